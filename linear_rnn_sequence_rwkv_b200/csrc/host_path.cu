// wkv7_forward on host buffers: the end-to-end path of a caller whose tokens and results live in
// host memory. The batch is cut into slices of whole sequences; each slice's host-to-device
// copies (one copy stream), its forward (the caller's stream) and its device-to-host copies (a
// second copy stream) overlap with those of the other slices, so both copy directions and the
// kernels run at the same time. The device copies live in the caller's workspace: nothing is
// allocated. The two copy streams and the events that order them are made once per device.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace {

using wkv7::set_error;
#define host_fail set_error

constexpr int kMaxSlices = 8;
constexpr size_t kMinSliceBytes = size_t(24) << 20;   // input bytes per slice: copies stay efficient
constexpr size_t kAlign = 256;

size_t up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Per-device copy streams and events (host-side objects; no device memory of the caller's).
struct Lane {
    bool ready = false;
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, done = nullptr, copied[kMaxSlices] = {}, computed[kMaxSlices] = {};
    std::mutex mu;   // one call at a time enqueues on a device (the events are reused)
};

cudaError_t lane_for(int dev, Lane *&out) {
    static std::mutex mu;
    static Lane lanes[64];
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    Lane &l = lanes[dev];
    if (!l.ready) {
        const unsigned fl = cudaEventDisableTiming;
        cudaError_t e = cudaStreamCreateWithFlags(&l.in, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&l.out, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&l.start, fl);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&l.done, fl);
        for (int i = 0; i < kMaxSlices && e == cudaSuccess; ++i) {
            e = cudaEventCreateWithFlags(&l.copied[i], fl);
            if (e == cudaSuccess) e = cudaEventCreateWithFlags(&l.computed[i], fl);
        }
        if (e != cudaSuccess) return e;   // partly made objects are kept and remade on the next call
        l.ready = true;
    }
    out = &l;
    return cudaSuccess;
}

// Whether p is host memory (pinned, registered or pageable), not device or managed memory.
bool is_host(const void *p) {
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return true;   // unknown to CUDA: pageable host memory on older drivers
    }
    return at.type == cudaMemoryTypeHost || at.type == cudaMemoryTypeUnregistered;
}

struct Layout {
    size_t in, s0, y, st, snap, par, total;
};

Layout layout(int B, int T, int H, int N, wkv7_dtype dt, int n_snap, bool s0, bool st, bool epi) {
    Layout L{};
    const size_t tok = size_t(B) * T * H * N, state = size_t(B) * H * N * N;
    L.in = up(tok * (dt == WKV7_BF16 ? 2 : 4));
    L.s0 = s0 ? up(state * 4) : 0;
    L.y = up(tok * 4);
    L.st = st ? up(state * 4) : 0;
    L.snap = up(state * 4 * size_t(n_snap));
    L.par = epi ? 3 * up(size_t(H) * N * 4) : 0;
    L.total = 6 * L.in + L.s0 + L.y + L.st + L.snap + L.par;
    return L;
}

}  // namespace

extern "C" {

size_t wkv7_forward_host_workspace_bytes(int B, int T, int H, int N, wkv7_dtype dt, const wkv7_opts *opts) {
    if (B <= 0 || T < 0 || H <= 0 || N <= 0 || (long long)B * T * H * N > (1ll << 40)) return 0;
    wkv7_opts o;
    wkv7_opts_default(&o);
    if (opts) o = *opts;
    const int n_snap = o.snap_every > 0 ? T / o.snap_every : 0;
    const bool epi = o.ln_w && o.ln_b && o.r_k;
    // S0 and S_T are counted whether or not the call passes them (the size does not depend on it)
    return layout(B, T, H, N, dt, n_snap, true, true, epi).total +
           wkv7_workspace_bytes(B, T, H, N, dt, opts);
}

wkv7_status wkv7_forward_host(int B, int T, int H, int N, wkv7_dtype dt, const void *r, const void *w,
                              const void *k, const void *v, const void *kk, const void *a, const float *S0,
                              float *y, float *S_T, const wkv7_opts *opts_in, void *workspace,
                              size_t workspace_bytes, void *stream) {
    wkv7_opts opts;
    wkv7_opts_default(&opts);
    if (opts_in) opts = *opts_in;
    if (B <= 0 || T < 0 || H <= 0 || N <= 0) return host_fail(WKV7_ERR_ARG, "B, H, N >= 1 and T >= 0 required");
    if (dt != WKV7_BF16 && dt != WKV7_F32) return host_fail(WKV7_ERR_ARG, "unknown dtype %d", int(dt));
    if ((long long)B * T * H * N > (1ll << 40)) return host_fail(WKV7_ERR_ARG, "sizes overflow");
    const int n_snap = opts.snap_every > 0 ? T / opts.snap_every : 0;
    const int n_epi = (opts.ln_w != nullptr) + (opts.ln_b != nullptr) + (opts.r_k != nullptr);
    if (n_epi != 0 && n_epi != 3) return host_fail(WKV7_ERR_ARG, "ln_w, ln_b, r_k: all three or none");
    if (T > 0) {
        const void *req[] = {r, w, k, v, kk, a, y};
        const char *names[] = {"r", "w", "k", "v", "kk", "a", "y"};
        for (int i = 0; i < 7; ++i)
            if (!req[i]) return host_fail(WKV7_ERR_ARG, "%s is NULL", names[i]);
    }
    if (n_snap > 0 && !opts.snapshots) return host_fail(WKV7_ERR_ARG, "snap_every=%d but snapshots is NULL", opts.snap_every);
    const void *hosts[] = {r, w, k, v, kk, a, S0, y, S_T, n_snap ? opts.snapshots : nullptr, opts.ln_w, opts.ln_b,
                           opts.r_k};
    const char *hn[] = {"r", "w", "k", "v", "kk", "a", "S0", "y", "S_T", "snapshots", "ln_w", "ln_b", "r_k"};
    for (int i = 0; i < 13; ++i)
        if (hosts[i] && !is_host(hosts[i]))
            return host_fail(WKV7_ERR_ARG, "%s: the host path takes host memory (use wkv7_forward for device buffers)",
                             hn[i]);
    const size_t need = wkv7_forward_host_workspace_bytes(B, T, H, N, dt, &opts);
    if (!workspace || workspace_bytes < need)
        return host_fail(WKV7_ERR_WORKSPACE, "workspace of %zu bytes required, %zu given", need,
                         workspace ? workspace_bytes : 0);
    if ((reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) != 0)
        return host_fail(WKV7_ERR_ALIGN, "workspace is not %zu-byte aligned", kAlign);

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    Lane *lane = nullptr;
    if (e == cudaSuccess) e = lane_for(dev, lane);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return host_fail(WKV7_ERR_CUDA, "copy streams: %s", cudaGetErrorName(e));
    }
    std::lock_guard<std::mutex> lk(lane->mu);
    const cudaStream_t main = static_cast<cudaStream_t>(stream);

    // device copies in the workspace
    const Layout L = layout(B, T, H, N, dt, n_snap, true, true, n_epi == 3);
    uint8_t *base = static_cast<uint8_t *>(workspace);
    uint8_t *d_in[6];
    for (int i = 0; i < 6; ++i) d_in[i] = base + i * L.in;
    float *d_s0 = reinterpret_cast<float *>(base + 6 * L.in);
    float *d_y = reinterpret_cast<float *>(base + 6 * L.in + L.s0);
    float *d_st = reinterpret_cast<float *>(base + 6 * L.in + L.s0 + L.y);
    float *d_snap = reinterpret_cast<float *>(base + 6 * L.in + L.s0 + L.y + L.st);
    float *d_par = reinterpret_cast<float *>(base + 6 * L.in + L.s0 + L.y + L.st + L.snap);
    uint8_t *d_ws = base + L.total;
    const size_t ws_bytes = workspace_bytes - L.total;
    const size_t par_stride = up(size_t(H) * N * 4) / 4;

    const size_t es = dt == WKV7_BF16 ? 2 : 4;
    const size_t tok_b = size_t(T) * H * N;          // elements per batch row
    const size_t st_b = size_t(H) * N * N;
    const size_t in_bytes = size_t(B) * tok_b * es * 6;
    const int pieces = T > 0 ? int(std::max<size_t>(1, std::min<size_t>({size_t(B), size_t(kMaxSlices),
                                                                         in_bytes / kMinSliceBytes}))) : 1;
    const void *src[6] = {r, w, k, v, kk, a};

    // the copy streams start after everything already on the caller's stream (which includes the
    // previous call's last copies: the workspace is free again)
#define WKV7_TRY(x)                                                                             \
    do {                                                                                        \
        const cudaError_t e_ = (x);                                                             \
        if (e_ != cudaSuccess) return host_fail(WKV7_ERR_CUDA, "%s: %s", #x, cudaGetErrorName(e_)); \
    } while (0)
    WKV7_TRY(cudaEventRecord(lane->start, main));
    WKV7_TRY(cudaStreamWaitEvent(lane->in, lane->start, 0));
    WKV7_TRY(cudaStreamWaitEvent(lane->out, lane->start, 0));
    wkv7_opts sl = opts;
    if (n_epi == 3) {
        const float *pars[3] = {opts.ln_w, opts.ln_b, opts.r_k};
        for (int i = 0; i < 3; ++i)
            WKV7_TRY(cudaMemcpyAsync(d_par + i * par_stride, pars[i], size_t(H) * N * 4, cudaMemcpyHostToDevice,
                                     lane->in));
        sl.ln_w = d_par;
        sl.ln_b = d_par + par_stride;
        sl.r_k = d_par + 2 * par_stride;
    }
    for (int p = 0; p < pieces; ++p) {
        const int b0 = int(size_t(B) * p / pieces), b1 = int(size_t(B) * (p + 1) / pieces), nb = b1 - b0;
        if (nb == 0) continue;
        for (int i = 0; i < 6 && T > 0; ++i)
            WKV7_TRY(cudaMemcpyAsync(d_in[i] + b0 * tok_b * es, static_cast<const uint8_t *>(src[i]) + b0 * tok_b * es,
                                     nb * tok_b * es, cudaMemcpyHostToDevice, lane->in));
        if (S0)
            WKV7_TRY(cudaMemcpyAsync(d_s0 + b0 * st_b, S0 + b0 * st_b, nb * st_b * 4, cudaMemcpyHostToDevice, lane->in));
        WKV7_TRY(cudaEventRecord(lane->copied[p], lane->in));
        WKV7_TRY(cudaStreamWaitEvent(main, lane->copied[p], 0));
        sl.snapshots = n_snap ? d_snap + size_t(b0) * n_snap * st_b : nullptr;
        const wkv7_status s = wkv7_forward(nb, T, H, N, dt, d_in[0] + b0 * tok_b * es, d_in[1] + b0 * tok_b * es,
                                           d_in[2] + b0 * tok_b * es, d_in[3] + b0 * tok_b * es,
                                           d_in[4] + b0 * tok_b * es, d_in[5] + b0 * tok_b * es,
                                           S0 ? d_s0 + b0 * st_b : nullptr, d_y + b0 * tok_b,
                                           S_T ? d_st + b0 * st_b : nullptr, &sl, ws_bytes ? d_ws : nullptr,
                                           ws_bytes, main);
        if (s != WKV7_OK) {
            char detail[400];
            snprintf(detail, sizeof(detail), "%s", wkv7_last_error());
            return host_fail(s, "slice %d: %s", p, detail);
        }
        WKV7_TRY(cudaEventRecord(lane->computed[p], main));
        WKV7_TRY(cudaStreamWaitEvent(lane->out, lane->computed[p], 0));
        if (T > 0)
            WKV7_TRY(cudaMemcpyAsync(y + b0 * tok_b, d_y + b0 * tok_b, nb * tok_b * 4, cudaMemcpyDeviceToHost,
                                     lane->out));
        if (S_T)
            WKV7_TRY(cudaMemcpyAsync(S_T + b0 * st_b, d_st + b0 * st_b, nb * st_b * 4, cudaMemcpyDeviceToHost,
                                     lane->out));
        if (n_snap)
            WKV7_TRY(cudaMemcpyAsync(opts.snapshots + size_t(b0) * n_snap * st_b, d_snap + size_t(b0) * n_snap * st_b,
                                     size_t(nb) * n_snap * st_b * 4, cudaMemcpyDeviceToHost, lane->out));
    }
    // the caller's stream completes once the last result is in host memory
    WKV7_TRY(cudaEventRecord(lane->done, lane->out));
    WKV7_TRY(cudaStreamWaitEvent(main, lane->done, 0));
#undef WKV7_TRY
    return WKV7_OK;
}

}  // extern "C"
