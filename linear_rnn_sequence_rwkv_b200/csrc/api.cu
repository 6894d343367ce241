// C ABI of the WKV-7 library: argument validation, workspace sizing, dispatch.
//
// Every check that can fail runs on the host before anything is enqueued, so a bad
// argument never reaches a kernel. Launches go to the caller's stream; nothing here
// allocates device memory or synchronises.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <set>
#include <utility>

#include "common.cuh"
#include "backward.cuh"
#include "decode.cuh"
#include "epilogue.cuh"

namespace wkv7 {

cudaError_t allow_dynamic_smem(const void *kernel, int bytes) {
    static std::mutex mu;
    static std::set<std::pair<int, const void *>> done;   // (device, kernel) pairs already raised
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lk(mu);
    if (done.count({dev, kernel})) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done.insert({dev, kernel});
    return e;
}

wkv7_status set_error(wkv7_status s, const char *fmt, ...);

}  // namespace wkv7

namespace {

thread_local char g_err[512] = "";

wkv7_status fail(wkv7_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

}  // namespace

wkv7_status wkv7::set_error(wkv7_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

namespace {

wkv7_status cuda_fail(cudaError_t e, const char *what) {
    return fail(WKV7_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// cuMemGetAddressRange through the runtime's driver entry point (no -lcuda needed).
typedef CUresult (*AddrRangeFn)(CUdeviceptr *, size_t *, CUdeviceptr);
AddrRangeFn addr_range_fn() {
    static std::once_flag once;
    static AddrRangeFn fn = nullptr;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<AddrRangeFn>(p);
    });
    return fn;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Buf {
    const char *name;
    const void *ptr;
    size_t bytes;
};

// Device-side checks of one buffer: device memory of the current device, large enough.
wkv7_status check_device_buffer(const Buf &b, int device) {
    if (!b.ptr || b.bytes == 0) return WKV7_OK;
    cudaPointerAttributes at;
    cudaError_t e = cudaPointerGetAttributes(&at, b.ptr);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(WKV7_ERR_ARG, "%s: cannot query pointer attributes (%s)", b.name, cudaGetErrorName(e));
    }
    if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged)
        return fail(WKV7_ERR_ARG, "%s: not device memory (memory type %d)", b.name, (int)at.type);
    if (at.type == cudaMemoryTypeDevice && at.device != device)
        return fail(WKV7_ERR_ARG, "%s: allocated on device %d, current device is %d", b.name, at.device, device);
    if (AddrRangeFn fn = addr_range_fn()) {
        CUdeviceptr base = 0;
        size_t size = 0;
        if (fn(&base, &size, reinterpret_cast<CUdeviceptr>(b.ptr)) == CUDA_SUCCESS) {
            const uintptr_t end = reinterpret_cast<uintptr_t>(b.ptr) + b.bytes;
            if (end > static_cast<uintptr_t>(base) + size)
                return fail(WKV7_ERR_ARG, "%s: needs %zu bytes but its allocation ends %zu bytes after it",
                            b.name, b.bytes, static_cast<size_t>(base + size - reinterpret_cast<uintptr_t>(b.ptr)));
        }
    }
    return WKV7_OK;
}

bool overlaps(const Buf &x, const Buf &y) {
    if (!x.ptr || !y.ptr || !x.bytes || !y.bytes) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(x.ptr), a1 = a0 + x.bytes;
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(y.ptr), b1 = b0 + y.bytes;
    return a0 < b1 && b0 < a1;
}

size_t elem_bytes(wkv7_dtype dt) { return dt == WKV7_BF16 ? 2 : 4; }

// Product of non-negative sizes with overflow detection (returns false on overflow).
bool mul_ok(size_t &acc, long long f) {
    if (f < 0) return false;
    if (f != 0 && acc > SIZE_MAX / static_cast<size_t>(f)) return false;
    acc *= static_cast<size_t>(f);
    return true;
}

}  // namespace

// Sizes and options, shared by wkv7_forward and wkv7_plan; fills `opts` (defaults if NULL).
wkv7_status check_args(int B, int T, int H, int N, wkv7_dtype dt, const wkv7_opts *opts_in, wkv7_opts &opts,
                       bool need_buffers = true) {
    if (N <= 0 || B <= 0 || H <= 0 || T < 0)
        return fail(WKV7_ERR_ARG, "bad sizes B=%d T=%d H=%d N=%d (need B,H,N >= 1, T >= 0)", B, T, H, N);
    if (static_cast<long long>(B) * H > INT_MAX) return fail(WKV7_ERR_ARG, "B*H=%lld heads: at most %d", static_cast<long long>(B) * H, INT_MAX);
    if (N != wkv7::kN && N != 128)
        return fail(WKV7_ERR_UNSUPPORTED, "head size N=%d: N=64 and N=128 (scan path) are implemented", N);
    if (dt != WKV7_F32 && dt != WKV7_BF16) return fail(WKV7_ERR_ARG, "unknown dtype %d", (int)dt);
    wkv7_opts_default(&opts);
    if (opts_in) opts = *opts_in;
    if (opts.algo < WKV7_ALGO_AUTO || opts.algo > WKV7_ALGO_SPLIT)
        return fail(WKV7_ERR_ARG, "unknown algo %d", opts.algo);
    if (!(opts.chunk == 0 || opts.chunk == 16 || opts.chunk == 32 || opts.chunk == 64))
        return fail(WKV7_ERR_ARG, "chunk=%d: must be 0 (default), 16, 32 or 64", opts.chunk);
    if (opts.snap_every < 0) return fail(WKV7_ERR_ARG, "snap_every=%d < 0", opts.snap_every);
    if (need_buffers && opts.snap_every > 0 && !opts.snapshots && T >= opts.snap_every)
        return fail(WKV7_ERR_ARG, "snap_every=%d but snapshots is NULL", opts.snap_every);
    const int n_epi = (opts.ln_w != nullptr) + (opts.ln_b != nullptr) + (opts.r_k != nullptr);
    if (n_epi != 0 && n_epi != 3) return fail(WKV7_ERR_ARG, "epilogue needs all of ln_w, ln_b, r_k (or none)");
    if (n_epi == 3 && !(std::isfinite(opts.gn_eps) && opts.gn_eps >= 0.f))
        return fail(WKV7_ERR_ARG, "gn_eps must be finite and >= 0");
    if (opts.segments < 0 || opts.segments > WKV7_MAX_SEGMENTS)
        return fail(WKV7_ERR_ARG, "segments=%d outside 0..%d", opts.segments, WKV7_MAX_SEGMENTS);
    if (opts.withhold_handoff != 0 &&
        (opts.withhold_handoff != 1 || opts.algo != WKV7_ALGO_SPLIT || opts.segments < 2))
        return fail(WKV7_ERR_ARG, "withhold_handoff=%d: only 1, with WKV7_ALGO_SPLIT and segments >= 2",
                    opts.withhold_handoff);
    return WKV7_OK;
}

// Whether the chunked kernel runs: forced by CHUNK / SPLIT (UNSUPPORTED if it cannot), chosen
// by AUTO for bf16 inputs of at least 16 tokens.
wkv7_status pick_chunk(const wkv7_opts &opts, const wkv7::FwdArgs &p, bool &use_chunk) {
    const bool chunk_ok = wkv7::chunk_supported(p) && (opts.chunk == 0 || opts.chunk == 64);
    use_chunk = false;
    if (opts.algo == WKV7_ALGO_CHUNK || opts.algo == WKV7_ALGO_SPLIT) {
        if (!chunk_ok)
            return fail(WKV7_ERR_UNSUPPORTED,
                        "chunked algorithm needs bf16 inputs, chunk 0 or 64 and snap_every a multiple of 64");
        use_chunk = true;
    } else if (opts.algo == WKV7_ALGO_AUTO) {
        use_chunk = chunk_ok && p.T >= 16;
    }
    return WKV7_OK;
}

// CTAs per (b, h) requested of the chunked path: CHUNK one, SPLIT the caller's count (0 = choose).
int requested_segments(const wkv7_opts &opts) {
    return opts.algo == WKV7_ALGO_CHUNK ? 1 : (opts.algo == WKV7_ALGO_SPLIT ? opts.segments : 0);
}

extern "C" {

void wkv7_opts_default(wkv7_opts *o) {
    if (!o) return;
    std::memset(o, 0, sizeof(*o));
    o->algo = WKV7_ALGO_AUTO;
    o->gn_eps = 64e-5f;
}

const char *wkv7_status_string(wkv7_status s) {
    switch (s) {
        case WKV7_OK: return "WKV7_OK";
        case WKV7_ERR_ARG: return "WKV7_ERR_ARG";
        case WKV7_ERR_UNSUPPORTED: return "WKV7_ERR_UNSUPPORTED";
        case WKV7_ERR_ALIGN: return "WKV7_ERR_ALIGN";
        case WKV7_ERR_CUDA: return "WKV7_ERR_CUDA";
        case WKV7_ERR_TIMEOUT: return "WKV7_ERR_TIMEOUT";
        case WKV7_ERR_WORKSPACE: return "WKV7_ERR_WORKSPACE";
    }
    return "WKV7_ERR_UNKNOWN";
}

const char *wkv7_last_error(void) { return g_err; }

int wkv7_abi_version(void) { return WKV7_ABI_VERSION; }

wkv7_status wkv7_probe_fp32_fma(int blocks, int iters, void *stream, double *flops) {
    if (blocks < 1 || iters < 1 || !flops) return fail(WKV7_ERR_ARG, "blocks and iters must be >= 1, flops non-NULL");
    const cudaError_t e = wkv7::launch_fma_peak(blocks, iters, static_cast<cudaStream_t>(stream), flops);
    return e == cudaSuccess ? WKV7_OK : cuda_fail(e, "FMA peak probe");
}

wkv7_status wkv7_probe_tf32_mma(int n, int iters, void *stream, double *flops) {
    if (!(n == 64 || n == 128 || n == 256) || iters < 1 || !flops)
        return fail(WKV7_ERR_ARG, "n must be 64, 128 or 256, iters >= 1, flops non-NULL");
    const cudaError_t e = wkv7::launch_tf32_mma_peak(n, iters, static_cast<cudaStream_t>(stream), flops);
    return e == cudaSuccess ? WKV7_OK : cuda_fail(e, "tf32 MMA peak probe");
}

size_t wkv7_workspace_bytes(int B, int T, int H, int N, wkv7_dtype dt, const wkv7_opts *opts) {
    (void)B; (void)T; (void)H; (void)N; (void)dt; (void)opts;
    return 0;
}

}  // extern "C"

namespace {

// wkv7_forward and wkv7_forward_raw. raw: w and a are the decay and rate logits, k the key
// before its update, kk is unused, k_k (required) and k_a (nullable) are the [H][N] parameters.
wkv7_status forward_impl(bool raw, int B, int T, int H, int N, wkv7_dtype dt, const void *r, const void *w,
                         const void *k, const void *v, const void *kk, const void *a, const float *k_k,
                         const float *k_a, const float *S0, float *y, float *S_T, const wkv7_opts *opts_in,
                         void *workspace, size_t workspace_bytes, void *stream) {
    g_err[0] = '\0';
    wkv7_opts opts;
    const wkv7_status vs = check_args(B, T, H, N, dt, opts_in, opts);
    if (vs != WKV7_OK) return vs;
    const int n_epi = (opts.ln_w != nullptr) + (opts.ln_b != nullptr) + (opts.r_k != nullptr);

    size_t tok = 1, st = 1;
    if (!mul_ok(tok, B) || !mul_ok(tok, T) || !mul_ok(tok, H) || !mul_ok(tok, N) || !mul_ok(st, B) ||
        !mul_ok(st, H) || !mul_ok(st, N) || !mul_ok(st, N) || tok > (size_t(1) << 40))
        return fail(WKV7_ERR_ARG, "sizes overflow");
    const size_t in_bytes = tok * elem_bytes(dt), y_bytes = tok * 4, st_bytes = st * 4;
    const int n_snap = opts.snap_every > 0 ? T / opts.snap_every : 0;
    const size_t snap_bytes = st_bytes * static_cast<size_t>(n_snap);
    const size_t par_bytes = size_t(H) * N * 4;
    const char *wn = raw ? "w_logit" : "w", *an = raw ? "a_logit" : "a";

    if (T > 0) {
        const void *req[] = {r, w, k, v, raw ? k_k : kk, a, y};
        const char *names[] = {"r", wn, "k", "v", raw ? "k_k" : "kk", an, "y"};
        for (int i = 0; i < 7; ++i)
            if (!req[i]) return fail(WKV7_ERR_ARG, "%s is NULL", names[i]);
    }
    const Buf bufs[] = {{"r", r, T ? in_bytes : 0},      {wn, w, T ? in_bytes : 0},
                        {"k", k, T ? in_bytes : 0},      {"v", v, T ? in_bytes : 0},
                        {"kk", raw ? nullptr : kk, T ? in_bytes : 0}, {an, a, T ? in_bytes : 0},
                        {"S0", S0, st_bytes},            {"y", y, T ? y_bytes : 0},
                        {"S_T", S_T, st_bytes},          {"snapshots", n_snap ? opts.snapshots : nullptr, snap_bytes},
                        {"ln_w", opts.ln_w, par_bytes},  {"ln_b", opts.ln_b, par_bytes},
                        {"r_k", opts.r_k, par_bytes},    {"workspace", workspace, workspace_bytes},
                        {"k_k", raw ? k_k : nullptr, par_bytes}, {"k_a", raw ? k_a : nullptr, par_bytes}};
    constexpr int nb = sizeof(bufs) / sizeof(bufs[0]);
    for (int i = 0; i < nb; ++i)
        if (bufs[i].ptr && !aligned16(bufs[i].ptr))
            return fail(WKV7_ERR_ALIGN, "%s is not 16-byte aligned", bufs[i].name);
    const size_t need_ws = wkv7_workspace_bytes(B, T, H, N, dt, &opts);
    if (need_ws > 0 && (!workspace || workspace_bytes < need_ws))
        return fail(WKV7_ERR_WORKSPACE, "workspace of %zu bytes required, %zu given", need_ws,
                    workspace ? workspace_bytes : 0);
    // Outputs must not overlap inputs (S_T == S0 exactly is the allowed in-place hand-off).
    const Buf &yb = bufs[7], &sb = bufs[8], &snb = bufs[9];
    for (int i = 0; i < 7; ++i) {
        if (i < 6 && overlaps(yb, bufs[i])) return fail(WKV7_ERR_ARG, "y overlaps %s", bufs[i].name);
        if (i < 6 && overlaps(sb, bufs[i])) return fail(WKV7_ERR_ARG, "S_T overlaps %s", bufs[i].name);
        if (overlaps(snb, bufs[i])) return fail(WKV7_ERR_ARG, "snapshots overlap %s", bufs[i].name);
    }
    if (overlaps(yb, sb)) return fail(WKV7_ERR_ARG, "y overlaps S_T");
    if (overlaps(sb, bufs[6]) && S_T != S0) return fail(WKV7_ERR_ARG, "S_T partially overlaps S0");
    if (overlaps(snb, sb) || overlaps(snb, bufs[6])) return fail(WKV7_ERR_ARG, "snapshots overlap a state");

    int device = 0;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e, "cudaGetDevice");
    }
    for (int i = 0; i < nb; ++i) {
        const wkv7_status s = check_device_buffer(bufs[i], device);
        if (s != WKV7_OK) return s;
    }

    wkv7::FwdArgs p{};
    p.B = B; p.T = T; p.H = H; p.N = N; p.dt = dt;
    p.r = r; p.w = w; p.k = k; p.v = v; p.kk = raw ? nullptr : kk; p.a = a;
    p.S0 = S0; p.y = y; p.S_T = S_T;
    p.snap_every = n_snap ? opts.snap_every : 0;
    p.snaps = n_snap ? opts.snapshots : nullptr;
    p.ln_w = opts.ln_w; p.ln_b = opts.ln_b; p.r_k = opts.r_k; p.gn_eps = opts.gn_eps;
    p.raw = raw; p.k_k = raw ? k_k : nullptr; p.k_a = raw ? k_a : nullptr;
    p.chunk = opts.chunk;
    p.segments = requested_segments(opts);
    p.handoff_wait_us = opts.handoff_wait_us;
    p.withhold_handoff = opts.withhold_handoff;
    p.ws = workspace; p.ws_bytes = workspace_bytes;
    p.stream = static_cast<cudaStream_t>(stream);

    if (T == 0) {
        if (!S_T || S_T == S0) return WKV7_OK;
        e = wkv7::launch_copy_state(p);
        return e == cudaSuccess ? WKV7_OK : cuda_fail(e, "state copy launch");
    }
    bool use_chunk = false;
    const wkv7_status ps = pick_chunk(opts, p, use_chunk);
    if (ps != WKV7_OK) return ps;
    if (use_chunk) {   // raw inputs are prepared in each kernel's load stage
        e = wkv7::launch_chunk(p);
        if (e != cudaSuccess) return cuda_fail(e, "chunked-prefill launch");
        return WKV7_OK;
    }
    e = wkv7::launch_seq(p);
    if (e != cudaSuccess) return cuda_fail(e, "sequential-scan launch");
    if (n_epi == 3) {
        e = wkv7::launch_epilogue(p);
        if (e != cudaSuccess) return cuda_fail(e, "epilogue launch");
    }
    return WKV7_OK;
}

// Defined with the other shared checks below.
wkv7_status decode_impl(int B, int H, int N, wkv7_dtype dt, const void *r, const void *w, const void *k,
                        const void *v, const void *kk, const void *a, float *S, float *y, bool raw,
                        const float *k_k, const float *k_a, const float *ln_w, const float *ln_b,
                        const float *r_k, float gn_eps, void *stream);

}  // namespace

extern "C" {

wkv7_status wkv7_forward(int B, int T, int H, int N, wkv7_dtype dt, const void *r, const void *w,
                         const void *k, const void *v, const void *kk, const void *a, const float *S0,
                         float *y, float *S_T, const wkv7_opts *opts_in, void *workspace,
                         size_t workspace_bytes, void *stream) {
    return forward_impl(false, B, T, H, N, dt, r, w, k, v, kk, a, nullptr, nullptr, S0, y, S_T, opts_in,
                        workspace, workspace_bytes, stream);
}

wkv7_status wkv7_forward_raw(int B, int T, int H, int N, wkv7_dtype dt, const void *r, const void *w_logit,
                             const void *k, const void *v, const void *a_logit, const float *k_k,
                             const float *k_a, const float *S0, float *y, float *S_T, const wkv7_opts *opts_in,
                             void *workspace, size_t workspace_bytes, void *stream) {
    return forward_impl(true, B, T, H, N, dt, r, w_logit, k, v, nullptr, a_logit, k_k, k_a, S0, y, S_T, opts_in,
                        workspace, workspace_bytes, stream);
}

wkv7_status wkv7_plan(int B, int T, int H, int N, wkv7_dtype dt, const wkv7_opts *opts_in, int *algo,
                      int *segments, int *launches) {
    g_err[0] = '\0';
    if (!algo || !segments || !launches) return fail(WKV7_ERR_ARG, "algo, segments and launches must not be NULL");
    wkv7_opts opts;
    const wkv7_status vs = check_args(B, T, H, N, dt, opts_in, opts, false);   // no buffers needed
    if (vs != WKV7_OK) return vs;
    wkv7::FwdArgs p{};
    p.B = B; p.T = T; p.H = H; p.N = N; p.dt = dt;
    p.snap_every = (opts.snap_every > 0 && T >= opts.snap_every) ? opts.snap_every : 0;
    p.chunk = opts.chunk;
    p.segments = requested_segments(opts);
    bool use_chunk = false;
    const wkv7_status ps = pick_chunk(opts, p, use_chunk);
    if (ps != WKV7_OK) return ps;
    *algo = WKV7_ALGO_SEQ;
    *segments = 0;
    if (T == 0) {   // the state copy (one launch) unless S_T is not requested; counted as one here
        *launches = 1;
        return WKV7_OK;
    }
    if (!use_chunk) {   // the scan, plus the stand-alone epilogue when it is on
        const int n_epi = (opts.ln_w != nullptr) + (opts.ln_b != nullptr) + (opts.r_k != nullptr);
        *launches = n_epi == 3 ? 2 : 1;
        return WKV7_OK;
    }
    int cs = 0, n = 0;
    const cudaError_t e = wkv7::chunk_segments(p, &cs, &n);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e, "querying the device for the chunked path");
    }
    *algo = WKV7_ALGO_CHUNK;
    *segments = cs;
    *launches = n;
    return WKV7_OK;
}

wkv7_status wkv7_poll_device_error(void *stream) {
    g_err[0] = '\0';
    unsigned int v = 0;
    const cudaError_t e = wkv7::read_device_error(static_cast<cudaStream_t>(stream), &v, true);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (v) return fail(WKV7_ERR_TIMEOUT, "a bounded device-side wait gave up (code %u)", v);
    return WKV7_OK;
}

wkv7_status wkv7_decode_step(int B, int H, int N, wkv7_dtype dt, const void *r, const void *w, const void *k,
                             const void *v, const void *kk, const void *a, float *S, float *y, void *stream) {
    g_err[0] = '\0';
    return decode_impl(B, H, N, dt, r, w, k, v, kk, a, S, y, false, nullptr, nullptr, nullptr, nullptr, nullptr,
                       64e-5f, stream);
}

wkv7_status wkv7_decode_step_ex(int B, int H, int N, wkv7_dtype dt, const void *r, const void *w, const void *k,
                                const void *v, const void *kk, const void *a, float *S, float *y,
                                const float *ln_w, const float *ln_b, const float *r_k, float gn_eps,
                                void *stream) {
    g_err[0] = '\0';
    return decode_impl(B, H, N, dt, r, w, k, v, kk, a, S, y, false, nullptr, nullptr, ln_w, ln_b, r_k, gn_eps,
                       stream);
}

wkv7_status wkv7_decode_step_raw(int B, int H, int N, wkv7_dtype dt, const void *r, const void *w_logit,
                                 const void *k, const void *v, const void *a_logit, const float *k_k,
                                 const float *k_a, float *S, float *y, const float *ln_w, const float *ln_b,
                                 const float *r_k, float gn_eps, void *stream) {
    g_err[0] = '\0';
    return decode_impl(B, H, N, dt, r, w_logit, k, v, nullptr, a_logit, S, y, true, k_k, k_a, ln_w, ln_b, r_k,
                       gn_eps, stream);
}

wkv7_status wkv7_backward_static(int B, int T, int H, int N, wkv7_dtype dt, const void *r, const void *w,
                                 const void *k, const void *v, const void *kk, const void *a, const float *S0,
                                 const float *snapshots, int snap_every, const float *dy, const float *dS_T,
                                 float *dr, float *dw, float *dk, float *dv, float *dkk, float *da, float *dS0,
                                 void *stream) {
    g_err[0] = '\0';
    const size_t need = wkv7_backward_workspace_bytes(B, T, H, N, snap_every);
    const size_t cap = wkv7::backward_static_scratch_bytes();
    if (need > cap)
        return fail(WKV7_ERR_WORKSPACE, "needs %zu bytes of scratch; the static scratch holds %zu (use wkv7_backward)",
                    need, cap);
    void *scratch = nullptr;
    if (need > 0) {
        const cudaError_t e = wkv7::backward_static_scratch(&scratch);
        if (e != cudaSuccess) {
            cudaGetLastError();
            return cuda_fail(e, "static scratch address");
        }
    }
    return wkv7_backward(B, T, H, N, dt, r, w, k, v, kk, a, S0, snapshots, snap_every, dy, dS_T, dr, dw, dk, dv,
                         dkk, da, dS0, scratch, need ? cap : 0, stream);
}

static bool layer_dims_ok(const wkv7_layer_dims *d) {
    return d && d->H > 0 && (d->N == wkv7::kN || d->N == 128) && d->d_w > 0 && d->d_a > 0 && d->d_v > 0 &&
           d->d_g > 0 && size_t(d->H) * d->N <= (size_t(1) << 20);
}

size_t wkv7_layer_workspace_bytes(int B, int T, wkv7_dtype dt, const wkv7_layer_dims *dims) {
    if (B <= 0 || T <= 0 || !layer_dims_ok(dims) || (dt != WKV7_F32 && dt != WKV7_BF16)) return 0;
    size_t m = 1;
    if (!mul_ok(m, B) || !mul_ok(m, T) || !mul_ok(m, dims->H) || !mul_ok(m, dims->N) || m > (size_t(1) << 36)) return 0;
    return wkv7::layer_workspace(B, T, dt, *dims);
}

wkv7_status wkv7_layer_forward(int B, int T, wkv7_dtype dt, const wkv7_layer_dims *dims,
                               const wkv7_layer_params *params, const void *x, const void *last_x, const void *v0,
                               float *S, float *out, void *v0_out, void *last_x_out, const wkv7_opts *opts_in,
                               void *workspace, size_t workspace_bytes, void *stream) {
    g_err[0] = '\0';
    if (B <= 0 || T < 0) return fail(WKV7_ERR_ARG, "bad sizes B=%d T=%d", B, T);
    if (dt != WKV7_F32 && dt != WKV7_BF16) return fail(WKV7_ERR_ARG, "unknown dtype %d", (int)dt);
    if (!dims || !params) return fail(WKV7_ERR_ARG, "dims and params are required");
    if (dims->N != wkv7::kN && dims->N != 128)
        return fail(WKV7_ERR_UNSUPPORTED, "head size N=%d: N=64 and N=128 are implemented", dims->N);
    if (!layer_dims_ok(dims)) return fail(WKV7_ERR_ARG, "bad layer dims (H, low-rank widths >= 1)");
    const wkv7_layer_params &P = *params;
    const int C = dims->H * dims->N;
    const size_t e = elem_bytes(dt), bc = size_t(B) * C;
    size_t mc = bc;
    if (!mul_ok(mc, T) || mc > (size_t(1) << 36)) return fail(WKV7_ERR_ARG, "sizes overflow");
    wkv7_opts opts;
    wkv7_opts_default(&opts);
    if (opts_in) opts = *opts_in;
    // required pointers and their sizes (bytes); optional ones may be NULL
    const size_t pc = size_t(C) * 4, ph = size_t(dims->H) * dims->N * 4, sq = size_t(C) * C * e;
    const Buf bufs[] = {
        {"mr", P.mr, pc}, {"mw", P.mw, pc}, {"mk", P.mk, pc}, {"mv", P.mv, pc}, {"ma", P.ma, pc}, {"mg", P.mg, pc},
        {"w_bias", P.w_bias, pc}, {"a_bias", P.a_bias, pc}, {"r_k", P.r_k, ph}, {"k_k", P.k_k, ph},
        {"ln_w", P.ln_w, ph}, {"ln_b", P.ln_b, ph}, {"Wr", P.Wr, sq}, {"Wk", P.Wk, sq}, {"Wv", P.Wv, sq},
        {"Wo", P.Wo, sq}, {"Ww1", P.Ww1, size_t(C) * dims->d_w * e}, {"Ww2", P.Ww2, size_t(C) * dims->d_w * e},
        {"Wa1", P.Wa1, size_t(C) * dims->d_a * e}, {"Wa2", P.Wa2, size_t(C) * dims->d_a * e},
        {"Wg1", P.Wg1, size_t(C) * dims->d_g * e}, {"Wg2", P.Wg2, size_t(C) * dims->d_g * e},
        {"x", x, mc * e}, {"out", out, mc * 4}};
    const Buf opt[] = {{"k_a", P.k_a, ph}, {"v_bias", v0 ? P.v_bias : nullptr, pc},
                       {"Wv1", v0 ? P.Wv1 : nullptr, size_t(C) * dims->d_v * e},
                       {"Wv2", v0 ? P.Wv2 : nullptr, size_t(C) * dims->d_v * e},
                       {"last_x", last_x, bc * e}, {"v0", v0, mc * e}, {"S", S, size_t(B) * dims->H * dims->N * dims->N * 4},
                       {"v0_out", v0_out, mc * e}, {"last_x_out", last_x_out, bc * e},
                       {"workspace", workspace, workspace_bytes}};
    for (const Buf &b : bufs) {
        if (!b.ptr && T > 0) return fail(WKV7_ERR_ARG, "%s is NULL", b.name);
        if (b.ptr && !aligned16(b.ptr)) return fail(WKV7_ERR_ALIGN, "%s is not 16-byte aligned", b.name);
    }
    if (v0 && (!P.v_bias || !P.Wv1 || !P.Wv2)) return fail(WKV7_ERR_ARG, "v0 given but v_bias / Wv1 / Wv2 is NULL");
    for (const Buf &b : opt)
        if (b.ptr && !aligned16(b.ptr)) return fail(WKV7_ERR_ALIGN, "%s is not 16-byte aligned", b.name);
    const size_t need = wkv7_layer_workspace_bytes(B, T, dt, dims);
    if (need > 0 && (!workspace || workspace_bytes < need))
        return fail(WKV7_ERR_WORKSPACE, "workspace of %zu bytes required, %zu given", need, workspace ? workspace_bytes : 0);
    const Buf outs[] = {{"out", out, T ? mc * 4 : 0}, {"v0_out", v0_out, T ? mc * e : 0},
                        {"last_x_out", last_x_out, bc * e}, {"S", S, size_t(B) * dims->H * dims->N * dims->N * 4},
                        {"workspace", workspace, need}};
    const Buf ins[] = {{"x", x, mc * e}, {"last_x", last_x, bc * e}, {"v0", v0, mc * e}};
    for (const Buf &o : outs) {
        for (const Buf &i : ins) {
            // last_x_out == last_x in place is allowed: last_x is read by the first kernel,
            // x[:, T-1] is written by the last one
            if (o.ptr == last_x_out && i.ptr == last_x && last_x_out == last_x) continue;
            if (overlaps(o, i)) return fail(WKV7_ERR_ARG, "%s overlaps %s", o.name, i.name);
        }
        for (const Buf &o2 : outs)
            if (&o2 != &o && overlaps(o, o2)) return fail(WKV7_ERR_ARG, "%s overlaps %s", o.name, o2.name);
    }
    int device = 0;
    cudaError_t ce = cudaGetDevice(&device);
    if (ce != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(ce, "cudaGetDevice");
    }
    for (const Buf &b : bufs) {
        const wkv7_status s = check_device_buffer(b, device);
        if (s != WKV7_OK) return s;
    }
    for (const Buf &b : opt) {
        const wkv7_status s = check_device_buffer(b, device);
        if (s != WKV7_OK) return s;
    }
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (T == 0) {   // nothing to mix: the previous token passes through
        if (last_x_out) {
            ce = last_x ? cudaMemcpyAsync(last_x_out, last_x, bc * e, cudaMemcpyDeviceToDevice, cs)
                        : cudaMemsetAsync(last_x_out, 0, bc * e, cs);
            if (ce != cudaSuccess) return cuda_fail(ce, "last_x copy");
        }
        return WKV7_OK;
    }
    char err[400] = "";
    const wkv7_status s = wkv7::layer_dispatch(B, T, dt, *dims, P, x, last_x, v0, S, out, v0_out, last_x_out, opts,
                                               workspace, cs, err, sizeof(err));
    if (s != WKV7_OK) return fail(s, "%s", err);
    return WKV7_OK;
}

size_t wkv7_backward_workspace_bytes(int B, int T, int H, int N, int snap_every) {
    if (B <= 0 || T <= 0 || H <= 0 || (N != wkv7::kN && N != 128) || snap_every < 0) return 0;
    size_t n = 1;
    if (!mul_ok(n, B) || !mul_ok(n, H) || !mul_ok(n, T)) return 0;
    return wkv7::backward_checkpoint_bytes_n(B, T, H, N, snap_every);
}

wkv7_status wkv7_backward(int B, int T, int H, int N, wkv7_dtype dt, const void *r, const void *w,
                          const void *k, const void *v, const void *kk, const void *a, const float *S0,
                          const float *snapshots, int snap_every, const float *dy, const float *dS_T,
                          float *dr, float *dw, float *dk, float *dv, float *dkk, float *da, float *dS0,
                          void *workspace, size_t workspace_bytes, void *stream) {
    g_err[0] = '\0';
    if (N <= 0 || B <= 0 || H <= 0 || T < 0)
        return fail(WKV7_ERR_ARG, "bad sizes B=%d T=%d H=%d N=%d (need B,H,N >= 1, T >= 0)", B, T, H, N);
    if (static_cast<long long>(B) * H > INT_MAX) return fail(WKV7_ERR_ARG, "B*H=%lld heads: at most %d", static_cast<long long>(B) * H, INT_MAX);
    if (N != wkv7::kN && N != 128)
        return fail(WKV7_ERR_UNSUPPORTED, "head size N=%d: the backward pass is implemented for N=64 and N=128", N);
    if (dt != WKV7_F32 && dt != WKV7_BF16) return fail(WKV7_ERR_ARG, "unknown dtype %d", (int)dt);
    if (snap_every < 0) return fail(WKV7_ERR_ARG, "snap_every=%d < 0", snap_every);
    const int n_snap = snap_every > 0 ? T / snap_every : 0;
    if (n_snap > 0 && !snapshots) return fail(WKV7_ERR_ARG, "snap_every=%d but snapshots is NULL", snap_every);
    size_t tok = 1, st = 1;
    if (!mul_ok(tok, B) || !mul_ok(tok, T) || !mul_ok(tok, H) || !mul_ok(tok, N) || !mul_ok(st, B) ||
        !mul_ok(st, H) || !mul_ok(st, N) || !mul_ok(st, N) || tok > (size_t(1) << 40))
        return fail(WKV7_ERR_ARG, "sizes overflow");
    const size_t in_bytes = T ? tok * elem_bytes(dt) : 0, g_bytes = T ? tok * 4 : 0, st_bytes = st * 4;
    if (T > 0) {
        const void *req[] = {r, w, k, v, kk, a, dy, dr, dw, dk, dv, dkk, da};
        const char *names[] = {"r", "w", "k", "v", "kk", "a", "dy", "dr", "dw", "dk", "dv", "dkk", "da"};
        for (int i = 0; i < 13; ++i)
            if (!req[i]) return fail(WKV7_ERR_ARG, "%s is NULL", names[i]);
    }
    // inputs 0-9, outputs 10-16, workspace 17
    const Buf bufs[] = {{"r", r, in_bytes},   {"w", w, in_bytes},   {"k", k, in_bytes},
                        {"v", v, in_bytes},   {"kk", kk, in_bytes}, {"a", a, in_bytes},
                        {"S0", S0, st_bytes}, {"snapshots", n_snap ? snapshots : nullptr, st_bytes * n_snap},
                        {"dy", dy, g_bytes},  {"dS_T", dS_T, st_bytes},
                        {"dr", dr, g_bytes},  {"dw", dw, g_bytes},  {"dk", dk, g_bytes},
                        {"dv", dv, g_bytes},  {"dkk", dkk, g_bytes}, {"da", da, g_bytes},
                        {"dS0", dS0, st_bytes}, {"workspace", workspace, workspace_bytes}};
    constexpr int nb = sizeof(bufs) / sizeof(bufs[0]);
    for (int i = 0; i < nb; ++i)
        if (bufs[i].ptr && !aligned16(bufs[i].ptr))
            return fail(WKV7_ERR_ALIGN, "%s is not 16-byte aligned", bufs[i].name);
    const size_t need_ws = wkv7_backward_workspace_bytes(B, T, H, N, snap_every);
    if (need_ws > 0 && (!workspace || workspace_bytes < need_ws))
        return fail(WKV7_ERR_WORKSPACE, "workspace of %zu bytes required, %zu given", need_ws,
                    workspace ? workspace_bytes : 0);
    const Buf ws_used{"workspace", workspace, need_ws};
    for (int o = 10; o < nb; ++o) {   // outputs (and the workspace) overlap nothing else
        const Buf &ob = o == nb - 1 ? ws_used : bufs[o];
        for (int i = 0; i < nb - 1; ++i)
            if (i != o && overlaps(ob, bufs[i]) && !(o == 16 && i == 9 && dS0 == dS_T))   // dS0 = dS_T in place
                return fail(WKV7_ERR_ARG, "%s overlaps %s", ob.name, bufs[i].name);
    }
    int device = 0;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e, "cudaGetDevice");
    }
    for (int i = 0; i < nb; ++i) {
        const wkv7_status s = check_device_buffer(i == nb - 1 ? ws_used : bufs[i], device);
        if (s != WKV7_OK) return s;
    }
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (T == 0) {   // dS0 <- dS_T (or zeros)
        if (!dS0) return WKV7_OK;
        wkv7::FwdArgs c{};
        c.B = B; c.H = H; c.N = N; c.S0 = dS_T; c.S_T = dS0; c.stream = cs;
        e = wkv7::launch_copy_state(c);
        return e == cudaSuccess ? WKV7_OK : cuda_fail(e, "state-gradient copy launch");
    }
    wkv7::BwdArgs p{};
    p.B = B; p.T = T; p.H = H; p.dt = dt;
    p.r = r; p.w = w; p.k = k; p.v = v; p.kk = kk; p.a = a;
    p.S0 = S0; p.snaps = n_snap ? snapshots : nullptr; p.snap_every = n_snap ? snap_every : 0;
    p.dy = dy; p.dS_T = dS_T;
    p.dr = dr; p.dw = dw; p.dk = dk; p.dv = dv; p.dkk = dkk; p.da = da; p.dS0 = dS0;
    p.ws = static_cast<float *>(workspace);
    p.stream = cs;
    e = wkv7::launch_backward_n(p, N);
    return e == cudaSuccess ? WKV7_OK : cuda_fail(e, "backward launch");
}

}  // extern "C"

namespace {

// Shared checks of the epilogue entries: sizes, dtype, head size, the epilogue's inputs.
wkv7_status epilogue_args(int B, int T, int H, int N, wkv7_dtype dt, float gn_eps, size_t &tok) {
    if (B <= 0 || H <= 0 || N <= 0 || T < 0) return fail(WKV7_ERR_ARG, "bad sizes B=%d T=%d H=%d N=%d", B, T, H, N);
    if (N != wkv7::kN && N != 128) return fail(WKV7_ERR_UNSUPPORTED, "head size N=%d: N=64 and N=128 are implemented", N);
    if (dt != WKV7_F32 && dt != WKV7_BF16) return fail(WKV7_ERR_ARG, "unknown dtype %d", (int)dt);
    if (!(gn_eps > 0.f) || !std::isfinite(gn_eps)) return fail(WKV7_ERR_ARG, "gn_eps must be finite and > 0");
    tok = 1;
    if (!mul_ok(tok, B) || !mul_ok(tok, T) || !mul_ok(tok, H) || !mul_ok(tok, N) || tok > (size_t(1) << 40))
        return fail(WKV7_ERR_ARG, "sizes overflow");
    return WKV7_OK;
}

// Alignment, device placement and overlaps of bufs[0 .. n): entries from `first_out` on are outputs
// and may overlap nothing else, except the pairs the caller allows through `allowed`.
template <class Allowed>
wkv7_status check_buffers(const Buf *bufs, int n, int first_out, Allowed allowed) {
    for (int i = 0; i < n; ++i) {
        if (bufs[i].bytes && !bufs[i].ptr) return fail(WKV7_ERR_ARG, "%s is NULL", bufs[i].name);
        if (bufs[i].ptr && !aligned16(bufs[i].ptr)) return fail(WKV7_ERR_ALIGN, "%s is not 16-byte aligned", bufs[i].name);
    }
    for (int o = first_out; o < n; ++o)
        for (int i = 0; i < n; ++i)
            if (i != o && overlaps(bufs[o], bufs[i]) && !allowed(o, i))
                return fail(WKV7_ERR_ARG, "%s overlaps %s", bufs[o].name, bufs[i].name);
    int device = 0;
    cudaError_t e = cudaGetDevice(&device);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return cuda_fail(e, "cudaGetDevice");
    }
    for (int i = 0; i < n; ++i) {
        const wkv7_status s = check_device_buffer(bufs[i], device);
        if (s != WKV7_OK) return s;
    }
    return WKV7_OK;
}

// The decode entries: sizes, the epilogue and raw-input arguments, then every buffer (inputs,
// per-head parameters, the in/out state S and y) checked before the launch.
wkv7_status decode_impl(int B, int H, int N, wkv7_dtype dt, const void *r, const void *w, const void *k,
                        const void *v, const void *kk, const void *a, float *S, float *y, bool raw,
                        const float *k_k, const float *k_a, const float *ln_w, const float *ln_b,
                        const float *r_k, float gn_eps, void *stream) {
    if (N <= 0 || B <= 0 || H <= 0) return fail(WKV7_ERR_ARG, "bad sizes B=%d H=%d N=%d", B, H, N);
    if (N != wkv7::kN && N != 128)
        return fail(WKV7_ERR_UNSUPPORTED, "head size N=%d: N=64 and N=128 are implemented", N);
    if (dt != WKV7_F32 && dt != WKV7_BF16) return fail(WKV7_ERR_ARG, "unknown dtype %d", (int)dt);
    size_t tok = 1;
    if (!mul_ok(tok, B) || !mul_ok(tok, H) || !mul_ok(tok, N) || tok > (size_t(1) << 36))
        return fail(WKV7_ERR_ARG, "sizes overflow");
    const int n_epi = (ln_w != nullptr) + (ln_b != nullptr) + (r_k != nullptr);
    if (n_epi != 0 && n_epi != 3) return fail(WKV7_ERR_ARG, "epilogue needs ln_w, ln_b and r_k (or none)");
    if (n_epi == 3 && (!(gn_eps > 0.f) || !std::isfinite(gn_eps)))
        return fail(WKV7_ERR_ARG, "gn_eps must be finite and > 0");
    if (raw && !k_k) return fail(WKV7_ERR_ARG, "k_k is NULL");
    const size_t in = tok * elem_bytes(dt), ph = size_t(H) * N * 4, pe = n_epi ? ph : 0;
    const Buf bufs[] = {{"r", r, in},
                        {raw ? "w_logit" : "w", w, in},
                        {"k", k, in},
                        {"v", v, in},
                        {"kk", kk, raw ? 0 : in},
                        {raw ? "a_logit" : "a", a, in},
                        {"k_k", k_k, raw ? ph : 0},
                        {"k_a", k_a, k_a ? ph : 0},
                        {"ln_w", ln_w, pe},
                        {"ln_b", ln_b, pe},
                        {"r_k", r_k, pe},
                        {"S", S, tok * N * 4},
                        {"y", y, tok * 4}};
    const wkv7_status st = check_buffers(bufs, 13, 11, [](int, int) { return false; });
    if (st != WKV7_OK) return st;
    wkv7::DecArgs p{B, H, N, dt, r, w, k, v, raw ? nullptr : kk, a, S, y, static_cast<cudaStream_t>(stream)};
    wkv7::DecOpts o;
    if (raw) {
        o.k_k = k_k;
        o.k_a = k_a;
    }
    if (n_epi) {
        o.ln_w = ln_w;
        o.ln_b = ln_b;
        o.r_k = r_k;
        o.gn_eps = gn_eps;
    }
    const cudaError_t e = wkv7::launch_decode_ex(p, o);
    return e == cudaSuccess ? WKV7_OK : cuda_fail(e, "decode launch");
}

}  // namespace

extern "C" {

wkv7_status wkv7_epilogue(int B, int T, int H, int N, wkv7_dtype dt, const float *y, const void *r, const void *k,
                          const void *v, const float *ln_w, const float *ln_b, const float *r_k, float gn_eps,
                          float *out, void *stream) {
    g_err[0] = '\0';
    size_t tok = 0;
    wkv7_status st = epilogue_args(B, T, H, N, dt, gn_eps, tok);
    if (st != WKV7_OK) return st;
    if (T == 0) return WKV7_OK;
    const size_t in = tok * elem_bytes(dt), f = tok * 4, ph = size_t(H) * N * 4;
    const Buf bufs[] = {{"y", y, f},         {"r", r, in},       {"k", k, in},     {"v", v, in},
                        {"ln_w", ln_w, ph},  {"ln_b", ln_b, ph}, {"r_k", r_k, ph}, {"out", out, f}};
    st = check_buffers(bufs, 8, 7, [&](int o, int i) { return o == 7 && i == 0 && out == y; });
    if (st != WKV7_OK) return st;
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaSuccess;
    if (out != y && (e = cudaMemcpyAsync(out, y, f, cudaMemcpyDeviceToDevice, cs)) != cudaSuccess)
        return cuda_fail(e, "copy of y");
    wkv7::FwdArgs p{};
    p.B = B; p.T = T; p.H = H; p.N = N; p.dt = dt;
    p.r = r; p.k = k; p.v = v; p.y = out;
    p.ln_w = ln_w; p.ln_b = ln_b; p.r_k = r_k; p.gn_eps = gn_eps; p.raw = false; p.stream = cs;
    e = wkv7::launch_epilogue(p);
    return e == cudaSuccess ? WKV7_OK : cuda_fail(e, "epilogue launch");
}

size_t wkv7_epilogue_backward_workspace_bytes(int B, int T, int H, int N) {
    if (B <= 0 || T < 0 || H <= 0 || (N != wkv7::kN && N != 128)) return 0;
    size_t tok = 1;
    if (!mul_ok(tok, B) || !mul_ok(tok, T) || !mul_ok(tok, H) || !mul_ok(tok, N) || tok > (size_t(1) << 40)) return 0;
    return wkv7::epilogue_backward_partials(B, T, H, N) * sizeof(float);
}

wkv7_status wkv7_epilogue_backward(int B, int T, int H, int N, wkv7_dtype dt, const float *y, const void *r,
                                   const void *k, const void *v, const float *ln_w, const float *ln_b,
                                   const float *r_k, float gn_eps, const float *dout, float *dy, float *dr,
                                   float *dk, float *dv, float *dln_w, float *dln_b, float *dr_k, void *workspace,
                                   size_t workspace_bytes, void *stream) {
    g_err[0] = '\0';
    size_t tok = 0;
    wkv7_status st = epilogue_args(B, T, H, N, dt, gn_eps, tok);
    if (st != WKV7_OK) return st;
    const size_t in = tok * elem_bytes(dt), f = tok * 4, ph = size_t(H) * N * 4;
    const size_t need = wkv7_epilogue_backward_workspace_bytes(B, T, H, N);
    if (need > 0 && (!workspace || workspace_bytes < need))
        return fail(WKV7_ERR_WORKSPACE, "workspace of %zu bytes required, %zu given", need, workspace ? workspace_bytes : 0);
    // inputs 0-7, outputs 8-14, workspace 15
    const Buf bufs[] = {{"y", y, f},          {"r", r, in},         {"k", k, in},         {"v", v, in},
                        {"ln_w", ln_w, ph},   {"ln_b", ln_b, ph},   {"r_k", r_k, ph},     {"dout", dout, f},
                        {"dy", dy, f},        {"dr", dr, f},        {"dk", dk, f},        {"dv", dv, f},
                        {"dln_w", dln_w, ph}, {"dln_b", dln_b, ph}, {"dr_k", dr_k, ph},   {"workspace", workspace, need}};
    st = check_buffers(bufs, 16, 8, [](int, int) { return false; });
    if (st != WKV7_OK) return st;
    wkv7::EpiBwdArgs a{};
    a.B = B; a.T = T; a.H = H; a.N = N; a.dt = dt;
    a.y = y; a.r = r; a.k = k; a.v = v; a.ln_w = ln_w; a.ln_b = ln_b; a.r_k = r_k; a.eps = gn_eps;
    a.dout = dout; a.dy = dy; a.dr = dr; a.dk = dk; a.dv = dv; a.dln_w = dln_w; a.dln_b = dln_b; a.dr_k = dr_k;
    a.ws = static_cast<float *>(workspace);
    a.stream = static_cast<cudaStream_t>(stream);
    const cudaError_t e = wkv7::launch_epilogue_backward(a);
    return e == cudaSuccess ? WKV7_OK : cuda_fail(e, "epilogue backward launch");
}

}  // extern "C"
