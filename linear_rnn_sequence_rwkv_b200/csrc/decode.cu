// One WKV-7 decode step for every (b, h): the recurrence for a single token with the
// fp32 state read from and written back to HBM (RWKV-7 paper summary, section 8:
// single-token inference at constant memory; update and readout as in the
// rebuttal page's numpy time_mixing listing).
//
// The step moves 16 KB of state in and 16 KB out per head for ~37 kflop, so it is
// bound by HBM bandwidth. One 256-thread CTA owns one head: thread t holds one
// float4 of columns 4*(t%16)..+3 in each of the rows t/16 + 16m, m = 0..3, so a
// half-warp covers one 256-byte row and a warp moves 512 contiguous bytes per load
// or store. All four rows are loaded before any arithmetic to keep 64 bytes per
// thread in flight. Row dot products (removed value, readout) reduce over the 16
// lanes of the half-warp.
#include "decode.cuh"

namespace wkv7 {
namespace {

constexpr int kDecThreads = 256;

// NN = 64: the layout above (THREADS = 128, as the fused steps run: rows t/16 + 8m, m = 0..7).
// NN = 128: a warp covers one 512-byte row (32 float4 columns) and a thread holds rows
// t/32 + 8m, m = 0..15; the row dot products reduce over the 32 lanes.
// RAW: w and a hold the decay and rate logits and k the key before its update; the load turns
// them into w, a, the unit-norm removal key kk (its norm reduced over the CL lanes that hold
// one row's channels) and the updated key k~ (rebuttal page, the time_mixing listing: decay,
// learning rate, removal key with its 1e-12 norm floor, key update).
// EPI: the head's N readouts meet in shared memory; the first N threads normalise them over
// the head (group_norm, population variance plus gn_eps) and add the bonus
// (sum_j r_j k_j r_k[j]) v_i (rebuttal page, the listing's output lines).
template <class Tin, int NN, bool RAW, bool EPI, int THREADS = kDecThreads>
__device__ __forceinline__ void decode_body(const DecArgs &p, const DecOpts &o) {
    constexpr int CL = NN / 4;                  // lanes per row (one float4 each)
    constexpr int RS = THREADS / CL;            // row stride between a thread's rows
    constexpr int RPT = NN / RS;                // rows per thread
    __shared__ float ys[EPI ? NN : 1];
    const int unit = blockIdx.x, h = unit % p.H;
    const int c4 = threadIdx.x % CL, rbase = threadIdx.x / CL;
    float *S = p.S + size_t(unit) * NN * NN;
    const size_t vo = size_t(unit) * NN;
    auto lanes_sum = [](float x) {
#pragma unroll
        for (int off = CL / 2; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        return x;
    };

    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = __ldcs(reinterpret_cast<const float4 *>(S + (rbase + RS * m) * NN + 4 * c4));

    const Tin *r = static_cast<const Tin *>(p.r), *w = static_cast<const Tin *>(p.w);
    const Tin *k = static_cast<const Tin *>(p.k), *v = static_cast<const Tin *>(p.v);
    const Tin *kk = static_cast<const Tin *>(p.kk), *a = static_cast<const Tin *>(p.a);
    float4 w4, kk4, a4, k4;
    if constexpr (RAW) {
        w4 = load4(w + vo + 4 * c4);
        a4 = load4(a + vo + 4 * c4);
        k4 = load4(k + vo + 4 * c4);
        const int pc = h * NN + 4 * c4;
        // fast divisions, as in the chunked kernel's load stage: exp overflow gives 0, the limit
        auto decay = [](float z) { return __expf(__fdividef(-0.60653065971263342f, 1.f + __expf(-z))); };   // e^-1/2
        auto sigm = [](float z) { return __fdividef(1.f, 1.f + __expf(-z)); };
        w4 = make_float4(decay(w4.x), decay(w4.y), decay(w4.z), decay(w4.w));
        a4 = make_float4(sigm(a4.x), sigm(a4.y), sigm(a4.z), sigm(a4.w));
        const float4 kkp = __ldg(reinterpret_cast<const float4 *>(o.k_k + pc));
        kk4 = make_float4(k4.x * kkp.x, k4.y * kkp.y, k4.z * kkp.z, k4.w * kkp.w);
        const float inv = rsqrtf(fmaxf(lanes_sum(dot4(kk4, kk4)), 1e-24f));   // 1 / max(||.||, 1e-12)
        kk4 = make_float4(kk4.x * inv, kk4.y * inv, kk4.z * inv, kk4.w * inv);
        if (o.k_a) {
            const float4 ka = __ldg(reinterpret_cast<const float4 *>(o.k_a + pc));
            k4 = make_float4(fmaf(k4.x * (a4.x - 1.f), ka.x, k4.x), fmaf(k4.y * (a4.y - 1.f), ka.y, k4.y),
                             fmaf(k4.z * (a4.z - 1.f), ka.z, k4.z), fmaf(k4.w * (a4.w - 1.f), ka.w, k4.w));
        }
    } else {
        w4 = load4(w + vo + 4 * c4);
        kk4 = load4(kk + vo + 4 * c4);
        a4 = load4(a + vo + 4 * c4);
        k4 = load4(k + vo + 4 * c4);
    }
    const float4 r4 = load4(r + vo + 4 * c4);
    float vi[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) vi[m] = load1(v + vo + rbase + RS * m);
    const float4 b4 = make_float4(kk4.x * a4.x, kk4.y * a4.y, kk4.z * a4.z, kk4.w * a4.w);

#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        const float sk = lanes_sum(dot4(s[m], kk4));
        float4 x;
        x.x = fmaf(vi[m], k4.x, fmaf(-sk, b4.x, s[m].x * w4.x));
        x.y = fmaf(vi[m], k4.y, fmaf(-sk, b4.y, s[m].y * w4.y));
        x.z = fmaf(vi[m], k4.z, fmaf(-sk, b4.z, s[m].z * w4.z));
        x.w = fmaf(vi[m], k4.w, fmaf(-sk, b4.w, s[m].w * w4.w));
        const float yv = lanes_sum(dot4(x, r4));
        __stcs(reinterpret_cast<float4 *>(S + (rbase + RS * m) * NN + 4 * c4), x);
        if (c4 == 0) {
            if constexpr (EPI) ys[rbase + RS * m] = yv;
            else p.y[vo + rbase + RS * m] = yv;
        }
    }
    if constexpr (EPI) {
        // bonus over the key channels: the CL lanes of every row group hold all of them
        const float4 rk = __ldg(reinterpret_cast<const float4 *>(o.r_k + h * NN + 4 * c4));
        const float bon = lanes_sum(fmaf(r4.x * k4.x, rk.x, fmaf(r4.y * k4.y, rk.y,
                                    fmaf(r4.z * k4.z, rk.z, r4.w * k4.w * rk.w))));
        __syncthreads();
        if (threadIdx.x >= NN) return;          // whole warps: NN is a multiple of 32
        constexpr int E = NN / 32;              // readouts per lane for the statistics
        const int lane = threadIdx.x & 31;
        float yv[E], sum = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            yv[e] = ys[E * lane + e];
            sum += yv[e];
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        const float mean = sum * (1.f / NN);
        float sq = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) sq = fmaf(yv[e] - mean, yv[e] - mean, sq);
#pragma unroll
        for (int off = 16; off; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
        const float inv = 1.f / sqrtf(sq * (1.f / NN) + o.gn_eps);
        const int i = threadIdx.x, pc = h * NN + i;
        p.y[vo + i] = (ys[i] - mean) * inv * o.ln_w[pc] + o.ln_b[pc] + bon * load1(v + vo + i);
    }
}

// The prepared-input step, and the steps with raw inputs and/or the epilogue. At N = 64 the fused
// steps run 128 threads per head (eight rows each): half as many row groups repeat the
// pre-processing and the bonus. Measured on B256 H40 against 256 threads: raw inputs with the
// epilogue 54.4 against 66.5 us (bound of eight CTAs per SM), raw inputs 55.9 against 58.1 and the
// epilogue alone 58.4 against 59.1 us (bound of six).
template <int NN> constexpr int kFusedThreads = NN == 64 ? 128 : kDecThreads;
template <int NN, bool RAW, bool EPI> constexpr int kFusedMinCtas = NN == 64 ? (RAW && EPI ? 8 : 6) : 2;
template <class Tin, int NN>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const DecArgs p) {
    decode_body<Tin, NN, false, false>(p, DecOpts{});
}
template <class Tin, int NN, bool RAW, bool EPI>
__global__ void __launch_bounds__(kFusedThreads<NN>, (kFusedMinCtas<NN, RAW, EPI>))
    decode_fused_kernel(const DecArgs p, const DecOpts o) {
    decode_body<Tin, NN, RAW, EPI, kFusedThreads<NN>>(p, o);
}

template <class Tin, int NN>
cudaError_t launch_dec_t(const DecArgs &p, const DecOpts &o) {
    const unsigned units = unsigned(p.B) * unsigned(p.H);
    const bool raw = o.k_k != nullptr, epi = o.ln_w != nullptr;
    if (raw && epi)
        decode_fused_kernel<Tin, NN, true, true><<<units, kFusedThreads<NN>, 0, p.stream>>>(p, o);
    else if (raw)
        decode_fused_kernel<Tin, NN, true, false><<<units, kFusedThreads<NN>, 0, p.stream>>>(p, o);
    else if (epi)
        decode_fused_kernel<Tin, NN, false, true><<<units, kFusedThreads<NN>, 0, p.stream>>>(p, o);
    else
        decode_kernel<Tin, NN><<<units, kDecThreads, 0, p.stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

// ---- host side ---------------------------------------------------------------------------------------

cudaError_t launch_decode_ex(const DecArgs &p, const DecOpts &o) {
    if (p.N == 128) return p.dt == WKV7_BF16 ? launch_dec_t<__nv_bfloat16, 128>(p, o) : launch_dec_t<float, 128>(p, o);
    return p.dt == WKV7_BF16 ? launch_dec_t<__nv_bfloat16, 64>(p, o) : launch_dec_t<float, 64>(p, o);
}

cudaError_t launch_decode(const DecArgs &p) { return launch_decode_ex(p, DecOpts{}); }

}  // namespace wkv7
