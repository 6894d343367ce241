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
#include "common.cuh"

namespace wkv7 {
namespace {

constexpr int kDecThreads = 256;

// NN = 64: the layout above. NN = 128: a warp covers one 512-byte row (32 float4 columns) and
// a thread holds rows t/32 + 8m, m = 0..15; the row dot products reduce over the 32 lanes.
template <class Tin, int NN>
__global__ void __launch_bounds__(kDecThreads) decode_kernel(const DecArgs p) {
    constexpr int CL = NN / 4;                  // lanes per row (one float4 each)
    constexpr int RS = kDecThreads / CL;        // row stride between a thread's rows
    constexpr int RPT = NN / RS;                // rows per thread
    const int unit = blockIdx.x;
    const int c4 = threadIdx.x % CL, rbase = threadIdx.x / CL;
    float *S = p.S + size_t(unit) * NN * NN;
    const size_t vo = size_t(unit) * NN;

    float4 s[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) s[m] = __ldcs(reinterpret_cast<const float4 *>(S + (rbase + RS * m) * NN + 4 * c4));

    const Tin *r = static_cast<const Tin *>(p.r), *w = static_cast<const Tin *>(p.w);
    const Tin *k = static_cast<const Tin *>(p.k), *v = static_cast<const Tin *>(p.v);
    const Tin *kk = static_cast<const Tin *>(p.kk), *a = static_cast<const Tin *>(p.a);
    const float4 w4 = load4(w + vo + 4 * c4), kk4 = load4(kk + vo + 4 * c4), a4 = load4(a + vo + 4 * c4);
    const float4 k4 = load4(k + vo + 4 * c4), r4 = load4(r + vo + 4 * c4);
    float vi[RPT];
#pragma unroll
    for (int m = 0; m < RPT; ++m) vi[m] = load1(v + vo + rbase + RS * m);
    const float4 b4 = make_float4(kk4.x * a4.x, kk4.y * a4.y, kk4.z * a4.z, kk4.w * a4.w);

#pragma unroll
    for (int m = 0; m < RPT; ++m) {
        float sk = dot4(s[m], kk4);
#pragma unroll
        for (int o = CL / 2; o; o >>= 1) sk += __shfl_xor_sync(0xffffffffu, sk, o);
        float4 x;
        x.x = fmaf(vi[m], k4.x, fmaf(-sk, b4.x, s[m].x * w4.x));
        x.y = fmaf(vi[m], k4.y, fmaf(-sk, b4.y, s[m].y * w4.y));
        x.z = fmaf(vi[m], k4.z, fmaf(-sk, b4.z, s[m].z * w4.z));
        x.w = fmaf(vi[m], k4.w, fmaf(-sk, b4.w, s[m].w * w4.w));
        float yv = dot4(x, r4);
#pragma unroll
        for (int o = CL / 2; o; o >>= 1) yv += __shfl_xor_sync(0xffffffffu, yv, o);
        __stcs(reinterpret_cast<float4 *>(S + (rbase + RS * m) * NN + 4 * c4), x);
        if (c4 == 0) p.y[vo + rbase + RS * m] = yv;
    }
}

}  // namespace

// ---- host side ---------------------------------------------------------------------------------------

cudaError_t launch_decode(const DecArgs &p) {
    const unsigned units = unsigned(p.B) * unsigned(p.H);
    if (p.N == 128) {
        if (p.dt == WKV7_BF16)
            decode_kernel<__nv_bfloat16, 128><<<units, kDecThreads, 0, p.stream>>>(p);
        else
            decode_kernel<float, 128><<<units, kDecThreads, 0, p.stream>>>(p);
    } else if (p.dt == WKV7_BF16) {
        decode_kernel<__nv_bfloat16, 64><<<units, kDecThreads, 0, p.stream>>>(p);
    } else {
        decode_kernel<float, 64><<<units, kDecThreads, 0, p.stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace wkv7
