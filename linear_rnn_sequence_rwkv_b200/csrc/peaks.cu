// Peak-rate probes: the FP32 FMA pipe and the tf32 tensor-core path (tcgen05.mma kind::tf32),
// each driven at full rate by a kernel that does nothing else, so that the caller can time a
// launch with CUDA events and divide the flops it reports by that time. They stand for the
// "alu" and "tensor" roofline denominators of the kernels in this library: the scan and the
// backward run on the FMA pipe, the chunked prefill on tf32 MMAs of M = 128 and N = 64..256.
#include "common.cuh"
#include "tc_util.cuh"

namespace wkv7 {
namespace {

using namespace tc;

constexpr int kFmaThreads = 256;
constexpr int kFmaChains = 8;    // independent FMA chains per thread (covers the pipe latency)
constexpr int kFmaUnroll = 16;

// a <- a * b + c on kFmaChains independent chains; b and c come from the host so nothing folds.
__global__ void __launch_bounds__(kFmaThreads) fma_peak_kernel(float b, float c, int iters, float *sink) {
    float a[kFmaChains];
#pragma unroll
    for (int i = 0; i < kFmaChains; ++i) a[i] = float(threadIdx.x) * 1e-3f + float(i);
    for (int it = 0; it < iters; ++it) {
#pragma unroll
        for (int u = 0; u < kFmaUnroll; ++u)
#pragma unroll
            for (int i = 0; i < kFmaChains; ++i) a[i] = fmaf(a[i], b, c);
    }
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kFmaChains; ++i) s += a[i];
    if (s == -1.2345f) sink[blockIdx.x] = s;   // keeps the chains live; never true for these inputs
}

// One CTA per SM: thread 0 issues `iters` rounds of four K = 8 steps of a 128 x N x 32 tf32 MMA
// from zeroed shared-memory operands into one TMEM accumulator, then waits (bounded) for the
// last one. The other threads only allocate and free tensor memory.
template <int N>
__global__ void __launch_bounds__(128, 1) tf32_mma_peak_kernel(int iters, unsigned int *err) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
    constexpr uint32_t kA = 128 * 128, kB = N * 128;   // bytes: 128 (A) and N (B) rows of 32 tf32
    __shared__ uint64_t bar;
    __shared__ uint32_t tmem_base;
    for (uint32_t i = threadIdx.x; i < (kA + kB) / 16; i += blockDim.x)
        reinterpret_cast<uint4 *>(sm)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async_smem();
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_fence_init();
    }
    if (threadIdx.x < 32) {
        tmem_alloc(&tmem_base, N < 32 ? 32 : N);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = tmem_base;
    if (threadIdx.x == 0) {
        const uint64_t dA = desc_sw128(smem_u32(sm)), dB = desc_sw128(smem_u32(sm + kA));
        for (int it = 0; it < iters; ++it)
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_tf32_ss(tb, dA + kstep_off(ks, 128), dB + kstep_off(ks, N), idesc_tf32(128, N), (it | ks) != 0);
        mma_commit(&bar);
        if (!mbar_wait(&bar, 0, 2000000000ull)) {
            atomicOr(err, 1u);
            mbar_wait(&bar, 0, 2000000000ull);   // the MMAs may still run: wait once more before freeing
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x < 32) tmem_dealloc(tb, N < 32 ? 32 : N);
}

template <int N>
cudaError_t launch_mma_peak(int ctas, int iters, cudaStream_t stream, unsigned int *err) {
    const int smem = 128 * 128 + N * 128 + 1024;
    cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void *>(tf32_mma_peak_kernel<N>), smem);
    if (e != cudaSuccess) return e;
    tf32_mma_peak_kernel<N><<<ctas, 128, smem, stream>>>(iters, err);
    return cudaGetLastError();
}

}  // namespace

// ---- host side ---------------------------------------------------------------------------------------

cudaError_t launch_fma_peak(int blocks, int iters, cudaStream_t stream, double *flops) {
    fma_peak_kernel<<<blocks, kFmaThreads, 0, stream>>>(0.9999999f, 1e-7f, iters, nullptr);
    *flops = 2.0 * kFmaChains * kFmaUnroll * double(iters) * kFmaThreads * blocks;
    return cudaGetLastError();
}

cudaError_t launch_tf32_mma_peak(int n, int iters, cudaStream_t stream, double *flops) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    unsigned int *err = nullptr;
    if ((e = device_error_word(&err)) != cudaSuccess) return e;
    switch (n) {
        case 64: e = launch_mma_peak<64>(sms, iters, stream, err); break;
        case 128: e = launch_mma_peak<128>(sms, iters, stream, err); break;
        case 256: e = launch_mma_peak<256>(sms, iters, stream, err); break;
        default: return cudaErrorInvalidValue;
    }
    *flops = 2.0 * 128.0 * n * 32.0 * double(iters) * sms;
    return e;
}

}  // namespace wkv7
