// The projections of the time-mixing layer: D[M][N] = op(A)[M][K] * W[N][K]^T with the operand's
// preparation fused into its load and the element-wise step after the product fused into the
// store (RWKV-7 rebuttal page, numpy time_mixing listing: the token-shift mixes feed the square
// projections and the low-rank first factors; tanh, sigmoid, the biases and the value residual
// follow them; the gate multiplies the readout before the output projection).
//
// Operand preparation (A, per element, in fp32, then rounded to the layer dtype):
//   PLAIN  A itself;
//   MIX    x + m (x_prev - x), x_prev the previous token of the same sequence (last_x, or 0,
//          for the first token);
//   GATE   y * g (both fp32).
// Store (per element of the fp32 accumulator z, column n):
//   STORE z;  TANH tanh(z);  SIGMOID sigmoid(z);  BIAS z + bias[n];
//   RESIDUAL v + (v0 - v) sigmoid(z + bias[n]) with v the value already in D;  F32 z in fp32.
//
// bf16 layers: tcgen05.mma kind::f16 (bf16 operands, fp32 accumulation in tensor memory), a
// 128 x BN output tile per CTA, K in blocks of 64. W arrives by TMA (128-byte swizzle); eight
// warps prepare A into the same swizzled layout and later read the accumulator back; one thread
// issues the MMAs. fp32 layers: a shared-memory tiled FMA GEMM with the same preparation and
// store steps (exact fp32 products, fp32 accumulation).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

#include "common.cuh"
#include "tc_util.cuh"

namespace wkv7 {
namespace {

using namespace tc;

__device__ __forceinline__ float sigmoidf_(float z) { return 1.f / (1.f + __expf(-z)); }

// Named barrier over `n` threads that also ORs a predicate (the result is uniform).
__device__ __forceinline__ bool bar_or(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(uint32_t(v)), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float apply_epi(int epi, float z, float bias, float v, float v0) {
    switch (epi) {
        case GEMM_TANH: return tanhf(z);
        case GEMM_SIGMOID: return sigmoidf_(z);
        case GEMM_BIAS: return z + bias;
        case GEMM_RESIDUAL: return fmaf(v0 - v, sigmoidf_(z + bias), v);
        default: return z;
    }
}

__device__ __forceinline__ float bf(uint32_t packed, int hi) {
    return __uint_as_float(hi ? (packed & 0xffff0000u) : (packed << 16));
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// ---- bf16 on tcgen05 -------------------------------------------------------------------------------
constexpr int kProdThreads = 256;                 // warps 0-7: A preparation (MIX, GATE), then the store
constexpr int kGemmThreads = kProdThreads + 64;   // warp 8: TMA; warp 9: MMA issue and TMEM
constexpr int kStages = 4;

// One stage: the A tile (128 rows x 64 K, bf16, 128-byte swizzle), the previous-token tile of the
// mix (the same rows shifted by one token), and the W tile (BN rows).
template <int BN>
struct GemmSmem {
    static constexpr uint32_t A = 128 * 128, XP = 128 * 128, B = BN * 128, STAGE = A + XP + B;
    static constexpr uint32_t bytes = kStages * STAGE + 1024 + 256;
};

// GATE: eight bf16 values of A's row m, columns k..k+7 (k a multiple of 8): y * g from fp32.
__device__ __forceinline__ uint4 gate_a8(const GemmArgs &a, int m, int k) {
    if (m >= a.M) return make_uint4(0u, 0u, 0u, 0u);
    const float *yr = a.y + size_t(m) * a.K + k, *gr = static_cast<const float *>(a.g) + size_t(m) * a.K + k;
    const float4 y0 = __ldg(reinterpret_cast<const float4 *>(yr)), y1 = __ldg(reinterpret_cast<const float4 *>(yr + 4));
    const float4 g0 = __ldg(reinterpret_cast<const float4 *>(gr)), g1 = __ldg(reinterpret_cast<const float4 *>(gr + 4));
    return make_uint4(pack_bf16(y0.x * g0.x, y0.y * g0.y), pack_bf16(y0.z * g0.z, y0.w * g0.w),
                      pack_bf16(y1.x * g1.x, y1.y * g1.y), pack_bf16(y1.z * g1.z, y1.w * g1.w));
}

// MIX, in place in the stage: A chunk (row r, 16-byte chunk at byte `off` of the swizzled tile)
// <- x + m (x_prev - x), with x_prev from the shifted tile, or last_x (0 without it) when row
// m0 + r starts a sequence.
__device__ __forceinline__ void mix_chunk(const GemmArgs &a, uint8_t *at, const uint8_t *xpt, int m, int k,
                                          uint32_t off) {
    if (m >= a.M) return;
    uint4 xc = *reinterpret_cast<const uint4 *>(at + off), xp;
    if (m % a.T != 0) xp = *reinterpret_cast<const uint4 *>(xpt + off);
    else if (a.last_x)
        xp = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.last_x) + size_t(m / a.T) * a.K + k));
    else xp = make_uint4(0u, 0u, 0u, 0u);
    const float4 m0 = __ldg(reinterpret_cast<const float4 *>(a.mix + k));
    const float4 m1 = __ldg(reinterpret_cast<const float4 *>(a.mix + k + 4));
    const float mv[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
    const uint32_t xcw[4] = {xc.x, xc.y, xc.z, xc.w}, xpw[4] = {xp.x, xp.y, xp.z, xp.w};
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float xi = bf(xcw[e >> 1], e & 1), pi = bf(xpw[e >> 1], e & 1);
        o[e] = fmaf(mv[e], pi - xi, xi);
    }
    *reinterpret_cast<uint4 *>(at + off) =
        make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7]));
}

// PLAIN: A by TMA straight into the stage. MIX: x and the previous-token rows by TMA, mixed in
// place by warps 0-7. GATE: A formed by warps 0-7 from global memory. W always by TMA.
template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_bf16_kernel(const __grid_constant__ CUtensorMap wmap,
                                                                    const __grid_constant__ CUtensorMap amap,
                                                                    const GemmArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
    using L = GemmSmem<BN>;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kStages * L::STAGE);
    uint64_t *full_t = bars, *full_a = bars + kStages, *empty = bars + 2 * kStages, *acc_full = bars + 3 * kStages;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 3 * kStages + 1);
    auto stA = [&](int s) { return sm + s * L::STAGE; };
    auto stXP = [&](int s) { return sm + s * L::STAGE + L::A; };
    auto stB = [&](int s) { return sm + s * L::STAGE + L::A + L::XP; };

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int m0 = blockIdx.x * 128, n0 = blockIdx.y * BN, nkb = a.K / 64;
    const bool tma_a = a.pro != GEMM_GATE, mix = a.pro == GEMM_MIX, prod = a.pro != GEMM_PLAIN;
    const uint64_t tmo = 2000000000ull;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_t[s], 1);
            mbar_init(&full_a[s], kProdThreads);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_fence_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tmem_slot;
    bool bad = false;

    if (warp < 8) {
        if (prod) {
            // 1024 16-byte chunks per stage, four per thread; chunk q of row r sits at chunk position
            // q ^ (r % 8) of the row (128-byte swizzle, K-major). Thread 0 polls the stage's barrier,
            // the others wait for it in a named barrier.
            for (int kb = 0; kb < nkb && !bad; ++kb) {
                const int s = kb % kStages;
                const uint32_t ph = (kb / kStages) & 1;
                const bool to = tid == 0 && (mix ? !mbar_wait_spin(&full_t[s], ph, tmo) : !mbar_wait_spin(&empty[s], ph ^ 1, tmo));
                if (bar_or(1, kProdThreads, to)) { bad = true; break; }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int idx = tid + kProdThreads * i, r = idx >> 3, q = idx & 7;
                    const uint32_t off = r * 128 + ((q ^ (r & 7)) << 4);
                    if (mix) mix_chunk(a, stA(s), stXP(s), m0 + r, kb * 64 + q * 8, off);
                    else *reinterpret_cast<uint4 *>(stA(s) + off) = gate_a8(a, m0 + r, kb * 64 + q * 8);
                }
                fence_proxy_async_smem();
                mbar_arrive(&full_a[s]);
            }
        }
    } else if (warp == 8) {
        if (lane == 0) {
            const uint32_t bytes = L::B + (tma_a ? L::A : 0u) + (mix ? L::XP : 0u);
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % kStages;
                if (!mbar_wait_spin(&empty[s], ((kb / kStages) & 1) ^ 1, tmo)) { bad = true; break; }
                mbar_arrive_expect_tx(&full_t[s], bytes);
                tma_load_2d(stB(s), &wmap, &full_t[s], kb * 64, n0);
                if (tma_a) tma_load_2d(stA(s), &amap, &full_t[s], kb * 64, m0);
                if (mix) tma_load_2d(stXP(s), &amap, &full_t[s], kb * 64, m0 - 1);   // row -1: zeros
            }
        }
    } else if (lane == 0) {
        // ---- MMA issue: four K = 16 steps per stage, then the stage goes back to its producers
        for (int kb = 0; kb < nkb; ++kb) {
            const int s = kb % kStages;
            const uint32_t ph = (kb / kStages) & 1;
            if (!mbar_wait_spin(&full_t[s], ph, tmo) || (prod && !mbar_wait_spin(&full_a[s], ph, tmo))) { bad = true; break; }
            tc_fence_after();
            const uint64_t dA = desc_sw128(smem_u32(stA(s))), dB = desc_sw128(smem_u32(stB(s)));
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma_bf16_ss(tb, dA + uint64_t(2 * ks), dB + uint64_t(2 * ks), idesc_bf16(128, BN), (kb | ks) != 0);
            mma_commit(&empty[s]);
        }
        mma_commit(acc_full);   // also after a failure: the store side waits for what was issued
    }

    // ---- store: warp w reads TMEM lanes 32 (w % 4) .. + 31 (rows), columns of its half
    if (warp < 8) {
        const bool ok = !bar_or(1, kProdThreads, tid == 0 && !mbar_wait_spin(acc_full, 0, tmo));
        if (!ok) bad = true;
        tc_fence_after();
        const int q = warp & 3, h = warp >> 2, m = m0 + 32 * q + lane;
        constexpr int HALF = BN / 2;
#pragma unroll 1
        for (int c0 = 0; c0 < HALF && ok; c0 += 32) {
            float z[32];
            tmem_ld32(tmem_addr(tb, 32 * q, h * HALF + c0), z);
            const int n = n0 + h * HALF + c0;
            if (m < a.M) {
                if (a.epi == GEMM_F32) {
                    float *d = static_cast<float *>(a.D) + size_t(m) * a.ldd + n;
#pragma unroll
                    for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4 *>(d + e) = make_float4(z[e], z[e + 1], z[e + 2], z[e + 3]);
                } else {
                    __nv_bfloat16 *d = static_cast<__nv_bfloat16 *>(a.D) + size_t(m) * a.ldd + n;
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        float o[8];
                        uint4 vv = make_uint4(0u, 0u, 0u, 0u), v0 = make_uint4(0u, 0u, 0u, 0u);
                        if (a.epi == GEMM_RESIDUAL) {
                            vv = *reinterpret_cast<const uint4 *>(d + e);
                            v0 = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(a.v0) +
                                                                       size_t(m) * a.ldd + n + e));
                        }
                        const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w}, v0w[4] = {v0.x, v0.y, v0.z, v0.w};
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            o[j] = apply_epi(a.epi, z[e + j], a.bias ? __ldg(a.bias + n + e + j) : 0.f, bf(vw[j >> 1], j & 1),
                                             bf(v0w[j >> 1], j & 1));
                        const uint4 w = make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]),
                                                   pack_bf16(o[6], o[7]));
                        *reinterpret_cast<uint4 *>(d + e) = w;
                        if (a.D2)
                            *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(a.D2) + size_t(m) * a.ldd + n + e) = w;
                    }
                }
            }
        }
    }
    if (bad && a.err) atomicOr(a.err, 1u);
    tc_fence_before();
    __syncthreads();
    if (warp == 9) tmem_dealloc(tb, BN);
}

// ---- fp32 on the FMA pipe ---------------------------------------------------------------------------
constexpr int kFT = 64, kFK = 16;   // 64 x 64 output tile, K in steps of 16; 256 threads, 4 x 4 each

__device__ __forceinline__ float prep_a1(const GemmArgs &a, int m, int k) {
    if (m >= a.M || k >= a.K) return 0.f;
    if (a.pro == GEMM_PLAIN) return static_cast<const float *>(a.A)[size_t(m) * a.lda + k];
    if (a.pro == GEMM_MIX) {
        const float *x = static_cast<const float *>(a.x);
        const float xi = x[size_t(m) * a.K + k];
        float xp = 0.f;
        if (m % a.T != 0) xp = x[size_t(m - 1) * a.K + k];
        else if (a.last_x) xp = static_cast<const float *>(a.last_x)[size_t(m / a.T) * a.K + k];
        return fmaf(a.mix[k], xp - xi, xi);
    }
    return a.y[size_t(m) * a.K + k] * static_cast<const float *>(a.g)[size_t(m) * a.K + k];
}

__global__ void __launch_bounds__(256) gemm_f32_kernel(const GemmArgs a) {
    __shared__ float As[kFK][kFT + 4], Bs[kFK][kFT + 4];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int m0 = blockIdx.x * kFT, n0 = blockIdx.y * kFT;
    const float *W = static_cast<const float *>(a.W);
    float acc[4][4] = {};
    for (int k0 = 0; k0 < a.K; k0 += kFK) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + 256 * i, r = e >> 4, k = e & 15;
            As[k][r] = prep_a1(a, m0 + r, k0 + k);
            const int n = n0 + r;
            Bs[k][r] = (n < a.N && k0 + k < a.K) ? W[size_t(n) * a.K + k0 + k] : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < kFK; ++k) {
            float av[4], bv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                av[i] = As[k][ty * 4 + i];
                bv[i] = Bs[k][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= a.M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= a.N) continue;
            float *d = static_cast<float *>(a.D) + size_t(m) * a.ldd + n;
            const float v = a.epi == GEMM_RESIDUAL ? *d : 0.f;
            const float v0 = a.epi == GEMM_RESIDUAL ? static_cast<const float *>(a.v0)[size_t(m) * a.ldd + n] : 0.f;
            const float o = apply_epi(a.epi, acc[i][j], a.bias ? a.bias[n] : 0.f, v, v0);
            *d = o;
            if (a.D2) static_cast<float *>(a.D2)[size_t(m) * a.ldd + n] = o;
        }
    }
}

// ---- transposed, zero-padded copies of the low-rank factors ------------------------------------------
template <class T>
__global__ void transpose_pad_kernel(const T *in, T *out, int rows, int cols, int out_rows, int out_cols) {
    // in [rows][cols] -> out [out_rows][out_cols], out[i][j] = in[j][i] inside, 0 in the padding
    const size_t n = size_t(out_rows) * out_cols;
    for (size_t e = blockIdx.x * size_t(blockDim.x) + threadIdx.x; e < n; e += size_t(gridDim.x) * blockDim.x) {
        const int i = int(e / out_cols), j = int(e % out_cols);
        out[e] = (i < cols && j < rows) ? in[size_t(j) * cols + i] : T(0.f);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

bool encode_bf16_2d(CUtensorMap *map, const void *base, int cols, int rows, int ld, int box_rows) {
    auto enc = tmap_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(ld) * 2};
    const cuuint32_t box[2] = {64, cuuint32_t(box_rows)}, es[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int BN>
cudaError_t launch_bf16(const GemmArgs &a, cudaStream_t stream) {
    CUtensorMap wmap, amap;
    std::memset(&amap, 0, sizeof(amap));
    if (!encode_bf16_2d(&wmap, a.W, a.K, a.N, a.K, BN)) return cudaErrorInvalidValue;
    if (a.pro == GEMM_PLAIN && !encode_bf16_2d(&amap, a.A, a.K, a.M, a.lda, 128)) return cudaErrorInvalidValue;
    if (a.pro == GEMM_MIX && !encode_bf16_2d(&amap, a.x, a.K, a.M, a.K, 128)) return cudaErrorInvalidValue;
    const int smem = int(GemmSmem<BN>::bytes);
    cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void *>(gemm_bf16_kernel<BN>), smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(unsigned((a.M + 127) / 128), unsigned(a.N / BN));
    gemm_bf16_kernel<BN><<<grid, kGemmThreads, smem, stream>>>(wmap, amap, a);
    return cudaGetLastError();
}

}  // namespace

// ---- host side ---------------------------------------------------------------------------------------

cudaError_t launch_gemm(const GemmArgs &a, wkv7_dtype dt, cudaStream_t stream) {
    if (a.M <= 0 || a.N <= 0 || a.K <= 0) return cudaSuccess;
    if (dt == WKV7_F32) {
        const dim3 grid(unsigned((a.M + kFT - 1) / kFT), unsigned((a.N + kFT - 1) / kFT));
        gemm_f32_kernel<<<grid, 256, 0, stream>>>(a);
        return cudaGetLastError();
    }
    if (a.K % 64 != 0 || a.N % 64 != 0) return cudaErrorInvalidValue;
    if (a.N % 128 == 0) return launch_bf16<128>(a, stream);
    return launch_bf16<64>(a, stream);
}

cudaError_t launch_transpose_pad(const void *in, void *out, int rows, int cols, int out_rows, int out_cols,
                                 wkv7_dtype dt, cudaStream_t stream) {
    const size_t n = size_t(out_rows) * out_cols;
    const unsigned grid = unsigned(std::min<size_t>((n + 255) / 256, 148 * 8));
    if (dt == WKV7_BF16)
        transpose_pad_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16 *>(in),
                                                                     static_cast<__nv_bfloat16 *>(out), rows, cols,
                                                                     out_rows, out_cols);
    else
        transpose_pad_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float *>(in), static_cast<float *>(out),
                                                             rows, cols, out_rows, out_cols);
    return cudaGetLastError();
}

}  // namespace wkv7
