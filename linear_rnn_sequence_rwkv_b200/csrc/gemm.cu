// The projections of the time-mixing layer: D_i[M][N_i] = op(A)[M][K_i] * W_i[N_i][K_i]^T for up to
// seven products per launch, with the operand's preparation fused into its load and the
// element-wise step after each product fused into its store (RWKV-7 rebuttal page, numpy
// time_mixing listing: the token-shift mixes feed the square projections and the low-rank first
// factors; tanh, sigmoid, the biases and the value residual follow them).
//
// Operand preparation:
//   PLAIN  A_i itself;
//   MIX    x + m_i (x_prev - x), x_prev the previous token of the same sequence (last_x, or 0,
//          for the first token), in fp32 and rounded once to the layer dtype.
// Store (per element of the fp32 accumulator z, column n of problem i):
//   STORE z;  TANH tanh(z);  SIGMOID sigmoid(z);  BIAS z + bias[n];
//   RESIDUAL v + (v0 - v) sigmoid(z + bias[n]) with v the value already in D;  F32 z in fp32.
//
// bf16: a persistent kernel, one CTA per SM, walking 128-row output tiles (all the launch's
// problems for one row block, then the next block, so that a block of x is read from HBM once).
// Warp 12 streams W (and A or x) by TMA into a ring of shared-memory stages (128-byte swizzle);
// warps 0-7 prepare the MIX operand into the stage; warp 13 issues tcgen05.mma (bf16
// operands, fp32 accumulation) into one of two tensor-memory accumulators of up to 256 columns;
// warps 8-11 read the other accumulator back (one TMEM lane quarter each) and store it, so that
// a tile's store overlaps the next tile's products. fp32: a shared-memory tiled FMA GEMM with the
// same preparation and store steps (exact fp32 products, fp32 accumulation), one launch per
// problem.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>

#include "gemm.cuh"
#include "tc_util.cuh"

namespace wkv7 {
namespace {

using namespace tc;

// 1 / (1 + e^-z) with the hardware reciprocal: no slow path for large or non-finite arguments
// (e^-z = inf gives 0, the limit).
__device__ __forceinline__ float sigmoidf_(float z) { return __fdividef(1.f, 1.f + __expf(-z)); }

__device__ __forceinline__ float bf(uint32_t packed, int hi) {
    return __uint_as_float(hi ? (packed & 0xffff0000u) : (packed << 16));
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Shared-memory accesses with an explicit state space (the staging tiles are addressed as
// 32-bit shared addresses).
__device__ __forceinline__ void st_shared_f4(uint32_t a, float4 v) {
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w) : "memory");
}
__device__ __forceinline__ float4 ld_shared_f4(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a) : "memory");
    return v;
}
// ---- bf16 on tcgen05 -------------------------------------------------------------------------------
constexpr int kProdWarps = 8;                 // warps 0-7: MIX operand preparation
constexpr int kEpiWarp0 = 8;                  // warps 8-11: accumulator read-back and store
constexpr int kTmaWarp = 12, kMmaWarp = 13;
constexpr int kGemmThreads = 14 * 32;
constexpr int kAccCols = 256;                 // one accumulator: 128 lanes x up to 256 fp32 columns
constexpr uint32_t kTileA = 128 * 128;        // 128 rows x 64 bf16
constexpr uint32_t kTileB = 256 * 128;        // up to 256 rows x 64 bf16
constexpr uint64_t kWaitNs = 2000000000ull;

// One stage: the W tile, the A tile as loaded (x for the mix), and for MIX the prepared operand
// (OP: where the products read A).
// After the ring: per store warp two 4 KB output staging tiles; for PLAIN three pairs of 2 KB
// tiles for the value residual's v and v0, for MIX per stage the mix values of its 64 columns
// (256 bytes) and the x row before the tile (128 bytes), loaded with the stage.
template <int PRO>
struct Ring {
    static constexpr uint32_t B = 0, A = kTileB, P = kTileB + kTileA, OP = PRO == GEMM_MIX ? P : A;
    static constexpr uint32_t stage = kTileB + kTileA + (PRO == GEMM_MIX ? kTileA : 0u);
    static constexpr int stages = 3;
    static constexpr uint32_t out_off = stages * stage;             // [warp][2] x 4096
    static constexpr uint32_t res_off = out_off + 4 * 2 * 4096;     // PLAIN: [warp][3] x (v 2048, v0 2048)
    static constexpr uint32_t mix_off = res_off;                     // MIX: [stage] x 384
    static constexpr uint32_t bar_off = res_off + (PRO == GEMM_PLAIN ? 4 * 3 * 4096u : stages * 384u);
    static constexpr uint32_t bytes = bar_off + 256 + 1024;   // + barriers, + 1 KB alignment slack
};

struct GemmProb {
    int N, K, bn, tile0;   // bn: columns per tile (64, 128 or 256); tile0: first column tile of the problem
    int epi, ldd, Kx;      // Kx: row length of x (MIX)
    const float *mix, *bias;
    const void *v0;
    void *D;
};
struct GemmDev {
    int M, T, nprob, ntn, ntiles;   // ntn: column tiles per row block over all problems
    const void *x, *last_x;
    unsigned int *err;
    GemmProb p[kGemmMaxProblems];
};
struct GemmParams {
    CUtensorMap wmap[kGemmMaxProblems];
    CUtensorMap amap[kGemmMaxProblems];   // PLAIN: problem i's A; MIX: amap[0] is x
    CUtensorMap dmap[kGemmMaxProblems];   // D in boxes of 32 x 32 (the stores; RESIDUAL also loads v)
    CUtensorMap v0map;                    // RESIDUAL: v0, same boxes
    GemmDev d;
};

static_assert(sizeof(GemmParams) <= 4096, "kernel parameters");
static_assert(Ring<GEMM_MIX>::bytes <= 232448 && Ring<GEMM_PLAIN>::bytes <= 232448, "shared memory per CTA");

struct Tile {
    int m0, pi, n0;
};
__device__ __forceinline__ Tile tile_of(const GemmDev &d, int t) {
    const int mt = t / d.ntn, nt = t - mt * d.ntn;
    int i = 0;
    while (i + 1 < d.nprob && nt >= d.p[i + 1].tile0) ++i;
    return Tile{mt * 128, i, (nt - d.p[i].tile0) * d.p[i].bn};
}

// Wait for a phase: at most kWaitNs, and not past an abort raised by another role.
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_test_wait(bar, parity)) return true;
        if ((i & 255u) == 0 && (*abort || globaltimer_ns() - t0 > kWaitNs)) {
            *abort = 1;
            return false;
        }
    }
}
// The same with a pause between polls, for waits that are long and not on the critical path:
// a tight poll takes issue slots from the warps that share the scheduler.
__device__ __forceinline__ bool wait_phase_idle(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (mbar_test_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 1;; ++i) {
        __nanosleep(100);
        if (mbar_test_wait(bar, parity)) return true;
        if ((i & 15u) == 0 && (*abort || globaltimer_ns() - t0 > kWaitNs)) {
            *abort = 1;
            return false;
        }
    }
}
// Lane 0 waits, the warp learns the outcome.
__device__ __forceinline__ bool warp_wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort, int lane,
                                                bool idle = false) {
    int ok = 0;
    if (lane == 0) ok = idle ? wait_phase_idle(bar, parity, abort) : wait_phase(bar, parity, abort);
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// The store warps. Each owns 32 accumulator rows (its TMEM lane quarter, token rows m0 .. m0 + 31)
// and moves them out 32 columns at a time: tcgen05.ld puts row `lane` in the lane's registers,
// the element-wise step runs there, the lane writes its row into a staging tile in the layout
// of the output's tensor map (bf16: 64-byte rows, 16-byte chunk c at c ^ ((row >> 1) & 3), the
// 64-byte swizzle; fp32: 128-byte rows, chunk c at c ^ (row & 7), the 128-byte swizzle), and one
// lane hands the tile to a TMA store. The value residual's v (the current D) and v0 arrive the
// same way, by TMA loads into the same 64-byte-swizzled layout, one chunk ahead.
// out: the warp's two 4 KB staging tiles; res: its three (v, v0) pairs of 2 KB tiles (PLAIN), with
// one barrier each in vbar, used in turn by the value residual's blocks (two blocks are in
// flight while a third is read); rc: the residual blocks this warp has taken so far (block a
// uses pair a % 3, whose barrier is then in its (a / 3)-th phase). Everything is passed by
// value (a context struct passed by reference would live in local memory and cost a round trip
// to the cache for every field read). Returns the updated rc.
template <int EPI>
__device__ __noinline__ uint32_t store_tile(const GemmProb p, const CUtensorMap *dmap, const CUtensorMap *v0map,
                                            uint32_t tacc, int m0, int n0, uint8_t *const out, uint8_t *const res,
                                            uint64_t *const vbar, uint32_t rc, volatile int *abort, int lane) {
    const int nch = p.bn / 32;
    const float *const bias_p = p.bias;
    auto fetch_res = [&](int j) {   // v and v0 of chunk j (block rc + j) into pair (rc + j) % 3
        if (lane == 0) {
            const uint32_t sl = (rc + uint32_t(j)) % 3u;
            uint8_t *r = res + sl * 4096;
            mbar_arrive_expect_tx(&vbar[sl], 4096);
            tma_load_2d(r, dmap, &vbar[sl], n0 + 32 * j, m0);
            tma_load_2d(r + 2048, v0map, &vbar[sl], n0 + 32 * j, m0);
        }
    };
    if constexpr (EPI == GEMM_RESIDUAL) {
        fetch_res(0);
        if (nch > 1) fetch_res(1);
    }
#pragma unroll 1
    for (int j = 0; j < nch; ++j) {
        if constexpr (EPI == GEMM_RESIDUAL)
            if (j + 2 < nch) fetch_res(j + 2);   // its pair was last read in chunk j - 1
        float z[32];
        tmem_ld32(tacc + uint32_t(32 * j), z);
        const int n = n0 + 32 * j;
        if constexpr (EPI == GEMM_BIAS || EPI == GEMM_RESIDUAL) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
                const float4 b = __ldg(reinterpret_cast<const float4 *>(bias_p + n + e));
                z[e] += b.x; z[e + 1] += b.y; z[e + 2] += b.z; z[e + 3] += b.w;
            }
        }
        if constexpr (EPI == GEMM_TANH) {
#pragma unroll
            for (int e = 0; e < 32; ++e) z[e] = tanhf(z[e]);
        } else if constexpr (EPI == GEMM_SIGMOID) {
#pragma unroll
            for (int e = 0; e < 32; ++e) z[e] = sigmoidf_(z[e]);
        } else if constexpr (EPI == GEMM_RESIDUAL) {
            const uint32_t a = rc + uint32_t(j), b = a % 3u;
            int ok = 1;
            if (lane == 0) ok = wait_phase(&vbar[b], (a / 3u) & 1u, abort);   // polled: wakes on time
            ok = __shfl_sync(0xffffffffu, ok, 0);
            const uint32_t rv = smem_u32(res + b * 4096) + uint32_t(lane * 64);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint32_t off = uint32_t((c ^ ((lane >> 1) & 3)) << 4);
                const float4 va = ld_shared_f4(rv + off), v0a = ld_shared_f4(rv + 2048 + off);
                const uint32_t vw[4] = {__float_as_uint(va.x), __float_as_uint(va.y), __float_as_uint(va.z),
                                        __float_as_uint(va.w)};
                const uint32_t v0w[4] = {__float_as_uint(v0a.x), __float_as_uint(v0a.y), __float_as_uint(v0a.z),
                                         __float_as_uint(v0a.w)};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float v = bf(vw[e >> 1], e & 1);
                    z[8 * c + e] = ok ? fmaf(bf(v0w[e >> 1], e & 1) - v, sigmoidf_(z[8 * c + e]), v) : 0.f;
                }
            }
        }
        // staging tile j & 1: its store from chunk j - 2 has finished reading it
        uint8_t *o = out + (j & 1) * 4096;
        if (lane == 0) tma_store_wait_read1();
        __syncwarp();
        if constexpr (EPI == GEMM_F32) {
            const uint32_t ro = smem_u32(o) + uint32_t(lane * 128);
#pragma unroll
            for (int c = 0; c < 8; ++c)
                st_shared_f4(ro + uint32_t((c ^ (lane & 7)) << 4), make_float4(z[4 * c], z[4 * c + 1], z[4 * c + 2], z[4 * c + 3]));
        } else {
            const uint32_t ro = smem_u32(o) + uint32_t(lane * 64);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float4 w = make_float4(__uint_as_float(pack_bf16(z[8 * c], z[8 * c + 1])),
                                             __uint_as_float(pack_bf16(z[8 * c + 2], z[8 * c + 3])),
                                             __uint_as_float(pack_bf16(z[8 * c + 4], z[8 * c + 5])),
                                             __uint_as_float(pack_bf16(z[8 * c + 6], z[8 * c + 7])));
                st_shared_f4(ro + uint32_t((c ^ ((lane >> 1) & 3)) << 4), w);
            }
        }
        fence_proxy_async_smem();   // the staging writes -> visible to the TMA unit
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(dmap, o, n, m0);   // rows past M are clipped by the tensor map
            tma_store_commit();
        }
    }
    return EPI == GEMM_RESIDUAL ? rc + uint32_t(nch) : rc;
}

// MIX: the thread's four chunks (rows rb + 32 i, 16-byte chunk q) of the prepared operand,
// x + m (x_prev - x) in fp32, rounded once to bf16. The row before comes from the loaded x tile,
// for tile row 0 from the stage's copy of the row before the tile, and for the first token of a
// sequence from last_x (or zeros), read from global memory (rare unless sequences are short).
// The operand sources, copied out of the kernel parameters into registers once (reads through a
// reference to the parameters would be repeated after every shared-memory store).
struct Src {
    const __nv_bfloat16 *last_x;
    int M, T, K;
};
__device__ __forceinline__ void mix_stage(const Src &d, const uint8_t *xt, const uint8_t *extra, uint8_t *pt, int m0,
                                          int k, int rb, int q, uint32_t first_mask) {
    // extra: the stage's 64 mix values (256 bytes), then the row before the tile (128 bytes)
    const float4 mA = *reinterpret_cast<const float4 *>(extra + q * 32), mB = *reinterpret_cast<const float4 *>(extra + q * 32 + 16);
    const float mv[8] = {mA.x, mA.y, mA.z, mA.w, mB.x, mB.y, mB.z, mB.w};
    uint4 xc[4], xp[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = rb + 32 * i;
        xc[i] = *reinterpret_cast<const uint4 *>(xt + uint32_t(r) * 128u + (uint32_t(q ^ (r & 7)) << 4));
        xp[i] = r > 0 ? *reinterpret_cast<const uint4 *>(xt + uint32_t(r - 1) * 128u + (uint32_t(q ^ ((r - 1) & 7)) << 4))
                      : *reinterpret_cast<const uint4 *>(extra + 256 + q * 16);
    }
    if (first_mask) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (first_mask >> i & 1u) {
                const int m = m0 + rb + 32 * i;
                xp[i] = d.last_x ? __ldg(reinterpret_cast<const uint4 *>(d.last_x + size_t(m / d.T) * d.K + k))
                                 : make_uint4(0u, 0u, 0u, 0u);
            }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = rb + 32 * i;
        const uint32_t cw[4] = {xc[i].x, xc[i].y, xc[i].z, xc[i].w}, pw[4] = {xp[i].x, xp[i].y, xp[i].z, xp[i].w};
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float xi = bf(cw[e >> 1], e & 1), pi = bf(pw[e >> 1], e & 1);
            o[e] = fmaf(mv[e], pi - xi, xi);
        }
        *reinterpret_cast<uint4 *>(pt + uint32_t(r) * 128u + (uint32_t(q ^ (r & 7)) << 4)) =
            make_uint4(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]), pack_bf16(o[6], o[7]));
    }
}

template <int PRO>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_bf16_kernel(const __grid_constant__ GemmParams P) {
    using R = Ring<PRO>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + R::bar_off);
    uint64_t *full_t = bars, *full_a = bars + 4, *empty = bars + 8, *acc_full = bars + 12, *acc_empty = bars + 14;
    uint64_t *drain = bars + 16, *vbars = bars + 17;   // vbars: [store warp][3]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 29);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 30);
    auto stage = [&](int s) { return sm + s * R::stage; };

    const GemmDev &d = P.d;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < R::stages; ++s) {
            mbar_init(&full_t[s], 1);
            mbar_init(&full_a[s], kProdWarps);   // one arrival per preparing warp
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);         // one arrival per store warp
        }
        mbar_init(drain, 1);
        for (int i = 0; i < 12; ++i) mbar_init(&vbars[i], 1);
        *abort = 0;
        mbar_fence_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, 2 * kAccCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *tmem_slot;

    if (warp == kTmaWarp) {
        if (lane == 0) {
            for (int i = 0; i < d.nprob; ++i) {
                prefetch_tensormap(&P.wmap[i]);
                if (PRO == GEMM_PLAIN || (PRO == GEMM_MIX && i == 0)) prefetch_tensormap(&P.amap[i]);
            }
            int it = 0;
            for (int t = blockIdx.x; t < d.ntiles && !*abort; t += gridDim.x) {
                const Tile tl = tile_of(d, t);
                const GemmProb &p = d.p[tl.pi];
                // MIX: the mix values, and the row before the tile unless the tile starts at row 0
                const uint32_t bytes = uint32_t(p.bn) * 128u + kTileA + (PRO == GEMM_MIX ? (tl.m0 > 0 ? 384u : 256u) : 0u);
                const CUtensorMap *am = &P.amap[PRO == GEMM_PLAIN ? tl.pi : 0];
                for (int kb = 0; kb < p.K / 64; ++kb, ++it) {
                    const int s = it % R::stages;
                    if (!wait_phase(&empty[s], ((it / R::stages) & 1) ^ 1, abort)) break;
                    mbar_arrive_expect_tx(&full_t[s], bytes);
                    tma_load_2d(stage(s) + R::B, &P.wmap[tl.pi], &full_t[s], kb * 64, tl.n0);
                    tma_load_2d(stage(s) + R::A, am, &full_t[s], kb * 64, tl.m0);
                    if (PRO == GEMM_MIX) {
                        uint8_t *ex = sm + R::mix_off + s * 384;
                        bulk_load_1d(ex, p.mix + kb * 64, 256u, &full_t[s]);
                        if (tl.m0 > 0)
                            bulk_load_1d(ex + 256, static_cast<const __nv_bfloat16 *>(d.x) + size_t(tl.m0 - 1) * p.Kx + kb * 64,
                                         128u, &full_t[s]);
                    }
                }
            }
            // the loads still in flight land before the CTA leaves
            for (int j = std::max(0, it - R::stages); j < it; ++j)
                mbar_wait_spin(&full_t[j % R::stages], (j / R::stages) & 1, kWaitNs);
        }
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            int it = 0, lt = 0;
            for (int t = blockIdx.x; t < d.ntiles && !*abort; t += gridDim.x, ++lt) {
                const Tile tl = tile_of(d, t);
                const GemmProb &p = d.p[tl.pi];
                const int b = lt & 1;
                if (!wait_phase(&acc_empty[b], ((lt >> 1) & 1) ^ 1, abort)) break;
                tc_fence_after();
                const uint32_t tacc = tb + uint32_t(b * kAccCols), idesc = idesc_bf16(128, p.bn);
                bool ok = true;
                for (int kb = 0; kb < p.K / 64; ++kb, ++it) {
                    const int s = it % R::stages;
                    const uint32_t ph = (it / R::stages) & 1;
                    if (!wait_phase(&full_t[s], ph, abort) || (PRO != GEMM_PLAIN && !wait_phase(&full_a[s], ph, abort))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint8_t *a_op = stage(s) + R::OP;
                    const uint64_t dA = desc_sw128(smem_u32(a_op)), dB = desc_sw128(smem_u32(stage(s) + R::B));
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16_ss(tacc, dA + uint64_t(2 * ks), dB + uint64_t(2 * ks), idesc, (kb | ks) != 0);
                    mma_commit(&empty[s]);
                }
                if (!ok) break;
                mma_commit(&acc_full[b]);
            }
            // every product issued has completed before the accumulators are freed
            mma_commit(drain);
            mbar_wait_spin(drain, 0, kWaitNs);   // polled: a suspended wait can wake late
        }
    } else if (warp >= kEpiWarp0) {
        const int quarter = warp & 3, ew = warp - kEpiWarp0;
        uint8_t *const out = sm + R::out_off + ew * 8192, *const res = sm + R::res_off + ew * 12288;
        uint64_t *const vbar = vbars + 3 * ew;
        uint32_t rc = 0;
        if (lane == 0) {
            for (int i = 0; i < d.nprob; ++i) prefetch_tensormap(&P.dmap[i]);
        }
        int lt = 0;
        for (int t = blockIdx.x; t < d.ntiles; t += gridDim.x, ++lt) {
            const Tile tl = tile_of(d, t);
            const GemmProb p = d.p[tl.pi];
            const int b = lt & 1;
            if (!warp_wait_phase(&acc_full[b], (lt >> 1) & 1, abort, lane, true)) break;
            tc_fence_after();
            const uint32_t tacc = tmem_addr(tb, 32 * quarter, b * kAccCols);
            const int m0 = tl.m0 + 32 * quarter;
            const CUtensorMap *dm = &P.dmap[tl.pi];
            switch (p.epi) {
                case GEMM_TANH: rc = store_tile<GEMM_TANH>(p, dm, &P.v0map, tacc, m0, tl.n0, out, res, vbar, rc, abort, lane); break;
                case GEMM_SIGMOID: rc = store_tile<GEMM_SIGMOID>(p, dm, &P.v0map, tacc, m0, tl.n0, out, res, vbar, rc, abort, lane); break;
                case GEMM_BIAS: rc = store_tile<GEMM_BIAS>(p, dm, &P.v0map, tacc, m0, tl.n0, out, res, vbar, rc, abort, lane); break;
                case GEMM_RESIDUAL:
                    if (PRO == GEMM_PLAIN) rc = store_tile<GEMM_RESIDUAL>(p, dm, &P.v0map, tacc, m0, tl.n0, out, res, vbar, rc, abort, lane);
                    break;
                case GEMM_F32: rc = store_tile<GEMM_F32>(p, dm, &P.v0map, tacc, m0, tl.n0, out, res, vbar, rc, abort, lane); break;
                default: rc = store_tile<GEMM_STORE>(p, dm, &P.v0map, tacc, m0, tl.n0, out, res, vbar, rc, abort, lane); break;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
        }
        if (lane == 0) tma_store_wait_all();   // the stores have landed before the CTA leaves
    } else if (PRO == GEMM_MIX) {
        // operand preparation: the thread owns chunk q of rows rb, rb + 32, rb + 64, rb + 96
        const int q = tid & 7, rb = tid >> 3;
        const Src src{static_cast<const __nv_bfloat16 *>(d.last_x), d.M, d.T, 0};
        int it = 0;
        for (int t = blockIdx.x; t < d.ntiles; t += gridDim.x) {
            const Tile tl = tile_of(d, t);
            Src sd = src;
            sd.K = d.p[tl.pi].Kx;
            const int nkb = d.p[tl.pi].K / 64;
            uint32_t first_mask = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int m = tl.m0 + rb + 32 * i;
                if (m < sd.M && m % sd.T == 0) first_mask |= 1u << i;
            }
            bool ok = true;
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const int s = it % R::stages;
                if (!warp_wait_phase(&full_t[s], (it / R::stages) & 1, abort, lane)) {
                    ok = false;
                    break;
                }
                mix_stage(sd, stage(s) + R::A, sm + R::mix_off + s * 384, stage(s) + R::OP, tl.m0, kb * 64 + q * 8, rb, q,
                          first_mask);
                fence_proxy_async_smem();   // generic-proxy writes -> visible to the tensor core
                __syncwarp();
                if (lane == 0) mbar_arrive(&full_a[s]);
            }
            if (!ok) break;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort && d.err) atomicOr(d.err, 1u);
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tb, 2 * kAccCols);
    }
}

// ---- fp32 on the FMA pipe ---------------------------------------------------------------------------
constexpr int kFT = 64, kFK = 16;   // 64 x 64 output tile, K in steps of 16; 256 threads, 4 x 4 each

struct F32Args {
    int M, T, pro;
    const float *x, *last_x;
    GemmProblem p;
};

__device__ __forceinline__ float prep_a1(const F32Args &a, int m, int k) {
    const int K = a.p.K;
    if (m >= a.M || k >= K) return 0.f;
    if (a.pro == GEMM_PLAIN) return static_cast<const float *>(a.p.A)[size_t(m) * a.p.lda + k];
    const float xi = a.x[size_t(m) * K + k];
    float xp = 0.f;
    if (m % a.T != 0) xp = a.x[size_t(m - 1) * K + k];
    else if (a.last_x) xp = a.last_x[size_t(m / a.T) * K + k];
    return fmaf(a.p.mix[k], xp - xi, xi);
}

__global__ void __launch_bounds__(256) gemm_f32_kernel(const F32Args a) {
    __shared__ float As[kFK][kFT + 4], Bs[kFK][kFT + 4];
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int m0 = blockIdx.x * kFT, n0 = blockIdx.y * kFT;
    const GemmProblem &p = a.p;
    const float *W = static_cast<const float *>(p.W);
    float acc[4][4] = {};
    for (int k0 = 0; k0 < p.K; k0 += kFK) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + 256 * i, r = e >> 4, k = e & 15;
            As[k][r] = prep_a1(a, m0 + r, k0 + k);
            const int n = n0 + r;
            Bs[k][r] = (n < p.N && k0 + k < p.K) ? W[size_t(n) * p.K + k0 + k] : 0.f;
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
            if (n >= p.N) continue;
            float *dp = static_cast<float *>(p.D) + size_t(m) * p.ldd + n;
            const float z = acc[i][j], bias = p.bias ? p.bias[n] : 0.f;
            float o = z;
            switch (p.epi) {
                case GEMM_TANH: o = tanhf(z); break;
                case GEMM_SIGMOID: o = sigmoidf_(z); break;
                case GEMM_BIAS: o = z + bias; break;
                case GEMM_RESIDUAL: {
                    const float v = *dp, v0 = static_cast<const float *>(p.v0)[size_t(m) * p.ldd + n];
                    o = fmaf(v0 - v, sigmoidf_(z + bias), v);
                    break;
                }
                default: break;
            }
            *dp = o;
        }
    }
}

// ---- transposed, zero-padded copies of the low-rank factors ------------------------------------------
struct PadCopies {
    PadCopy c[kMaxPadCopies];
};

template <class T>
__global__ void transpose_pad_kernel(const PadCopies cs) {
    // blockIdx.y selects the copy: out[i][j] = in[j][i] inside, 0 in the padding
    const PadCopy &c = cs.c[blockIdx.y];
    const T *in = static_cast<const T *>(c.in);
    T *out = static_cast<T *>(c.out);
    const size_t n = size_t(c.out_rows) * c.out_cols;
    for (size_t e = blockIdx.x * size_t(blockDim.x) + threadIdx.x; e < n; e += size_t(gridDim.x) * blockDim.x) {
        const int i = int(e / c.out_cols), j = int(e % c.out_cols);
        out[e] = (i < c.cols && j < c.rows) ? in[size_t(j) * c.cols + i] : T(0.f);
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

// A [rows][cols] matrix (bf16, or fp32 when f32) with row stride ld elements, moved in boxes of
// box_cols x box_rows.
bool encode_2d(CUtensorMap *map, bool f32, const void *base, int cols, int rows, int ld, int box_cols, int box_rows,
               CUtensorMapSwizzle swz) {
    auto enc = tmap_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    const cuuint64_t strides[1] = {cuuint64_t(ld) * (f32 ? 4 : 2)};
    const cuuint32_t box[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)}, es[2] = {1, 1};
    return enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base),
               dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// Operand tiles: 64 bf16 columns (128 bytes, the 128-byte swizzle) x box_rows rows.
bool encode_operand(CUtensorMap *map, const void *base, int cols, int rows, int ld, int box_rows) {
    return encode_2d(map, false, base, cols, rows, ld, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}
// Store-side tiles: 32 x 32, bf16 rows of 64 bytes (64-byte swizzle) or fp32 rows of 128 bytes
// (128-byte swizzle), the layouts the store warps write.
bool encode_out(CUtensorMap *map, bool f32, const void *base, int cols, int rows, int ld) {
    return encode_2d(map, f32, base, cols, rows, ld, 32, 32, f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
}

int tile_cols(int N) { return N % 256 == 0 ? 256 : N % 128 == 0 ? 128 : 64; }

template <int PRO>
cudaError_t launch_bf16(const GemmGroup &g, cudaStream_t stream) {
    GemmParams P;
    std::memset(&P, 0, sizeof(P));
    GemmDev &d = P.d;
    d.M = g.M; d.T = g.T; d.nprob = g.nprob;
    d.x = g.x; d.last_x = g.last_x; d.err = g.err;
    int ntn = 0;
    const void *v0 = nullptr;
    for (int i = 0; i < g.nprob; ++i) {
        const GemmProblem &q = g.p[i];
        if (q.K <= 0 || q.N <= 0 || q.K % 64 != 0 || q.N % 64 != 0) return cudaErrorInvalidValue;
        GemmProb &p = d.p[i];
        p.N = q.N; p.K = q.K; p.bn = tile_cols(q.N); p.tile0 = ntn;
        p.epi = q.epi; p.ldd = q.ldd; p.Kx = q.K;
        p.mix = q.mix; p.bias = q.bias; p.v0 = q.v0; p.D = q.D;
        ntn += q.N / p.bn;
        if (!encode_operand(&P.wmap[i], q.W, q.K, q.N, q.K, p.bn)) return cudaErrorInvalidValue;
        if (PRO == GEMM_PLAIN && !encode_operand(&P.amap[i], q.A, q.K, g.M, q.lda, 128)) return cudaErrorInvalidValue;
        if (!encode_out(&P.dmap[i], q.epi == GEMM_F32, q.D, q.N, g.M, q.ldd)) return cudaErrorInvalidValue;
        if (q.epi == GEMM_RESIDUAL) {
            // the value residual: PLAIN launches only (the others have no room for its tiles), one v0
            if (PRO != GEMM_PLAIN || !q.v0 || (v0 && v0 != q.v0)) return cudaErrorInvalidValue;
            v0 = q.v0;
            if (!encode_out(&P.v0map, false, q.v0, q.N, g.M, q.ldd)) return cudaErrorInvalidValue;
        }
    }
    if (PRO == GEMM_MIX) {
        for (int i = 1; i < g.nprob; ++i)
            if (g.p[i].K != g.p[0].K) return cudaErrorInvalidValue;   // every mix reads the same x
        for (int i = 0; i < g.nprob; ++i)   // the mix values are copied in 256-byte pieces
            if (!g.p[i].mix || reinterpret_cast<uintptr_t>(g.p[i].mix) % 16 != 0) return cudaErrorInvalidValue;
        if (!encode_operand(&P.amap[0], g.x, g.p[0].K, g.M, g.p[0].K, 128)) return cudaErrorInvalidValue;
    }
    d.ntn = ntn;
    const long long ntiles = (long long)((g.M + 127) / 128) * ntn;
    if (ntiles > INT32_MAX) return cudaErrorInvalidValue;
    d.ntiles = int(ntiles);
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int smem = int(Ring<PRO>::bytes);
    if ((e = allow_dynamic_smem(reinterpret_cast<const void *>(gemm_bf16_kernel<PRO>), smem)) != cudaSuccess) return e;
    const unsigned grid = unsigned(std::min<long long>(ntiles, sms));
    gemm_bf16_kernel<PRO><<<grid, kGemmThreads, smem, stream>>>(P);
    return cudaGetLastError();
}

}  // namespace

// ---- host side ---------------------------------------------------------------------------------------

cudaError_t launch_gemm_group(const GemmGroup &g, wkv7_dtype dt, cudaStream_t stream) {
    if (g.nprob < 1 || g.nprob > kGemmMaxProblems) return cudaErrorInvalidValue;
    if (g.M <= 0) return cudaSuccess;
    if (g.pro == GEMM_MIX && g.T <= 0) return cudaErrorInvalidValue;
    if (dt == WKV7_F32) {
        for (int i = 0; i < g.nprob; ++i) {
            F32Args a{};
            a.M = g.M; a.T = g.T; a.pro = g.pro;
            a.x = static_cast<const float *>(g.x); a.last_x = static_cast<const float *>(g.last_x);
            a.p = g.p[i];
            if (a.p.N <= 0 || a.p.K <= 0) return cudaErrorInvalidValue;
            const dim3 grid(unsigned((g.M + kFT - 1) / kFT), unsigned((a.p.N + kFT - 1) / kFT));
            gemm_f32_kernel<<<grid, 256, 0, stream>>>(a);
            const cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
        return cudaSuccess;
    }
    switch (g.pro) {
        case GEMM_PLAIN: return launch_bf16<GEMM_PLAIN>(g, stream);
        case GEMM_MIX: return launch_bf16<GEMM_MIX>(g, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_transpose_pad(const PadCopy *copies, int n, wkv7_dtype dt, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    if (n > kMaxPadCopies) return cudaErrorInvalidValue;
    PadCopies cs{};
    size_t most = 0;
    for (int i = 0; i < n; ++i) {
        cs.c[i] = copies[i];
        most = std::max(most, size_t(copies[i].out_rows) * copies[i].out_cols);
    }
    const dim3 grid(unsigned(std::min<size_t>((most + 255) / 256, 148 * 4)), unsigned(n));
    if (dt == WKV7_BF16) transpose_pad_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(cs);
    else transpose_pad_kernel<float><<<grid, 256, 0, stream>>>(cs);
    return cudaGetLastError();
}

}  // namespace wkv7
