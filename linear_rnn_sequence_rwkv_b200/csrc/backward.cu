// WKV-7 backward pass: fp32 reverse sweep with state recomputation.
//
// The pages time a backward pass and quote the precision of an fp32 one (RWKV-7 rebuttal
// page, the answer on numerical precision; paper summary, the speed figures for the
// forward that keeps its states and for the backward) without printing it. This is the
// chain rule through the update and the readout (rebuttal page, numpy time_mixing
// listing), one token at a time in reverse. With b = kk * a, s = S_{t-1} kk and dS the
// gradient reaching S_t:
//     dS += dy_t r_t^T;           dr_t = S_t^T dy_t
//     dv_t = dS k_t;              dk_t = dS^T v_t
//     dw_t[j] = sum_i S_{t-1}[i, j] dS[i, j]
//     db = -dS^T s;  ds = -dS b;  dkk_t = S_{t-1}^T ds + db * a_t;  da_t = db * kk_t
//     dS_{t-1} = dS diag(w_t) + ds kk_t^T.
//
// One CTA of 256 threads per (b, h). The sweep needs S_{t-1} at every t in reverse order. The sequence is cut into segments (between the
// forward's snapshots, or the whole sequence); a segment's forward is run once to write one
// state per block of kLb tokens to the workspace, then the blocks are taken in reverse: each
// block's states are recomputed from its checkpoint into shared memory, the reverse
// recurrence runs over the block, and the per-token gradient vectors are summed over the 64
// rows from shared memory. Two thread layouts:
//   row owner   (recurrence): thread (g = tid / 8, q = tid % 8) holds columns
//                4q + 32m + c (m < 2, c < 4) of rows g and g + 32 of S and of dS in
//                registers; the dot products per row and token reduce over the eight lanes
//                of a row group. Two rows per thread halve the shared-memory wavefronts of
//                the token vectors, which every row group reads.
//   column pass (gradient vectors): thread (token tt, column quad cq, row quarter rq) sums
//                the 16 rows 4r + rq of five products; the quarters combine by two shuffles.
// A split of a head's rows over a cluster of two CTAs (the rows are independent; only the
// gradient vectors need both halves, exchanged through distributed shared memory) measured
// slower on the 96-head prefill: the busiest SMs still carry a whole head's work.
// Shared rows are 80 floats apart (320 B = 64 mod 128), so the column pass's float4 loads
// are free of bank conflicts (the row owners' stores are: eight lanes write one row's 128 B).
#include <mutex>

#include "common.cuh"

namespace wkv7 {
namespace {

// Scratch of the allocation-free backward entry: the recomputation checkpoints live in this
// module-scope array instead of a caller's workspace. Every checkpoint is written before it is
// read, so nothing in it needs to start at zero.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;   // 2048 states of 64 x 64 fp32
static __device__ __align__(256) float g_bwd_scratch[kStaticScratchBytes / sizeof(float)];

constexpr int kBwdThreads = 256;
constexpr int kRows = 64;
constexpr int kLb = 4;          // tokens per block
constexpr int kRS = 80;         // shared row stride (floats)

// Tokens between recomputation anchors: the snapshot interval, or the whole sequence.
__host__ __device__ inline int segment_length(int T, int snap_every) {
    return (snap_every > 0 && snap_every < T) ? snap_every : (T > 0 ? T : 1);
}

enum { VW = 0, VKK, VB, VK, VR, VV, VDY, VA, kVecs };
enum { GU = 0, GZ, GK, GB, GW, kGrads };   // partial sums: S_t^T dy, S_{t-1}^T ds, dS^T v, db, dw

struct BwdSmem {
    float S[kLb + 1][kRows][kRS];    // S_{t0} .. S_{t0 + L}, this CTA's rows
    float D[kLb][kRows][kRS];        // the gradient reaching S_t, t in the block
    float vec[kVecs][kLb][kN];       // w, kk, b = kk*a, k, r, v, dy, a (fp32, all 64 channels)
    float sa[kLb][kRows];            // s_i = S_{t-1}[i, :] . kk_t
    float ds[kLb][kRows];            // ds_i = -dS_t[i, :] . b_t
};

template <class Tin>
__device__ __forceinline__ float ld_in(const void *p, size_t i) {
    return load1(static_cast<const Tin *>(p) + i);
}

template <class Tin>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_kernel(const BwdArgs p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    BwdSmem &sm = *reinterpret_cast<BwdSmem *>(smem_raw);
    const int T = p.T, H = p.H;
    const int unit = blockIdx.x, b = unit / H, h = unit % H;
    const int tid = threadIdx.x;
    // row owner: rows rg and rg + 32, columns 4q + 32m + c (m < 2, c < 4)
    const int rg = tid >> 3, q = tid & 7;
    constexpr int row0 = 0;
    auto tok = [&](int t) { return ((size_t(b) * T + t) * H + h) * kN; };

    float s[2][8], d[2][8];
    auto load_rows = [&](const float *base, float (&x)[2][8]) {   // this thread's part of a [64][64] state
#pragma unroll
        for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (base) v = *reinterpret_cast<const float4 *>(base + (row0 + rg + 32 * rr) * kN + 4 * q + 32 * m);
                x[rr][4 * m] = v.x; x[rr][4 * m + 1] = v.y; x[rr][4 * m + 2] = v.z; x[rr][4 * m + 3] = v.w;
            }
    };
    auto store_rows = [&](float *base, const float (&x)[2][8]) {
#pragma unroll
        for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int m = 0; m < 2; ++m)
                *reinterpret_cast<float4 *>(base + (row0 + rg + 32 * rr) * kN + 4 * q + 32 * m) =
                    make_float4(x[rr][4 * m], x[rr][4 * m + 1], x[rr][4 * m + 2], x[rr][4 * m + 3]);
    };
    auto store_rows_sm = [&](float (*dst)[kRS], const float (&x)[2][8]) {
#pragma unroll
        for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int m = 0; m < 2; ++m)
                *reinterpret_cast<float4 *>(&dst[rg + 32 * rr][4 * q + 32 * m]) =
                    make_float4(x[rr][4 * m], x[rr][4 * m + 1], x[rr][4 * m + 2], x[rr][4 * m + 3]);
    };
    // this thread's eight columns of a staged token vector
    auto vec8 = [&](int slot, int tt, float (&o)[8]) {
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const float4 v = *reinterpret_cast<const float4 *>(&sm.vec[slot][tt][4 * q + 32 * m]);
            o[4 * m] = v.x; o[4 * m + 1] = v.y; o[4 * m + 2] = v.z; o[4 * m + 3] = v.w;
        }
    };
    auto rowsum = [&](float x) {   // over the eight lanes of a row group
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        return x + __shfl_xor_sync(0xffffffffu, x, 4);
    };

    // Token vectors of [t0, t0 + L) -> shared fp32: thread (tt = tid / 32) takes channels
    // 2 (tid % 32) and the next. `full` also loads r and dy (the backward block).
    float pre[kVecs][2];
    auto fetch = [&](int t0, int L, bool full) {
        const int tt = tid >> 5, c = 2 * (tid & 31);
        if (tt < L) {
            const size_t o = tok(t0 + tt) + c;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                pre[VW][e] = ld_in<Tin>(p.w, o + e);
                pre[VKK][e] = ld_in<Tin>(p.kk, o + e);
                pre[VA][e] = ld_in<Tin>(p.a, o + e);
                pre[VK][e] = ld_in<Tin>(p.k, o + e);
                pre[VV][e] = ld_in<Tin>(p.v, o + e);
                if (full) {
                    pre[VR][e] = ld_in<Tin>(p.r, o + e);
                    pre[VDY][e] = __ldg(p.dy + o + e);
                }
            }
        }
    };
    auto stage = [&](int L, bool full) {
        const int tt = tid >> 5, c = 2 * (tid & 31);
        if (tt < L) {
            auto put = [&](int slot, float x0, float x1) {
                *reinterpret_cast<float2 *>(&sm.vec[slot][tt][c]) = make_float2(x0, x1);
            };
            put(VW, pre[VW][0], pre[VW][1]);
            put(VKK, pre[VKK][0], pre[VKK][1]);
            put(VB, pre[VKK][0] * pre[VA][0], pre[VKK][1] * pre[VA][1]);
            put(VA, pre[VA][0], pre[VA][1]);
            put(VK, pre[VK][0], pre[VK][1]);
            put(VV, pre[VV][0], pre[VV][1]);
            if (full) {
                put(VR, pre[VR][0], pre[VR][1]);
                put(VDY, pre[VDY][0], pre[VDY][1]);
            }
        }
    };
    // One forward token on the row owner's registers: s <- s diag(w) - (s . kk) b^T + v_i k^T.
    // Returns s . kk of the thread's two rows.
    auto forward_step = [&](int tt, float (&sa)[2]) {
        float kk[8], w[8], bb[8], kv[8];
        vec8(VKK, tt, kk);
        float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
        for (int rr = 0; rr < 2; ++rr)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[rr][c & 1] = fmaf(s[rr][c], kk[c], acc[rr][c & 1]);
        sa[0] = rowsum(acc[0][0] + acc[0][1]);
        sa[1] = rowsum(acc[1][0] + acc[1][1]);
        vec8(VW, tt, w);
        vec8(VB, tt, bb);
        vec8(VK, tt, kv);
        const float v0 = sm.vec[VV][tt][row0 + rg], v1 = sm.vec[VV][tt][row0 + rg + 32];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            s[0][c] = fmaf(v0, kv[c], fmaf(-sa[0], bb[c], s[0][c] * w[c]));
            s[1][c] = fmaf(v1, kv[c], fmaf(-sa[1], bb[c], s[1][c] * w[c]));
        }
    };

    load_rows(p.dS_T ? p.dS_T + size_t(unit) * kN * kN : nullptr, d);
    const int K = segment_length(T, p.snap_every);
    const int nseg = (T + K - 1) / K;
    const int n_snap = p.snap_every > 0 ? T / p.snap_every : 0;
    float *ck = p.ws + size_t(unit) * size_t((K + kLb - 1) / kLb) * kN * kN;   // this head's checkpoints

    for (int seg = nseg - 1; seg >= 0; --seg) {
        const int tb = seg * K, te = min(T, tb + K);
        const float *start = seg == 0 ? (p.S0 ? p.S0 + size_t(unit) * kN * kN : nullptr)
                                      : p.snaps + ((size_t(b) * n_snap + (seg - 1)) * H + h) * kN * kN;
        load_rows(start, s);
        // ---- segment forward: one checkpoint per block start (the last block's end is not needed)
        if (tb + kLb < te) fetch(tb, min(kLb, te - tb), false);
        for (int t0 = tb; t0 < te; t0 += kLb) {
            store_rows(ck + size_t((t0 - tb) / kLb) * kN * kN, s);
            if (t0 + kLb >= te) break;
            const int L = min(kLb, te - t0);
            __syncthreads();   // the previous block's vectors are consumed
            stage(L, false);
            __syncthreads();
            if (t0 + kLb + kLb < te) fetch(t0 + kLb, min(kLb, te - t0 - kLb), false);
            for (int tt = 0; tt < L; ++tt) {
                float sa[2];
                forward_step(tt, sa);
            }
        }
        // ---- blocks in reverse; each block's checkpoint is loaded one block ahead
        const int last0 = tb + ((te - tb - 1) / kLb) * kLb;
        fetch(last0, te - last0, true);
        float cnext[2][8];
        load_rows(ck + size_t((last0 - tb) / kLb) * kN * kN, cnext);
        for (int t0 = last0; t0 >= tb; t0 -= kLb) {
            const int L = min(kLb, te - t0);
#pragma unroll
            for (int rr = 0; rr < 2; ++rr)
#pragma unroll
                for (int c = 0; c < 8; ++c) s[rr][c] = cnext[rr][c];
            __syncthreads();   // the previous block's shared data are consumed
            stage(L, true);
            __syncthreads();
            if (t0 - kLb >= tb) {
                fetch(t0 - kLb, kLb, true);
                load_rows(ck + size_t((t0 - kLb - tb) / kLb) * kN * kN, cnext);
            }
            // recompute S_{t0} .. S_{t0 + L} (this CTA's rows) into shared memory
            for (int tt = 0; tt < L; ++tt) {
                store_rows_sm(sm.S[tt], s);
                float sa[2];
                forward_step(tt, sa);
                if (q == 0) {
                    sm.sa[tt][rg] = sa[0];
                    sm.sa[tt][rg + 32] = sa[1];
                }
            }
            store_rows_sm(sm.S[L], s);
            // reverse recurrence over the block on the row owner's registers
            for (int tt = L - 1; tt >= 0; --tt) {
                float rv[8], kv[8], bb[8];
                vec8(VR, tt, rv);
                vec8(VK, tt, kv);
                vec8(VB, tt, bb);
                const float dy0 = sm.vec[VDY][tt][row0 + rg], dy1 = sm.vec[VDY][tt][row0 + rg + 32];
                float av[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, ab[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    d[0][c] = fmaf(dy0, rv[c], d[0][c]);
                    d[1][c] = fmaf(dy1, rv[c], d[1][c]);
                    av[0][c & 1] = fmaf(d[0][c], kv[c], av[0][c & 1]);
                    av[1][c & 1] = fmaf(d[1][c], kv[c], av[1][c & 1]);
                    ab[0][c & 1] = fmaf(d[0][c], bb[c], ab[0][c & 1]);
                    ab[1][c & 1] = fmaf(d[1][c], bb[c], ab[1][c & 1]);
                }
                const float dv0 = rowsum(av[0][0] + av[0][1]), dv1 = rowsum(av[1][0] + av[1][1]);
                const float ds0 = -rowsum(ab[0][0] + ab[0][1]), ds1 = -rowsum(ab[1][0] + ab[1][1]);
                if (q == 0) {
                    p.dv[tok(t0 + tt) + row0 + rg] = dv0;
                    p.dv[tok(t0 + tt) + row0 + rg + 32] = dv1;
                    sm.ds[tt][rg] = ds0;
                    sm.ds[tt][rg + 32] = ds1;
                }
                store_rows_sm(sm.D[tt], d);
                float w[8], kk[8];
                vec8(VW, tt, w);
                vec8(VKK, tt, kk);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    d[0][c] = fmaf(ds0, kk[c], d[0][c] * w[c]);
                    d[1][c] = fmaf(ds1, kk[c], d[1][c] * w[c]);
                }
            }
            __syncthreads();
            // ---- column pass: the per-token gradient vectors, summed over the 64 rows
            {
                const int cq = (tid & 3) | (((tid >> 3) & 1) << 2) | (((tid >> 5) & 1) << 3);
                const int rq = ((tid >> 2) & 1) | (((tid >> 4) & 1) << 1);
                const int tt = tid >> 6;
                if (tt < L) {   // warp-uniform
                    float g[kGrads][4] = {};
#pragma unroll 4
                    for (int r = 0; r < 16; ++r) {
                        const int i = 4 * r + rq;
                        const float4 sp = *reinterpret_cast<const float4 *>(&sm.S[tt][i][4 * cq]);
                        const float4 sn = *reinterpret_cast<const float4 *>(&sm.S[tt + 1][i][4 * cq]);
                        const float4 dd = *reinterpret_cast<const float4 *>(&sm.D[tt][i][4 * cq]);
                        const float cdy = sm.vec[VDY][tt][i], cv = sm.vec[VV][tt][i];
                        const float csa = sm.sa[tt][i], cds = sm.ds[tt][i];
                        const float spv[4] = {sp.x, sp.y, sp.z, sp.w}, snv[4] = {sn.x, sn.y, sn.z, sn.w};
                        const float ddv[4] = {dd.x, dd.y, dd.z, dd.w};
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            g[GU][c] = fmaf(cdy, snv[c], g[GU][c]);
                            g[GZ][c] = fmaf(cds, spv[c], g[GZ][c]);
                            g[GK][c] = fmaf(cv, ddv[c], g[GK][c]);
                            g[GB][c] = fmaf(-csa, ddv[c], g[GB][c]);
                            g[GW][c] = fmaf(spv[c], ddv[c], g[GW][c]);
                        }
                    }
#pragma unroll
                    for (int x = 0; x < kGrads; ++x)
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            g[x][c] += __shfl_xor_sync(0xffffffffu, g[x][c], 4);
                            g[x][c] += __shfl_xor_sync(0xffffffffu, g[x][c], 16);
                        }
                    if (rq == 0) {
                        const size_t o = tok(t0 + tt) + 4 * cq;
                        const float4 a4 = *reinterpret_cast<const float4 *>(&sm.vec[VA][tt][4 * cq]);
                        const float4 kk4 = *reinterpret_cast<const float4 *>(&sm.vec[VKK][tt][4 * cq]);
                        *reinterpret_cast<float4 *>(p.dr + o) = make_float4(g[GU][0], g[GU][1], g[GU][2], g[GU][3]);
                        *reinterpret_cast<float4 *>(p.dk + o) = make_float4(g[GK][0], g[GK][1], g[GK][2], g[GK][3]);
                        *reinterpret_cast<float4 *>(p.dw + o) = make_float4(g[GW][0], g[GW][1], g[GW][2], g[GW][3]);
                        *reinterpret_cast<float4 *>(p.dkk + o) =
                            make_float4(fmaf(g[GB][0], a4.x, g[GZ][0]), fmaf(g[GB][1], a4.y, g[GZ][1]),
                                        fmaf(g[GB][2], a4.z, g[GZ][2]), fmaf(g[GB][3], a4.w, g[GZ][3]));
                        *reinterpret_cast<float4 *>(p.da + o) =
                            make_float4(g[GB][0] * kk4.x, g[GB][1] * kk4.y, g[GB][2] * kk4.z, g[GB][3] * kk4.w);
                    }
                }
            }
        }
    }
    if (p.dS0) store_rows(p.dS0 + size_t(unit) * kN * kN, d);
}

// ---- host side ---------------------------------------------------------------------------------------

template <class Tin>
cudaError_t launch_bwd_t(const BwdArgs &p) {
    const int smem = int(sizeof(BwdSmem));
    const cudaError_t attr = allow_dynamic_smem(reinterpret_cast<const void *>(bwd_kernel<Tin>), smem);
    if (attr != cudaSuccess) return attr;
    bwd_kernel<Tin><<<p.B * p.H, kBwdThreads, smem, p.stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

size_t backward_checkpoint_bytes(int B, int T, int H, int snap_every) {
    if (T <= 0) return 0;
    const int K = segment_length(T, snap_every);
    return size_t(B) * H * size_t((K + kLb - 1) / kLb) * kN * kN * sizeof(float);
}

size_t backward_static_scratch_bytes() { return kStaticScratchBytes; }

// Device address of the static scratch on the current device. A successful lookup is kept per
// device; a failed one is not, so the next call tries again. The kept address belongs to the
// device's current context and is not valid after cudaDeviceReset.
cudaError_t backward_static_scratch(void **ptr) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static void *addr[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void *a = nullptr;
        if ((e = cudaGetSymbolAddress(&a, g_bwd_scratch)) != cudaSuccess) return e;
        addr[dev] = a;
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

cudaError_t launch_backward(const BwdArgs &p) {
    return p.dt == WKV7_BF16 ? launch_bwd_t<__nv_bfloat16>(p) : launch_bwd_t<float>(p);
}

}  // namespace wkv7
