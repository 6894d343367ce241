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
// One CTA per (b, h), 256 threads. The sweep needs S_{t-1} at every t in reverse order.
// The sequence is cut into segments (between the forward's snapshots, or the whole
// sequence); a segment's forward is run once to write one state per block of kLb tokens
// to the workspace, then the blocks are taken in reverse: each block's states are
// recomputed from its checkpoint into shared memory, the reverse recurrence runs over the
// block, and the per-token gradient vectors are reduced over the 64 rows from shared
// memory. Two thread layouts:
//   row owner   (recurrence): thread (i = tid / 4, q = tid % 4) holds columns
//                4q + 16m + c (m, c < 4) of row i of S and of dS in registers; the three
//                dot products per row and token reduce over the four lanes of a row.
//   column pass (gradient vectors): thread (token tt, column quad cq, row quarter rq)
//                sums 16 rows 4r + rq of five products, then the quarters combine by
//                two shuffles.
// Shared rows are 80 floats apart (320 B = 64 mod 128), so the row owners' float4 stores
// and the column pass's float4 loads are both free of bank conflicts.
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
constexpr int kLb = 4;          // tokens per block
constexpr int kRS = 80;         // shared row stride (floats)

// Tokens between recomputation anchors: the snapshot interval, or the whole sequence.
__host__ __device__ inline int segment_length(int T, int snap_every) {
    return (snap_every > 0 && snap_every < T) ? snap_every : (T > 0 ? T : 1);
}

enum { VW = 0, VKK, VB, VK, VR, VV, VDY, VA, kVecs };

struct BwdSmem {
    float S[kLb + 1][kN][kRS];   // S_{t0} .. S_{t0 + L}
    float D[kLb][kN][kRS];       // the gradient reaching S_t, t in the block
    float vec[kVecs][kLb][kN];   // w, kk, b = kk*a, k, r, v, dy, a (fp32)
    float sa[kLb][kN];           // s_i = S_{t-1}[i, :] . kk_t
    float ds[kLb][kN];           // ds_i = -dS_t[i, :] . b_t
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
    const int row = tid >> 2, q = tid & 3;
    auto tok = [&](int t) { return ((size_t(b) * T + t) * H + h) * kN; };

    float s[16], d[16];
    auto load_row = [&](const float *base, float (&x)[16]) {   // row `row` of a [64][64] state, nullable
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (base) v = *reinterpret_cast<const float4 *>(base + row * kN + 4 * q + 16 * m);
            x[4 * m] = v.x; x[4 * m + 1] = v.y; x[4 * m + 2] = v.z; x[4 * m + 3] = v.w;
        }
    };
    auto store_row = [&](float *base, const float (&x)[16]) {
#pragma unroll
        for (int m = 0; m < 4; ++m)
            *reinterpret_cast<float4 *>(base + row * kN + 4 * q + 16 * m) =
                make_float4(x[4 * m], x[4 * m + 1], x[4 * m + 2], x[4 * m + 3]);
    };
    auto store_row_sm = [&](float (*dst)[kRS], const float (&x)[16]) {
#pragma unroll
        for (int m = 0; m < 4; ++m)
            *reinterpret_cast<float4 *>(&dst[row][4 * q + 16 * m]) =
                make_float4(x[4 * m], x[4 * m + 1], x[4 * m + 2], x[4 * m + 3]);
    };
    auto vec4 = [&](int slot, int tt, int m) {
        return *reinterpret_cast<const float4 *>(&sm.vec[slot][tt][4 * q + 16 * m]);
    };
    auto rowsum = [&](float x) {
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        return x + __shfl_xor_sync(0xffffffffu, x, 2);
    };

    // Token vectors of [t0, t0 + L) -> shared fp32 (one channel of one token per thread).
    // `full` also loads r, dy and a (the backward block); otherwise only what the forward reads.
    float pre[kVecs];
    auto fetch = [&](int t0, int L, bool full) {
        const int tt = tid >> 6, c = tid & 63;
        if (tt < L) {
            const size_t o = tok(t0 + tt) + c;
            pre[VW] = ld_in<Tin>(p.w, o);
            pre[VKK] = ld_in<Tin>(p.kk, o);
            pre[VA] = ld_in<Tin>(p.a, o);
            pre[VK] = ld_in<Tin>(p.k, o);
            pre[VV] = ld_in<Tin>(p.v, o);
            if (full) {
                pre[VR] = ld_in<Tin>(p.r, o);
                pre[VDY] = __ldg(p.dy + o);
            }
        }
    };
    auto stage = [&](int L, bool full) {
        const int tt = tid >> 6, c = tid & 63;
        if (tt < L) {
            sm.vec[VW][tt][c] = pre[VW];
            sm.vec[VKK][tt][c] = pre[VKK];
            sm.vec[VB][tt][c] = pre[VKK] * pre[VA];
            sm.vec[VA][tt][c] = pre[VA];
            sm.vec[VK][tt][c] = pre[VK];
            sm.vec[VV][tt][c] = pre[VV];
            if (full) {
                sm.vec[VR][tt][c] = pre[VR];
                sm.vec[VDY][tt][c] = pre[VDY];
            }
        }
    };
    // One forward token on the row owner's registers: s <- s diag(w) - (s . kk) b^T + v_i k^T.
    auto forward_step = [&](int tt) {
        float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
        for (int m = 0; m < 4; m += 2) {
            const float4 k0 = vec4(VKK, tt, m), k1 = vec4(VKK, tt, m + 1);
            acc0 = fmaf(s[4 * m], k0.x, acc0); acc0 = fmaf(s[4 * m + 1], k0.y, acc0);
            acc0 = fmaf(s[4 * m + 2], k0.z, acc0); acc0 = fmaf(s[4 * m + 3], k0.w, acc0);
            acc1 = fmaf(s[4 * m + 4], k1.x, acc1); acc1 = fmaf(s[4 * m + 5], k1.y, acc1);
            acc1 = fmaf(s[4 * m + 6], k1.z, acc1); acc1 = fmaf(s[4 * m + 7], k1.w, acc1);
        }
        const float sa = rowsum(acc0 + acc1);
        const float vi = sm.vec[VV][tt][row];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float4 w4 = vec4(VW, tt, m), b4 = vec4(VB, tt, m), k4 = vec4(VK, tt, m);
            const float wv[4] = {w4.x, w4.y, w4.z, w4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
            const float kv[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
            for (int c = 0; c < 4; ++c) s[4 * m + c] = fmaf(vi, kv[c], fmaf(-sa, bv[c], s[4 * m + c] * wv[c]));
        }
        return sa;
    };

    load_row(p.dS_T ? p.dS_T + size_t(unit) * kN * kN : nullptr, d);
    const int K = segment_length(T, p.snap_every);
    const int nseg = (T + K - 1) / K;
    const int n_snap = p.snap_every > 0 ? T / p.snap_every : 0;
    float *ck = p.ws + size_t(unit) * size_t((K + kLb - 1) / kLb) * kN * kN;   // this head's checkpoints

    for (int seg = nseg - 1; seg >= 0; --seg) {
        const int tb = seg * K, te = min(T, tb + K);
        const float *start = seg == 0 ? (p.S0 ? p.S0 + size_t(unit) * kN * kN : nullptr)
                                      : p.snaps + ((size_t(b) * n_snap + (seg - 1)) * H + h) * kN * kN;
        load_row(start, s);
        // ---- segment forward: one checkpoint per block start (the last block's end is not needed)
        if (tb + kLb < te) fetch(tb, min(kLb, te - tb), false);
        for (int t0 = tb; t0 < te; t0 += kLb) {
            store_row(ck + size_t((t0 - tb) / kLb) * kN * kN, s);
            if (t0 + kLb >= te) break;
            const int L = min(kLb, te - t0);
            __syncthreads();   // the previous block's vectors are consumed
            stage(L, false);
            __syncthreads();
            if (t0 + kLb + kLb < te) fetch(t0 + kLb, min(kLb, te - t0 - kLb), false);
            for (int tt = 0; tt < L; ++tt) forward_step(tt);
        }
        // ---- blocks in reverse
        const int last0 = tb + ((te - tb - 1) / kLb) * kLb;
        fetch(last0, te - last0, true);
        for (int t0 = last0; t0 >= tb; t0 -= kLb) {
            const int L = min(kLb, te - t0);
            load_row(ck + size_t((t0 - tb) / kLb) * kN * kN, s);
            __syncthreads();   // the previous block's shared data are consumed
            stage(L, true);
            __syncthreads();
            if (t0 - kLb >= tb) fetch(t0 - kLb, kLb, true);
            // recompute S_{t0} .. S_{t0 + L} into shared memory
            for (int tt = 0; tt < L; ++tt) {
                store_row_sm(sm.S[tt], s);
                const float sa = forward_step(tt);
                if (q == 0) sm.sa[tt][row] = sa;
            }
            store_row_sm(sm.S[L], s);
            // reverse recurrence over the block on the row owner's registers
            for (int tt = L - 1; tt >= 0; --tt) {
                const float dyi = sm.vec[VDY][tt][row];
                float acc_v = 0.f, acc_b = 0.f;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float4 r4 = vec4(VR, tt, m), k4 = vec4(VK, tt, m), b4 = vec4(VB, tt, m);
                    const float rv[4] = {r4.x, r4.y, r4.z, r4.w}, kv[4] = {k4.x, k4.y, k4.z, k4.w};
                    const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        d[4 * m + c] = fmaf(dyi, rv[c], d[4 * m + c]);
                        acc_v = fmaf(d[4 * m + c], kv[c], acc_v);
                        acc_b = fmaf(d[4 * m + c], bv[c], acc_b);
                    }
                }
                const float dv = rowsum(acc_v), ds = -rowsum(acc_b);
                if (q == 0) {
                    p.dv[tok(t0 + tt) + row] = dv;
                    sm.ds[tt][row] = ds;
                }
                store_row_sm(sm.D[tt], d);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float4 w4 = vec4(VW, tt, m), kk4 = vec4(VKK, tt, m);
                    const float wv[4] = {w4.x, w4.y, w4.z, w4.w}, kv[4] = {kk4.x, kk4.y, kk4.z, kk4.w};
#pragma unroll
                    for (int c = 0; c < 4; ++c) d[4 * m + c] = fmaf(ds, kv[c], d[4 * m + c] * wv[c]);
                }
            }
            __syncthreads();
            // ---- column pass: the per-token gradient vectors, summed over the 64 rows
            {
                const int cq = (tid & 3) | (((tid >> 3) & 1) << 2) | (((tid >> 5) & 1) << 3);
                const int rq = ((tid >> 2) & 1) | (((tid >> 4) & 1) << 1);
                const int tt = tid >> 6;
                if (tt < L) {   // warp-uniform
                    float u[4] = {0.f, 0.f, 0.f, 0.f}, z[4] = {0.f, 0.f, 0.f, 0.f}, gk[4] = {0.f, 0.f, 0.f, 0.f};
                    float gb[4] = {0.f, 0.f, 0.f, 0.f}, gw[4] = {0.f, 0.f, 0.f, 0.f};
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
                            u[c] = fmaf(cdy, snv[c], u[c]);
                            z[c] = fmaf(cds, spv[c], z[c]);
                            gk[c] = fmaf(cv, ddv[c], gk[c]);
                            gb[c] = fmaf(-csa, ddv[c], gb[c]);
                            gw[c] = fmaf(spv[c], ddv[c], gw[c]);
                        }
                    }
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
#pragma unroll
                        for (int o = 4; o <= 16; o <<= 2) {
                            u[c] += __shfl_xor_sync(0xffffffffu, u[c], o);
                            z[c] += __shfl_xor_sync(0xffffffffu, z[c], o);
                            gk[c] += __shfl_xor_sync(0xffffffffu, gk[c], o);
                            gb[c] += __shfl_xor_sync(0xffffffffu, gb[c], o);
                            gw[c] += __shfl_xor_sync(0xffffffffu, gw[c], o);
                        }
                    }
                    if (rq == 0) {
                        const size_t o = tok(t0 + tt) + 4 * cq;
                        const float4 a4 = *reinterpret_cast<const float4 *>(&sm.vec[VA][tt][4 * cq]);
                        const float4 kk4 = *reinterpret_cast<const float4 *>(&sm.vec[VKK][tt][4 * cq]);
                        *reinterpret_cast<float4 *>(p.dr + o) = make_float4(u[0], u[1], u[2], u[3]);
                        *reinterpret_cast<float4 *>(p.dk + o) = make_float4(gk[0], gk[1], gk[2], gk[3]);
                        *reinterpret_cast<float4 *>(p.dw + o) = make_float4(gw[0], gw[1], gw[2], gw[3]);
                        *reinterpret_cast<float4 *>(p.dkk + o) =
                            make_float4(fmaf(gb[0], a4.x, z[0]), fmaf(gb[1], a4.y, z[1]), fmaf(gb[2], a4.z, z[2]),
                                        fmaf(gb[3], a4.w, z[3]));
                        *reinterpret_cast<float4 *>(p.da + o) =
                            make_float4(gb[0] * kk4.x, gb[1] * kk4.y, gb[2] * kk4.z, gb[3] * kk4.w);
                    }
                }
            }
        }
    }
    if (p.dS0) store_row(p.dS0 + size_t(unit) * kN * kN, d);
}

template <class Tin>
cudaError_t launch_bwd_t(const BwdArgs &p) {
    const int smem = int(sizeof(BwdSmem));
    static const cudaError_t attr =
        cudaFuncSetAttribute(bwd_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
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

// Device address of the static scratch on the current device, looked up once per device.
cudaError_t backward_static_scratch(void **ptr) {
    constexpr int kMaxDevices = 64;
    static std::once_flag once[kMaxDevices];
    static void *addr[kMaxDevices];
    static cudaError_t err[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::call_once(once[dev], [dev] { err[dev] = cudaGetSymbolAddress(&addr[dev], g_bwd_scratch); });
    *ptr = addr[dev];
    return err[dev];
}

cudaError_t launch_backward(const BwdArgs &p) {
    return p.dt == WKV7_BF16 ? launch_bwd_t<__nv_bfloat16>(p) : launch_bwd_t<float>(p);
}

}  // namespace wkv7
