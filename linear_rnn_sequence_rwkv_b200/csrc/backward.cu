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
// A CTA of 256 threads owns 64 rows of one (b, h): all of them at N = 64, one half at N = 128
// (a cluster of two CTAs per head; rows are independent, only the gradient vectors dr, dk, dw,
// dkk, da sum over all rows). The sweep needs S_{t-1} at every t in reverse order. The sequence
// is cut into segments (between the forward's snapshots, or the whole sequence); a segment's
// forward is run once to write one state per block of kLb tokens to the workspace, then the
// blocks are taken in reverse: each block's states are recomputed from its checkpoint into
// shared memory, the reverse recurrence runs over the block, and the per-token gradient vectors
// are summed over the CTA's rows from shared memory. Two thread layouts:
//   row owner   (recurrence): LPR = N / 8 lanes share a row, lane q holding columns
//                4q + (N/2) m + c (m < 2, c < 4); thread (g = tid / LPR, q) holds rows
//                g + (256 / LPR) rr of S and dS in registers (rr < 2 at N = 64, < 4 at N = 128);
//                the dot products per row and token reduce over the LPR lanes. Several rows per
//                thread divide the shared-memory wavefronts of the token vectors, which every row
//                group reads, by the rows each read serves.
//   column pass (gradient vectors): thread (token tt, column quad cq, row quarter rq) sums
//                the 16 rows 4r + rq of five products; the quarters combine by two shuffles. At
//                N = 128 each CTA of the pair finishes half of the columns: it stores the partial
//                sums of the other half into its partner's shared memory (distributed shared
//                memory), and after one cluster barrier per block adds the partner's partials
//                to its own (a double-buffered exchange area, so the next block's stores never
//                meet unread data).
// A split of a 64-wide head's rows over a cluster of two CTAs measured slower on the 96-head
// prefill (the busiest SMs still carry a whole head's work), so N = 64 keeps one CTA per head.
// Shared rows are N + 16 floats apart (64 mod 128 bytes), so the column pass's float4 loads
// are free of bank conflicts (the row owners' stores are: LPR lanes write one row's contiguous
// columns).
#include <mutex>
#include <type_traits>

#include "backward.cuh"
#include "tc_util.cuh"

namespace wkv7 {
namespace {

// Scratch of the allocation-free backward entry: the recomputation checkpoints live in this
// module-scope array instead of a caller's workspace. Every checkpoint is written before it is
// read, so nothing in it needs to start at zero.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;   // 2048 states of 64 x 64 fp32
static __device__ __align__(256) float g_bwd_scratch[kStaticScratchBytes / sizeof(float)];

constexpr int kBwdThreads = 256;
constexpr int kRows = 64;       // rows of S per CTA

// Shape of the kernel at head size NN.
template <int NN> struct BwdShape;
template <> struct BwdShape<64> {
    static constexpr int kCPH = 1;   // CTAs per head (a cluster)
    static constexpr int kRPT = 2;   // rows per row-owner thread
    static constexpr int kLb = 4;    // tokens per block
    static constexpr int kRS = 80;   // shared row stride (floats)
};
template <> struct BwdShape<128> {
    static constexpr int kCPH = 2, kRPT = 4, kLb = 2, kRS = 144;
};
template <int NN> constexpr int kLPR = NN / 8;                      // lanes per row
template <int NN> constexpr int kNRG = kBwdThreads / kLPR<NN>;      // row groups
static_assert(kNRG<64> * BwdShape<64>::kRPT == kRows && kNRG<128> * BwdShape<128>::kRPT == kRows, "rows");
static_assert(64 * BwdShape<64>::kCPH == 64 && 64 * BwdShape<128>::kCPH == 128, "rows per head");

// Tokens between recomputation anchors: the snapshot interval, or the whole sequence.
__host__ __device__ inline int segment_length(int T, int snap_every) {
    return (snap_every > 0 && snap_every < T) ? snap_every : (T > 0 ? T : 1);
}

// Token vectors indexed by column (the key index); v and dy, indexed by row, go to BwdSmem::sc.
enum { VW = 0, VKK, VA, VK, VR, VB, kVecs };
enum { GU = 0, GZ, GK, GB, GW, kGrads };   // partial sums: S_t^T dy, S_{t-1}^T ds, dS^T v, db, dw

// The staged column vectors of a block. Each row-owner thread reads its eight columns
// 4q + (N/2) m + c of every vector, once per row group, so the bytes a lane reads per token set
// the shared-memory traffic of the recurrence phases.
//   fp32 inputs: w, kk, a, k, r and b = kk * a in fp32, in column order.
//   bf16 inputs: w, kk, a, k, r as loaded (bf16 is exact in fp32, so nothing is lost), with the
//                columns permuted so that a thread's eight sit in one 16-byte word (column j at
//                8 ((j / 4) % LPR) + 4 (j / (N/2)) + j % 4); b is formed in registers as kk * a,
//                the same fp32 product the fp32 layout stores.
template <class Tin, int NN> struct VecTile;
template <int NN> struct VecTile<float, NN> {
    float x[kVecs][BwdShape<NN>::kLb][NN];
    __device__ __forceinline__ void put(int slot, int tt, int c, float2 v) {
        *reinterpret_cast<float2 *>(&x[slot][tt][c]) = v;
    }
    __device__ __forceinline__ void get8(int slot, int tt, int q, float (&o)[8]) const {
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const float4 v = *reinterpret_cast<const float4 *>(&x[slot][tt][4 * q + (NN / 2) * m]);
            o[4 * m] = v.x; o[4 * m + 1] = v.y; o[4 * m + 2] = v.z; o[4 * m + 3] = v.w;
        }
    }
    __device__ __forceinline__ void b8(int tt, int q, const float (&)[8], float (&o)[8]) const { get8(VB, tt, q, o); }
    __device__ __forceinline__ float4 get4(int slot, int tt, int cq) const {
        return *reinterpret_cast<const float4 *>(&x[slot][tt][4 * cq]);
    }
};
template <int NN> struct VecTile<__nv_bfloat16, NN> {
    unsigned short x[VB][BwdShape<NN>::kLb][NN];
    static __device__ __forceinline__ int perm(int j) {
        return 8 * ((j >> 2) % kLPR<NN>) + 4 * (j / (NN / 2)) + (j & 3);
    }
    __device__ __forceinline__ void put(int slot, int tt, int c, unsigned int bits) {   // channels c, c + 1 (c even)
        *reinterpret_cast<unsigned int *>(&x[slot][tt][perm(c)]) = bits;
    }
    __device__ __forceinline__ void get8(int slot, int tt, int q, float (&o)[8]) const {
        const uint4 u = *reinterpret_cast<const uint4 *>(&x[slot][tt][8 * q]);
        o[0] = bf16_lo(u.x); o[1] = bf16_hi(u.x); o[2] = bf16_lo(u.y); o[3] = bf16_hi(u.y);
        o[4] = bf16_lo(u.z); o[5] = bf16_hi(u.z); o[6] = bf16_lo(u.w); o[7] = bf16_hi(u.w);
    }
    __device__ __forceinline__ void b8(int tt, int q, const float (&kk)[8], float (&o)[8]) const {
        get8(VA, tt, q, o);
#pragma unroll
        for (int c = 0; c < 8; ++c) o[c] = kk[c] * o[c];
    }
    __device__ __forceinline__ float4 get4(int slot, int tt, int cq) const {
        const uint2 u = *reinterpret_cast<const uint2 *>(&x[slot][tt][perm(4 * cq)]);
        return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
    }
};

// N = 128: the partner's partial sums of this CTA's 64 columns (16 quads), by block parity.
template <int NN> struct XBuf {
    float4 x[2][BwdShape<NN>::kLb][16][kGrads];
};
template <> struct XBuf<64> {};

template <class Tin, int NN>
struct BwdSmem {
    using Sh = BwdShape<NN>;
    float S[Sh::kLb + 1][kRows][Sh::kRS];   // S_{t0} .. S_{t0 + L}, this CTA's rows
    float D[Sh::kLb][kRows][Sh::kRS];       // the gradient reaching S_t, t in the block
    float4 sc[Sh::kLb][kRows];              // per row i: dy_i, v_i, s_i = S_{t-1}[i, :] . kk_t, ds_i = -dS_t[i, :] . b_t
    VecTile<Tin, NN> vec;
    XBuf<NN> xb;
};

// Two adjacent channels as loaded; converted to fp32 only when staged, so that the loads of
// the next block stay in flight across the current one.
template <class Tin> struct Pair;
template <> struct Pair<float> {
    float2 x;
    __device__ __forceinline__ void load(const void *p, size_t i) {
        x = __ldg(reinterpret_cast<const float2 *>(static_cast<const float *>(p) + i));
    }
    __device__ __forceinline__ float2 get() const { return x; }
};
template <> struct Pair<__nv_bfloat16> {
    unsigned int x;
    __device__ __forceinline__ void load(const void *p, size_t i) {
        x = __ldg(reinterpret_cast<const unsigned int *>(static_cast<const __nv_bfloat16 *>(p) + i));
    }
    __device__ __forceinline__ float2 get() const { return make_float2(bf16_lo(x), bf16_hi(x)); }   // exact
};

template <int NN>
__device__ __forceinline__ void put_pair(VecTile<float, NN> &t, int slot, int tt, int c, const Pair<float> &v) {
    t.put(slot, tt, c, v.get());
}
template <int NN>
__device__ __forceinline__ void put_pair(VecTile<__nv_bfloat16, NN> &t, int slot, int tt, int c,
                                         const Pair<__nv_bfloat16> &v) {
    t.put(slot, tt, c, v.x);
}

__device__ __forceinline__ void st_cluster4(uint32_t cluster_addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(cluster_addr), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w)
                 : "memory");
}

template <class Tin, int NN>
__global__ void __launch_bounds__(kBwdThreads, 1) bwd_kernel(const BwdArgs p) {
    using Sh = BwdShape<NN>;
    constexpr int kLb = Sh::kLb, kRS = Sh::kRS, RPT = Sh::kRPT, CPH = Sh::kCPH;
    constexpr int LPR = kLPR<NN>, NRG = kNRG<NN>, HALF = NN / 2;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    BwdSmem<Tin, NN> &sm = *reinterpret_cast<BwdSmem<Tin, NN> *>(smem_raw);
    const int T = p.T, H = p.H;
    const int unit = blockIdx.x / CPH, b = unit / H, h = unit % H;
    const int rank = CPH > 1 ? int(tc::cluster_rank()) : 0;   // which 64 rows of the head
    if constexpr (CPH > 1) tc::cluster_sync();   // both CTAs running before any remote store
    const int row0 = kRows * rank;
    const int tid = threadIdx.x;
    // row owner: rows rg + NRG rr (rr < RPT), columns 4q + (N/2) m + c (m < 2, c < 4)
    const int rg = tid / LPR, q = tid % LPR;
    auto tok = [&](int t) { return ((size_t(b) * T + t) * H + h) * NN; };

    float s[RPT][8], d[RPT][8];
    // this thread's part of the CTA's 64 rows of a state: rows roff + local row of `base`
    auto load_rows = [&](const float *base, int roff, float (&x)[RPT][8]) {
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (base) v = *reinterpret_cast<const float4 *>(base + (roff + rg + NRG * rr) * NN + 4 * q + HALF * m);
                x[rr][4 * m] = v.x; x[rr][4 * m + 1] = v.y; x[rr][4 * m + 2] = v.z; x[rr][4 * m + 3] = v.w;
            }
    };
    auto store_rows = [&](float *base, int roff, const float (&x)[RPT][8]) {
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
            for (int m = 0; m < 2; ++m)
                *reinterpret_cast<float4 *>(base + (roff + rg + NRG * rr) * NN + 4 * q + HALF * m) =
                    make_float4(x[rr][4 * m], x[rr][4 * m + 1], x[rr][4 * m + 2], x[rr][4 * m + 3]);
    };
    auto store_rows_sm = [&](float (*dst)[kRS], const float (&x)[RPT][8]) {
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
            for (int m = 0; m < 2; ++m)
                *reinterpret_cast<float4 *>(&dst[rg + NRG * rr][4 * q + HALF * m]) =
                    make_float4(x[rr][4 * m], x[rr][4 * m + 1], x[rr][4 * m + 2], x[rr][4 * m + 3]);
    };
    // this thread's eight columns of a staged token vector
    auto vec8 = [&](int slot, int tt, float (&o)[8]) { sm.vec.get8(slot, tt, q, o); };
    auto rowsum = [&](float x) {   // over the LPR lanes of a row group
#pragma unroll
        for (int off = 1; off < LPR; off <<= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
        return x;
    };

    // Token vectors of [t0, t0 + L) -> shared memory: thread (tt = tid / (N/2)) takes key
    // channels c = 2 (tid % (N/2)) and c + 1, and v and dy of the CTA's rows c, c + 1 when
    // c < 64. `full` also loads r and dy (the backward block).
    Pair<Tin> pre[VB], pre_v;
    float2 pre_dy;
    constexpr bool kAllRows = CPH == 1;   // every staged channel pair is also a pair of this CTA's rows
    auto fetch = [&](int t0, int L, bool full) {
        const int tt = tid / HALF, c = 2 * (tid % HALF);
        if (tt < L) {
            const size_t o = tok(t0 + tt);
            pre[VW].load(p.w, o + c);
            pre[VKK].load(p.kk, o + c);
            pre[VA].load(p.a, o + c);
            pre[VK].load(p.k, o + c);
            if (kAllRows || c < kRows) pre_v.load(p.v, o + row0 + c);
            if (full) {
                pre[VR].load(p.r, o + c);
                if (kAllRows || c < kRows) pre_dy = __ldg(reinterpret_cast<const float2 *>(p.dy + o + row0 + c));
            }
        }
    };
    auto stage = [&](int L, bool full) {
        const int tt = tid / HALF, c = 2 * (tid % HALF);
        if (tt < L) {
            put_pair(sm.vec, VW, tt, c, pre[VW]);
            put_pair(sm.vec, VKK, tt, c, pre[VKK]);
            put_pair(sm.vec, VA, tt, c, pre[VA]);
            put_pair(sm.vec, VK, tt, c, pre[VK]);
            if constexpr (std::is_same<Tin, float>::value) {
                const float2 kk = pre[VKK].get(), a = pre[VA].get();
                sm.vec.put(VB, tt, c, make_float2(kk.x * a.x, kk.y * a.y));
            }
            if (kAllRows || c < kRows) {
                const float2 v = pre_v.get();
                sm.sc[tt][c].y = v.x;
                sm.sc[tt][c + 1].y = v.y;
            }
            if (full) {
                put_pair(sm.vec, VR, tt, c, pre[VR]);
                if (kAllRows || c < kRows) {
                    sm.sc[tt][c].x = pre_dy.x;
                    sm.sc[tt][c + 1].x = pre_dy.y;
                }
            }
        }
    };
    // One forward token on the row owner's registers: s <- s diag(w) - (s . kk) b^T + v_i k^T.
    // Returns s . kk of the thread's rows.
    auto forward_step = [&](int tt, float (&sa)[RPT]) {
        float kk[8], w[8], bb[8], kv[8];
        vec8(VKK, tt, kk);
        float acc[RPT][2];
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) {
            acc[rr][0] = acc[rr][1] = 0.f;
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[rr][c & 1] = fmaf(s[rr][c], kk[c], acc[rr][c & 1]);
        }
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) sa[rr] = rowsum(acc[rr][0] + acc[rr][1]);
        vec8(VW, tt, w);
        sm.vec.b8(tt, q, kk, bb);
        vec8(VK, tt, kv);
        float vr[RPT];
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr) vr[rr] = sm.sc[tt][rg + NRG * rr].y;
#pragma unroll
        for (int c = 0; c < 8; ++c)
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) s[rr][c] = fmaf(vr[rr], kv[c], fmaf(-sa[rr], bb[c], s[rr][c] * w[c]));
    };

    load_rows(p.dS_T ? p.dS_T + size_t(unit) * NN * NN : nullptr, row0, d);
    const int K = segment_length(T, p.snap_every);
    const int nseg = (T + K - 1) / K;
    const int n_snap = p.snap_every > 0 ? T / p.snap_every : 0;
    // this CTA's checkpoints: [64][N] states of its rows, one per block of a segment
    float *ck = p.ws + size_t(blockIdx.x) * size_t((K + kLb - 1) / kLb) * kRows * NN;
    uint32_t parity = 0;   // N = 128: exchange buffer of the current block

    for (int seg = nseg - 1; seg >= 0; --seg) {
        const int tb = seg * K, te = min(T, tb + K);
        const float *start = seg == 0 ? (p.S0 ? p.S0 + size_t(unit) * NN * NN : nullptr)
                                      : p.snaps + ((size_t(b) * n_snap + (seg - 1)) * H + h) * NN * NN;
        load_rows(start, row0, s);
        // ---- segment forward: one checkpoint per block start (the last block's end is not needed)
        if (tb + kLb < te) fetch(tb, min(kLb, te - tb), false);
        for (int t0 = tb; t0 < te; t0 += kLb) {
            store_rows(ck + size_t((t0 - tb) / kLb) * kRows * NN, 0, s);
            if (t0 + kLb >= te) break;
            const int L = min(kLb, te - t0);
            __syncthreads();   // the previous block's vectors are consumed
            stage(L, false);
            __syncthreads();
            if (t0 + kLb + kLb < te) fetch(t0 + kLb, min(kLb, te - t0 - kLb), false);
            auto seg_tok = [&](int tt) {
                float sa[RPT];
                forward_step(tt, sa);
            };
            if (L == kLb) {
#pragma unroll
                for (int tt = 0; tt < kLb; ++tt) seg_tok(tt);
            } else {
                for (int tt = 0; tt < L; ++tt) seg_tok(tt);
            }
        }
        // ---- blocks in reverse; each block's checkpoint is loaded one block ahead
        const int last0 = tb + ((te - tb - 1) / kLb) * kLb;
        fetch(last0, te - last0, true);
        float cnext[RPT][8];
        load_rows(ck + size_t((last0 - tb) / kLb) * kRows * NN, 0, cnext);
        for (int t0 = last0; t0 >= tb; t0 -= kLb) {
            const int L = min(kLb, te - t0);
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
                for (int c = 0; c < 8; ++c) s[rr][c] = cnext[rr][c];
            __syncthreads();   // the previous block's shared data are consumed
            stage(L, true);
            __syncthreads();
            if (t0 - kLb >= tb) {
                fetch(t0 - kLb, kLb, true);
                load_rows(ck + size_t((t0 - kLb - tb) / kLb) * kRows * NN, 0, cnext);
            }
            // recompute S_{t0} .. S_{t0 + L} (this CTA's rows) into shared memory
            auto rec_tok = [&](int tt) {
                store_rows_sm(sm.S[tt], s);
                float sa[RPT];
                forward_step(tt, sa);
                if (q == 0) {
#pragma unroll
                    for (int rr = 0; rr < RPT; ++rr) sm.sc[tt][rg + NRG * rr].z = sa[rr];
                }
            };
            if (L == kLb) {
#pragma unroll
                for (int tt = 0; tt < kLb; ++tt) rec_tok(tt);
            } else {
                for (int tt = 0; tt < L; ++tt) rec_tok(tt);
            }
            store_rows_sm(sm.S[L], s);
            // reverse recurrence over the block on the row owner's registers
            auto rev_tok = [&](int tt) {
                float rv[8], kv[8], bb[8], kk[8];
                vec8(VR, tt, rv);
                vec8(VK, tt, kv);
                vec8(VKK, tt, kk);
                sm.vec.b8(tt, q, kk, bb);
                float dyr[RPT], av[RPT][2], ab[RPT][2];
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr) {
                    dyr[rr] = sm.sc[tt][rg + NRG * rr].x;
                    av[rr][0] = av[rr][1] = ab[rr][0] = ab[rr][1] = 0.f;
                }
#pragma unroll
                for (int c = 0; c < 8; ++c)
#pragma unroll
                    for (int rr = 0; rr < RPT; ++rr) {
                        d[rr][c] = fmaf(dyr[rr], rv[c], d[rr][c]);
                        av[rr][c & 1] = fmaf(d[rr][c], kv[c], av[rr][c & 1]);
                        ab[rr][c & 1] = fmaf(d[rr][c], bb[c], ab[rr][c & 1]);
                    }
                float dvr[RPT], dsr[RPT];
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr) {
                    dvr[rr] = rowsum(av[rr][0] + av[rr][1]);
                    dsr[rr] = -rowsum(ab[rr][0] + ab[rr][1]);
                }
                if (q == 0) {
#pragma unroll
                    for (int rr = 0; rr < RPT; ++rr) {
                        p.dv[tok(t0 + tt) + row0 + rg + NRG * rr] = dvr[rr];
                        sm.sc[tt][rg + NRG * rr].w = dsr[rr];
                    }
                }
                store_rows_sm(sm.D[tt], d);
                float w[8];
                vec8(VW, tt, w);
#pragma unroll
                for (int c = 0; c < 8; ++c)
#pragma unroll
                    for (int rr = 0; rr < RPT; ++rr) d[rr][c] = fmaf(dsr[rr], kk[c], d[rr][c] * w[c]);
            };
            if (L == kLb) {
#pragma unroll
                for (int tt = kLb - 1; tt >= 0; --tt) rev_tok(tt);
            } else {
                for (int tt = L - 1; tt >= 0; --tt) rev_tok(tt);
            }
            __syncthreads();
            // ---- column pass: the per-token gradient vectors, summed over the CTA's 64 rows
            {
                // lanes: column-quad bits 0, 1, 2 from tid bits 0, 1, 3, row-quarter bits from
                // tid bits 2, 4; the higher column-quad bits and the token from the warp index
                constexpr int kQuads = NN / 4, kHiQ = kQuads / 8;   // column quads; their groups over warps
                const int cq = (tid & 3) | (((tid >> 3) & 1) << 2) | (((tid >> 5) & (kHiQ - 1)) << 3);
                const int rq = ((tid >> 2) & 1) | (((tid >> 4) & 1) << 1);
                const int tt = (tid >> 5) / kHiQ;
                float g[kGrads][4] = {};
                if (tt < L) {   // warp-uniform
#pragma unroll 4
                    for (int r = 0; r < kRows / 4; ++r) {
                        const int i = 4 * r + rq;
                        const float4 sp = *reinterpret_cast<const float4 *>(&sm.S[tt][i][4 * cq]);
                        const float4 sn = *reinterpret_cast<const float4 *>(&sm.S[tt + 1][i][4 * cq]);
                        const float4 dd = *reinterpret_cast<const float4 *>(&sm.D[tt][i][4 * cq]);
                        const float4 sc = sm.sc[tt][i];   // one 16-byte load for the row's four scalars
                        const float cdy = sc.x, cv = sc.y, csa = sc.z, cds = sc.w;
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
                }
                bool mine = true;   // this CTA writes the columns of quad cq
                if constexpr (CPH > 1) {
                    // partials of the partner's half go to its exchange area; one cluster barrier
                    // (all threads of both CTAs), then the partner's partials of this half are added
                    mine = cq / 16 == rank;
                    if (tt < L && rq == 0 && !mine) {
                        const uint32_t base = tc::map_to_rank(tc::smem_u32(&sm.xb.x[parity][tt][cq % 16][0]), 1 - rank);
#pragma unroll
                        for (int x = 0; x < kGrads; ++x)
                            st_cluster4(base + 16 * x, make_float4(g[x][0], g[x][1], g[x][2], g[x][3]));
                    }
                    tc::cluster_sync();
                    if (tt < L && rq == 0 && mine) {
#pragma unroll
                        for (int x = 0; x < kGrads; ++x) {
                            const float4 o = sm.xb.x[parity][tt][cq % 16][x];
                            g[x][0] += o.x; g[x][1] += o.y; g[x][2] += o.z; g[x][3] += o.w;
                        }
                    }
                    parity ^= 1u;
                }
                if (tt < L && rq == 0 && mine) {
                    const size_t o = tok(t0 + tt) + 4 * cq;
                    const float4 a4 = sm.vec.get4(VA, tt, cq);
                    const float4 kk4 = sm.vec.get4(VKK, tt, cq);
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
    if (p.dS0) store_rows(p.dS0 + size_t(unit) * NN * NN, row0, d);
}

// ---- host side ---------------------------------------------------------------------------------------

template <class Tin, int NN>
cudaError_t launch_bwd_t(const BwdArgs &p) {
    constexpr int CPH = BwdShape<NN>::kCPH;
    const int smem = int(sizeof(BwdSmem<Tin, NN>));
    const cudaError_t attr = allow_dynamic_smem(reinterpret_cast<const void *>(bwd_kernel<Tin, NN>), smem);
    if (attr != cudaSuccess) return attr;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(unsigned(p.B) * unsigned(p.H) * CPH, 1, 1);
    cfg.blockDim = dim3(kBwdThreads, 1, 1);
    cfg.dynamicSmemBytes = size_t(smem);
    cfg.stream = p.stream;
    cudaLaunchAttribute at{};
    at.id = cudaLaunchAttributeClusterDimension;
    at.val.clusterDim.x = CPH;
    at.val.clusterDim.y = 1;
    at.val.clusterDim.z = 1;
    cfg.attrs = &at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, bwd_kernel<Tin, NN>, p);
}

template <int NN>
size_t checkpoint_bytes_t(int B, int T, int H, int snap_every) {
    if (T <= 0) return 0;
    constexpr int kLb = BwdShape<NN>::kLb, CPH = BwdShape<NN>::kCPH;
    const int K = segment_length(T, snap_every);
    return size_t(B) * H * CPH * size_t((K + kLb - 1) / kLb) * kRows * NN * sizeof(float);
}

}  // namespace

size_t backward_checkpoint_bytes_n(int B, int T, int H, int N, int snap_every) {
    return N == 128 ? checkpoint_bytes_t<128>(B, T, H, snap_every) : checkpoint_bytes_t<64>(B, T, H, snap_every);
}

size_t backward_checkpoint_bytes(int B, int T, int H, int snap_every) {
    return backward_checkpoint_bytes_n(B, T, H, kN, snap_every);
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

cudaError_t launch_backward_n(const BwdArgs &p, int N) {
    if (N == 128) return p.dt == WKV7_BF16 ? launch_bwd_t<__nv_bfloat16, 128>(p) : launch_bwd_t<float, 128>(p);
    return p.dt == WKV7_BF16 ? launch_bwd_t<__nv_bfloat16, 64>(p) : launch_bwd_t<float, 64>(p);
}

cudaError_t launch_backward(const BwdArgs &p) { return launch_backward_n(p, kN); }

}  // namespace wkv7
