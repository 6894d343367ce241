// Sequential-scan WKV-7 forward (fp32 FMA), the state-copy kernel for T = 0, and the
// stand-alone group_norm + bonus epilogue used after the scan.
//
// The recurrence (RWKV-7 rebuttal page, numpy time_mixing listing, update and
// readout lines): per (b, h),
//     removed = S_{t-1} kk_t;  S_t = S_{t-1} diag(w_t) - removed (kk_t*a_t)^T + v_t k_t^T;
//     y_t = S_t r_t.
// Every row i of S (one value channel) evolves independently of the other rows:
// row i needs only v_t[i] and the key-side vectors w, kk, a, k, r. The scan
// therefore spreads the 64 rows of one head over CTAs and threads: a CTA owns 16*RPT
// rows of one (b, h); four threads share a row, each holding 16 of its 64 columns
// in registers for the whole sequence. The two dot products per row and token
// (removed value, readout) are reduced with two butterfly shuffles.
//
// Key-side vectors of TB tokens are staged once per CTA in shared memory as fp32
// (b = kk*a precomputed) and read back as broadcast float4; the raw loads of the
// next token block are in flight while the current block is scanned.
#include "common.cuh"

namespace wkv7 {
namespace {

constexpr int kSeqThreads = 64;   // 16 row groups x 4 column quarters

template <class Tin> struct SeqTile;
template <> struct SeqTile<__nv_bfloat16> { static constexpr int TB = 32; };
template <> struct SeqTile<float> { static constexpr int TB = 16; };

// Shared-memory slots of the key-side vectors.
enum { kW = 0, kB = 1, kK = 2, kKK = 3, kR = 4, kSlots = 5 };

template <class Tin, int RPT, int NN>
struct SeqSmem {
    static constexpr int TB = SeqTile<Tin>::TB * 64 / NN;   // the same prefetch registers at any NN
    static constexpr int ROWS = 16 * RPT;
    float vec[kSlots][TB][NN];
    float v[TB][ROWS];
};

// 16 raw bytes -> 4 (fp32) or 8 (bf16) floats.
__device__ __forceinline__ void unpack16(const uint4 &u, const float *, float (&o)[4]) {
    o[0] = __uint_as_float(u.x); o[1] = __uint_as_float(u.y); o[2] = __uint_as_float(u.z); o[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void unpack16(const uint4 &u, const __nv_bfloat16 *, float (&o)[8]) {
    o[0] = bf16_lo(u.x); o[1] = bf16_hi(u.x); o[2] = bf16_lo(u.y); o[3] = bf16_hi(u.y);
    o[4] = bf16_lo(u.z); o[5] = bf16_hi(u.z); o[6] = bf16_lo(u.w); o[7] = bf16_hi(u.w);
}
template <int E>
__device__ __forceinline__ void store_vals(float *dst, const float (&o)[E]) {
#pragma unroll
    for (int j = 0; j < E; j += 4) *reinterpret_cast<float4 *>(dst + j) = make_float4(o[j], o[j + 1], o[j + 2], o[j + 3]);
}

// RAW: w and a hold the decay and rate logits, k the key before its update and kk is not read;
// the staging step turns them into w, b = kk * a, k~ and the unit-norm removal key (rebuttal
// page, the time_mixing listing: decay, learning rate, removal key with its 1e-12 norm floor,
// key update), with the formulas of the chunked kernel's load stage.
template <class Tin, int RPT, bool RAW, int NN>
__global__ void __launch_bounds__(kSeqThreads) seq_kernel(const FwdArgs p) {
    using Sm = SeqSmem<Tin, RPT, NN>;
    constexpr int NM = NN / 16;                           // float4 column groups per thread
    constexpr int TB = Sm::TB, ROWS = Sm::ROWS;
    constexpr int EPC = 16 / sizeof(Tin);                 // elements per 16-byte chunk
    constexpr int CPT = NN / EPC;                         // chunks per token vector
    constexpr int VEC_CH = TB * CPT / kSeqThreads;        // chunks per thread per vector
    constexpr int VCPT = ROWS / EPC;                      // v chunks per token
    constexpr int V_CH = (TB * VCPT + kSeqThreads - 1) / kSeqThreads;
    static_assert(TB * CPT % kSeqThreads == 0, "tile");

    extern __shared__ __align__(16) unsigned char smem_raw[];
    Sm &sm = *reinterpret_cast<Sm *>(smem_raw);

    const int T = p.T, H = p.H;
    const int unit = blockIdx.x, b = unit / H, h = unit % H;
    const int q = threadIdx.x & 3, rg = threadIdx.x >> 2;
    const int row0 = blockIdx.y * ROWS;
    const Tin *src[6] = {static_cast<const Tin *>(p.w), static_cast<const Tin *>(p.kk),
                         static_cast<const Tin *>(p.a), static_cast<const Tin *>(p.k),
                         static_cast<const Tin *>(p.r), static_cast<const Tin *>(p.v)};
    auto tok_off = [&](int t) { return ((size_t(b) * T + t) * H + h) * NN; };

    // state: s[rr][4m + c] = S[row(rr)][4q + 16m + c]
    float s[RPT][4 * NM];
#pragma unroll
    for (int rr = 0; rr < RPT; ++rr) {
        const int row = row0 + rg * RPT + rr;
#pragma unroll
        for (int m = 0; m < NM; ++m) {
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (p.S0) x = __ldg(reinterpret_cast<const float4 *>(p.S0 + (size_t(unit) * NN + row) * NN + 4 * q + 16 * m));
            s[rr][4 * m + 0] = x.x; s[rr][4 * m + 1] = x.y; s[rr][4 * m + 2] = x.z; s[rr][4 * m + 3] = x.w;
        }
    }

    uint4 raw[5][VEC_CH];   // w, kk, a, k, r
    uint4 rawv[V_CH];
    auto issue_loads = [&](int t0) {
#pragma unroll
        for (int x = 0; x < 5; ++x)
#pragma unroll
            for (int i = 0; i < VEC_CH; ++i) {
                if (RAW && x == 1) continue;   // the removal key is derived from k
                const int c = threadIdx.x + kSeqThreads * i, t = c / CPT, e = (c % CPT) * EPC;
                raw[x][i] = t0 + t < T ? __ldg(reinterpret_cast<const uint4 *>(src[x] + tok_off(t0 + t) + e))
                                       : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
        for (int i = 0; i < V_CH; ++i) {
            const int c = threadIdx.x + kSeqThreads * i, t = c / VCPT, e = (c % VCPT) * EPC;
            rawv[i] = (c < TB * VCPT && t0 + t < T)
                          ? __ldg(reinterpret_cast<const uint4 *>(src[5] + tok_off(t0 + t) + row0 + e))
                          : make_uint4(0, 0, 0, 0);
        }
    };
    auto stage = [&]() {
        const Tin *tag = nullptr;
#pragma unroll
        for (int i = 0; i < VEC_CH; ++i) {
            const int c = threadIdx.x + kSeqThreads * i, t = c / CPT, e = (c % CPT) * EPC;
            float w_[EPC], kk_[EPC], a_[EPC], k_[EPC], r_[EPC], b_[EPC];
            unpack16(raw[0][i], tag, w_);
            unpack16(raw[2][i], tag, a_);
            unpack16(raw[3][i], tag, k_);
            unpack16(raw[4][i], tag, r_);
            if (RAW) {
                // the CPT consecutive threads that hold one token reduce ||k * k_k|| by shuffles
                const float *kk_p = p.k_k + h * NN + e, *ka_p = p.k_a ? p.k_a + h * NN + e : nullptr;
                float ss = 0.f;
#pragma unroll
                for (int j = 0; j < EPC; ++j) {
                    w_[j] = __expf(-0.60653065971263342f / (1.f + __expf(-w_[j])));   // e^-1/2 = 1/sqrt(e)
                    a_[j] = 1.f / (1.f + __expf(-a_[j]));
                    kk_[j] = k_[j] * __ldg(kk_p + j);
                    ss = fmaf(kk_[j], kk_[j], ss);
                    if (ka_p) k_[j] = fmaf(k_[j] * (a_[j] - 1.f), __ldg(ka_p + j), k_[j]);
                }
#pragma unroll
                for (int o = 1; o < CPT; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
                const float inv = 1.f / fmaxf(sqrtf(ss), 1e-12f);
#pragma unroll
                for (int j = 0; j < EPC; ++j) kk_[j] *= inv;
            } else {
                unpack16(raw[1][i], tag, kk_);
            }
#pragma unroll
            for (int j = 0; j < EPC; ++j) b_[j] = kk_[j] * a_[j];
            store_vals(&sm.vec[kW][t][e], w_);
            store_vals(&sm.vec[kKK][t][e], kk_);
            store_vals(&sm.vec[kB][t][e], b_);
            store_vals(&sm.vec[kK][t][e], k_);
            store_vals(&sm.vec[kR][t][e], r_);
        }
#pragma unroll
        for (int i = 0; i < V_CH; ++i) {
            const int c = threadIdx.x + kSeqThreads * i, t = c / VCPT, e = (c % VCPT) * EPC;
            float v_[EPC];
            unpack16(rawv[i], tag, v_);
            if (c < TB * VCPT) store_vals(&sm.v[t][e], v_);
        }
    };

    const int n_snap = p.snap_every > 0 ? T / p.snap_every : 0;
    issue_loads(0);
    for (int t0 = 0; t0 < T; t0 += TB) {
        __syncthreads();            // previous block fully consumed
        stage();
        __syncthreads();
        if (t0 + TB < T) issue_loads(t0 + TB);
        const int tn = min(TB, T - t0);
        // Two rows per thread: two tokens per loop pass let the next token's loads start early
        // (measured faster); one row per thread: faster rolled.
#pragma unroll (RPT)
        for (int t = 0; t < tn; ++t) {
            float4 kk4[NM];
#pragma unroll
            for (int m = 0; m < NM; ++m) kk4[m] = reinterpret_cast<const float4 *>(&sm.vec[kKK][t][0])[q + 4 * m];
            float sk[RPT];
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) {
                float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
                for (int m = 0; m < NM; m += 2) {
                    acc0 = fmaf(s[rr][4 * m + 0], kk4[m].x, acc0);
                    acc0 = fmaf(s[rr][4 * m + 1], kk4[m].y, acc0);
                    acc0 = fmaf(s[rr][4 * m + 2], kk4[m].z, acc0);
                    acc0 = fmaf(s[rr][4 * m + 3], kk4[m].w, acc0);
                    acc1 = fmaf(s[rr][4 * m + 4], kk4[m + 1].x, acc1);
                    acc1 = fmaf(s[rr][4 * m + 5], kk4[m + 1].y, acc1);
                    acc1 = fmaf(s[rr][4 * m + 6], kk4[m + 1].z, acc1);
                    acc1 = fmaf(s[rr][4 * m + 7], kk4[m + 1].w, acc1);
                }
                sk[rr] = acc0 + acc1;
            }
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) {
                sk[rr] += __shfl_xor_sync(0xffffffffu, sk[rr], 1);
                sk[rr] += __shfl_xor_sync(0xffffffffu, sk[rr], 2);
            }
            float yv[RPT];
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) yv[rr] = 0.f;
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                const float4 w4 = reinterpret_cast<const float4 *>(&sm.vec[kW][t][0])[q + 4 * m];
                const float4 b4 = reinterpret_cast<const float4 *>(&sm.vec[kB][t][0])[q + 4 * m];
                const float4 k4 = reinterpret_cast<const float4 *>(&sm.vec[kK][t][0])[q + 4 * m];
                const float4 r4 = reinterpret_cast<const float4 *>(&sm.vec[kR][t][0])[q + 4 * m];
                const float wv[4] = {w4.x, w4.y, w4.z, w4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
                const float kv[4] = {k4.x, k4.y, k4.z, k4.w}, rv[4] = {r4.x, r4.y, r4.z, r4.w};
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr) {
                    const float vi = sm.v[t][rg * RPT + rr];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        float x = s[rr][4 * m + c] * wv[c];
                        x = fmaf(-sk[rr], bv[c], x);
                        x = fmaf(vi, kv[c], x);
                        s[rr][4 * m + c] = x;
                        yv[rr] = fmaf(x, rv[c], yv[rr]);
                    }
                }
            }
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) {
                yv[rr] += __shfl_xor_sync(0xffffffffu, yv[rr], 1);
                yv[rr] += __shfl_xor_sync(0xffffffffu, yv[rr], 2);
                if (q == 0) p.y[tok_off(t0 + t) + row0 + rg * RPT + rr] = yv[rr];
            }
            const int tt = t0 + t + 1;
            if (n_snap && tt % p.snap_every == 0) {
                const int m_idx = tt / p.snap_every - 1;
                float *dst = p.snaps + (((size_t(b) * n_snap + m_idx) * H + h) * NN) * NN;
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
                    for (int m = 0; m < NM; ++m)
                        *reinterpret_cast<float4 *>(dst + (row0 + rg * RPT + rr) * NN + 4 * q + 16 * m) =
                            make_float4(s[rr][4 * m], s[rr][4 * m + 1], s[rr][4 * m + 2], s[rr][4 * m + 3]);
            }
        }
    }
    if (p.S_T) {
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
            for (int m = 0; m < NM; ++m)
                *reinterpret_cast<float4 *>(p.S_T + (size_t(unit) * NN + row0 + rg * RPT + rr) * NN + 4 * q + 16 * m) =
                    make_float4(s[rr][4 * m], s[rr][4 * m + 1], s[rr][4 * m + 2], s[rr][4 * m + 3]);
    }
}

// ---- host side ---------------------------------------------------------------------------------------

template <class Tin, int RPT, bool RAW, int NN>
cudaError_t launch_seq_t(const FwdArgs &p) {
    const size_t smem = sizeof(SeqSmem<Tin, RPT, NN>);
    const cudaError_t attr =
        allow_dynamic_smem(reinterpret_cast<const void *>(seq_kernel<Tin, RPT, RAW, NN>), int(smem));
    if (attr != cudaSuccess) return attr;
    dim3 grid(p.B * p.H, NN / (16 * RPT));
    seq_kernel<Tin, RPT, RAW, NN><<<grid, kSeqThreads, smem, p.stream>>>(p);
    return cudaGetLastError();
}

template <class Tin, int RPT>
cudaError_t launch_seq_r(const FwdArgs &p) {
    if constexpr (RPT <= 2) {   // four rows of 32 columns would not fit the registers at N = 128
        if (p.N == 128)
            return p.raw ? launch_seq_t<Tin, RPT, true, 128>(p) : launch_seq_t<Tin, RPT, false, 128>(p);
    }
    return p.raw ? launch_seq_t<Tin, RPT, true, 64>(p) : launch_seq_t<Tin, RPT, false, 64>(p);
}

// ---- T = 0: S_T <- S0 (or zeros) -------------------------------------------------------------
__global__ void copy_state_kernel(const float4 *__restrict__ src, float4 *__restrict__ dst, size_t n4) {
    for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < n4; i += size_t(gridDim.x) * blockDim.x)
        dst[i] = src ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
}

// ---- group_norm + bonus epilogue (one warp per (b, t, h) row of NN channels) ----------------
// RAW: k is the key before its update and a the rate logit; the bonus uses k~ = k + k (a-1) k_a.
template <class Tin, bool RAW, int NN>
__global__ void __launch_bounds__(256) epilogue_kernel(const FwdArgs p, size_t rows) {
    constexpr int E = NN / 32;   // channels per lane
    const size_t row = blockIdx.x * size_t(8) + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31, h = int(row % p.H);
    const size_t base = row * NN + E * lane;
    const int pc = h * NN + E * lane;
    const Tin *r = static_cast<const Tin *>(p.r), *k = static_cast<const Tin *>(p.k), *v = static_cast<const Tin *>(p.v);
    float yv[E], bon = 0.f, sum = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        yv[e] = p.y[base + e];
        float ke = load1(k + base + e);
        if (RAW && p.k_a) {
            const float ae = 1.f / (1.f + __expf(-load1(static_cast<const Tin *>(p.a) + base + e)));
            ke = fmaf(ke * (ae - 1.f), p.k_a[pc + e], ke);
        }
        bon = fmaf(load1(r + base + e) * ke, p.r_k[pc + e], bon);
        sum += yv[e];
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
        bon += __shfl_xor_sync(0xffffffffu, bon, o);
    }
    const float mean = sum * (1.f / NN);
    float sq = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        yv[e] -= mean;
        sq = fmaf(yv[e], yv[e], sq);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    const float inv = 1.f / sqrtf(sq * (1.f / NN) + p.gn_eps);
#pragma unroll
    for (int e = 0; e < E; ++e)
        p.y[base + e] = yv[e] * inv * p.ln_w[pc + e] + p.ln_b[pc + e] + bon * load1(v + base + e);
}

}  // namespace

cudaError_t launch_seq(const FwdArgs &p) {
    // Rows per thread (a CTA holds 16 of them per thread): more rows let each token-vector read
    // serve more rows, fewer give a head more CTAs and an SM more warps. Measured at N = 64,
    // B8 T1024: 96 heads one row 0.389 ms against two 0.401; 128 heads two rows 0.395 against
    // four 0.414; 160 heads four rows 0.414 against two 0.467 and 512 heads (T4096) 2.61 against
    // 4.08 ms, from the head count at which one CTA per head fills the 148 SMs. N = 128 takes two
    // rows (0.59 against 0.69 ms at 48 heads; four would spill).
    const size_t heads = size_t(p.B) * p.H;
    const int rpt = p.N == 128 ? 2 : heads >= 148 ? 4 : heads >= 128 ? 2 : 1;
    if (p.dt == WKV7_BF16)
        return rpt == 4 ? launch_seq_r<__nv_bfloat16, 4>(p)
                        : rpt == 2 ? launch_seq_r<__nv_bfloat16, 2>(p) : launch_seq_r<__nv_bfloat16, 1>(p);
    return rpt == 4 ? launch_seq_r<float, 4>(p) : rpt == 2 ? launch_seq_r<float, 2>(p) : launch_seq_r<float, 1>(p);
}

cudaError_t launch_copy_state(const FwdArgs &p) {
    const size_t n4 = size_t(p.B) * p.H * p.N * p.N / 4;
    const int blocks = int(std::min<size_t>((n4 + 255) / 256, 148 * 8));
    copy_state_kernel<<<blocks, 256, 0, p.stream>>>(reinterpret_cast<const float4 *>(p.S0),
                                                    reinterpret_cast<float4 *>(p.S_T), n4);
    return cudaGetLastError();
}

template <class Tin, bool RAW>
void launch_epilogue_t(const FwdArgs &p, size_t rows, unsigned blocks) {
    if (p.N == 128)
        epilogue_kernel<Tin, RAW, 128><<<blocks, 256, 0, p.stream>>>(p, rows);
    else
        epilogue_kernel<Tin, RAW, 64><<<blocks, 256, 0, p.stream>>>(p, rows);
}

cudaError_t launch_epilogue(const FwdArgs &p) {
    const size_t rows = size_t(p.B) * p.T * p.H;
    const unsigned blocks = unsigned((rows + 7) / 8);
    if (p.dt == WKV7_BF16) {
        if (p.raw) launch_epilogue_t<__nv_bfloat16, true>(p, rows, blocks);
        else launch_epilogue_t<__nv_bfloat16, false>(p, rows, blocks);
    } else {
        if (p.raw) launch_epilogue_t<float, true>(p, rows, blocks);
        else launch_epilogue_t<float, false>(p, rows, blocks);
    }
    return cudaGetLastError();
}

}  // namespace wkv7
