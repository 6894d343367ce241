// Chunked WKV-7 prefill on tcgen05 tensor cores (tf32 operands, fp32 accumulation),
// with the state carried from chunk to chunk in fp32.
//
// The recurrence (RWKV-7 rebuttal page, numpy time_mixing listing, update and
// readout lines; the paper summary, section 4: the transition is a diagonal matrix plus a
// rank-one one, so products over time can be formed in parallel) is, per (b, h),
//     S_t = S_{t-1} diag(w_t) + u_t b_t^T + v_t k_t^T,  u_t = -S_{t-1} kk_t,  b_t = kk_t*a_t,
//     y_t = S_t r_t.
// Over a chunk of C tokens with start state S_0, let g_t = prod_{s<=t} w_s (per key
// channel, g_{-1} = 1) and gC = g_{C-1}. Unrolling gives (rows of the C x N matrices
// are tokens; the derivation is this file's own, the pages give no chunk formula):
//     KKd = kk*g_{t-1}, Rd = r*g_t, Bi = b/g_s, Ki = k/g_s, Bc = b*gC/g_s, Kc = k*gC/g_s
//     M_ab = tril(KKd Bi^T, -1), M_kb = tril(KKd Ki^T, -1), Q_b = tril(Rd Bi^T), Q_k = tril(Rd Ki^T)
//     A = (I + M_ab)^{-1}                              (the removed values U = A(-KKd S_0^T - M_kb V))
//     [Z] = [Bi^T; Q_b] A,   [X] = Z [KKd | M_kb]
//     P  = diag(gC) (I - Bi^T A KKd)      R~ = Rd  - Q_b A KKd
//     K~ = diag(gC) (Ki^T - Bi^T A M_kb)  Q~ = Q_k - Q_b A M_kb
// (Bc = Bi*gC and Kc = Ki*gC column-wise, so gC is applied once, per key row of P and K~.)
//     [S_C^T; Y] = [P; R~] S_0^T + [K~; Q~] V
// Only the last line depends on the state, so the chain from chunk to chunk is one
// fused M=128 MMA; everything else is computed from the chunk's own inputs.
//
// Mapping onto one B200 SM (one CTA per SM, persistent over (b, h) heads):
//  * TMA (no multicast) stages the six bf16 [64 x 64] input tiles of the next chunk
//    (128-byte swizzle) while the current chunk is processed.
//  * Every MMA is tcgen05.mma kind::tf32, M=128, with the A operand in tensor memory
//    (lane = row) or shared memory and the B operand in shared memory (K-major, 128-byte
//    swizzle); rounds that share an A operand are merged into N = 128.
//  * 512 threads = 16 warps. A warp reaches only its quarter (warp % 4) of the TMEM lanes:
//    lanes 0-63 hold key channels or the first 64 rows, lanes 64-127 tokens.
//  * Software pipeline over the CTA's chunks. After chunk c's inverse, warps 0-3 run the
//    dependent MMA rounds of chunk c and its output (state, y, epilogue) while warps 4-15
//    wait for chunk c+1's tiles and compute its decay products and scaled operands
//    (shared memory only). Everything that writes tensor memory waits for the join.
//  * The unit-lower-triangular inverse: 16x16 diagonal blocks and one merge level on the
//    CUDA cores in fp32, the merge of the two 32x32 halves on the tensor core.
//  * Operands are rounded to tf32 (round to nearest) before the tensor core sees them;
//    the carried state, the accumulators and all element-wise work stay fp32.
// Every wait is bounded; a wait that gives up sets the device error word, the CTA
// drains what it issued (bounded), frees its tensor memory and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "tc_util.cuh"

namespace wkv7 {

__device__ unsigned int g_device_error;   // non-zero: a bounded wait in a kernel gave up

namespace {

using namespace tc;

constexpr int C = 64;             // chunk length (tokens)
constexpr int kThreads = 512;     // 16 warps
constexpr int kBackThreads = 128; // warps 0-3: MMA rounds after the inverse, and the output
constexpr int kFrontThreads = kThreads - kBackThreads;   // warps 4-15: the next chunk's operands
constexpr int kSendThreads = 256; // split mode: the 8 warps of TMEM lanes 0-63 write the next CTA's state
constexpr int kMaxSegments = WKV7_MAX_SEGMENTS;   // CTAs per (b, h) in split mode (portable cluster size)
constexpr int GTS = 68;           // row stride (floats) of the decay table
constexpr int LWS = 68;           // row stride of the inverse workspaces (16-byte aligned rows)
constexpr int BAR_BACK = 1, BAR_FRONT = 2, BAR_ROWS = 3;   // named barriers: warps 0-3, 4-15, TMEM lanes 64-127

// Shared-memory layout (byte offsets from a 1024-byte aligned base).
constexpr uint32_t OFF_B1 = 0;        // [Bi; Ki] 128x64 tf32 (B of R1 and of the transpose round); then the
                                      // inverse workspace
constexpr uint32_t OFF_B3 = 32768;    // [M_kb^T; KKd^T] 128x64 (B of R3)
constexpr uint32_t OFF_B2 = 65536;    // A^T 64x64 (B of R2); after R2, the y tile of the TMA store
                                      // (2 x [64][32] fp32), stored during the next chunk's R1
constexpr uint32_t OFF_B4 = 81920;    // V^T 64x64 (B of R4; exact bf16 values)
constexpr uint32_t OFF_B5 = 98304;    // S 64x64, row = value channel (B of R5)
constexpr uint32_t OFF_A1 = 114688;   // [KKd; Rd] 128x64 (A of R1)
constexpr uint32_t OFF_IN = 147456;   // six bf16 [64][64] input tiles, TMA destination (swizzled)
constexpr uint32_t OFF_GT = 196608;   // decay table [65][GTS] fp32; later the inverse [64][LWS]
constexpr uint32_t OFF_L21 = (OFF_GT + 65 * GTS * 4 + 1023) & ~1023u;   // L21^T 32x32 (B of R2b)
constexpr uint32_t OFF_SMALL = OFF_L21 + 4096;

struct Small {
    float gC[2][C];           // decay over the chunk per key channel, by chunk parity
    float tq[4][C];           // decay product over each quarter of the chunk
    float bon[2][C];          // epilogue bonus r_t . (k_t * r_k) per token, by chunk parity
    float red[4][C];          // epilogue: partial sums over the four column parts of each y row
    float dk[C];              // r_t . k_t (exact current-token Gram entry)
    float db[C];              // r_t . (kk_t * a_t)
    float ln_w[2][C], ln_b[2][C], r_k[2][C];   // epilogue parameters, by head parity
    float k_k[2][C], k_a[2][C];                 // raw inputs: removal-key scale, key-update rate
    float inv_norm[C];                          // raw inputs: 1 / max(||k_t * k_k||, 1e-12) per token
    uint64_t bar_tma;
    uint64_t bar_mma;
    uint64_t bar_state;       // split mode: the carried state has arrived in B5 (kSendThreads arrivals)
    uint64_t bar_credit;      // split mode: the next CTA has consumed the state last sent to it
    uint32_t tmem_base;
};
constexpr uint32_t SMEM_BYTES = OFF_SMALL + sizeof(Small) + 1024;   // + alignment slack
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

// TMEM columns (512 allocated). A tf32 MMA with N = 64 costs nearly as much issue time as one
// with N = 128, so products that share an A operand are merged into N = 128 rounds.
constexpr uint32_t T_D1 = 0;     // Grams [M_ab | M_kb ; Q_b | Q_k] (R1); once read, Z (R2, 64 columns)
constexpr uint32_t T_A2 = 128;   // A of R2: [Bi^T (transpose round); Q_b]
constexpr uint32_t T_D3R = 192;  // [Ki^T (transpose round); Q_k] -> R3 subtracts Z M_kb -> [K~; Q~] (A of R4)
constexpr uint32_t T_D3L = 256;  // [I; Rd] -> R3 subtracts Z KKd -> [I - X; R~] (A of R5)
constexpr uint32_t T_D4 = 320;   // [S'^T; Y] (R4 + R5); the new state is diag(gC) S'^T
constexpr uint32_t T_V = 384;    // R2b: U[:, 32:64] L21 (32 columns)
constexpr uint32_t T_ID = 448;   // identity (lanes 0-63) over zeros: A of the transpose round, written once
static_assert(T_A2 + 64 == T_D3R && T_D3R + 64 == T_D3L, "transpose round and R3 write adjacent blocks");

enum { XR = 0, XW = 1, XK = 2, XV = 3, XKK = 4, XA = 5 };

struct ChunkMaps {
    CUtensorMap m[6];     // inputs r, w, k, v, kk, a: bf16 [B][T][H][64], box 64 tokens x 64 channels
    CUtensorMap y;        // output y: fp32 [B][T][H][64], box 64 tokens x 32 channels
};
constexpr int kStoreThread = 32;   // issues and completes the TMA stores of y (lane 0 of warp 1)

// y tile of one chunk (in B2) -> global through the y tensor map; the two channel halves.
__device__ __forceinline__ void store_y_tile(const ChunkMaps &maps, const uint8_t *tile, int hh, int c0, int b) {
    tma_store_4d(&maps.y, tile, 0, hh, c0, b);
    tma_store_4d(&maps.y, tile + 8192, 32, hh, c0, b);
    tma_store_commit();
}

struct ChunkArgs {
    int B, T, H;
    int unit0, unit_end;      // the heads (b * H + h) of this launch: [unit0, unit_end)
    const float *S0;
    float *S_T, *snaps;
    int snap_every, n_snap;
    const float *ln_w, *ln_b, *r_k;
    float gn_eps;
    const float *k_k, *k_a;   // raw inputs: the removal-key scale and the key-update rate ([H][64]; k_a nullable)
    unsigned int *err;
    unsigned long long timeout_ns;           // every bounded wait but the split-mode hand-off
    unsigned long long handoff_timeout_ns;   // split mode: waits for a state and for its receipt
    int withhold_handoff;     // failure-path test: CTA 0 of each cluster does not send its first state
};

// bf16 element (t, j) of a 128-byte-swizzled [64][64] tile.
__device__ __forceinline__ float in_elem(const uint8_t *tile, int t, int j) {
    const uint32_t off = t * 128 + ((((j >> 3) ^ (t & 7))) << 4) + ((j & 7) << 1);
    return __uint_as_float(uint32_t(*reinterpret_cast<const uint16_t *>(tile + off)) << 16);
}
// Byte offsets, within a token row, of key channel j in a 128-byte-swizzled bf16 tile, for
// the eight row phases t % 8 (hoisted out of column walks).
__device__ __forceinline__ void col_offsets(int j, uint32_t (&xo)[8]) {
#pragma unroll
    for (int e = 0; e < 8; ++e) xo[e] = ((((j >> 3) ^ e)) << 4) + ((j & 7) << 1);
}
__device__ __forceinline__ float in_col(const uint8_t *tile, int t, const uint32_t (&xo)[8], int e) {
    return __uint_as_float(uint32_t(*reinterpret_cast<const uint16_t *>(tile + t * 128 + xo[e])) << 16);
}
// Byte offsets of column k of a K-major swizzled tf32 tile with `rows` rows, for the eight
// row phases r % 8: element (r0 + e, k) with r0 a multiple of 8 is at r0 * 128 + e * 128 + xo[e].
__device__ __forceinline__ void kcol_offsets(int k, int rows, uint32_t (&xo)[8]) {
    const int kb = k >> 5, kk = k & 31;
#pragma unroll
    for (int e = 0; e < 8; ++e) xo[e] = uint32_t(kb * rows * 128 + ((((kk >> 2) ^ e)) << 4) + ((kk & 3) << 2));
}
// Eight bf16 elements (t, j..j+7), j a multiple of 8.
__device__ __forceinline__ void in_row8(const uint8_t *tile, int t, int j, float (&o)[8]) {
    const uint32_t off = t * 128 + ((((j >> 3) ^ (t & 7))) << 4);
    const uint4 u = *reinterpret_cast<const uint4 *>(tile + off);
    o[0] = bf16_lo(u.x); o[1] = bf16_hi(u.x); o[2] = bf16_lo(u.y); o[3] = bf16_hi(u.y);
    o[4] = bf16_lo(u.z); o[5] = bf16_hi(u.z); o[6] = bf16_lo(u.w); o[7] = bf16_hi(u.w);
}
__device__ __forceinline__ void st_f4(uint8_t *base, uint32_t off, float a, float b, float c, float d) {
    *reinterpret_cast<float4 *>(base + off) = make_float4(a, b, c, d);
}
__device__ __forceinline__ void bar_named(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }
// Named barrier that also ORs a predicate over its participants (the result is uniform).
__device__ __forceinline__ bool bar_named_or(int id, int n, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(uint32_t(v)), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// RAW: the inputs are the pages' time-mixing values before their pre-processing (the decay and
// rate logits, the raw key, the per-head removal-key scale k_k and key-update rate k_a); the
// load stage computes w = exp(-sigmoid(w_logit) / sqrt(e)), a = sigmoid(a_logit),
// kk = (k * k_k) / max(||k * k_k||, 1e-12) and k~ = k + k (a - 1) k_a (rebuttal page, the
// time_mixing listing) in fp32. Otherwise the inputs are r, w, k~, v, kk, a themselves.
template <bool RAW>
__global__ void __launch_bounds__(kThreads, 1) chunk_kernel(const __grid_constant__ ChunkMaps maps, const ChunkArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = smem_raw + (((smem_u32(smem_raw) + 1023u) & ~1023u) - smem_u32(smem_raw));
    Small &S = *reinterpret_cast<Small *>(sm + OFF_SMALL);
    const uint8_t *IN = sm + OFF_IN;
    float *GT = reinterpret_cast<float *>(sm + OFF_GT);
    float *Lw = reinterpret_cast<float *>(sm + OFF_B1);      // strictly lower M_ab [64][LWS]
    float *Tw = Lw + 64 * LWS;                               // level-1 temps [2][16][20]
    float *Aw = reinterpret_cast<float *>(sm + OFF_GT);      // inverse [64][LWS]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Lq = (warp & 3) * 32;         // first TMEM lane of this warp's quarter
    const int L = Lq + lane;                // this thread's TMEM lane
    const int pq = warp >> 2;               // which 16-wide part of the 64 columns / tokens
    const int c16 = 16 * pq;
    const bool colg = L < 64;
    const bool back = warp < 4;             // warps 0-3: one per TMEM lane quarter
    const int ft = tid - kBackThreads;      // index among the front warps 4-15
    const int units = p.unit_end;
    const int nchunks = (p.T + C - 1) / C;
    const bool epi = p.ln_w != nullptr;

    // Split mode: the CTAs of a cluster share each (b, h); CTA `rank` takes chunks rank,
    // rank + cs, ... and hands the state after each of them to CTA rank + 1 (mod cs).
    const int cs = int(cluster_size()), rank = int(cluster_rank());
    const int cid = int(cluster_index()), ncl = int(cluster_count());
    if (tid < 7) asm volatile("prefetch.tensormap [%0];" ::"l"(tid < 6 ? &maps.m[tid] : &maps.y) : "memory");
    if (tid == 0) {
        mbar_init(&S.bar_tma, 1);
        mbar_init(&S.bar_mma, 1);
        mbar_init(&S.bar_state, kSendThreads);
        mbar_init(&S.bar_credit, 1);
        mbar_fence_init();
    }
    if (warp == 0) {
        tmem_alloc(&S.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    if (cs > 1) cluster_sync();   // every CTA's barriers are initialised before anyone arrives remotely
    tc_fence_after();
    const uint32_t tb = S.tmem_base;
    const int next_rank = rank + 1 == cs ? 0 : rank + 1, prev_rank = rank == 0 ? cs - 1 : rank - 1;
    const uint32_t next_b5 = map_to_rank(smem_u32(sm + OFF_B5), uint32_t(next_rank));
    const uint32_t own_b5 = map_to_rank(smem_u32(sm + OFF_B5), uint32_t(rank));
    const uint32_t next_bar = map_to_rank(smem_u32(&S.bar_state), uint32_t(next_rank));
    const uint32_t prev_credit = map_to_rank(smem_u32(&S.bar_credit), uint32_t(prev_rank));
    // matrix descriptors of the shared-memory operands at K-step 0
    const uint64_t dB1 = desc_sw128(smem_u32(sm + OFF_B1)), dB2 = desc_sw128(smem_u32(sm + OFF_B2));
    const uint64_t dB3 = desc_sw128(smem_u32(sm + OFF_B3)), dB4 = desc_sw128(smem_u32(sm + OFF_B4));
    const uint64_t dB5 = desc_sw128(smem_u32(sm + OFF_B5)), dA1 = desc_sw128(smem_u32(sm + OFF_A1));
    const uint64_t dL21 = desc_sw128(smem_u32(sm + OFF_L21));
    {   // identity over zeros in T_ID (A operand of the transposes; never overwritten)
        float id8[8];
#pragma unroll 1
        for (int g = 0; g < 2; ++g) {
            const int c8 = c16 + 8 * g;
#pragma unroll
            for (int e = 0; e < 8; ++e) id8[e] = (c8 + e == L) ? 1.f : 0.f;
            tmem_st8(tmem_addr(tb, Lq, T_ID + c8), id8);
        }
        tmem_st_wait();
    }
    uint32_t tma_parity = 0, mma_parity = 0, state_parity = 0, credit_parity = 0;
    int sends = 0;                     // states sent to the next CTA (warps 0-1)
    bool y_pending = false;            // the y tile in B2 still has to be stored (uniform)
    int y_h = 0, y_c0 = 0, y_b = 0;    // its coordinates
    bool tma_pending = false, mma_pending = false, failed = false;

    constexpr uint32_t kTileBytes = (RAW ? 5 : 6) * 8192;   // RAW has no kk tile
    auto issue_tma = [&](int u, int c) {   // one thread: the input tiles of chunk c of head u
        const int b = u / p.H, hh = u % p.H;
        mbar_arrive_expect_tx(&S.bar_tma, kTileBytes);
#pragma unroll
        for (int x = 0; x < 6; ++x)
            if (!(RAW && x == XKK)) tma_load_4d(sm + OFF_IN + x * 8192, &maps.m[x], &S.bar_tma, 0, hh, c * C, b);
    };
    // Waits: one thread polls the mbarrier (bounded, acquire) and the others wait in a hardware
    // barrier with it; many polling threads would crowd the shared-memory pipe that the other
    // warp group is using. All threads; true on timeout (uniform across the CTA).
    // On a timeout the issuing thread keeps the parity of the phase that did not complete and
    // stays `mma_pending`, so the drain on the way out waits (bounded) for that phase.
    auto wait_mma_all = [&]() -> bool {
        const bool to = tid == 0 && !mbar_wait_spin(&S.bar_mma, mma_parity, p.timeout_ns);
        if (!to) mma_parity ^= 1u;
        mma_pending = to;
        const bool f = __syncthreads_or(to) != 0;
        tc_fence_after();
        return f;
    };
    // warps 0-3 only; true on timeout here or (`extra`) in any of them
    auto wait_mma_back = [&](bool extra) -> bool {
        const bool to = tid == 0 && !mbar_wait_spin(&S.bar_mma, mma_parity, p.timeout_ns);
        if (!to) mma_parity ^= 1u;
        const bool f = bar_named_or(BAR_BACK, kBackThreads, to || extra);
        tc_fence_after();
        mma_pending = to;   // a round that did not complete may still be running: drain it before exit
        return f;
    };
    auto sync_for_mma = [&]() {            // writes to smem/TMEM -> visible to the next MMA
        fence_proxy_async_smem();
        tmem_st_wait();
        tc_fence_before();
        __syncthreads();
    };
    auto load_params = [&](int u, int slot, int i) {   // per-head parameters of head u, element i
        const int hh = u % p.H;
        S.ln_w[slot][i] = epi ? p.ln_w[hh * 64 + i] : 1.f;
        S.ln_b[slot][i] = epi ? p.ln_b[hh * 64 + i] : 0.f;
        S.r_k[slot][i] = epi ? p.r_k[hh * 64 + i] : 0.f;
        if (RAW) {
            S.k_k[slot][i] = p.k_k[hh * 64 + i];
            S.k_a[slot][i] = p.k_a ? p.k_a[hh * 64 + i] : 0.f;
        }
    };
    auto load_state = [&](int u) {   // all threads: S_0 of head u (or zeros) -> B5, tf32, row = value channel
        for (int e = tid; e < 1024; e += kThreads) {
            const int i = e >> 4, j4 = (e & 15) * 4;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (p.S0) x = __ldg(reinterpret_cast<const float4 *>(p.S0 + size_t(u) * 4096 + i * 64 + j4));
            st_f4(sm + OFF_B5, sw128_off(i, j4, 64), to_tf32(x.x), to_tf32(x.y), to_tf32(x.z), to_tf32(x.w));
        }
    };

    // ---- front: the operands of chunk c of head u (warps 4-15, shared memory only): decay
    //      products g_t (table GT, gC[ip]), KKd, Rd -> A1; Bi, Ki -> B1; exact current-token Grams.
    //      Returns true (uniform over the front warps) if the input tiles did not arrive.
    auto front = [&](int u, int c, int ip, int us) -> bool {
        const int Lc = min(C, p.T - c * C);
        const bool to = ft == 0 && !mbar_wait_spin(&S.bar_tma, tma_parity, p.timeout_ns);
        tma_parity ^= 1u;
        if (bar_named_or(BAR_FRONT, kFrontThreads, to)) return true;
        if (RAW) {
            // P0: the decay multipliers w = exp(-sigmoid(z)/sqrt(e)) of the whole tile into the decay
            //     table's rows, four channels per item over all front threads (independent items,
            //     so the transcendental latencies overlap), before the products run over them
            for (int it = ft; it < C * 16; it += kFrontThreads) {
                const int t = it >> 4, j0 = (it & 15) * 4;
                const uint2 u = *reinterpret_cast<const uint2 *>(IN + XW * 8192 + t * 128 +
                                                                 ((((j0 >> 3) ^ (t & 7))) << 4) + (j0 & 4) * 2);
                const float z[4] = {bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y)};
                float wv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) wv[e] = __expf(__fdividef(-0.60653065971263342f, 1.f + __expf(-z[e])));
                *reinterpret_cast<float4 *>(GT + (t + 1) * GTS + j0) = make_float4(wv[0], wv[1], wv[2], wv[3]);
            }
            bar_named(BAR_FRONT, kFrontThreads);
        }
        // P1: decay products per key channel j over each quarter of the chunk (256 threads)
        if (ft < 256) {
            const int j = ft & 63, q = ft >> 6;
            const uint8_t *wt = IN + XW * 8192;
            uint32_t xo[8];
            col_offsets(j, xo);
            float run = 1.f;
#pragma unroll 1
            for (int h8 = 0; h8 < 2; ++h8) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int t = 16 * q + 8 * h8 + e;
                    const float w = RAW ? GT[(t + 1) * GTS + j] : in_col(wt, t, xo, e);
                    run *= (t < Lc) ? w : 1.f;   // padded tokens: w = 1
                    GT[(t + 1) * GTS + j] = run;
                }
            }
            S.tq[q][j] = run;
        }
        bar_named(BAR_FRONT, kFrontThreads);
        // P2: absolute products g_t (the quarters before this one as prefix)
        if (ft < 256) {
            const int j = ft & 63, q = ft >> 6;
            if (q > 0) {
                float pre = 1.f;
                for (int qq = 0; qq < q; ++qq) pre *= S.tq[qq][j];
#pragma unroll
                for (int e = 0; e < 16; ++e) GT[(16 * q + e + 1) * GTS + j] *= pre;
            } else {
                GT[j] = 1.f;
                S.gC[ip][j] = S.tq[0][j] * S.tq[1][j] * S.tq[2][j] * S.tq[3][j];
            }
            if (RAW) {   // removal-key norms: four threads per token, sixteen channels each
                const int t = ft >> 2, j0 = 16 * (ft & 3);
                float k8[8], ss = 0.f;
#pragma unroll
                for (int hlf = 0; hlf < 2; ++hlf) {
                    in_row8(IN + XK * 8192, t, j0 + 8 * hlf, k8);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float x = k8[e] * S.k_k[us][j0 + 8 * hlf + e];
                        ss = fmaf(x, x, ss);
                    }
                }
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                ss += __shfl_xor_sync(0xffffffffu, ss, 2);
                if ((ft & 3) == 0) S.inv_norm[t] = rsqrtf(fmaxf(ss, 1e-24f));   // 1 / max(||.||, 1e-12)
            }
        }
        bar_named(BAR_FRONT, kFrontThreads);
        // P3: one (token t, channel octet o) per thread and pass. In a quarter-warp, token t takes
        //     octets 0-3 and token t+1 octets 4-7 (or the reverse), so the swizzled bf16 reads, the
        //     decay-table rows and the tf32 stores of the eight lanes all fall on distinct banks.
        const int fw = ft >> 5, half = lane >> 4, qa = (lane >> 3) & 1, s8 = lane & 7;
        const int hi = s8 >> 2, sub = s8 & 3;
        const int j0 = 8 * (sub + 4 * (qa ^ hi));
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
            const int tbase = 4 * (fw + 12 * pass);
            if (tbase >= C) break;   // warp-uniform
            const int t = tbase + 2 * half + hi;
            float r8[8], kk8[8], k8[8], a8[8];
            in_row8(IN + XR * 8192, t, j0, r8);
            in_row8(IN + XK * 8192, t, j0, k8);
            in_row8(IN + XA * 8192, t, j0, a8);
            if (RAW) {
                // a = sigmoid(a_logit); kk = k*k_k / max(||k*k_k||, 1e-12) with the norm from P2;
                // k~ = k + k (a - 1) k_a, from the key before its update
                const float inv_norm = S.inv_norm[t];
                float kkp[8], kap[8];
                *reinterpret_cast<float4 *>(kkp) = *reinterpret_cast<const float4 *>(&S.k_k[us][j0]);
                *reinterpret_cast<float4 *>(kkp + 4) = *reinterpret_cast<const float4 *>(&S.k_k[us][j0 + 4]);
                *reinterpret_cast<float4 *>(kap) = *reinterpret_cast<const float4 *>(&S.k_a[us][j0]);
                *reinterpret_cast<float4 *>(kap + 4) = *reinterpret_cast<const float4 *>(&S.k_a[us][j0 + 4]);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    a8[e] = __fdividef(1.f, 1.f + __expf(-a8[e]));   // exp overflow -> 0, the limit
                    kk8[e] = k8[e] * kkp[e] * inv_norm;
                    k8[e] = fmaf(k8[e] * (a8[e] - 1.f), kap[e], k8[e]);
                }
            } else {
                in_row8(IN + XKK * 8192, t, j0, kk8);
            }
            const float4 ga = *reinterpret_cast<const float4 *>(GT + t * GTS + j0);         // g_{t-1}
            const float4 gb = *reinterpret_cast<const float4 *>(GT + t * GTS + j0 + 4);
            const float4 gc = *reinterpret_cast<const float4 *>(GT + (t + 1) * GTS + j0);   // g_t
            const float4 gd = *reinterpret_cast<const float4 *>(GT + (t + 1) * GTS + j0 + 4);
            const float gpv[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
            const float gtv[8] = {gc.x, gc.y, gc.z, gc.w, gd.x, gd.y, gd.z, gd.w};
            float kkd[8], rd[8], bi[8], ki[8], dk = 0.f, db = 0.f, bon = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float inv = __fdividef(1.f, gtv[e]);
                const float bb = kk8[e] * a8[e];
                kkd[e] = to_tf32(kk8[e] * gpv[e]);
                rd[e] = to_tf32(r8[e] * gtv[e]);
                bi[e] = to_tf32(bb * inv);
                ki[e] = to_tf32(k8[e] * inv);
                dk = fmaf(r8[e], k8[e], dk);
                db = fmaf(r8[e], bb, db);
                bon = fmaf(r8[e] * k8[e], S.r_k[us][j0 + e], bon);   // r_k = 0 without the epilogue
            }
            st_f4(sm + OFF_A1, sw128_off(t, j0, 128), kkd[0], kkd[1], kkd[2], kkd[3]);
            st_f4(sm + OFF_A1, sw128_off(t, j0 + 4, 128), kkd[4], kkd[5], kkd[6], kkd[7]);
            st_f4(sm + OFF_A1, sw128_off(64 + t, j0, 128), rd[0], rd[1], rd[2], rd[3]);
            st_f4(sm + OFF_A1, sw128_off(64 + t, j0 + 4, 128), rd[4], rd[5], rd[6], rd[7]);
            st_f4(sm + OFF_B1, sw128_off(t, j0, 128), bi[0], bi[1], bi[2], bi[3]);
            st_f4(sm + OFF_B1, sw128_off(t, j0 + 4, 128), bi[4], bi[5], bi[6], bi[7]);
            st_f4(sm + OFF_B1, sw128_off(64 + t, j0, 128), ki[0], ki[1], ki[2], ki[3]);
            st_f4(sm + OFF_B1, sw128_off(64 + t, j0 + 4, 128), ki[4], ki[5], ki[6], ki[7]);
            // the eight octets of token t sit in lanes differing in bits 0, 1 and 3
#pragma unroll
            for (int m = 1; m <= 8; m <<= 1) {
                if (m == 4) continue;
                dk += __shfl_xor_sync(0xffffffffu, dk, m);
                db += __shfl_xor_sync(0xffffffffu, db, m);
                bon += __shfl_xor_sync(0xffffffffu, bon, m);
            }
            if (sub == 0 && qa == 0) {
                S.dk[t] = dk;
                S.db[t] = db;
                S.bon[ip][t] = bon;
            }
        }
        // the operand tiles are read next by the tensor core (R1 and the transpose round at the
        // top of the chunk): generic-proxy writes -> visible to the async proxy
        fence_proxy_async_smem();
        return false;
    };

    // ---- output of chunk c of head u from T_D4, by all warps (each owns 16 columns of its lane
    //      quarter). Lanes 0-63 (key channel j): the new state diag(gC) S'^T -> B5, or the next CTA's
    //      B5 in split mode, and at the end of the sequence or of a snapshot interval fp32 to S_T /
    //      the snapshot. Lanes 64-127 (token t): y -> epilogue -> the swizzled y tile in B2.
    auto out = [&](int u, int c, int ip, int us, bool send) {
        const int b = u / p.H, hh = u % p.H, done = c * C + min(C, p.T - c * C);
        float v[2][8];
        tmem_ld8_nowait(tmem_addr(tb, Lq, T_D4 + c16), v[0]);
        tmem_ld8_nowait(tmem_addr(tb, Lq, T_D4 + c16 + 8), v[1]);
        tmem_ld_wait(v[0], v[1]);
        if (colg) {
            const int j = L;
            const float gCj = S.gC[ip][j];
            uint32_t xo[8];
            kcol_offsets(j, 64, xo);
            const uint32_t b5_dst = cs == 1 ? own_b5 : next_b5;
            // failure-path test: CTA 0 of the cluster keeps its first state to itself, so the next
            // CTA's bounded wait for it runs out
            const bool deliver = send && !(p.withhold_handoff && rank == 0 && sends == 0);
            const bool write_b5 = cs == 1 || deliver;
#pragma unroll
            for (int g = 0; g < 2; ++g)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    v[g][e] *= gCj;                                             // S_C = S' diag(gC)
                    if (write_b5) st_cluster(b5_dst + (c16 + 8 * g + e) * 128 + xo[e], to_tf32(v[g][e]));
                }
            if (deliver) {
                fence_proxy_async_cluster();
                mbar_arrive_remote(next_bar);
            }
            float *gdst = (c == nchunks - 1 && p.S_T) ? p.S_T + size_t(u) * 4096 : nullptr;
            float *sdst = (p.snap_every > 0 && done % p.snap_every == 0)
                              ? p.snaps + ((size_t(b) * p.n_snap + (done / p.snap_every - 1)) * p.H + hh) * 4096
                              : nullptr;
            if (gdst || sdst) {
#pragma unroll
                for (int g = 0; g < 2; ++g)
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = c16 + 8 * g + e;
                        if (gdst) gdst[i * 64 + j] = v[g][e];
                        if (sdst) sdst[i * 64 + j] = v[g][e];
                    }
            }
        } else {
            const int t = L - 64;
            if (epi) {   // group_norm over the head's 64 channels, then the bonus (r.(k*r_k)) v
                float s1 = 0.f, s2 = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) s1 += v[0][e] + v[1][e];
                S.red[pq][t] = s1;
                bar_named(BAR_ROWS, 256);
                const float mean = (S.red[0][t] + S.red[1][t] + S.red[2][t] + S.red[3][t]) * (1.f / 64.f);
                bar_named(BAR_ROWS, 256);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    s2 = fmaf(v[0][e] - mean, v[0][e] - mean, s2);
                    s2 = fmaf(v[1][e] - mean, v[1][e] - mean, s2);
                }
                S.red[pq][t] = s2;
                bar_named(BAR_ROWS, 256);
                const float inv =
                    1.f / sqrtf((S.red[0][t] + S.red[1][t] + S.red[2][t] + S.red[3][t]) * (1.f / 64.f) + p.gn_eps);
                const float bon = S.bon[ip][t];
                uint32_t xv[8];
                kcol_offsets(t, 64, xv);
#pragma unroll
                for (int g = 0; g < 2; ++g)
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int i = c16 + 8 * g + e;
                        const float vi = *reinterpret_cast<const float *>(sm + OFF_B4 + i * 128 + xv[e]);
                        v[g][e] = fmaf((v[g][e] - mean) * inv, S.ln_w[us][i], S.ln_b[us][i]) + bon * vi;
                    }
            }
            // y row t, channels c16..c16+15 -> the swizzled [64][32] fp32 tile of its channel half
            // (the layout the y tensor map expects); rows past the end of T are clipped by the store
            uint8_t *row = sm + OFF_B2 + (c16 >> 5) * 8192 + t * 128;
            const int q0 = (c16 & 31) >> 2;
#pragma unroll
            for (int m = 0; m < 4; ++m)
                *reinterpret_cast<float4 *>(row + (((q0 + m) ^ (t & 7)) << 4)) =
                    make_float4(v[m >> 1][4 * (m & 1)], v[m >> 1][4 * (m & 1) + 1], v[m >> 1][4 * (m & 1) + 2],
                                v[m >> 1][4 * (m & 1) + 3]);
        }
    };

    // ---- the CTA's chunks: (head u, chunk c), c = rank, rank + cs, ... of heads cid, cid + ncl, ...
    int u = p.unit0 + cid, c = rank;
    bool valid = u < units && rank < nchunks;
    int ip = 0, us = 0;                // parity slots of the current chunk and head
    if (valid) {
        if (tid == 0) issue_tma(u, c);
        tma_pending = true;
        if (tid < 64) load_params(u, 0, tid);
        if (rank == 0) load_state(u);
    }
    __syncthreads();
    {
        const bool f = valid && !back ? front(u, c, 0, 0) : false;
        failed = __syncthreads_or(f) != 0;
        if (valid && back) tma_parity ^= 1u;
        if (!failed) tma_pending = false;
    }

    while (valid && !failed) {
        const int b = u / p.H, hh = u % p.H, c0 = c * C;
        int nu = u, nc = c + cs;
        if (nc >= nchunks) { nu = u + ncl; nc = rank; }
        const bool more = nu < units && nc < nchunks;
        const bool new_unit = more && nu != u;
        const bool recv = cs > 1 && c > 0;   // split mode: this chunk's start state comes from CTA rank-1

        if (tid == 0) {
            // the next chunk's six input tiles are issued by six warps in P5; their byte count
            // is registered here, ordered before those issues by the barrier after R1
            if (more) mbar_arrive_expect_tx(&S.bar_tma, kTileBytes);
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)   // R1: Grams = [KKd; Rd] [Bi; Ki]^T
                mma_tf32_ss(tb + T_D1, dA1 + kstep_off(ks, 128), dB1 + kstep_off(ks, 128), idesc_tf32(128, 128), ks > 0);
            // transpose round on the tensor core (exact: identity times tf32 operands), N = 128:
            // lanes 0-63 of T_A2 <- Bi^T (A of R2), of T_D3R <- Ki^T (start of K~)
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                mma_tf32_ts(tb + T_A2, tb + T_ID + 8 * ks, dB1 + kstep_off(ks, 128), idesc_tf32(128, 128), ks > 0);
            mma_commit(&S.bar_mma);
        }
        mma_pending = true;
        // the previous chunk's y tile goes out now: every warp has slack while R1 runs
        if (y_pending && tid == kStoreThread) store_y_tile(maps, sm + OFF_B2, y_h, y_c0, y_b);
        y_pending = false;
        // ---- P4 (while the MMAs run): transposes through shared memory and the start of
        //      T_D3L (the previous chunk's R5 has read it).
        //      Lanes 0-63 (key/value channel j = L): V^T row j -> B4; identity row -> T_D3L.
        //      Lanes 64-127 (key j = L - 64): KKd^T row j -> B3 rows 64-127; Rd row t = j -> T_D3L.
        if (colg) {
            const int j = L;
            uint32_t xo[8];
            col_offsets(j, xo);
#pragma unroll 1
            for (int g = 0; g < 2; ++g) {
                const int t0 = c16 + 8 * g;
                float vv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) vv[e] = in_col(IN + XV * 8192, t0 + e, xo, e);
                st_f4(sm + OFF_B4, sw128_off(j, t0, 64), vv[0], vv[1], vv[2], vv[3]);
                st_f4(sm + OFF_B4, sw128_off(j, t0 + 4, 64), vv[4], vv[5], vv[6], vv[7]);
#pragma unroll
                for (int e = 0; e < 8; ++e) vv[e] = (t0 + e == L) ? 1.f : 0.f;
                tmem_st8(tmem_addr(tb, Lq, T_D3L + t0), vv);
            }
        } else {
            const int j = L - 64;
            uint32_t xo[8];
            kcol_offsets(j, 128, xo);
            const uint8_t *b6 = sm + OFF_A1;
#pragma unroll 1
            for (int g = 0; g < 2; ++g) {
                const int t0 = c16 + 8 * g;
                float kkd[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) kkd[e] = *reinterpret_cast<const float *>(b6 + (t0 + e) * 128 + xo[e]);
                st_f4(sm + OFF_B3, sw128_off(64 + j, t0, 128), kkd[0], kkd[1], kkd[2], kkd[3]);
                st_f4(sm + OFF_B3, sw128_off(64 + j, t0 + 4, 128), kkd[4], kkd[5], kkd[6], kkd[7]);
                const float4 ra = *reinterpret_cast<const float4 *>(b6 + sw128_off(64 + j, t0, 128));
                const float4 rb = *reinterpret_cast<const float4 *>(b6 + sw128_off(64 + j, t0 + 4, 128));
                const float rd[8] = {ra.x, ra.y, ra.z, ra.w, rb.x, rb.y, rb.z, rb.w};
                tmem_st8(tmem_addr(tb, Lq, T_D3L + t0), rd);   // Rd row (token j), channels t0..t0+7
            }
        }
        if (wait_mma_all()) { failed = true; break; }
        // ---- P5: masks. Lanes 0-63 (token t): M_ab row -> inverse workspace; M_kb row t ->
        //      column t of B3 rows 0-63 (M_kb^T, scalar stores along K: conflict-free).
        //      Lanes 64-127 (token t): Q_b row -> T_A2 lanes 64-127; Q_k row -> T_D3R lanes 64-127.
        if (more && lane == 0 && colg && (warp >> 2) < 3) {
            // the input tiles were last read in P4: six warps each issue one tile of the next chunk
            const int x = (warp >> 2) * 2 + (warp & 1);
            if (!(RAW && x == XKK)) tma_load_4d(sm + OFF_IN + x * 8192, &maps.m[x], &S.bar_tma, 0, nu % p.H, nc * C, nu / p.H);
        }
        if (colg) {
            const int t = L;
            float m[2][8], mk[2][8];
            tmem_ld8_nowait(tmem_addr(tb, Lq, T_D1 + c16), m[0]);
            tmem_ld8_nowait(tmem_addr(tb, Lq, T_D1 + c16 + 8), m[1]);
            tmem_ld8_nowait(tmem_addr(tb, Lq, T_D1 + 64 + c16), mk[0]);
            tmem_ld8_nowait(tmem_addr(tb, Lq, T_D1 + 64 + c16 + 8), mk[1]);
            tmem_ld_wait(m[0], m[1], mk[0], mk[1]);
            uint32_t xo[8];
            kcol_offsets(t, 128, xo);
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                const int s0 = c16 + 8 * g;
#pragma unroll
                for (int e = 0; e < 8; ++e) m[g][e] = (s0 + e < t) ? m[g][e] : 0.f;
                *reinterpret_cast<float4 *>(Lw + t * LWS + s0) = make_float4(m[g][0], m[g][1], m[g][2], m[g][3]);
                *reinterpret_cast<float4 *>(Lw + t * LWS + s0 + 4) = make_float4(m[g][4], m[g][5], m[g][6], m[g][7]);
#pragma unroll
                for (int e = 0; e < 8; ++e)   // B3[s][t] = M_kb[t][s], nonzero for s < t
                    *reinterpret_cast<float *>(sm + OFF_B3 + (s0 + e) * 128 + xo[e]) =
                        (s0 + e < t) ? to_tf32(mk[g][e]) : 0.f;
            }
            if (t >= 32 && c16 < 32) {   // L21^T[s][t - 32] = M_ab[t][s] (s < 32 <= t: no mask)
                uint32_t xl[8];
                kcol_offsets(t - 32, 32, xl);
#pragma unroll
                for (int g = 0; g < 2; ++g)
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        *reinterpret_cast<float *>(sm + OFF_L21 + (c16 + 8 * g + e) * 128 + xl[e]) = to_tf32(m[g][e]);
            }
        } else {
            const int t = L - 64;
            // the current-token entries are taken exactly in fp32: they dominate short sequences
            const float dgb = to_tf32(S.db[t]);
            const float dgk = S.dk[t];
            float qb[2][8], qk[2][8];
            tmem_ld8_nowait(tmem_addr(tb, Lq, T_D1 + c16), qb[0]);            // Q_b row t
            tmem_ld8_nowait(tmem_addr(tb, Lq, T_D1 + c16 + 8), qb[1]);
            tmem_ld8_nowait(tmem_addr(tb, Lq, T_D1 + 64 + c16), qk[0]);       // Q_k row t
            tmem_ld8_nowait(tmem_addr(tb, Lq, T_D1 + 64 + c16 + 8), qk[1]);
            tmem_ld_wait(qb[0], qb[1], qk[0], qk[1]);
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                const int s0 = c16 + 8 * g;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int ss = s0 + e;
                    qb[g][e] = ss < t ? to_tf32(qb[g][e]) : (ss == t ? dgb : 0.f);
                    qk[g][e] = ss < t ? qk[g][e] : (ss == t ? dgk : 0.f);
                }
                tmem_st8(tmem_addr(tb, Lq, T_A2 + s0), qb[g]);
                tmem_st8(tmem_addr(tb, Lq, T_D3R + s0), qk[g]);
            }
        }
        if (tid == kStoreThread) tma_store_wait_read();   // the y tile in B2 has been read
        sync_for_mma();
        tma_pending = more;
        // ---- A = (I + M_ab)^{-1}. Diagonal 16x16 blocks: one thread per (block, column)
        //      solves (I + L_dd) x = e_c by forward substitution in registers (warps 2, 3).
        if (tid >= 64 && tid < 128) {
            const int d = (tid - 64) >> 4, cc = tid & 15;
            const float *Lb = Lw + 16 * d * LWS + 16 * d;
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                float acc = (r == cc) ? 1.f : 0.f;
#pragma unroll
                for (int k = 0; k < r; ++k) acc = fmaf(-Lb[r * LWS + k], x[k], acc);
                x[r] = acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) Aw[(16 * d + r) * LWS + 16 * d + cc] = x[r];
            // column cc of the block is row 16d + cc of B2 = D^T (K = t), tf32
#pragma unroll
            for (int m = 0; m < 4; ++m)
                st_f4(sm + OFF_B2, sw128_off(16 * d + cc, 16 * d + 4 * m, 64), to_tf32(x[4 * m]), to_tf32(x[4 * m + 1]),
                      to_tf32(x[4 * m + 2]), to_tf32(x[4 * m + 3]));
        } else {
            // B2 = D^T, D = blockdiag(Y0, Y1): zero where t and s lie in different 32-halves or
            // t's 16-block precedes s's (the diagonal blocks and the level-1 blocks are written by
            // their producers)
            const int z = tid < 64 ? tid : tid - 64;
#pragma unroll 1
            for (int e = z; e < 1024; e += kThreads - 64) {
                const int sr = e & 63, t4 = (e >> 6) * 4;
                if (((t4 ^ sr) >= 32) || ((t4 >> 4) < (sr >> 4))) st_f4(sm + OFF_B2, sw128_off(sr, t4, 64), 0.f, 0.f, 0.f, 0.f);
            }
        }
        __syncthreads();
        // level 1: X[2p+1][2p] = -X[2p+1] (L[2p+1][2p] X[2p]), p = 0, 1. Threads 0-127 each
        // compute four adjacent outputs from one broadcast scalar and one float4 per step.
        if (tid < 128) {
            const int pp = tid >> 6, i = (tid >> 2) & 15, j4 = (tid & 3) * 4;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kq = 0; kq < 16; ++kq) {
                const float lv = Lw[(32 * pp + 16 + i) * LWS + 32 * pp + kq];
                const float4 xv = *reinterpret_cast<const float4 *>(Aw + (32 * pp + kq) * LWS + 32 * pp + j4);
                acc[0] = fmaf(lv, xv.x, acc[0]); acc[1] = fmaf(lv, xv.y, acc[1]);
                acc[2] = fmaf(lv, xv.z, acc[2]); acc[3] = fmaf(lv, xv.w, acc[3]);
            }
            *reinterpret_cast<float4 *>(Tw + (pp * 16 + i) * 20 + j4) = make_float4(acc[0], acc[1], acc[2], acc[3]);
        }
        __syncthreads();
        if (tid < 128) {
            const int pp = tid >> 6, i = (tid >> 2) & 15, j4 = (tid & 3) * 4;
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int kq = 0; kq < 16; ++kq) {
                const float xv = Aw[(32 * pp + 16 + i) * LWS + 32 * pp + 16 + kq];
                const float4 tv = *reinterpret_cast<const float4 *>(Tw + (pp * 16 + kq) * 20 + j4);
                acc[0] = fmaf(xv, tv.x, acc[0]); acc[1] = fmaf(xv, tv.y, acc[1]);
                acc[2] = fmaf(xv, tv.z, acc[2]); acc[3] = fmaf(xv, tv.w, acc[3]);
            }
            // the block X[2p+1][2p] of D goes transposed into B2 (row s = column of D, K = t), tf32
            const int t = 32 * pp + 16 + i;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<float *>(sm + OFF_B2 + sw128_off(32 * pp + j4 + q, t, 64)) = to_tf32(-acc[q]);
        }
        // B2 now holds D^T, D = blockdiag(Y0, Y1) the inverses of the two diagonal 32x32 blocks of
        // I + M_ab; the off-diagonal block of the inverse, -Y1 L21 Y0, is applied by R2b/R2c.
        sync_for_mma();

        // ---- the window: warps 0-3 run this chunk's dependent MMA rounds and its output,
        //      warps 4-15 prepare the next chunk's operands.
        bool wfail = false;
        if (back) {
            if (tid == 0) {
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)   // R2a: U = W D, W = [Bi^T; Q_b]
                    mma_tf32_ts(tb + T_D1, tb + T_A2 + 8 * ks, dB2 + kstep_off(ks, 64), idesc_tf32(128, 64), ks > 0);
                mma_commit(&S.bar_mma);
            }
            wfail = wait_mma_back(false);
            // Z = W A with A = D - [0 0; Y1 L21 Y0 0]: Z[:, 32:64] = U[:, 32:64] and
            // Z[:, 0:32] = U[:, 0:32] - (U[:, 32:64] L21) Y0 (block back-substitution on the tensor core)
            if (!wfail) {
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)   // R2b: V = U[:, 32:64] L21
                        mma_tf32_ts(tb + T_V, tb + T_D1 + 32 + 8 * ks, dL21 + kstep_off(ks, 32), idesc_tf32(128, 32), ks > 0);
                    mma_commit(&S.bar_mma);
                }
                wfail = wait_mma_back(false);
            }
            if (!wfail) {
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)   // R2c: U[:, 0:32] -= V Y0 (B2 rows 0-31 hold Y0^T)
                        mma_tf32_ts(tb + T_D1, tb + T_V + 8 * ks, dB2 + kstep_off(ks, 64), idesc_neg_a(idesc_tf32(128, 32)), 1);
                    mma_commit(&S.bar_mma);
                }
                wfail = wait_mma_back(false);
            }
            if (!wfail) {
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)   // R3: [T_D3R | T_D3L] -= Z [M_kb | KKd]
                        mma_tf32_ts(tb + T_D3R, tb + T_D1 + 8 * ks, dB3 + kstep_off(ks, 128),
                                    idesc_neg_a(idesc_tf32(128, 128)), 1);
                    mma_commit(&S.bar_mma);
                }
                wfail = wait_mma_back(false);
            }
            if (!wfail) {
                bool state_to = false;
                if (tid == 0) {
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)   // R4: [Ki^T - X; Q~] V
                        mma_tf32_ts(tb + T_D4, tb + T_D3R + 8 * ks, dB4 + kstep_off(ks, 64), idesc_tf32(128, 64), ks > 0);
                    if (recv) {
                        // the only wait on another CTA: everything above used this chunk's inputs only
                        state_to = !mbar_wait_cluster(&S.bar_state, state_parity, p.handoff_timeout_ns);
                        fence_proxy_async_smem();
                        tc_fence_after();
                    }
                    if (!state_to) {
#pragma unroll
                        for (int ks = 0; ks < 8; ++ks)   // R5: += [I - X; R~] S_0^T
                            mma_tf32_ts(tb + T_D4, tb + T_D3L + 8 * ks, dB5 + kstep_off(ks, 64), idesc_tf32(128, 64), 1);
                    }
                    mma_commit(&S.bar_mma);
                }
                if (recv) state_parity ^= 1u;
                wfail = wait_mma_back(state_to);
                // split mode: this CTA's B5 is consumed; the previous CTA may send the next state
                if (!wfail && recv && tid == 0) mbar_arrive_remote(prev_credit);
            }
        } else if (more) {
            if (new_unit && ft < 64) load_params(nu, us ^ 1, ft);
            wfail = front(nu, nc, ip ^ 1, new_unit ? (us ^ 1) : us);
            if (!wfail) tma_pending = false;   // these threads saw the tiles arrive
        }
        // split mode: before writing the next CTA's B5, its credit for the state sent before
        const bool send = cs > 1 && c + 1 < nchunks;
        if (send && sends > 0) {
            if (tid == 0 && !wfail) wfail = !mbar_wait_cluster(&S.bar_credit, credit_parity, p.handoff_timeout_ns);
            credit_parity ^= 1u;
        }
        tc_fence_before();
        if (__syncthreads_or(wfail)) { failed = true; break; }
        tc_fence_after();
        out(u, c, ip, us, send);
        if (send) ++sends;
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // keep the barrier parities uniform: warps 0-3 completed five MMA rounds, warps 4-15
        // consumed the next chunk's tiles
        if (!back) mma_parity ^= 1u;
        if (back && more) tma_parity ^= 1u;
        tma_pending = false;
        mma_pending = false;
        y_pending = true;
        y_h = hh; y_c0 = c0; y_b = b;
        if (new_unit && rank == 0) load_state(nu);   // R5 of the previous head has read B5
        u = nu; c = nc; valid = more;
        ip ^= 1;
        if (new_unit) us ^= 1;
    }
    if (tid == kStoreThread) {
        if (y_pending && !failed) store_y_tile(maps, sm + OFF_B2, y_h, y_c0, y_b);
        tma_store_wait_all();
    }

    if (failed) {
        if (tid == 0) atomicOr(p.err, 1u);
        // drain what this CTA issued (bounded), then release tensor memory
        if (mma_pending) mbar_wait(&S.bar_mma, mma_parity, p.timeout_ns);
        if (tma_pending) mbar_wait(&S.bar_tma, tma_parity, p.timeout_ns);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tb, 512);
    // no CTA leaves while another CTA of its cluster may still write to its shared memory
    if (cs > 1) cluster_sync();
}

// ---- host side ---------------------------------------------------------------------------------------

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

struct DeviceInfo {
    int sms = 0;
    unsigned int *err = nullptr;
    bool attr_set = false;
    int clusters[kMaxSegments + 1] = {};   // co-resident clusters of each size (0: that size does not fit)
};

cudaLaunchConfig_t launch_config(int grid, int cs, cudaStream_t stream, cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(unsigned(grid), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = stream;
    attr->id = cudaLaunchAttributeClusterDimension;
    attr->val.clusterDim.x = unsigned(cs);
    attr->val.clusterDim.y = 1;
    attr->val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

cudaError_t device_info(DeviceInfo *&out) {
    static std::mutex mu;
    static DeviceInfo info[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    DeviceInfo &d = info[dev];
    if (!d.attr_set) {
        if ((e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaGetSymbolAddress(reinterpret_cast<void **>(&d.err), g_device_error)) != cudaSuccess) return e;
        if ((e = cudaFuncSetAttribute(chunk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(SMEM_BYTES))) != cudaSuccess ||
            (e = cudaFuncSetAttribute(chunk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      int(SMEM_BYTES))) != cudaSuccess)
            return e;
        d.clusters[1] = d.sms;
        for (int cs = 2; cs <= kMaxSegments; ++cs) {
            cudaLaunchAttribute attr;
            const cudaLaunchConfig_t cfg = launch_config(cs * (d.sms / cs), cs, nullptr, &attr);
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, chunk_kernel<false>, &cfg) != cudaSuccess) {
                cudaGetLastError();
                n = 0;
            }
            d.clusters[cs] = n;
        }
        d.attr_set = true;
    }
    out = &d;
    return cudaSuccess;
}

// CTAs per (b, h). Each CTA of a cluster runs every cs-th chunk, so a head takes about
// ceil(nchunks / cs) chunk times plus the hand-off latency, and the heads run in
// ceil(units / clusters) waves. Pick the size with the smallest estimate (ties: fewer CTAs);
// the 15.5% and 0.35-chunk terms are the measured cost of the hand-off per chunk and per head
// (B8 T1024 H12 and B16 T4096 H32 timed with 1-4 CTAs per head).
double launch_cost(int units, int nchunks, int cs, const DeviceInfo &d) {
    const double waves = double((units + d.clusters[cs] - 1) / d.clusters[cs]);
    const double per = double((nchunks + cs - 1) / cs);
    return waves * (per * (cs > 1 ? 1.155 : 1.0) + 0.35 * (cs - 1));
}
int choose_segments(int units, int nchunks, const DeviceInfo &d, double *cost_out = nullptr) {
    int best = 1;
    double best_cost = 1e300;
    for (int cs = 1; cs <= kMaxSegments; ++cs) {
        if (d.clusters[cs] <= 0) continue;
        const double cost = launch_cost(units, nchunks, cs, d);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = cs;
        }
    }
    if (cost_out) *cost_out = best_cost;
    return best;
}

// The launches of one forward call: the heads that fill whole waves of one CTA per head, then
// the rest with the CTAs per head that suit them (a partial last wave would otherwise leave
// SMs idle), when that is cheaper than one launch; the second launch costs about half a chunk.
struct ChunkPlan {
    int n = 1;
    int units[2] = {0, 0};   // heads per launch
    int cs[2] = {1, 1};
};
ChunkPlan plan_launches(const FwdArgs &p, const DeviceInfo &d) {
    const int units = p.B * p.H, nchunks = (p.T + C - 1) / C;
    ChunkPlan pl;
    pl.units[0] = units;
    if (p.segments > 0) {
        pl.cs[0] = p.segments;
        return pl;
    }
    double one = 0.0, tail_cost = 0.0;
    pl.cs[0] = choose_segments(units, nchunks, d, &one);
    const int full = (units / d.clusters[1]) * d.clusters[1];
    if (full > 0 && full < units) {
        const int tail_cs = choose_segments(units - full, nchunks, d, &tail_cost);
        const double two = double(full / d.clusters[1]) * nchunks + tail_cost + 0.5;
        if (tail_cs > 1 && two < one - 1e-9) {
            pl.n = 2;
            pl.units[0] = full;
            pl.cs[0] = 1;
            pl.units[1] = units - full;
            pl.cs[1] = tail_cs;
        }
    }
    return pl;
}

}  // namespace

cudaError_t chunk_segments(const FwdArgs &p, int *segments, int *launches) {
    DeviceInfo *di = nullptr;
    const cudaError_t e = device_info(di);
    if (e != cudaSuccess) return e;
    const ChunkPlan pl = plan_launches(p, *di);
    for (int i = 0; i < pl.n; ++i)
        if (pl.cs[i] > kMaxSegments || di->clusters[pl.cs[i]] <= 0) return cudaErrorInvalidClusterSize;
    *segments = pl.cs[pl.n - 1];   // the CTAs per head of the last launch (the first is 1 when there are two)
    if (launches) *launches = pl.n;
    return cudaSuccess;
}

bool chunk_supported(const FwdArgs &p) {
    return p.N == kN && p.dt == WKV7_BF16 && (p.snap_every == 0 || p.snap_every % C == 0);
}

cudaError_t launch_chunk(const FwdArgs &p) {
    auto enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    DeviceInfo *di = nullptr;
    cudaError_t e = device_info(di);
    if (e != cudaSuccess) return e;
    ChunkMaps maps;
    // raw inputs: slot XW holds the decay logit, XA the rate logit, and the kk slot is not loaded
    const void *src[6] = {p.r, p.w, p.k, p.v, p.raw ? p.k : p.kk, p.a};
    const cuuint64_t dims[4] = {cuuint64_t(kN), cuuint64_t(p.H), cuuint64_t(p.T), cuuint64_t(p.B)};
    const cuuint64_t strides[3] = {cuuint64_t(kN) * 2, cuuint64_t(p.H) * kN * 2, cuuint64_t(p.T) * p.H * kN * 2};
    const cuuint32_t box[4] = {cuuint32_t(kN), 1, cuuint32_t(C), 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    for (int x = 0; x < 6; ++x) {
        const CUresult r = enc(&maps.m[x], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(src[x]), dims,
                               strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    {
        const cuuint64_t ydims[4] = {cuuint64_t(kN), cuuint64_t(p.H), cuuint64_t(p.T), cuuint64_t(p.B)};
        const cuuint64_t ystrides[3] = {cuuint64_t(kN) * 4, cuuint64_t(p.H) * kN * 4, cuuint64_t(p.T) * p.H * kN * 4};
        const cuuint32_t ybox[4] = {32, 1, cuuint32_t(C), 1};
        const CUresult r = enc(&maps.y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, p.y, ydims, ystrides, ybox, es,
                               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    ChunkArgs a{};
    a.B = p.B; a.T = p.T; a.H = p.H;
    a.S0 = p.S0; a.S_T = p.S_T; a.snaps = p.snaps;
    a.snap_every = p.snap_every;
    a.n_snap = p.snap_every > 0 ? p.T / p.snap_every : 0;
    a.ln_w = p.ln_w; a.ln_b = p.ln_b; a.r_k = p.r_k; a.gn_eps = p.gn_eps;
    a.k_k = p.k_k; a.k_a = p.k_a;
    a.err = di->err;
    a.timeout_ns = 2000000000ull;
    a.handoff_timeout_ns = p.handoff_wait_us ? 1000ull * p.handoff_wait_us : a.timeout_ns;
    a.withhold_handoff = p.withhold_handoff;
    int cs = 1;
    if ((e = chunk_segments(p, &cs)) != cudaSuccess) return e;
    const ChunkPlan pl = plan_launches(p, *di);
    a.unit0 = 0;
    for (int i = 0; i < pl.n; ++i) {
        a.unit_end = a.unit0 + pl.units[i];
        const int ncl = pl.units[i] < di->clusters[pl.cs[i]] ? pl.units[i] : di->clusters[pl.cs[i]];
        cudaLaunchAttribute attr;
        const cudaLaunchConfig_t cfg = launch_config(ncl * pl.cs[i], pl.cs[i], p.stream, &attr);
        e = p.raw ? cudaLaunchKernelEx(&cfg, chunk_kernel<true>, maps, a) : cudaLaunchKernelEx(&cfg, chunk_kernel<false>, maps, a);
        if (e != cudaSuccess) return e;
        a.unit0 = a.unit_end;
    }
    return cudaSuccess;
}

cudaError_t device_error_word(unsigned int **ptr) {
    DeviceInfo *di = nullptr;
    const cudaError_t e = device_info(di);
    if (e == cudaSuccess) *ptr = di->err;
    return e;
}

cudaError_t read_device_error(cudaStream_t stream, unsigned int *value, bool clear) {
    DeviceInfo *di = nullptr;
    cudaError_t e = device_info(di);
    if (e != cudaSuccess) return e;
    if ((e = cudaStreamSynchronize(stream)) != cudaSuccess) return e;
    if ((e = cudaMemcpy(value, di->err, sizeof(unsigned int), cudaMemcpyDeviceToHost)) != cudaSuccess) return e;
    if (clear && *value) e = cudaMemset(di->err, 0, sizeof(unsigned int));
    return e;
}

}  // namespace wkv7
