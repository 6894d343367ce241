// Backward of the optional epilogue: the per-head group_norm (population variance, eps inside
// the square root, a per-channel affine ln_w, ln_b) and the current-token bonus
// (sum_j r_j k_j r_k[j]) v, from the RWKV-7 rebuttal page's numpy time_mixing listing (the
// group_norm lambda and the two lines after the readout). The pages print the forward only; this
// is its chain rule. For one (b, t, h) row, with yc = y - mean(y), inv = (mean(yc^2) + eps)^-1/2,
// yn = yc inv, beta = sum_j r_j k_j r_k[j] and dout the gradient arriving at the epilogue's output:
//     dv = beta dout;  dbeta = sum_i dout_i v_i;  dr = dbeta k r_k;  dk = dbeta r r_k
//     dr_k += dbeta r k;  dln_w += dout yn;  dln_b += dout
//     g = dout ln_w;  dy = inv (g - mean(g) - yn mean(g yn))
// One warp per row (each lane N / 32 adjacent channels; the row sums by shuffles), eight warps per
// CTA over 64 rows of one head. The parameter gradients are summed in a fixed order: per lane
// over its rows, over the CTA's warps in shared memory into one partial per CTA, then over the
// CTAs of a head by a second kernel, so repeated calls give identical results.
#include "epilogue.cuh"

namespace wkv7 {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

template <class Tin, int NN>
__global__ void __launch_bounds__(kWarps * 32) epilogue_bwd_kernel(const EpiBwdArgs a) {
    constexpr int E = NN / 32;
    __shared__ float red[kWarps][3][NN];
    // one CTA per (block of kEpiRows rows, head); the heads of a row block are adjacent CTAs
    const size_t part = blockIdx.x / unsigned(a.H);
    const int h = int(blockIdx.x % unsigned(a.H)), warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const size_t rows = size_t(a.B) * a.T;
    const int j0 = lane * E;
    const Tin *r = static_cast<const Tin *>(a.r), *k = static_cast<const Tin *>(a.k), *v = static_cast<const Tin *>(a.v);
    float lw[E], rk[E], acc_w[E], acc_b[E], acc_k[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        lw[e] = a.ln_w[h * NN + j0 + e];
        rk[e] = a.r_k[h * NN + j0 + e];
        acc_w[e] = acc_b[e] = acc_k[e] = 0.f;
    }
    const float inv_n = 1.f / NN;
    // the warp's rows one at a time (batching two or four rows per warp cost more in occupancy)
    for (int i0 = warp; i0 < kEpiRows; i0 += kWarps) {
        const size_t rr = part * kEpiRows + i0;
        if (rr >= rows) break;                          // uniform over the warp
        const size_t base = (rr * a.H + h) * NN + j0;   // row (b, t) = rr of head h
        float y[E], rv[E], kv[E], vv[E], d[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            y[e] = a.y[base + e];
            rv[e] = load1(r + base + e);
            kv[e] = load1(k + base + e);
            vv[e] = load1(v + base + e);
            d[e] = a.dout[base + e];
        }
        float sy = 0.f, beta = 0.f, dbeta = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            sy += y[e];
            beta = fmaf(rv[e] * kv[e], rk[e], beta);
            dbeta = fmaf(d[e], vv[e], dbeta);
        }
        sy = warp_sum(sy);
        beta = warp_sum(beta);
        dbeta = warp_sum(dbeta);
        const float mean = sy * inv_n;
        float sq = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            y[e] -= mean;
            sq = fmaf(y[e], y[e], sq);
        }
        const float inv = 1.f / sqrtf(warp_sum(sq) * inv_n + a.eps);
        float g[E], sg = 0.f, sgy = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            y[e] *= inv;   // yn
            g[e] = d[e] * lw[e];
            sg += g[e];
            sgy = fmaf(g[e], y[e], sgy);
            acc_w[e] = fmaf(d[e], y[e], acc_w[e]);
            acc_b[e] += d[e];
            acc_k[e] = fmaf(dbeta * rv[e], kv[e], acc_k[e]);
        }
        const float mg = warp_sum(sg) * inv_n, mgy = warp_sum(sgy) * inv_n;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            a.dy[base + e] = inv * (g[e] - mg - y[e] * mgy);
            a.dr[base + e] = dbeta * kv[e] * rk[e];
            a.dk[base + e] = dbeta * rv[e] * rk[e];
            a.dv[base + e] = beta * d[e];
        }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
        red[warp][0][j0 + e] = acc_w[e];
        red[warp][1][j0 + e] = acc_b[e];
        red[warp][2][j0 + e] = acc_k[e];
    }
    __syncthreads();
    float *ws = a.ws + (part * a.H + h) * 3 * NN;
    for (int q = threadIdx.x; q < 3 * NN; q += blockDim.x) {
        const int which = q / NN, j = q % NN;
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) s += red[w][which][j];
        ws[q] = s;
    }
}

// One parameter gradient (blockIdx.y: dln_w, dln_b, dr_k) of head blockIdx.x: the sum of the
// CTAs' partials. Warp w sums partials w, w + 8, ... (lane: N / 32 adjacent channels), then the
// eight warp sums are added in warp order.
template <int NN>
__global__ void __launch_bounds__(kWarps * 32) epilogue_param_sum_kernel(const EpiBwdArgs a, int parts) {
    constexpr int E = NN / 32;
    __shared__ float red[kWarps][NN];
    const int h = blockIdx.x, which = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float s[E];
#pragma unroll
    for (int e = 0; e < E; ++e) s[e] = 0.f;
#pragma unroll 4
    for (int pp = warp; pp < parts; pp += kWarps) {
        const float *src = a.ws + ((size_t(pp) * a.H + h) * 3 + which) * NN + lane * E;
#pragma unroll
        for (int e = 0; e < E; ++e) s[e] += src[e];
    }
#pragma unroll
    for (int e = 0; e < E; ++e) red[warp][lane * E + e] = s[e];
    __syncthreads();
    float *out = which == 0 ? a.dln_w : which == 1 ? a.dln_b : a.dr_k;
    for (int j = threadIdx.x; j < NN; j += blockDim.x) {
        float t = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) t += red[w][j];
        out[h * NN + j] = t;
    }
}

template <class Tin, int NN>
cudaError_t launch_t(const EpiBwdArgs &a) {
    const size_t rows = size_t(a.B) * a.T;
    const int parts = int((rows + kEpiRows - 1) / kEpiRows);
    if (parts > 0) {
        // parts * H: at most 2^29 under the size limit B * T * H * N <= 2^40 (H alone when B * T <= 64)
        epilogue_bwd_kernel<Tin, NN><<<unsigned(size_t(parts) * a.H), kWarps * 32, 0, a.stream>>>(a);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    epilogue_param_sum_kernel<NN><<<dim3(unsigned(a.H), 3u), kWarps * 32, 0, a.stream>>>(a, parts);
    return cudaGetLastError();
}

}  // namespace

// ---- host side ---------------------------------------------------------------------------------------

cudaError_t launch_epilogue_backward(const EpiBwdArgs &a) {
    if (a.dt == WKV7_BF16) return a.N == 128 ? launch_t<__nv_bfloat16, 128>(a) : launch_t<__nv_bfloat16, 64>(a);
    return a.N == 128 ? launch_t<float, 128>(a) : launch_t<float, 64>(a);
}

}  // namespace wkv7
