// One RWKV-7 time-mixing layer over a sequence (RWKV-7 rebuttal page, the numpy time_mixing
// listing): every projection is this library's GEMM (gemm.cu) with the token-shift mix fused
// into its operand load and the bias, activation or value residual fused into its store; the
// recurrence with its pre-processing and epilogue runs through wkv7_forward_raw (chunked
// tensor-core kernel for bf16, scan for fp32); the gate multiplies the readout in one
// element-wise pass before the output projection.
//
// Data flow for M = B*T token rows of C = H*N channels, in the layer dtype unless noted
// (x_m = x + m (x_prev - x), x_prev the token before):
//   r = x_r Wr^T, k = x_k Wk^T, v = x_v Wv^T          (the first layer writes v to v0_out)
//   hw = tanh(x_w Ww1);   w_logit = hw Ww2 + w_bias
//   ha = x_a Wa1;         a_logit = ha Wa2 + a_bias
//   hv = x_v Wv1;         v <- v + (v0 - v) sigmoid(hv Wv2 + v_bias)     (layers after the first)
//   hg = sigmoid(x_g Wg1); g = hg Wg2 (fp32)
//   y = wkv7_forward_raw(r, w_logit, k, v, a_logit, k_k, k_a; S in place; epilogue) (fp32)
//   out = (y * g) Wo^T (fp32; y * g rounded to the layer dtype, in r's buffer)
// The low-rank factors are stored [in][out] (applied as x W); each call copies them transposed
// and zero-padded to a multiple of 64 into the workspace, so that every GEMM takes W as
// [out][in] with K and N multiples of 64 (the padding adds exact zeros).
// Launches, in stream order: the factor copies (one launch); the seven products of the mixed x
// (r, k, v and the four first factors, one grouped launch); the four second factors (one
// grouped launch); the recurrence; the gate product; the output projection; the last-token copy.
#include <algorithm>
#include <cstdio>

#include "gemm.cuh"

namespace wkv7 {
namespace {

#define GRID_STRIDE(i, n) for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < (n); i += size_t(gridDim.x) * blockDim.x)

// last_x_out[b] = x[b, T - 1].
template <class T>
__global__ void last_kernel(const T *x, T *out, int Tn, int C, size_t n) {
    GRID_STRIDE(i, n) out[i] = x[((i / C) * Tn + (Tn - 1)) * C + i % C];
}

unsigned grid_for(size_t n) { return unsigned(std::min<size_t>((n + 255) / 256, size_t(148) * 16)); }

// out[i] = y[i] * g[i], four elements per step (n a multiple of 4).
template <class T>
__global__ void gate_kernel(const float4 *y, const float4 *g, T *out, size_t n4) {
    GRID_STRIDE(i, n4) {
        const float4 a = y[i], b = g[i];
        if constexpr (sizeof(T) == 2) {
            const __nv_bfloat162 lo = __floats2bfloat162_rn(a.x * b.x, a.y * b.y), hi = __floats2bfloat162_rn(a.z * b.z, a.w * b.w);
            reinterpret_cast<uint2 *>(out)[i] =
                make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
        } else {
            reinterpret_cast<float4 *>(out)[i] = make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
        }
    }
}

int pad64(int d) { return (d + 63) / 64 * 64; }

// Byte offsets of the layer's intermediates in the caller's workspace (256-byte aligned).
struct LayerPlan {
    size_t r, k, v, wl, al, hw, ha, hv, hg, g, y;
    size_t w1[4], w2[4];   // transposed low-rank factors: Ww, Wa, Wv, Wg
    size_t total;
};

LayerPlan layer_plan(size_t M, int C, const wkv7_layer_dims &d, size_t e) {
    LayerPlan p{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        const size_t o = off;
        off += (bytes + 255) & ~size_t(255);
        return o;
    };
    const size_t mc = M * size_t(C);
    const int dp[4] = {pad64(d.d_w), pad64(d.d_a), pad64(d.d_v), pad64(d.d_g)};
    p.r = take(mc * e); p.k = take(mc * e); p.v = take(mc * e); p.wl = take(mc * e); p.al = take(mc * e);
    p.hw = take(M * dp[0] * e); p.ha = take(M * dp[1] * e); p.hv = take(M * dp[2] * e); p.hg = take(M * dp[3] * e);
    p.g = take(mc * 4); p.y = take(mc * 4);
    for (int i = 0; i < 4; ++i) {
        p.w1[i] = take(size_t(dp[i]) * C * e);
        p.w2[i] = take(size_t(C) * dp[i] * e);
    }
    p.total = off;
    return p;
}

}  // namespace

// Everything after validation: the launches of one layer call, in stream order.
template <class T>
wkv7_status layer_run(int B, int Tn, const wkv7_layer_dims &d, const wkv7_layer_params &P, const void *x,
                      const void *last_x, const void *v0, float *S, float *out, void *v0_out, void *last_x_out,
                      const wkv7_opts &opts, uint8_t *ws, cudaStream_t stream, char *err, size_t err_len) {
    const int C = d.H * d.N;
    const size_t M = size_t(B) * Tn, e = sizeof(T);
    const wkv7_dtype dt = sizeof(T) == 2 ? WKV7_BF16 : WKV7_F32;
    const LayerPlan L = layer_plan(M, C, d, e);
    auto at = [&](size_t off) { return static_cast<void *>(ws + off); };
    auto fail = [&](cudaError_t c, const char *what) {
        snprintf(err, err_len, "%s: %s", what, cudaGetErrorString(c));
        return WKV7_ERR_CUDA;
    };
    unsigned int *dev_err = nullptr;
    cudaError_t c = device_error_word(&dev_err);
    if (c != cudaSuccess) return fail(c, "device error word");
    // the low-rank factors, transposed to [out][in] and zero-padded to multiples of 64 (one launch)
    const void *w1[4] = {P.Ww1, P.Wa1, P.Wv1, P.Wg1}, *w2[4] = {P.Ww2, P.Wa2, P.Wv2, P.Wg2};
    const int dims[4] = {d.d_w, d.d_a, d.d_v, d.d_g};
    PadCopy copies[kMaxPadCopies];
    int ncopies = 0;
    for (int i = 0; i < 4; ++i) {
        if (i == 2 && !v0) continue;   // the value residual's factors are unused in the first layer
        const int dp = pad64(dims[i]);
        copies[ncopies++] = PadCopy{w1[i], at(L.w1[i]), C, dims[i], dp, C};
        copies[ncopies++] = PadCopy{w2[i], at(L.w2[i]), dims[i], C, C, dp};
    }
    if ((c = launch_transpose_pad(copies, ncopies, dt, stream)) != cudaSuccess) return fail(c, "low-rank factor copy");

    const int dw = pad64(d.d_w), da = pad64(d.d_a), dv = pad64(d.d_v), dg = pad64(d.d_g);
    void *v_buf = v0 ? at(L.v) : (v0_out ? v0_out : at(L.v));   // the first layer's v is its v0
    auto problem = [&](int N, int K, int epi, const void *A, const float *mix, const void *W, void *D,
                       const float *bias) {
        GemmProblem q{};
        q.N = N; q.K = K; q.epi = epi; q.A = A; q.lda = K; q.mix = mix; q.W = W; q.D = D; q.ldd = N;
        q.bias = bias; q.v0 = v0;
        return q;
    };
    auto group = [&](int pro) {
        GemmGroup g{};
        g.M = int(M); g.pro = pro; g.x = x; g.last_x = last_x; g.T = Tn;
        g.err = dev_err;
        return g;
    };
    // every product of the mixed x in one launch: the square projections and the low-rank
    // first factors (tanh for the decay, sigmoid for the gate)
    GemmGroup gm = group(GEMM_MIX);
    gm.p[gm.nprob++] = problem(C, C, GEMM_STORE, nullptr, P.mr, P.Wr, at(L.r), nullptr);
    gm.p[gm.nprob++] = problem(C, C, GEMM_STORE, nullptr, P.mk, P.Wk, at(L.k), nullptr);
    gm.p[gm.nprob++] = problem(C, C, GEMM_STORE, nullptr, P.mv, P.Wv, v_buf, nullptr);
    gm.p[gm.nprob++] = problem(dw, C, GEMM_TANH, nullptr, P.mw, at(L.w1[0]), at(L.hw), nullptr);
    gm.p[gm.nprob++] = problem(da, C, GEMM_STORE, nullptr, P.ma, at(L.w1[1]), at(L.ha), nullptr);
    if (v0) gm.p[gm.nprob++] = problem(dv, C, GEMM_STORE, nullptr, P.mv, at(L.w1[2]), at(L.hv), nullptr);
    gm.p[gm.nprob++] = problem(dg, C, GEMM_SIGMOID, nullptr, P.mg, at(L.w1[3]), at(L.hg), nullptr);
    if ((c = launch_gemm_group(gm, dt, stream)) != cudaSuccess) return fail(c, "mixed projections");
    // the second factors: decay and rate logits with their biases, the value residual (layers
    // after the first; it reads v written above), the gate in fp32
    GemmGroup gp = group(GEMM_PLAIN);
    gp.p[gp.nprob++] = problem(C, dw, GEMM_BIAS, at(L.hw), nullptr, at(L.w2[0]), at(L.wl), P.w_bias);
    gp.p[gp.nprob++] = problem(C, da, GEMM_BIAS, at(L.ha), nullptr, at(L.w2[1]), at(L.al), P.a_bias);
    if (v0) gp.p[gp.nprob++] = problem(C, dv, GEMM_RESIDUAL, at(L.hv), nullptr, at(L.w2[2]), v_buf, P.v_bias);
    gp.p[gp.nprob++] = problem(C, dg, GEMM_F32, at(L.hg), nullptr, at(L.w2[3]), at(L.g), nullptr);
    if ((c = launch_gemm_group(gp, dt, stream)) != cudaSuccess) return fail(c, "low-rank second factors");
    // recurrence with its pre-processing and epilogue
    wkv7_status s;
    wkv7_opts o = opts;
    o.ln_w = P.ln_w; o.ln_b = P.ln_b; o.r_k = P.r_k;
    s = wkv7_forward_raw(B, Tn, d.H, d.N, dt, at(L.r), at(L.wl), at(L.k), v_buf, at(L.al), P.k_k, P.k_a, S,
                         static_cast<float *>(at(L.y)), S, &o, nullptr, 0, stream);
    if (s != WKV7_OK) {
        snprintf(err, err_len, "recurrence: %s", wkv7_last_error());
        return s;
    }
    // the gate, then the output projection; y * g goes to r's buffer (r has been consumed)
    if ((c = launch_gate_product(static_cast<const float *>(at(L.y)), static_cast<const float *>(at(L.g)), at(L.r),
                                 M * size_t(C), dt, stream)) != cudaSuccess)
        return fail(c, "gate product");
    GemmGroup go = group(GEMM_PLAIN);
    go.p[go.nprob++] = problem(C, C, GEMM_F32, at(L.r), nullptr, P.Wo, out, nullptr);
    if ((c = launch_gemm_group(go, dt, stream)) != cudaSuccess) return fail(c, "out = Wo (y g)");
    if (last_x_out) {
        last_kernel<T><<<grid_for(size_t(B) * C), 256, 0, stream>>>(static_cast<const T *>(x),
                                                                     static_cast<T *>(last_x_out), Tn, C,
                                                                     size_t(B) * C);
        if ((c = cudaGetLastError()) != cudaSuccess) return fail(c, "last-token copy");
    }
    return WKV7_OK;
}

cudaError_t launch_gate_product(const float *y, const float *g, void *out, size_t n, wkv7_dtype dt,
                                cudaStream_t stream) {
    const size_t n4 = n / 4;
    if (n % 4 != 0) return cudaErrorInvalidValue;
    if (n4 == 0) return cudaSuccess;
    const float4 *y4 = reinterpret_cast<const float4 *>(y), *g4 = reinterpret_cast<const float4 *>(g);
    if (dt == WKV7_BF16) gate_kernel<__nv_bfloat16><<<grid_for(n4), 256, 0, stream>>>(y4, g4, static_cast<__nv_bfloat16 *>(out), n4);
    else gate_kernel<float><<<grid_for(n4), 256, 0, stream>>>(y4, g4, static_cast<float *>(out), n4);
    return cudaGetLastError();
}

size_t layer_workspace(int B, int T, wkv7_dtype dt, const wkv7_layer_dims &d) {
    if (B <= 0 || T <= 0) return 0;
    return layer_plan(size_t(B) * T, d.H * d.N, d, dt == WKV7_BF16 ? 2 : 4).total;
}

wkv7_status layer_dispatch(int B, int T, wkv7_dtype dt, const wkv7_layer_dims &d, const wkv7_layer_params &P,
                           const void *x, const void *last_x, const void *v0, float *S, float *out, void *v0_out,
                           void *last_x_out, const wkv7_opts &opts, void *ws, cudaStream_t stream, char *err,
                           size_t err_len) {
    uint8_t *w = static_cast<uint8_t *>(ws);
    if (dt == WKV7_BF16)
        return layer_run<__nv_bfloat16>(B, T, d, P, x, last_x, v0, S, out, v0_out, last_x_out, opts, w, stream, err,
                                        err_len);
    return layer_run<float>(B, T, d, P, x, last_x, v0, S, out, v0_out, last_x_out, opts, w, stream, err, err_len);
}

}  // namespace wkv7
