// One RWKV-7 time-mixing layer over a sequence (RWKV-7 rebuttal page, the numpy time_mixing
// listing): every projection is this library's GEMM (gemm.cu) with the token-shift mix fused
// into its operand load and the bias, activation or value residual fused into its store; the
// recurrence with its pre-processing and epilogue runs through wkv7_forward_raw (chunked
// tensor-core kernel for bf16, scan for fp32); the gate multiplies the readout inside the
// output projection's operand load.
//
// Data flow for M = B*T token rows of C = H*N channels, in the layer dtype unless noted
// (x_m = x + m (x_prev - x), x_prev the token before):
//   r = x_r Wr^T, k = x_k Wk^T, v = x_v Wv^T          (the first layer writes v to v0_out)
//   hw = tanh(x_w Ww1);   w_logit = hw Ww2 + w_bias
//   ha = x_a Wa1;         a_logit = ha Wa2 + a_bias
//   hv = x_v Wv1;         v <- v + (v0 - v) sigmoid(hv Wv2 + v_bias)     (layers after the first)
//   hg = sigmoid(x_g Wg1); g = hg Wg2 (fp32)
//   y = wkv7_forward_raw(r, w_logit, k, v, a_logit, k_k, k_a; S in place; epilogue) (fp32)
//   out = (y * g) Wo^T (fp32)
// The low-rank factors are stored [in][out] (applied as x W); each call copies them transposed
// and zero-padded to a multiple of 64 into the workspace, so that every GEMM takes W as
// [out][in] with K and N multiples of 64 (the padding adds exact zeros).
#include <algorithm>
#include <cstdio>

#include "common.cuh"

namespace wkv7 {
namespace {

#define GRID_STRIDE(i, n) for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < (n); i += size_t(gridDim.x) * blockDim.x)

// last_x_out[b] = x[b, T - 1].
template <class T>
__global__ void last_kernel(const T *x, T *out, int Tn, int C, size_t n) {
    GRID_STRIDE(i, n) out[i] = x[((i / C) * Tn + (Tn - 1)) * C + i % C];
}

unsigned grid_for(size_t n) { return unsigned(std::min<size_t>((n + 255) / 256, size_t(148) * 16)); }

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
    // the low-rank factors, transposed to [out][in] and zero-padded to multiples of 64
    const void *w1[4] = {P.Ww1, P.Wa1, P.Wv1, P.Wg1}, *w2[4] = {P.Ww2, P.Wa2, P.Wv2, P.Wg2};
    const int dims[4] = {d.d_w, d.d_a, d.d_v, d.d_g};
    for (int i = 0; i < 4; ++i) {
        if (i == 2 && !v0) continue;   // the value residual's factors are unused in the first layer
        const int dp = pad64(dims[i]);
        if ((c = launch_transpose_pad(w1[i], at(L.w1[i]), C, dims[i], dp, C, dt, stream)) != cudaSuccess ||
            (c = launch_transpose_pad(w2[i], at(L.w2[i]), dims[i], C, C, dp, dt, stream)) != cudaSuccess)
            return fail(c, "low-rank factor copy");
    }
    auto gemm = [&](int pro, const float *mix, const void *A, int lda, const void *W, int N, int K, int epi, void *D,
                    const float *bias, const char *what) -> wkv7_status {
        GemmArgs g{};
        g.M = int(M); g.N = N; g.K = K; g.pro = pro;
        g.A = A; g.lda = lda;
        g.x = x; g.last_x = last_x; g.mix = mix; g.T = Tn;
        g.y = static_cast<const float *>(at(L.y)); g.g = at(L.g);
        g.W = W; g.epi = epi; g.D = D; g.ldd = N; g.bias = bias; g.v0 = v0; g.D2 = nullptr; g.err = dev_err;
        const cudaError_t ce = launch_gemm(g, dt, stream);
        return ce == cudaSuccess ? WKV7_OK : fail(ce, what);
    };
    const int dw = pad64(d.d_w), da = pad64(d.d_a), dv = pad64(d.d_v), dg = pad64(d.d_g);
    void *v_buf = v0 ? at(L.v) : (v0_out ? v0_out : at(L.v));   // the first layer's v is its v0
    wkv7_status s;
    if ((s = gemm(GEMM_MIX, P.mr, nullptr, 0, P.Wr, C, C, GEMM_STORE, at(L.r), nullptr, "r = Wr x_r"))) return s;
    if ((s = gemm(GEMM_MIX, P.mk, nullptr, 0, P.Wk, C, C, GEMM_STORE, at(L.k), nullptr, "k = Wk x_k"))) return s;
    if ((s = gemm(GEMM_MIX, P.mv, nullptr, 0, P.Wv, C, C, GEMM_STORE, v_buf, nullptr, "v = Wv x_v"))) return s;
    // decay logits
    if ((s = gemm(GEMM_MIX, P.mw, nullptr, 0, at(L.w1[0]), dw, C, GEMM_TANH, at(L.hw), nullptr, "tanh(x_w Ww1)")))
        return s;
    if ((s = gemm(GEMM_PLAIN, nullptr, at(L.hw), dw, at(L.w2[0]), C, dw, GEMM_BIAS, at(L.wl), P.w_bias,
                  "(.) Ww2 + w_bias")))
        return s;
    // value residual (layers after the first)
    if (v0) {
        if ((s = gemm(GEMM_MIX, P.mv, nullptr, 0, at(L.w1[2]), dv, C, GEMM_STORE, at(L.hv), nullptr, "x_v Wv1")))
            return s;
        if ((s = gemm(GEMM_PLAIN, nullptr, at(L.hv), dv, at(L.w2[2]), C, dv, GEMM_RESIDUAL, v_buf, P.v_bias,
                      "value residual")))
            return s;
    }
    // rate logits
    if ((s = gemm(GEMM_MIX, P.ma, nullptr, 0, at(L.w1[1]), da, C, GEMM_STORE, at(L.ha), nullptr, "x_a Wa1"))) return s;
    if ((s = gemm(GEMM_PLAIN, nullptr, at(L.ha), da, at(L.w2[1]), C, da, GEMM_BIAS, at(L.al), P.a_bias,
                  "(.) Wa2 + a_bias")))
        return s;
    // gate (fp32)
    if ((s = gemm(GEMM_MIX, P.mg, nullptr, 0, at(L.w1[3]), dg, C, GEMM_SIGMOID, at(L.hg), nullptr,
                  "sigmoid(x_g Wg1)")))
        return s;
    if ((s = gemm(GEMM_PLAIN, nullptr, at(L.hg), dg, at(L.w2[3]), C, dg, GEMM_F32, at(L.g), nullptr, "(.) Wg2")))
        return s;
    // recurrence with its pre-processing and epilogue
    wkv7_opts o = opts;
    o.ln_w = P.ln_w; o.ln_b = P.ln_b; o.r_k = P.r_k;
    s = wkv7_forward_raw(B, Tn, d.H, d.N, dt, at(L.r), at(L.wl), at(L.k), v_buf, at(L.al), P.k_k, P.k_a, S,
                         static_cast<float *>(at(L.y)), S, &o, nullptr, 0, stream);
    if (s != WKV7_OK) {
        snprintf(err, err_len, "recurrence: %s", wkv7_last_error());
        return s;
    }
    if ((s = gemm(GEMM_GATE, nullptr, nullptr, 0, P.Wo, C, C, GEMM_F32, out, nullptr, "out = Wo (y g)"))) return s;
    if (last_x_out) {
        last_kernel<T><<<grid_for(size_t(B) * C), 256, 0, stream>>>(static_cast<const T *>(x),
                                                                     static_cast<T *>(last_x_out), Tn, C,
                                                                     size_t(B) * C);
        if ((c = cudaGetLastError()) != cudaSuccess) return fail(c, "last-token copy");
    }
    return WKV7_OK;
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
