// One RWKV-7 time-mixing layer over a sequence (RWKV-7 rebuttal page, the numpy time_mixing
// listing): token shift, the four square projections and the four low-rank paths as
// library GEMMs (cuBLASLt, fp32 accumulation, workspace from the caller), the element-wise
// steps between them as the kernels below, and the recurrence with its pre-processing and
// epilogue through wkv7_forward_raw (chunked tensor-core kernel for bf16, scan for fp32).
//
// Data flow for M = B*T token rows of C = H*N channels, in the layer dtype unless noted:
//   mix:   xm[j] = x + m_j (x_prev - x), j in r, w, k, v, a, g        (x_prev: token before)
//   GEMM:  r = xm_r Wr^T, k = xm_k Wk^T, v = xm_v Wv^T                 (v written to v0_out
//                                                                        in the first layer)
//   GEMM:  hw = xm_w Ww1 (fp32) -> tanh -> hw' ; w_logit = hw' Ww2 (fp32) + w_bias
//   GEMM:  ha = xm_a Wa1 ; a_logit = ha Wa2 (fp32) + a_bias
//   GEMM:  hv = xm_v Wv1 ; lv = hv Wv2 (fp32) ; v <- v + (v0 - v) sigmoid(lv + v_bias)
//   GEMM:  hg = xm_g Wg1 (fp32) -> sigmoid -> hg' ; g = hg' Wg2 (fp32)
//   WKV:   y = wkv7_forward_raw(r, w_logit, k, v, a_logit, k_k, k_a; S in place; epilogue)
//   out  = (y * g) Wo^T (fp32)
#include <cublasLt.h>

#include <cstdio>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"

namespace wkv7 {
namespace {

template <class T> struct Cvt;
template <> struct Cvt<float> {
    static __device__ __forceinline__ float load(const float *p) { return *p; }
    static __device__ __forceinline__ void store(float *p, float x) { *p = x; }
};
template <> struct Cvt<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

#define GRID_STRIDE(i, n) for (size_t i = blockIdx.x * size_t(blockDim.x) + threadIdx.x; i < (n); i += size_t(gridDim.x) * blockDim.x)

// Six token-shift mixes of every (b, t, c); the previous token of t = 0 is last_x (or 0).
template <class T>
__global__ void mix_table_kernel(const T *x, const T *last_x, const float *m0, const float *m1, const float *m2,
                                 const float *m3, const float *m4, const float *m5, T *o0, T *o1, T *o2, T *o3,
                                 T *o4, T *o5, int Tn, int C, size_t n) {
    GRID_STRIDE(i, n) {
        const int c = int(i % C);
        const size_t bt = i / C;
        const int t = int(bt % Tn);
        const float xi = Cvt<T>::load(x + i);
        float xp = 0.f;
        if (t > 0) xp = Cvt<T>::load(x + i - C);
        else if (last_x) xp = Cvt<T>::load(last_x + (bt / Tn) * C + c);
        const float dxp = xp - xi;
        Cvt<T>::store(o0 + i, fmaf(m0[c], dxp, xi));
        Cvt<T>::store(o1 + i, fmaf(m1[c], dxp, xi));
        Cvt<T>::store(o2 + i, fmaf(m2[c], dxp, xi));
        Cvt<T>::store(o3 + i, fmaf(m3[c], dxp, xi));
        Cvt<T>::store(o4 + i, fmaf(m4[c], dxp, xi));
        Cvt<T>::store(o5 + i, fmaf(m5[c], dxp, xi));
    }
}

// Element-wise activation of an fp32 GEMM result into the layer dtype: 0 tanh, 1 sigmoid.
template <class T>
__global__ void act_kernel(const float *in, T *out, int op, size_t n) {
    GRID_STRIDE(i, n) {
        const float z = in[i];
        Cvt<T>::store(out + i, op == 0 ? tanhf(z) : 1.f / (1.f + expf(-z)));
    }
}

// out = in + bias[c] in the layer dtype (the decay and rate logits).
template <class T>
__global__ void bias_kernel(const float *in, const float *bias, T *out, int C, size_t n) {
    GRID_STRIDE(i, n) Cvt<T>::store(out + i, in[i] + bias[i % C]);
}

// v <- v + (v0 - v) sigmoid(lv + v_bias): the value residual towards the first layer's values.
template <class T>
__global__ void residual_kernel(T *v, const T *v0, const float *lv, const float *bias, int C, size_t n) {
    GRID_STRIDE(i, n) {
        const float vi = Cvt<T>::load(v + i), s = 1.f / (1.f + expf(-(lv[i] + bias[i % C])));
        Cvt<T>::store(v + i, fmaf(Cvt<T>::load(v0 + i) - vi, s, vi));
    }
}

// out = y * g in the layer dtype (the gated readout before the output projection).
template <class T>
__global__ void gate_kernel(const float *y, const float *g, T *out, size_t n) {
    GRID_STRIDE(i, n) Cvt<T>::store(out + i, y[i] * g[i]);
}

// last_x_out[b] = x[b, T - 1].
template <class T>
__global__ void last_kernel(const T *x, T *out, int Tn, int C, size_t n) {
    GRID_STRIDE(i, n) out[i] = x[((i / C) * Tn + (Tn - 1)) * C + i % C];
}

unsigned grid_for(size_t n) { return unsigned(std::min<size_t>((n + 255) / 256, size_t(148) * 16)); }

// ---- cuBLASLt ------------------------------------------------------------------------------

cublasLtHandle_t lt_handle(cublasStatus_t *st) {
    static std::once_flag once;
    static cublasLtHandle_t h = nullptr;
    static cublasStatus_t s = CUBLAS_STATUS_SUCCESS;
    std::call_once(once, [] { s = cublasLtCreate(&h); });
    *st = s;
    return h;
}

// Row-major Y[M][Nout] (+)= X[M][K] * op(W): square projections store W as [Nout][K]
// (Y = X W^T, `w_out_major`), low-rank factors as [K][Nout] (Y = X W).
struct Gemm {
    const void *X, *W;
    void *Y;
    int M, K, Nout;
    bool w_out_major;
    cudaDataType_t in_t, out_t;
};

// A GEMM shape's cuBLASLt descriptors and chosen algorithm, made once per process and shape
// (descriptor creation and the heuristic query cost more host time than a small GEMM runs).
struct GemmPlan {
    cublasLtMatmulDesc_t desc = nullptr;
    cublasLtMatrixLayout_t la = nullptr, lb = nullptr, ld = nullptr;
    cublasLtMatmulAlgo_t algo{};
    cublasStatus_t status = CUBLAS_STATUS_NOT_INITIALIZED;
};

cublasStatus_t make_plan(cublasLtHandle_t h, const Gemm &g, size_t ws_bytes, GemmPlan &p) {
    const cublasOperation_t ta = g.w_out_major ? CUBLAS_OP_T : CUBLAS_OP_N, tb = CUBLAS_OP_N;
    cublasLtMatmulPreference_t pref = nullptr;
    cublasLtMatmulHeuristicResult_t heur{};
    int found = 0;
    cublasStatus_t st;
    do {
        if ((st = cublasLtMatmulDescCreate(&p.desc, CUBLAS_COMPUTE_32F, CUDA_R_32F))) break;
        if ((st = cublasLtMatmulDescSetAttribute(p.desc, CUBLASLT_MATMUL_DESC_TRANSA, &ta, sizeof(ta)))) break;
        if ((st = cublasLtMatmulDescSetAttribute(p.desc, CUBLASLT_MATMUL_DESC_TRANSB, &tb, sizeof(tb)))) break;
        // column-major view: Y^T[Nout][M] = op(A)[Nout][K] * X^T[K][M]
        if (g.w_out_major) st = cublasLtMatrixLayoutCreate(&p.la, g.in_t, g.K, g.Nout, g.K);
        else st = cublasLtMatrixLayoutCreate(&p.la, g.in_t, g.Nout, g.K, g.Nout);
        if (st) break;
        if ((st = cublasLtMatrixLayoutCreate(&p.lb, g.in_t, g.K, g.M, g.K))) break;
        if ((st = cublasLtMatrixLayoutCreate(&p.ld, g.out_t, g.Nout, g.M, g.Nout))) break;
        if ((st = cublasLtMatmulPreferenceCreate(&pref))) break;
        if ((st = cublasLtMatmulPreferenceSetAttribute(pref, CUBLASLT_MATMUL_PREF_MAX_WORKSPACE_BYTES, &ws_bytes,
                                                       sizeof(ws_bytes))))
            break;
        if ((st = cublasLtMatmulAlgoGetHeuristic(h, p.desc, p.la, p.lb, p.ld, p.ld, pref, 1, &heur, &found))) break;
        if (found == 0) st = CUBLAS_STATUS_NOT_SUPPORTED;
        else p.algo = heur.algo;
    } while (false);
    if (pref) cublasLtMatmulPreferenceDestroy(pref);
    return st;
}

cublasStatus_t run_gemm(const Gemm &g, void *ws, size_t ws_bytes, cudaStream_t stream) {
    cublasStatus_t st;
    cublasLtHandle_t h = lt_handle(&st);
    if (st != CUBLAS_STATUS_SUCCESS) return st;
    typedef std::tuple<int, int, int, bool, int, int, int> Key;   // shape, types, device
    static std::mutex mu;
    static std::map<Key, GemmPlan> plans;
    int dev = 0;
    cudaGetDevice(&dev);
    const Key key(g.M, g.K, g.Nout, g.w_out_major, int(g.in_t), int(g.out_t), dev);
    GemmPlan *p;
    {
        std::lock_guard<std::mutex> lock(mu);
        p = &plans[key];
        if (p->status == CUBLAS_STATUS_NOT_INITIALIZED) p->status = make_plan(h, g, ws_bytes, *p);
    }
    if (p->status != CUBLAS_STATUS_SUCCESS) return p->status;
    const float alpha = 1.f, beta = 0.f;
    return cublasLtMatmul(h, p->desc, &alpha, g.W, p->la, g.X, p->lb, &beta, g.Y, p->ld, g.Y, p->ld, &p->algo, ws,
                          ws_bytes, stream);
}

constexpr size_t kGemmWorkspace = size_t(32) << 20;

// Byte offsets of the layer's intermediates in the caller's workspace (256-byte aligned).
struct LayerPlan {
    size_t xm[6], r, k, v, wl, al, hw32, hw, ha, hv, hg32, hg, lw32, la32, lv32, g32, y, yg, gemm, total;
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
    for (int j = 0; j < 6; ++j) p.xm[j] = take(mc * e);
    p.r = take(mc * e); p.k = take(mc * e); p.v = take(mc * e); p.wl = take(mc * e); p.al = take(mc * e);
    p.hw32 = take(M * d.d_w * 4); p.hw = take(M * d.d_w * e);
    p.ha = take(M * d.d_a * e); p.hv = take(M * d.d_v * e);
    p.hg32 = take(M * d.d_g * 4); p.hg = take(M * d.d_g * e);
    p.lw32 = take(mc * 4); p.la32 = take(mc * 4); p.lv32 = take(mc * 4); p.g32 = take(mc * 4);
    p.y = take(mc * 4); p.yg = take(mc * e);
    p.gemm = take(kGemmWorkspace);
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
    const size_t M = size_t(B) * Tn, mc = M * size_t(C), e = sizeof(T);
    const LayerPlan L = layer_plan(M, C, d, e);
    const cudaDataType_t dt_t = sizeof(T) == 2 ? CUDA_R_16BF : CUDA_R_32F;
    auto at = [&](size_t off) { return static_cast<void *>(ws + off); };
    auto cuda_err = [&](cudaError_t c, const char *what) {
        snprintf(err, err_len, "%s: %s", what, cudaGetErrorString(c));
        return WKV7_ERR_CUDA;
    };
    auto gemm = [&](const void *X, const void *W, void *Y, int K, int Nout, bool out_major, cudaDataType_t ot,
                    const char *what) -> wkv7_status {
        const cublasStatus_t st = run_gemm(Gemm{X, W, Y, int(M), K, Nout, out_major, dt_t, ot}, at(L.gemm),
                                           kGemmWorkspace, stream);
        if (st == CUBLAS_STATUS_SUCCESS) return WKV7_OK;
        snprintf(err, err_len, "cuBLASLt GEMM %s failed with status %d", what, int(st));
        return WKV7_ERR_CUDA;
    };
    wkv7_status s;
    cudaError_t c;
    // token shift
    mix_table_kernel<T><<<grid_for(mc), 256, 0, stream>>>(
        static_cast<const T *>(x), static_cast<const T *>(last_x), P.mr, P.mw, P.mk, P.mv, P.ma, P.mg,
        static_cast<T *>(at(L.xm[0])), static_cast<T *>(at(L.xm[1])), static_cast<T *>(at(L.xm[2])),
        static_cast<T *>(at(L.xm[3])), static_cast<T *>(at(L.xm[4])), static_cast<T *>(at(L.xm[5])), Tn, C, mc);
    if ((c = cudaGetLastError()) != cudaSuccess) return cuda_err(c, "token-shift launch");
    enum { XR = 0, XW, XK, XV, XA, XG };
    void *v_buf = v0 ? at(L.v) : (v0_out ? v0_out : at(L.v));   // the first layer's v is its v0
    if ((s = gemm(at(L.xm[XR]), P.Wr, at(L.r), C, C, true, dt_t, "r = Wr x_r"))) return s;
    if ((s = gemm(at(L.xm[XK]), P.Wk, at(L.k), C, C, true, dt_t, "k = Wk x_k"))) return s;
    if ((s = gemm(at(L.xm[XV]), P.Wv, v_buf, C, C, true, dt_t, "v = Wv x_v"))) return s;
    // decay logits
    if ((s = gemm(at(L.xm[XW]), P.Ww1, at(L.hw32), C, d.d_w, false, CUDA_R_32F, "x_w Ww1"))) return s;
    act_kernel<T><<<grid_for(M * d.d_w), 256, 0, stream>>>(static_cast<const float *>(at(L.hw32)),
                                                           static_cast<T *>(at(L.hw)), 0, M * d.d_w);
    if ((s = gemm(at(L.hw), P.Ww2, at(L.lw32), d.d_w, C, false, CUDA_R_32F, "tanh(.) Ww2"))) return s;
    bias_kernel<T><<<grid_for(mc), 256, 0, stream>>>(static_cast<const float *>(at(L.lw32)), P.w_bias,
                                                     static_cast<T *>(at(L.wl)), C, mc);
    // value residual (layers after the first)
    if (v0) {
        if ((s = gemm(at(L.xm[XV]), P.Wv1, at(L.hv), C, d.d_v, false, dt_t, "x_v Wv1"))) return s;
        if ((s = gemm(at(L.hv), P.Wv2, at(L.lv32), d.d_v, C, false, CUDA_R_32F, "(.) Wv2"))) return s;
        residual_kernel<T><<<grid_for(mc), 256, 0, stream>>>(static_cast<T *>(v_buf), static_cast<const T *>(v0),
                                                             static_cast<const float *>(at(L.lv32)), P.v_bias, C, mc);
    }
    // rate logits
    if ((s = gemm(at(L.xm[XA]), P.Wa1, at(L.ha), C, d.d_a, false, dt_t, "x_a Wa1"))) return s;
    if ((s = gemm(at(L.ha), P.Wa2, at(L.la32), d.d_a, C, false, CUDA_R_32F, "(.) Wa2"))) return s;
    bias_kernel<T><<<grid_for(mc), 256, 0, stream>>>(static_cast<const float *>(at(L.la32)), P.a_bias,
                                                     static_cast<T *>(at(L.al)), C, mc);
    // gate
    if ((s = gemm(at(L.xm[XG]), P.Wg1, at(L.hg32), C, d.d_g, false, CUDA_R_32F, "x_g Wg1"))) return s;
    act_kernel<T><<<grid_for(M * d.d_g), 256, 0, stream>>>(static_cast<const float *>(at(L.hg32)),
                                                           static_cast<T *>(at(L.hg)), 1, M * d.d_g);
    if ((s = gemm(at(L.hg), P.Wg2, at(L.g32), d.d_g, C, false, CUDA_R_32F, "sigmoid(.) Wg2"))) return s;
    if ((c = cudaGetLastError()) != cudaSuccess) return cuda_err(c, "element-wise launch");
    // recurrence with its pre-processing and epilogue
    wkv7_opts o = opts;
    o.ln_w = P.ln_w; o.ln_b = P.ln_b; o.r_k = P.r_k;
    s = wkv7_forward_raw(B, Tn, d.H, d.N, sizeof(T) == 2 ? WKV7_BF16 : WKV7_F32, at(L.r), at(L.wl), at(L.k), v_buf,
                         at(L.al), P.k_k, P.k_a, S, static_cast<float *>(at(L.y)), S, &o, nullptr, 0, stream);
    if (s != WKV7_OK) {
        snprintf(err, err_len, "recurrence: %s", wkv7_last_error());
        return s;
    }
    gate_kernel<T><<<grid_for(mc), 256, 0, stream>>>(static_cast<const float *>(at(L.y)),
                                                     static_cast<const float *>(at(L.g32)),
                                                     static_cast<T *>(at(L.yg)), mc);
    if ((s = gemm(at(L.yg), P.Wo, out, C, C, true, CUDA_R_32F, "out = Wo (y g)"))) return s;
    if (last_x_out) {
        last_kernel<T><<<grid_for(size_t(B) * C), 256, 0, stream>>>(static_cast<const T *>(x),
                                                                     static_cast<T *>(last_x_out), Tn, C,
                                                                     size_t(B) * C);
    }
    if ((c = cudaGetLastError()) != cudaSuccess) return cuda_err(c, "element-wise launch");
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
