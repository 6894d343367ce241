// Internal interface of the time-mixing layer's kernels (gemm.cu, layer.cu).
#pragma once

#include "common.cuh"

namespace wkv7 {

// The projections of the time-mixing layer (gemm.cu): one launch computes up to
// kGemmMaxProblems products D_i[M][N_i] = op(A)[M][K_i] * W_i[N_i][K_i]^T that share the row count
// M and the operand preparation op (GEMM_PLAIN: A_i itself; GEMM_MIX: the token-shift mix of x
// with the problem's own mix vector). Each problem's store applies its own GEMM_STORE / TANH /
// SIGMOID / BIAS / RESIDUAL (layer dtype out) or GEMM_F32 (fp32 out). All matrices are row-major
// in the layer dtype unless noted; bf16 needs K_i and N_i multiples of 64, and takes the value
// residual in PLAIN launches only, with one v0 per launch.
enum { GEMM_PLAIN = 0, GEMM_MIX = 1 };
enum { GEMM_STORE = 0, GEMM_TANH = 1, GEMM_SIGMOID = 2, GEMM_BIAS = 3, GEMM_RESIDUAL = 4, GEMM_F32 = 5 };
constexpr int kGemmMaxProblems = 7;
struct GemmProblem {
    int N, K;
    int epi;
    const void *A;          // PLAIN: [M][lda]
    int lda;
    const float *mix;       // MIX: [K] fp32
    const void *W;          // [N][K]
    void *D;                // [M][ldd]; RESIDUAL reads v from it
    int ldd;
    const float *bias;      // [N] fp32 (BIAS, RESIDUAL)
    const void *v0;         // RESIDUAL: [M][ldd]
};
struct GemmGroup {
    int M, pro, nprob;
    const void *x;          // MIX: x [M][K] (rows b * T + t); last_x [M / T][K] or null (zeros)
    const void *last_x;
    int T;
    GemmProblem p[kGemmMaxProblems];
    unsigned int *err;      // device error word (a bounded wait that gave up)
};
cudaError_t launch_gemm_group(const GemmGroup &g, wkv7_dtype dt, cudaStream_t stream);
// out[i] = y[i] * g[i] (fp32 in, layer dtype out), i < n.
cudaError_t launch_gate_product(const float *y, const float *g, void *out, size_t n, wkv7_dtype dt,
                                cudaStream_t stream);
// Up to kMaxPadCopies copies in one launch: out [out_rows][out_cols] = the transpose of
// in [rows][cols], zero outside it.
struct PadCopy {
    const void *in;
    void *out;
    int rows, cols, out_rows, out_cols;
};
constexpr int kMaxPadCopies = 8;
cudaError_t launch_transpose_pad(const PadCopy *copies, int n, wkv7_dtype dt, cudaStream_t stream);

}  // namespace wkv7
