// Internal interface of the epilogue's backward (epilogue_bwd.cu).
#pragma once

#include "common.cuh"

namespace wkv7 {

// Backward of the group_norm + bonus epilogue for every (b, t, h) row of N channels: dy, and the
// bonus's dr, dk, dv ([B][T][H][N] fp32, overwritten); dln_w, dln_b, dr_k ([H][N] fp32, sums over
// B and T, overwritten). ws: epilogue_backward_partials(B, T, H, N) floats (one partial sum of the
// three parameter gradients per block of kEpiRows rows of a head), written before they are read.
struct EpiBwdArgs {
    int B, T, H, N;
    wkv7_dtype dt;
    const float *y;
    const void *r, *k, *v;
    const float *ln_w, *ln_b, *r_k;
    float eps;
    const float *dout;
    float *dy, *dr, *dk, *dv;
    float *dln_w, *dln_b, *dr_k;
    float *ws;
    cudaStream_t stream;
};
constexpr int kEpiRows = 64;   // (b, t) rows of one head per CTA
inline size_t epilogue_backward_partials(int B, int T, int H, int N) {
    const size_t rows = size_t(B) * T;
    return (rows + kEpiRows - 1) / kEpiRows * size_t(H) * 3 * N;
}
cudaError_t launch_epilogue_backward(const EpiBwdArgs &a);

}  // namespace wkv7
