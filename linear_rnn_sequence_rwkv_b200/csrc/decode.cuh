// Options of the decode step beyond the prepared-input recurrence: raw inputs (the pre-processing
// of the time-mixing values fused into the load) and the fused group_norm + bonus epilogue.
#pragma once

#include "common.cuh"

namespace wkv7 {

struct DecOpts {
    const float *k_k = nullptr;    // non-NULL: raw inputs (w, a hold the decay and rate logits,
    const float *k_a = nullptr;    // k the key before its update; kk is derived); [H][N] fp32
    const float *ln_w = nullptr;   // epilogue: all three [H][N] fp32, or all NULL (off)
    const float *ln_b = nullptr;
    const float *r_k = nullptr;
    float gn_eps = 64e-5f;
};

cudaError_t launch_decode_ex(const DecArgs &p, const DecOpts &o);

}  // namespace wkv7
