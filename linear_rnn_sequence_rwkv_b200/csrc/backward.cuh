// The backward pass at head sizes 64 and 128 (the entries of common.cuh take N = 64).
#pragma once

#include "common.cuh"

namespace wkv7 {

cudaError_t launch_backward_n(const BwdArgs &p, int N);                    // T >= 1; N 64 or 128
size_t backward_checkpoint_bytes_n(int B, int T, int H, int N, int snap_every);

}  // namespace wkv7
