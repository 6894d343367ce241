// Shared device helpers and the internal launcher interface of the WKV-7 library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "wkv7.h"

namespace wkv7 {

constexpr int kN = WKV7_HEAD_SIZE;   // head size: the state of one (b, h) is kN x kN fp32

// Arguments of one forward call after validation (device pointers, caller's stream).
struct FwdArgs {
    int B, T, H;
    int N;                 // head size: 64, or 128 on the scan path
    wkv7_dtype dt;
    const void *r, *w, *k, *v, *kk, *a;
    const float *S0;       // nullable: zero initial state
    float *y;
    float *S_T;            // nullable
    int snap_every;        // 0 = off
    float *snaps;          // [B][T/snap_every][H][N][N]
    const float *ln_w, *ln_b, *r_k;   // all null = no epilogue
    bool raw;              // w and a hold the decay / rate logits, k the raw key; kk unused
    const float *k_k, *k_a;   // raw: [H][N] removal-key scale and key-update rate (k_a nullable)
    float gn_eps;
    int chunk;
    int segments;          // CTAs per (b, h) on the chunked path; 0 = automatic
    unsigned int handoff_wait_us;   // split mode: limit of the hand-off waits (0 = default)
    int withhold_handoff;  // split mode, failure-path test: withhold the first hand-off of each head
    void *ws;
    size_t ws_bytes;
    cudaStream_t stream;
};

struct DecArgs {
    int B, H;
    int N;                 // head size: 64 or 128
    wkv7_dtype dt;
    const void *r, *w, *k, *v, *kk, *a;
    float *S;
    float *y;
    cudaStream_t stream;
};

// Arguments of one backward call after validation.
struct BwdArgs {
    int B, T, H;
    wkv7_dtype dt;
    const void *r, *w, *k, *v, *kk, *a;
    const float *S0;        // nullable: zero initial state
    const float *snaps;     // the forward's states every snap_every tokens, or null (snap_every 0)
    int snap_every;
    const float *dy;        // [B][T][H][N] gradient of y
    const float *dS_T;      // nullable: no gradient on the final state
    float *dr, *dw, *dk, *dv, *dkk, *da;   // [B][T][H][N]
    float *dS0;             // nullable
    float *ws;              // backward_checkpoint_bytes(...) of scratch
    cudaStream_t stream;
};

// Launchers (each returns the launch status; no synchronisation).
cudaError_t launch_seq(const FwdArgs &p);
cudaError_t launch_epilogue(const FwdArgs &p);
cudaError_t launch_decode(const DecArgs &p);
cudaError_t launch_copy_state(const FwdArgs &p);   // T == 0: S_T <- S0 (or zeros)
cudaError_t launch_backward(const BwdArgs &p);     // T >= 1
size_t backward_checkpoint_bytes(int B, int T, int H, int snap_every);
size_t backward_static_scratch_bytes();             // capacity of the module's static scratch
// One time-mixing layer (validated arguments): launches on `stream`, error text into err.
size_t layer_workspace(int B, int T, wkv7_dtype dt, const wkv7_layer_dims &d);
wkv7_status layer_dispatch(int B, int T, wkv7_dtype dt, const wkv7_layer_dims &d, const wkv7_layer_params &P,
                           const void *x, const void *last_x, const void *v0, float *S, float *out, void *v0_out,
                           void *last_x_out, const wkv7_opts &opts, void *ws, cudaStream_t stream, char *err,
                           size_t err_len);
cudaError_t backward_static_scratch(void **ptr);    // its address on the current device
bool chunk_supported(const FwdArgs &p);            // bf16 inputs, snapshots on chunk boundaries
cudaError_t launch_chunk(const FwdArgs &p);        // chunked prefill on tcgen05 (epilogue fused)
// CTAs per (b, h) of launch_chunk's last launch, and its number of launches (1 or 2)
cudaError_t chunk_segments(const FwdArgs &p, int *segments, int *launches = nullptr);
// Synchronises `stream` and reads the device error word (bounded waits that gave up).
cudaError_t read_device_error(cudaStream_t stream, unsigned int *value, bool clear);
// Records the calling thread's error text (wkv7_last_error) and returns s.
wkv7_status set_error(wkv7_status s, const char *fmt, ...);
// The device error word of the current device (set by a bounded wait that gave up).
cudaError_t device_error_word(unsigned int **ptr);
// Peak-rate probes: launch on `stream`, *flops = the floating-point operations of the launch.
cudaError_t launch_fma_peak(int blocks, int iters, cudaStream_t stream, double *flops);
cudaError_t launch_tf32_mma_peak(int n, int iters, cudaStream_t stream, double *flops);
// Raises `kernel`'s dynamic shared-memory limit to `bytes` on the current device. The attribute
// belongs to the device's context, so it is set once per (device, kernel); failures are not
// remembered (the next call tries again).
cudaError_t allow_dynamic_smem(const void *kernel, int bytes);

// ---- device helpers -------------------------------------------------------------------------

__device__ __forceinline__ float bf16_lo(uint32_t packed) { return __uint_as_float(packed << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t packed) { return __uint_as_float(packed & 0xffff0000u); }

// Four consecutive elements starting at p (16-byte aligned for float, 8-byte for bf16).
__device__ __forceinline__ float4 load4(const float *p) { return __ldg(reinterpret_cast<const float4 *>(p)); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p));
    return make_float4(bf16_lo(u.x), bf16_hi(u.x), bf16_lo(u.y), bf16_hi(u.y));
}
__device__ __forceinline__ float load1(const float *p) { return __ldg(p); }
__device__ __forceinline__ float load1(const __nv_bfloat16 *p) { return __bfloat162float(*p); }

__device__ __forceinline__ float dot4(float4 a, float4 b) {
    return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

}  // namespace wkv7
