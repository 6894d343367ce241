"""Seeded synthetic inputs for the WKV-7 recurrence.

This module is shared by the CUDA path's tests/benchmarks and by the CPU oracle's
tests. It draws random tensors with the shapes and value ranges of the workloads
described for RWKV-7 "Goose" and performs only the *input pre-processing* that the
pages place upstream of the WKV kernel (decay parametrisation, learning-rate sigmoid,
removal-key normalisation). It contains none of the recurrence's arithmetic.

Recipe (RWKV-7 rebuttal page, the numpy ``time_mixing`` listing; RWKV-7 paper
summary, section F "Numerical stability"):

* r, k, v ~ N(0, 1)
* z ~ N(mu_z, 1) (mu_z = 0, or 2 for the long-context workload);
  w = exp(-sigmoid(z) / sqrt(e))  -> w in (exp(-e^-1/2), 1) = (0.5452, 1)
* a = sigmoid(N(0, 1))            -> a in (0, 1)
* k_k ~ U(0.5, 1.5), one [H, N] parameter; kk = (k * k_k) / max(||k * k_k||_2, 1e-12)
  per head (the replacement-rate booster k_a is taken as 0, so the kernel's k is k)
* S0 = 0, or ~ N(0, 0.1^2) where the workload says so
* epilogue parameters (group_norm affine + bonus): ln_w ~ 1 + N(0, 0.1^2),
  ln_b ~ N(0, 0.1^2), r_k ~ N(0, 0.5^2), all fp32 [H, N]

All draws are fp32 from one seeded ``torch.Generator`` in a fixed order; bf16
workloads are then rounded to nearest-even with ``.to(torch.bfloat16)``. Both
sides of every comparison consume the same bytes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

HEAD_SIZE = 64
SEED_BASE = 20260

# Lower end of the decay range: exp(-e^{-1/2}) (RWKV-7 paper summary, section F).
W_MIN = math.exp(-math.exp(-0.5))


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, dtype and draw recipe."""

    cid: int
    name: str
    B: int
    T: int
    H: int
    N: int = HEAD_SIZE
    dtype: str = "bf16"          # "bf16" or "f32" for r,w,k,v,kk,a
    s0: str = "zeros"            # "zeros" | "normal"  (std 0.1)
    z_mean: float = 0.0          # mean of the decay logit
    epilogue: bool = False       # group_norm + bonus fused after the readout
    snap_every: int = 0          # state snapshot interval (0 = off)
    decode_steps: int = 0        # >0: T tokens are consumed one decode step at a time
    chunks: tuple = field(default=(64,))

    @property
    def token_heads(self) -> int:
        return self.B * self.T * self.H


WORKLOADS = {
    0: Workload(0, "tiny-f32 B1 T64 H2", B=1, T=64, H=2, dtype="f32"),
    1: Workload(1, "prefill-0.19B B8 T1024 H12", B=8, T=1024, H=12, s0="normal"),
    2: Workload(2, "prefill-1.5B B16 T4096 H32 +epilogue", B=16, T=4096, H=32,
                epilogue=True, chunks=(16, 32, 64)),
    3: Workload(3, "decode-2.9B B256 H40 x128 steps", B=256, T=128, H=40, decode_steps=128),
    4: Workload(4, "long-context B1 T65536 H40 z~N(2,1)", B=1, T=65536, H=40, z_mean=2.0,
                snap_every=4096),
}


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def make_inputs(wl: Workload, *, seed: int | None = None, device: str = "cpu",
                B: int | None = None, T: int | None = None, H: int | None = None,
                s0: str | None = None, dtype: str | None = None) -> dict:
    """Draw the inputs of workload ``wl`` (optionally with overridden sizes).

    Returns a dict with r, w, k, v, kk, a ([B, T, H, N] in the workload dtype,
    contiguous), S0 ([B, H, N, N] fp32 or None) and, when the workload has the
    epilogue, ln_w, ln_b, r_k ([H, N] fp32).
    """
    B = wl.B if B is None else B
    T = wl.T if T is None else T
    H = wl.H if H is None else H
    N = wl.N
    s0 = wl.s0 if s0 is None else s0
    dt = torch_dtype(wl.dtype if dtype is None else dtype)
    g = torch.Generator(device=device)
    g.manual_seed(SEED_BASE + wl.cid if seed is None else seed)
    shape = (B, T, H, N)

    def randn(*s):
        return torch.randn(*s, generator=g, device=device, dtype=torch.float32)

    def rand(*s):
        return torch.rand(*s, generator=g, device=device, dtype=torch.float32)

    r = randn(*shape)
    k = randn(*shape)
    v = randn(*shape)
    z = randn(*shape) + wl.z_mean
    w = torch.exp(-torch.sigmoid(z) / math.sqrt(math.e))
    del z
    a = torch.sigmoid(randn(*shape))
    k_k = 0.5 + rand(H, N)
    kk = k * k_k
    kk = kk / torch.clamp(torch.linalg.vector_norm(kk, dim=-1, keepdim=True), min=1e-12)
    out = {}
    for name, t in (("r", r), ("w", w), ("k", k), ("v", v), ("kk", kk), ("a", a)):
        out[name] = t.to(dt).contiguous()
    if s0 == "normal":
        out["S0"] = (0.1 * randn(B, H, N, N)).contiguous()
    elif s0 == "zeros":
        out["S0"] = None
    else:
        raise ValueError(f"unknown S0 recipe {s0!r}")
    if wl.epilogue:
        out["ln_w"] = (1.0 + 0.1 * randn(H, N)).contiguous()
        out["ln_b"] = (0.1 * randn(H, N)).contiguous()
        out["r_k"] = (0.5 * randn(H, N)).contiguous()
    return out


def make_raw_inputs(wl: Workload, *, seed: int | None = None, device: str = "cpu",
                    B: int | None = None, T: int | None = None, H: int | None = None,
                    s0: str | None = None, dtype: str | None = None, k_a: bool = True) -> dict:
    """The same workload's draws *before* the pre-processing, for the path that fuses it
    into the kernel: r, w_logit (= z), k, v, a_logit ([B, T, H, N] in the workload dtype),
    k_k ~ U(0.5, 1.5) and k_a ~ U(0, 1) (zeros if ``k_a`` is False) as [H, N] fp32, S0 and
    the epilogue parameters as in ``make_inputs``. No arithmetic of the method is applied.
    """
    B = wl.B if B is None else B
    T = wl.T if T is None else T
    H = wl.H if H is None else H
    N = wl.N
    s0 = wl.s0 if s0 is None else s0
    dt = torch_dtype(wl.dtype if dtype is None else dtype)
    g = torch.Generator(device=device)
    g.manual_seed(SEED_BASE + 500 + wl.cid if seed is None else seed)
    shape = (B, T, H, N)

    def randn(*s):
        return torch.randn(*s, generator=g, device=device, dtype=torch.float32)

    def rand(*s):
        return torch.rand(*s, generator=g, device=device, dtype=torch.float32)

    out = {}
    for name in ("r", "k", "v"):
        out[name] = randn(*shape).to(dt).contiguous()
    out["w_logit"] = (randn(*shape) + wl.z_mean).to(dt).contiguous()
    out["a_logit"] = randn(*shape).to(dt).contiguous()
    out["k_k"] = (0.5 + rand(H, N)).contiguous()
    out["k_a"] = rand(H, N).contiguous() if k_a else torch.zeros(H, N, device=device)
    if s0 == "normal":
        out["S0"] = (0.1 * randn(B, H, N, N)).contiguous()
    elif s0 == "zeros":
        out["S0"] = None
    else:
        raise ValueError(f"unknown S0 recipe {s0!r}")
    if wl.epilogue:
        out["ln_w"] = (1.0 + 0.1 * randn(H, N)).contiguous()
        out["ln_b"] = (0.1 * randn(H, N)).contiguous()
        out["r_k"] = (0.5 * randn(H, N)).contiguous()
    return out


LAYER_RANKS = {"d_w": 64, "d_a": 64, "d_v": 32, "d_g": 128}   # low-rank widths of the synthetic layer


def make_layer(B: int, T: int, H: int, N: int = HEAD_SIZE, *, seed: int = SEED_BASE + 900, device: str = "cpu",
               dtype: str = "bf16", first_layer: bool = False, ranks: dict | None = None) -> dict:
    """Synthetic weights and activations for one time-mixing layer (no trained weights are
    available): x, last_x, v0 ([B, T, C] / [B, C], C = H * N) and the projections in the layer
    dtype; mixes, biases and the per-head parameters fp32. Scales keep every projection's
    output near unit variance: square projections N(0, 1/C), low-rank factors N(0, 1/fan_in).
    No arithmetic of the method is applied."""
    rk = dict(LAYER_RANKS if ranks is None else ranks)
    C = H * N
    dt = torch_dtype(dtype)
    g = torch.Generator(device=device)
    g.manual_seed(seed)

    def randn(*s, std=1.0):
        return std * torch.randn(*s, generator=g, device=device, dtype=torch.float32)

    def rand(*s):
        return torch.rand(*s, generator=g, device=device, dtype=torch.float32)

    out = {"x": randn(B, T, C).to(dt), "last_x": randn(B, C).to(dt)}
    out["v0"] = None if first_layer else randn(B, T, C).to(dt)
    for m in ("mr", "mw", "mk", "mv", "ma", "mg"):
        out[m] = rand(C)
    out["w_bias"] = randn(C, std=0.5)
    out["a_bias"] = randn(C, std=0.5)
    out["v_bias"] = randn(C, std=0.5)
    out["r_k"] = randn(H, N, std=0.5)
    out["k_k"] = 0.5 + rand(H, N)
    out["k_a"] = rand(H, N)
    out["ln_w"] = 1.0 + randn(H, N, std=0.1)
    out["ln_b"] = randn(H, N, std=0.1)
    for n in ("Wr", "Wk", "Wv", "Wo"):
        out[n] = randn(C, C, std=C ** -0.5).to(dt)
    for lo, hi, d in (("Ww1", "Ww2", rk["d_w"]), ("Wa1", "Wa2", rk["d_a"]), ("Wv1", "Wv2", rk["d_v"]),
                      ("Wg1", "Wg2", rk["d_g"])):
        out[lo] = randn(C, d, std=C ** -0.5).to(dt)
        out[hi] = randn(d, C, std=d ** -0.5).to(dt)
    out["S0"] = randn(B, H, N, N, std=0.1)
    return out
