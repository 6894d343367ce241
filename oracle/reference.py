"""Plain fp64 numpy statement of the WKV-7 recurrence and its epilogue.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import this module;
only tests, the graft smoke check and the benchmark's CPU-baseline leg do.

Sources (RWKV-7 "Goose"):
* State update and readout: the rebuttal page's numpy ``time_mixing`` listing, the
  update line ``S = S*w.mT - S@kk*(kk*a).mT + v*k.mT`` and readout ``y = S@r``; the
  same update in row-vector form in the ARWKV verdict page (``key_machinery``):
  S_t = S_{t-1}(diag(w_t) - kk_t^T (a_t * kk_t)) + v_t^T k_t.
* Per-head group_norm (population variance, eps 64e-5 inside the square root, then
  a per-channel affine) and the bonus term sum_j(r_j k_j r_k[j]) * v added after the
  norm: same listing, the ``group_norm`` lambda and the two lines after the readout.

Readings taken where the pages leave a step open (each listed in the design doc):
* S is N x N with row i = value channel, column j = key channel (the listing's
  column vectors make ``S*w.mT`` scale columns and ``S@r`` contract the key index).
* The removal term uses the state *before* this token's update, S_{t-1}: the
  right-hand side is evaluated before assignment, and the row-vector form factors
  S_{t-1} out of both terms.
* ``S@kk*(kk*a).mT`` is ``(S@kk) * (kk*a)^T``: the outer product of the removed value
  S_{t-1} kk with kk*a (``@`` and ``*`` share precedence, left to right).
* The readout uses the updated state S_t (the current token is included).
* kk arrives already L2-normalised, k is the replacement key, w is the decay
  multiplier itself; nothing is renormalised in the recurrence. ``prepare_inputs``
  states the pre-processing that produces them from the raw time-mixing values
  (the path that fuses it into the kernel's load stage).

Parity pins: every function here is pinned in tests/test_oracle.py against closed
forms, brute-force transition products, the paper's elementary-transition
constructions and a finite-difference SGD reading of the delta rule.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    """Exact conversion of a torch tensor / array of bf16, fp32 or fp64 to fp64."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # local: only needed for tensor inputs
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def wkv7_recurrence(r, w, k, v, kk, a, S0=None, snap_every=0):
    """Run the WKV-7 recurrence token by token in fp64.

    r, w, k, v, kk, a: [B, T, H, N]. S0: [B, H, N, N] or None (zeros).
    Returns (y [B, T, H, N], S_T [B, H, N, N], snaps [B, T//snap_every, H, N, N] or None).
    """
    r, w, k, v, kk, a = (_f64(x) for x in (r, w, k, v, kk, a))
    B, T, H, N = r.shape
    S = np.zeros((B, H, N, N)) if S0 is None else _f64(S0).copy()
    y = np.empty((B, T, H, N))
    n_snap = T // snap_every if snap_every else 0
    snaps = np.empty((B, n_snap, H, N, N)) if n_snap else None
    for t in range(T):
        w_t, k_t, v_t, kk_t, a_t, r_t = w[:, t], k[:, t], v[:, t], kk[:, t], a[:, t], r[:, t]
        # value currently stored at the removal key, read from S_{t-1}
        removed = np.einsum("bhij,bhj->bhi", S, kk_t)
        decayed = S * w_t[:, :, None, :]                       # S diag(w): scale key columns
        erase = removed[:, :, :, None] * (kk_t * a_t)[:, :, None, :]
        write = v_t[:, :, :, None] * k_t[:, :, None, :]
        S = decayed - erase + write
        y[:, t] = np.einsum("bhij,bhj->bhi", S, r_t)          # readout of S_t
        if n_snap and (t + 1) % snap_every == 0:
            snaps[:, (t + 1) // snap_every - 1] = S
    return y, S, snaps


def group_norm_bonus(y, r, k, v, ln_w, ln_b, r_k, eps=64e-5):
    """Per-head group_norm of the readout, then the current-token bonus.

    y, r, k, v: [B, T, H, N]; ln_w, ln_b, r_k: [H, N]. Returns [B, T, H, N] fp64.
    """
    y, r, k, v, ln_w, ln_b, r_k = (_f64(x) for x in (y, r, k, v, ln_w, ln_b, r_k))
    mean = y.mean(axis=-1, keepdims=True)
    var = ((y - mean) ** 2).mean(axis=-1, keepdims=True)   # population variance
    normed = (y - mean) / np.sqrt(var + eps) * ln_w + ln_b
    bonus = (r * k * r_k).sum(axis=-1, keepdims=True) * v
    return normed + bonus


def prepare_inputs(w_logit, a_logit, k, k_k, k_a=None):
    """The pre-processing the pages place before the update, in fp64 (the rebuttal page's
    ``time_mixing`` listing: the decay, the in-context learning rate, the removal key formed
    from the key before its update and normalised with a 1e-12 floor, and the key update).

    w_logit, a_logit, k: [B, T, H, N]; k_k, k_a: [H, N] (k_a None = 0).
    Returns (w, a, kk, k_tilde), each [B, T, H, N] fp64:
      w = exp(-sigmoid(w_logit) / sqrt(e)), a = sigmoid(a_logit),
      kk = (k * k_k) / max(||k * k_k||_2, 1e-12) over the head's N channels (from the key
      before its update), k_tilde = k + k * (a - 1) * k_a.
    """
    w_logit, a_logit, k, k_k = (_f64(x) for x in (w_logit, a_logit, k, k_k))
    k_a = np.zeros_like(k_k) if k_a is None else _f64(k_a)
    sig = lambda x: 1.0 / (1.0 + np.exp(-x))
    w = np.exp(-sig(w_logit) / np.e ** 0.5)
    a = sig(a_logit)
    kk = k * k_k
    k_tilde = k + k * (a - 1.0) * k_a
    kk = kk / np.maximum(np.linalg.norm(kk, axis=-1, keepdims=True), 1e-12)
    return w, a, kk, k_tilde


def transition_matrix(w_t, kk_t, a_t):
    """A_t = diag(w_t) - kk_t (kk_t * a_t)^T for one head (vectors of length N)."""
    w_t, kk_t, a_t = (_f64(x) for x in (w_t, kk_t, a_t))
    return np.diag(w_t) - np.outer(kk_t, kk_t * a_t)
