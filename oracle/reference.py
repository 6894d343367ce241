"""Plain fp64 numpy statement of the WKV-7 recurrence and its epilogue.

TEST INFRASTRUCTURE ONLY. Nothing in the product path may import this module;
only tests, the graft smoke check and the benchmark's CPU-baseline leg do.

Sources (RWKV-7 "Goose"):
* State update and readout: the rebuttal page's numpy ``time_mixing`` listing (its
  state-update line and its readout line): S_t = S_{t-1} diag(w_t) - (S_{t-1} kk_t)
  (kk_t * a_t)^T + v_t k_t^T and y_t = S_t r_t with column vectors; the same update in
  row-vector form in the ARWKV verdict page (``key_machinery``):
  S_t = S_{t-1}(diag(w_t) - kk_t^T (a_t * kk_t)) + v_t^T k_t.
* Per-head group_norm (population variance, eps 64e-5 inside the square root, then
  a per-channel affine) and the bonus term sum_j(r_j k_j r_k[j]) * v added after the
  norm: same listing, the ``group_norm`` lambda and the two lines after the readout.

Readings taken where the pages leave a step open:
* S is N x N with row i = value channel, column j = key channel (with the listing's
  column vectors the decay multiplies the key columns and the readout contracts the
  key index).
* The removal term uses the state *before* this token's update, S_{t-1}: the
  right-hand side is evaluated before assignment, and the row-vector form factors
  S_{t-1} out of both terms.
* The removal term, a matrix product followed by an elementwise product of equal
  precedence, evaluates left to right: (S kk)(kk*a)^T, the outer product of the removed
  value S_{t-1} kk with kk*a.
* The readout uses the updated state S_t (the current token is included).
* kk arrives already L2-normalised, k is the replacement key, w is the decay
  multiplier itself; nothing is renormalised in the recurrence. ``prepare_inputs``
  states the pre-processing that produces them from the raw time-mixing values
  (the path that fuses it into the kernel's load stage).

Parity pins: every function here is pinned in tests/test_oracle.py against closed
forms, brute-force transition products, the paper's elementary-transition
constructions and a finite-difference SGD reading of the delta rule; the backward in
tests/test_oracle_backward.py by finite differences; the layer (``layer_projections`` and
``time_mixing_layer``) in tests/test_oracle_layer.py by a second transcription in plain C
(oracle/wkv7_oracle.c, ``wkv7_oracle_layer``) and by properties of each activation (tanh
saturation and slope on the decay path, linearity of the rate and value-residual paths
between their factors, the gate's sigmoid limits, the orientation of the projections).
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


def wkv7_backward(r, w, k, v, kk, a, S0=None, dy=None, dS_T=None):
    """Gradients of the recurrence, in fp64: reverse-mode differentiation of
    ``wkv7_recurrence`` for the scalar L = <dy, y> + <dS_T, S_T> (dy, dS_T: the
    gradients arriving from above; None = 0). The pages time a backward pass and quote its
    fp32 precision (rebuttal page, the answer on numerical precision; paper summary, the
    speed figures for the forward that keeps its states and for the backward) but do not
    print it; this is the chain rule through the update and the readout, one token at a
    time in reverse, with every state kept from a forward sweep.

    For one token, with b = kk * a, s = S_{t-1} kk and dS the gradient of S_t:
      y_t = S_t r_t                      -> dS += dy_t r_t^T, dr_t = S_t^T dy_t
      + v_t k_t^T                        -> dv_t = dS k_t, dk_t = dS^T v_t
      S_{t-1} diag(w_t)                  -> dw_t[j] = sum_i S_{t-1}[i, j] dS[i, j]
      - s b^T                            -> db = -dS^T s, ds = -dS b
      s = S_{t-1} kk, b = kk * a         -> dkk_t = S_{t-1}^T ds + db * a_t, da_t = db * kk_t
      dS_{t-1} = dS diag(w_t) + ds kk_t^T.
    Returns dict of dr, dw, dk, dv, dkk, da ([B, T, H, N]) and dS0 ([B, H, N, N]), fp64.
    """
    r, w, k, v, kk, a = (_f64(x) for x in (r, w, k, v, kk, a))
    B, T, H, N = r.shape
    states = np.empty((T + 1, B, H, N, N))
    states[0] = 0.0 if S0 is None else _f64(S0)
    if T:
        _, _, snaps = wkv7_recurrence(r, w, k, v, kk, a, states[0], snap_every=1)
        states[1:] = np.moveaxis(snaps, 1, 0)
    dy = np.zeros((B, T, H, N)) if dy is None else _f64(dy)
    dS = np.zeros((B, H, N, N)) if dS_T is None else _f64(dS_T).copy()
    out = {n: np.zeros((B, T, H, N)) for n in ("dr", "dw", "dk", "dv", "dkk", "da")}
    for t in range(T - 1, -1, -1):
        S_prev, S_t = states[t], states[t + 1]
        w_t, k_t, v_t, kk_t, a_t, r_t, dy_t = (x[:, t] for x in (w, k, v, kk, a, r, dy))
        dS = dS + dy_t[:, :, :, None] * r_t[:, :, None, :]
        out["dr"][:, t] = np.einsum("bhij,bhi->bhj", S_t, dy_t)
        out["dv"][:, t] = np.einsum("bhij,bhj->bhi", dS, k_t)
        out["dk"][:, t] = np.einsum("bhij,bhi->bhj", dS, v_t)
        out["dw"][:, t] = np.sum(S_prev * dS, axis=-2)
        b_t = kk_t * a_t
        s = np.einsum("bhij,bhj->bhi", S_prev, kk_t)
        db = -np.einsum("bhij,bhi->bhj", dS, s)
        ds = -np.einsum("bhij,bhj->bhi", dS, b_t)
        out["dkk"][:, t] = np.einsum("bhij,bhi->bhj", S_prev, ds) + db * a_t
        out["da"][:, t] = db * kk_t
        dS = dS * w_t[:, :, None, :] + ds[:, :, :, None] * kk_t[:, :, None, :]
    out["dS0"] = dS
    return out


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


def group_norm_bonus_backward(y, r, k, v, ln_w, ln_b, r_k, dout, eps=64e-5):
    """Gradients of L = <dout, group_norm_bonus(y, r, k, v, ln_w, ln_b, r_k)> in fp64: the
    chain rule through the per-head group_norm and the bonus (the pages print the forward
    only; same listing as ``group_norm_bonus``). With yc = y - mean(y), inv = (mean(yc^2) +
    eps)^(-1/2), yn = yc inv and beta = sum_j r_j k_j r_k[j], per (b, t, h):
      out = yn ln_w + ln_b + beta v
      -> dv = beta dout, dbeta = sum_i dout_i v_i, dr = dbeta k r_k, dk = dbeta r r_k,
         dr_k += dbeta r k, dln_w += dout yn, dln_b += dout,
         g = dout ln_w, dy = inv (g - mean(g) - yn mean(g yn)).
    y, r, k, v, dout: [B, T, H, N]; ln_w, ln_b, r_k: [H, N]. Returns a dict of fp64 arrays:
    dy, dr, dk, dv [B, T, H, N] and dln_w, dln_b, dr_k [H, N] (summed over B and T).
    """
    y, r, k, v, ln_w, ln_b, r_k, dout = (_f64(x) for x in (y, r, k, v, ln_w, ln_b, r_k, dout))
    yc = y - y.mean(axis=-1, keepdims=True)
    inv = 1.0 / np.sqrt((yc ** 2).mean(axis=-1, keepdims=True) + eps)
    yn = yc * inv
    beta = (r * k * r_k).sum(axis=-1, keepdims=True)
    dbeta = (dout * v).sum(axis=-1, keepdims=True)
    g = dout * ln_w
    dy = inv * (g - g.mean(axis=-1, keepdims=True) - yn * (g * yn).mean(axis=-1, keepdims=True))
    return {"dy": dy, "dr": dbeta * k * r_k, "dk": dbeta * r * r_k, "dv": beta * dout,
            "dln_w": (dout * yn).sum(axis=(0, 1)), "dln_b": dout.sum(axis=(0, 1)),
            "dr_k": (dbeta * r * k).sum(axis=(0, 1))}


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


LAYER_PARAM_NAMES = ("mr", "mw", "mk", "mv", "ma", "mg", "w_bias", "a_bias", "v_bias", "r_k", "k_k", "k_a",
                     "ln_w", "ln_b", "Wr", "Wk", "Wv", "Wo", "Ww1", "Ww2", "Wa1", "Wa2", "Wv1", "Wv2", "Wg1", "Wg2")


def layer_projections(x, P, last_x=None, v0=None):
    """The per-token values one time-mixing layer feeds to its recurrence, in fp64 (the rebuttal
    page's numpy ``time_mixing`` listing, from the token shift to the gate), for a whole
    sequence at once.

    x: [B, T, C]; P: dict of fp64 parameters as in ``time_mixing_layer``; last_x [B, C] or None
    (zeros); v0 [B, T, C] or None (first layer). Returns a dict of [B, T, C] arrays: r, k, v (v
    after the value residual), w_logit, a_logit, g, and v0 (the first layer's values). Per token,
    with x_p the previous token (last_x for the first):
      x_m = x + m (x_p - x) for the six mixes m
      r = Wr x_r, k = Wk x_k, v = Wv x_v                      (W stored [out][in])
      w_logit = tanh(x_w Ww1) Ww2 + w_bias                    (low-rank factors [in][out])
      v <- v + (v0 - v) sigmoid(x_v Wv1 Wv2 + v_bias)         (layers after the first)
      a_logit = x_a Wa1 Wa2 + a_bias                          (no activation between the factors)
      g = sigmoid(x_g Wg1) Wg2
    """
    B, T, C = x.shape
    prev = np.concatenate([np.zeros((B, 1, C)) if last_x is None else _f64(last_x)[:, None], x[:, :-1]], axis=1)
    mix = {m: x + P[m] * (prev - x) for m in ("mr", "mw", "mk", "mv", "ma", "mg")}
    sig = lambda z: 1.0 / (1.0 + np.exp(-z))
    out = {"r": mix["mr"] @ P["Wr"].T, "k": mix["mk"] @ P["Wk"].T}
    v = mix["mv"] @ P["Wv"].T
    out["w_logit"] = np.tanh(mix["mw"] @ P["Ww1"]) @ P["Ww2"] + P["w_bias"]
    if v0 is None:
        v0 = v
    else:
        v = v + (_f64(v0) - v) * sig(mix["mv"] @ P["Wv1"] @ P["Wv2"] + P["v_bias"])
    out["v"], out["v0"] = v, v0
    out["a_logit"] = mix["ma"] @ P["Wa1"] @ P["Wa2"] + P["a_bias"]
    out["g"] = sig(mix["mg"] @ P["Wg1"]) @ P["Wg2"]
    return out


def time_mixing_layer(x, params, last_x=None, v0=None, S0=None, eps=64e-5):
    """One RWKV-7 time-mixing layer over a sequence, in fp64 (the rebuttal page's numpy
    ``time_mixing`` listing, applied token after token with the state, the previous token
    and the first layer's values carried along).

    x: [B, T, C] with C = H * N. params (arrays, fp64-convertible): token-shift mixes
    mr, mw, mk, mv, ma, mg [C]; biases w_bias, a_bias, v_bias [C]; r_k, k_k, k_a, ln_w, ln_b
    [H, N]; square projections Wr, Wk, Wv, Wo [C_out, C_in] applied as W x; low-rank factors
    Ww1 [C, Dw], Ww2 [Dw, C], Wa1, Wa2, Wv1, Wv2, Wg1, Wg2 likewise, applied as x W.
    last_x: [B, C] (the token before x[:, 0]; None = zeros). v0: [B, T, C] values of the
    first layer (None: this is the first layer, and its own v is returned as v0).
    S0: [B, H, N, N] or None. Returns (out [B, T, C], v0 [B, T, C], last x [B, C], S_T).

    The per-token values come from ``layer_projections``; then the pre-processing
    (w = exp(-sigmoid(w_logit) / sqrt(e)), a = sigmoid(a_logit), kk = normalised (k * k_k) per
    head, k <- k + k (a - 1) k_a), the recurrence and readout per head, group_norm + bonus, and
    out = Wo (y * g).
    """
    P = {n: _f64(params[n]) for n in LAYER_PARAM_NAMES}
    x = _f64(x)
    B, T, C = x.shape
    H, N = P["r_k"].shape
    z = layer_projections(x, P, last_x, v0)
    heads = lambda u: u.reshape(B, T, H, N)
    w, a, kk, k_t = prepare_inputs(heads(z["w_logit"]), heads(z["a_logit"]), heads(z["k"]), P["k_k"], P["k_a"])
    y, S_T, _ = wkv7_recurrence(heads(z["r"]), w, k_t, heads(z["v"]), kk, a, S0)
    y = group_norm_bonus(y, heads(z["r"]), k_t, heads(z["v"]), P["ln_w"], P["ln_b"], P["r_k"], eps)
    out = (y.reshape(B, T, C) * z["g"]) @ P["Wo"].T
    return out, z["v0"], x[:, -1].copy(), S_T


def transition_matrix(w_t, kk_t, a_t):
    """A_t = diag(w_t) - kk_t (kk_t * a_t)^T for one head (vectors of length N)."""
    w_t, kk_t, a_t = (_f64(x) for x in (w_t, kk_t, a_t))
    return np.diag(w_t) - np.outer(kk_t, kk_t * a_t)
