"""Pins for the oracle's backward pass (CPU, fp64). Each checks the reverse sweep against
something other than itself: central finite differences of the (pinned) forward, the
closed form of the linear-attention special case, Euler's identity for the parts of the
map that are linear, and the split of a sequence at a state hand-off."""
import numpy as np
import pytest

from oracle import reference

NAMES = ("r", "w", "k", "v", "kk", "a")


def _inputs(rng, B, T, H, N, *, s0=True):
    x = {n: rng.standard_normal((B, T, H, N)) for n in ("r", "k", "v")}
    x["w"] = rng.uniform(0.55, 1.0, (B, T, H, N))
    x["a"] = rng.uniform(0.0, 1.0, (B, T, H, N))
    kk = rng.standard_normal((B, T, H, N))
    x["kk"] = kk / np.linalg.norm(kk, axis=-1, keepdims=True)
    x["S0"] = rng.standard_normal((B, H, N, N)) if s0 else None
    x["dy"] = rng.standard_normal((B, T, H, N))
    x["dS_T"] = rng.standard_normal((B, H, N, N))
    return x


def _loss(x):
    y, S_T, _ = reference.wkv7_recurrence(*(x[n] for n in NAMES), x["S0"])
    return float(np.sum(x["dy"] * y) + np.sum(x["dS_T"] * S_T))


def _grads(x):
    return reference.wkv7_backward(*(x[n] for n in NAMES), x["S0"], x["dy"], x["dS_T"])


def test_backward_matches_finite_differences():
    """Every gradient entry (all six token inputs and S0) against a central difference."""
    rng = np.random.default_rng(40)
    x = _inputs(rng, 1, 5, 2, 3)
    g = _grads(x)
    h = 1e-6
    for name, gname in list(zip(NAMES, ("dr", "dw", "dk", "dv", "dkk", "da"))) + [("S0", "dS0")]:
        fd = np.zeros_like(x[name])
        for idx in np.ndindex(x[name].shape):
            orig = x[name][idx]
            x[name][idx] = orig + h
            lp = _loss(x)
            x[name][idx] = orig - h
            lm = _loss(x)
            x[name][idx] = orig
            fd[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(fd - g[gname])) / max(1.0, np.max(np.abs(fd)))
        assert err < 1e-7, (gname, err)


def test_linear_attention_closed_form():
    """w = 1, a = 0: S_t = S0 + sum_{s<=t} v_s k_s^T, so dr_t = S_t^T dy_t,
    dv_t = sum_{s>=t} (k_t . r_s) dy_s + dS_T k_t, dk_t = sum_{s>=t} (v_t . dy_s) r_s + dS_T^T v_t,
    dS0 = sum_s dy_s r_s^T + dS_T, dw_t and da_t from S_{t-1} and the gradient reaching S_t;
    summed directly, token pair by token pair."""
    rng = np.random.default_rng(41)
    B, T, H, N = 1, 7, 2, 5
    x = _inputs(rng, B, T, H, N)
    x["w"] = np.ones((B, T, H, N))
    x["a"] = np.zeros((B, T, H, N))
    g = _grads(x)
    r, k, v, dy, dS_T, S0 = x["r"][0], x["k"][0], x["v"][0], x["dy"][0], x["dS_T"][0], x["S0"][0]
    kk = x["kk"][0]
    for h in range(H):
        S = S0[h].copy()
        for t in range(T):
            S_prev = S
            S = S + np.outer(v[t, h], k[t, h])
            np.testing.assert_allclose(g["dr"][0, t, h], S.T @ dy[t, h], rtol=0, atol=1e-12)
            # the gradient reaching S_t is dS_T plus every later readout's dy_s r_s^T
            dS_t = dS_T[h] + sum(np.outer(dy[s, h], r[s, h]) for s in range(t, T))
            np.testing.assert_allclose(g["dw"][0, t, h], np.sum(S_prev * dS_t, axis=0), rtol=0, atol=1e-12)
            da = -kk[t, h] * (dS_t.T @ (S_prev @ kk[t, h]))
            np.testing.assert_allclose(g["da"][0, t, h], da, rtol=0, atol=1e-12)
            dv = dS_T[h] @ k[t, h] + sum((k[t, h] @ r[s, h]) * dy[s, h] for s in range(t, T))
            dk = dS_T[h].T @ v[t, h] + sum((v[t, h] @ dy[s, h]) * r[s, h] for s in range(t, T))
            np.testing.assert_allclose(g["dv"][0, t, h], dv, rtol=0, atol=1e-12)
            np.testing.assert_allclose(g["dk"][0, t, h], dk, rtol=0, atol=1e-12)
        dS0 = dS_T[h] + sum(np.outer(dy[s, h], r[s, h]) for s in range(T))
        np.testing.assert_allclose(g["dS0"][0, h], dS0, rtol=0, atol=1e-12)
    # a = 0: the removal term is absent, so nothing flows to kk
    assert np.max(np.abs(g["dkk"])) == 0


def test_euler_identities():
    """y is linear in r and (y, S_T) is linear in (S0, v) jointly, so
    <dr, r> = <dy, y> and <dS0, S0> + <dv, v> = L."""
    rng = np.random.default_rng(42)
    x = _inputs(rng, 2, 9, 3, 6)
    g = _grads(x)
    y, S_T, _ = reference.wkv7_recurrence(*(x[n] for n in NAMES), x["S0"])
    L = np.sum(x["dy"] * y) + np.sum(x["dS_T"] * S_T)
    assert abs(np.sum(g["dr"] * x["r"]) - np.sum(x["dy"] * y)) < 1e-9 * max(1.0, abs(L))
    assert abs(np.sum(g["dS0"] * x["S0"]) + np.sum(g["dv"] * x["v"]) - L) < 1e-9 * max(1.0, abs(L))


@pytest.mark.parametrize("T1", [1, 4, 8])
def test_split_at_state_handoff(T1):
    """Backward over [T1, T) from dS_T, then over [0, T1) from the dS it returns (with the
    state after T1 tokens as the second part's S0) equals one backward over [0, T)."""
    rng = np.random.default_rng(43)
    T = 11
    x = _inputs(rng, 1, T, 2, 4)
    g = _grads(x)
    _, S_mid, _ = reference.wkv7_recurrence(*(x[n][:, :T1] for n in NAMES), x["S0"])
    g2 = reference.wkv7_backward(*(x[n][:, T1:] for n in NAMES), S_mid, x["dy"][:, T1:], x["dS_T"])
    g1 = reference.wkv7_backward(*(x[n][:, :T1] for n in NAMES), x["S0"], x["dy"][:, :T1], g2["dS0"])
    for n in ("dr", "dw", "dk", "dv", "dkk", "da"):
        np.testing.assert_allclose(np.concatenate([g1[n], g2[n]], axis=1), g[n], rtol=0, atol=1e-12)
    np.testing.assert_allclose(g1["dS0"], g["dS0"], rtol=0, atol=1e-12)


def test_empty_sequence_passes_the_state_gradient_through():
    rng = np.random.default_rng(44)
    x = _inputs(rng, 1, 0, 2, 4)
    g = _grads(x)
    np.testing.assert_array_equal(g["dS0"], x["dS_T"])
    assert g["dr"].shape == (1, 0, 2, 4)
