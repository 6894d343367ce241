"""Pins for the oracle's full time-mixing layer (CPU, fp64): reductions to the pinned
recurrence, invariants of the token shift, the value residual and the gate, linearity in the
output projection, and the carry of state and previous token across calls."""
import numpy as np
import pytest

from linear_rnn_sequence_rwkv_b200 import inputs
from oracle import reference

P_NAMES = reference.LAYER_PARAM_NAMES


def _layer(B=2, T=6, H=2, N=8, seed=1, first=False):
    d = inputs.make_layer(B, T, H, N, seed=seed, first_layer=first, dtype="f32",
                          ranks={"d_w": 5, "d_a": 4, "d_v": 3, "d_g": 6})
    d = {k: (None if v is None else v.double().numpy()) for k, v in d.items()}
    return d


def _run(d, **over):
    p = {n: over.get(n, d[n]) for n in P_NAMES}
    return reference.time_mixing_layer(over.get("x", d["x"]), p, over.get("last_x", d["last_x"]),
                                       over.get("v0", d["v0"]), over.get("S0", d["S0"]))


def test_reduces_to_the_recurrence_and_epilogue():
    """Zero mixes, identity projections, zero low-rank factors but Wg2 = 2/d_g (g = 1): the
    layer is the pre-processing, the recurrence and the epilogue on x itself, per head."""
    d = _layer(first=True)
    B, T, C = d["x"].shape
    H, N = d["r_k"].shape
    over = {m: np.zeros(C) for m in ("mr", "mw", "mk", "mv", "ma", "mg")}
    over.update({n: np.eye(C) for n in ("Wr", "Wk", "Wv", "Wo")})
    for n in ("Ww1", "Ww2", "Wa1", "Wa2", "Wv1", "Wv2", "Wg1"):
        over[n] = np.zeros_like(d[n])
    over["Wg2"] = np.full_like(d["Wg2"], 2.0 / d["Wg2"].shape[0])
    out, v0, last, S_T = _run(d, **over)
    xh = d["x"].reshape(B, T, H, N)
    wl = np.broadcast_to(d["w_bias"], (B, T, C)).reshape(B, T, H, N)
    al = np.broadcast_to(d["a_bias"], (B, T, C)).reshape(B, T, H, N)
    w, a, kk, kt = reference.prepare_inputs(wl, al, xh, d["k_k"], d["k_a"])
    y, S_ref, _ = reference.wkv7_recurrence(xh, w, kt, xh, kk, a, d["S0"])
    ref = reference.group_norm_bonus(y, xh, kt, xh, d["ln_w"], d["ln_b"], d["r_k"]).reshape(B, T, C)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(S_T, S_ref, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(v0, d["x"])          # first layer: v0 is its own v (= x here)
    np.testing.assert_array_equal(last, d["x"][:, -1])


def test_full_mix_reads_only_the_previous_token():
    """Every mix 1: all projections see the previous token, so the first output depends on
    last_x and not on x[:, 0]."""
    d = _layer()
    C = d["x"].shape[-1]
    ones = {m: np.ones(C) for m in ("mr", "mw", "mk", "mv", "ma", "mg")}
    x2 = d["x"].copy()
    x2[:, 0] += 3.0
    o1 = _run(d, **ones)[0]
    o2 = _run(d, x=x2, **ones)[0]
    np.testing.assert_allclose(o1[:, 0], o2[:, 0], rtol=0, atol=1e-12)
    assert np.max(np.abs(o1[:, 1] - o2[:, 1])) > 1e-3   # the second token sees the change


def test_value_residual_limits():
    """v_bias -> -inf: the first layer's values are ignored (as in the first layer);
    v_bias -> +inf: v is replaced by v0, so Wv no longer matters."""
    d = _layer()
    C = d["x"].shape[-1]
    lo = _run(d, v_bias=np.full(C, -60.0))[0]
    first = _run(d, v0=None)[0]
    np.testing.assert_allclose(lo, first, rtol=0, atol=1e-12)
    hi1 = _run(d, v_bias=np.full(C, 60.0))[0]
    hi2 = _run(d, v_bias=np.full(C, 60.0), Wv=2.0 * d["Wv"] + 1.0)[0]
    np.testing.assert_allclose(hi1, hi2, rtol=0, atol=1e-12)


def test_linear_in_output_projection_and_gate_output_factor():
    d = _layer()
    W2 = np.random.default_rng(3).standard_normal(d["Wo"].shape)
    o1, o2, o12 = _run(d)[0], _run(d, Wo=W2)[0], _run(d, Wo=d["Wo"] + W2)[0]
    np.testing.assert_allclose(o12, o1 + o2, rtol=0, atol=1e-10)
    np.testing.assert_allclose(_run(d, Wg2=3.0 * d["Wg2"])[0], 3.0 * o1, rtol=0, atol=1e-10)


@pytest.mark.parametrize("T1", [1, 3])
def test_sequence_split_carries_state_and_previous_token(T1):
    d = _layer(T=7)
    out, v0, last, S_T = _run(d)
    a = _run(d, x=d["x"][:, :T1], v0=d["v0"][:, :T1])
    b = _run(d, x=d["x"][:, T1:], v0=d["v0"][:, T1:], last_x=a[2], S0=a[3])
    np.testing.assert_allclose(np.concatenate([a[0], b[0]], axis=1), out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(b[3], S_T, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(b[2], last)


# ---- second transcription and the activations of the low-rank paths ----------------------------

from oracle import native  # noqa: E402


@pytest.mark.parametrize("first,with_last,with_s0", [(True, True, True), (False, True, True), (False, False, False)])
def test_numpy_layer_matches_the_c_transcription(first, with_last, with_s0):
    """The numpy layer (whole sequences at once) equals the plain-C transcription of the
    listing (one token at a time, plain loops) with every low-rank factor non-zero."""
    d = _layer(B=2, T=5, H=2, N=4, seed=11 + int(first), first=first)
    p = {n: d[n] for n in P_NAMES}
    args = (d["x"], p, d["last_x"] if with_last else None, d["v0"], d["S0"] if with_s0 else None)
    a = reference.time_mixing_layer(*args)
    b = native.time_mixing_layer(*args)
    for u, v, name in zip(a, b, ("out", "v0", "last_x", "S_T")):
        np.testing.assert_allclose(u, v, rtol=0, atol=1e-11 * max(1.0, np.max(np.abs(v))), err_msg=name)


def _proj(d, **over):
    P = {n: over.get(n, d[n]) for n in P_NAMES}
    return reference.layer_projections(over.get("x", d["x"]), P, over.get("last_x", d["last_x"]),
                                       over.get("v0", d["v0"]))


def _mixed(d, m):
    prev = np.concatenate([d["last_x"][:, None], d["x"][:, :-1]], axis=1)
    return d["x"] + d[m] * (prev - d["x"])


def test_decay_path_is_tanh_between_its_factors():
    """tanh saturates at +-1 for a large first factor, so the logit minus its bias becomes
    sign(x_w Ww1) Ww2; for a tiny first factor tanh is the identity to first order."""
    d = _layer()
    xw = _mixed(d, "mw")
    big = _proj(d, Ww1=1e4 * d["Ww1"])["w_logit"] - d["w_bias"]
    np.testing.assert_allclose(big, np.sign(xw @ d["Ww1"]) @ d["Ww2"], rtol=0, atol=1e-9)
    eps = 1e-6
    small = (_proj(d, Ww1=eps * d["Ww1"])["w_logit"] - d["w_bias"]) / eps
    np.testing.assert_allclose(small, (xw @ d["Ww1"]) @ d["Ww2"], rtol=0, atol=1e-6)


def test_rate_path_is_linear_between_its_factors():
    """Nothing sits between Wa1 and Wa2: the logit minus its bias is linear in Wa1."""
    d = _layer()
    base = _proj(d)["a_logit"] - d["a_bias"]
    for alpha in (3.0, -2.0):
        np.testing.assert_allclose(_proj(d, Wa1=alpha * d["Wa1"])["a_logit"] - d["a_bias"], alpha * base,
                                   rtol=0, atol=1e-12)
    np.testing.assert_allclose(base, _mixed(d, "ma") @ d["Wa1"] @ d["Wa2"], rtol=0, atol=1e-12)


def test_value_residual_path_is_linear_between_its_factors():
    """The residual's mixing weight is sigmoid(x_v Wv1 Wv2 + v_bias): recovered from v, v0 and
    the first-layer v, its logit minus the bias is x_v Wv1 Wv2 (no activation in between)."""
    d = _layer()
    v_lin = _proj(d, v0=None)["v"]
    got = _proj(d)
    lam = (got["v"] - v_lin) / (d["v0"] - v_lin)
    logit = np.log(lam / (1.0 - lam))
    np.testing.assert_allclose(logit - d["v_bias"], _mixed(d, "mv") @ d["Wv1"] @ d["Wv2"], rtol=0, atol=1e-8)


def test_gate_is_sigmoid_of_the_hidden_value_then_the_second_factor():
    """g = sigmoid(x_g Wg1) Wg2: with Wg1 = 0 every hidden unit is 1/2; with a large Wg1 the
    hidden units become the step of x_g Wg1."""
    d = _layer()
    g0 = _proj(d, Wg1=np.zeros_like(d["Wg1"]))["g"]
    np.testing.assert_allclose(g0, np.broadcast_to(0.5 * d["Wg2"].sum(axis=0), g0.shape), rtol=0, atol=1e-14)
    gb = _proj(d, Wg1=1e4 * d["Wg1"])["g"]
    np.testing.assert_allclose(gb, (_mixed(d, "mg") @ d["Wg1"] > 0) @ d["Wg2"], rtol=0, atol=1e-9)


def test_square_projections_take_the_stored_row_as_output_channel():
    """W x with W stored [out][in]: a one-hot token at channel i (no mixing, first layer) gives
    column i of Wr, Wk and Wv; the matrices are not symmetric, so a transposed use fails."""
    d = _layer(B=1, T=1)
    C = d["x"].shape[-1]
    i = 3
    x = np.zeros((1, 1, C))
    x[0, 0, i] = 1.0
    zero = {m: np.zeros(C) for m in ("mr", "mw", "mk", "mv", "ma", "mg")}
    z = _proj(d, x=x, last_x=np.zeros((1, C)), v0=None, **zero)
    for name, W in (("r", "Wr"), ("k", "Wk"), ("v", "Wv")):
        assert np.max(np.abs(d[W] - d[W].T)) > 1e-3
        np.testing.assert_allclose(z[name][0, 0], d[W][:, i], rtol=0, atol=1e-15)
