"""Pins for the CPU fp64 oracle (runs without a GPU).

Each test checks the oracle against something other than itself: a closed form
the pages fix, a brute-force product of transition matrices, the paper's
elementary-transition constructions, a finite-difference gradient, or an
invariant of the mathematics. Sources are RWKV-7 "Goose" pages: the rebuttal's
numpy ``time_mixing`` listing (update, readout, group_norm, bonus), the ARWKV
verdict's row-vector statement of the update, and the paper summary's sections
2 (linear attention, decay, DeltaNet), 4 (eigenvalues in [-1, 1]), D.3
(elementary transitions with c = 2) and F (SGD reading, decay above 0.545).
"""
import math

import numpy as np
import pytest

from oracle import native, reference
from linear_rnn_sequence_rwkv_b200 import inputs

RTOL = 1e-12


def _rand_inputs(rng, B, T, H, N, *, a_scale=1.0, unit_kk=True, w_lo=inputs.W_MIN):
    r = rng.standard_normal((B, T, H, N))
    k = rng.standard_normal((B, T, H, N))
    v = rng.standard_normal((B, T, H, N))
    w = rng.uniform(w_lo, 1.0, (B, T, H, N))
    a = a_scale * rng.uniform(0.0, 1.0, (B, T, H, N))
    kk = rng.standard_normal((B, T, H, N))
    if unit_kk:
        kk /= np.linalg.norm(kk, axis=-1, keepdims=True)
    return r, w, k, v, kk, a


def _close(x, ref, tol=RTOL):
    x, ref = np.asarray(x), np.asarray(ref)
    scale = max(1.0, float(np.max(np.abs(ref))))
    err = float(np.max(np.abs(x - ref))) / scale
    assert err <= tol, f"max abs err {err:.3e} (scaled) > {tol:.1e}"


both = pytest.mark.parametrize("impl", ["numpy", "c"])


def _run(impl, *args, **kw):
    fn = reference.wkv7_recurrence if impl == "numpy" else native.forward
    return fn(*args, **kw)


# --- closed forms --------------------------------------------------------------------

@both
def test_single_token_from_zero_state(impl):
    """T=1 from S0=0: S_1 = v k^T and y = v (k . r) (update + readout lines)."""
    rng = np.random.default_rng(1)
    r, w, k, v, kk, a = _rand_inputs(rng, 2, 1, 3, 64)
    y, S, _ = _run(impl, r, w, k, v, kk, a)
    S_exp = v[:, 0, :, :, None] * k[:, 0, :, None, :]
    y_exp = v[:, 0] * np.sum(k[:, 0] * r[:, 0], axis=-1, keepdims=True)
    _close(S, S_exp)
    _close(y[:, 0], y_exp)


@both
def test_linear_attention_reduction(impl):
    """a=0, w=1 reduces to linear attention: S_t = S0 + sum_{s<=t} v_s k_s^T, y_t = S_t r_t."""
    rng = np.random.default_rng(2)
    B, T, H, N = 2, 9, 2, 64
    r, w, k, v, kk, a = _rand_inputs(rng, B, T, H, N)
    w[:] = 1.0
    a[:] = 0.0
    S0 = rng.standard_normal((B, H, N, N))
    y, S, _ = _run(impl, r, w, k, v, kk, a, S0)
    outer = v[..., :, None] * k[..., None, :]                 # [B,T,H,N,N]
    S_t = S0[:, None] + np.cumsum(outer, axis=1)
    _close(S, S_t[:, -1])
    _close(y, np.einsum("bthij,bthj->bthi", S_t, r))


@both
def test_diagonal_decay_brute_force(impl):
    """a=0: S_T[i,j] = S0[i,j] prod_t w_t[j] + sum_t v_t[i] k_t[j] prod_{s>t} w_s[j]."""
    rng = np.random.default_rng(3)
    B, T, H, N = 1, 6, 1, 8
    r, w, k, v, kk, a = _rand_inputs(rng, B, T, H, N)
    a[:] = 0.0
    S0 = rng.standard_normal((B, H, N, N))
    y, S, _ = _run(impl, r, w, k, v, kk, a, S0)
    for t_end in range(1, T + 1):
        St = np.zeros((N, N))
        for i in range(N):
            for j in range(N):
                acc = S0[0, 0, i, j] * np.prod(w[0, :t_end, 0, j])
                for t in range(t_end):
                    acc += v[0, t, 0, i] * k[0, t, 0, j] * np.prod(w[0, t + 1:t_end, 0, j])
                St[i, j] = acc
        _close(y[0, t_end - 1, 0], St @ r[0, t_end - 1, 0])
        if t_end == T:
            _close(S[0, 0], St)


# --- delta rule semantics ---------------------------------------------------------------

@both
def test_delta_rule_replaces_value_at_key(impl):
    """w=1, a=1, unit kk, k=kk: after each token the state maps kk_t exactly to v_t.

    With a=1 the transition I - kk kk^T erases the kk direction before the write,
    so S_t kk_t = v_t (section 2, DeltaNet replacement; section F)."""
    rng = np.random.default_rng(4)
    B, T, H, N = 2, 12, 2, 64
    r, w, k, v, kk, a = _rand_inputs(rng, B, T, H, N)
    w[:] = 1.0
    a[:] = 1.0
    k = kk.copy()
    S0 = rng.standard_normal((B, H, N, N))
    _, _, snaps = _run(impl, r, w, k, v, kk, a, S0, snap_every=1)
    got = np.einsum("bthij,bthj->bthi", snaps, kk)
    _close(got, v, 1e-11)


@both
def test_delta_rule_with_general_replacement_key(impl):
    """w=1, a=1, unit kk: S_t kk_t = v_t (k_t . kk_t), whatever S_{t-1} held."""
    rng = np.random.default_rng(5)
    B, T, H, N = 1, 10, 3, 64
    r, w, k, v, kk, a = _rand_inputs(rng, B, T, H, N)
    w[:] = 1.0
    a[:] = 1.0
    _, _, snaps = _run(impl, r, w, k, v, kk, a, rng.standard_normal((B, H, N, N)), snap_every=1)
    got = np.einsum("bthij,bthj->bthi", snaps, kk)
    _close(got, v * np.sum(k * kk, axis=-1, keepdims=True), 1e-11)


@both
def test_sgd_step_reading(impl):
    """Section F: the update is an SGD step on L(S) = 1/2 ||S kk - v||^2.

    With w=1, a=eta (every channel), k = eta*kk and unit kk, one token gives
    S_1 = S_0 - eta * dL/dS. The gradient here is taken by central finite
    differences, independently of the update formula."""
    rng = np.random.default_rng(6)
    N, eta, h = 5, 0.37, 1e-5
    S0 = rng.standard_normal((1, 1, N, N))
    kk = rng.standard_normal((1, 1, 1, N))
    kk /= np.linalg.norm(kk)
    v = rng.standard_normal((1, 1, 1, N))
    r = rng.standard_normal((1, 1, 1, N))
    w = np.ones((1, 1, 1, N))
    a = np.full((1, 1, 1, N), eta)
    k = eta * kk

    def loss(S):
        res = S @ kk[0, 0, 0] - v[0, 0, 0]
        return 0.5 * float(res @ res)

    grad = np.zeros((N, N))
    for i in range(N):
        for j in range(N):
            Sp = S0[0, 0].copy()
            Sm = S0[0, 0].copy()
            Sp[i, j] += h
            Sm[i, j] -= h
            grad[i, j] = (loss(Sp) - loss(Sm)) / (2 * h)
    _, S1, _ = _run(impl, r, w, k, v, kk, a, S0)
    _close(S1[0, 0], S0[0, 0] - eta * grad, 1e-8)


# --- the paper's elementary transitions (appendix D.3, c = 2) ------------------------

def _elementary(impl, N, kk_vec, a_vec, S0):
    one = lambda x: np.asarray(x, dtype=np.float64).reshape(1, 1, 1, N)
    zeros = np.zeros((1, 1, 1, N))
    _, S1, _ = _run(impl, zeros, one(np.ones(N)), zeros, zeros, one(kk_vec), one(a_vec),
                    S0.reshape(1, 1, N, N))
    return S1[0, 0]


@both
@pytest.mark.parametrize("i,j", [(0, 1), (2, 5), (7, 3)])
def test_swap_transition(impl, i, j):
    """kk = (e_i - e_j)/sqrt2, a = 2 (c=2, gate on): the transition swaps key columns i, j."""
    N = 8
    S0 = np.random.default_rng(7).standard_normal((N, N))
    e = np.eye(N)
    kk = (e[i] - e[j]) / math.sqrt(2.0)
    S1 = _elementary(impl, N, kk, 2.0 * (e[i] + e[j]), S0)
    expected = S0.copy()
    expected[:, [i, j]] = S0[:, [j, i]]
    _close(S1, expected)


@both
@pytest.mark.parametrize("i,j", [(0, 1), (4, 2), (6, 7)])
def test_copy_transition(impl, i, j):
    """kk = (e_i - e_j)/sqrt2, a = 2 e_j (binary gate on j only): column j := column i.

    This pins the placement of a on the right factor (kk*a)^T: with a on the
    left factor the same inputs would also change column i."""
    N = 8
    S0 = np.random.default_rng(8).standard_normal((N, N))
    e = np.eye(N)
    kk = (e[i] - e[j]) / math.sqrt(2.0)
    S1 = _elementary(impl, N, kk, 2.0 * e[j], S0)
    expected = S0.copy()
    expected[:, j] = S0[:, i]
    _close(S1, expected)


@both
def test_identity_transition(impl):
    """Gate off (a = 0), w = 1, no write: the state is unchanged."""
    N = 8
    S0 = np.random.default_rng(9).standard_normal((N, N))
    kk = np.random.default_rng(10).standard_normal(N)
    kk /= np.linalg.norm(kk)
    _close(_elementary(impl, N, kk, np.zeros(N), S0), S0)


# --- brute-force products of transition matrices ------------------------------------------

@both
@pytest.mark.parametrize("N,T", [(4, 1), (4, 7), (64, 5)])
def test_transition_product(impl, N, T):
    """Row-vector form (ARWKV verdict): S_T = S0 A_1..A_T + sum_t v_t k_t^T A_{t+1}..A_T,
    A_t = diag(w_t) - kk_t (a_t * kk_t)^T, built here as explicit N x N matrices."""
    rng = np.random.default_rng(11 + N + T)
    r, w, k, v, kk, a = _rand_inputs(rng, 1, T, 1, N)
    S0 = rng.standard_normal((1, 1, N, N))
    y, S, _ = _run(impl, r, w, k, v, kk, a, S0)
    A = [np.diag(w[0, t, 0]) - np.outer(kk[0, t, 0], a[0, t, 0] * kk[0, t, 0]) for t in range(T)]
    for t_end in range(1, T + 1):
        P = np.eye(N)
        for t in range(t_end):
            P = P @ A[t]
        St = S0[0, 0] @ P
        for t in range(t_end):
            tail = np.eye(N)
            for s in range(t + 1, t_end):
                tail = tail @ A[s]
            St = St + np.outer(v[0, t, 0], k[0, t, 0]) @ tail
        _close(y[0, t_end - 1, 0], St @ r[0, t_end - 1, 0], 1e-11)
        if t_end == T:
            _close(S[0, 0], St, 1e-11)


def test_transition_matrix_helper_matches_lemma():
    """reference.transition_matrix reproduces the swap construction (a Householder
    reflection) and its eigenvalues {+1 (N-1 times), -1}."""
    N = 6
    e = np.eye(N)
    kk = (e[1] - e[4]) / math.sqrt(2)
    A = reference.transition_matrix(np.ones(N), kk, 2.0 * np.ones(N))
    P = np.eye(N)
    P[:, [1, 4]] = P[:, [4, 1]]
    _close(A, P)
    ev = np.sort(np.linalg.eigvals(A).real)
    _close(ev, np.array([-1.0] + [1.0] * (N - 1)))


@pytest.mark.parametrize("seed", range(5))
def test_transition_spectrum_in_unit_interval(seed):
    """Section 4: eigenvalues of diag(w) - kk (kk*a)^T lie in [-1, 1]; for a in [0, 1]
    and unit kk they are real and within [min w - 1, max w] (similar, via diag(a)^1/2,
    to the symmetric diag(w) - u u^T with |u|^2 <= 1)."""
    rng = np.random.default_rng(100 + seed)
    N = 64
    w = rng.uniform(inputs.W_MIN, 1.0, N)
    a = rng.uniform(0.0, 1.0, N)
    kk = rng.standard_normal(N)
    kk /= np.linalg.norm(kk)
    ev = np.linalg.eigvals(reference.transition_matrix(w, kk, a))
    assert np.max(np.abs(ev.imag)) < 1e-9
    assert ev.real.min() >= w.min() - 1.0 - 1e-12
    assert ev.real.max() <= w.max() + 1e-12
    assert np.all(np.abs(ev.real) <= 1.0 + 1e-12)


# --- structural properties ----------------------------------------------------------------

@both
@pytest.mark.parametrize("T1", [1, 17, 40])
def test_state_handoff(impl, T1):
    """Running T1 tokens, handing S over and running the rest equals one pass."""
    rng = np.random.default_rng(12)
    B, T, H, N = 2, 41, 2, 64
    r, w, k, v, kk, a = _rand_inputs(rng, B, T, H, N)
    S0 = rng.standard_normal((B, H, N, N))
    y, S, _ = _run(impl, r, w, k, v, kk, a, S0)
    sl = lambda x, s: x[:, s]
    y1, S1, _ = _run(impl, *(sl(x, slice(0, T1)) for x in (r, w, k, v, kk, a)), S0)
    y2, S2, _ = _run(impl, *(sl(x, slice(T1, T)) for x in (r, w, k, v, kk, a)), S1)
    np.testing.assert_array_equal(np.concatenate([y1, y2], axis=1), y)
    np.testing.assert_array_equal(S2, S)


@both
def test_linear_in_state_and_values(impl):
    """For fixed r, w, k, kk, a the map (S0, v) -> (y, S_T) is linear."""
    rng = np.random.default_rng(13)
    B, T, H, N = 1, 8, 2, 64
    r, w, k, v, kk, a = _rand_inputs(rng, B, T, H, N)
    # the write term v k^T is bilinear in (v, k): superpose with k fixed
    v2 = rng.standard_normal(v.shape)
    S0 = rng.standard_normal((B, H, N, N))
    S02 = rng.standard_normal((B, H, N, N))
    al, be = 0.7, -1.9
    y1, S1, _ = _run(impl, r, w, k, v, kk, a, S0)
    y2, S2, _ = _run(impl, r, w, k, v2, kk, a, S02)
    y3, S3, _ = _run(impl, r, w, k, al * v + be * v2, kk, a, al * S0 + be * S02)
    _close(y3, al * y1 + be * y2, 1e-11)
    _close(S3, al * S1 + be * S2, 1e-11)


@both
def test_snapshots_are_intermediate_states(impl):
    """Snapshot m equals the state after (m+1)*snap_every tokens; the last equals S_T."""
    rng = np.random.default_rng(14)
    B, T, H, N = 1, 12, 2, 16
    r, w, k, v, kk, a = _rand_inputs(rng, B, T, H, N)
    _, S, snaps = _run(impl, r, w, k, v, kk, a, snap_every=4)
    assert snaps.shape == (B, 3, H, N, N)
    _close(snaps[:, -1], S, 0.0)
    for m in range(3):
        _, Sm, _ = _run(impl, *(x[:, :4 * (m + 1)] for x in (r, w, k, v, kk, a)))
        _close(snaps[:, m], Sm, 0.0)


def test_c_and_numpy_statements_agree():
    """The two oracle statements (numpy, plain C) agree on random shapes incl. S0."""
    rng = np.random.default_rng(15)
    for (B, T, H, N) in [(1, 1, 1, 64), (2, 33, 3, 64), (3, 7, 2, 8)]:
        r, w, k, v, kk, a = _rand_inputs(rng, B, T, H, N)
        S0 = rng.standard_normal((B, H, N, N))
        yn, Sn, _ = reference.wkv7_recurrence(r, w, k, v, kk, a, S0)
        for nt in (1, 4):
            yc, Sc, _ = native.forward(r, w, k, v, kk, a, S0, nthreads=nt)
            _close(yc, yn, 1e-12)
            _close(Sc, Sn, 1e-12)


# --- epilogue ---------------------------------------------------------------------------

@pytest.mark.parametrize("impl", ["numpy", "c"])
def test_group_norm_moments(impl):
    """ln_w=1, ln_b=0, r_k=0: each head row has mean 0 and variance var/(var+eps)."""
    rng = np.random.default_rng(16)
    B, T, H, N = 2, 5, 3, 64
    y = 0.05 * rng.standard_normal((B, T, H, N)) + 3.0
    r, k, v = (rng.standard_normal((B, T, H, N)) for _ in range(3))
    ones, zeros = np.ones((H, N)), np.zeros((H, N))
    fn = reference.group_norm_bonus if impl == "numpy" else native.epilogue
    out = fn(y, r, k, v, ones, zeros, zeros, eps=64e-5)
    var = y.var(axis=-1)
    _close(out.mean(axis=-1), np.zeros_like(var), 1e-12)
    _close(out.var(axis=-1), var / (var + 64e-5), 1e-12)


@pytest.mark.parametrize("impl", ["numpy", "c"])
def test_group_norm_affine_and_bonus_closed_form(impl):
    """Constant rows normalise to 0, leaving ln_b + bonus; one-hot r, k, r_k make
    the bonus r_p k_p r_k[p] v (added after the norm)."""
    B, T, H, N = 1, 2, 2, 64
    rng = np.random.default_rng(17)
    y = np.full((B, T, H, N), 2.5)
    r = np.zeros((B, T, H, N))
    k = np.zeros((B, T, H, N))
    p = 11
    r[..., p] = 1.5
    k[..., p] = -2.0
    r_k = np.zeros((H, N))
    r_k[:, p] = 0.25
    v = rng.standard_normal((B, T, H, N))
    ln_w = rng.standard_normal((H, N))
    ln_b = rng.standard_normal((H, N))
    fn = reference.group_norm_bonus if impl == "numpy" else native.epilogue
    out = fn(y, r, k, v, ln_w, ln_b, r_k, eps=64e-5)
    _close(out, ln_b + (1.5 * -2.0 * 0.25) * v, 1e-12)


def test_epilogue_c_matches_numpy():
    rng = np.random.default_rng(18)
    B, T, H, N = 2, 6, 3, 64
    y, r, k, v = (rng.standard_normal((B, T, H, N)) for _ in range(4))
    ln_w, ln_b, r_k = (rng.standard_normal((H, N)) for _ in range(3))
    _close(native.epilogue(y, r, k, v, ln_w, ln_b, r_k),
           reference.group_norm_bonus(y, r, k, v, ln_w, ln_b, r_k), 1e-12)


# --- the synthetic input recipe ---------------------------------------------------------------

@pytest.mark.parametrize("cid", [0, 1, 4])
def test_input_ranges(cid):
    """w in (exp(-e^-1/2), 1] (section F: decay multiplier above 0.545), a in (0, 1),
    |kk| = 1 up to the rounding of the stored dtype."""
    import torch
    wl = inputs.WORKLOADS[cid]
    d = inputs.make_inputs(wl, B=1, T=256, H=2)
    w = d["w"].double()
    ulp = 2.0 ** -8 if wl.dtype == "bf16" else 2.0 ** -23
    assert float(w.min()) >= inputs.W_MIN * (1 - ulp) and float(w.max()) <= 1.0
    a = d["a"].double()
    assert float(a.min()) >= 0.0 and float(a.max()) <= 1.0
    nrm = torch.linalg.vector_norm(d["kk"].double(), dim=-1)
    assert float((nrm - 1).abs().max()) <= 4 * ulp
    if wl.z_mean > 0:   # long-context recipe: decay near the lower end of its range
        assert float(w.mean()) < 0.62


def test_inputs_are_seeded():
    wl = inputs.WORKLOADS[1]
    d1 = inputs.make_inputs(wl, B=1, T=8, H=2)
    d2 = inputs.make_inputs(wl, B=1, T=8, H=2)
    for name in ("r", "w", "k", "v", "kk", "a", "S0"):
        assert bool((d1[name] == d2[name]).all())


# --- golden fixture: appendix D.3 construction, expected values are column maps ---------

@both
def test_golden_elementary_transitions(impl):
    """tests/golden/elementary_transitions.json (appendix D.3, c = 2): the state
    after each token is a column map of S0 and y_t reads one column."""
    from tests.golden_util import elementary_transitions
    g = elementary_transitions()
    y, S, snaps = _run(impl, g["r"], g["w"], g["k"], g["v"], g["kk"], g["a"], g["S0"],
                       snap_every=1)
    _close(snaps[0, :, 0], g["S_expected"], 1e-13)
    _close(y[0, :, 0], g["y_expected"], 1e-13)
    _close(S[0, 0], g["S_expected"][-1], 1e-13)


# ---- the input pre-processing (fused into the kernel's load stage on the raw path) ----------

def test_prepare_inputs_closed_forms():
    """Decay and rate at known logits, the decay range, and the removal key's norm."""
    B, T, H, N = 1, 3, 2, 8
    rng = np.random.default_rng(7)
    k = rng.standard_normal((B, T, H, N))
    k_k = 0.5 + rng.random((H, N))
    z = np.zeros((B, T, H, N))
    w, a, kk, kt = reference.prepare_inputs(z, z, k, k_k)
    assert np.allclose(w, math.exp(-0.5 / math.sqrt(math.e)), rtol=0, atol=1e-15)
    assert np.allclose(a, 0.5, rtol=0, atol=1e-15)
    big = np.full((B, T, H, N), 20.0)
    w_hi, a_hi, _, _ = reference.prepare_inputs(-big, big, k, k_k)             # sigmoid -> 0 / 1
    w_lo, a_lo, _, _ = reference.prepare_inputs(big, -big, k, k_k)
    lo = math.exp(-math.exp(-0.5))                                              # w in (e^-e^-1/2, 1)
    assert np.all(w_hi < 1.0) and np.all(w_hi > 1.0 - 1e-8)
    assert np.all(w_lo > lo) and np.all(w_lo < lo + 1e-8)
    assert np.allclose(a_hi, 1.0, atol=1e-8) and np.allclose(a_lo, 0.0, atol=1e-8)
    assert np.allclose(np.linalg.norm(kk, axis=-1), 1.0, atol=1e-14)
    assert np.allclose(kt, k, rtol=0, atol=0)                                 # k_a = 0: k unchanged


def test_prepare_inputs_removal_key_uses_the_key_before_its_update():
    """kk is the normalised k * k_k of the raw key whatever k_a is; k_tilde = k * (1 + (a-1) k_a)."""
    B, T, H, N = 2, 4, 3, 16
    rng = np.random.default_rng(8)
    k = rng.standard_normal((B, T, H, N))
    k_k = 0.5 + rng.random((H, N))
    k_a = rng.random((H, N))
    zw, za = rng.standard_normal((B, T, H, N)), rng.standard_normal((B, T, H, N))
    w, a, kk, kt = reference.prepare_inputs(zw, za, k, k_k, k_a)
    _, _, kk0, _ = reference.prepare_inputs(zw, za, k, k_k, None)
    assert np.array_equal(kk, kk0)
    direction = (k * k_k) / np.linalg.norm(k * k_k, axis=-1, keepdims=True)
    assert np.allclose(kk, direction, atol=1e-14)
    assert np.allclose(kt, k * (1.0 + (a - 1.0) * k_a), atol=1e-14)
    _, a1, _, kt1 = reference.prepare_inputs(zw, np.full_like(za, 60.0), k, k_k, k_a)   # a -> 1
    assert np.allclose(kt1, k, atol=1e-12)
    _, _, _, kt2 = reference.prepare_inputs(zw, za, k, k_k, np.ones((H, N)))            # k_a = 1
    assert np.allclose(kt2, k * a, atol=1e-14)


def test_prepare_inputs_zero_key_is_finite():
    """A zero key gives a zero removal key (the 1e-12 floor), not a division by zero."""
    k = np.zeros((1, 1, 1, 64))
    _, _, kk, _ = reference.prepare_inputs(np.zeros_like(k), np.zeros_like(k), k, np.ones((1, 64)))
    assert np.all(np.isfinite(kk)) and np.all(kk == 0.0)


def test_raw_generator_matches_prepared_recipe_ranges():
    """The raw draws, prepared by the oracle, land in the ranges the prepared recipe states."""
    d = inputs.make_raw_inputs(inputs.WORKLOADS[1], B=1, T=40, H=2, seed=11)
    w, a, kk, kt = reference.prepare_inputs(d["w_logit"], d["a_logit"], d["k"], d["k_k"], d["k_a"])
    assert np.all((w > math.exp(-math.exp(-0.5))) & (w <= 1.0))
    assert np.all((a > 0.0) & (a < 1.0))
    assert np.allclose(np.linalg.norm(kk, axis=-1), 1.0, atol=1e-12)
    assert np.all(np.abs(kt) <= np.abs(reference._f64(d["k"])) + 1e-12)        # 0 < 1 + (a-1) k_a <= 1
