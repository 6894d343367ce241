"""Planted mistakes in the oracle (CPU only): each mutant below changes one step of an
oracle function — a sign, an index, a transposed operand, a factor in the wrong place —
and must make at least one pin fail. A mutant that every pin let through would show a
pin set too weak to trust the oracle with."""
import math

import numpy as np
import pytest

from oracle import reference
from tests import test_oracle as P
from tests import test_oracle_backward as PB

_f64 = reference._f64


# ---- forward mutants ---------------------------------------------------------------------

def _forward(kind):
    def run(r, w, k, v, kk, a, S0=None, snap_every=0):
        r, w, k, v, kk, a = (_f64(x) for x in (r, w, k, v, kk, a))
        B, T, H, N = r.shape
        S = np.zeros((B, H, N, N)) if S0 is None else _f64(S0).copy()
        y = np.empty((B, T, H, N))
        n_snap = T // snap_every if snap_every else 0
        snaps = np.empty((B, n_snap, H, N, N)) if n_snap else None
        for t in range(T):
            w_t, k_t, v_t, kk_t, a_t, r_t = w[:, t], k[:, t], v[:, t], kk[:, t], a[:, t], r[:, t]
            decayed = S * (w_t[:, :, :, None] if kind == "decay_rows" else w_t[:, :, None, :])
            src = decayed if kind == "removal_after_decay" else S
            if kind == "a_on_left":
                removed = np.einsum("bhij,bhj->bhi", src, kk_t * a_t)
                erase = removed[:, :, :, None] * kk_t[:, :, None, :]
            else:
                removed = np.einsum("bhij,bhj->bhi", src, kk_t)
                erase = removed[:, :, :, None] * (kk_t * a_t)[:, :, None, :]
            if kind == "transposed_write":
                write = k_t[:, :, :, None] * v_t[:, :, None, :]
            else:
                write = v_t[:, :, :, None] * k_t[:, :, None, :]
            S_new = decayed + erase + write if kind == "erase_sign" else decayed - erase + write
            y[:, t] = np.einsum("bhij,bhj->bhi", S if kind == "readout_before_update" else S_new, r_t)
            S = S_new
            if n_snap and (t + 1) % snap_every == 0:
                snaps[:, (t + 1) // snap_every - 1] = S
        return y, S, snaps
    return run


FORWARD_PINS = [
    lambda: P.test_single_token_from_zero_state("numpy"),
    lambda: P.test_linear_attention_reduction("numpy"),
    lambda: P.test_diagonal_decay_brute_force("numpy"),
    lambda: P.test_delta_rule_replaces_value_at_key("numpy"),
    lambda: P.test_delta_rule_with_general_replacement_key("numpy"),
    lambda: P.test_sgd_step_reading("numpy"),
    lambda: P.test_swap_transition("numpy", 2, 5),
    lambda: P.test_copy_transition("numpy", 4, 2),
    lambda: P.test_identity_transition("numpy"),
    lambda: P.test_transition_product("numpy", 4, 7),
    lambda: P.test_golden_elementary_transitions("numpy"),
]


def _failures(pins):
    n = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            n += 1
    return n


def test_unmutated_oracle_passes_the_pins_used_here():
    assert _failures(FORWARD_PINS + EPILOGUE_PINS + PREP_PINS + BACKWARD_PINS) == 0


@pytest.mark.parametrize("kind", ["erase_sign", "a_on_left", "readout_before_update", "decay_rows",
                                  "transposed_write", "removal_after_decay"])
def test_forward_mutant_is_caught(monkeypatch, kind):
    monkeypatch.setattr(reference, "wkv7_recurrence", _forward(kind))
    assert _failures(FORWARD_PINS) >= 1


# ---- epilogue mutants -----------------------------------------------------------------------

def _epilogue(kind):
    def run(y, r, k, v, ln_w, ln_b, r_k, eps=64e-5):
        y, r, k, v, ln_w, ln_b, r_k = (_f64(x) for x in (y, r, k, v, ln_w, ln_b, r_k))
        mean = y.mean(axis=-1, keepdims=True)
        var = y.var(axis=-1, keepdims=True, ddof=1 if kind == "sample_variance" else 0)
        den = np.sqrt(var) + eps if kind == "eps_outside_sqrt" else np.sqrt(var + eps)
        bonus = (r * k * r_k).sum(axis=-1, keepdims=True) * v
        if kind == "bonus_before_norm":
            y = y + bonus
            mean = y.mean(axis=-1, keepdims=True)
            den = np.sqrt(y.var(axis=-1, keepdims=True) + eps)
            return (y - mean) / den * ln_w + ln_b
        return (y - mean) / den * ln_w + ln_b + bonus
    return run


EPILOGUE_PINS = [
    lambda: P.test_group_norm_moments("numpy"),
    lambda: P.test_group_norm_affine_and_bonus_closed_form("numpy"),
]


@pytest.mark.parametrize("kind", ["sample_variance", "eps_outside_sqrt", "bonus_before_norm"])
def test_epilogue_mutant_is_caught(monkeypatch, kind):
    monkeypatch.setattr(reference, "group_norm_bonus", _epilogue(kind))
    assert _failures(EPILOGUE_PINS) >= 1


# ---- pre-processing mutants -----------------------------------------------------------------

def _prepare(kind):
    def run(w_logit, a_logit, k, k_k, k_a=None):
        w_logit, a_logit, k, k_k = (_f64(x) for x in (w_logit, a_logit, k, k_k))
        k_a = np.zeros_like(k_k) if k_a is None else _f64(k_a)
        sig = lambda x: 1.0 / (1.0 + np.exp(-x))
        w = np.exp(-sig(w_logit) / (math.e if kind == "decay_over_e" else math.sqrt(math.e)))
        a = sig(a_logit)
        k_tilde = k + k * (a - 1.0) * k_a
        kk = (k_tilde if kind == "kk_from_updated_key" else k) * k_k
        kk = kk / np.maximum(np.linalg.norm(kk, axis=-1, keepdims=True), 1e-12)
        return w, a, kk, k_tilde
    return run


PREP_PINS = [
    P.test_prepare_inputs_closed_forms,
    P.test_prepare_inputs_removal_key_uses_the_key_before_its_update,
    P.test_prepare_inputs_zero_key_is_finite,
]


@pytest.mark.parametrize("kind", ["decay_over_e", "kk_from_updated_key"])
def test_prepare_mutant_is_caught(monkeypatch, kind):
    monkeypatch.setattr(reference, "prepare_inputs", _prepare(kind))
    assert _failures(PREP_PINS) >= 1


# ---- backward mutants -----------------------------------------------------------------------

def _backward(kind):
    def run(r, w, k, v, kk, a, S0=None, dy=None, dS_T=None):
        r, w, k, v, kk, a = (_f64(x) for x in (r, w, k, v, kk, a))
        B, T, H, N = r.shape
        states = np.empty((T + 1, B, H, N, N))
        states[0] = 0.0 if S0 is None else _f64(S0)
        if T:
            _, _, snaps = reference.wkv7_recurrence(r, w, k, v, kk, a, states[0], snap_every=1)
            states[1:] = np.moveaxis(snaps, 1, 0)
        dy = np.zeros((B, T, H, N)) if dy is None else _f64(dy)
        dS = np.zeros((B, H, N, N)) if dS_T is None else _f64(dS_T).copy()
        out = {n: np.zeros((B, T, H, N)) for n in ("dr", "dw", "dk", "dv", "dkk", "da")}
        for t in range(T - 1, -1, -1):
            S_prev, S_t = states[t], states[t + 1]
            w_t, k_t, v_t, kk_t, a_t, r_t, dy_t = (x[:, t] for x in (w, k, v, kk, a, r, dy))
            dS = dS + dy_t[:, :, :, None] * r_t[:, :, None, :]
            out["dr"][:, t] = np.einsum("bhij,bhi->bhj", S_prev if kind == "dr_from_prev" else S_t, dy_t)
            out["dv"][:, t] = np.einsum("bhij,bhj->bhi", dS, k_t)
            out["dk"][:, t] = (np.einsum("bhij,bhj->bhi", dS, v_t) if kind == "dk_transposed"
                               else np.einsum("bhij,bhi->bhj", dS, v_t))
            out["dw"][:, t] = np.sum((S_t if kind == "dw_from_new" else S_prev) * dS, axis=-2)
            b_t = kk_t * a_t
            s = np.einsum("bhij,bhj->bhi", S_prev, kk_t)
            db = -np.einsum("bhij,bhi->bhj", dS, s)
            ds = -np.einsum("bhij,bhj->bhi", dS, b_t)
            out["dkk"][:, t] = np.einsum("bhij,bhi->bhj", S_prev, ds) + (0 if kind == "dkk_no_rate" else db * a_t)
            out["da"][:, t] = db * kk_t
            dS = dS * w_t[:, :, None, :]
            if kind != "no_removal_in_state_gradient":
                dS = dS + ds[:, :, :, None] * kk_t[:, :, None, :]
        out["dS0"] = dS
        return out
    return run


BACKWARD_PINS = [
    PB.test_backward_matches_finite_differences,
    PB.test_linear_attention_closed_form,
    PB.test_euler_identities,
]


@pytest.mark.parametrize("kind", ["dr_from_prev", "dk_transposed", "dw_from_new", "dkk_no_rate",
                                  "no_removal_in_state_gradient"])
def test_backward_mutant_is_caught(monkeypatch, kind):
    monkeypatch.setattr(reference, "wkv7_backward", _backward(kind))
    assert _failures(BACKWARD_PINS) >= 1


# ---- layer mutants --------------------------------------------------------------------------

from tests import test_oracle_layer as PL   # noqa: E402


def _layer_mutant(kind):
    def run(x, params, last_x=None, v0=None, S0=None, eps=64e-5):
        P = {n: _f64(params[n]) for n in reference.LAYER_PARAM_NAMES}
        x = _f64(x)
        B, T, C = x.shape
        H, N = P["r_k"].shape
        first = np.zeros((B, 1, C)) if (last_x is None or kind == "ignores_last_x") else _f64(last_x)[:, None]
        prev = np.concatenate([first, x[:, :-1]], axis=1)
        sgn = -1.0 if kind == "mix_sign" else 1.0
        mix = {m: x + sgn * P[m] * (prev - x) for m in ("mr", "mw", "mk", "mv", "ma", "mg")}
        sig = lambda z: 1.0 / (1.0 + np.exp(-z))
        r = mix["mr"] @ P["Wr"].T
        k = mix["mk"] @ P["Wk"].T
        v = mix["mv"] @ P["Wv"].T
        w_logit = np.tanh(mix["mw"] @ P["Ww1"]) @ P["Ww2"] + P["w_bias"]
        if v0 is None:
            v0 = v
        else:
            lerp = sig(mix["mv"] @ P["Wv1"] @ P["Wv2"] + P["v_bias"])
            v = v + ((v - _f64(v0)) if kind == "residual_sign" else (_f64(v0) - v)) * lerp
        a_logit = mix["ma"] @ P["Wa1"] @ P["Wa2"] + P["a_bias"]
        g = sig(mix["mg"] @ P["Wg1"] @ P["Wg2"]) if kind == "gate_sigmoid_outside" else sig(mix["mg"] @ P["Wg1"]) @ P["Wg2"]
        heads = lambda z: z.reshape(B, T, H, N)
        w, a, kk, k_t = reference.prepare_inputs(heads(w_logit), heads(a_logit), heads(k), P["k_k"], P["k_a"])
        y, S_T, _ = reference.wkv7_recurrence(heads(r), w, k_t, heads(v), kk, a, S0)
        y = reference.group_norm_bonus(y, heads(r), k_t, heads(v), P["ln_w"], P["ln_b"], P["r_k"], eps)
        return (y.reshape(B, T, C) * g) @ P["Wo"].T, v0, x[:, -1].copy(), S_T
    return run


LAYER_PINS = [
    PL.test_reduces_to_the_recurrence_and_epilogue,
    PL.test_full_mix_reads_only_the_previous_token,
    PL.test_value_residual_limits,
    PL.test_linear_in_output_projection_and_gate_output_factor,
    lambda: PL.test_sequence_split_carries_state_and_previous_token(3),
    lambda: PL.test_numpy_layer_matches_the_c_transcription(False, True, True),
    lambda: PL.test_numpy_layer_matches_the_c_transcription(True, True, True),
    PL.test_decay_path_is_tanh_between_its_factors,
    PL.test_rate_path_is_linear_between_its_factors,
    PL.test_value_residual_path_is_linear_between_its_factors,
    PL.test_gate_is_sigmoid_of_the_hidden_value_then_the_second_factor,
    PL.test_square_projections_take_the_stored_row_as_output_channel,
]


@pytest.mark.parametrize("kind", ["mix_sign", "residual_sign", "gate_sigmoid_outside", "ignores_last_x"])
def test_layer_mutant_is_caught(monkeypatch, kind):
    monkeypatch.setattr(reference, "time_mixing_layer", _layer_mutant(kind))
    assert _failures(LAYER_PINS) >= 1


def _projection_mutant(kind):
    """reference.layer_projections with one activation or one operand orientation changed."""
    def run(x, P, last_x=None, v0=None):
        B, T, C = x.shape
        prev = np.concatenate([np.zeros((B, 1, C)) if last_x is None else _f64(last_x)[:, None], x[:, :-1]], axis=1)
        mix = {m: x + P[m] * (prev - x) for m in ("mr", "mw", "mk", "mv", "ma", "mg")}
        sig = lambda z: 1.0 / (1.0 + np.exp(-z))
        ident = lambda z: z
        sq = (lambda xm, W: xm @ W) if kind == "transposed_square_projection" else (lambda xm, W: xm @ W.T)
        out = {"r": sq(mix["mr"], P["Wr"]), "k": sq(mix["mk"], P["Wk"])}
        v = sq(mix["mv"], P["Wv"])
        act_w = {"decay_no_tanh": ident, "decay_sigmoid": sig}.get(kind, np.tanh)
        out["w_logit"] = act_w(mix["mw"] @ P["Ww1"]) @ P["Ww2"] + P["w_bias"]
        if v0 is None:
            v0 = v
        else:
            act_v = np.tanh if kind == "residual_tanh" else ident
            v = v + (_f64(v0) - v) * sig(act_v(mix["mv"] @ P["Wv1"]) @ P["Wv2"] + P["v_bias"])
        out["v"], out["v0"] = v, v0
        act_a = {"rate_tanh": np.tanh, "rate_sigmoid": sig}.get(kind, ident)
        out["a_logit"] = act_a(mix["ma"] @ P["Wa1"]) @ P["Wa2"] + P["a_bias"]
        act_g = {"gate_no_sigmoid": ident, "gate_tanh": np.tanh}.get(kind, sig)
        out["g"] = act_g(mix["mg"] @ P["Wg1"]) @ P["Wg2"]
        return out
    return run


@pytest.mark.parametrize("kind", ["decay_no_tanh", "decay_sigmoid", "rate_tanh", "rate_sigmoid", "residual_tanh",
                                  "gate_no_sigmoid", "gate_tanh", "transposed_square_projection"])
def test_layer_projection_mutant_is_caught(monkeypatch, kind):
    monkeypatch.setattr(reference, "layer_projections", _projection_mutant(kind))
    assert _failures(LAYER_PINS) >= 1


def test_layer_with_transposed_output_projection_is_caught(monkeypatch):
    orig = reference.time_mixing_layer

    def run(x, params, last_x=None, v0=None, S0=None, eps=64e-5):
        p = dict(params)
        p["Wo"] = _f64(params["Wo"]).T
        return orig(x, p, last_x, v0, S0, eps)
    monkeypatch.setattr(reference, "time_mixing_layer", run)
    assert _failures(LAYER_PINS) >= 1


def test_unmutated_layer_passes_its_pins():
    assert _failures(LAYER_PINS) == 0


# ---- epilogue backward mutants -----------------------------------------------------------

from tests import test_oracle_epilogue_backward as PE  # noqa: E402


def _epilogue_backward(kind):
    def run(y, r, k, v, ln_w, ln_b, r_k, dout, eps=64e-5):
        y, r, k, v, ln_w, ln_b, r_k, dout = (_f64(x) for x in (y, r, k, v, ln_w, ln_b, r_k, dout))
        N = y.shape[-1]
        yc = y - y.mean(axis=-1, keepdims=True)
        var = (yc ** 2).sum(axis=-1, keepdims=True) / (N - 1 if kind == "sample_variance" else N)
        inv = 1.0 / np.sqrt(var + eps)
        yn = yc * inv
        beta = (r * k * r_k).sum(axis=-1, keepdims=True)
        dbeta = (dout * v).sum(axis=-1, keepdims=True)
        g = dout * ln_w
        corr = 0.0 if kind == "no_variance_term" else yn * (g * yn).mean(axis=-1, keepdims=True)
        dy = inv * (g - (0.0 if kind == "no_mean_term" else g.mean(axis=-1, keepdims=True)) - corr)
        dk = dbeta * (r if kind != "dk_uses_k" else k) * r_k
        return {"dy": dy, "dr": dbeta * k * r_k, "dk": dk, "dv": beta * dout,
                "dln_w": (dout * (yc if kind == "dln_w_unnormalised" else yn)).sum(axis=(0, 1)),
                "dln_b": dout.sum(axis=(0, 1)), "dr_k": (dbeta * r * k).sum(axis=(0, 1))}
    return run


@pytest.mark.parametrize("kind", ["sample_variance", "no_variance_term", "no_mean_term", "dk_uses_k",
                                  "dln_w_unnormalised"])
def test_epilogue_backward_mutant_is_caught(monkeypatch, kind):
    monkeypatch.setattr(reference, "group_norm_bonus_backward", _epilogue_backward(kind))
    failures = 0
    for name in ("y", "r", "k", "v", "ln_w", "ln_b", "r_k"):
        try:
            PE.test_matches_central_differences(name)
        except AssertionError:
            failures += 1
    for pin in (PE.test_normalisation_invariants, PE.test_branches_cut_off):
        try:
            pin()
        except AssertionError:
            failures += 1
    assert failures > 0, f"mutant {kind} passed every pin"
