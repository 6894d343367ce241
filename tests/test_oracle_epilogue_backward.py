"""Pins for the oracle's backward of the epilogue (group_norm + bonus), CPU fp64: central
finite differences of the pinned forward oracle for every input, the invariants of the
normalisation (a per-row shift of y changes nothing, so dy sums to zero per row; a scaling
of y changes the output only through eps), and the cases that cut a branch off."""
import numpy as np
import pytest

from oracle import reference


def _case(B=2, T=3, H=2, N=8, seed=5):
    g = np.random.default_rng(seed)
    x = {n: g.standard_normal((B, T, H, N)) for n in ("y", "r", "k", "v", "dout")}
    x.update({n: g.standard_normal((H, N)) for n in ("ln_w", "ln_b", "r_k")})
    return x


def _loss(x, eps=64e-5):
    out = reference.group_norm_bonus(x["y"], x["r"], x["k"], x["v"], x["ln_w"], x["ln_b"], x["r_k"], eps)
    return float((x["dout"] * out).sum())


@pytest.mark.parametrize("name", ["y", "r", "k", "v", "ln_w", "ln_b", "r_k"])
def test_matches_central_differences(name):
    x = _case()
    grad = reference.group_norm_bonus_backward(x["y"], x["r"], x["k"], x["v"], x["ln_w"], x["ln_b"], x["r_k"],
                                               x["dout"])["d" + name]
    h = 1e-6
    fd = np.zeros_like(x[name])
    for idx in np.ndindex(*x[name].shape):
        up = {n: a.copy() for n, a in x.items()}
        dn = {n: a.copy() for n, a in x.items()}
        up[name][idx] += h
        dn[name][idx] -= h
        fd[idx] = (_loss(up) - _loss(dn)) / (2 * h)
    np.testing.assert_allclose(grad, fd, rtol=1e-6, atol=1e-7 * max(1.0, np.abs(fd).max()))


def test_normalisation_invariants():
    """out(y + c) = out(y) per row: dy sums to zero over a head's channels. out(s y) differs
    from out(y) only through eps: sum_j dy_j y_j is small against |dy| |y| (zero as eps -> 0)."""
    x = _case(B=3, T=4, H=3, N=16, seed=7)
    d = reference.group_norm_bonus_backward(x["y"], x["r"], x["k"], x["v"], x["ln_w"], x["ln_b"], x["r_k"],
                                            x["dout"], eps=0.0)
    np.testing.assert_allclose(d["dy"].sum(axis=-1), 0.0, atol=1e-12)
    np.testing.assert_allclose((d["dy"] * x["y"]).sum(axis=-1), 0.0, atol=1e-11)


def test_branches_cut_off():
    """ln_w = 0: the normalised branch carries no gradient to y. r_k = 0: no bonus, so dr,
    dk, dv vanish. v = 0: dr, dk, dr_k vanish but dv = beta dout."""
    x = _case(seed=9)
    f = lambda **o: reference.group_norm_bonus_backward(*[o.get(n, x[n]) for n in ("y", "r", "k", "v", "ln_w", "ln_b",
                                                                                   "r_k", "dout")])
    assert np.abs(f(ln_w=np.zeros_like(x["ln_w"]))["dy"]).max() == 0.0
    d = f(r_k=np.zeros_like(x["r_k"]))
    assert max(np.abs(d[n]).max() for n in ("dr", "dk", "dv")) == 0.0
    d = f(v=np.zeros_like(x["v"]))
    assert max(np.abs(d[n]).max() for n in ("dr", "dk", "dr_k")) == 0.0
    beta = (x["r"] * x["k"] * x["r_k"]).sum(axis=-1, keepdims=True)
    np.testing.assert_allclose(d["dv"], beta * x["dout"], rtol=1e-14)
