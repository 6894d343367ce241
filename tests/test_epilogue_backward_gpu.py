"""GPU parity of the epilogue on its own and of its backward (wkv7_epilogue,
wkv7_epilogue_backward) against the fp64 oracle, and the training chain they make with the
forward and backward of the recurrence.

Bounds (max relative error per (b, h) slice, as everywhere): 2e-5 for the per-row gradients
and the epilogue (fp32 arithmetic over a head's N channels: row sums of N terms, then one
division by the standard deviation); 1e-4 for the parameter gradients, which sum B * T rows
in fp32."""
import numpy as np
import pytest
import torch

from linear_rnn_sequence_rwkv_b200 import inputs, wkv7
from oracle import reference
from tests.parity_util import slice_rel_err

pytestmark = pytest.mark.gpu

TOL_ROW, TOL_PARAM = 2e-5, 1e-4


def _case(B, T, H, N, dtype, seed, dev):
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = {n: torch.randn(B, T, H, N, generator=g) for n in ("y", "dout")}
    x.update({n: torch.randn(B, T, H, N, generator=g).to(dt) for n in ("r", "k", "v")})
    x["ln_w"] = 1.0 + 0.1 * torch.randn(H, N, generator=g)
    x["ln_b"] = 0.1 * torch.randn(H, N, generator=g)
    x["r_k"] = 0.5 * torch.randn(H, N, generator=g)
    return x, {n: t.to(dev) for n, t in x.items()}


def _param_err(got, ref):
    ref = np.asarray(ref)
    return float(np.abs(got.double().cpu().numpy() - ref).max() / max(np.abs(ref).max(), 1e-30))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("T", [1, 37, 200])
def test_epilogue_backward_matches_oracle(cuda_device, dtype, N, T):
    x, d = _case(2, T, 3, N, dtype, seed=1000 + T + N, dev=cuda_device)
    ref = reference.group_norm_bonus_backward(x["y"], x["r"], x["k"], x["v"], x["ln_w"], x["ln_b"], x["r_k"], x["dout"])
    got = wkv7.epilogue_backward(d["y"], d["r"], d["k"], d["v"], d["ln_w"], d["ln_b"], d["r_k"], d["dout"])
    for n in ("dy", "dr", "dk", "dv"):
        assert slice_rel_err(got[n], ref[n], (0, 2)) <= TOL_ROW, n
    for n in ("dln_w", "dln_b", "dr_k"):
        assert _param_err(got[n], ref[n]) <= TOL_PARAM, n


def test_epilogue_backward_more_heads_than_a_grid_row(cuda_device):
    """H = 70,000 heads, more than a grid's y extent: one CTA per (row block, head) in x."""
    x, d = _case(1, 3, 70000, 64, "bf16", seed=1090, dev=cuda_device)
    ref = reference.group_norm_bonus_backward(x["y"], x["r"], x["k"], x["v"], x["ln_w"], x["ln_b"], x["r_k"], x["dout"])
    got = wkv7.epilogue_backward(d["y"], d["r"], d["k"], d["v"], d["ln_w"], d["ln_b"], d["r_k"], d["dout"])
    for n in ("dy", "dr", "dk", "dv"):
        assert slice_rel_err(got[n], ref[n], (0, 2)) <= TOL_ROW, n
    for n in ("dln_w", "dln_b", "dr_k"):
        assert _param_err(got[n], ref[n]) <= TOL_PARAM, n


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_epilogue_out_of_place_matches_oracle_and_fused(cuda_device, dtype):
    """wkv7_epilogue equals the oracle, leaves y untouched, and equals the epilogue fused into
    the forward (same fp32 arithmetic per row; the fused path reads the same y)."""
    x, d = _case(2, 50, 3, 64, dtype, seed=1100, dev=cuda_device)
    y0 = d["y"].clone()
    out = wkv7.epilogue(d["y"], d["r"], d["k"], d["v"], d["ln_w"], d["ln_b"], d["r_k"])
    ref = reference.group_norm_bonus(x["y"], x["r"], x["k"], x["v"], x["ln_w"], x["ln_b"], x["r_k"])
    assert slice_rel_err(out, ref, (0, 2)) <= TOL_ROW
    assert torch.equal(d["y"], y0)
    inplace = d["y"].clone()
    wkv7.epilogue(inplace, d["r"], d["k"], d["v"], d["ln_w"], d["ln_b"], d["r_k"], out=inplace)
    assert torch.equal(inplace, out)


def test_parameter_gradients_are_reproducible_and_T0_gives_zeros(cuda_device):
    x, d = _case(4, 300, 2, 64, "bf16", seed=1200, dev=cuda_device)
    a = wkv7.epilogue_backward(d["y"], d["r"], d["k"], d["v"], d["ln_w"], d["ln_b"], d["r_k"], d["dout"])
    b = wkv7.epilogue_backward(d["y"], d["r"], d["k"], d["v"], d["ln_w"], d["ln_b"], d["r_k"], d["dout"])
    for n in wkv7.EPILOGUE_GRAD_NAMES:
        assert torch.equal(a[n], b[n]), n
    e = {n: d[n][:, :0].contiguous() for n in ("y", "r", "k", "v", "dout")}
    z = wkv7.epilogue_backward(e["y"], e["r"], e["k"], e["v"], d["ln_w"], d["ln_b"], d["r_k"], e["dout"])
    for n in ("dln_w", "dln_b", "dr_k"):
        assert torch.count_nonzero(z[n]) == 0


def test_epilogue_backward_at_the_bench_shape(cuda_device):
    """B8 T1024 H12 N64, bf16 inputs: every row and every parameter gradient."""
    x, d = _case(8, 1024, 12, 64, "bf16", seed=1300, dev=cuda_device)
    ref = reference.group_norm_bonus_backward(x["y"], x["r"], x["k"], x["v"], x["ln_w"], x["ln_b"], x["r_k"], x["dout"])
    got = wkv7.epilogue_backward(d["y"], d["r"], d["k"], d["v"], d["ln_w"], d["ln_b"], d["r_k"], d["dout"])
    for n in ("dy", "dr", "dk", "dv"):
        assert slice_rel_err(got[n], ref[n], (0, 2)) <= TOL_ROW, n
    for n in ("dln_w", "dln_b", "dr_k"):
        assert _param_err(got[n], ref[n]) <= TOL_PARAM, n


def test_training_chain_with_the_epilogue(cuda_device):
    """forward without the epilogue -> wkv7_epilogue -> L = <dout, out>; the gradients from
    wkv7_epilogue_backward then wkv7_backward (dr, dk, dv summed) equal the oracle's chain
    (group_norm_bonus_backward, then wkv7_backward with its dy) within the backward's bound."""
    B, T, H = 2, 96, 3
    x = inputs.make_inputs(inputs.WORKLOADS[0], seed=1400, device="cpu", B=B, T=T, H=H, dtype="f32")
    g = torch.Generator().manual_seed(1401)
    ln_w, ln_b, r_k = 1.0 + 0.1 * torch.randn(H, 64, generator=g), 0.1 * torch.randn(H, 64, generator=g), \
        0.5 * torch.randn(H, 64, generator=g)
    dout = torch.randn(B, T, H, 64, generator=g)
    names = ("r", "w", "k", "v", "kk", "a")
    d = {n: x[n].to(cuda_device) for n in names}
    y, _, _ = wkv7.forward(*(d[n] for n in names), None, return_state=False)
    ep = wkv7.epilogue_backward(y, d["r"], d["k"], d["v"], ln_w.to(cuda_device), ln_b.to(cuda_device),
                                r_k.to(cuda_device), dout.to(cuda_device))
    gr = wkv7.backward(*(d[n] for n in names), ep["dy"], return_state_grad=False)
    y_ref, _, _ = reference.wkv7_recurrence(*(x[n] for n in names))
    e_ref = reference.group_norm_bonus_backward(y_ref, x["r"], x["k"], x["v"], ln_w, ln_b, r_k, dout)
    g_ref = reference.wkv7_backward(*(x[n] for n in names), dy=e_ref["dy"])
    for n in ("dr", "dk", "dv"):
        assert slice_rel_err(gr[n] + ep[n], g_ref[n] + e_ref[n], (0, 2)) <= 1e-4, n
    for n in ("dw", "dkk", "da"):
        assert slice_rel_err(gr[n], g_ref[n], (0, 2)) <= 1e-4, n
