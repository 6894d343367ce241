"""GPU parity of the backward pass (through the C ABI) against the oracle's fp64 reverse
sweep on the same seeded inputs. The kernel works in fp32 from inputs that are exact in
fp32 (bf16 or fp32), so one bound serves both: max relative error per (b, h) slice
<= 9e-5, the precision the pages report for their fp32 backward."""
import dataclasses

import numpy as np
import pytest
import torch

from linear_rnn_sequence_rwkv_b200 import inputs, wkv7
from oracle import reference
from tests.parity_util import slice_rel_err, state_err, y_err

pytestmark = pytest.mark.gpu

TOL_BWD = 9e-5
NAMES = ("r", "w", "k", "v", "kk", "a")


def _case(B, T, H, *, dtype="bf16", seed=0, s0="normal", ds_t=True, wl=1, N=64):
    work = dataclasses.replace(inputs.WORKLOADS[wl], N=N)
    d = inputs.make_inputs(work, B=B, T=T, H=H, dtype=dtype, seed=seed, s0=s0)
    g = torch.Generator().manual_seed(seed + 1)
    d["dy"] = torch.randn(B, T, H, N, generator=g)
    d["dS_T"] = 0.1 * torch.randn(B, H, N, N, generator=g) if ds_t else None
    return d


def _oracle(d):
    return reference.wkv7_backward(*(d[n] for n in NAMES), d.get("S0"), d["dy"], d["dS_T"])


def _dev(d, device):
    return {k: (None if v is None else v.to(device)) for k, v in d.items()}


def _check(got, ref, tol=TOL_BWD):
    errs = {n: y_err(got[n], ref[n]) for n in wkv7.GRAD_NAMES}
    if got.get("dS0") is not None:
        errs["dS0"] = state_err(got["dS0"], ref["dS0"])
    assert max(errs.values()) <= tol, errs
    return errs


@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 8, 37, 130])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_ragged_lengths(cuda_device, T, dtype):
    d = _case(2, T, 3, dtype=dtype, seed=500 + T)
    ref = _oracle(d)
    dd = _dev(d, cuda_device)
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"], dd["S0"], dd["dS_T"])
    _check(got, ref)


def test_backward_zero_state_and_no_state_gradient(cuda_device):
    d = _case(1, 45, 2, seed=520, s0="zeros", ds_t=False)
    ref = _oracle(d)
    dd = _dev(d, cuda_device)
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"])
    _check(got, ref)


@pytest.mark.parametrize("snap_every", [7, 16, 50, 64])
def test_backward_from_forward_snapshots(cuda_device, snap_every):
    """Recomputation anchored at the snapshots an fp32 scan forward wrote gives the same
    gradients as recomputation from S0 alone."""
    d = _case(2, 200, 2, seed=530 + snap_every)
    ref = _oracle(d)
    dd = _dev(d, cuda_device)
    _, _, snaps = wkv7.forward(*(dd[n] for n in NAMES), dd["S0"], snap_every=snap_every, algo="seq")
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"], dd["S0"], dd["dS_T"], snapshots=snaps,
                        snap_every=snap_every)
    _check(got, ref)


def test_backward_empty_sequence_and_in_place_state_gradient(cuda_device):
    d = _case(2, 0, 3, seed=540)
    dd = _dev(d, cuda_device)
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"], dd["S0"], dd["dS_T"])
    assert torch.equal(got["dS0"], dd["dS_T"])
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"], dd["S0"], None)
    assert torch.count_nonzero(got["dS0"]) == 0
    d = _case(1, 21, 2, seed=541)
    ref = _oracle(d)
    dd = _dev(d, cuda_device)
    g_in = dd["dS_T"].clone()
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"], dd["S0"], g_in, dS0=g_in)
    assert got["dS0"] is g_in
    _check(got, ref)


def test_backward_from_chunked_forward_snapshots(cuda_device):
    """Anchored at the tf32 chunked forward's snapshots, the gradients that read the states
    (dr, dw, dkk, da, through S) inherit the forward's precision (the bf16 forward bound,
    2e-3); dk, dv and dS0 read only the state gradient and keep the fp32 bound."""
    d = _case(2, 256, 3, seed=545)
    ref = _oracle(d)
    dd = _dev(d, cuda_device)
    _, _, snaps = wkv7.forward(*(dd[n] for n in NAMES), dd["S0"], snap_every=64, algo="chunk")
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"], dd["S0"], dd["dS_T"], snapshots=snaps, snap_every=64)
    errs = _check(got, ref, tol=2e-3)
    assert max(errs["dk"], errs["dv"], errs["dS0"]) <= TOL_BWD


def test_backward_prefill_019b_sampled_heads(cuda_device):
    """0.19B-shaped workload (B8 T1024 H12, bf16, S0), snapshots every 64 tokens from the
    fp32 scan forward; the oracle runs on six sampled (b, h) pairs."""
    wl = inputs.WORKLOADS[1]
    d = _case(wl.B, wl.T, wl.H, seed=550)
    dd = _dev(d, cuda_device)
    _, _, snaps = wkv7.forward(*(dd[n] for n in NAMES), dd["S0"], snap_every=64, algo="seq")
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"], dd["S0"], dd["dS_T"], snapshots=snaps, snap_every=64)
    pairs = [(0, 0), (3, 7), (7, 11), (5, 2), (1, 9), (6, 4)]
    sub = {n: torch.stack([d[n][b, :, h] for b, h in pairs])[:, :, None] for n in NAMES + ("dy",)}
    sub["S0"] = torch.stack([d["S0"][b, h] for b, h in pairs])[:, None]
    sub["dS_T"] = torch.stack([d["dS_T"][b, h] for b, h in pairs])[:, None]
    ref = _oracle(sub)
    sel = {n: torch.stack([got[n][b, :, h] for b, h in pairs])[:, :, None] for n in wkv7.GRAD_NAMES}
    sel["dS0"] = torch.stack([got["dS0"][b, h] for b, h in pairs])[:, None]
    _check(sel, ref)


def test_backward_prefill_15b_sampled_heads(cuda_device):
    """The backward bench's launch: B16 T4096 H32 bf16 with S0 and dS_T, snapshots every 64
    tokens from the fp32 scan forward, all 512 heads in one launch (3.5 waves of CTAs). Inputs
    are drawn on the device; the oracle runs on four sampled (b, h) pairs, one from each wave."""
    wl = inputs.WORKLOADS[2]
    d = inputs.make_inputs(wl, device=str(cuda_device), seed=560)
    g = torch.Generator(device=cuda_device).manual_seed(561)
    d["dy"] = torch.randn(wl.B, wl.T, wl.H, 64, device=cuda_device, generator=g)
    d["dS_T"] = 0.1 * torch.randn(wl.B, wl.H, 64, 64, device=cuda_device, generator=g)
    if d["S0"] is None:
        d["S0"] = 0.1 * torch.randn(wl.B, wl.H, 64, 64, device=cuda_device, generator=g)
    _, _, snaps = wkv7.forward(*(d[n] for n in NAMES), d["S0"], snap_every=64, algo="seq")
    got = wkv7.backward(*(d[n] for n in NAMES), d["dy"], d["S0"], d["dS_T"], snapshots=snaps, snap_every=64)
    pairs = [(0, 0), (4, 20), (9, 17), (15, 31)]   # units b*H + h = 0, 148, 305, 511
    sub = {n: torch.stack([d[n][b, :, h] for b, h in pairs])[:, :, None].cpu() for n in NAMES + ("dy",)}
    sub["S0"] = torch.stack([d["S0"][b, h] for b, h in pairs])[:, None].cpu()
    sub["dS_T"] = torch.stack([d["dS_T"][b, h] for b, h in pairs])[:, None].cpu()
    ref = _oracle(sub)
    sel = {n: torch.stack([got[n][b, :, h] for b, h in pairs])[:, :, None].cpu() for n in wkv7.GRAD_NAMES}
    sel["dS0"] = torch.stack([got["dS0"][b, h] for b, h in pairs])[:, None].cpu()
    _check(sel, ref)


def test_gpu_gradients_match_finite_difference_of_the_oracle_forward(cuda_device):
    """A directional derivative of the oracle's fp64 forward (central difference along a
    random direction of every input) equals the GPU gradients contracted with that direction.
    The fp64 oracle is differentiated, not the GPU forward: an fp32 forward's rounding would
    swamp a central difference."""
    d = _case(1, 24, 2, dtype="f32", seed=560)
    dd = _dev(d, cuda_device)
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"], dd["S0"], dd["dS_T"])
    g = torch.Generator().manual_seed(561)
    dirs = {n: torch.randn(d[n].shape, generator=g, dtype=torch.float64) for n in NAMES}
    eps = 1e-3

    def loss(sign):
        x = {n: (d[n].double() + sign * eps * dirs[n]) for n in NAMES}
        y, S, _ = reference.wkv7_recurrence(*(x[n] for n in NAMES), d["S0"])
        return float(np.sum(d["dy"].double().numpy() * y) + np.sum(d["dS_T"].double().numpy() * S))
    fd = (loss(1) - loss(-1)) / (2 * eps)
    lin = sum(float((got["d" + n].double().cpu() * dirs[n]).sum()) for n in NAMES)
    assert abs(fd - lin) <= 1e-4 * max(1.0, abs(fd))


# ---- head size 128: the rows of a head split over a cluster of two CTAs, two-token blocks ----

@pytest.mark.parametrize("T", [1, 2, 3, 5, 37, 130])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_n128_ragged_lengths(cuda_device, T, dtype):
    d = _case(2, T, 3, dtype=dtype, seed=1700 + T, N=128)
    ref = _oracle(d)
    dd = _dev(d, cuda_device)
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"], dd["S0"], dd["dS_T"])
    _check(got, ref)


@pytest.mark.parametrize("snap_every", [7, 64])
def test_backward_n128_from_forward_snapshots(cuda_device, snap_every):
    d = _case(2, 150, 2, seed=1750 + snap_every, N=128)
    ref = _oracle(d)
    dd = _dev(d, cuda_device)
    _, _, snaps = wkv7.forward(*(dd[n] for n in NAMES), dd["S0"], snap_every=snap_every, algo="seq")
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"], dd["S0"], dd["dS_T"], snapshots=snaps,
                        snap_every=snap_every)
    _check(got, ref)


def test_backward_n128_no_state_and_in_place_state_gradient(cuda_device):
    d = _case(1, 20, 2, seed=1770, s0="zeros", N=128)
    ref = _oracle(d)
    dd = _dev(d, cuda_device)
    dS = dd["dS_T"].clone()
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"], None, dS, dS0=dS)
    _check(got, ref)
    assert got["dS0"].data_ptr() == dS.data_ptr()


def test_backward_n128_sampled_heads(cuda_device):
    """B8 T1024 H6 N128 (the 0.19B channel count in 128-wide heads, bf16, S0), snapshots every 64
    tokens from the scan forward; the oracle runs on four sampled (b, h) pairs."""
    d = _case(8, 1024, 6, seed=1790, N=128)
    dd = _dev(d, cuda_device)
    _, _, snaps = wkv7.forward(*(dd[n] for n in NAMES), dd["S0"], snap_every=64, algo="seq")
    got = wkv7.backward(*(dd[n] for n in NAMES), dd["dy"], dd["S0"], dd["dS_T"], snapshots=snaps, snap_every=64)
    pairs = [(0, 0), (3, 5), (6, 2), (7, 5)]
    sub = {n: torch.stack([d[n][b, :, h] for b, h in pairs])[:, :, None] for n in NAMES + ("dy",)}
    sub["S0"] = torch.stack([d["S0"][b, h] for b, h in pairs])[:, None]
    sub["dS_T"] = torch.stack([d["dS_T"][b, h] for b, h in pairs])[:, None]
    ref = _oracle(sub)
    sel = {n: torch.stack([got[n][b, :, h] for b, h in pairs])[:, :, None] for n in wkv7.GRAD_NAMES}
    sel["dS0"] = torch.stack([got["dS0"][b, h] for b, h in pairs])[:, None]
    _check(sel, ref)
