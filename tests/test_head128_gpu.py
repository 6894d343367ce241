"""GPU parity for head size N = 128 (scan, its epilogue, the raw-input staging and the decode
step) against the fp64 oracle, which takes any N; tolerances as for N = 64."""
import dataclasses

import pytest
import torch

from linear_rnn_sequence_rwkv_b200 import inputs, wkv7
from oracle import native, reference
from tests.parity_util import TOL, snaps_err, state_err, y_err

pytestmark = pytest.mark.gpu

NAMES = ("r", "w", "k", "v", "kk", "a")
WL = dataclasses.replace(inputs.WORKLOADS[1], N=128)
WL_EPI = dataclasses.replace(inputs.WORKLOADS[2], N=128)


def _dev(d, device):
    return {k: (None if v is None else v.to(device)) for k, v in d.items()}


def _oracle(d, snap_every=0):
    return native.forward(*(d[n] for n in NAMES), d.get("S0"), snap_every=snap_every)


@pytest.mark.parametrize("T", [1, 5, 17, 33, 100, 257])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_scan_n128_ragged(cuda_device, T, dtype):
    d = inputs.make_inputs(WL, B=2, T=T, H=3, dtype=dtype, seed=700 + T, s0="normal")
    y_ref, S_ref, _ = _oracle(d)
    dd = _dev(d, cuda_device)
    y, S, _ = wkv7.forward(*(dd[n] for n in NAMES), dd["S0"], algo="auto")
    assert y.shape == (2, T, 3, 128)
    assert y_err(y, y_ref) <= TOL[dtype]
    assert state_err(S, S_ref) <= TOL[dtype]


def test_scan_n128_many_heads_and_auto_is_scan(cuda_device):
    """Enough heads for the two-rows-per-thread layout; AUTO equals SEQ bit for bit."""
    d = inputs.make_inputs(WL, B=8, T=200, H=40, seed=720, s0="normal")
    dd = _dev(d, cuda_device)
    y, S, _ = wkv7.forward(*(dd[n] for n in NAMES), dd["S0"], algo="seq")
    y2, S2, _ = wkv7.forward(*(dd[n] for n in NAMES), dd["S0"])
    assert torch.equal(y, y2) and torch.equal(S, S2)
    pairs = [(0, 0), (3, 17), (7, 39)]
    sub = {n: torch.stack([d[n][b, :, h] for b, h in pairs])[:, :, None] for n in NAMES}
    sub["S0"] = torch.stack([d["S0"][b, h] for b, h in pairs])[:, None]
    y_ref, S_ref, _ = _oracle(sub)
    ys = torch.stack([y[b, :, h] for b, h in pairs])[:, :, None]
    Ss = torch.stack([S[b, h] for b, h in pairs])[:, None]
    assert y_err(ys, y_ref) <= TOL["bf16"]
    assert state_err(Ss, S_ref) <= TOL["bf16"]


@pytest.mark.parametrize("snap_every", [7, 64])
def test_scan_n128_snapshots(cuda_device, snap_every):
    d = inputs.make_inputs(WL, B=1, T=150, H=2, seed=730, s0="normal")
    y_ref, S_ref, sn_ref = _oracle(d, snap_every)
    dd = _dev(d, cuda_device)
    y, S, sn = wkv7.forward(*(dd[n] for n in NAMES), dd["S0"], snap_every=snap_every)
    assert snaps_err(sn, sn_ref) <= TOL["bf16"]
    assert y_err(y, y_ref) <= TOL["bf16"]


def test_scan_n128_epilogue(cuda_device):
    d = inputs.make_inputs(WL_EPI, B=2, T=70, H=3, seed=740)
    y_ref, _, _ = _oracle(d)
    out_ref = native.epilogue(y_ref, d["r"], d["k"], d["v"], d["ln_w"], d["ln_b"], d["r_k"])
    dd = _dev(d, cuda_device)
    y, _, _ = wkv7.forward(*(dd[n] for n in NAMES), dd["S0"], ln_w=dd["ln_w"], ln_b=dd["ln_b"], r_k=dd["r_k"])
    assert y_err(y, out_ref) <= TOL["bf16"]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_raw_n128(cuda_device, dtype):
    d = inputs.make_raw_inputs(WL_EPI, B=2, T=45, H=2, seed=750, s0="normal", dtype=dtype)
    w, a, kk, kt = reference.prepare_inputs(d["w_logit"], d["a_logit"], d["k"], d["k_k"], d["k_a"])
    y_ref, S_ref, _ = native.forward(d["r"], w, kt, d["v"], kk, a, d["S0"])
    out_ref = native.epilogue(y_ref, d["r"], kt, d["v"], d["ln_w"], d["ln_b"], d["r_k"])
    dd = _dev(d, cuda_device)
    y, S, _ = wkv7.forward_raw(dd["r"], dd["w_logit"], dd["k"], dd["v"], dd["a_logit"], dd["k_k"], dd["k_a"],
                               dd["S0"], ln_w=dd["ln_w"], ln_b=dd["ln_b"], r_k=dd["r_k"])
    assert y_err(y, out_ref) <= TOL[dtype]
    assert state_err(S, S_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_n128(cuda_device, dtype):
    T = 12
    d = inputs.make_inputs(WL, B=3, T=T, H=4, dtype=dtype, seed=760, s0="normal")
    y_ref, S_ref, _ = _oracle(d)
    dd = _dev(d, cuda_device)
    S = dd["S0"].clone()
    ys = [wkv7.decode_step(*(dd[n][:, t].contiguous() for n in NAMES), S).clone() for t in range(T)]
    assert y_err(torch.stack(ys, dim=1), y_ref) <= TOL[dtype]
    assert state_err(S, S_ref) <= TOL[dtype]


def test_n128_refused_where_unsupported(cuda_device):
    d = _dev(inputs.make_inputs(WL, B=1, T=64, H=1, seed=770), cuda_device)
    with pytest.raises(wkv7.Wkv7Error) as e:
        wkv7.forward(*(d[n] for n in NAMES), algo="chunk")
    assert e.value.status == wkv7.ERR_UNSUPPORTED
