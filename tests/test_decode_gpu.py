"""GPU parity of the decode step's fused options (through the C ABI): the group_norm + bonus
epilogue and the raw time-mixing inputs, each against the fp64 oracle run over the same tokens
(decode steps are the recurrence one token at a time), and against the library's own
full-sequence forward with the same options."""
import dataclasses

import pytest
import torch

from linear_rnn_sequence_rwkv_b200 import inputs, wkv7
from oracle import native, reference
from tests.parity_util import TOL, state_err, y_err

pytestmark = pytest.mark.gpu

NAMES = ("r", "w", "k", "v", "kk", "a")
RAW = ("r", "w_logit", "k", "v", "a_logit")


def _wl(N):
    return dataclasses.replace(inputs.WORKLOADS[2], N=N)   # the workload with the epilogue


def _dev(d, device):
    return {k: (None if v is None else v.to(device)) for k, v in d.items()}


def _epi(d):
    return dict(ln_w=d["ln_w"], ln_b=d["ln_b"], r_k=d["r_k"])


@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_epilogue_matches_oracle(cuda_device, N, dtype):
    T = 6
    d = inputs.make_inputs(_wl(N), B=3, T=T, H=2, dtype=dtype, seed=1200 + N, s0="normal")
    y_ref, S_ref, _ = native.forward(*(d[n] for n in NAMES), d["S0"])
    out_ref = native.epilogue(y_ref, d["r"], d["k"], d["v"], d["ln_w"], d["ln_b"], d["r_k"])
    dd = _dev(d, cuda_device)
    S = dd["S0"].clone()
    ys = [wkv7.decode_step(*(dd[n][:, t].contiguous() for n in NAMES), S, **_epi(dd)).clone() for t in range(T)]
    assert y_err(torch.stack(ys, 1), out_ref) <= TOL[dtype]
    assert state_err(S, S_ref) <= TOL[dtype]


@pytest.mark.parametrize("N", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("epilogue", [False, True])
@pytest.mark.parametrize("with_k_a", [True, False])
def test_decode_raw_matches_oracle(cuda_device, N, dtype, epilogue, with_k_a):
    """Raw inputs: the oracle's fp64 pre-processing, then its recurrence (and epilogue, whose
    bonus uses the updated key)."""
    T = 5
    d = inputs.make_raw_inputs(_wl(N), B=2, T=T, H=3, dtype=dtype, seed=1300 + N + 7 * with_k_a,
                               s0="normal", k_a=with_k_a)
    w, a, kk, kt = reference.prepare_inputs(d["w_logit"], d["a_logit"], d["k"], d["k_k"], d["k_a"])
    y_ref, S_ref, _ = native.forward(d["r"], w, kt, d["v"], kk, a, d["S0"])
    if epilogue:
        y_ref = native.epilogue(y_ref, d["r"], kt, d["v"], d["ln_w"], d["ln_b"], d["r_k"])
    dd = _dev(d, cuda_device)
    S = dd["S0"].clone()
    kw = _epi(dd) if epilogue else {}
    ka = dd["k_a"] if with_k_a else None
    ys = [wkv7.decode_step_raw(*(dd[n][:, t].contiguous() for n in RAW), dd["k_k"], S, k_a=ka, **kw).clone()
          for t in range(T)]
    assert y_err(torch.stack(ys, 1), y_ref) <= TOL[dtype]
    assert state_err(S, S_ref) <= TOL[dtype]


@pytest.mark.parametrize("N", [64, 128])
def test_decode_raw_epilogue_matches_forward_raw(cuda_device, N):
    """Decode steps chained over T tokens give the full-sequence raw forward's output and state
    (both fp32 arithmetic on the same inputs; the scan and the decode step reduce in other
    orders)."""
    T = 9
    d = _dev(inputs.make_raw_inputs(_wl(N), B=2, T=T, H=4, seed=1400 + N, s0="normal"), cuda_device)
    yf, Sf, _ = wkv7.forward_raw(*(d[n] for n in RAW), d["k_k"], d["k_a"], d["S0"], algo="seq", **_epi(d))
    S = d["S0"].clone()
    ys = [wkv7.decode_step_raw(*(d[n][:, t].contiguous() for n in RAW), d["k_k"], S, k_a=d["k_a"],
                               **_epi(d)).clone() for t in range(T)]
    assert y_err(torch.stack(ys, 1), yf) <= 1e-5
    assert state_err(S, Sf) <= 1e-5


def test_decode_29b_raw_epilogue_sampled(cuda_device):
    """2.9B-shaped decode (B256 H40) from raw inputs with the epilogue, 16 steps; six heads
    checked against the oracle."""
    wl = dataclasses.replace(inputs.WORKLOADS[3], T=16, epilogue=True)
    d = inputs.make_raw_inputs(wl, device=str(cuda_device), seed=1500)
    B, T, H, N = d["r"].shape
    S = torch.zeros(B, H, N, N, device=cuda_device)
    ys = torch.empty(T, B, H, N, device=cuda_device)
    for t in range(T):
        wkv7.decode_step_raw(*(d[n][:, t].contiguous() for n in RAW), d["k_k"], S, k_a=d["k_a"], y=ys[t],
                             **_epi(d))
    pairs = [(0, 0), (17, 39), (100, 3), (200, 20), (255, 0), (255, 39)]
    pick = lambda x: torch.stack([x[b, :, h] for b, h in pairs])[:, :, None].cpu()
    sub = {n: pick(d[n]) for n in RAW}
    y_ref, S_ref = [], []
    for i, (_, h) in enumerate(pairs):
        one = {n: sub[n][i:i + 1] for n in RAW}
        kk_, ka_ = d["k_k"][h:h + 1].cpu(), d["k_a"][h:h + 1].cpu()
        w, a, kk, kt = reference.prepare_inputs(one["w_logit"], one["a_logit"], one["k"], kk_, ka_)
        y1, S1, _ = native.forward(one["r"], w, kt, one["v"], kk, a, None)
        y1 = native.epilogue(y1, one["r"], kt, one["v"], d["ln_w"][h:h + 1].cpu(), d["ln_b"][h:h + 1].cpu(),
                             d["r_k"][h:h + 1].cpu())
        y_ref.append(y1)
        S_ref.append(S1)
    y_got = torch.stack([ys[:, b, h] for b, h in pairs])[:, :, None, :]
    S_got = torch.stack([S[b, h] for b, h in pairs])[:, None]
    assert y_err(y_got, torch.cat([torch.as_tensor(y) for y in y_ref])) <= TOL["bf16"]
    assert state_err(S_got, torch.cat([torch.as_tensor(s) for s in S_ref])) <= TOL["bf16"]


def test_decode_options_rejected(cuda_device):
    d = _dev(inputs.make_raw_inputs(_wl(64), B=1, T=1, H=2, seed=1600, s0="normal"), cuda_device)
    S = d["S0"].clone()
    step = [d[n][:, 0].contiguous() for n in RAW]
    with pytest.raises(wkv7.Wkv7Error) as e:
        wkv7.decode_step_raw(*step, d["k_k"], S, ln_w=d["ln_w"], ln_b=d["ln_b"])   # r_k missing
    assert e.value.status == wkv7.ERR_ARG
    with pytest.raises(wkv7.Wkv7Error) as e:
        wkv7.decode_step_raw(*step, None, S)
    assert e.value.status == wkv7.ERR_ARG
    with pytest.raises(wkv7.Wkv7Error) as e:
        wkv7.decode_step_raw(*step, d["k_k"].cpu(), S)                               # host parameter
    assert e.value.status == wkv7.ERR_ARG
    with pytest.raises(wkv7.Wkv7Error) as e:
        wkv7.decode_step_raw(*step, d["k_k"], S, gn_eps=0.0, **_epi(d))
    assert e.value.status == wkv7.ERR_ARG
