"""GPU parity of the raw-input forward (decay and rate logits, the key before its update,
per-head k_k and k_a) against the oracle's fp64 pre-processing followed by its recurrence."""
import numpy as np
import pytest
import torch

from linear_rnn_sequence_rwkv_b200 import inputs, wkv7
from oracle import native, reference
from tests.parity_util import TOL, snaps_err, state_err, y_err

pytestmark = pytest.mark.gpu


def _oracle(d, snap_every=0, epilogue=False):
    w, a, kk, kt = reference.prepare_inputs(d["w_logit"], d["a_logit"], d["k"], d["k_k"], d["k_a"])
    y, S, sn = native.forward(d["r"], w, kt, d["v"], kk, a, d.get("S0"), snap_every=snap_every)
    if epilogue:
        y = native.epilogue(y, d["r"], kt, d["v"], d["ln_w"], d["ln_b"], d["r_k"])
    return y, S, sn


def _gpu(d, device, **kw):
    dd = {k: (None if v is None else v.to(device)) for k, v in d.items()}
    return wkv7.forward_raw(dd["r"], dd["w_logit"], dd["k"], dd["v"], dd["a_logit"], dd["k_k"], dd["k_a"],
                            dd.get("S0"), **kw), dd


@pytest.mark.parametrize("algo", ["seq", "chunk", "split"])
@pytest.mark.parametrize("T", [1, 37, 64, 65, 200, 449])
def test_raw_ragged_lengths(cuda_device, algo, T):
    """bf16 raw inputs with a carried-in state, lengths off every tile boundary."""
    d = inputs.make_raw_inputs(inputs.WORKLOADS[1], B=2, T=T, H=3, s0="normal", seed=3000 + T)
    y_ref, S_ref, _ = _oracle(d)
    (y, S, _), _ = _gpu(d, cuda_device, algo=algo)
    assert y_err(y, y_ref) <= TOL["bf16"]
    assert state_err(S, S_ref) <= TOL["bf16"]


@pytest.mark.parametrize("T", [1, 16, 17, 100])
def test_raw_fp32_scan(cuda_device, T):
    d = inputs.make_raw_inputs(inputs.WORKLOADS[1], B=2, T=T, H=2, s0="normal", dtype="f32", seed=3100 + T)
    y_ref, S_ref, _ = _oracle(d)
    (y, S, _), _ = _gpu(d, cuda_device, algo="seq")
    assert y_err(y, y_ref) <= TOL["f32"]
    assert state_err(S, S_ref) <= TOL["f32"]


@pytest.mark.parametrize("algo", ["auto", "seq"])
def test_raw_prefill_019b_full(cuda_device, algo):
    """0.19B-shaped prefill (B8 T1024 H12, bf16) from raw inputs; every head."""
    d = inputs.make_raw_inputs(inputs.WORKLOADS[1])
    y_ref, S_ref, _ = _oracle(d)
    (y, S, _), _ = _gpu(d, cuda_device, algo=algo)
    assert y_err(y, y_ref) <= TOL["bf16"]
    assert state_err(S, S_ref) <= TOL["bf16"]


@pytest.mark.parametrize("algo", ["seq", "chunk", "split"])
@pytest.mark.parametrize("with_k_a", [True, False])
def test_raw_epilogue_uses_updated_key(cuda_device, algo, with_k_a):
    """The bonus term reads k~ = k + k (a-1) k_a (k_a absent = 0: k~ = k)."""
    d = inputs.make_raw_inputs(inputs.WORKLOADS[2], B=2, T=300, H=4, seed=3200, k_a=with_k_a)
    if not with_k_a:
        d["k_a"] = None
    y_ref, _, _ = _oracle(d, epilogue=True)
    dd = {k: (None if v is None else v.to(cuda_device)) for k, v in d.items()}
    y, _, _ = wkv7.forward_raw(dd["r"], dd["w_logit"], dd["k"], dd["v"], dd["a_logit"], dd["k_k"], dd["k_a"],
                               dd.get("S0"), algo=algo, ln_w=dd["ln_w"], ln_b=dd["ln_b"], r_k=dd["r_k"])
    assert y_err(y, y_ref) <= TOL["bf16"]


@pytest.mark.parametrize("algo,snap_every", [("chunk", 64), ("seq", 50), ("seq", 64)])
def test_raw_snapshots(cuda_device, algo, snap_every):
    d = inputs.make_raw_inputs(inputs.WORKLOADS[1], B=1, T=256, H=3, s0="normal", seed=3300)
    y_ref, S_ref, sn_ref = _oracle(d, snap_every=snap_every)
    (y, S, sn), _ = _gpu(d, cuda_device, algo=algo, snap_every=snap_every)
    assert snaps_err(sn, sn_ref) <= TOL["bf16"]
    assert y_err(y, y_ref) <= TOL["bf16"]
    assert state_err(S, S_ref) <= TOL["bf16"]


@pytest.mark.parametrize("algo", ["seq", "chunk"])
def test_raw_zero_keys_stay_finite(cuda_device, algo):
    """A token whose key is zero has ||k * k_k|| = 0: the 1e-12 floor keeps kk = 0, the update
    reduces to the decay, and nothing turns non-finite."""
    d = inputs.make_raw_inputs(inputs.WORKLOADS[1], B=1, T=130, H=2, s0="normal", seed=3400)
    d["k"][:, 5:70] = 0
    y_ref, S_ref, _ = _oracle(d)
    (y, S, _), _ = _gpu(d, cuda_device, algo=algo)
    assert torch.isfinite(y).all() and torch.isfinite(S).all()
    assert y_err(y, y_ref) <= TOL["bf16"]
    assert state_err(S, S_ref) <= TOL["bf16"]
