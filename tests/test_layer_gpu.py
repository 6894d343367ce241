"""GPU parity of the full time-mixing layer (this library's GEMMs with the token-shift mixes,
activations, biases, value residual and gate fused into them, and its recurrence) against the
oracle's fp64 layer.

Bounds (max relative error per (b, h) slice of the output, as everywhere):
* fp32 layer: 1e-4. The GEMMs accumulate in fp32 over at most C = 256 products (first-order
  relative error near C * 2^-24 = 1.5e-5 each), the fp32 recurrence stays within its 1e-5
  bound, and a few such steps lie in series.
* bf16 layer: 2.2e-2. Every intermediate stored in bf16 is a relative rounding of at most
  2^-9 = 1.95e-3. The readout y = S r sees, to first order and in the worst case, r's two
  roundings (mixed input, projection), v's two, k's two, the decay's three (mixed input,
  low-rank hidden value, logit) and then the gated readout's one: 10 * 1.95e-3 = 1.95e-2,
  plus the tf32 recurrence's 2e-3 bound. (g and y stay fp32; y * g is rounded once, as the
  output projection's bf16 operand.)
"""
import pytest
import torch

from linear_rnn_sequence_rwkv_b200 import inputs, wkv7
from oracle import reference
from tests.parity_util import slice_rel_err, state_err

pytestmark = pytest.mark.gpu

TOL_LAYER = {"f32": 1e-4, "bf16": 2.2e-2}
RANKS = {"d_w": 16, "d_a": 16, "d_v": 8, "d_g": 32}


def _out_err(got, ref, H):
    B, T, C = ref.shape
    return slice_rel_err(got.reshape(B, T, H, C // H), ref.reshape(B, T, H, C // H), (0, 2))


def _case(B, T, H, dtype, first, seed):
    d = inputs.make_layer(B, T, H, seed=seed, dtype=dtype, first_layer=first, ranks=RANKS)
    ref = reference.time_mixing_layer(d["x"], d, d["last_x"], d["v0"], d["S0"])
    return d, ref


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("first", [True, False])
@pytest.mark.parametrize("T", [1, 37, 130])
def test_layer_matches_oracle(cuda_device, dtype, first, T):
    H = 4
    d, (out_ref, v0_ref, last_ref, S_ref) = _case(2, T, H, dtype, first, seed=900 + T + 7 * first)
    dd = {k: (None if v is None else v.to(cuda_device)) for k, v in d.items()}
    S = dd["S0"].clone()
    out, v0_out, last_out, S = wkv7.layer_forward(dd["x"], dd, H, last_x=dd["last_x"], v0=dd["v0"], S=S)
    assert _out_err(out, out_ref, H) <= TOL_LAYER[dtype]
    assert state_err(S, S_ref) <= TOL_LAYER[dtype]
    assert torch.equal(last_out.cpu(), d["x"][:, -1])
    if first:
        v_err = _out_err(v0_out.float(), torch.as_tensor(v0_ref), H)
        assert v_err <= TOL_LAYER[dtype]
    else:
        assert v0_out is None


def test_layer_two_calls_carry_state_and_previous_token(cuda_device):
    """Two calls (the second fed the first's state and last token) equal the oracle's layer
    over the whole sequence."""
    H, T1 = 4, 40
    d, (out_ref, _, _, S_ref) = _case(2, 100, H, "f32", False, seed=950)
    dd = {k: (None if v is None else v.to(cuda_device)) for k, v in d.items()}
    S = dd["S0"].clone()
    o1, _, last1, S = wkv7.layer_forward(dd["x"][:, :T1].contiguous(), dd, H, last_x=dd["last_x"],
                                         v0=dd["v0"][:, :T1].contiguous(), S=S)
    o2, _, _, S = wkv7.layer_forward(dd["x"][:, T1:].contiguous(), dd, H, last_x=last1,
                                     v0=dd["v0"][:, T1:].contiguous(), S=S)
    assert _out_err(torch.cat([o1, o2], dim=1), out_ref, H) <= TOL_LAYER["f32"]
    assert state_err(S, S_ref) <= TOL_LAYER["f32"]


def test_layer_empty_sequence_passes_last_token(cuda_device):
    d = inputs.make_layer(2, 0, 2, seed=960, dtype="bf16", ranks=RANKS)
    dd = {k: (None if v is None else v.to(cuda_device)) for k, v in d.items()}
    _, _, last_out, _ = wkv7.layer_forward(dd["x"], dd, 2, last_x=dd["last_x"], v0=dd["v0"], S=dd["S0"])
    assert torch.equal(last_out, dd["last_x"])


def test_layer_head_size_128(cuda_device):
    """N = 128 heads (the recurrence on the scan) in the fp32 layer."""
    H, N = 2, 128
    d = inputs.make_layer(2, 33, H, N, seed=970, dtype="f32", ranks=RANKS)
    out_ref, _, _, S_ref = reference.time_mixing_layer(d["x"], d, d["last_x"], d["v0"], d["S0"])
    dd = {k: (None if v is None else v.to(cuda_device)) for k, v in d.items()}
    S = dd["S0"].clone()
    out, _, _, S = wkv7.layer_forward(dd["x"], dd, H, N=N, last_x=dd["last_x"], v0=dd["v0"], S=S)
    assert _out_err(out, out_ref, H) <= TOL_LAYER["f32"]
    assert state_err(S, S_ref) <= TOL_LAYER["f32"]


def test_layer_bench_shape_bf16(cuda_device):
    """The bench's layer: B8 T1024 H12 N64 (C = 768), bf16, default low-rank widths, a layer
    after the first; every output slice against the fp64 oracle layer."""
    d = inputs.make_layer(8, 1024, 12, seed=980, dtype="bf16")
    out_ref, _, _, S_ref = reference.time_mixing_layer(d["x"], d, d["last_x"], d["v0"], d["S0"])
    dd = {k: (None if v is None else v.to(cuda_device)) for k, v in d.items()}
    S = dd["S0"].clone()
    out, _, _, S = wkv7.layer_forward(dd["x"], dd, 12, last_x=dd["last_x"], v0=dd["v0"], S=S)
    assert _out_err(out, out_ref, 12) <= TOL_LAYER["bf16"]
    assert state_err(S, S_ref) <= TOL_LAYER["bf16"]


def test_layer_previous_token_in_place(cuda_device):
    """last_x_out may be last_x itself: the next call's previous token is updated in place."""
    d, (out_ref, _, last_ref, _) = _case(2, 20, 4, "f32", False, seed=990)
    dd = {k: (None if v is None else v.to(cuda_device)) for k, v in d.items()}
    last = dd["last_x"].clone()
    out, _, last_out, _ = wkv7.layer_forward(dd["x"], dd, 4, last_x=last, v0=dd["v0"], S=dd["S0"].clone(),
                                             last_x_out=last)
    assert last_out is last and torch.equal(last.cpu(), d["x"][:, -1])
    assert _out_err(out, out_ref, 4) <= TOL_LAYER["f32"]


def test_layer_at_the_large_shape_sampled(cuda_device):
    """B16 T4096 H32 (C 2048): the whole batch runs on the GPU; the first and the last sequence
    are checked against the oracle run on those two sequences alone (sequences are independent)."""
    H = 32
    d = inputs.make_layer(16, 4096, H, seed=971, dtype="bf16")
    rows = [0, 15]
    pick = {k: v for k, v in d.items()}
    for k in ("x", "last_x", "v0", "S0"):
        pick[k] = d[k][rows]
    out_ref, _, _, S_ref = reference.time_mixing_layer(pick["x"], pick, pick["last_x"], pick["v0"], pick["S0"])
    dd = {k: (None if v is None else v.to(cuda_device)) for k, v in d.items()}
    S = dd["S0"].clone()
    out, _, _, S = wkv7.layer_forward(dd["x"], dd, H, last_x=dd["last_x"], v0=dd["v0"], S=S)
    assert _out_err(out[rows], out_ref, H) <= TOL_LAYER["bf16"]
    assert state_err(S[rows], S_ref) <= TOL_LAYER["bf16"]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_layer_odd_widths(cuda_device, dtype):
    """C = 192 (three heads) and low-rank widths 70, 130, 1, 257 (padded to 128, 192, 64, 320):
    column tiles of 64 and 128 next to each other in one launch, second-factor K of 64 to 320,
    and 3 x 101 = 303 token rows (a partial last row block)."""
    H = 3
    ranks = {"d_w": 70, "d_a": 130, "d_v": 1, "d_g": 257}
    d = inputs.make_layer(3, 101, H, seed=990 + (dtype == "f32"), dtype=dtype, ranks=ranks)
    out_ref, _, _, S_ref = reference.time_mixing_layer(d["x"], d, d["last_x"], d["v0"], d["S0"])
    dd = {k: (None if v is None else v.to(cuda_device)) for k, v in d.items()}
    S = dd["S0"].clone()
    out, _, _, S = wkv7.layer_forward(dd["x"], dd, H, last_x=dd["last_x"], v0=dd["v0"], S=S)
    assert _out_err(out, out_ref, H) <= TOL_LAYER[dtype]
    assert state_err(S, S_ref) <= TOL_LAYER[dtype]
