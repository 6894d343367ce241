"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle on the
same seeded inputs, element by element, within the stated tolerances (max
relative error per (b, h) slice: 2e-3 for bf16 inputs, 1e-5 for fp32 inputs)."""
import numpy as np
import pytest
import torch

from linear_rnn_sequence_rwkv_b200 import inputs, wkv7
from oracle import native, reference
from tests.golden_util import elementary_transitions
from tests.parity_util import TOL, as_np, heads_slice, snaps_err, state_err, y_err

pytestmark = pytest.mark.gpu

ALGOS_ANY = ["seq", "chunk", "split"]   # algorithms that accept bf16 inputs (split: automatic CTAs per head)
CHUNKED = ("chunk", "split")


def _dev(d, device):
    return {k: (None if v is None else v.to(device)) for k, v in d.items()}


def _oracle(d, snap_every=0):
    return native.forward(d["r"], d["w"], d["k"], d["v"], d["kk"], d["a"], d.get("S0"), snap_every=snap_every)


def _gpu(dd, **kw):
    return wkv7.forward(dd["r"], dd["w"], dd["k"], dd["v"], dd["kk"], dd["a"], dd.get("S0"), **kw)


@pytest.mark.parametrize("algo", ["seq", "auto"])
def test_tiny_fp32_workload(cuda_device, algo):
    """Tiny oracle check (B1 T64 H2, fp32 in/out, S0 = 0): error <= 1e-5."""
    wl = inputs.WORKLOADS[0]
    d = inputs.make_inputs(wl)
    y_ref, S_ref, _ = _oracle(d)
    y, S, _ = _gpu(_dev(d, cuda_device), algo=algo)
    assert y_err(y, y_ref) <= TOL["f32"]
    assert state_err(S, S_ref) <= TOL["f32"]


@pytest.mark.parametrize("algo", ALGOS_ANY)
@pytest.mark.parametrize("T", [1, 2, 3, 17, 31, 33, 63, 65, 100, 257])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_ragged_lengths(cuda_device, algo, T, dtype):
    """Lengths that are not multiples of any tile, with a carried-in state."""
    if dtype == "f32" and algo in CHUNKED:
        pytest.skip("the chunked algorithms take bf16 inputs")
    wl = inputs.WORKLOADS[1]
    d = inputs.make_inputs(wl, B=2, T=T, H=3, dtype=dtype, seed=1000 + T)
    y_ref, S_ref, _ = _oracle(d)
    y, S, _ = _gpu(_dev(d, cuda_device), algo=algo)
    assert y_err(y, y_ref) <= TOL[dtype]
    assert state_err(S, S_ref) <= TOL[dtype]


@pytest.mark.parametrize("algo", ALGOS_ANY)
def test_prefill_019b_full(cuda_device, algo):
    """0.19B-shaped prefill at full size (B8 T1024 H12, bf16, S0 ~ N(0, 0.1^2)); every head."""
    wl = inputs.WORKLOADS[1]
    d = inputs.make_inputs(wl)
    y_ref, S_ref, _ = _oracle(d)
    y, S, _ = _gpu(_dev(d, cuda_device), algo=algo)
    assert y_err(y, y_ref) <= TOL["bf16"]
    assert state_err(S, S_ref) <= TOL["bf16"]


def test_golden_elementary_transitions(cuda_device):
    """Appendix-D.3 swap/copy/identity fixture through the fp32 path: states are
    column maps of S0 and each y_t reads one column."""
    g = elementary_transitions()
    to = lambda x: torch.as_tensor(x, dtype=torch.float32, device=cuda_device).contiguous()
    y, S, snaps = wkv7.forward(*(to(g[n]) for n in ("r", "w", "k", "v", "kk", "a")), to(g["S0"]),
                               snap_every=1)
    np.testing.assert_allclose(as_np(snaps)[0, :, 0], g["S_expected"], rtol=0, atol=1e-5 * 8)
    np.testing.assert_allclose(as_np(y)[0, :, 0], g["y_expected"], rtol=0, atol=1e-5 * 8)
    np.testing.assert_allclose(as_np(S)[0, 0], g["S_expected"][-1], rtol=0, atol=1e-5 * 8)


@pytest.mark.parametrize("algo", ALGOS_ANY)
@pytest.mark.parametrize("T1", [1, 37, 64, 100])
def test_state_handoff_split(cuda_device, algo, T1):
    """forward(T1) then forward(T - T1, S0 = S_mid) equals one pass (and the oracle)."""
    wl = inputs.WORKLOADS[1]
    d = _dev(inputs.make_inputs(wl, B=2, T=160, H=3, seed=77), cuda_device)
    y, S, _ = _gpu(d, algo=algo)
    first = {k: (v[:, :T1].contiguous() if k != "S0" else v) for k, v in d.items()}
    rest = {k: (v[:, T1:].contiguous() if k != "S0" else None) for k, v in d.items()}
    y1, S1, _ = _gpu(first, algo=algo)
    rest["S0"] = S1
    y2, S2, _ = _gpu(rest, algo=algo)
    y_ref, S_ref, _ = _oracle({k: v.cpu() if v is not None else None for k, v in d.items()})
    assert y_err(torch.cat([y1, y2], dim=1), y_ref) <= TOL["bf16"]
    assert state_err(S2, S_ref) <= TOL["bf16"]
    # the fp32 scan is reproducible to rounding; the chunked path moves its chunk
    # boundaries with the split, so the two runs differ at tf32 operand rounding
    self_tol = 1e-5 if algo == "seq" else TOL["bf16"]
    assert y_err(torch.cat([y1, y2], dim=1), y) <= self_tol
    assert state_err(S2, S) <= self_tol


def test_in_place_state_handoff(cuda_device):
    """S_T may be the S0 buffer itself."""
    wl = inputs.WORKLOADS[1]
    d = _dev(inputs.make_inputs(wl, B=1, T=50, H=2, seed=5), cuda_device)
    y_ref, S_ref, _ = _oracle({k: v.cpu() if v is not None else None for k, v in d.items()})
    S = d["S0"].clone()
    y, S_out, _ = _gpu({**d, "S0": S}, S_T=S)
    assert S_out.data_ptr() == S.data_ptr()
    assert state_err(S, S_ref) <= TOL["bf16"]
    assert y_err(y, y_ref) <= TOL["bf16"]


def test_zero_length_copies_state(cuda_device):
    wl = inputs.WORKLOADS[1]
    d = _dev(inputs.make_inputs(wl, B=2, T=0, H=3, seed=6), cuda_device)
    _, S, _ = _gpu(d)
    assert torch.equal(S, d["S0"])
    d["S0"] = None
    _, S, _ = _gpu(d)
    assert torch.count_nonzero(S) == 0


@pytest.mark.parametrize("algo", ALGOS_ANY)
def test_snapshots(cuda_device, algo):
    wl = inputs.WORKLOADS[4]
    d = inputs.make_inputs(wl, B=1, T=512, H=3, seed=9)
    y_ref, S_ref, sn_ref = _oracle(d, snap_every=128)
    y, S, sn = _gpu(_dev(d, cuda_device), algo=algo, snap_every=128)
    assert sn.shape == (1, 4, 3, 64, 64)
    assert snaps_err(sn, sn_ref) <= TOL["bf16"]
    assert y_err(y, y_ref) <= TOL["bf16"]
    assert torch.equal(sn[:, -1], S)


@pytest.mark.parametrize("algo", ALGOS_ANY)
def test_epilogue(cuda_device, algo):
    """group_norm (eps 64e-5) + r.k.r_k bonus fused after the readout."""
    wl = inputs.WORKLOADS[2]
    d = inputs.make_inputs(wl, B=2, T=300, H=4, seed=10)
    y_ref, _, _ = _oracle(d)
    out_ref = native.epilogue(y_ref, d["r"], d["k"], d["v"], d["ln_w"], d["ln_b"], d["r_k"])
    dd = _dev(d, cuda_device)
    y, _, _ = _gpu(dd, algo=algo, ln_w=dd["ln_w"], ln_b=dd["ln_b"], r_k=dd["r_k"])
    assert y_err(y, out_ref) <= TOL["bf16"]


def test_decode_matches_forward_and_oracle(cuda_device):
    """T decode steps equal one forward pass over the same tokens (and the oracle)."""
    wl = inputs.WORKLOADS[3]
    T = 24
    d = inputs.make_inputs(wl, B=4, T=T, H=5, seed=11, s0="normal")
    y_ref, S_ref, _ = _oracle(d)
    dd = _dev(d, cuda_device)
    S = dd["S0"].clone()
    ys = []
    for t in range(T):
        step = [dd[n][:, t].contiguous() for n in ("r", "w", "k", "v", "kk", "a")]
        ys.append(wkv7.decode_step(*step, S).clone())
    y = torch.stack(ys, dim=1)
    assert y_err(y, y_ref) <= TOL["bf16"]
    assert state_err(S, S_ref) <= TOL["bf16"]
    yf, Sf, _ = _gpu(dd, algo="seq")
    assert y_err(y, yf) <= 1e-5 and state_err(S, Sf) <= 1e-5


def test_decode_fp32_inputs(cuda_device):
    wl = inputs.WORKLOADS[0]
    d = inputs.make_inputs(wl, B=3, T=5, H=2, seed=12, s0="normal")
    y_ref, S_ref, _ = _oracle(d)
    dd = _dev(d, cuda_device)
    S = dd["S0"].clone()
    ys = [wkv7.decode_step(*(dd[n][:, t].contiguous() for n in ("r", "w", "k", "v", "kk", "a")), S).clone()
          for t in range(5)]
    assert y_err(torch.stack(ys, 1), y_ref) <= TOL["f32"]
    assert state_err(S, S_ref) <= TOL["f32"]


def test_host_pointer_rejected_before_launch(cuda_device):
    d = _dev(inputs.make_inputs(inputs.WORKLOADS[1], B=1, T=8, H=1, seed=13), cuda_device)
    d["kk"] = d["kk"].cpu()
    with pytest.raises(wkv7.Wkv7Error) as e:
        wkv7.forward(d["r"], d["w"], d["k"], d["v"], d["kk"], d["a"], d["S0"])
    assert e.value.status == wkv7.ERR_ARG


def test_too_small_allocation_rejected(cuda_device):
    """An output buffer whose allocation ends before the stated size is rejected on
    the host (allocation range from the driver), so no kernel writes past it."""
    import ctypes
    from cuda.bindings import runtime as cudart
    d = _dev(inputs.make_inputs(inputs.WORKLOADS[1], B=1, T=8, H=1, seed=14), cuda_device)
    err, raw = cudart.cudaMalloc(1024)          # y needs 8 * 64 * 4 = 2048 bytes
    assert err == cudart.cudaError_t.cudaSuccess
    try:
        lib = wkv7.load()
        p = lambda t: ctypes.c_void_p(t.data_ptr())
        o = wkv7.make_opts()
        st = lib.wkv7_forward(1, 8, 1, 64, wkv7.BF16, *(p(d[n]) for n in ("r", "w", "k", "v", "kk", "a")),
                              p(d["S0"]), ctypes.c_void_p(int(raw)), None, ctypes.byref(o), None, 0, None)
        assert st == wkv7.ERR_ARG, lib.wkv7_last_error()
        assert b"allocation" in lib.wkv7_last_error()
    finally:
        cudart.cudaFree(raw)


@pytest.mark.slow
@pytest.mark.parametrize("algo", ALGOS_ANY)
def test_prefill_15b_sampled_heads(cuda_device, algo):
    """1.5B-shaped prefill (B16 T4096 H32, epilogue on) at full size on the GPU;
    8 sampled (b, h) heads recomputed by the oracle."""
    wl = inputs.WORKLOADS[2]
    d = inputs.make_inputs(wl, device="cuda")
    y, S, _ = _gpu(d, algo=algo, ln_w=d["ln_w"], ln_b=d["ln_b"], r_k=d["r_k"])
    pairs = [(0, 0), (3, 7), (5, 31), (8, 16), (11, 2), (12, 29), (15, 0), (15, 31)]
    hs = heads_slice({k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}, pairs)
    y_ref, S_ref, _ = native.forward(hs["r"], hs["w"], hs["k"], hs["v"], hs["kk"], hs["a"], hs["S0"])
    hsel = torch.tensor([h for _, h in pairs])
    ln = {n: d[n].cpu()[hsel][:, None, :] for n in ("ln_w", "ln_b", "r_k")}   # per-sample head params
    out_ref = np.empty_like(y_ref)
    for i in range(len(pairs)):
        out_ref[i:i + 1] = native.epilogue(y_ref[i:i + 1], hs["r"][i:i + 1], hs["k"][i:i + 1], hs["v"][i:i + 1],
                                           ln["ln_w"][i], ln["ln_b"][i], ln["r_k"][i])
    y_got = torch.stack([y[b, :, h] for b, h in pairs])[:, :, None, :]
    S_got = torch.stack([S[b, h] for b, h in pairs])[:, None]
    assert y_err(y_got, out_ref) <= TOL["bf16"]
    assert state_err(S_got, S_ref) <= TOL["bf16"]


@pytest.mark.slow
def test_decode_29b_full_steps_sampled(cuda_device):
    """2.9B-shaped decode (B256 H40, 128 steps, fp32 state in HBM); 6 heads checked."""
    wl = inputs.WORKLOADS[3]
    d = inputs.make_inputs(wl, device="cuda")
    B, T, H, N = d["r"].shape
    steps = {n: d[n].transpose(0, 1).contiguous() for n in ("r", "w", "k", "v", "kk", "a")}
    S = torch.zeros(B, H, N, N, device="cuda")
    ys = torch.empty(T, B, H, N, device="cuda")
    for t in range(T):
        wkv7.decode_step(*(steps[n][t] for n in ("r", "w", "k", "v", "kk", "a")), S, y=ys[t])
    pairs = [(0, 0), (17, 39), (100, 3), (200, 20), (255, 0), (255, 39)]
    hs = heads_slice({k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}, pairs)
    y_ref, S_ref, _ = native.forward(hs["r"], hs["w"], hs["k"], hs["v"], hs["kk"], hs["a"], None)
    y_got = torch.stack([ys[:, b, h] for b, h in pairs])[:, :, None, :]
    S_got = torch.stack([S[b, h] for b, h in pairs])[:, None]
    assert y_err(y_got, y_ref) <= TOL["bf16"]
    assert state_err(S_got, S_ref) <= TOL["bf16"]


@pytest.mark.slow
@pytest.mark.parametrize("algo", ALGOS_ANY)
def test_long_context_sampled_heads(cuda_device, algo):
    """Long context (B1 T65536 H40, z ~ N(2,1), snapshots every 4096); 4 heads checked
    over the whole sequence, plus all 16 snapshots of those heads."""
    wl = inputs.WORKLOADS[4]
    d = inputs.make_inputs(wl, device="cuda")
    y, S, sn = _gpu(d, algo=algo, snap_every=4096)
    pairs = [(0, 0), (0, 13), (0, 27), (0, 39)]
    hs = heads_slice({k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}, pairs)
    y_ref, S_ref, sn_ref = native.forward(hs["r"], hs["w"], hs["k"], hs["v"], hs["kk"], hs["a"], None,
                                          snap_every=4096)
    y_got = torch.stack([y[b, :, h] for b, h in pairs])[:, :, None, :]
    S_got = torch.stack([S[b, h] for b, h in pairs])[:, None]
    sn_got = torch.stack([sn[b, :, h] for b, h in pairs])[:, :, None]
    assert y_err(y_got, y_ref) <= TOL["bf16"]
    assert state_err(S_got, S_ref) <= TOL["bf16"]
    assert snaps_err(sn_got, sn_ref) <= TOL["bf16"]


@pytest.mark.parametrize("algo", ALGOS_ANY)
def test_more_heads_than_sms(cuda_device, algo):
    """200 (b, h) heads: the persistent chunked kernel walks several heads per CTA and
    prefetches the next head's first chunk."""
    wl = inputs.WORKLOADS[1]
    d = inputs.make_inputs(wl, B=4, T=200, H=50, seed=21)
    y_ref, S_ref, _ = _oracle(d)
    y, S, _ = _gpu(_dev(d, cuda_device), algo=algo)
    assert y_err(y, y_ref) <= TOL["bf16"]
    assert state_err(S, S_ref) <= TOL["bf16"]


@pytest.mark.parametrize("algo", ALGOS_ANY)
@pytest.mark.parametrize("case", ["linear_attention", "full_erase", "no_decay_a0", "slowest_decay"])
def test_degenerate_inputs(cuda_device, algo, case):
    """Edge cases of the method: w = 1 with a = 0 (linear attention), w = 1 with a = 1
    (delta-rule erasure), all-zero removal keys, and decay at the lower end of its range."""
    wl = inputs.WORKLOADS[1]
    d = inputs.make_inputs(wl, B=2, T=130, H=3, seed=22)
    one = torch.ones_like(d["w"])
    if case == "linear_attention":
        d["w"], d["a"] = one.clone(), torch.zeros_like(d["a"])
    elif case == "full_erase":
        d["w"], d["a"] = one.clone(), one.clone()
    elif case == "no_decay_a0":
        d["kk"] = torch.zeros_like(d["kk"])
    else:
        d["w"] = torch.full_like(d["w"], inputs.W_MIN).to(torch.float32).to(d["w"].dtype)
    y_ref, S_ref, _ = _oracle(d)
    y, S, _ = _gpu(_dev(d, cuda_device), algo=algo)
    assert y_err(y, y_ref) <= TOL["bf16"]
    assert state_err(S, S_ref) <= TOL["bf16"]


def test_chunk_rejects_unsupported_requests(cuda_device):
    d = _dev(inputs.make_inputs(inputs.WORKLOADS[0], B=1, T=70, H=1, seed=23), cuda_device)
    with pytest.raises(wkv7.Wkv7Error) as e:
        _gpu(d, algo="chunk")                       # fp32 inputs
    assert e.value.status == wkv7.ERR_UNSUPPORTED
    d = _dev(inputs.make_inputs(inputs.WORKLOADS[1], B=1, T=70, H=1, seed=23), cuda_device)
    with pytest.raises(wkv7.Wkv7Error) as e:
        _gpu(d, algo="chunk", snap_every=10)        # snapshot inside a chunk
    assert e.value.status == wkv7.ERR_UNSUPPORTED
    y, S, sn = _gpu(d, snap_every=10)               # auto falls back to the scan
    assert sn.shape[1] == 7


def test_no_device_error_after_runs(cuda_device):
    d = _dev(inputs.make_inputs(inputs.WORKLOADS[1], B=1, T=64, H=2, seed=24), cuda_device)
    _gpu(d, algo="chunk")
    wkv7.poll_device_error()


def test_handoff_wait_runs_out_and_reports_timeout(cuda_device):
    """Split mode with each head's first state hand-off withheld: the receiving CTA's bounded
    wait (2 ms here) runs out, the kernel records the error, drains what it issued and
    returns. wkv7_poll_device_error reports WKV7_ERR_TIMEOUT once and clears it; the context
    stays usable, and a normal forward afterwards matches the oracle."""
    d = inputs.make_inputs(inputs.WORKLOADS[1], B=1, T=256, H=2, seed=4242)
    dd = _dev(d, cuda_device)
    wkv7.poll_device_error()                       # nothing pending before
    _gpu(dd, algo="split", segments=2, handoff_wait_us=2000, withhold_handoff=1)
    with pytest.raises(wkv7.Wkv7Error) as e:
        wkv7.poll_device_error()
    assert e.value.status == wkv7.ERR_TIMEOUT
    wkv7.poll_device_error()                       # cleared by the poll
    y, S, _ = _gpu(dd, algo="split", segments=2)
    wkv7.poll_device_error()
    y_ref, S_ref, _ = _oracle(d)
    assert y_err(y, y_ref) <= TOL["bf16"]
    assert state_err(S, S_ref) <= TOL["bf16"]


@pytest.mark.parametrize("segments", [2, 3, 4, 7, 8])
@pytest.mark.parametrize("T", [130, 64 * 9 + 17, 1024])
def test_split_matches_oracle_and_single_cta(cuda_device, segments, T):
    """Chunks of one head spread over a cluster of `segments` CTAs, the state handed on
    through distributed shared memory: within tolerance of the oracle, and bit-identical
    to the one-CTA chunked path (same operations in the same order, only the CTA differs).
    Covers clusters wider than the chunk count (T = 130: three chunks), a ragged last
    chunk, snapshots and S_T written by different CTAs, and the fused epilogue."""
    wl = inputs.WORKLOADS[2]
    d = _dev(inputs.make_inputs(wl, B=2, T=T, H=3, seed=30 + segments), cuda_device)
    kw = dict(ln_w=d["ln_w"], ln_b=d["ln_b"], r_k=d["r_k"], snap_every=64)
    y1, S1, sn1 = _gpu(d, algo="chunk", **kw)
    ys, Ss, sns = _gpu(d, algo="split", segments=segments, **kw)
    assert torch.equal(ys, y1) and torch.equal(Ss, S1) and torch.equal(sns, sn1)
    dc = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    y_ref, S_ref, sn_ref = _oracle(dc, snap_every=64)
    out_ref = native.epilogue(y_ref, dc["r"], dc["k"], dc["v"], dc["ln_w"], dc["ln_b"], dc["r_k"])
    assert y_err(ys, out_ref) <= TOL["bf16"]
    assert state_err(Ss, S_ref) <= TOL["bf16"]
    assert snaps_err(sns, sn_ref) <= TOL["bf16"]
    wkv7.poll_device_error()


def test_split_many_heads_per_cluster(cuda_device):
    """More heads than clusters: each cluster walks several heads, CTA 0 reloads S0 for
    every head and the ring of hand-offs restarts at each head's first chunk."""
    d = _dev(inputs.make_inputs(inputs.WORKLOADS[1], B=8, T=64 * 5 + 3, H=40, seed=31), cuda_device)
    y1, S1, _ = _gpu(d, algo="chunk")
    for seg in (2, 3, 8):
        ys, Ss, _ = _gpu(d, algo="split", segments=seg)
        assert torch.equal(ys, y1) and torch.equal(Ss, S1), seg
    wkv7.poll_device_error()


def test_plan_matches_dispatch(cuda_device):
    """wkv7_plan reports the path wkv7_forward takes: forced sizes are echoed, automatic ones
    lie in 1..8, and the long-context shape (40 heads) is split across several CTAs."""
    assert wkv7.plan(1, 1024, 2, algo="chunk") == ("chunk", 1)
    assert wkv7.plan(1, 1024, 2, algo="split", segments=5) == ("chunk", 5)
    algo, seg = wkv7.plan(1, 65536, 40)
    assert algo == "chunk" and 2 <= seg <= 8
    algo, seg = wkv7.plan(8, 1024, 12)
    assert algo == "chunk" and 1 <= seg <= 8


def test_partial_wave_tail_launch(cuda_device):
    """320 heads of 6 chunks: two whole waves run with one CTA per head, the 24 heads left over
    run in a second launch with several CTAs per head. Bit-identical to one CTA per head, and
    the plan reports the second launch's CTAs per head."""
    d = _dev(inputs.make_inputs(inputs.WORKLOADS[1], B=8, T=64 * 5 + 3, H=40, seed=32), cuda_device)
    algo, seg = wkv7.plan(8, 64 * 5 + 3, 40)
    assert algo == "chunk" and seg >= 1
    y1, S1, _ = _gpu(d, algo="chunk")
    ya, Sa, _ = _gpu(d)
    assert torch.equal(ya, y1) and torch.equal(Sa, S1)
    wkv7.poll_device_error()


def test_plan_launch_counts_on_device(cuda_device):
    """One launch per forward call, except the partial-wave split (two)."""
    assert wkv7.plan(8, 1024, 12, launches=True)[2] == 1
    algo, seg, n = wkv7.plan(16, 4096, 32, launches=True)
    assert algo == "chunk" and n in (1, 2) and (n == 1 or seg > 1)


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("T", [1, 15, 33, 100, 257])
def test_chunk_option_with_epilogue(cuda_device, chunk, T):
    """The chunk-length option (16, 32, 64) under AUTO on ragged lengths, with the fused
    group_norm + bonus epilogue and a carried-in state, against the oracle recurrence and
    epilogue; the path AUTO picks is whichever the library dispatches the option to."""
    wl = inputs.WORKLOADS[2]
    d = inputs.make_inputs(wl, B=2, T=T, H=3, seed=1500 + 7 * T + chunk, s0="normal")
    y_ref, S_ref, _ = _oracle(d)
    y_ref = native.epilogue(y_ref, d["r"], d["k"], d["v"], d["ln_w"], d["ln_b"], d["r_k"])
    dd = _dev(d, cuda_device)
    y, S, _ = _gpu(dd, chunk=chunk, ln_w=dd["ln_w"], ln_b=dd["ln_b"], r_k=dd["r_k"])
    assert y_err(y, y_ref) <= TOL["bf16"]
    assert state_err(S, S_ref) <= TOL["bf16"]


@pytest.mark.parametrize("chunk", [16, 32])
def test_chunk_option_on_the_prefill_15b_shape_sampled(cuda_device, chunk):
    """The 1.5B prefill shape (B16 T4096 H32, epilogue) at chunk 16 and 32; the oracle runs
    on four sampled (b, h) pairs."""
    wl = inputs.WORKLOADS[2]
    d = inputs.make_inputs(wl)
    dd = _dev(d, cuda_device)
    y, S, _ = _gpu(dd, chunk=chunk, ln_w=dd["ln_w"], ln_b=dd["ln_b"], r_k=dd["r_k"])
    pairs = [(0, 0), (5, 31), (11, 17), (15, 3)]
    for b, h in pairs:
        sub = {n: d[n][b:b + 1, :, h:h + 1] for n in ("r", "w", "k", "v", "kk", "a")}
        sub["S0"] = None if d["S0"] is None else d["S0"][b:b + 1, h:h + 1]
        y_ref, S_ref, _ = _oracle(sub)
        y_ref = native.epilogue(y_ref, sub["r"], sub["k"], sub["v"], d["ln_w"][h:h + 1], d["ln_b"][h:h + 1],
                                d["r_k"][h:h + 1])
        assert y_err(y[b:b + 1, :, h:h + 1], y_ref) <= TOL["bf16"], (b, h)
        assert state_err(S[b:b + 1, h:h + 1], S_ref) <= TOL["bf16"], (b, h)


@pytest.mark.parametrize("B,H", [(4, 32), (4, 37), (8, 20)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_scan_launch_shapes_by_head_count(cuda_device, B, H, dtype):
    """The scan's launch by head count: 128 heads (two rows per thread, two CTAs per head), 148
    and 160 (four rows per thread, one CTA per head); ragged T, S0, snapshots and the epilogue."""
    wl = inputs.WORKLOADS[2]   # with the epilogue parameters
    T, snap = 45, 9
    d = inputs.make_inputs(wl, B=B, T=T, H=H, dtype=dtype, seed=1800 + B * H, s0="normal")
    y_ref, S_ref, sn_ref = _oracle(d, snap_every=snap)
    out_ref = native.epilogue(y_ref, d["r"], d["k"], d["v"], d["ln_w"], d["ln_b"], d["r_k"])
    dd = _dev(d, cuda_device)
    y, S, sn = _gpu(dd, algo="seq", snap_every=snap, ln_w=dd["ln_w"], ln_b=dd["ln_b"], r_k=dd["r_k"])
    assert y_err(y, out_ref) <= TOL[dtype]
    assert state_err(S, S_ref) <= TOL[dtype]
    assert snaps_err(sn, sn_ref) <= TOL[dtype]


@pytest.mark.parametrize("H", [32, 40])
def test_scan_raw_inputs_by_head_count(cuda_device, H):
    """Raw inputs on the scan at 128 and 160 heads (two and four rows per thread)."""
    d = inputs.make_raw_inputs(inputs.WORKLOADS[1], B=4, T=33, H=H, s0="normal", seed=1900 + H)
    w, a, kk, kt = reference.prepare_inputs(d["w_logit"], d["a_logit"], d["k"], d["k_k"], d["k_a"])
    y_ref, S_ref, _ = native.forward(d["r"], w, kt, d["v"], kk, a, d["S0"])
    dd = _dev(d, cuda_device)
    y, S, _ = wkv7.forward_raw(dd["r"], dd["w_logit"], dd["k"], dd["v"], dd["a_logit"], dd["k_k"], dd["k_a"],
                               dd["S0"], algo="seq")
    assert y_err(y, y_ref) <= TOL["bf16"]
    assert state_err(S, S_ref) <= TOL["bf16"]
