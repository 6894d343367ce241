"""C-ABI checks that need no GPU: the library loads, exports every symbol that
include/wkv7.h declares, and rejects bad arguments on the host before any CUDA
call (these calls return before touching the device)."""
import ctypes
import os
import re

import pytest
import torch

from linear_rnn_sequence_rwkv_b200 import build, wkv7

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return wkv7.load()


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"WKV7_API\s+[\w\s\*]*?\b(wkv7_\w+)\s*\(", text))
    return names


def test_exports_every_declared_symbol(lib):
    declared = _declared_symbols()
    assert {"wkv7_forward", "wkv7_decode_step", "wkv7_workspace_bytes"} <= declared
    for name in declared:
        assert hasattr(lib, name), f"{name} declared in include/ but not exported"
    assert set(wkv7.EXPORTED) <= declared


def test_abi_version_and_strings(lib):
    assert lib.wkv7_abi_version() == 6
    assert lib.wkv7_status_string(0) == b"WKV7_OK"
    assert lib.wkv7_status_string(3) == b"WKV7_ERR_ALIGN"
    assert lib.wkv7_status_string(99) == b"WKV7_ERR_UNKNOWN"
    o = wkv7.Opts()
    lib.wkv7_opts_default(ctypes.byref(o))
    assert o.algo == 0 and o.chunk == 0 and o.snap_every == 0 and abs(o.gn_eps - 64e-5) < 1e-9
    assert o.handoff_wait_us == 0 and o.withhold_handoff == 0


FAKE = 0x10000   # 16-byte aligned, never dereferenced: validation fails first


def _fwd(lib, B=1, T=4, H=1, N=64, dt=1, ptrs=None, opts=None, ws=None, ws_bytes=0):
    p = ptrs or {}
    get = lambda n, d=FAKE: ctypes.c_void_p(p.get(n, d)) if p.get(n, d) is not None else None
    return lib.wkv7_forward(B, T, H, N, dt, *(get(n) for n in ("r", "w", "k", "v", "kk", "a")),
                            get("S0", None), get("y"), get("S_T", None),
                            ctypes.byref(opts) if opts else None, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(N=63), wkv7.ERR_UNSUPPORTED),
    (dict(N=96), wkv7.ERR_UNSUPPORTED),
    (dict(N=256), wkv7.ERR_UNSUPPORTED),
    (dict(N=0), wkv7.ERR_ARG),
    (dict(B=0), wkv7.ERR_ARG),
    (dict(H=-1), wkv7.ERR_ARG),
    (dict(T=-1), wkv7.ERR_ARG),
    (dict(dt=7), wkv7.ERR_ARG),
    (dict(ptrs={"kk": None}), wkv7.ERR_ARG),
    (dict(ptrs={"y": None}), wkv7.ERR_ARG),
    (dict(ptrs={"r": FAKE + 8}), wkv7.ERR_ALIGN),
    (dict(ptrs={"S0": FAKE + 4}), wkv7.ERR_ALIGN),
    (dict(B=1 << 30, T=1 << 30, H=1 << 30), wkv7.ERR_ARG),
])
def test_forward_rejects_bad_arguments(lib, kw, status):
    assert _fwd(lib, **kw) == status
    assert lib.wkv7_last_error() != b""


@pytest.mark.parametrize("field,value", [("algo", 9), ("chunk", 24), ("snap_every", -1), ("segments", -2),
                                         ("segments", 9)])
def test_forward_rejects_bad_options(lib, field, value):
    o = wkv7.Opts()
    lib.wkv7_opts_default(ctypes.byref(o))
    setattr(o, field, value)
    assert _fwd(lib, opts=o) == wkv7.ERR_ARG


@pytest.mark.parametrize("algo,segments,value", [(0, 0, 1), (2, 0, 1), (3, 1, 1), (3, 2, 2), (3, 2, -1)])
def test_withheld_handoff_only_in_split_mode(lib, algo, segments, value):
    """The failure-path switch is refused unless the chunks of a head are spread over at
    least two CTAs (the only place a hand-off happens)."""
    o = wkv7.Opts()
    lib.wkv7_opts_default(ctypes.byref(o))
    o.algo, o.segments, o.withhold_handoff = algo, segments, value
    assert _fwd(lib, opts=o) == wkv7.ERR_ARG
    assert b"withhold_handoff" in lib.wkv7_last_error()


def test_forward_rejects_partial_epilogue_and_missing_snapshots(lib):
    o = wkv7.Opts()
    lib.wkv7_opts_default(ctypes.byref(o))
    o.ln_w = FAKE
    assert _fwd(lib, opts=o) == wkv7.ERR_ARG
    lib.wkv7_opts_default(ctypes.byref(o))
    o.snap_every = 2
    assert _fwd(lib, opts=o) == wkv7.ERR_ARG


def test_forward_rejects_overlapping_outputs(lib):
    # y overlapping an input is caught on the host (pure address arithmetic)
    assert _fwd(lib, ptrs={"y": FAKE}) == wkv7.ERR_ARG
    assert b"overlap" in lib.wkv7_last_error()


def test_decode_rejects_bad_arguments(lib):
    P = lambda x: ctypes.c_void_p(x) if x is not None else None
    args = [P(FAKE + 0x1000 * i) for i in range(8)]
    assert lib.wkv7_decode_step(1, 1, 32, 1, *args, None) == wkv7.ERR_UNSUPPORTED
    assert lib.wkv7_decode_step(0, 1, 64, 1, *args, None) == wkv7.ERR_ARG
    bad = list(args)
    bad[3] = None
    assert lib.wkv7_decode_step(1, 1, 64, 1, *bad, None) == wkv7.ERR_ARG
    bad = list(args)
    bad[6] = P(FAKE + 0x6000 + 4)
    assert lib.wkv7_decode_step(1, 1, 64, 1, *bad, None) == wkv7.ERR_ALIGN


def test_workspace_query_is_host_only(lib):
    assert wkv7.workspace_bytes(2, 128, 4) >= 0


def test_plan_without_device(lib):
    """The dispatch query answers the scan cases on the host and reports a CUDA error, not a
    crash, when the chunked path would need the (absent) device."""
    import torch
    assert wkv7.plan(2, 8, 4) == ("seq", 0)                               # AUTO: < 16 tokens -> scan
    assert wkv7.plan(2, 128, 4, dtype=torch.float32) == ("seq", 0)        # fp32 inputs -> scan
    assert wkv7.plan(2, 0, 4) == ("seq", 0)                               # T = 0: state copy
    with pytest.raises(wkv7.Wkv7Error) as e:
        wkv7.plan(2, 128, 4, algo="split", segments=9)
    assert e.value.status == wkv7.ERR_ARG
    with pytest.raises(wkv7.Wkv7Error) as e:
        wkv7.plan(2, 128, 4, algo="chunk", dtype=torch.float32)
    assert e.value.status == wkv7.ERR_UNSUPPORTED
    if not torch.cuda.is_available():
        with pytest.raises(wkv7.Wkv7Error) as e:
            wkv7.plan(2, 128, 4)
        assert e.value.status == wkv7.ERR_CUDA


def test_plan_with_snapshot_interval_needs_no_buffer(lib):
    """The dispatch query takes snap_every without a snapshots buffer (it runs nothing)."""
    import torch
    assert wkv7.plan(1, 8, 2, snap_every=4) == ("seq", 0)                 # off chunk boundaries -> scan
    with pytest.raises(wkv7.Wkv7Error) as e:
        wkv7.plan(1, 128, 2, algo="chunk", snap_every=10)                  # chunked path cannot take it
    assert e.value.status == wkv7.ERR_UNSUPPORTED
    if not torch.cuda.is_available():
        with pytest.raises(wkv7.Wkv7Error) as e:
            wkv7.plan(1, 8192, 2, snap_every=4096)                         # chunked: needs the device
        assert e.value.status == wkv7.ERR_CUDA


def test_plan_counts_launches(lib):
    """The launch count the bench reports: the scan is one launch, plus one for the stand-alone
    epilogue; T = 0 is the state copy."""
    import torch
    assert wkv7.plan(2, 8, 4, launches=True) == ("seq", 0, 1)
    ln = torch.zeros(4, 64)
    assert wkv7.plan(2, 8, 4, launches=True, ln_w=ln, ln_b=ln, r_k=ln) == ("seq", 0, 2)
    assert wkv7.plan(2, 0, 4, launches=True) == ("seq", 0, 1)


def _fwd_raw(lib, ptrs=None, B=1, T=4, H=1, N=64, dt=1):
    p = ptrs or {}
    get = lambda n, d=FAKE: ctypes.c_void_p(p.get(n, d)) if p.get(n, d) is not None else None
    return lib.wkv7_forward_raw(B, T, H, N, dt, *(get(n) for n in ("r", "w_logit", "k", "v", "a_logit", "k_k")),
                                get("k_a", None), get("S0", None), get("y", FAKE + 0x100000), get("S_T", None),
                                None, None, 0, None)


@pytest.mark.parametrize("ptrs,status,word", [
    ({"k_k": None}, wkv7.ERR_ARG, b"k_k"),
    ({"a_logit": None}, wkv7.ERR_ARG, b"a_logit"),
    ({"w_logit": None}, wkv7.ERR_ARG, b"w_logit"),
    ({"k_a": FAKE + 0x200004}, wkv7.ERR_ALIGN, b"k_a"),
    ({"k_k": FAKE + 0x200008}, wkv7.ERR_ALIGN, b"k_k"),
])
def test_forward_raw_rejects_bad_arguments(lib, ptrs, status, word):
    assert _fwd_raw(lib, ptrs) == status
    assert word in lib.wkv7_last_error()


def test_forward_raw_shares_the_size_checks(lib):
    assert _fwd_raw(lib, N=32) == wkv7.ERR_UNSUPPORTED
    assert _fwd_raw(lib, B=0) == wkv7.ERR_ARG
    assert _fwd_raw(lib, {"y": FAKE}) == wkv7.ERR_ARG   # y overlapping r


def _bwd(lib, ptrs=None, B=1, T=4, H=1, N=64, dt=1, snap_every=0, ws=None, ws_bytes=0):
    p = ptrs or {}
    names_in = ("r", "w", "k", "v", "kk", "a")
    names_out = ("dr", "dw", "dk", "dv", "dkk", "da")
    base = {n: FAKE + 0x100000 * (i + 1) for i, n in enumerate(names_in + ("dy",) + names_out)}
    get = lambda n: (ctypes.c_void_p(p.get(n, base.get(n))) if p.get(n, base.get(n)) is not None else None)
    return lib.wkv7_backward(B, T, H, N, dt, *(get(n) for n in names_in), get("S0"), get("snapshots"),
                             snap_every, get("dy"), get("dS_T"), *(get(n) for n in names_out), get("dS0"),
                             ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status,word", [
    (dict(N=32), wkv7.ERR_UNSUPPORTED, b"N=32"),
    (dict(T=-1), wkv7.ERR_ARG, b"bad sizes"),
    (dict(dt=5), wkv7.ERR_ARG, b"dtype"),
    (dict(snap_every=-1), wkv7.ERR_ARG, b"snap_every"),
    (dict(snap_every=2), wkv7.ERR_ARG, b"snapshots"),
    (dict(ptrs={"dy": None}), wkv7.ERR_ARG, b"dy"),
    (dict(ptrs={"dkk": None}), wkv7.ERR_ARG, b"dkk"),
    (dict(ptrs={"kk": None}), wkv7.ERR_ARG, b"kk"),
    (dict(ptrs={"dr": FAKE + 0x100000 * 8 + 4}), wkv7.ERR_ALIGN, b"dr"),
    (dict(ptrs={"dS0": FAKE + 0x40000004}), wkv7.ERR_ALIGN, b"dS0"),
])
def test_backward_rejects_bad_arguments(lib, kw, status, word):
    assert _bwd(lib, **kw) == status
    assert word in lib.wkv7_last_error()


def test_backward_rejects_overlaps_and_small_workspace(lib):
    need = wkv7.backward_workspace_bytes(1, 4, 1)
    ws = ctypes.c_void_p(FAKE + 0x10000000)
    assert _bwd(lib, {"dw": FAKE + 0x100000 * 8}, ws=ws, ws_bytes=need) == wkv7.ERR_ARG   # dw on top of dr
    assert b"overlaps" in lib.wkv7_last_error()
    assert _bwd(lib, {"dr": FAKE + 0x100000}, ws=ws, ws_bytes=need) == wkv7.ERR_ARG       # dr on top of r
    assert _bwd(lib, ws=ctypes.c_void_p(FAKE + 0x100000 * 9), ws_bytes=need) == wkv7.ERR_ARG   # ws on dw
    assert need == 64 * 64 * 4                                              # one checkpoint per 4 tokens
    assert _bwd(lib, ws=ctypes.c_void_p(FAKE + 0x10000000), ws_bytes=need - 16) == wkv7.ERR_WORKSPACE
    assert _bwd(lib, ws=None, ws_bytes=0) == wkv7.ERR_WORKSPACE


def test_backward_workspace_query():
    assert wkv7.backward_workspace_bytes(2, 0, 3) == 0
    assert wkv7.backward_workspace_bytes(2, 10, 3) == 2 * 3 * 3 * 16384           # ceil(10 / 4) states
    assert wkv7.backward_workspace_bytes(2, 100, 3, snap_every=16) == 2 * 3 * 4 * 16384
    assert wkv7.backward_workspace_bytes(2, 100, 3, snap_every=200) == 2 * 3 * 25 * 16384
    assert wkv7.backward_workspace_bytes(2, 100, 3, N=32) == 0


def test_head_size_128_runs_on_the_scan():
    """N = 128: AUTO plans the scan and the chunked algorithms refuse it; the backward takes it
    (checkpoints every 2 tokens: B * H * ceil(K / 2) * N * N * 4 bytes)."""
    assert wkv7.plan(2, 300, 4, 128, torch.bfloat16) == ("seq", 0)
    assert wkv7.plan(2, 300, 4, 128, torch.float32, algo="seq") == ("seq", 0)
    with pytest.raises(wkv7.Wkv7Error) as e:
        wkv7.plan(2, 300, 4, 128, torch.bfloat16, algo="chunk")
    assert e.value.status == wkv7.ERR_UNSUPPORTED
    assert wkv7.backward_workspace_bytes(2, 300, 4, N=128) == 2 * 4 * 150 * 128 * 128 * 4
    assert wkv7.backward_workspace_bytes(2, 300, 4, N=128, snap_every=64) == 2 * 4 * 32 * 128 * 128 * 4
    assert wkv7.backward_workspace_bytes(2, 300, 4, N=96) == 0


def _layer_call(lib, B=1, T=4, H=1, N=64, dt=1, drop=None, over=None, ws=None, ws_bytes=0, v0=None):
    dims = wkv7.LayerDims(H, N, 8, 8, 8, 8)
    vals = {n: FAKE + 0x100000 * (i + 1) for i, n in enumerate(wkv7.LAYER_PARAMS)}
    vals.update(over or {})
    if drop:
        vals[drop] = None
    lp = wkv7.LayerParams(*(vals[n] for n in wkv7.LAYER_PARAMS))
    P = lambda a: None if a is None else ctypes.c_void_p(a)
    base = FAKE + 0x10000000
    return lib.wkv7_layer_forward(B, T, dt, ctypes.byref(dims), ctypes.byref(lp), P(base), None, P(v0), None,
                                  P(base + 0x1000000), None, None, None, ws, ws_bytes, None)


def test_layer_rejects_bad_arguments(lib):
    assert _layer_call(lib, N=96) == wkv7.ERR_UNSUPPORTED
    assert _layer_call(lib, drop="Wr") == wkv7.ERR_ARG and b"Wr" in lib.wkv7_last_error()
    assert _layer_call(lib, drop="ln_b") == wkv7.ERR_ARG
    assert _layer_call(lib, over={"Wg2": FAKE + 0x100000 * 30 + 8}) == wkv7.ERR_ALIGN
    assert _layer_call(lib, v0=FAKE + 0x20000000, drop="Wv1") == wkv7.ERR_ARG   # a later layer needs Wv1
    assert _layer_call(lib) == wkv7.ERR_WORKSPACE
    dims = wkv7.LayerDims(2, 64, 8, 8, 8, 8)
    assert lib.wkv7_layer_workspace_bytes(2, 0, 1, ctypes.byref(dims)) == 0
    # B2 T10, C = 128 channels, bf16, low-rank widths 8 (padded to 64): r, k, v and the two logits
    # (bf16), four hidden values (bf16, 64 wide), g and y (fp32), and the transposed factors
    up = lambda n: (n + 255) // 256 * 256
    M, C = 20, 128
    want = 5 * up(M * C * 2) + 4 * up(M * 64 * 2) + 2 * up(M * C * 4) + 8 * up(64 * C * 2)
    assert lib.wkv7_layer_workspace_bytes(2, 10, 1, ctypes.byref(dims)) == want


def _epi(lib, B=1, T=4, H=1, N=64, dt=1, eps=64e-5, ptrs=None):
    p = ptrs or {}
    get = lambda n: ctypes.c_void_p(p.get(n, FAKE)) if p.get(n, FAKE) is not None else None
    return lib.wkv7_epilogue(B, T, H, N, dt, *(get(n) for n in ("y", "r", "k", "v", "ln_w", "ln_b", "r_k")),
                             ctypes.c_float(eps), get("out"), None)


def _epi_bwd(lib, B=1, T=4, H=1, N=64, dt=1, ptrs=None, ws=None, ws_bytes=0):
    p = ptrs or {}
    names = ("y", "r", "k", "v", "ln_w", "ln_b", "r_k")
    outs = ("dy", "dr", "dk", "dv", "dln_w", "dln_b", "dr_k")
    # distinct fake addresses far apart, so that only the overlaps a test asks for exist
    base = {n: FAKE + (i + 1) * (1 << 24) for i, n in enumerate(names + ("dout",) + outs)}
    get = lambda n: ctypes.c_void_p(p.get(n, base[n]))
    return lib.wkv7_epilogue_backward(B, T, H, N, dt, *(get(n) for n in names), ctypes.c_float(64e-5), get("dout"),
                                      *(get(n) for n in outs), ws, ws_bytes, None)


def test_epilogue_entries_validate_before_touching_memory(lib):
    assert _epi(lib, N=32) == wkv7.ERR_UNSUPPORTED
    assert _epi(lib, eps=0.0) == wkv7.ERR_ARG
    assert _epi(lib, eps=float("nan")) == wkv7.ERR_ARG
    assert _epi(lib, dt=7) == wkv7.ERR_ARG
    assert _epi(lib, ptrs={"y": FAKE + 4}) == wkv7.ERR_ALIGN
    assert _epi(lib, ptrs={"r": None}) == wkv7.ERR_ARG
    assert _epi(lib, T=0, ptrs={n: None for n in ("y", "r", "k", "v", "ln_w", "ln_b", "r_k", "out")}) == wkv7.OK
    assert _epi_bwd(lib, N=96) == wkv7.ERR_UNSUPPORTED
    assert _epi_bwd(lib) == wkv7.ERR_WORKSPACE                      # one partial block needed, none given
    need = lib.wkv7_epilogue_backward_workspace_bytes(1, 4, 1, 64)
    ws = ctypes.c_void_p(FAKE + (1 << 30))
    assert _epi_bwd(lib, ptrs={"dr": FAKE + 8 * (1 << 24)}, ws=ws, ws_bytes=need) == wkv7.ERR_ARG   # dr on dout


def test_epilogue_backward_workspace_formula(lib):
    """One partial sum of the three parameter gradients (fp32, [3][N]) per head and per block of
    64 (b, t) rows."""
    assert lib.wkv7_epilogue_backward_workspace_bytes(2, 100, 3, 64) == 4 * 3 * 3 * 64 * 4
    assert lib.wkv7_epilogue_backward_workspace_bytes(1, 64, 2, 128) == 1 * 2 * 3 * 128 * 4
    assert lib.wkv7_epilogue_backward_workspace_bytes(1, 0, 2, 64) == 0
    assert lib.wkv7_epilogue_backward_workspace_bytes(1, 4, 2, 32) == 0


def _dec(lib, raw=False, N=64, eps=64e-5, ptrs=None, B=1, H=1):
    """A decode entry with distinct fake addresses far apart (host checks only)."""
    p = ptrs or {}
    ins = ("r", "w", "k", "v", "kk", "a") if not raw else ("r", "w_logit", "k", "v", "a_logit", "k_k", "k_a")
    names = ins + ("S", "y", "ln_w", "ln_b", "r_k")
    base = {n: FAKE + (i + 1) * (1 << 24) for i, n in enumerate(names)}
    get = lambda n: (lambda x: None if x is None else ctypes.c_void_p(x))(p.get(n, base[n]))
    if raw:
        return lib.wkv7_decode_step_raw(B, H, N, 1, *(get(n) for n in names), ctypes.c_float(eps), None)
    return lib.wkv7_decode_step_ex(B, H, N, 1, *(get(n) for n in names), ctypes.c_float(eps), None)


@pytest.mark.parametrize("raw", [False, True])
def test_decode_options_validate_before_touching_memory(lib, raw):
    assert _dec(lib, raw, N=32) == wkv7.ERR_UNSUPPORTED
    assert _dec(lib, raw, B=0) == wkv7.ERR_ARG
    assert _dec(lib, raw, ptrs={"ln_b": None}) == wkv7.ERR_ARG            # partial epilogue
    assert _dec(lib, raw, eps=0.0) == wkv7.ERR_ARG
    assert _dec(lib, raw, eps=float("inf")) == wkv7.ERR_ARG
    assert _dec(lib, raw, ptrs={"ln_w": FAKE + (1 << 30) + 4}) == wkv7.ERR_ALIGN
    s_base = FAKE + (8 if raw else 7) * (1 << 24)                            # where _dec puts S
    assert _dec(lib, raw, ptrs={"y": s_base + 256}) == wkv7.ERR_ARG          # y inside S
    assert b"overlaps" in lib.wkv7_last_error()
    if raw:
        assert _dec(lib, raw, ptrs={"k_k": None}) == wkv7.ERR_ARG
        assert b"k_k" in lib.wkv7_last_error()


def test_head_count_bound(lib):
    """B * H heads index the grids of the scan and the backward: more than INT_MAX is refused."""
    assert _fwd(lib, B=1 << 16, H=1 << 15, T=1) == wkv7.ERR_ARG
    assert b"heads" in lib.wkv7_last_error()
