"""Python binding of the WKV-7 C ABI (include/wkv7.h), loaded with ctypes.

Argument marshalling only: torch tensors supply device memory and the current
CUDA stream; every step of the computation runs in the library's CUDA kernels.
There is no CPU fallback: without the built library or a CUDA device these
functions raise.

Host (CPU) tensors are accepted by ``forward`` for callers that keep their data
on the host: the inputs are copied to the device, the kernels run, and the
outputs are copied back (the end-to-end path).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libwkv7.so")
HEAD_SIZE = 64
ABI_VERSION = 6          # WKV7_ABI_VERSION of include/wkv7.h this binding follows

# wkv7_status
OK, ERR_ARG, ERR_UNSUPPORTED, ERR_ALIGN, ERR_CUDA, ERR_TIMEOUT, ERR_WORKSPACE = range(7)
# wkv7_dtype
F32, BF16 = 0, 1
# wkv7_algo
ALGOS = {"auto": 0, "seq": 1, "chunk": 2, "split": 3}

EXPORTED = ("wkv7_opts_default", "wkv7_forward", "wkv7_decode_step", "wkv7_workspace_bytes",
            "wkv7_status_string", "wkv7_last_error", "wkv7_abi_version", "wkv7_poll_device_error",
            "wkv7_plan", "wkv7_forward_raw", "wkv7_backward", "wkv7_backward_workspace_bytes",
            "wkv7_backward_static", "wkv7_layer_forward", "wkv7_layer_workspace_bytes", "wkv7_probe_fp32_fma",
            "wkv7_probe_tf32_mma", "wkv7_forward_host", "wkv7_forward_host_workspace_bytes", "wkv7_epilogue",
            "wkv7_epilogue_backward", "wkv7_epilogue_backward_workspace_bytes", "wkv7_decode_step_ex",
            "wkv7_decode_step_raw")


class Wkv7Error(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: status {status} ({detail})")
        self.status = status


class LayerDims(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("N", ctypes.c_int), ("d_w", ctypes.c_int), ("d_a", ctypes.c_int),
                ("d_v", ctypes.c_int), ("d_g", ctypes.c_int)]


LAYER_PARAMS = ("mr", "mw", "mk", "mv", "ma", "mg", "w_bias", "a_bias", "v_bias", "r_k", "k_k", "k_a", "ln_w",
                "ln_b", "Wr", "Wk", "Wv", "Wo", "Ww1", "Ww2", "Wa1", "Wa2", "Wv1", "Wv2", "Wg1", "Wg2")


class LayerParams(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in LAYER_PARAMS]


class Opts(ctypes.Structure):
    _fields_ = [("algo", ctypes.c_int), ("chunk", ctypes.c_int), ("snap_every", ctypes.c_int),
                ("snapshots", ctypes.c_void_p), ("ln_w", ctypes.c_void_p), ("ln_b", ctypes.c_void_p),
                ("r_k", ctypes.c_void_p), ("gn_eps", ctypes.c_float), ("segments", ctypes.c_int),
                ("handoff_wait_us", ctypes.c_uint), ("withhold_handoff", ctypes.c_int)]


_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load libwkv7.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m linear_rnn_sequence_rwkv_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        vp, ci = ctypes.c_void_p, ctypes.c_int
        lib.wkv7_opts_default.argtypes = [ctypes.POINTER(Opts)]
        lib.wkv7_opts_default.restype = None
        lib.wkv7_forward.argtypes = [ci, ci, ci, ci, ci] + [vp] * 6 + [vp, vp, vp, ctypes.POINTER(Opts),
                                                                       vp, ctypes.c_size_t, vp]
        lib.wkv7_forward.restype = ci
        lib.wkv7_decode_step.argtypes = [ci, ci, ci, ci] + [vp] * 6 + [vp, vp, vp]
        lib.wkv7_decode_step.restype = ci
        lib.wkv7_decode_step_ex.argtypes = [ci, ci, ci, ci] + [vp] * 6 + [vp, vp] + [vp] * 3 + [ctypes.c_float, vp]
        lib.wkv7_decode_step_ex.restype = ci
        lib.wkv7_decode_step_raw.argtypes = [ci, ci, ci, ci] + [vp] * 5 + [vp, vp] + [vp, vp] + [vp] * 3 + [
            ctypes.c_float, vp]
        lib.wkv7_decode_step_raw.restype = ci
        lib.wkv7_backward.argtypes = [ci, ci, ci, ci, ci] + [vp] * 6 + [vp, vp, ci, vp, vp] + [vp] * 7 + [
            vp, ctypes.c_size_t, vp]
        lib.wkv7_backward.restype = ci
        lib.wkv7_backward_static.argtypes = [ci, ci, ci, ci, ci] + [vp] * 6 + [vp, vp, ci, vp, vp] + [vp] * 7 + [vp]
        lib.wkv7_backward_static.restype = ci
        lib.wkv7_epilogue.argtypes = [ci, ci, ci, ci, ci] + [vp] * 7 + [ctypes.c_float, vp, vp]
        lib.wkv7_epilogue.restype = ci
        lib.wkv7_epilogue_backward_workspace_bytes.argtypes = [ci, ci, ci, ci]
        lib.wkv7_epilogue_backward_workspace_bytes.restype = ctypes.c_size_t
        lib.wkv7_epilogue_backward.argtypes = [ci, ci, ci, ci, ci] + [vp] * 7 + [ctypes.c_float] + [vp] * 8 + [
            vp, ctypes.c_size_t, vp]
        lib.wkv7_epilogue_backward.restype = ci
        lib.wkv7_layer_forward.argtypes = [ci, ci, ci, ctypes.POINTER(LayerDims), ctypes.POINTER(LayerParams)] + [
            vp] * 7 + [ctypes.POINTER(Opts), vp, ctypes.c_size_t, vp]
        lib.wkv7_layer_forward.restype = ci
        lib.wkv7_layer_workspace_bytes.argtypes = [ci, ci, ci, ctypes.POINTER(LayerDims)]
        lib.wkv7_layer_workspace_bytes.restype = ctypes.c_size_t
        lib.wkv7_backward_workspace_bytes.argtypes = [ci, ci, ci, ci, ci]
        lib.wkv7_backward_workspace_bytes.restype = ctypes.c_size_t
        lib.wkv7_workspace_bytes.argtypes = [ci, ci, ci, ci, ci, ctypes.POINTER(Opts)]
        lib.wkv7_workspace_bytes.restype = ctypes.c_size_t
        lib.wkv7_status_string.argtypes = [ci]
        lib.wkv7_status_string.restype = ctypes.c_char_p
        lib.wkv7_last_error.argtypes = []
        lib.wkv7_last_error.restype = ctypes.c_char_p
        lib.wkv7_abi_version.argtypes = []
        lib.wkv7_abi_version.restype = ci
        lib.wkv7_poll_device_error.argtypes = [vp]
        lib.wkv7_poll_device_error.restype = ci
        lib.wkv7_plan.argtypes = [ci, ci, ci, ci, ci, ctypes.POINTER(Opts), ctypes.POINTER(ci), ctypes.POINTER(ci),
                                  ctypes.POINTER(ci)]
        lib.wkv7_plan.restype = ci
        lib.wkv7_forward_raw.argtypes = [ci, ci, ci, ci, ci] + [vp] * 5 + [vp, vp] + [vp, vp, vp, ctypes.POINTER(Opts),
                                                                               vp, ctypes.c_size_t, vp]
        lib.wkv7_forward_raw.restype = ci
        lib.wkv7_forward_host.argtypes = lib.wkv7_forward.argtypes
        lib.wkv7_forward_host.restype = ci
        lib.wkv7_forward_host_workspace_bytes.argtypes = [ci, ci, ci, ci, ci, ctypes.POINTER(Opts)]
        lib.wkv7_forward_host_workspace_bytes.restype = ctypes.c_size_t
        lib.wkv7_probe_fp32_fma.argtypes = [ci, ci, vp, ctypes.POINTER(ctypes.c_double)]
        lib.wkv7_probe_fp32_fma.restype = ci
        lib.wkv7_probe_tf32_mma.argtypes = [ci, ci, vp, ctypes.POINTER(ctypes.c_double)]
        lib.wkv7_probe_tf32_mma.restype = ci
        if lib.wkv7_abi_version() != ABI_VERSION:
            raise RuntimeError(f"{_LIB_PATH} has ABI version {lib.wkv7_abi_version()}, the binding expects "
                               f"{ABI_VERSION}: rebuild it")
        _lib = lib
        return lib


def _check(status: int, where: str):
    if status != OK:
        lib = load()
        detail = lib.wkv7_last_error().decode() or lib.wkv7_status_string(status).decode()
        raise Wkv7Error(status, where, detail)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}: use bfloat16 or float32")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(device, stream):
    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_opts(algo="auto", chunk=0, snap_every=0, snapshots=None, ln_w=None, ln_b=None, r_k=None,
              gn_eps=64e-5, segments=0, handoff_wait_us=0, withhold_handoff=0) -> Opts:
    o = Opts()
    load().wkv7_opts_default(ctypes.byref(o))
    o.algo = ALGOS[algo] if isinstance(algo, str) else int(algo)
    o.chunk = int(chunk)
    o.snap_every = int(snap_every)
    o.snapshots = None if snapshots is None else snapshots.data_ptr()
    o.ln_w = None if ln_w is None else ln_w.data_ptr()
    o.ln_b = None if ln_b is None else ln_b.data_ptr()
    o.r_k = None if r_k is None else r_k.data_ptr()
    o.gn_eps = float(gn_eps)
    o.segments = int(segments)
    o.handoff_wait_us = int(handoff_wait_us)
    o.withhold_handoff = int(withhold_handoff)
    return o


def plan(B, T, H, N=HEAD_SIZE, dtype=torch.bfloat16, launches=False, **opt_kw):
    """(algorithm, CTAs per head) wkv7_forward would use on the current device: ("seq", 0) or
    ("chunk", n) with n = 1 for one CTA per head and n > 1 for a cluster split; with
    launches=True also the number of kernel launches of the call."""
    algo, seg, n = ctypes.c_int(0), ctypes.c_int(0), ctypes.c_int(0)
    st = load().wkv7_plan(B, T, H, N, BF16 if dtype == torch.bfloat16 else F32, ctypes.byref(make_opts(**opt_kw)),
                          ctypes.byref(algo), ctypes.byref(seg), ctypes.byref(n))
    _check(st, "wkv7_plan")
    out = ("seq" if algo.value == ALGOS["seq"] else "chunk"), int(seg.value)
    return out + (int(n.value),) if launches else out


def workspace_bytes(B, T, H, N=HEAD_SIZE, dtype=torch.bfloat16, **opt_kw) -> int:
    return int(load().wkv7_workspace_bytes(B, T, H, N, BF16 if dtype == torch.bfloat16 else F32,
                                           ctypes.byref(make_opts(**opt_kw))))


def forward(r, w, k, v, kk, a, S0=None, *, algo="auto", chunk=0, snap_every=0, ln_w=None, ln_b=None,
            r_k=None, gn_eps=64e-5, segments=0, y=None, S_T=None, snapshots=None, workspace=None,
            return_state=True, stream=None, out_host=None, handoff_wait_us=0, withhold_handoff=0):
    """WKV-7 forward over [B, T, H, 64] inputs (bf16 or fp32, all the same dtype).

    Returns (y, S_T, snapshots): y [B, T, H, 64] fp32, S_T [B, H, 64, 64] fp32
    (None if return_state is False), snapshots [B, T//snap_every, H, 64, 64] or None.
    Output tensors may be passed in (y=, S_T=, snapshots=) to avoid allocation; S_T
    may be S0 for an in-place hand-off. CPU inputs run the end-to-end path (pinned
    host tensors make its copies asynchronous; ``out_host=(y_host, S_host)`` names
    pinned destinations for the results).
    """
    if r.device.type == "cpu":
        return _forward_host(r, w, k, v, kk, a, S0, algo=algo, chunk=chunk, snap_every=snap_every,
                             ln_w=ln_w, ln_b=ln_b, r_k=r_k, gn_eps=gn_eps, segments=segments,
                             return_state=return_state, out_host=out_host)
    lib = load()
    B, T, H, N = r.shape
    dev = r.device
    if y is None:
        y = torch.empty((B, T, H, N), device=dev, dtype=torch.float32)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, N, N), device=dev, dtype=torch.float32)
    n_snap = T // snap_every if snap_every else 0
    if snapshots is None and n_snap:
        snapshots = torch.empty((B, n_snap, H, N, N), device=dev, dtype=torch.float32)
    opts = make_opts(algo, chunk, snap_every, snapshots, ln_w, ln_b, r_k, gn_eps, segments, handoff_wait_us,
                     withhold_handoff)
    need = int(lib.wkv7_workspace_bytes(B, T, H, N, _dt(r), ctypes.byref(opts)))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = lib.wkv7_forward(B, T, H, N, _dt(r), _ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(kk), _ptr(a),
                              _ptr(S0), _ptr(y), _ptr(S_T), ctypes.byref(opts), _ptr(workspace),
                              ws_bytes, _stream_handle(dev, stream))
    _check(st, "wkv7_forward")
    return y, S_T, snapshots


def forward_raw(r, w_logit, k, v, a_logit, k_k, k_a=None, S0=None, *, algo="auto", chunk=0, snap_every=0,
                ln_w=None, ln_b=None, r_k=None, gn_eps=64e-5, segments=0, y=None, S_T=None, snapshots=None,
                workspace=None, return_state=True, stream=None):
    """WKV-7 forward from the raw time-mixing values (decay and rate logits, the key before its
    update, the per-head k_k and k_a): the pre-processing runs on the device (see
    wkv7_forward_raw in include/wkv7.h). Same outputs as ``forward``; device tensors only."""
    lib = load()
    B, T, H, N = r.shape
    dev = r.device
    if y is None:
        y = torch.empty((B, T, H, N), device=dev, dtype=torch.float32)
    if S_T is None and return_state:
        S_T = torch.empty((B, H, N, N), device=dev, dtype=torch.float32)
    n_snap = T // snap_every if snap_every else 0
    if snapshots is None and n_snap:
        snapshots = torch.empty((B, n_snap, H, N, N), device=dev, dtype=torch.float32)
    opts = make_opts(algo, chunk, snap_every, snapshots, ln_w, ln_b, r_k, gn_eps, segments)
    need = int(lib.wkv7_workspace_bytes(B, T, H, N, _dt(r), ctypes.byref(opts)))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = lib.wkv7_forward_raw(B, T, H, N, _dt(r), _ptr(r), _ptr(w_logit), _ptr(k), _ptr(v), _ptr(a_logit),
                                  _ptr(k_k), _ptr(k_a), _ptr(S0), _ptr(y), _ptr(S_T), ctypes.byref(opts),
                                  _ptr(workspace), ws_bytes, _stream_handle(dev, stream))
    _check(st, "wkv7_forward_raw")
    return y, S_T, snapshots


GRAD_NAMES = ("dr", "dw", "dk", "dv", "dkk", "da")


def backward_workspace_bytes(B, T, H, N=HEAD_SIZE, snap_every=0) -> int:
    return int(load().wkv7_backward_workspace_bytes(B, T, H, N, snap_every))


def backward(r, w, k, v, kk, a, dy, S0=None, dS_T=None, *, snapshots=None, snap_every=0, grads=None,
             dS0=None, return_state_grad=True, workspace=None, stream=None):
    """Gradients of <dy, y> + <dS_T, S_T> with respect to the forward's inputs (see
    wkv7_backward in include/wkv7.h). ``snapshots``/``snap_every``: the states a forward with
    the same ``snap_every`` wrote, bounding the recomputation. Device tensors only. Returns a
    dict of dr, dw, dk, dv, dkk, da ([B, T, H, 64] fp32) and dS0 ([B, H, 64, 64] or None)."""
    lib = load()
    B, T, H, N = r.shape
    dev = r.device
    if grads is None:
        grads = {n: torch.empty((B, T, H, N), device=dev, dtype=torch.float32) for n in GRAD_NAMES}
    if dS0 is None and return_state_grad:
        dS0 = torch.empty((B, H, N, N), device=dev, dtype=torch.float32)
    need = int(lib.wkv7_backward_workspace_bytes(B, T, H, N, snap_every))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = lib.wkv7_backward(B, T, H, N, _dt(r), _ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(kk), _ptr(a),
                               _ptr(S0), _ptr(snapshots), int(snap_every), _ptr(dy), _ptr(dS_T),
                               *(_ptr(grads[n]) for n in GRAD_NAMES), _ptr(dS0), _ptr(workspace), ws_bytes,
                               _stream_handle(dev, stream))
    _check(st, "wkv7_backward")
    out = dict(grads)
    out["dS0"] = dS0
    return out


def epilogue(y, r, k, v, ln_w, ln_b, r_k, *, gn_eps=64e-5, out=None, stream=None):
    """The group_norm + bonus epilogue on its own (wkv7_epilogue): returns out [B, T, H, N] fp32;
    ``out=y`` applies it in place. Device tensors only; r, k, v prepared inputs of one dtype."""
    lib = load()
    B, T, H, N = y.shape
    if out is None:
        out = torch.empty_like(y)
    with torch.cuda.device(y.device):
        st = lib.wkv7_epilogue(B, T, H, N, _dt(r), _ptr(y), _ptr(r), _ptr(k), _ptr(v), _ptr(ln_w), _ptr(ln_b),
                               _ptr(r_k), float(gn_eps), _ptr(out), _stream_handle(y.device, stream))
    _check(st, "wkv7_epilogue")
    return out


EPILOGUE_GRAD_NAMES = ("dy", "dr", "dk", "dv", "dln_w", "dln_b", "dr_k")


def epilogue_backward(y, r, k, v, ln_w, ln_b, r_k, dout, *, gn_eps=64e-5, grads=None, workspace=None, stream=None):
    """Backward of the epilogue (wkv7_epilogue_backward) for <dout, out>: returns a dict of dy,
    and the bonus's dr, dk, dv ([B, T, H, N] fp32) and dln_w, dln_b, dr_k ([H, N] fp32). y is
    the readout before the epilogue; dy is what ``backward`` takes, and its dr, dk, dv add to
    these."""
    lib = load()
    B, T, H, N = y.shape
    dev = y.device
    if grads is None:
        grads = {n: torch.empty((B, T, H, N) if n in ("dy", "dr", "dk", "dv") else (H, N), device=dev,
                                dtype=torch.float32) for n in EPILOGUE_GRAD_NAMES}
    need = int(lib.wkv7_epilogue_backward_workspace_bytes(B, T, H, N))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = lib.wkv7_epilogue_backward(B, T, H, N, _dt(r), _ptr(y), _ptr(r), _ptr(k), _ptr(v), _ptr(ln_w),
                                        _ptr(ln_b), _ptr(r_k), float(gn_eps), _ptr(dout),
                                        *(_ptr(grads[n]) for n in EPILOGUE_GRAD_NAMES), _ptr(workspace), ws_bytes,
                                        _stream_handle(dev, stream))
    _check(st, "wkv7_epilogue_backward")
    return dict(grads)


STATIC_SCRATCH_BYTES = 32 << 20   # capacity of the library's static backward scratch


def backward_static(r, w, k, v, kk, a, dy, S0=None, dS_T=None, *, snapshots=None, snap_every=0, grads=None,
                    dS0=None, return_state_grad=True, stream=None):
    """``backward`` through the allocation-free entry (wkv7_backward_static): the library's
    static scratch replaces the workspace; calls on one device must not overlap in time."""
    lib = load()
    B, T, H, N = r.shape
    dev = r.device
    if grads is None:
        grads = {n: torch.empty((B, T, H, N), device=dev, dtype=torch.float32) for n in GRAD_NAMES}
    if dS0 is None and return_state_grad:
        dS0 = torch.empty((B, H, N, N), device=dev, dtype=torch.float32)
    with torch.cuda.device(dev):
        st = lib.wkv7_backward_static(B, T, H, N, _dt(r), _ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(kk), _ptr(a),
                                      _ptr(S0), _ptr(snapshots), int(snap_every), _ptr(dy), _ptr(dS_T),
                                      *(_ptr(grads[n]) for n in GRAD_NAMES), _ptr(dS0), _stream_handle(dev, stream))
    _check(st, "wkv7_backward_static")
    out = dict(grads)
    out["dS0"] = dS0
    return out


def layer_dims(params, H, N=HEAD_SIZE):
    return LayerDims(H, N, params["Ww1"].shape[1], params["Wa1"].shape[1], params["Wv1"].shape[1],
                     params["Wg1"].shape[1])


def layer_forward(x, params, H, *, N=HEAD_SIZE, last_x=None, v0=None, S=None, out=None, v0_out=None,
                  last_x_out=None, algo="auto", chunk=0, segments=0, workspace=None, stream=None):
    """One time-mixing layer over x [B, T, C] (bf16 or fp32; C = H * N) with the weights in
    ``params`` (names as in LAYER_PARAMS; see wkv7_layer_forward in include/wkv7.h). S
    [B, H, N, N] fp32 is updated in place. Returns (out, v0_out, last_x_out, S): v0_out is the
    layer's v when v0 is None (the first layer), else None."""
    lib = load()
    B, T, C = x.shape
    dev = x.device
    dims = layer_dims(params, H, N)
    if out is None:
        out = torch.empty((B, T, C), device=dev, dtype=torch.float32)
    if v0 is None and v0_out is None:
        v0_out = torch.empty((B, T, C), device=dev, dtype=x.dtype)
    if last_x_out is None:
        last_x_out = torch.empty((B, C), device=dev, dtype=x.dtype)
    lp = LayerParams(*(None if params.get(n) is None else params[n].data_ptr() for n in LAYER_PARAMS))
    opts = make_opts(algo, chunk, 0, None, None, None, None, 64e-5, segments)
    need = int(lib.wkv7_layer_workspace_bytes(B, T, _dt(x), ctypes.byref(dims)))
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    with torch.cuda.device(dev):
        st = lib.wkv7_layer_forward(B, T, _dt(x), ctypes.byref(dims), ctypes.byref(lp), _ptr(x), _ptr(last_x),
                                    _ptr(v0), _ptr(S), _ptr(out), _ptr(v0_out), _ptr(last_x_out), ctypes.byref(opts),
                                    _ptr(workspace), ws_bytes, _stream_handle(dev, stream))
    _check(st, "wkv7_layer_forward")
    return out, (v0_out if v0 is None else None), last_x_out, S


def layer_workspace_bytes(B, T, params, H, N=HEAD_SIZE, dtype=torch.bfloat16) -> int:
    return int(load().wkv7_layer_workspace_bytes(B, T, BF16 if dtype == torch.bfloat16 else F32,
                                                 ctypes.byref(layer_dims(params, H, N))))


def decode_step(r, w, k, v, kk, a, S, *, y=None, ln_w=None, ln_b=None, r_k=None, gn_eps=64e-5, stream=None):
    """One decode step; inputs [B, H, N]; S [B, H, N, N] fp32 updated in place. Returns y
    ([B, H, N] fp32), with the group_norm + bonus epilogue applied when ln_w, ln_b, r_k are given."""
    lib = load()
    B, H, N = r.shape
    if y is None:
        y = torch.empty((B, H, N), device=r.device, dtype=torch.float32)
    args = (B, H, N, _dt(r), _ptr(r), _ptr(w), _ptr(k), _ptr(v), _ptr(kk), _ptr(a), _ptr(S), _ptr(y))
    with torch.cuda.device(r.device):
        if ln_w is None and ln_b is None and r_k is None:
            st, name = lib.wkv7_decode_step(*args, _stream_handle(r.device, stream)), "wkv7_decode_step"
        else:
            st = lib.wkv7_decode_step_ex(*args, _ptr(ln_w), _ptr(ln_b), _ptr(r_k), ctypes.c_float(gn_eps),
                                         _stream_handle(r.device, stream))
            name = "wkv7_decode_step_ex"
    _check(st, name)
    return y


def decode_step_raw(r, w_logit, k, v, a_logit, k_k, S, *, k_a=None, y=None, ln_w=None, ln_b=None, r_k=None,
                    gn_eps=64e-5, stream=None):
    """One decode step from the raw time-mixing values (decay and rate logits, the key before its
    update; per-head k_k [H, N] and optional k_a), optionally with the epilogue. Returns y."""
    lib = load()
    B, H, N = r.shape
    if y is None:
        y = torch.empty((B, H, N), device=r.device, dtype=torch.float32)
    with torch.cuda.device(r.device):
        st = lib.wkv7_decode_step_raw(B, H, N, _dt(r), _ptr(r), _ptr(w_logit), _ptr(k), _ptr(v), _ptr(a_logit),
                                      _ptr(k_k), _ptr(k_a), _ptr(S), _ptr(y), _ptr(ln_w), _ptr(ln_b), _ptr(r_k),
                                      ctypes.c_float(gn_eps), _stream_handle(r.device, stream))
    _check(st, "wkv7_decode_step_raw")
    return y


def poll_device_error(stream=None):
    """Synchronise the stream and raise Wkv7Error(ERR_TIMEOUT) if a kernel gave up a
    bounded device-side wait since the last poll."""
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(load().wkv7_poll_device_error(_stream_handle(dev, stream)), "wkv7_poll_device_error")


_copy_streams = {}


def _side_streams(dev):
    """Two copy streams per device (host->device and device->host), made once."""
    if dev not in _copy_streams:
        _copy_streams[dev] = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    return _copy_streams[dev]


def _forward_host(r, w, k, v, kk, a, S0, *, return_state, out_host, **kw):
    """End-to-end path for host tensors. The batch is cut into up to eight slices of whole
    sequences (at least 24 MB of input each, so per-copy overheads stay small); slice i's host->device copies (one stream), its forward (the current stream)
    and its device->host copies (another stream) overlap with those of the other slices, so
    the two copy directions and the kernels run at the same time. Returns after the
    current stream has waited for everything and been synchronised."""
    dev = torch.device("cuda", torch.cuda.current_device())
    main = torch.cuda.current_stream(dev)
    s_in, s_out = _side_streams(dev)
    B, T, H, N = r.shape
    snap_every = kw.get("snap_every", 0)
    n_snap = T // snap_every if snap_every else 0
    ins = {"r": r, "w": w, "k": k, "v": v, "kk": kk, "a": a, "S0": S0}
    dv = {n: None if t is None else torch.empty(t.shape, dtype=t.dtype, device=dev) for n, t in ins.items()}
    y_d = torch.empty((B, T, H, N), device=dev, dtype=torch.float32)
    S_d = torch.empty((B, H, N, N), device=dev, dtype=torch.float32) if return_state else None
    sn_d = torch.empty((B, n_snap, H, N, N), device=dev, dtype=torch.float32) if n_snap else None
    y_h, S_h = out_host if out_host is not None else (None, None)
    if y_h is None:
        y_h = torch.empty((B, T, H, N), dtype=torch.float32, pin_memory=True)
    if S_d is not None and S_h is None:
        S_h = torch.empty((B, H, N, N), dtype=torch.float32, pin_memory=True)
    sn_h = torch.empty((B, n_snap, H, N, N), dtype=torch.float32, pin_memory=True) if n_snap else None
    s_in.wait_stream(main)   # the device buffers above were made on the current stream
    ep = {}
    with torch.cuda.stream(s_in):
        for n in ("ln_w", "ln_b", "r_k"):
            t = kw.pop(n, None)
            ep[n] = None if t is None else t.to(dev, non_blocking=True)
    for t in [*dv.values(), *ep.values()]:
        if t is not None:
            t.record_stream(s_in)
    in_bytes = sum(t.numel() * t.element_size() for t in ins.values() if t is not None)
    pieces = max(1, min(B, 8, in_bytes // (24 << 20))) if T > 0 else 1   # slices of >= 24 MB of input
    cuts = [B * i // pieces for i in range(pieces + 1)]
    for b0, b1 in zip(cuts[:-1], cuts[1:]):
        if b0 == b1:
            continue
        with torch.cuda.stream(s_in):
            for n, t in ins.items():
                if t is not None:
                    dv[n][b0:b1].copy_(t[b0:b1], non_blocking=True)
        main.wait_stream(s_in)
        sl = lambda t: None if t is None else t[b0:b1]
        forward(*(dv[n][b0:b1] for n in ("r", "w", "k", "v", "kk", "a")), sl(dv["S0"]), y=y_d[b0:b1],
                S_T=sl(S_d), snapshots=sl(sn_d), return_state=return_state, **ep, **kw)
        s_out.wait_stream(main)
        with torch.cuda.stream(s_out):
            y_h[b0:b1].copy_(y_d[b0:b1], non_blocking=True)
            if S_d is not None:
                S_h[b0:b1].copy_(S_d[b0:b1], non_blocking=True)
            if sn_d is not None:
                sn_h[b0:b1].copy_(sn_d[b0:b1], non_blocking=True)
    for t in (y_d, S_d, sn_d):
        if t is not None:
            t.record_stream(s_out)
    main.wait_stream(s_out)
    main.synchronize()
    return y_h, (S_h if return_state else None), sn_h


def probe_peak(kind, *, n=256, iters=None, blocks=None, reps=5, device=None):
    """Measured rate (TFLOP/s) of one pipe: kind "fp32_fma" (the FMA pipe, all SMs) or
    "tf32_mma" (tcgen05 kind::tf32, M = 128 and N = n, one CTA per SM). Each of `reps` launches
    is timed with CUDA events on the current stream after a warm-up launch; the median is kept."""
    lib = load()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    stream = torch.cuda.current_stream(dev)
    flops = ctypes.c_double(0.0)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    def launch():
        if kind == "fp32_fma":
            st = lib.wkv7_probe_fp32_fma(blocks or 8 * sms, iters or 4096, ctypes.c_void_p(stream.cuda_stream),
                                         ctypes.byref(flops))
        elif kind == "tf32_mma":
            st = lib.wkv7_probe_tf32_mma(int(n), iters or 20000, ctypes.c_void_p(stream.cuda_stream),
                                         ctypes.byref(flops))
        else:
            raise ValueError(kind)
        _check(st, "wkv7_probe_" + kind)

    with torch.cuda.device(dev):
        launch()
        times = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            launch()
            e1.record(stream)
            e1.synchronize()
            times.append(e0.elapsed_time(e1))
        poll_device_error()
    times.sort()
    return flops.value / (times[len(times) // 2] * 1e-3) / 1e12


def _host_ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _host_opts(algo, chunk, snap_every, snapshots, ln_w, ln_b, r_k, gn_eps, segments):
    o = make_opts(algo, chunk, snap_every, None, None, None, None, gn_eps, segments)
    o.snapshots = None if snapshots is None else snapshots.data_ptr()
    o.ln_w = None if ln_w is None else ln_w.data_ptr()
    o.ln_b = None if ln_b is None else ln_b.data_ptr()
    o.r_k = None if r_k is None else r_k.data_ptr()
    return o


def forward_host_workspace_bytes(B, T, H, N=HEAD_SIZE, dtype=torch.bfloat16, *, snap_every=0, epilogue=False,
                                 algo="auto", chunk=0, segments=0) -> int:
    o = make_opts(algo, chunk, snap_every, None, None, None, None, 64e-5, segments)
    if epilogue:   # any non-null value marks the epilogue as on for the size query
        o.ln_w = o.ln_b = o.r_k = 16
    return int(load().wkv7_forward_host_workspace_bytes(B, T, H, N, _dt_of(dtype), ctypes.byref(o)))


def _dt_of(dtype):
    return BF16 if dtype == torch.bfloat16 else F32


def forward_host(r, w, k, v, kk, a, S0, y, S_T, workspace, *, algo="auto", chunk=0, snap_every=0,
                 snapshots=None, ln_w=None, ln_b=None, r_k=None, gn_eps=64e-5, segments=0, stream=None):
    """wkv7_forward_host: every tensor but ``workspace`` is a host (CPU) tensor, pinned for
    asynchronous copies; ``workspace`` is a device uint8 tensor of at least
    ``forward_host_workspace_bytes`` bytes. Enqueues the copies and kernels on the current
    stream of the workspace's device and returns; synchronise that stream before reading y,
    S_T and the snapshots."""
    lib = load()
    B, T, H, N = r.shape
    dev = workspace.device
    opts = _host_opts(algo, chunk, snap_every, snapshots, ln_w, ln_b, r_k, gn_eps, segments)
    with torch.cuda.device(dev):
        st = lib.wkv7_forward_host(B, T, H, N, _dt(r), *(_host_ptr(t) for t in (r, w, k, v, kk, a, S0, y, S_T)),
                                   ctypes.byref(opts), ctypes.c_void_p(workspace.data_ptr()),
                                   workspace.numel() * workspace.element_size(), _stream_handle(dev, stream))
    _check(st, "wkv7_forward_host")
    return y, S_T, snapshots
