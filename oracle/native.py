"""ctypes binding and build step for the plain-C fp64 oracle (wkv7_oracle.c).

TEST INFRASTRUCTURE ONLY (tests, the graft smoke check, the benchmark's CPU
baseline). The C source states the recurrence of the rebuttal page's numpy
``time_mixing`` listing with plain loops; see its header.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from .reference import _f64

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv7_oracle.c")
_LIB = os.path.join(_HERE, "libwkv7_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math: the loops keep their order)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-o", tmp, _SRC, "-lm"],
                       check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            d = ctypes.POINTER(ctypes.c_double)
            lib.wkv7_oracle_forward.argtypes = [ctypes.c_int] * 4 + [d] * 6 + [d, d, d, ctypes.c_int, d,
                                                                             ctypes.c_int]
            lib.wkv7_oracle_forward.restype = ctypes.c_int
            lib.wkv7_oracle_epilogue.argtypes = [ctypes.c_int] * 4 + [d] * 7 + [ctypes.c_double, d]
            lib.wkv7_oracle_epilogue.restype = ctypes.c_int
            lib.wkv7_oracle_layer.argtypes = [ctypes.c_int] * 8 + [d] * 30 + [ctypes.c_double] + [d] * 4
            lib.wkv7_oracle_layer.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(x):
    if x is None:
        return None
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def host_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def forward(r, w, k, v, kk, a, S0=None, snap_every=0, nthreads=0):
    """fp64 recurrence on host threads. Same contract as reference.wkv7_recurrence."""
    lib = _load()
    arrs = [np.ascontiguousarray(_f64(x)) for x in (r, w, k, v, kk, a)]
    B, T, H, N = arrs[0].shape
    s0 = None if S0 is None else np.ascontiguousarray(_f64(S0))
    y = np.empty((B, T, H, N))
    S_T = np.empty((B, H, N, N))
    n_snap = T // snap_every if snap_every else 0
    snaps = np.empty((B, n_snap, H, N, N)) if n_snap else None
    rc = lib.wkv7_oracle_forward(B, T, H, N, *[_ptr(x) for x in arrs], _ptr(s0), _ptr(y), _ptr(S_T),
                                 int(snap_every), _ptr(snaps), int(nthreads or host_threads()))
    if rc != 0:
        raise RuntimeError(f"wkv7_oracle_forward failed with {rc}")
    return y, S_T, snaps


def epilogue(y, r, k, v, ln_w, ln_b, r_k, eps=64e-5):
    """fp64 group_norm + bonus. Same contract as reference.group_norm_bonus."""
    lib = _load()
    ys, rs, ks, vs = (np.ascontiguousarray(_f64(x)) for x in (y, r, k, v))
    lw, lb, rk = (np.ascontiguousarray(_f64(x)) for x in (ln_w, ln_b, r_k))
    B, T, H, N = ys.shape
    out = np.empty_like(ys)
    rc = lib.wkv7_oracle_epilogue(B, T, H, N, _ptr(ys), _ptr(rs), _ptr(ks), _ptr(vs), _ptr(lw),
                                  _ptr(lb), _ptr(rk), float(eps), _ptr(out))
    if rc != 0:
        raise RuntimeError(f"wkv7_oracle_epilogue failed with {rc}")
    return out


_LAYER_ORDER = ("mr", "mw", "mk", "mv", "ma", "mg", "w_bias", "a_bias", "v_bias", "r_k", "k_k", "k_a", "ln_w",
                "ln_b", "Wr", "Wk", "Wv", "Wo", "Ww1", "Ww2", "Wa1", "Wa2", "Wv1", "Wv2", "Wg1", "Wg2")


def time_mixing_layer(x, params, last_x=None, v0=None, S0=None, eps=64e-5):
    """The C transcription of one time-mixing layer (wkv7_oracle_layer: the listing token by
    token with plain loops). Same contract as reference.time_mixing_layer; k_a must be given."""
    lib = _load()
    P = {n: np.ascontiguousarray(_f64(params[n])) for n in _LAYER_ORDER}
    xs = np.ascontiguousarray(_f64(x))
    B, T, C = xs.shape
    H, N = P["r_k"].shape
    dims = [P[n].shape[1] for n in ("Ww1", "Wa1", "Wv1", "Wg1")]
    lx = None if last_x is None else np.ascontiguousarray(_f64(last_x))
    v0s = None if v0 is None else np.ascontiguousarray(_f64(v0))
    s0 = None if S0 is None else np.ascontiguousarray(_f64(S0))
    out = np.empty((B, T, C))
    v0_out = np.empty((B, T, C))
    last = np.empty((B, C))
    S_T = np.empty((B, H, N, N))
    rc = lib.wkv7_oracle_layer(B, T, H, N, *dims, _ptr(xs), _ptr(lx), _ptr(v0s), _ptr(s0),
                               *(_ptr(P[n]) for n in _LAYER_ORDER), float(eps), _ptr(out), _ptr(v0_out),
                               _ptr(last), _ptr(S_T))
    if rc != 0:
        raise RuntimeError(f"wkv7_oracle_layer failed with {rc}")
    return out, v0_out, last, S_T
