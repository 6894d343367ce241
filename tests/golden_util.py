"""Loads the golden fixtures under tests/golden/ into recurrence inputs."""
import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def elementary_transitions():
    """Inputs [1, T, 1, N] (fp64) and the expected states / readouts of the
    appendix-D.3 construction fixture."""
    with open(os.path.join(GOLDEN, "elementary_transitions.json")) as f:
        doc = json.load(f)
    N = doc["N"]
    steps = doc["steps"]
    T = len(steps)
    S0 = np.asarray(doc["S0"], dtype=np.float64)
    e = np.eye(N)
    shape = (1, T, 1, N)
    w = np.ones(shape)
    k = np.zeros(shape)
    v = np.zeros(shape)
    kk = np.zeros(shape)
    a = np.zeros(shape)
    r = np.zeros(shape)
    S_exp = np.empty((T, N, N))
    y_exp = np.empty((T, N))
    for t, st in enumerate(steps):
        i, j = st["i"], st["j"]
        if st["op"] in ("swap", "copy"):
            kk[0, t, 0] = (e[i] - e[j]) / math.sqrt(2.0)
            a[0, t, 0] = 2.0 * (e[i] + e[j] if st["op"] == "swap" else e[j])
        else:
            kk[0, t, 0] = e[0]
        r[0, t, 0, st["read"]] = 1.0
        src = np.asarray(st["src_after"])
        S_exp[t] = S0[:, src]
        y_exp[t] = S0[:, src[st["read"]]]
    return dict(r=r, w=w, k=k, v=v, kk=kk, a=a, S0=S0.reshape(1, 1, N, N),
                S_expected=S_exp, y_expected=y_exp)
