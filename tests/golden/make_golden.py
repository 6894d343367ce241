"""Writes tests/golden/elementary_transitions.json.

Source: RWKV-7 "Goose" paper summary, appendix D.3 ("Lemmas for Theorem 3"):
every elementary transition (identity, swap, copy) is realised by one RWKV-7
step with a unit-norm removal key and a binary gate, using c = 2 (the in-context
learning rate a = 2 * gate). With w = 1 and no write (k = v = 0):

* swap(i, j):  kk = (e_i - e_j)/sqrt(2), gate on i and j  -> key columns i, j swap
* copy(i->j):  kk = (e_i - e_j)/sqrt(2), gate on j only    -> column j := column i
* identity:    gate off                                    -> state unchanged

Each op is a map of key columns, so the expected state after token t is
S_t[:, c] = S0[:, src_t[c]] and, with a one-hot readout r_t = e_{m_t},
y_t = S0[:, src_t[m_t]]. S0 holds small integers. The stored values are these
column maps; no arithmetic of the recurrence is involved in writing them.
"""
import json
import os

import numpy as np

N = 64
OPS = [("swap", 3, 17), ("copy", 5, 40), ("identity", 0, 0), ("swap", 0, 63),
       ("copy", 63, 1), ("swap", 3, 17), ("copy", 40, 2), ("swap", 2, 5)]
READ = [17, 40, 9, 63, 1, 3, 2, 5]


def main():
    rng = np.random.default_rng(2503_14456)
    S0 = rng.integers(-8, 9, size=(N, N))
    src = np.arange(N)
    steps = []
    for (op, i, j), m in zip(OPS, READ):
        nxt = src.copy()
        if op == "swap":
            nxt[i], nxt[j] = src[j], src[i]
        elif op == "copy":
            nxt[j] = src[i]
        steps.append({"op": op, "i": i, "j": j, "read": m, "src_after": nxt.tolist()})
        src = nxt
    doc = {
        "citation": "RWKV-7 'Goose' paper summary, appendix D.3 (elementary transitions, c = 2)",
        "N": N,
        "S0": S0.tolist(),
        "steps": steps,
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "elementary_transitions.json")
    with open(path, "w") as f:
        json.dump(doc, f, separators=(",", ":"))
    print("wrote", path)


if __name__ == "__main__":
    main()
