"""CPU fp64 oracle for the WKV-7 recurrence (RWKV-7 "Goose").

TEST INFRASTRUCTURE: only tests/, ``__graft_entry__.smoke()`` and the benchmark's
``cpu_baseline`` / ``--impl reference`` legs may import, call, link or execute
anything under this directory. The product path (the CUDA library and its Python
binding) never does, and fails loudly when its extension is missing.

* ``reference``: numpy fp64 statement of the recurrence and epilogue.
* ``native``: the same definition in plain C (fp64, POSIX threads over independent
  (batch, head) units), for full-size sampling and the CPU baseline.

Parity pins: see tests/test_oracle.py. Every function is pinned against closed
forms, brute-force transition products or the paper's transition constructions;
no function here is "parity unpinned".
"""
