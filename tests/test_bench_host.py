"""Host-side arithmetic of bench.py (CPU): the algorithmic bytes the roofline divides by, and
the device-code digest that ties a profile's measured traffic to the code it was taken on."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from linear_rnn_sequence_rwkv_b200 import inputs  # noqa: E402


def test_algorithmic_bytes_of_the_prefill_workloads():
    """1,024 B per token-head (six bf16 inputs of 64 channels, fp32 y) plus 16 KiB per head for
    every state read or written; five inputs and the per-head k_k, k_a on the raw path."""
    wl = inputs.WORKLOADS[1]                                   # B8 T1024 H12, S0 in, S_T out
    assert bench.algorithmic_bytes(wl, 8, 1024, 12, 2, True, True, 0, False) == 98304 * 1024 + 96 * 16384 * 2
    assert bench.algorithmic_bytes(wl, 8, 1024, 12, 2, True, True, 0, False, raw=True) == \
        98304 * 896 + 96 * 16384 * 2 + 12 * 64 * 2 * 4
    wl2 = inputs.WORKLOADS[2]                                  # with the epilogue parameters
    assert bench.algorithmic_bytes(wl2, 16, 4096, 32, 2, False, True, 0, True) == \
        16 * 4096 * 32 * 1024 + 512 * 16384 + 32 * 64 * 3 * 4


def test_digest_ignores_comments_only():
    src = "int f(int x) { return x + 1; }  // one\n"
    assert bench._strip_comments(src) == bench._strip_comments("/* a */ int f(int x) { return x + 1; }\n")
    assert bench._strip_comments(src) != bench._strip_comments("int f(int x) { return x + 2; }")
    assert bench._strip_comments('const char *s = "a // b";') == 'const char *s = "a // b";'


def test_profiles_match_the_current_device_code():
    """Every committed profile summary that records traffic was taken on the device code now in
    the tree (otherwise the bench reports its traffic as null)."""
    for kernel, workload, raw in (("chunk_kernel", "prefill-0.19b", False), ("chunk_kernel", "prefill-1.5b", False),
                                  ("chunk_kernel", "long-context", False), ("chunk_kernel", "prefill-0.19b", True),
                                  ("decode_kernel", "decode", False), ("seq_kernel", "prefill-0.19b", False),
                                  ("bwd_kernel", "prefill-0.19b", False)):
        assert bench.measured_traffic(kernel, workload, raw) is not None, (kernel, workload, raw)
