"""The allocation-free backward entry (wkv7_backward_static): the library's static scratch
in place of a caller's workspace. Collected last, so that it also runs after every other
test has used the device; it must pass alone as well."""
import ctypes
import dataclasses

import pytest
import torch

from linear_rnn_sequence_rwkv_b200 import inputs, wkv7

NAMES = ("r", "w", "k", "v", "kk", "a")
FAKE = 0x10000


def _case(B, T, H, seed, N=64):
    d = inputs.make_inputs(dataclasses.replace(inputs.WORKLOADS[1], N=N), B=B, T=T, H=H, seed=seed, s0="normal")
    g = torch.Generator().manual_seed(seed + 1)
    d["dy"] = torch.randn(B, T, H, N, generator=g)
    d["dS_T"] = 0.1 * torch.randn(B, H, N, N, generator=g)
    return d


def test_static_entry_rejects_requests_above_its_capacity():
    """B*H*ceil(K/4) checkpoints of 16 KiB must fit 32 MiB; one more is refused on the host."""
    lib = wkv7.load()
    assert wkv7.backward_workspace_bytes(2, 1024, 4) == wkv7.STATIC_SCRATCH_BYTES      # exactly full
    B, T, H = 1, 4 * 2048 + 1, 1
    assert wkv7.backward_workspace_bytes(B, T, H) > wkv7.STATIC_SCRATCH_BYTES
    P = lambda i: ctypes.c_void_p(FAKE + 0x1000000 * i)
    st = lib.wkv7_backward_static(B, T, H, 64, 1, *(P(i) for i in range(1, 7)), None, None, 0, P(7), None,
                                  *(P(i) for i in range(8, 14)), None, None)
    assert st == wkv7.ERR_WORKSPACE
    assert b"static scratch" in lib.wkv7_last_error()
    # N = 128: a head's two CTAs hold 64 KB states, one per two tokens of a segment
    assert wkv7.backward_workspace_bytes(1, 1024, 1, N=128) == wkv7.STATIC_SCRATCH_BYTES   # exactly full
    st = lib.wkv7_backward_static(1, 1026, 1, 128, 1, *(P(i) for i in range(1, 7)), None, None, 0, P(7), None,
                                  *(P(i) for i in range(8, 14)), None, None)
    assert st == wkv7.ERR_WORKSPACE


@pytest.mark.gpu
@pytest.mark.parametrize("B,T,H,snap_every,N", [(2, 130, 3, 0, 64), (2, 1024, 4, 0, 64), (3, 300, 2, 64, 64),
                                                (2, 130, 2, 0, 128), (2, 300, 3, 64, 128)])
def test_static_entry_matches_workspace_entry_on_consecutive_calls(cuda_device, B, T, H, snap_every, N):
    """Two calls in a row with different inputs: each equals wkv7_backward bit for bit (the
    second call sees the first one's leftovers in the scratch and must not depend on them)."""
    for seed in (900 + T, 901 + T):
        d = {k: (None if v is None else v.to(cuda_device)) for k, v in _case(B, T, H, seed, N).items()}
        snaps = None
        if snap_every:
            _, _, snaps = wkv7.forward(*(d[n] for n in NAMES), d["S0"], snap_every=snap_every, algo="seq")
        got = wkv7.backward_static(*(d[n] for n in NAMES), d["dy"], d["S0"], d["dS_T"], snapshots=snaps,
                                   snap_every=snap_every)
        ref = wkv7.backward(*(d[n] for n in NAMES), d["dy"], d["S0"], d["dS_T"], snapshots=snaps,
                            snap_every=snap_every)
        for n in wkv7.GRAD_NAMES + ("dS0",):
            assert torch.equal(got[n], ref[n]), n


@pytest.mark.gpu
def test_static_entry_takes_no_device_memory(cuda_device):
    """With every argument allocated up front, further calls leave the device's free memory
    unchanged: the entry itself allocates nothing (its scratch is part of the loaded module)."""
    B, T, H = 2, 200, 3
    d = {k: (None if v is None else v.to(cuda_device)) for k, v in _case(B, T, H, 950).items()}
    grads = {n: torch.empty(B, T, H, 64, device=cuda_device) for n in wkv7.GRAD_NAMES}
    dS0 = torch.empty(B, H, 64, 64, device=cuda_device)
    call = lambda: wkv7.backward_static(*(d[n] for n in NAMES), d["dy"], d["S0"], d["dS_T"], grads=grads,
                                        dS0=dS0)
    call()                                   # first call on the device: the scratch address lookup
    torch.cuda.synchronize(cuda_device)
    free0 = torch.cuda.mem_get_info(cuda_device)[0]
    for _ in range(3):
        call()
    torch.cuda.synchronize(cuda_device)
    assert torch.cuda.mem_get_info(cuda_device)[0] == free0


@pytest.mark.gpu
def test_static_and_workspace_entries_on_a_second_device(cuda_device):
    """Kernel attributes and the scratch address are per device: the backward runs on device 1
    after device 0 in the same process (skipped with one visible device)."""
    if torch.cuda.device_count() < 2:
        pytest.skip("one visible CUDA device")
    B, T, H = 1, 130, 2
    for dev in (torch.device("cuda:0"), torch.device("cuda:1")):
        d = {k: (None if v is None else v.to(dev)) for k, v in _case(B, T, H, 960).items()}
        got = wkv7.backward_static(*(d[n] for n in NAMES), d["dy"], d["S0"], d["dS_T"])
        ref = wkv7.backward(*(d[n] for n in NAMES), d["dy"], d["S0"], d["dS_T"])
        for n in wkv7.GRAD_NAMES + ("dS0",):
            assert torch.equal(got[n], ref[n]), (dev, n)
