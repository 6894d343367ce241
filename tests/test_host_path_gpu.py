"""The end-to-end path of the binding (host tensors in, host tensors out): the batch is
pipelined in slices over two copy streams and the current stream; the results must equal
the device path bit for bit (every slice runs the same kernels on the same bytes; the
chunked kernel's results do not depend on how many CTAs share a head)."""
import pytest
import torch

from linear_rnn_sequence_rwkv_b200 import inputs, wkv7

pytestmark = pytest.mark.gpu

NAMES = ("r", "w", "k", "v", "kk", "a")


@pytest.mark.parametrize("B,T,H,epi,snap", [(8, 300, 3, False, 0), (5, 130, 2, True, 64), (1, 64, 4, False, 0),
                                            (3, 0, 2, False, 0), (6, 1, 2, False, 0)])
def test_host_path_equals_device_path(cuda_device, B, T, H, epi, snap):
    wl = inputs.WORKLOADS[2 if epi else 1]
    d = inputs.make_inputs(wl, B=B, T=T, H=H, seed=800 + B + T, s0="normal")
    host = {n: (t.pin_memory() if isinstance(t, torch.Tensor) else t) for n, t in d.items()}
    ep_h = {n: host[n] for n in ("ln_w", "ln_b", "r_k")} if epi else {}
    y_h, S_h, sn_h = wkv7.forward(*(host[n] for n in NAMES), host["S0"], snap_every=snap, **ep_h)
    assert y_h.device.type == "cpu" and S_h.device.type == "cpu"
    dd = {n: (t.to(cuda_device) if isinstance(t, torch.Tensor) else t) for n, t in d.items()}
    ep_d = {n: dd[n] for n in ("ln_w", "ln_b", "r_k")} if epi else {}
    y, S, sn = wkv7.forward(*(dd[n] for n in NAMES), dd["S0"], snap_every=snap, **ep_d)
    assert torch.equal(y_h, y.cpu())
    assert torch.equal(S_h, S.cpu())
    if snap and T >= snap:
        assert torch.equal(sn_h, sn.cpu())


def test_host_path_into_given_buffers(cuda_device):
    d = inputs.make_inputs(inputs.WORKLOADS[1], B=4, T=100, H=2, seed=830, s0="normal")
    host = {n: (t.pin_memory() if isinstance(t, torch.Tensor) else t) for n, t in d.items()}
    y_h = torch.full((4, 100, 2, 64), float("nan")).pin_memory()
    S_h = torch.full((4, 2, 64, 64), float("nan")).pin_memory()
    y, S, _ = wkv7.forward(*(host[n] for n in NAMES), host["S0"], out_host=(y_h, S_h))
    assert y is y_h and S is S_h and torch.isfinite(y_h).all() and torch.isfinite(S_h).all()


@pytest.mark.parametrize("B,T,H,epi,snap", [(3, 200, 2, False, 0), (16, 512, 8, True, 128), (2, 0, 3, False, 0)])
def test_c_abi_host_entry_matches_the_device_path(cuda_device, B, T, H, epi, snap):
    """wkv7_forward_host (pinned host buffers, device copies in the caller's workspace) gives
    the device path's results bit for bit; a second call reuses the workspace."""
    wl = inputs.WORKLOADS[2] if epi else inputs.WORKLOADS[1]
    for seed in (71, 72):
        d = inputs.make_inputs(wl, B=B, T=T, H=H, seed=seed, s0="normal")
        host = {n: (v.pin_memory() if isinstance(v, torch.Tensor) else v) for n, v in d.items()}
        ep = {n: host[n] for n in ("ln_w", "ln_b", "r_k")} if epi else {}
        y_h = torch.empty(B, T, H, 64).pin_memory()
        S_h = torch.empty(B, H, 64, 64).pin_memory()
        sn_h = torch.empty(B, T // snap, H, 64, 64).pin_memory() if snap else None
        ws = torch.empty(wkv7.forward_host_workspace_bytes(B, T, H, snap_every=snap, epilogue=epi),
                         dtype=torch.uint8, device=cuda_device)
        wkv7.forward_host(*(host[n] for n in NAMES), host["S0"], y_h, S_h, ws, snap_every=snap, snapshots=sn_h,
                          **ep)
        torch.cuda.synchronize(cuda_device)
        dd = {n: (None if v is None else v.to(cuda_device)) for n, v in d.items()}
        dep = {n: dd[n] for n in ("ln_w", "ln_b", "r_k")} if epi else {}
        y, S, sn = wkv7.forward(*(dd[n] for n in NAMES), dd["S0"], snap_every=snap, **dep)
        assert torch.equal(y_h, y.cpu())
        assert torch.equal(S_h, S.cpu())
        if snap:
            assert torch.equal(sn_h, sn.cpu())


def test_c_abi_host_entry_rejects_device_buffers(cuda_device):
    d = inputs.make_inputs(inputs.WORKLOADS[1], B=1, T=64, H=2, seed=3)
    dd = {n: (None if v is None else v.to(cuda_device)) for n, v in d.items()}
    ws = torch.empty(wkv7.forward_host_workspace_bytes(1, 64, 2), dtype=torch.uint8, device=cuda_device)
    y_h = torch.empty(1, 64, 2, 64).pin_memory()
    with pytest.raises(wkv7.Wkv7Error) as e:
        wkv7.forward_host(*(dd[n] for n in NAMES), dd["S0"], y_h, None, ws)
    assert e.value.status == wkv7.ERR_ARG
