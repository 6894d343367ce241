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
