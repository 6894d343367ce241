"""The multi-rank path of bench.py on CPU: two processes over gloo (127.0.0.1). The path has
no data-parallel collective; what the ranks share is the barrier around the timed region and
the max-over-ranks reduction of the device time, and each rank draws its own batch."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    from linear_rnn_sequence_rwkv_b200 import inputs
    w, r, _ = bench.dist_setup()
    assert (w, r) == (world, rank)
    bench.barrier(world)
    got = bench.max_over_ranks(1.5 + rank, world, torch.device("cpu"))
    wl = inputs.WORKLOADS[1]
    d = inputs.make_inputs(wl, B=1, T=8, H=2, seed=bench.rank_seed(wl, rank))
    out[rank] = (got, float(d["r"].float().sum()))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_ranks_share_only_the_barrier_and_the_max():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.5              # max over ranks of 1.5 and 2.5
    assert res[0][1] != res[1][1]                      # each rank drew its own batch


def test_reference_arm_prints_once_under_torchrun():
    """`bench.py --impl reference` under a two-rank launcher: rank 0 alone runs the oracle and
    prints the one JSON line; rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "decode"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0


def test_reference_arm_line_carries_the_contract_keys():
    """The reference arm's JSON line (the oracle on the host cores) has every key the bench
    contract names, with the reference's own e2e and cpu_baseline objects."""
    cmd = [sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", "decode"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    d = json.loads([l for l in r.stdout.splitlines() if l.startswith("{")][-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
        assert key in d, key
    assert d["impl"] == "reference" and d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert "workload" in d["config"]
