#!/usr/bin/env python
"""Throughput benchmark of the WKV-7 recurrence on B200 (synthetic inputs).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the hot path over one batch of the workload:
  prefill-1.5b (default): wkv7_forward on B16 T4096 H32 N64, bf16 inputs, fp32 state out,
      y fp32 with the fused group_norm + bonus epilogue (the largest prefill shape that
      fits one GPU). The same line carries a `decode` record (B256 H40, 128 steps replayed
      from a CUDA graph) and a `chunk_sweep` record (the same shape at chunk 16, 32, 64);
  prefill-0.19b: B8 T1024 H12, state carried in (S0 ~ N(0, 0.1^2)) and out;
  long-context: B1 T65536 H40, decay logits ~ N(2, 1), snapshots every 4096 tokens;
  decode: one wkv7_decode_step on B256 H40 (fp32 state in HBM); with --inputs raw, one
      wkv7_decode_step_raw with the epilogue (the pre-processing and group_norm + bonus fused).
Prints ONE JSON line (rank 0). Under torchrun every rank runs its own independent
batch (weak scaling over (b, h) units, no collective on the data path); the timed
region is bracketed by a barrier and a device synchronisation, and the time is the
max over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from linear_rnn_sequence_rwkv_b200 import inputs  # noqa: E402

METRIC = "WKV-7 Mtokens·heads/s (prefill, decode) at N=64 bf16; % of HBM/FP32/TC roofline"
UNIT = "Mtoken·heads/s"
L2_BYTES = 126 * 2 ** 20
NAMES = ("r", "w", "k", "v", "kk", "a")
RAW_NAMES = ("r", "w_logit", "k", "v", "a_logit")   # raw time-mixing values (pre-processing fused)

WORKLOADS = {
    "prefill-0.19b": dict(cid=1, default_steps=200),
    "prefill-1.5b": dict(cid=2, default_steps=20),
    "long-context": dict(cid=4, default_steps=10),
    "decode": dict(cid=3, default_steps=256),
}


# ---- measured DRAM traffic of the dominant kernel (committed ncu summaries under profiles/) -------

KERNEL_SOURCES = {"chunk_kernel": ("chunk.cu", "tc_util.cuh", "common.cuh"),
                  "bwd_kernel": ("backward.cu", "backward.cuh", "tc_util.cuh", "common.cuh"),
                  "decode_kernel": ("decode.cu", "decode.cuh", "common.cuh"),
                  "seq_kernel": ("seq.cu", "common.cuh")}
PROFILE_TAGS = {"prefill-0.19b": "prefill-0.19B", "prefill-1.5b": "prefill-1.5B",
                "long-context": "long-context", "decode": "decode-2.9B"}


def _strip_comments(text: str) -> str:
    """C/C++ source without its comments, blank lines and indentation (string and character
    literals kept), so that a comment edit does not count as a change of the compiled code."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            i = text.find("\n", i)
            i = n if i < 0 else i
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return "\n".join(l.strip() for l in "".join(out).splitlines() if l.strip())


def kernel_digest(kernel: str) -> str:
    """sha256 (16 hex digits) of the device code a kernel is built from: its .cu file up to the
    host-side section, plus the headers it includes, comments removed."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "linear_rnn_sequence_rwkv_b200", "csrc", f)) as fh:
            text = fh.read()
        cut = text.find("// ---- host side")
        h.update(_strip_comments(text if cut < 0 else text[:cut]).encode())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str, raw: bool = False):
    """dram__bytes_read.sum + dram__bytes_write.sum per launch recorded in
    profiles/<kernel>_<workload>.md, or None without a capture or when the kernel's device
    code has changed since it was taken (the summary records the digest it was taken at)."""
    tag = PROFILE_TAGS.get(workload, workload) + ("-raw-inputs" if raw else "")
    path = os.path.join(ROOT, "profiles", f"{kernel}_{tag}.md")
    try:
        with open(path) as f:
            text = f.read()
    except OSError:
        return None
    t = re.search(r"^traffic_bytes_per_launch:\s*(\d+)\s*$", text, re.M)
    d = re.search(r"^device_code_sha256_16:\s*([0-9a-f]{16})\s*$", text, re.M)
    if not (t and d) or d.group(1) != kernel_digest(kernel):
        return None
    return int(t.group(1))


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}, "fallback"


_PIPE_PEAKS = {}


def pipe_peaks(dev):
    """FP32 FMA and tf32 tensor-core rates measured on this device in this run (the library's
    peak probes, CUDA-event timed): the denominators of the "alu" and "tensor" rooflines."""
    key = str(dev)
    if key not in _PIPE_PEAKS:
        from linear_rnn_sequence_rwkv_b200 import wkv7
        with torch.cuda.device(dev):
            _PIPE_PEAKS[key] = {"fp32_fma_tflops": round(wkv7.probe_peak("fp32_fma"), 2),
                                "tf32_mma_tflops": {str(n): round(wkv7.probe_peak("tf32_mma", n=n), 1)
                                                    for n in (64, 128, 256)},
                                "source": "wkv7_probe_fp32_fma / wkv7_probe_tf32_mma, CUDA events, this run"}
    return _PIPE_PEAKS[key]


def fp32_roof(flops_per_launch, launch_ms, dev):
    pk = pipe_peaks(dev)
    peak = pk["fp32_fma_tflops"]
    achieved = flops_per_launch / (launch_ms * 1e-3) / 1e12
    return {"bound": "alu", "achieved": round(achieved, 3), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "peak_source": "measured FP32 FMA rate (" + pk["source"] + ")"}


# ---- clocks sampled during the timed region (NVML, polled from a thread) -------------------------

class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = torch.cuda.get_device_properties(device_index).uuid
            self._h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if str(uuid) in u:
                    self._h = h
            if self._h is None:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - depends on the box
            self._nv = None
            self.error = str(e)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "")}
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ---- distributed plumbing -------------------------------------------------------------------------

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def rank_seed(wl, rank: int, salt: int = 0) -> int:
    """Seed of rank `rank`'s batch: every rank draws its own batch of the workload (weak
    scaling over independent (b, h) units; no data crosses ranks)."""
    return inputs.SEED_BASE + wl.cid + 1000 * rank + salt


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---- workload set-up ---------------------------------------------------------------------------

def algorithmic_bytes(wl, B, T, H, dt_bytes, s0: bool, s_out: bool, snaps: int, epilogue: bool,
                      raw: bool = False) -> int:
    """Bytes one forward must move at minimum: inputs once, y once, states once (raw inputs:
    five token vectors instead of six, plus the per-head k_k and k_a)."""
    N = wl.N
    per_tok = (5 if raw else 6) * N * dt_bytes + N * 4
    st = N * N * 4
    extra = (H * N * 3 * 4 if epilogue else 0) + (H * N * 2 * 4 if raw else 0)
    return B * T * H * per_tok + B * H * st * (int(s0) + int(s_out) + snaps) + extra


def run_gpu(args, world, rank, local):
    from linear_rnn_sequence_rwkv_b200 import wkv7
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    spec = WORKLOADS[args.workload]
    wl = inputs.WORKLOADS[spec["cid"]]
    if args.head_size != wl.N:   # same channel count per token, wider heads
        wl = dataclasses.replace(wl, N=args.head_size, H=max(1, wl.H * wl.N // args.head_size),
                                 name=f"{wl.name} as N={args.head_size}")
    steps = args.steps if args.steps is not None else spec["default_steps"]
    warmup = args.warmup
    peaks, peak_kind = _peaks()
    stream = torch.cuda.current_stream(dev)
    decode = args.workload == "decode"
    raw = args.inputs == "raw"
    snap_every = wl.snap_every

    # independent batches per rank (seed offset), rotating input sets larger than L2
    seed0 = rank_seed(wl, rank)
    if decode:
        # raw: the fused step (raw inputs pre-processed in the load, group_norm + bonus epilogue)
        n_tok = 128
        if raw:
            d = inputs.make_raw_inputs(dataclasses.replace(wl, epilogue=True), device=str(dev), seed=seed0, T=n_tok)
        else:
            d = inputs.make_inputs(wl, device=str(dev), seed=seed0, T=n_tok)
        B, H, N = wl.B, wl.H, wl.N
        steps_in = {n: d[n].transpose(0, 1).contiguous() for n in (RAW_NAMES if raw else NAMES)}   # [128, B, H, N]
        S = torch.zeros(B, H, N, N, device=dev)
        y = torch.empty(B, H, N, device=dev)
        T = 1
        n_sets = 1

        def step(i):
            j = i % n_tok
            if raw:
                wkv7.decode_step_raw(*(steps_in[n][j] for n in RAW_NAMES), d["k_k"], S, k_a=d["k_a"], y=y,
                                     ln_w=d["ln_w"], ln_b=d["ln_b"], r_k=d["r_k"])
            else:
                wkv7.decode_step(*(steps_in[n][j] for n in NAMES), S, y=y)
        n_in = 5 if raw else 6
        bytes_per_launch = B * H * (n_in * N * 2 + N * 4 + 2 * N * N * 4) + (H * N * 5 * 4 if raw else 0)
        launches_per_step = 1
        epilogue = raw
    else:
        B, T, H, N = wl.B, wl.T, wl.H, wl.N
        n_vec = 5 if raw else 6
        set_bytes = B * T * H * N * (n_vec * 2)
        n_sets = max(1, min(8, math.ceil(2 * L2_BYTES / set_bytes)))
        make = inputs.make_raw_inputs if raw else inputs.make_inputs
        sets = [make(wl, device=str(dev), seed=seed0 + 17 * i) for i in range(n_sets)]
        y = torch.empty(B, T, H, N, device=dev)
        S_T = torch.empty(B, H, N, N, device=dev)
        snaps = torch.empty(B, T // snap_every, H, N, N, device=dev) if snap_every else None
        epilogue = wl.epilogue
        ws_need = wkv7.workspace_bytes(B, T, H, N, torch.bfloat16, algo=args.algo, chunk=args.chunk,
                                       snap_every=snap_every)
        ws = torch.empty(max(ws_need, 1), dtype=torch.uint8, device=dev)

        def step(i):
            s = sets[i % n_sets]
            ep = dict(ln_w=s["ln_w"], ln_b=s["ln_b"], r_k=s["r_k"]) if epilogue else {}
            if raw:
                wkv7.forward_raw(*(s[n] for n in RAW_NAMES), s["k_k"], s["k_a"], s["S0"], algo=args.algo,
                                 chunk=args.chunk, y=y, S_T=S_T, snap_every=snap_every, snapshots=snaps,
                                 workspace=ws, **ep)
            else:
                wkv7.forward(*(s[n] for n in NAMES), s["S0"], algo=args.algo, chunk=args.chunk, y=y, S_T=S_T,
                             snap_every=snap_every, snapshots=snaps, workspace=ws, **ep)
        bytes_per_launch = algorithmic_bytes(wl, B, T, H, 2, sets[0]["S0"] is not None, True,
                                             T // snap_every if snap_every else 0, epilogue, raw)
        launches_per_step = 1 + (1 if epilogue and _path_name(args) == "seq" else 0)

    units_per_step = B * T * H
    ctas_per_head = None
    if not decode:
        ep = dict(ln_w=sets[0]["ln_w"], ln_b=sets[0]["ln_b"], r_k=sets[0]["r_k"]) if epilogue else {}
        plan_algo, ctas_per_head, launches_per_step = wkv7.plan(
            B, T, H, N, torch.bfloat16, launches=True, algo=args.algo, chunk=args.chunk, snap_every=snap_every, **ep)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(dev)

    # decode: the 128 token steps are captured once in a CUDA graph and replayed (a step is
    # launch-bound at this size); each replay is timed and divided by its 128 steps
    graph = None
    if decode:
        graph = _decode_graph(lambda: [step(j) for j in range(n_tok)], dev)
        if graph is not None:
            reps = max(1, -(-steps // n_tok))
            steps = reps * n_tok
            graph.replay()   # warm-up replay (128 steps)
            torch.cuda.synchronize(dev)

    # timed region: K steps, one event pair per step (per replay for decode) on the launching stream
    n_ev = steps if graph is None else steps // n_tok
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n_ev + 1)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        ev[0].record(stream)
        for i in range(n_ev):
            if graph is None:
                step(warmup + i)
            else:
                graph.replay()
            ev[i + 1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    per_step_ms = [ev[i].elapsed_time(ev[i + 1]) / (1 if graph is None else n_tok) for i in range(n_ev)]
    total_ms = ev[0].elapsed_time(ev[n_ev])
    total_ms = max_over_ranks(total_ms, world, dev)
    value = units_per_step * steps * world / (total_ms * 1e-3) / 1e6
    launch_ms = statistics.mean(per_step_ms)

    # roofline of the dominant kernel
    hbm_peak = float(peaks["hbm_gbs"])
    achieved_gbs = bytes_per_launch / (launch_ms * 1e-3) / 1e9
    flops_per_launch = 9 * N * N * units_per_step   # 9 N^2 per token-head: the exact recurrence
    wtag = args.workload if N == 64 else f"{args.workload}-N{N}"   # profiles are per head size
    path = "decode" if decode else plan_algo
    if path == "seq":
        roof = fp32_roof(flops_per_launch, launch_ms, dev)
        roof.update({"traffic": measured_traffic("seq_kernel", wtag, raw), "kernel": "seq_kernel",
                     "hbm_gbs": round(achieved_gbs, 1), "hbm_frac": round(achieved_gbs / hbm_peak, 4)})
    else:
        roof = {"bound": "hbm", "achieved": round(achieved_gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved_gbs / hbm_peak, 4), "peak_source": f"{peak_kind} hbm_gbs",
                "traffic": measured_traffic("decode_kernel" if decode else "chunk_kernel", wtag, raw),
                "kernel": "decode_kernel" if decode else "chunk_kernel",
                "recurrence_tflops": round(flops_per_launch / (launch_ms * 1e-3) / 1e12, 3)}
    roof["algorithmic_bytes_per_launch"] = bytes_per_launch

    # end to end through the public API with pinned host buffers (copies inside the timed region)
    e2e = None
    if not decode and not getattr(args, "no_e2e", False):
        e2e = run_e2e(args, wl, dev, stream, B, T, H, N, seed0, epilogue, snap_every, warmup, steps, world, raw)

    out = {
        "metric": METRIC.replace("N=64", f"N={N}"), "value": round(value, 3), "unit": UNIT, "n_gpus": world, "steps": steps,
        "warmup": warmup, "ms_per_step": round(total_ms / steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32" if path in ("seq", "decode") else "tf32+f32",
        "data": "synthetic (seeded torch Philox; shapes and value ranges of the RWKV-7 pages' workloads)",
        "config": {"workload": f"{args.workload}: {wl.name}", "B": B, "T": T, "H": H, "N": N,
                   "input_dtype": "bf16", "path": path, "chunk": args.chunk or None,
                   "inputs": ("raw: decay/rate logits and the key before its update, pre-processing fused"
                              if raw else "prepared: w, a, kk, k~"),
                   "ctas_per_head": ctas_per_head,
                   "global_batch": B * world, "seq_len": T, "parallelism": f"dp{world} (independent (b,h) units)",
                   "l2": (f"{n_sets} rotating input sets, {n_sets * set_bytes / 1e6:.0f} MB > 126 MB L2"
                          if not decode else "fp32 state 168 MB > 126 MB L2, 128 rotating token inputs"),
                   "timing": ("CUDA graph of the 128 decode steps, replay time / 128" if graph is not None
                              else "one event pair per step")},
        "roofline": roof,
        "pipe_peaks": pipe_peaks(dev),
        "e2e": e2e,
        "gpu_launches": steps * launches_per_step,
        "clocks": clocks.summary(),
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, decode)
    if (args.workload == "prefill-1.5b" and not args.no_extras and not raw and N == 64 and args.algo == "auto"
            and not args.chunk):
        out["decode"] = run_decode_record(args, world, rank, local)
        out["chunk_sweep"] = run_chunk_sweep(args, world, rank, local, steps)
    return out


def _sub_args(args, **over):
    d = dict(vars(args))
    d.update(no_cpu_baseline=True, no_extras=True, no_e2e=True)
    d.update(over)
    return argparse.Namespace(**d)


def run_decode_record(args, world, rank, local):
    """The decode half of the metric on its own workload (B256 H40, fp32 state in HBM, 128 steps
    per CUDA graph replay), measured in the same run as the prefill line."""
    d = run_gpu(_sub_args(args, workload="decode", steps=256), world, rank, local)
    keep = ("value", "unit", "ms_per_step", "steps", "warmup", "dtype", "config", "roofline", "gpu_launches", "clocks")
    rec = {k: d[k] for k in keep}
    # the same steps from raw inputs with the epilogue fused (wkv7_decode_step_raw)
    f = run_gpu(_sub_args(args, workload="decode", steps=256, inputs="raw"), world, rank, local)
    rec["raw_inputs_with_epilogue"] = {k: f[k] for k in ("value", "ms_per_step", "roofline", "gpu_launches", "clocks")}
    return rec


def run_chunk_sweep(args, world, rank, local, steps):
    """The prefill workload at the three chunk lengths the option takes (16, 32, 64): the path
    the library dispatches each to, and its time."""
    rows = []
    for c in (16, 32, 64):
        d = run_gpu(_sub_args(args, chunk=c, steps=max(3, min(steps, 10))), world, rank, local)
        rows.append({"chunk": c, "path": d["config"]["path"], "ctas_per_head": d["config"]["ctas_per_head"],
                     "ms_per_step": d["ms_per_step"], "value": d["value"], "unit": d["unit"],
                     "bound": d["roofline"]["bound"], "frac": d["roofline"]["frac"],
                     "hbm_frac": d["roofline"].get("hbm_frac", d["roofline"]["frac"]), "clocks": d["clocks"]})
    return rows


BWD_FLOPS_PER_UNIT = 21 * 64 * 64   # gradient arithmetic per token-head at N = 64 (21 N^2; recomputation not counted)


def run_backward(args, world, rank, local):
    """Backward pass on the prefill workload: one step = wkv7.backward over the batch, with
    the snapshots (every 64 tokens) of a forward that kept its states, dy and dS_T resident."""
    from linear_rnn_sequence_rwkv_b200 import wkv7
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    spec = WORKLOADS[args.workload]
    wl = inputs.WORKLOADS[spec["cid"]]
    if args.head_size != wl.N:   # same channel count per token, wider heads
        wl = dataclasses.replace(wl, N=args.head_size, H=max(1, wl.H * wl.N // args.head_size),
                                 name=f"{wl.name} as N={args.head_size}")
    steps = args.steps if args.steps is not None else max(5, spec["default_steps"] // 10)
    warmup = args.warmup
    peaks, _ = _peaks()
    stream = torch.cuda.current_stream(dev)
    B, T, H, N = wl.B, wl.T, wl.H, wl.N
    snap = 64
    seed0 = rank_seed(wl, rank, 77)
    set_bytes = B * T * H * N * (6 * 2 + 4) + B * (T // snap) * H * N * N * 4
    n_sets = max(1, min(4, math.ceil(2 * L2_BYTES / set_bytes)))
    sets = []
    for i in range(n_sets):
        d = inputs.make_inputs(wl, device=str(dev), seed=seed0 + 17 * i)
        g = torch.Generator(device=dev).manual_seed(seed0 + 17 * i + 1)
        d["dy"] = torch.randn(B, T, H, N, device=dev, generator=g)
        d["dS_T"] = 0.1 * torch.randn(B, H, N, N, device=dev, generator=g)
        d["y"], _, d["snaps"] = wkv7.forward(*(d[n] for n in NAMES), d["S0"], snap_every=snap)
        sets.append(d)
    grads = {n: torch.empty(B, T, H, N, device=dev) for n in wkv7.GRAD_NAMES}
    dS0 = torch.empty(B, H, N, N, device=dev)
    ws = torch.empty(wkv7.backward_workspace_bytes(B, T, H, N, snap), dtype=torch.uint8, device=dev)

    def step(i):
        s = sets[i % n_sets]
        wkv7.backward(*(s[n] for n in NAMES), s["dy"], s["S0"], s["dS_T"], snapshots=s["snaps"],
                      snap_every=snap, grads=grads, dS0=dS0, workspace=ws)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        ev[0].record(stream)
        for i in range(steps):
            step(warmup + i)
            ev[i + 1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    per_step_ms = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[steps]), world, dev)
    units = B * T * H
    value = units * steps * world / (total_ms * 1e-3) / 1e6
    launch_ms = statistics.mean(per_step_ms)
    hbm_bytes = units * (6 * N * 2 + N * 4 + 6 * N * 4) + B * H * N * N * 4 * (3 + T // snap)
    flops_per_unit = BWD_FLOPS_PER_UNIT * (N // 64) ** 2
    roof = fp32_roof(flops_per_unit * units, launch_ms, dev)
    roof.update({"traffic": measured_traffic("bwd_kernel", args.workload) if N == 64 else None, "kernel": "bwd_kernel",
            "flops_per_unit": flops_per_unit, "algorithmic_bytes_per_launch": hbm_bytes,
            "hbm_gbs": round(hbm_bytes / (launch_ms * 1e-3) / 1e9, 1),
            "hbm_frac": round(hbm_bytes / (launch_ms * 1e-3) / 1e9 / float(peaks["hbm_gbs"]), 4)})

    # end to end: host inputs (pinned) -> device, backward, gradients -> host, all timed
    hd = {n: (v.to("cpu").pin_memory() if isinstance(v, torch.Tensor) else v) for n, v in sets[0].items()}
    host_out = {n: torch.empty(B, T, H, N).pin_memory() for n in wkv7.GRAD_NAMES}
    host_ds0 = torch.empty(B, H, N, N).pin_memory()
    in_names = NAMES + ("S0", "dy", "dS_T", "snaps")
    h2d = sum(hd[n].numel() * hd[n].element_size() for n in in_names if hd[n] is not None)
    d2h = sum(t.numel() * 4 for t in host_out.values()) + host_ds0.numel() * 4

    def once():
        dv = {n: (None if hd[n] is None else hd[n].to(dev, non_blocking=True)) for n in in_names}
        out = wkv7.backward(*(dv[n] for n in NAMES), dv["dy"], dv["S0"], dv["dS_T"], snapshots=dv["snaps"],
                            snap_every=snap, workspace=ws)
        for n in wkv7.GRAD_NAMES:
            host_out[n].copy_(out[n], non_blocking=True)
        host_ds0.copy_(out["dS0"], non_blocking=True)

    once()
    torch.cuda.synchronize(dev)
    e_steps = max(1, min(steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    e0.record(stream)
    for _ in range(e_steps):
        once()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e = {"value": round(units * e_steps * world / (e_ms * 1e-3) / 1e6, 3), "unit": UNIT,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
           "ms_per_step": round(e_ms / e_steps, 4)}
    epi = run_epilogue_backward_record(sets, wl, steps, warmup, world, dev, stream, peaks)
    out = {
        "metric": METRIC.replace("(prefill, decode)", "(backward)").replace("N=64", f"N={N}"), "value": round(value, 3),
        "unit": UNIT,
        "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": round(total_ms / steps, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (seeded torch Philox; shapes and value ranges of the RWKV-7 pages' workloads)",
        "config": {"workload": f"{args.workload} backward: {wl.name}", "B": B, "T": T, "H": H, "N": N,
                   "input_dtype": "bf16", "path": "backward", "snap_every": snap,
                   "global_batch": B * world, "seq_len": T, "parallelism": f"dp{world} (independent (b,h) units)",
                   "l2": f"{n_sets} rotating input sets, {n_sets * set_bytes / 1e6:.0f} MB"},
        "roofline": roof, "e2e": e2e, "gpu_launches": steps, "clocks": clocks.summary(),
        "epilogue_backward": epi,
    }
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_backward(wl)
    return out


def run_epilogue_backward_record(sets, wl, steps, warmup, world, dev, stream, peaks):
    """The epilogue's backward (wkv7.epilogue_backward) over the same batch, the forward's
    readout as y and dy as the gradient arriving at the epilogue: a record of the backward line.
    HBM-bound: per token-head it reads y and dout (fp32) and r, k, v, and writes dy, dr, dk, dv
    (fp32)."""
    from linear_rnn_sequence_rwkv_b200 import wkv7
    B, T, H, N = wl.B, wl.T, wl.H, wl.N
    g = torch.Generator(device=dev).manual_seed(4242)
    ln_w = 1.0 + 0.1 * torch.randn(H, N, device=dev, generator=g)
    ln_b = 0.1 * torch.randn(H, N, device=dev, generator=g)
    r_k = 0.5 * torch.randn(H, N, device=dev, generator=g)
    grads = {n: torch.empty((B, T, H, N) if n in ("dy", "dr", "dk", "dv") else (H, N), device=dev)
             for n in wkv7.EPILOGUE_GRAD_NAMES}
    ws = torch.empty(max(1, int(wkv7.load().wkv7_epilogue_backward_workspace_bytes(B, T, H, N))), dtype=torch.uint8,
                     device=dev)

    def step(i):
        s = sets[i % len(sets)]
        wkv7.epilogue_backward(s["y"], s["r"], s["k"], s["v"], ln_w, ln_b, r_k, s["dy"], grads=grads, workspace=ws)

    for i in range(max(3, warmup)):
        step(i)
    torch.cuda.synchronize(dev)
    n = max(steps, 20)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    with ClockSampler(dev.index) as clocks:
        e0.record(stream)
        for i in range(n):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / n
    units = B * T * H
    elem = sets[0]["r"].element_size()
    nbytes = units * N * (4 + 3 * elem + 4 + 4 * 4)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"ms_per_step": round(ms, 5), "value": round(units * world / (ms * 1e-3) / 1e6, 3), "unit": UNIT,
            "steps": n, "gpu_launches_per_step": 2,
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                         "frac": round(gbs / float(peaks["hbm_gbs"]), 4), "traffic": None,
                         "kernel": "epilogue_bwd_kernel", "algorithmic_bytes_per_launch": nbytes},
            "clocks": clocks.summary()}


def run_layer(args, world, rank, local):
    """Full time-mixing layer (a layer after the first: value residual on) with synthetic
    weights over the prefill workload's batch: one step = wkv7.layer_forward over the batch."""
    from linear_rnn_sequence_rwkv_b200 import wkv7
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    spec = WORKLOADS[args.workload]
    wl = inputs.WORKLOADS[spec["cid"]]
    steps = args.steps if args.steps is not None else max(5, spec["default_steps"] // 4)
    warmup = args.warmup
    B, T, H, N = wl.B, wl.T, wl.H, wl.N
    C = H * N
    d = inputs.make_layer(B, T, H, N, seed=rank_seed(wl, rank, 55), device=str(dev), dtype="bf16")
    S = d["S0"].clone()
    out = torch.empty(B, T, C, device=dev)
    last = torch.empty(B, C, device=dev, dtype=torch.bfloat16)
    ws = torch.empty(wkv7.layer_workspace_bytes(B, T, d, H, N), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i):
        S.copy_(d["S0"])
        wkv7.layer_forward(d["x"], d, H, N=N, last_x=d["last_x"], v0=d["v0"], S=S, out=out, last_x_out=last,
                           workspace=ws)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(dev.index) as clocks:
        ev[0].record(stream)
        for i in range(steps):
            step(warmup + i)
            ev[i + 1].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    total_ms = max_over_ranks(ev[0].elapsed_time(ev[steps]), world, dev)
    ms = total_ms / steps
    units = B * T * H
    rk = inputs.LAYER_RANKS
    rec_launches = wkv7.plan(B, T, H, N, torch.bfloat16, launches=True, ln_w=d["ln_w"], ln_b=d["ln_b"],
                             r_k=d["r_k"])[2]
    gemm_flops = 2 * B * T * C * (4 * C + 2 * (rk["d_w"] + rk["d_a"] + rk["d_v"] + rk["d_g"]))
    peaks, peak_kind = _peaks()
    tc_peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops", 1590.0)))
    achieved = gemm_flops / (ms * 1e-3) / 1e12
    return {
        "metric": METRIC.replace("(prefill, decode)", "(time-mixing layer)"), "value": round(units * steps * world /
                                                                                             (total_ms * 1e-3) / 1e6, 3),
        "unit": UNIT, "n_gpus": world, "steps": steps, "warmup": warmup, "ms_per_step": round(ms, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16+f32",
        "data": "synthetic weights and activations (seeded torch Philox)",
        "config": {"workload": f"{args.workload} layer: {wl.name}, C={C}, low-rank {rk}", "B": B, "T": T, "H": H,
                   "N": N, "path": "layer", "global_batch": B * world, "seq_len": T,
                   "parallelism": f"dp{world} (independent sequences)"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": round(achieved / tc_peak, 4), "traffic": None,
                     "kernel": "whole layer step (GEMM flops over the step time; the recurrence runs inside it)",
                     "peak_source": f"{peak_kind} bf16 (sustained)", "gemm_flops_per_step": gemm_flops},
        "e2e": None, "clocks": clocks.summary(),
        # this library's kernels per step: the low-rank factor copies, the grouped GEMM over the
        # mixed x (7 products), the grouped second factors (4), the recurrence, the output
        # projection (gate fused into its operand), the last-token copy
        "gpu_launches": steps * (1 + 1 + 1 + rec_launches + 1 + 1),
    }


def cpu_baseline_backward(wl, budget_s: float = 12.0):
    """The fp64 oracle's backward (numpy, vectorised over (b, h)) on a bounded sample."""
    from oracle import reference
    B, T, H = 1, min(wl.T, 1024), wl.H
    d = inputs.make_inputs(wl, B=B, T=T, H=H)
    g = torch.Generator().manual_seed(5)
    dy = torch.randn(B, T, H, wl.N, generator=g)
    dS_T = 0.1 * torch.randn(B, H, wl.N, wl.N, generator=g)
    reps, t0 = 0, time.perf_counter()
    while True:
        reference.wkv7_backward(*(d[n] for n in NAMES), d["S0"], dy, dS_T)
        reps += 1
        el = time.perf_counter() - t0
        if el > budget_s / 4 or reps >= 50:
            break
    return {"value": round(B * T * H * reps / el / 1e6, 5), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"B{B} T{T} H{H} of the workload (numpy fp64 backward); {reps} run(s), {el:.1f} s wall"}


def _decode_graph(body, dev):
    """CUDA graph of `body` (the 128 decode steps) captured on a side stream, or None when the
    capture is refused (the eager loop is timed instead)."""
    try:
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                body()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        return g
    except Exception as e:   # pragma: no cover - depends on the driver
        print(f"decode graph capture refused ({e}); timing the eager loop", file=sys.stderr)
        torch.cuda.synchronize(dev)
        return None


def _path_name(args):
    """Kernel the library dispatches to for the bf16 workloads (AUTO picks the chunked one)."""
    return {"auto": "chunk", "seq": "seq", "chunk": "chunk", "split": "chunk"}[args.algo]


def run_e2e(args, wl, dev, stream, B, T, H, N, seed, epilogue, snap_every, warmup, steps, world, raw=False):
    """Same metric through the C ABI's host-buffer entry (wkv7_forward_host) with pinned HOST
    tensors: every step's host-to-device copies of the inputs, the kernels and the
    device-to-host copies of y and S_T are inside the timed region. The raw-input workload has
    no host-buffer entry; it copies through torch around wkv7_forward_raw instead."""
    from linear_rnn_sequence_rwkv_b200 import wkv7
    d = (inputs.make_raw_inputs if raw else inputs.make_inputs)(wl, device="cpu", seed=seed + 999)
    host = {n: (v.pin_memory() if isinstance(v, torch.Tensor) else v) for n, v in d.items()}
    h2d = sum(host[n].numel() * host[n].element_size() for n in (RAW_NAMES if raw else NAMES))
    h2d += 0 if host["S0"] is None else host["S0"].numel() * 4
    if epilogue:
        h2d += 3 * H * N * 4
    if raw:
        h2d += 2 * H * N * 4
    d2h = B * T * H * N * 4 + B * H * N * N * 4 + (B * (T // snap_every) * H * N * N * 4 if snap_every else 0)
    y_h = torch.empty(B, T, H, N).pin_memory()
    S_h = torch.empty(B, H, N, N).pin_memory()
    sn_h = torch.empty(B, T // snap_every, H, N, N).pin_memory() if snap_every else None
    ep = {n: host[n] for n in ("ln_w", "ln_b", "r_k")} if epilogue else {}
    ws = None
    if not raw:
        ws = torch.empty(wkv7.forward_host_workspace_bytes(B, T, H, N, torch.bfloat16, snap_every=snap_every,
                                                           epilogue=epilogue, algo=args.algo, chunk=args.chunk),
                         dtype=torch.uint8, device=dev)

    def once():
        if raw:   # copy in, run, copy out, all on this stream
            dv = {n: (None if host[n] is None else host[n].to(dev, non_blocking=True))
                  for n in RAW_NAMES + ("k_k", "k_a", "S0")}
            dep = {n: v.to(dev, non_blocking=True) for n, v in ep.items()}
            y, S, _ = wkv7.forward_raw(*(dv[n] for n in RAW_NAMES), dv["k_k"], dv["k_a"], dv["S0"], algo=args.algo,
                                       chunk=args.chunk, snap_every=snap_every, **dep)
            y_h.copy_(y, non_blocking=True)
            S_h.copy_(S, non_blocking=True)
            return
        wkv7.forward_host(*(host[n] for n in NAMES), host["S0"], y_h, S_h, ws, algo=args.algo, chunk=args.chunk,
                          snap_every=snap_every, snapshots=sn_h, **ep)

    for _ in range(max(1, min(warmup, 3))):
        once()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        once()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    return {"value": round(B * T * H * steps * world / (ms * 1e-3) / 1e6, 3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 4),
            "api": "wkv7_forward_raw with torch copies" if raw else "wkv7_forward_host (C ABI, pinned host buffers)"}


def cpu_baseline(wl, decode: bool, budget_s: float = 12.0):
    """The fp64 oracle (plain C, threads over (b, h)) on a bounded sample of the workload."""
    import numpy as np
    from oracle import native
    if decode:
        B, T, H = 16, 1, wl.H
        d = inputs.make_inputs(wl, B=B, T=T, H=H, s0="normal")
        sample = f"{B * H} heads x 1 decode step (S0 ~ N(0, 0.1^2)), repeated"
    else:
        T = min(wl.T, 4096)
        H = wl.H
        B = max(1, min(wl.B, 2 if wl.T > 2048 else wl.B))
        d = inputs.make_inputs(wl, B=B, T=T, H=H)
        sample = f"B{B} T{T} H{H} of the workload's first batch rows"
    arrs = {n: np.ascontiguousarray(d[n].to(torch.float64).numpy()) for n in NAMES}
    s0 = None if d["S0"] is None else np.ascontiguousarray(d["S0"].to(torch.float64).numpy())
    units = B * T * H
    reps, t0 = 0, time.perf_counter()
    while True:
        native.forward(*(arrs[n] for n in NAMES), s0)
        reps += 1
        el = time.perf_counter() - t0
        if el > budget_s / 4 or reps >= 200:
            break
    return {"value": round(units * reps / el / 1e6, 5), "unit": UNIT, "cores": native.host_threads(),
            "kind": "oracle", "sample": f"{sample}; {reps} run(s), {el:.1f} s wall"}


def run_reference(args, world, rank):
    """Reference arm: the fp64 CPU oracle, as it stands, on host cores (rank 0 only)."""
    if rank != 0:
        return None
    spec = WORKLOADS[args.workload]
    wl = inputs.WORKLOADS[spec["cid"]]
    steps = args.steps if args.steps is not None else 3
    decode = args.workload == "decode"
    import numpy as np
    from oracle import native
    if decode:
        B, T, H = 32, 1, wl.H
    else:
        B, T, H = min(wl.B, 2), min(wl.T, 1024), wl.H
    d = inputs.make_inputs(wl, B=B, T=T, H=H)
    arrs = {n: np.ascontiguousarray(d[n].to(torch.float64).numpy()) for n in NAMES}
    s0 = None if d["S0"] is None else np.ascontiguousarray(d["S0"].to(torch.float64).numpy())
    for _ in range(args.warmup):
        native.forward(*(arrs[n] for n in NAMES), s0)
    t0 = time.perf_counter()
    for _ in range(steps):
        native.forward(*(arrs[n] for n in NAMES), s0)
    el = time.perf_counter() - t0
    value = B * T * H * steps / el / 1e6
    cores = native.host_threads()
    sample = f"B{B} T{T} H{H} sample of {wl.name} per step"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": round(el / steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": f"{args.workload}: {wl.name}", "sample": sample},
            "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="prefill-1.5b")
    ap.add_argument("--no-extras", action="store_true",
                    help="prefill-1.5b: leave out the decode and chunk-sweep records")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--algo", choices=["auto", "seq", "chunk", "split"], default="auto")
    ap.add_argument("--chunk", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--head-size", type=int, choices=[64, 128], default=64,
                    help="128: the same channels per token in heads of 128 (scan path)")
    ap.add_argument("--pass", dest="pass_", choices=["forward", "backward", "layer"], default="forward",
                    help="backward: gradients of every input from a forward's snapshots")
    ap.add_argument("--inputs", choices=["prepared", "raw"], default="prepared",
                    help="raw: decay/rate logits and the key before its update, pre-processing fused "
                         "(decode: with the epilogue too)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out))
        return 0

    world, rank, local = dist_setup()
    if world != args.gpus and rank == 0:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    try:
        if args.pass_ == "layer":
            out = run_layer(args, world, rank, local)
        elif args.pass_ == "backward":
            if args.workload == "decode" or args.inputs == "raw":
                raise SystemExit("--pass backward takes a prefill workload with prepared inputs")
            out = run_backward(args, world, rank, local)
        else:
            out = run_gpu(args, world, rank, local)
        if rank == 0:
            print(json.dumps(out))
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
