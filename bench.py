#!/usr/bin/env python
"""Benchmark of the DSpark draft MLA attention (forward + backward) on B200.

One step = one pass of the whole hot path over one batch: build the mask
descriptor, forward (O, LSE), backward (dQ, dK^C, dK^R, dV), all through the C
ABI. Default workload: B=2, S=8192, N=512, W=128, 64 heads, 192+64 / 256, bf16.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload ID]
                  [--impl reference] [--no-cpu-baseline] [--no-e2e] [--desc-timing]
                  [--part attention|draft-inputs|loss]

Prints one JSON line (rank 0). With N > 1 (torchrun) every rank processes its
own batch (batch sharding, weak scaling, no collective on the data path); the
time is the max over ranks and the value the rows of all ranks over that time.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload instead. ``--part draft-inputs`` times instead the step before the
attention: GPU anchor sampling and the draft block's inputs (ids, positions,
labels, predecessors, eval_mask) for the workload's batch shape, on one GPU;
``--part loss`` times the training loss over the workload's B * 5N draft steps
(V = 154880 synthetic bf16 student and teacher logits) with its gradient.
"""
import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from speculative_draft_mla_b200 import synth  # noqa: E402

METRIC = "query-head rows/sec fwd+bwd (bf16, 1 B200) and % of roofline"
UNIT = "rows/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 2 ** 20


# ---------------------------------------------------------------- work model
def algorithmic_work(wl, anchors, keep):
    """Algorithmic bytes and FLOPs of one forward and one backward.

    Bytes: every input element the method must read at least once and every
    output element it must write: Q, the K/V of context positions inside at
    least one window (union) and of the draft positions, O, LSE; the backward
    adds O, dO and LSE reads and writes all of dQ, dK^C, dK^R and dV.
    FLOPs: 2 per multiply-add over each (row, visible key) pair; forward
    d_c+d_r (scores) + d_v (PV); backward 3(d_c+d_r) + 2 d_v (scores, dP, dV,
    dQ, dK)."""
    e = 4 if wl.dtype == "f32" else 2
    an = anchors.numpy()
    kp = keep.numpy().astype(bool)
    dqk = wl.d_c + wl.d_r
    union = 0
    pairs = 0
    for b in range(wl.B):
        cov = np.zeros(wl.S + 1, np.int64)
        a = an[b][kp[b]]
        lo = np.maximum(0, a - wl.W + 1)
        np.add.at(cov, lo, 1)
        np.add.at(cov, a, -1)
        union += int((np.cumsum(cov)[:wl.S] > 0).sum())
        pairs += int((a - lo + 5).sum()) * 5
    R = 5 * wl.N
    rows = wl.B * wl.n_h * R
    per_pos = wl.n_h * (wl.d_c + wl.d_v) * e + wl.d_r * e
    kv = union * per_pos + wl.B * R * per_pos
    q = rows * dqk * e
    o = rows * wl.d_v * e
    lse = rows * 4
    fwd_bytes = q + kv + o + lse
    full_k = wl.B * wl.L * per_pos
    bwd_bytes = q + kv + o + o + lse + q + full_k
    fwd_flops = 2 * pairs * wl.n_h * (dqk + wl.d_v)
    bwd_flops = 2 * pairs * wl.n_h * (3 * dqk + 2 * wl.d_v)
    return dict(fwd_bytes=fwd_bytes, bwd_bytes=bwd_bytes, fwd_flops=fwd_flops, bwd_flops=bwd_flops,
                union_positions=union, rows=rows)


# The device sources each C-ABI call's kernels at the benchmark workload are
# built from (the host-side argument checks, the SIMT family, the no-workspace
# entry point and the host sampler play no part in a call's DRAM traffic).
_CALL_SOURCES = {
    "fwd": ("dspark_internal.cuh", "dspark_prep.cu", "dspark_tc_common.cuh", "dspark_tc_fwd.cu"),
    "bwd": ("dspark_internal.cuh", "dspark_prep.cu", "dspark_tc_common.cuh", "dspark_tc_bwd.cu"),
}


def sources_sha256(call):
    """sha256 over (basename, content) of the kernel sources one C-ABI call is built from."""
    import hashlib
    h = hashlib.sha256()
    for name in sorted(_CALL_SOURCES[call]):
        h.update(name.encode())
        with open(os.path.join(ROOT, "speculative_draft_mla_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(call):
    """DRAM bytes of one call (sum over its kernels) from the committed ncu capture of the
    benchmark workload, or None when that call's kernel sources have changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic_s8192_n512_b2.json")) as f:
            d = json.load(f)
        if sources_sha256(call) != d["sources_sha256"][call]:
            return None
        return sum(k["dram_read_bytes"] + k["dram_write_bytes"] for k in d["calls"][call])
    except Exception:
        return None


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), \
            "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# ------------------------------------------------------------ distribution
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def reduce_max(value, device, world):
    """Max of a float over ranks (identity on one rank)."""
    if world == 1:
        return value
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def aggregate(rows_per_rank, world, ms_max):
    """Whole-job throughput: rows of all ranks over the slowest rank's time."""
    return rows_per_rank * world / (ms_max / 1e3)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML on a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device, period=0.002):
        self.samples, self.reasons, self.period = [], set(), period
        self.max_mhz = None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            # match the CUDA device to its NVML handle by UUID (indices differ
            # under CUDA_VISIBLE_DEVICES)
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None
        self.t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv is not None:
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- oracle leg
def oracle_sample(wl, c, heads, with_bwd=True):
    """Run the fp64 oracle on the workload restricted to the first `heads`
    heads (all batch rows and blocks); returns (seconds, rows)."""
    import oracle
    oracle.build()
    q = c["q"][:, :heads].double().numpy()
    kc = c["kc"][:, :heads].double().numpy()
    kr = c["kr"].double().numpy()
    v = c["v"][:, :heads].double().numpy()
    do = c["dout"][:, :heads].double().numpy()
    an, kp = c["anchors"].numpy(), c["keep"].numpy()
    t0 = time.perf_counter()
    oracle.attn_fwd(q, kc, kr, v, an, kp, wl.S, wl.W, wl.rope_base)
    if with_bwd:
        oracle.attn_bwd(q, kc, kr, v, an, kp, do, wl.S, wl.W, wl.rope_base)
    return time.perf_counter() - t0, wl.B * 5 * wl.N * heads


def oracle_threads():
    n = os.environ.get("OMP_NUM_THREADS")
    return int(n) if n else (len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count())


def cpu_baseline(wl, c, target_s=10.0):
    t1, r1 = oracle_sample(wl, c, 1)
    heads = 1
    if t1 < target_s:
        # enough heads for ~target_s of work and for every thread to get a (batch, head) task
        heads = int(min(wl.n_h, max(-(-oracle_threads() // wl.B), round(target_s / max(t1, 1e-3)))))
    if heads > 1:
        t, r = oracle_sample(wl, c, heads)
    else:
        t, r = t1, r1
    return {"value": r / t, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": "workload %s restricted to the first %d of %d heads (all %d blocks x %d batch rows), "
                      "fp64 forward + backward, %.1f s" % (wl.name, heads, wl.n_h, wl.N, wl.B, t)}


def run_reference(args, wl):
    world, rank, local = dist_env()
    if rank != 0:
        return
    c = synth.make_inputs(wl)
    t1, _ = oracle_sample(wl, c, 1)
    budget = 150.0 / max(1, args.steps + args.warmup)  # whole run within a few minutes
    heads = int(min(wl.n_h, max(1, budget // max(t1, 1e-3))))
    times, rows = [], 0
    for i in range(args.warmup + args.steps):
        t, rows = oracle_sample(wl, c, heads)
        if i >= args.warmup:
            times.append(t)
    sec = sum(times) / len(times)
    value = rows / sec
    sample = "workload %s restricted to the first %d of %d heads, fp64 forward + backward per step" % (
        wl.name, heads, wl.n_h)
    out = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": config_of(wl),
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_draft_inputs(args, wl, capi, device):
    """Anchor sampling + draft-block inputs for the workload's (B, S, N): one
    step = dspark_sample_anchors_gpu + dspark_build_draft_inputs. Algorithmic
    bytes: the loss_mask, the six input ids a block reads (x_A .. x_{A+5}), the
    anchors and keep written and the five [B, 5N] outputs."""
    from oracle import draft_inputs as odi
    # the workload's loss mask (the first draw of its input generator)
    lm_h = synth._draw_loss_mask(wl, torch.Generator().manual_seed(1000 + wl.id)).to(torch.uint8)
    g = torch.Generator().manual_seed(77)
    ids_h = torch.randint(0, 154880, (wl.B, wl.S), generator=g, dtype=torch.int32)
    lm, ids = lm_h.to(device), ids_h.to(device)
    stream = torch.cuda.current_stream(device)

    def step(i):
        an, kp = capi.sample_anchors_gpu(lm, wl.N, 1000 + i)
        return capi.build_draft_inputs(ids, lm, an, kp)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device) as clk:
        torch.cuda.synchronize()
        n0 = capi.launch_counter()
        start.record(stream)
        for i in range(args.steps):
            step(args.warmup + i)
        end.record(stream)
        torch.cuda.synchronize()
        n1 = capi.launch_counter()
    ms = start.elapsed_time(end) / args.steps
    rows = wl.B * 5 * wl.N
    nbytes = wl.B * wl.S + wl.B * wl.N * (6 * 4 + 4 + 1) + rows * (4 * 4 + 1)
    hbm, _, _, src = measured_peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    t0 = time.perf_counter()
    an_o, kp_o = odi.sample_anchors(lm_h.numpy(), wl.N, 1000)
    odi.build_draft_inputs(ids_h.numpy(), lm_h.numpy(), an_o, kp_o)
    cpu_s = time.perf_counter() - t0
    out = {"metric": "draft rows/sec (anchor sampling + draft-block inputs, 1 B200)", "value": rows / (ms * 1e-3),
           "unit": "rows/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int32", "data": "synthetic",
           "config": {"workload": wl.name, "B": wl.B, "S": wl.S, "N": wl.N, "part": "draft-inputs",
                      "l2": "inputs far smaller than L2 (the step is launch- and latency-bound)"},
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                        "traffic": None, "kernel": "k_sample_anchors + k_build_draft_inputs",
                        "peak_source": src + " (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else src,
                        "bytes": nbytes},
           "cpu_baseline": {"value": rows / cpu_s, "unit": "rows/s", "cores": 1, "kind": "oracle",
                            "sample": "the whole step once (oracle.draft_inputs, pure Python), %.2f s" % cpu_s},
           "clocks": clk.summary(), "gpu_launches": n1 - n0}
    print(json.dumps(out))


def run_loss(args, wl, capi, device):
    """The DSpark loss over the workload's B * 5N draft steps, V = 154880: one
    step = dspark_loss_fwd_bwd (loss means and the gradients with respect to
    the student logits and the confidence logits). Algorithmic bytes: student
    and teacher logits read once, the logit gradient written once, the per-step
    scalars (label, confidence logit, eval_mask, its gradient)."""
    from oracle import dspark_loss as odl
    V = 154880
    R = wl.B * 5 * wl.N
    g = torch.Generator(device=device).manual_seed(4242)
    L = (torch.randn(R, V, generator=g, device=device) * 3).to(torch.bfloat16)
    T = (torch.randn(R, V, generator=g, device=device) * 3).to(torch.bfloat16)
    y = torch.randint(0, V, (R,), generator=g, device=device, dtype=torch.int32)
    c = torch.randn(R, generator=g, device=device)
    m = (torch.rand(R, generator=g, device=device) < 0.9).to(torch.uint8)
    out, grad, gconf, ws = capi.dspark_loss(L, T, y, c, m)
    lib = capi.load()
    st = capi._stream(None, device)
    ptr = capi._ptr

    def step():
        capi._check(lib.dspark_loss_fwd_bwd(R, V, ptr(L), ptr(T), ptr(y), ptr(c), ptr(m), 1.0, 0.9, 1.0, ptr(out),
                                            ptr(grad), ptr(gconf), ptr(ws), ws.numel(), st), "dspark_loss_fwd_bwd")

    for _ in range(args.warmup):
        step()
    capi.get_error(ws)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device) as clk:
        torch.cuda.synchronize()
        n0 = capi.launch_counter()
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize()
        n1 = capi.launch_counter()
    capi.get_error(ws)
    ms = start.elapsed_time(end) / args.steps
    nbytes = 3 * R * V * 2 + R * (4 + 4 + 1 + 4 + 16)
    hbm, _, _, src = measured_peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    # the oracle (fp64 NumPy) on a few steps, scaled to steps/s
    k = 4
    t0 = time.perf_counter()
    odl.loss_fwd_bwd(L[:k].double().cpu().numpy(), T[:k].double().cpu().numpy(), y[:k].cpu().numpy(),
                     c[:k].double().cpu().numpy(), m[:k].cpu().numpy())
    cpu_s = time.perf_counter() - t0
    res = {"metric": "draft steps/sec (DSpark loss + gradient, V=154880, bf16, 1 B200)", "value": R / (ms * 1e-3),
           "unit": "steps/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
           "config": {"workload": wl.name, "rows": R, "V": V, "part": "loss",
                      "l2": "inputs larger than L2 (no flush between steps)"},
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                        "traffic": None, "kernel": "dspark_loss_fwd_bwd call (all its kernels)",
                        "peak_source": src + " (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else src,
                        "bytes": nbytes},
           "cpu_baseline": {"value": k / cpu_s, "unit": "steps/s", "cores": 1, "kind": "oracle",
                            "sample": "%d of the %d steps (fp64 NumPy, one thread), %.2f s" % (k, R, cpu_s)},
           "clocks": clk.summary(), "gpu_launches": n1 - n0}
    print(json.dumps(res))


def config_of(wl):
    return {"workload": wl.name, "B": wl.B, "S": wl.S, "N": wl.N, "W": wl.W, "n_h": wl.n_h, "d_c": wl.d_c,
            "d_r": wl.d_r, "d_v": wl.d_v, "rope_base": wl.rope_base, "rows": wl.rows,
            "l2": "inputs larger than L2 (no flush between steps)", "parallelism": "batch-sharded replicas, no collective"}


# --------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=3)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--part", default="attention", choices=["attention", "draft-inputs", "loss"])
    ap.add_argument("--desc-timing", action="store_true",
                    help="also time the descriptor build alone (an event between it and the forward call)")
    args = ap.parse_args()
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
        return
    args.warmup = max(args.warmup, 3)

    from speculative_draft_mla_b200 import build as dbuild
    from speculative_draft_mla_b200 import capi

    world, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    if rank == 0:
        dbuild.build()
    barrier(world)
    capi.load()
    if args.part != "attention":
        if rank == 0:
            (run_draft_inputs if args.part == "draft-inputs" else run_loss)(args, wl, capi, device)
        return

    host = synth.make_inputs(wl)
    in_bytes = sum(t.numel() * t.element_size() for t in host.values())
    # inputs well above L2 need no flush; smaller workloads get an L2 flush
    # (a 256 MiB write) before every step, kept outside the timed events
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=device) if in_bytes < 4 * L2_BYTES else None
    pinned = {k: v.pin_memory() for k, v in host.items() if k != "loss_mask"}
    dev = {k: v.to(device, non_blocking=True) for k, v in pinned.items()}
    dt = dev["q"].dtype
    prob = capi.problem_of(dev["q"], dev["kc"], dev["kr"], dev["v"], dev["anchors"], wl.S, wl.W, wl.rope_base)
    ws = capi.alloc_workspace(prob, device)
    o = torch.empty(dev["q"].shape[:3] + (wl.d_v,), dtype=dt, device=device)
    lse = torch.empty(dev["q"].shape[:3], dtype=torch.float32, device=device)
    grads = (torch.empty_like(dev["q"]), torch.empty_like(dev["kc"]), torch.empty_like(dev["kr"]),
             torch.empty_like(dev["v"]))
    stream = torch.cuda.current_stream(device)
    R = capi.FLAG_REUSE_DESCRIPTOR

    def step(ev=None, d=None, outs=None):
        d = dev if d is None else d
        o_, lse_, g_ = (o, lse, grads) if outs is None else outs
        if ev is not None:
            ev[0].record(stream)
        capi.build_descriptor(prob, d["anchors"], d["keep"], ws)
        if ev is not None and args.desc_timing:
            ev[3].record(stream)
        capi.attn_fwd(d["q"], d["kc"], d["kr"], d["v"], d["anchors"], d["keep"], wl.S, wl.W,
                      wl.rope_base, workspace=ws, flags=R, out=(o_, lse_))
        if ev is not None:
            ev[1].record(stream)
        capi.attn_bwd(d["q"], d["kc"], d["kr"], d["v"], d["anchors"], d["keep"], o_, lse_, d["dout"],
                      wl.S, wl.W, wl.rope_base, workspace=ws, flags=R, out=g_)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    capi.get_error(ws)
    torch.cuda.synchronize()

    # timed region: exactly K steps, events on the launching stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device) as clk:
        barrier(world)
        torch.cuda.synchronize()
        n0 = capi.launch_counter()
        start.record(stream)
        for i in range(args.steps):
            if flush is not None:
                flush.fill_(i & 0xFF)
            step(evs[i])
        end.record(stream)
        torch.cuda.synchronize()
        n1 = capi.launch_counter()
        barrier(world)
    capi.get_error(ws)
    if flush is None:
        ms = start.elapsed_time(end) / args.steps
    else:  # per-step events exclude the flushes
        ms = statistics.mean(e[0].elapsed_time(e[2]) for e in evs)
    ms_max = reduce_max(ms, device, world)
    fwd_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    # the descriptor build, inside fwd_ms (only on request: the extra event sits
    # between two launches that otherwise overlap)
    desc_ms = statistics.mean(e[0].elapsed_time(e[3]) for e in evs) if args.desc_timing else None
    value = aggregate(wl.rows, world, ms_max)

    work = algorithmic_work(wl, host["anchors"], host["keep"])
    hbm, tfl, tfl_sus, src = measured_peaks()
    dominant = "bwd" if bwd_ms >= fwd_ms else "fwd"
    dom_ms = bwd_ms if dominant == "bwd" else fwd_ms
    dom_bytes = work["%s_bytes" % dominant]
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    roof_ms = max((work["fwd_bytes"] + work["bwd_bytes"]) / (hbm * 1e9),
                  (work["fwd_flops"] + work["bwd_flops"]) / (tfl_sus * 1e12)) * 1e3
    roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "traffic": (measured_traffic(dominant) if wl.name == "s8192_n512_b2" else None),
                "kernel": "attn_%s call (all its kernels)" % dominant,
                "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % src if src == "measured" else "fallback",
                "step_frac": roof_ms / ms_max, "fwd_ms": fwd_ms, "bwd_ms": bwd_ms, "desc_ms": desc_ms,
                "fwd_bytes": work["fwd_bytes"], "bwd_bytes": work["bwd_bytes"],
                "fwd_flops": work["fwd_flops"], "bwd_flops": work["bwd_flops"]}

    # End to end through the public API with host buffers: every step copies
    # its inputs in from pinned host memory and all of its outputs back. As a
    # training loop would, the copies run on their own streams into and out of
    # two device buffer sets, so that step i+1's inputs arrive and step i's
    # outputs leave while a step computes.
    e2e = None
    if not args.no_e2e:
        ins = ("q", "kc", "kr", "v", "anchors", "keep", "dout")
        outs_host = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (o, lse) + grads]
        h2d = sum(pinned[k].numel() * pinned[k].element_size() for k in ins)
        d2h = sum(t.numel() * t.element_size() for t in outs_host)
        dsets = [dev, {k: (torch.empty_like(dev[k]) if k in ins else dev[k]) for k in dev}]
        osets = [(o, lse, grads), (torch.empty_like(o), torch.empty_like(lse), tuple(torch.empty_like(g) for g in grads))]
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        in_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(n, a=None, b=None):
            if a is not None:
                a.record(s_in)
            for i in range(n):
                j = i & 1
                if i >= 2:  # set j's inputs were last read by step i - 2
                    s_in.wait_event(comp_done[j])
                with torch.cuda.stream(s_in):
                    for k in ins:
                        dsets[j][k].copy_(pinned[k], non_blocking=True)
                in_done[j].record(s_in)
                stream.wait_event(in_done[j])
                if i >= 2:  # set j's outputs were last read by step i - 2's copy out
                    stream.wait_event(out_done[j])
                step(d=dsets[j], outs=(osets[j][0], osets[j][1], osets[j][2]))
                comp_done[j].record(stream)
                s_out.wait_event(comp_done[j])
                with torch.cuda.stream(s_out):
                    for hdst, src_t in zip(outs_host, (osets[j][0], osets[j][1]) + osets[j][2]):
                        hdst.copy_(src_t, non_blocking=True)
                out_done[j].record(s_out)
            if b is not None:
                b.record(s_out)

        e2e_run(2)
        torch.cuda.synchronize()
        ke = max(2, min(args.steps, 5))
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_run(ke, a, b)
        torch.cuda.synchronize()
        ems = reduce_max(a.elapsed_time(b) / ke, device, world)
        e2e = {"value": aggregate(wl.rows, world, ems), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": ems,
               "copies": "own streams, two device buffer sets: step i+1's inputs in and step i's outputs out "
                         "while a step computes"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, host)

    if rank == 0:
        out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "bf16" if dt == torch.bfloat16 else "f32", "data": "synthetic",
               "config": dict(config_of(wl), **({} if flush is None else {
                   "l2": "L2 flushed (256 MiB write) before every step, outside the per-step events"})),
               "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
               "clocks": clk.summary(), "gpu_launches": n1 - n0}
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
