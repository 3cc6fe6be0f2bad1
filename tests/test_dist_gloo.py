"""Host logic of the benchmark on CPU: the multi-process steps (gloo, world
size 2), the work model and the lookup of the stored DRAM traffic.

The attention shards by batch with no collective on the data path; the only
cross-rank steps are the barrier around the timed region, the max over ranks
of the step time and the whole-job aggregation. These run here on gloo.
"""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    w, r, lr = bench.dist_env()
    bench.barrier(w)
    ms = bench.reduce_max(10.0 + rank, torch.device("cpu"), w)
    val = bench.aggregate(327680, w, ms)
    q.put((r, w, ms, val))
    dist.destroy_process_group()


def test_two_rank_reduction():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 for r in res)
    assert all(r[2] == 11.0 for r in res)  # max over ranks
    assert all(abs(r[3] - 327680 * 2 / 0.011) < 1e-6 for r in res)


def test_work_model_counts():
    sys.path.insert(0, ROOT)
    import bench
    from speculative_draft_mla_b200 import synth
    wl = synth.WORKLOADS[1].with_(S=20, N=2, W=4, n_h=1, d_c=2, d_r=2, d_v=4)
    an = torch.tensor([[0, 10]], dtype=torch.int32)
    kp = torch.tensor([[1, 1]], dtype=torch.uint8)
    w = bench.algorithmic_work(wl, an, kp)
    # windows: A=0 -> none; A=10 -> [7, 10): 3 positions
    assert w["union_positions"] == 3
    pairs = 5 * (0 + 5) + 5 * (3 + 5)
    assert w["fwd_flops"] == 2 * pairs * (4 + 4)


def test_traffic_follows_each_calls_sources(tmp_path, monkeypatch):
    """A call's stored DRAM traffic is reported while the device sources it is
    built from are unchanged, whatever happens to host-only files or to the
    other call's kernel file."""
    import json
    import shutil
    sys.path.insert(0, ROOT)
    import bench
    csrc = tmp_path / "speculative_draft_mla_b200" / "csrc"
    shutil.copytree(os.path.join(ROOT, "speculative_draft_mla_b200", "csrc"), csrc)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    calls = {c: [{"kernel": "k", "dram_read_bytes": 100 * (i + 1), "dram_write_bytes": 7}]
             for i, c in enumerate(("fwd", "bwd"))}
    stored = {"sources_sha256": {c: bench.sources_sha256(c) for c in calls}, "calls": calls}
    (tmp_path / "profiles" / "dram_traffic_s8192_n512_b2.json").write_text(json.dumps(stored))
    assert bench.measured_traffic("fwd") == 107 and bench.measured_traffic("bwd") == 207
    # host-only and unrelated sources do not invalidate either call's figure
    for name in ("dspark_capi.cu", "dspark_noalloc.cu", "dspark_simt.cu", "dspark_host.cpp"):
        with open(csrc / name, "a") as f:
            f.write("\n// edited\n")
    assert bench.measured_traffic("fwd") == 107 and bench.measured_traffic("bwd") == 207
    with open(csrc / "dspark_tc_fwd.cu", "a") as f:
        f.write("\n// edited\n")
    assert bench.measured_traffic("fwd") is None and bench.measured_traffic("bwd") == 207
    with open(csrc / "dspark_tc_common.cuh", "a") as f:
        f.write("\n// edited\n")
    assert bench.measured_traffic("bwd") is None
