"""The N > 1 path of bench.py on CPU with gloo, world size 2: every rank draws
its own shard, elapsed times reduce to the maximum over ranks, the whole-job
value counts all ranks' units, and the reference arm runs on rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        m = bench.max_over_ranks(1.5 + rank, "cpu")
        wl = bench.make_workload("sweep7", rank, tokens=3)
        out.put((rank, m, wl["bits"].tobytes()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[1] for r in res] == [2.5, 2.5]  # max over ranks on every rank
    assert res[0][2] != res[1][2]             # each rank has its own shard


def test_aggregate_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    gbs, tok = bench.aggregate(world=4, unit_bytes=1000, unit_count=10, steps=5, ms=2.0)
    assert np.isclose(gbs, 4 * 1000 * 5 / 2e-3 / 1e9) and np.isclose(tok, 4 * 10 * 5 / 2e-3)
    assert bench.max_over_ranks(3.25, "cpu") == 3.25  # single process: identity


def test_reference_arm_only_rank0_prints():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "sweep7", "--steps", "1", "--warmup", "3"], capture_output=True, text=True, env=env,
                       timeout=600)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_int8_line():
    """The reference arm on the INT8 workload (a reduced token count): its line names
    the INT8 metric, counts 3n + 4 bytes per token and describes the oracle run."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "r4_prefill_int8", "--tokens", "16", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and "INT8" in line["metric"]
    assert line["config"]["tokens"] == 16 and line["config"]["n"] == 16384
    n = 16384
    assert np.isclose(line["value"], 16 * (3 * n + 4) / (line["ms_per_step"] / 1e3) / 1e9, rtol=1e-6)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_cpu_baseline_leg_reports_one_and_all_cores():
    sys.path.insert(0, ROOT)
    import bench
    wl = bench.make_workload("sweep12", 0, tokens=24)
    cpu, ref = bench.cpu_baseline_leg(wl)
    assert cpu["kind"] == "oracle" and cpu["cores"] == 1 and cpu["value"] > 0
    assert cpu["all_cores"]["cores"] >= 1 and cpu["all_cores"]["value"] > 0
    assert ref[1].shape == (24, 2048) and ref[2].shape == (24,) and ref[3] == 24  # kept for the spot check
    wl8 = bench.make_workload("r4_prefill_int8", 0, tokens=2)
    cpu8, ref8 = bench.cpu_baseline_leg(wl8)
    assert cpu8["all_cores"]["cores"] == 1 and ref8 is None  # the INT8 rows run one call at a time
