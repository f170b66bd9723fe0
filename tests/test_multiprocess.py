"""The multi-rank host logic of bench.py on CPU: two gloo ranks for the
barrier and the max-over-ranks timing, per-rank replica seeding (weak
scaling, no collective on the data path), and the reference arm launched by
torchrun with two ranks (rank 0 prints the line, rank 1 exits 0 without
work)."""
import importlib.util
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        bench = _bench()
        barrier, max_over_ranks = bench.dist_helpers(world, "cpu")
        barrier()
        m = max_over_ranks(1.5 + rank)           # each rank's own "elapsed"
        from m3_inputs import make_prefill
        s = bench.replica_shape("siso_f32_b1_t256_h4_p64_n64", rank)
        x = make_prefill(s.with_(seqlen=8))["x"]
        out.put((rank, m, s.seed, float(x.sum()), bench.job_tokens_per_s(world, 3, s, m)))
        barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_barrier_max_and_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, seed0, sum0, v0), (r1, m1, seed1, sum1, v1) = res
    assert m0 == m1 == 2.5                      # the slowest rank's time, on every rank
    assert seed1 == seed0 + 1 and sum0 != sum1  # each rank its own inputs (replicas)
    s = _bench().replica_shape("siso_f32_b1_t256_h4_p64_n64", 0)
    assert v0 == v1 == pytest.approx(2 * 3 * s.batch * s.seqlen / 2.5)


def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "siso_f32_b1_t256_h4_p64_n64"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1                      # rank 0 only
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
