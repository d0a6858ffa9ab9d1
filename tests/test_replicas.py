"""The multi-GPU (replica) path of bench.py on CPU: two gloo ranks.

The encoder shards over the batch with no collective on the data path; the
only cross-rank step is the max-over-ranks of the step times, and every rank
runs its own seeded batch.  The reference arm, launched with torchrun, prints
one line on rank 0 and exits 0 on the others.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    import encoder_inputs as EI
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms, e2e = 3.0 + rank, 5.0 - rank          # rank 1 slower on ms, rank 0 slower on e2e
        got = bench.max_over_ranks([ms, e2e])
        wl = bench.replica_workload(EI.named_workload("pruned-s32", 4), rank)
        inp = EI.make_inputs(wl)
        results[rank] = (got, wl.seed, float(inp.x.astype("float64").sum()),
                         bench.job_throughput(wl.batch, world, got[0]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_own_batches():
    world, port = 2, _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        r0, r1 = results[0], results[1]
    assert r0[0] == r1[0] == [4.0, 5.0]          # both ranks see the slowest rank's times
    assert r0[1] != r1[1] and r0[2] != r1[2]      # distinct seeds, distinct batches
    assert r0[3] == pytest.approx(4 * 2 / 4.0e-3)  # all ranks' sequences in the slowest time


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "3", "--ref-sample", "1", "--workload", "pruned-s32:4"]
    res = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600,
                         env=dict(os.environ, OMP_NUM_THREADS="2"))
    assert res.returncode == 0, res.stderr[-2000:]
    lines = [l for l in res.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0
