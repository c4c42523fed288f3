"""The multi-rank host logic of bench.py on CPU: two gloo ranks agree on the
slowest rank's time and on the whole-job value, get distinct replica seeds,
and the reference arm prints only on rank 0."""
import json
import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [2.0, 3.5][rank]
        got = bench.max_over_ranks(ms, world, "cpu")
        val = bench.whole_job_gbs(1_000_000, world, got)
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.rank_seed_offset(rank))
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump([got, val, seeds], f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree(tmp_path):
    # the ranks are spawned (never forked: this process already runs threads)
    # and hand their results back through files
    port = 29500 + (os.getpid() % 1000)
    mp.spawn(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    res = {}
    for r in range(2):
        with open(tmp_path / f"rank{r}.json") as f:
            got, val, seeds = json.load(f)
        res[r] = (got, val, tuple(seeds))
    assert res[0] == res[1]
    got, val, seeds = res[0]
    assert got == 3.5                                   # the slower rank sets the time
    assert val == pytest.approx(2 * 1_000_000 / 3.5e-3 / 1e9)
    assert len(set(seeds)) == 2                         # independent replicas


def test_single_rank_identity():
    assert bench.max_over_ranks(1.25, 1, "cpu") == 1.25
    assert bench.whole_job_gbs(6_500_000, 1, 1.0) == pytest.approx(6.5)


@pytest.mark.parametrize("rank", [0, 1])
def test_reference_arm_prints_on_rank0_only(rank):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "1", "--gpus", "2"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    if rank == 0:
        d = json.loads(lines[-1])
        assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
        assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0
    else:
        assert lines == []
