"""Host logic of bench.py's multi-process path on CPU: two gloo ranks, replica
timing reduced by max over ranks, and the reference arm printed by rank 0 only."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    w, r, _ = bench.dist_setup(world)
    try:
        got = bench.max_over_ranks(10.0 * (r + 1), w, "cpu")
        bench.barrier(w)
        q.put((r, w, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_with_two_gloo_ranks():
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    res = sorted(q.get(timeout=5) for _ in range(2))
    assert [x[1] for x in res] == [2, 2]
    assert all(x[2] == 20.0 for x in res)  # max over ranks


@pytest.mark.slow
def test_reference_arm_two_ranks_prints_one_line():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(29600 + os.getpid() % 1000), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--config", "tiny"]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "weight-cols/s" and d["value"] > 0


def test_hessian_traffic_profile_parses_per_launch():
    """The bench's roofline takes the Hessian's DRAM traffic per launch from the committed
    ncu summary: one figure per distinct Hessian of the Llama-2-7B layer, in launch order,
    each at least the launch's algorithmic bytes (X once + H once)."""
    import bench
    from post_weight_quantization_layer_b200 import synth

    cfg = synth.CONFIGS["llama7b"]
    traffic = bench.load_traffic()
    assert traffic is not None and len(traffic) == len(cfg.hessian_n)
    for n, t in zip(cfg.hessian_n, traffic):
        assert t >= cfg.tokens * n * 2 + n * n * 4
