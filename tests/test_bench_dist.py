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


def test_hessian_traffic_from_small_case_counters(tmp_path, monkeypatch):
    """The bench's roofline `traffic` comes from committed ncu counters of small-case
    launches: per width a line through two token counts, evaluated at the layer's T; it is
    null when the counters belong to another version of the kernel or a width is missing."""
    import bench
    from post_weight_quantization_layer_b200 import synth

    cfg = synth.CONFIGS["llama7b"]
    f = tmp_path / "traffic.json"
    caps = [{"n": n, "tokens": t, "dram_bytes": 1000 * n + 3 * t * n} for n in (4096, 11008) for t in (16384, 32768)]
    f.write_text(json.dumps({"kernel_sha": bench.kernel_source_sha(), "captures": caps}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", str(f))
    tr = bench.hessian_traffic(cfg, cfg.tokens)
    assert tr["per_launch"] == [1000 * n + 3 * cfg.tokens * n for n in cfg.hessian_n]
    f.write_text(json.dumps({"kernel_sha": "other", "captures": caps}))
    assert bench.hessian_traffic(cfg, cfg.tokens) is None
    f.write_text(json.dumps({"kernel_sha": bench.kernel_source_sha(), "captures": caps[:2]}))
    assert bench.hessian_traffic(cfg, cfg.tokens) is None
