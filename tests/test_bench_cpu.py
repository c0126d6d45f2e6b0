"""bench.py host logic on CPU: the reference arm's JSON line, and the multi-rank
plumbing (max over ranks, per-rank seeds) with world_size 2 over gloo."""
import json
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny-16x16-w4", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["higher_is_better"] is True


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    bench.init_dist(world, "gloo")
    got = bench.max_over_ranks(1.5 + rank)
    from shifted_window_attention_pad_b200 import WORKLOADS
    seed = bench.rank_seed(WORKLOADS["tiny-16x16-w4"], rank)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got, seed))


def test_max_over_ranks_and_rank_seeds_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.5, 2.5]
    assert res[0][2] != res[1][2]


def test_l2_flush_only_for_workloads_smaller_than_twice_l2():
    import bench
    from shifted_window_attention_pad_b200 import WORKLOADS
    want = {"ragged-90x180-w8": True, "twelfth-degree-256x544-w8": False,
            "downsampled-128x272-w16": False, "small-patch-2x512x1088-w8": False}
    for name, flush in want.items():
        assert bench.needs_l2_flush(WORKLOADS[name]) == flush, name
    assert bench.input_bytes(WORKLOADS["twelfth-degree-256x544-w8"]) == 4 * 256 * 544 * 16 * 64 * 2


def test_roofline_entry_holds_1024_token_windows_to_the_tensor_peak():
    """32 x 32 windows do N/2 = 512 FLOP per byte, past the ridge of the
    measured peaks: their backward is held to the bf16 tensor peak in
    TFLOP/s; every other family to HBM bandwidth in GB/s."""
    import bench
    from shifted_window_attention_pad_b200 import WORKLOADS
    hbm, tf, _ = bench.measured_peaks()
    assert tf / hbm * 1e3 < 512                      # the ridge in FLOP per byte
    wl = WORKLOADS["table5-large-256x544-8x128-w32"]
    assert wl.flops_bwd() == 8 * 1024 * 128 * 256 * 544 * 8
    e = bench.roofline_entry(4, wl, 5.0, 400.0, hbm, "measured", None, wl.alg_bytes_bwd())
    assert e["bound"] == "tensor" and e["unit"] == "TFLOP/s" and e["peak"] == tf
    assert abs(e["achieved"] - wl.flops_bwd() / 5e-3 / 1e12) < 1e-9
    assert abs(e["frac"] - e["achieved"] / tf) < 1e-12
    wl8 = WORKLOADS["twelfth-degree-256x544-w8"]
    e = bench.roofline_entry(1, wl8, 0.75, 2660.0, hbm, "measured", None, wl8.alg_bytes_bwd())
    assert e["bound"] == "hbm" and e["unit"] == "GB/s" and e["achieved"] == 2660.0
