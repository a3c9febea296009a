"""The N > 1 benchmark plumbing on CPU: world-size-2 gloo ranks take the max of their step times
and the reference arm runs on rank 0 only (replicas need no data-path collective)."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_setup("gloo")
    assert (w, r) == (world, rank)
    got = bench.reduce_max(10.0 + 5 * rank, "cpu")
    bench.barrier()
    q.put((rank, got))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res == {0: 15.0, 1: 15.0}


def test_reference_arm_only_on_rank_zero():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_byte_model_matches_the_stated_formula():
    sys.path.insert(0, ROOT)
    import bench
    import workloads as W
    wl = W.WORKLOADS["deepseek"]
    T, H, k = wl.tokens, wl.hidden, wl.topk
    b = bench.algorithmic_bytes(wl, valid_pairs=T * k, pad_rows=1000)
    row = H + 4 * H // 128
    assert b["dispatch"] == T * H * 2 + T * k * row + 1000 * row + T * k * 8
    assert b["combine"] == T * k * H * 2 + T * H * 2 + T * k * 8
