"""Host logic of bench.py that needs no GPU: the max-over-ranks reduction used to
time multi-GPU runs (two gloo ranks on the CPU), and the reference arm's line."""

import json
import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    got = bench.max_over_ranks(10.0 + 3.0 * rank, world)
    bench.barrier(world)
    out[rank] = got
    dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
        assert dict(out) == {0: 13.0, 1: 13.0}


def test_single_rank_passthrough():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.5, 1) == 4.5


def test_reference_arm_prints_contract_line():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "1"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "1"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_work_flops_counts_the_window_visible_pairs():
    """Without a window the bench uses the headline formula; with one it counts the
    visible (q, k) pairs: checked against a brute-force double loop."""
    sys.path.insert(0, ROOT)
    import bench
    from attention_forward_flash_b200.inputs import Workload
    w = Workload("t", 2, 4, 2, 37, 61, 64, causal=True, start_pos=20)
    assert bench.work_flops(w) == w.flops()
    for W, lo in ((1, 0), (5, 0), (16, 30), (200, 0)):
        ww = w.scaled(window_size=W, window_lo=lo)
        pairs = sum(1 for i in range(ww.q_len) for j in range(ww.kv_len)
                    if j >= lo and j <= ww.start_pos + i and ww.start_pos + i - j < W)
        assert bench.work_flops(ww) == 4.0 * ww.batch * ww.n_q_heads * pairs * ww.head_dim
