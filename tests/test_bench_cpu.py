"""CPU tests of bench.py's host logic: algorithmic accounting against hand-computed
values, roofline arithmetic, and the multi-rank plumbing (barrier, max over ranks) on a
world-size-2 gloo group."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench
from mixture_experts_layer_35_b200 import inputs as gen


def test_layer_accounting_qwen36_decode():
    # 8 experts x (2I + I) x H x 2 B + router E x H x 2 + x and out + 4E bias bytes
    acc = bench.accounting(gen.QWEN36, T=1, U=8, router=True, Is=0)["layer"]
    assert acc["bytes"] == 8 * 3 * 2048 * 512 * 2 + 256 * 2048 * 2 + 2 * 2048 * 2 + 4 * 256
    assert acc["flops"] == 2 * 8 * 3 * 2048 * 512 + 2 * 256 * 2048
    assert abs(acc["bytes"] / 1e6 - 51.39) < 0.01


def test_layer_accounting_large_e_with_shared():
    acc = bench.accounting(gen.LARGE_E, T=4, U=40, router=True, Is=640)["layer"]
    per_expert = 3 * 2560 * 640 * 2
    assert acc["bytes"] == 40 * per_expert + 512 * 2560 * 2 + 2 * 4 * 2560 * 2 + per_expert + 4 * 512
    k = bench.accounting(gen.LARGE_E, T=4, U=40, router=True, Is=640)["kernels"]
    assert k["fc1"]["flops"] == 2 * 4 * 10 * 1280 * 2560 + 2 * 4 * 1280 * 2560


def test_roofline_bound_choice():
    peaks = {"hbm_gbs": 1000.0, "bf16_tflops": 100.0}
    r = bench.roofline_of({"bytes": 1e9, "flops": 1e9}, 2e-3, peaks)
    assert r["bound"] == "hbm" and abs(r["achieved"] - 500.0) < 1e-9 and abs(r["frac"] - 0.5) < 1e-12
    r = bench.roofline_of({"bytes": 1e6, "flops": 1e12}, 20e-3, peaks)
    assert r["bound"] == "tensor" and abs(r["frac"] - 0.5) < 1e-12


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    r, local, w = bench.dist_env()
    bench.dist_init(w, "gloo")
    bench.barrier(w)
    m = bench.max_over_ranks(10.0 * (r + 1), w, torch.device("cpu"))
    bench.barrier(w)
    torch.distributed.destroy_process_group()
    q.put((r, m))


def test_max_over_ranks_gloo_world2():
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
    assert res == [(0, 20.0), (1, 20.0)]


def test_single_rank_passthrough():
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    bench.barrier(1)
