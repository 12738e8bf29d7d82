"""bench.py's multi-rank logic on CPU: two gloo ranks (the GPU runs use NCCL with
the same calls).  Checks the max-over-ranks step time, the whole-job weak-scaling
value and that the reference arm does no work off rank 0."""
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = load_bench()
        # per-rank step times 3.0 ms and 4.5 ms: every rank must see the slower one
        ms = bench.max_over_ranks(3.0 + 1.5 * rank, torch.device("cpu"), world)
        value = bench.whole_job_tokens_per_s(220800, world, ms)

        class Args:
            steps, warmup, gpus = 1, 0, world

        # the reference arm returns at once on rank != 0 (rank 0 would run the oracle; not called here)
        ref = bench.run_reference(Args, rank) if rank != 0 else None
        dist.barrier()
        out.put((rank, ms, value, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_step_time_and_value():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [4.5, 4.5]
    # 2 ranks x 220,800 tokens in 4.5 ms
    assert res[0][2] == pytest.approx(2 * 220800 / 4.5e-3)
    assert res[1][3] is None


def test_single_rank_is_identity():
    bench = load_bench()
    assert bench.max_over_ranks(3.25, torch.device("cpu"), 1) == 3.25
    assert bench.whole_job_tokens_per_s(1000, 1, 2.0) == pytest.approx(500000.0)
