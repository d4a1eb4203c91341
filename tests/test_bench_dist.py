"""The multi-rank logic of bench.py on CPU: two gloo ranks agree on the
slowest rank's time, verify different batches against the same weights,
and report the same config."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from mxfp4_moe_block_b200 import synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        sh = synth.SHAPES["tiny"]
        mx = bench.max_over_ranks(1.5 + rank, world, "cpu")
        tot = bench.sum_over_ranks(2 + rank, world, "cpu")
        shr = bench.rank_shape(sh, rank)
        x = synth.x_bf16_bits(shr)
        w = synth.weight_codes_np(sh, "w13", 0)
        cfg = bench.workload_config(sh, world)
        out.put((rank, mx, tot, int(x.astype("int64").sum()), int(w.astype("int64").sum()),
                 repr(sorted(cfg.items()))))
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, t0, x0, w0, c0), (r1, m1, t1, x1, w1, c1) = res
    assert m0 == m1 == 2.5                 # slowest rank's value on both
    assert t0 == t1 == 5.0                 # all ranks' accepted tokens on both
    assert x0 != x1                        # different activations per rank
    assert w0 == w1                        # same weights
    assert c0 == c1 and "'global_batch_tokens', 16" in c0


def test_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, 1, "cpu") == 3.25
    assert bench.sum_over_ranks(3.25, 1, "cpu") == 3.25
