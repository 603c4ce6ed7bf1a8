"""The N > 1 pieces of bench.py on CPU, on two gloo ranks: the views each rank
holds in a sharded run (one collection, contiguous halves), the independent
replicas of ``--replicas``, the max-over-ranks step time, and the reference
arm.  The sharded write itself is tested in tests/test_multirank_sharded.py.

Checked: with ``--replicas`` each rank draws its own scene; the step time is
the slowest rank's (an all-reduce MAX that every rank calls); value = all
ranks' tokens over that time; the reference arm runs on rank 0 alone while
the other ranks exit 0 without work.
"""
import contextlib
import datetime
import io
import json
import os
import socket
import types

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from test_layer_reconstruction_b200 import inputs as tin

TINY = tin.CONFIGS["tiny_2v_8x8_d16_h32"]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [3.0, 5.0][rank]
        ms_max = bench.max_over_ranks(ms, world, "cpu")
        rcfg = bench.replica_config(TINY, rank)
        scene, views = bench.shard_views(TINY, rank, world)
        k = tin.make_inputs(rcfg)["K"]
        mine = torch.tensor([float(k.double().sum())], dtype=torch.float64)
        sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(sums, mine)
        args = types.SimpleNamespace(steps=1, warmup=0, gpus=world)
        out = io.StringIO()
        with contextlib.redirect_stdout(out):
            ret = bench.run_reference(args, TINY)
        q.put((rank, ms_max, bench.whole_job_tokens_per_s(world, TINY.n, ms_max), rcfg.seed,
               [float(t) for t in sums], ret, out.getvalue(), (scene.n_views, scene.seed, list(views))))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicas_timing_and_reference_arm():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, max0, val0, seed0, sums0, ret0, out0, sv0), (r1, max1, val1, seed1, sums1, ret1, out1, sv1) = results
    # sharded runs: one collection of 2 x n_views views (the workload's seed), contiguous halves
    assert sv0 == (2 * TINY.n_views, TINY.seed, list(range(TINY.n_views)))
    assert sv1 == (2 * TINY.n_views, TINY.seed, list(range(TINY.n_views, 2 * TINY.n_views)))
    assert (r0, r1) == (0, 1)
    # the slowest rank's time, on every rank
    assert max0 == max1 == 5.0
    assert val0 == val1 == 2 * TINY.n / 5e-3
    # independent scenes: different seeds, different draws, agreed on by both ranks
    assert seed0 != seed1 and sums0 == sums1 and sums0[0] != sums0[1]
    # reference arm: rank 0 prints one JSON line, rank 1 exits 0 without output
    assert ret0 == 0 and ret1 == 0 and out1 == ""
    line = json.loads(out0.strip())
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
