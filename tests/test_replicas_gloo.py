"""Host logic of the multi-GPU benchmark path (token-parallel replicas), run as two
gloo ranks on the CPU: per-rank token seeds, max-over-ranks timing, whole-job
throughput, and the reference arm leaving the work to rank 0."""
import os
import socket
import sys

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime
    import json

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import gen.workloads as W

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [30.0, 45.5][rank]
        mx = bench.max_over_ranks(local_ms, world)
        x = W.x_bf16_bits(4, 256, seed=bench.replica_seed(rank))
        xs = [None] * world
        dist.all_gather_object(xs, x.tolist())

        class A:
            steps, warmup = 2, 1
        ref = bench.run_reference(A, rank, world) if rank != 0 else "skipped"
        res = {"max": mx, "value": bench.job_tokens_per_s(2048, 10, world, mx),
               "x_differ": not np.array_equal(np.array(xs[0]), np.array(xs[1])), "ref": ref}
        json.dump(res, open(os.path.join(out_dir, f"r{rank}.json"), "w"))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    import json
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"r{r}.json")) for r in range(world)]
    for r in res:
        assert r["max"] == 45.5                       # the slowest rank's time
        assert abs(r["value"] - 2 * 2048 * 10 / 0.0455) < 1e-6 * r["value"]
        assert r["x_differ"]                          # replicas run different tokens
    assert res[1]["ref"] is None                      # only rank 0 runs the reference arm
