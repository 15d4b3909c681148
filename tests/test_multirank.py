"""The N > 1 host logic of bench.py on world-size-2 gloo ranks (CPU, no GPU).

Weak scaling over independent problems: each rank seeds its own inputs, timing is the max
over ranks, and the whole-job value is all ranks' tokens over that time.  There is no
collective on the data path, so these are the only cross-rank steps.
"""

import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, outdir):
    sys.path.insert(0, ROOT)
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port),
                       "WORLD_SIZE": str(world), "RANK": str(rank), "LOCAL_RANK": str(rank),
                       "CUDA_VISIBLE_DEVICES": ""})
    import torch
    import torch.distributed as dist

    import bench
    from block_sparse_long_meanpool_b200 import workloads as W

    w_world, w_rank, _ = bench.dist_setup()
    assert (w_world, w_rank) == (world, rank) and dist.get_backend() == "gloo"
    ms_max = bench.max_over_ranks(10.0 + 5.0 * rank, world)
    bench.barrier(world)
    wl = W.custom("mr", [300, 200], 2, 1, 64, 128, 3, "k_offsets", 99)
    x = W.make_inputs(wl, device="cpu", seed=bench.rank_seed(wl, rank))
    digest = float(x["q"].float().sum())
    digests = [None] * world
    dist.all_gather_object(digests, digest)
    value = bench.job_value(wl.total_tokens, world, ms_max)
    with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
        json.dump({"ms_max": ms_max, "digests": digests, "value": value}, f)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert all(r["ms_max"] == 15.0 for r in res)          # the slowest rank's time
    assert res[0]["digests"][0] != res[0]["digests"][1]   # independent problems per rank
    assert res[0]["value"] == pytest.approx(world * 500 / 15e-3)
