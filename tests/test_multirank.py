"""Data-parallel replicas on CPU: two gloo ranks run the benchmark's multi-GPU
plumbing without a GPU.

Each replica holds the same weights and its own token batch; the masks are a
deterministic function of the weights, so every replica computes the same mask
with no collective on the data path (checked here by gathering the oracle's
masks, a test-only exchange).  Timing takes the maximum over ranks.
"""
import datetime
import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        import synthetic_inputs as si
        wl = si.FFNWorkload("tiny", d=64, ff=128, tokens=32, dtype="f16")
        seeds = bench.rank_seeds(wl, rank)
        local = si.FFNWorkload(wl.name, wl.d, wl.ff, wl.tokens, wl.dtype, wl.steps, wl.lam, seeds)
        W1, _ = local.weights()
        X, _ = local.activations()
        mask = torch.from_numpy(oracle.mask_search(si.bits16(W1), "f16").astype(np.int64))
        gathered = [torch.zeros_like(mask) for _ in range(world)]
        dist.all_gather(gathered, mask)
        xs = [torch.zeros(X.shape, dtype=torch.float32) for _ in range(world)]
        dist.all_gather(xs, X.float())
        slowest = bench.max_over_ranks(float(10 * (rank + 1)), world)
        queue.put({"rank": rank, "masks_equal": all(torch.equal(g, gathered[0]) for g in gathered),
                   "batches_differ": not torch.equal(xs[0], xs[1]), "max": slowest,
                   "env": bench.dist_env()})
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicate_masks_and_time_by_max():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = [queue.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in results:
        assert r["masks_equal"]
        assert r["batches_differ"]
        assert r["max"] == 20.0
        assert r["env"][1] == 2
    assert sorted(r["rank"] for r in results) == [0, 1]
