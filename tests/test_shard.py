"""Batch sharding over ranks (the multi-GPU path), run on CPU as gloo ranks.

Each rank takes a contiguous block of batch rows and runs the whole cycle on
it; the rank's draws come from the rows' global indices (row_offset), so the
gathered output equals one unsharded run.  Here the per-rank compute is the
oracle over the rank's rows; the GPU kernels' row_offset is checked against
the same property in the GPU parity tests."""
import os
import pickle
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import synth
import oracle
from draft_sampling_verification_head_b200 import shard

W = synth.Workload("shard", B=7, K=3, V=96, r=8, dtype="f32", sigma=0.7, seed=5, uw_std=0.4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir, mode):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch.distributed as dist
    result = {}
    try:
        assert shard.init("gloo", timeout_s=20)
        if mode == "cycle":
            d = synth.make(W)
            P = oracle.Params(B=W.B, K=W.K, V=W.V, r=W.r, dtype=W.dtype, temperature=1.0, seed=3,
                              cycle=2)
            raw = [synth.to_numpy_raw(d[k]) for k in ("base", "target", "U", "W")]
            b0, b1 = shard.shard_range(W.B, world, rank)
            o = oracle.cycle(P, *raw, d["last_token"].numpy(), b_begin=b0, b_end=b1)
            got = {k: shard.gather_rows(torch.from_numpy(np.ascontiguousarray(o[k])), W.B)
                   for k in ("draft", "out", "tau")}
            result["gathered"] = None if rank else {k: v.numpy() for k, v in got.items()}
            result["max"] = shard.max_over_ranks(1.5 + rank)
            result["sum"] = shard.sum_over_ranks(b1 - b0)
            shard.barrier()
        elif mode == "rank_exits":
            if rank == 1:
                result["left"] = True
                return  # leaves between steps, with nothing in flight
            try:
                shard.max_over_ranks(1.0)
                result["error"] = None
            except Exception as e:  # the collective ends with an error, not a wait
                result["error"] = type(e).__name__
    finally:
        with open(os.path.join(outdir, f"r{rank}.pkl"), "wb") as f:
            pickle.dump(result, f)
        if mode != "rank_exits" and dist.is_initialized():
            dist.destroy_process_group()


def _run(world, mode, tmp_path):
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, str(tmp_path), mode))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
    out = []
    for r in range(world):
        with open(tmp_path / f"r{r}.pkl", "rb") as f:
            out.append(pickle.load(f))
    return out


@pytest.mark.parametrize("rows,world", [(7, 2), (8, 2), (5, 3), (2, 4), (0, 3), (64, 8)])
def test_shard_range_partitions_rows(rows, world):
    spans = [shard.shard_range(rows, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == rows
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 == b0
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    assert shard.shard_counts(rows, world) == sizes


def test_shard_range_rejects_bad_splits():
    for args in ((4, 0, 0), (4, 2, 2), (-1, 2, 0)):
        with pytest.raises(ValueError):
            shard.shard_range(*args)


def test_two_ranks_reproduce_the_unsharded_cycle(tmp_path):
    oracle.build()
    res = _run(2, "cycle", tmp_path)
    d = synth.make(W)
    P = oracle.Params(B=W.B, K=W.K, V=W.V, r=W.r, dtype=W.dtype, temperature=1.0, seed=3, cycle=2)
    raw = [synth.to_numpy_raw(d[k]) for k in ("base", "target", "U", "W")]
    full = oracle.cycle(P, *raw, d["last_token"].numpy())
    g = res[0]["gathered"]
    for k in ("draft", "out", "tau"):
        assert np.array_equal(g[k], full[k]), k
    assert all(r["max"] == 2.5 for r in res)  # the slowest rank's time
    assert all(r["sum"] == W.B for r in res)  # units of the whole job


def test_a_rank_that_leaves_ends_the_others_collective(tmp_path):
    res = _run(2, "rank_exits", tmp_path)
    assert res[1]["left"]
    assert res[0]["error"] is not None
