"""The N > 1 host logic on CPU: two gloo ranks (no GPU), as bench.py runs it under
torchrun with one rank per GPU.  The data path has no collective (every (b, h)
slice is independent); the ranks only agree on the step time, the maximum of
their own timings."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from lsh_attention_hash_b200 import multi, synth
from oracle import oracle_lsh_attention


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # the step time of the run is the maximum of the ranks' own timings
        got = multi.max_over_ranks([10.0 + rank, 5.0 - rank])
        # weak scaling: each rank generates its own batch
        w = synth.small_workload("multi", 1, 1, 256, 64, "bf16", 16, 64, 1)
        qk, _, _ = synth.make_inputs(w, seed=multi.rank_seed(0, rank))
        digest = float(qk.float().sum())
        digests = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(digests, torch.tensor([digest], dtype=torch.float64))
        out[rank] = (got, [float(d) for d in digests])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_timing_and_draw_distinct_batches():
    world = 2
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn", join=True)
    assert sorted(out.keys()) == [0, 1]
    for rank in range(world):
        got, digests = out[rank]
        assert got == [11.0, 5.0]                # max over ranks of (10 + r, 5 - r)
        assert digests[0] != digests[1]          # the ranks' inputs differ
    assert out[0][1] == out[1][1]


def _shard_main(rank, world, port, out):
    """Strong scaling by slices: the rank computes the (b, h) slices of its shard of one batch
    (the float64 oracle stands in for a GPU's four calls), then the ranks all-gather the outputs."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.small_workload("shard", 2, 3, 128, 16, "f32", 8, 32, 2)
        qk, v, R = synth.make_inputs(w, seed=7)
        mine = multi.shard_slices(w.B, w.H, rank, world)
        local = np.zeros((len(mine), w.L, w.D))
        local_lse = np.zeros((len(mine), w.L))
        for n, (b, h) in enumerate(mine):
            res = oracle_lsh_attention(qk[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1], R, w.n_buckets, w.chunk)
            local[n] = res["out"][0, 0]
            local_lse[n] = res["lse"][0, 0]
        # equal-size buffers for all_gather: pad to the largest shard
        n_max = max(len(multi.shard_slices(w.B, w.H, r, world)) for r in range(world))
        send = torch.zeros((n_max, w.L, w.D + 1), dtype=torch.float64)
        send[:len(mine), :, :w.D] = torch.from_numpy(local)
        send[:len(mine), :, w.D] = torch.from_numpy(local_lse)
        recv = [torch.zeros_like(send) for _ in range(world)]
        dist.all_gather(recv, send)
        full = np.zeros((w.B * w.H, w.L, w.D + 1))
        for r in range(world):
            lo, hi = multi.slice_shard(w.B, w.H, r, world)
            full[lo:hi] = recv[r][:hi - lo].numpy()
        out[rank] = full
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_slice_shards_gathered_equal_one_process_run(world):
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    mp.start_processes(_shard_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn",
                       join=True)
    w = synth.small_workload("shard", 2, 3, 128, 16, "f32", 8, 32, 2)
    qk, v, R = synth.make_inputs(w, seed=7)
    ref = oracle_lsh_attention(qk, v, R, w.n_buckets, w.chunk)
    want = np.concatenate([ref["out"].reshape(w.B * w.H, w.L, w.D),
                           ref["lse"].reshape(w.B * w.H, w.L, 1)], axis=2)
    for rank in range(world):
        assert np.array_equal(out[rank], want), f"rank {rank}"


@pytest.mark.parametrize("world", [2, 3, 8])
def test_shard_inputs_are_the_batch_slices(world):
    """bench.py --split slices: the ranks' shard inputs, concatenated in rank order, are exactly the
    batch that one process generates (same slices, same values), and R is the same on every rank."""
    w = synth.small_workload("shard_inputs", 2, 4, 64, 16, "bf16", 8, 32, 2)
    qk, v, R = synth.make_inputs(w, seed=0)
    parts_qk, parts_v = [], []
    for rank in range(world):
        sl = multi.shard_slices(w.B, w.H, rank, world)
        if not sl:
            continue
        q_r, v_r, R_r = synth.make_shard_inputs(w, sl, seed=0)
        assert torch.equal(R_r, R)
        parts_qk.append(q_r[0])
        parts_v.append(v_r[0])
    assert torch.equal(torch.cat(parts_qk), qk.reshape(w.B * w.H, w.L, w.D))
    assert torch.equal(torch.cat(parts_v), v.reshape(w.B * w.H, w.L, w.D))


def test_max_over_ranks_without_process_group_is_identity():
    assert multi.max_over_ranks([1.5, 2.0]) == [1.5, 2.0]


@pytest.mark.parametrize("B,H,world", [(8, 8, 2), (8, 8, 3), (1, 8, 4), (3, 5, 8), (1, 1, 2)])
def test_slice_shards_cover_every_slice_once(B, H, world):
    seen = []
    sizes = []
    for rank in range(world):
        sl = multi.shard_slices(B, H, rank, world)
        sizes.append(len(sl))
        seen += sl
    assert sorted(seen) == [(b, h) for b in range(B) for h in range(H)]
    assert max(sizes) - min(sizes) <= 1


def test_slice_shard_rejects_bad_rank():
    with pytest.raises(ValueError):
        multi.slice_shard(8, 8, 2, 2)
