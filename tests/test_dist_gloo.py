"""The N > 1 path on CPU: whole-prompt sharding over 2 gloo ranks reproduces the
single-process result, the weak-scaling batches differ per rank, and the
timing reduction takes the slowest rank."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
from vlm_decoder_positional_b200 import inputs, shard


def test_shards_cover_every_prompt_once_and_balance_tokens():
    for cfg in (2, 3, 5):
        wl = inputs.make_config(cfg, with_qk=False)
        for world in (1, 2, 3, 4, 8):
            shards = [shard.shard_sequences(wl.cu_seqlens, world, r) for r in range(world)]
            assert shards[0].seq_lo == 0 and shards[-1].seq_hi == wl.num_seqs
            for a, b in zip(shards, shards[1:]):
                assert a.seq_hi == b.seq_lo and a.tok_hi == b.tok_lo
            sizes = [s.n_tokens for s in shards]
            assert sum(sizes) == wl.n_tokens
            longest = int(np.diff(wl.cu_seqlens).max())
            assert max(sizes) - min(sizes) <= 2 * longest


def test_shard_of_empty_and_tiny_batches():
    cu = np.array([0, 0, 0, 5], np.int32)
    shards = [shard.shard_sequences(cu, 4, r) for r in range(4)]
    assert sum(s.n_tokens for s in shards) == 5
    assert shards[-1].seq_hi == 3
    with pytest.raises(ValueError):
        shard.shard_sequences(cu, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        wl = inputs.make_config(2)
        sh = shard.shard_sequences(wl.cu_seqlens, world, rank)
        ids, cu = shard.local_batch(wl.ids, wl.cu_seqlens, sh)
        pos, start, amount = oracle.positions(ids, cu, wl.image_token_id)
        q = wl.q.view(torch.int16).numpy().view(np.uint16)[:, sh.tok_lo:sh.tok_hi]
        rq = oracle.rotate_bf16(q, pos)
        gathered = [None] * world
        dist.all_gather_object(gathered, (sh, pos, start, amount, rq))
        # weak scaling: each rank's own batch differs
        own = inputs.make_config(2, with_qk=False,
                                 seed=shard.rank_seed(inputs.BASE_SEED + 2, rank))
        heads = [None] * world
        dist.all_gather_object(heads, own.ids[:64].tolist())
        slowest = shard.max_over_ranks(10.0 + rank, dist)
        if rank == 0:
            np.save(os.path.join(out_dir, "ok.npy"), np.array([0]))
            full_pos, full_start, full_amount = oracle.positions(wl.ids, wl.cu_seqlens,
                                                                 wl.image_token_id)
            full_q = oracle.rotate_bf16(wl.q.view(torch.int16).numpy().view(np.uint16),
                                        full_pos)
            got_pos = np.concatenate([g[1] for g in gathered], axis=1)
            got_start = np.concatenate([g[2] for g in gathered])
            got_amount = np.concatenate([g[3] for g in gathered])
            got_q = np.concatenate([g[4] for g in gathered], axis=1)
            assert [g[0].seq_lo for g in gathered] == sorted(g[0].seq_lo for g in gathered)
            np.testing.assert_array_equal(got_pos, full_pos)
            np.testing.assert_array_equal(got_start, full_start)
            np.testing.assert_array_equal(got_amount, full_amount)
            np.testing.assert_array_equal(got_q, full_q)
            assert heads[0] != heads[1]
            assert slowest == 10.0 + world - 1
            np.save(os.path.join(out_dir, "ok.npy"), np.array([1]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reproduce_the_single_process_result():
    world = 2
    with tempfile.TemporaryDirectory() as d:
        mp.spawn(_worker, args=(world, _free_port(), d), nprocs=world, join=True)
        assert int(np.load(os.path.join(d, "ok.npy"))[0]) == 1
