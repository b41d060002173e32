"""Head partitioning of one layer over ranks and the sequence <-> head
all-to-all (block_sparse_attention_candidate_b200/sharding.py), on CPU with
world-size-2 gloo process groups: every head owned once, the exchange exact
and invertible, and attention on head shards equal to attention on the whole
layer (float64 oracle on a tiny layer)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from block_sparse_attention_candidate_b200.sharding import head_range  # noqa: E402


@pytest.mark.parametrize("heads,world", [(40, 8), (40, 3), (24, 7), (12, 12), (1, 1), (5, 8)])
def test_head_ranges_cover_every_head_once_and_balance(heads, world):
    if heads < world:
        sizes = [head_range(heads, world, r)[1] - head_range(heads, world, r)[0] for r in range(world)]
        assert sum(sizes) == heads and max(sizes) <= 1
        return
    owned = []
    for r in range(world):
        h0, h1 = head_range(heads, world, r)
        owned.extend(range(h0, h1))
    assert owned == list(range(heads))
    sizes = [head_range(heads, world, r)[1] - head_range(heads, world, r)[0] for r in range(world)]
    assert max(sizes) - min(sizes) <= 1


def test_head_range_rejects_bad_arguments():
    for args in ((0, 2, 0), (4, 0, 0), (4, 2, 2), (4, 2, -1)):
        with pytest.raises(ValueError):
            head_range(*args)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from block_sparse_attention_candidate_b200.sharding import head_to_seq_shards, seq_to_head_shards
    from block_sparse_attention_candidate_b200.workloads import random_qkv_bf16, bf16_bits_to_f64
    from oracle import attention as OA
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, D, block = 1, 4, 96, 16, 16
        # the same seeded layer on every rank; each keeps its sequence slice
        full = torch.arange(B * H * N * D, dtype=torch.float32).reshape(B, H, N, D)
        n_loc = N // world
        mine = full[:, :, rank * n_loc:(rank + 1) * n_loc].contiguous()
        by_head = seq_to_head_shards(mine)
        hw = H // world
        ok_fwd = torch.equal(by_head, full[:, rank * hw:(rank + 1) * hw])
        back = head_to_seq_shards(by_head)
        ok_back = torch.equal(back, mine)
        # attention per head shard (oracle, float64) equals the whole layer's
        bits = random_qkv_bf16(7, B, H, N, D)
        q, k, v = (torch.from_numpy(bf16_bits_to_f64(bits[t])) for t in "qkv")
        nb = N // block
        rp = np.arange(nb + 1) * nb
        col = np.tile(np.arange(nb), nb)
        qs, ks, vs = (seq_to_head_shards(t[:, :, rank * n_loc:(rank + 1) * n_loc].contiguous()) for t in (q, k, v))
        o_sh = torch.zeros_like(qs)
        lse_sh = torch.zeros(qs.shape[:3], dtype=torch.float64)
        for h in range(hw):
            o, lse = OA.sparse_attention(qs[0, h].numpy(), ks[0, h].numpy(), vs[0, h].numpy(), block, rp, col)
            o_sh[0, h] = torch.from_numpy(o)
            lse_sh[0, h] = torch.from_numpy(lse)
        o_back = head_to_seq_shards(o_sh)
        lse_back = head_to_seq_shards(lse_sh.unsqueeze(-1)).squeeze(-1)
        err_o, err_l = 0.0, 0.0
        for h in range(H):
            o_ref, lse_ref = OA.sparse_attention(q[0, h].numpy(), k[0, h].numpy(), v[0, h].numpy(), block, rp, col)
            sl = slice(rank * n_loc, (rank + 1) * n_loc)
            err_o = max(err_o, float(np.abs(o_back[0, h].numpy() - o_ref[sl]).max()))
            err_l = max(err_l, float(np.abs(lse_back[0, h].numpy() - lse_ref[sl]).max()))
        out[rank] = (ok_fwd, ok_back, err_o, err_l)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_sequence_head_all_to_all_world2():
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    for rank in range(2):
        ok_fwd, ok_back, err_o, err_l = out[rank]
        assert ok_fwd and ok_back
        assert err_o == 0.0 and err_l == 0.0
