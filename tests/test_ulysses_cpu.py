"""Ulysses sequence parallelism ("Video Diffusion Models, in depth": an all-to-all
swaps the split of a clip from tokens to heads around attention) on 2 and 4
gloo ranks on the CPU: the exchanges move exactly the right elements, and
attention run through them equals attention on the whole clip.  The float64
oracle stands in for the single-device attention call (the kernels need a GPU;
the exchange logic is what is tested here)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import synthetic
        from oracle import reference as ref
        from spacetime_attention_vdit_b200 import ulysses

        T, HW, H, D = 4, 6, 4 * world, 16          # 24 tokens, heads divisible by the ranks
        L = T * HW
        q, k, v = (torch.from_numpy(synthetic.bf16_bits_to_f64(x))
                   for x in synthetic.qkv_bf16(2, L, H, D, seed=11, q_scale=2.0))
        Ls, Hp = L // world, H // world
        shard = lambda x: x[:, rank * Ls:(rank + 1) * Ls].contiguous()

        # the exchanges: exact element movement, and a round trip
        qh = ulysses.tokens_to_heads(shard(q))
        exact_heads = torch.equal(qh, q[:, :, rank * Hp:(rank + 1) * Hp])
        exact_back = torch.equal(ulysses.heads_to_tokens(qh), shard(q))

        def oracle_full(a, b, c):
            return torch.from_numpy(ref.attention(a.numpy(), b.numpy(), c.numpy())[0])

        def oracle_time(a, b, c):
            return torch.from_numpy(ref.divided_time(a.numpy(), b.numpy(), c.numpy(), T, HW)[0])

        o = ulysses.attention_ulysses(shard(q), shard(k), shard(v), attn=oracle_full)
        o_ref = ref.attention(q.numpy(), k.numpy(), v.numpy())[0][:, rank * Ls:(rank + 1) * Ls]
        ot = ulysses.attention_ulysses(shard(q), shard(k), shard(v), attn=oracle_time)
        ot_ref = ref.divided_time(q.numpy(), k.numpy(), v.numpy(), T, HW)[0][:, rank * Ls:(rank + 1) * Ls]
        # Ulysses is limited by the head count: heads that do not split over the
        # ranks are refused on every rank before any exchange
        try:
            ulysses.tokens_to_heads(torch.zeros(1, 2, world + 1, 8))
            refused = False
        except ValueError:
            refused = True
        out[rank] = (exact_heads, exact_back, float(np.abs(o.numpy() - o_ref).max()),
                     float(np.abs(ot.numpy() - ot_ref).max()), refused)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_ulysses_gloo(world):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        exact_heads, exact_back, err_full, err_time, refused = out[r]
        assert exact_heads and exact_back and refused
        assert err_full < 1e-12 and err_time < 1e-12
