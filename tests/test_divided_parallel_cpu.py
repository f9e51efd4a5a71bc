"""Divided attention over a frame-sharded clip on 2 and 4 gloo ranks (CPU): the
frame <-> site exchanges move exactly the right elements, and both passes run
through them equal the passes on the whole clip.  The float64 oracle stands in
for the single-device attention calls (the kernels need a GPU; the exchange
logic is what is tested here)."""
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
        from spacetime_attention_vdit_b200 import divided_parallel as dp

        T, HW, H, D = 8, 12, 2, 16                 # frames and sites split over 2 and 4 ranks
        L = T * HW
        q, k, v = (torch.from_numpy(synthetic.bf16_bits_to_f64(x))
                   for x in synthetic.qkv_bf16(2, L, H, D, seed=13, q_scale=2.0))
        Tl, HWl = T // world, HW // world
        frames = lambda x: x[:, rank * Tl * HW:(rank + 1) * Tl * HW].contiguous()
        # this rank's sites of every frame, frame-major: the layout frames_to_sites returns
        sites = lambda x: x.reshape(2, T, HW, H, D)[:, :, rank * HWl:(rank + 1) * HWl].reshape(2, T * HWl, H, D)

        qs = dp.frames_to_sites(frames(q), T, HW)
        exact_sites = torch.equal(qs, sites(q))
        exact_back = torch.equal(dp.sites_to_frames(qs, T, HW), frames(q))

        def oracle_time(a, b, c, t, hw):
            return torch.from_numpy(ref.divided_time(a.numpy(), b.numpy(), c.numpy(), t, hw)[0])

        def oracle_space(a, b, c, t, hw):
            return torch.from_numpy(ref.divided_space(a.numpy(), b.numpy(), c.numpy(), t, hw)[0])

        ot, os_ = dp.divided_attention_frame_sharded(frames(q), frames(k), frames(v), T, HW,
                                                     time_attn=oracle_time, space_attn=oracle_space)
        ot_ref = ref.divided_time(q.numpy(), k.numpy(), v.numpy(), T, HW)[0]
        os_ref = ref.divided_space(q.numpy(), k.numpy(), v.numpy(), T, HW)[0]
        sl = slice(rank * Tl * HW, (rank + 1) * Tl * HW)
        # extents that do not split over the ranks are refused before any exchange
        try:
            dp.frames_to_sites(torch.zeros(1, 2 * (HW + 1), 1, 8), 2 * world, HW + 1)
            refused = False
        except ValueError:
            refused = True
        out[rank] = (exact_sites, exact_back, float(np.abs(ot.numpy() - ot_ref[:, sl]).max()),
                     float(np.abs(os_.numpy() - os_ref[:, sl]).max()), refused)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_divided_frame_sharded_gloo(world):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        exact_sites, exact_back, err_time, err_space, refused = out[r]
        assert exact_sites and exact_back and refused
        assert err_time < 1e-12 and err_space < 1e-12
