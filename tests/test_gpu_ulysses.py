"""Ulysses on the GPU with NCCL and one rank (the only GPU a test gets here): the
exchanges are identities and the default attention is the library's kernel, so
the result equals vdit_attn_full bit for bit.  The exchange logic itself is
tested on 2 and 4 gloo ranks in tests/test_ulysses_cpu.py."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

import synthetic
from tests.gpu_util import to_dev_bf16, watchdog_clear

pytestmark = pytest.mark.gpu


def test_ulysses_single_rank_nccl():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import spacetime_attention_vdit_b200 as v
    from spacetime_attention_vdit_b200 import ulysses
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        q, k, vv = (to_dev_bf16(x) for x in synthetic.qkv_bf16(1, 700, 4, 128, seed=12))
        o = ulysses.attention_ulysses(q, k, vv)
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), v.attn_full(q, k, vv).view(torch.int16))
    finally:
        dist.destroy_process_group()
    watchdog_clear()
