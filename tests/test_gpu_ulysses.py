"""Sequence parallelism on the GPU with NCCL and one rank (the only GPU a test
gets here), compared with the float64 oracle: Ulysses attention over a
token-sharded clip ("Video Diffusion Models, in depth", Training and
Inference: an all-to-all swaps the split from tokens to heads) and divided
attention over a frame-sharded clip (cheatsheet "Divided attention": the time
pass needs every frame of a site, so the split swaps from frames to sites).
With one rank the exchanges move nothing between GPUs, but every permutation
and NCCL call of the real path runs on the device.  The exchange logic across
ranks is tested on 2 and 4 gloo ranks in tests/test_ulysses_cpu.py and
tests/test_divided_parallel_cpu.py."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

import synthetic
from oracle import reference as ref
from tests.gpu_util import assert_attention_close, dev_f64, to_dev_bf16, watchdog_clear

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_one_rank():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import spacetime_attention_vdit_b200  # noqa: F401
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    yield
    torch.cuda.synchronize()
    dist.destroy_process_group()
    watchdog_clear()


def f64(bits):
    return synthetic.bf16_bits_to_f64(bits)


def test_ulysses_full_attention_matches_oracle(nccl_one_rank):
    """700 tokens (a ragged last tile), 4 heads x 128: every row against the oracle."""
    from spacetime_attention_vdit_b200 import ulysses
    q, k, v = synthetic.qkv_bf16(1, 700, 4, 128, seed=12)
    o = ulysses.attention_ulysses(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v))
    eo, _ = ref.attention(f64(q), f64(k), f64(v))
    assert_attention_close(dev_f64(o), eo, what="ulysses full")


def test_ulysses_with_a_divided_pass_matches_oracle(nccl_one_rank):
    """Ulysses around the space pass (6 frames x 48 sites, 2 heads)."""
    import spacetime_attention_vdit_b200 as v_
    from spacetime_attention_vdit_b200 import ulysses
    T, HW = 6, 48
    q, k, v = synthetic.qkv_bf16(2, T * HW, 2, 128, seed=13)
    o = ulysses.attention_ulysses(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v),
                                  attn=lambda a, b, c: v_.attn_divided_space(a, b, c, T, HW))
    eo, _ = ref.divided_space(f64(q), f64(k), f64(v), T, HW)
    assert_attention_close(dev_f64(o), eo, what="ulysses space pass")


def test_divided_frame_sharded_matches_oracle(nccl_one_rank):
    """Both passes over a frame-sharded clip: 21 frames x 39 sites, 2 heads x 128,
    batch 2; every row of each pass against the oracle."""
    from spacetime_attention_vdit_b200 import divided_parallel
    T, HW = 21, 39
    q, k, v = synthetic.qkv_bf16(2, T * HW, 2, 128, seed=14)
    o_time, o_space = divided_parallel.divided_attention_frame_sharded(
        to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), T, HW)
    eo, _ = ref.divided_time(f64(q), f64(k), f64(v), T, HW)
    assert_attention_close(dev_f64(o_time), eo, what="frame-sharded time pass")
    eo, _ = ref.divided_space(f64(q), f64(k), f64(v), T, HW)
    assert_attention_close(dev_f64(o_space), eo, what="frame-sharded space pass")
