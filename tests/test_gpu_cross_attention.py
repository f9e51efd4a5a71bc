"""GPU parity of text cross-attention (the video tokens query the text tokens'
keys and values: "How AI Generates Video: Inside Sora and Wan2.1 on a Real GPU",
section 5, Sub-Layer 2) against the float64 oracle.  Small cases are compared on
every row; the 480p and 720p clips against 512 prompt tokens on 4,096 seeded
query rows per (batch, head).  Tolerances: tests/gpu_util.py."""
import numpy as np
import pytest
import torch

import synthetic
from oracle import reference as ref
from tests.gpu_util import assert_attention_close, dev_f64, from_dev_bf16, to_dev_bf16, watchdog_clear

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import spacetime_attention_vdit_b200 as v  # noqa: F401
    yield
    watchdog_clear()


def f64(bits):
    return synthetic.bf16_bits_to_f64(bits)


def cross_inputs(B, Lq, Lk, H, D, seed, q_scale=1.0):
    """Queries from one seeded draw, keys and values from another (the text side)."""
    q, _, _ = synthetic.qkv_bf16(B, Lq, H, D, seed=seed, q_scale=q_scale)
    _, k, v = synthetic.qkv_bf16(B, Lk, H, D, seed=seed + 1000)
    return q, k, v


@pytest.mark.parametrize("B,Lq,Lk,H,D,q_scale", [
    (1, 64, 1, 2, 32, 1.0),       # a single key: O = V for every query
    (1, 300, 77, 2, 128, 1.0),    # one short key tile (a short prompt)
    (1, 257, 129, 1, 128, 1.0),   # ragged on both sides: 2 query tiles + 1 row, 2 key tiles
    (2, 1000, 512, 3, 128, 1.0),  # 512 prompt tokens, several query blocks
    (1, 500, 512, 2, 128, 8.0),   # peaked rows
    (1, 130, 700, 2, 64, 1.0),    # more keys than queries
    (2, 300, 2200, 2, 128, 1.0),  # 18 key tiles: the per-row-store variant of the kernel
])
def test_cross_small(B, Lq, Lk, H, D, q_scale):
    import spacetime_attention_vdit_b200 as v_
    q, k, v = cross_inputs(B, Lq, Lk, H, D, seed=Lq + Lk, q_scale=q_scale)
    o, lse = v_.attn_cross(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), lse=True)
    assert o.shape == (B, Lq, H, D) and lse.shape == (B, H, Lq)
    eo, el = ref.attention(f64(q), f64(k), f64(v))
    assert_attention_close(dev_f64(o), eo, lse.cpu().numpy(), el, f"cross {B, Lq, Lk, H, D}")
    if Lk == 1:
        assert np.array_equal(from_dev_bf16(o), np.broadcast_to(v, o.shape))


def test_cross_equals_full_when_lengths_match():
    """With Lq = Lk and the same tensors, cross-attention is full attention, bit for bit."""
    import spacetime_attention_vdit_b200 as v_
    q, k, v = synthetic.qkv_bf16(1, 700, 2, 128, seed=21)
    Q, K, V = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    oc, lc = v_.attn_cross(Q, K, V, lse=True)
    of, lf = v_.attn_full(Q, K, V, lse=True)
    assert torch.equal(oc.view(torch.int16), of.view(torch.int16))
    assert torch.equal(lc, lf)


def _sampled_cross(B, Lq, Lk, H):
    import spacetime_attention_vdit_b200 as v_
    q, k, v = cross_inputs(B, Lq, Lk, H, 128, seed=0)
    o, lse = v_.attn_cross(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), lse=True)
    rows = synthetic.sample_rows(Lq, 4096, seed=0)
    og = from_dev_bf16(o[:, rows])
    lg = lse[:, :, rows].cpu().numpy()
    del o, lse
    for h in range(H):
        eo, el = ref.attention(f64(q[:, rows, h:h + 1]), f64(k[:, :, h:h + 1]), f64(v[:, :, h:h + 1]))
        assert_attention_close(f64(og[:, :, h:h + 1]), eo, lg[:, h:h + 1], el, f"head {h}")


def test_cross_480p_81_frames_cfg_pair_sampled():
    """32,760 video tokens (21x30x52) against 512 prompt tokens, 40 heads x 128, batch 2."""
    _sampled_cross(2, 32760, 512, 40)


def test_cross_720p_81_frames_sampled():
    """75,600 video tokens (21x45x80) against 512 prompt tokens, 40 heads x 128."""
    _sampled_cross(1, 75600, 512, 40)
