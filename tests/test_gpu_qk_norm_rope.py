"""GPU parity of the fused Q/K RMSNorm + 3D RoPE ("How AI Generates Video: Inside
Sora and Wan2.1 on a Real GPU", section 5, Sub-Layer 1: RMSNorm on Q and K, then
the rotation) against the float64 oracle.

Bound (floating point; bf16 in, float32 arithmetic, one bf16 rounding): the
result is within one bf16 ulp of the float64 definition plus the float32 error
of the normalisation (the group's sum of squares in float32 and the reciprocal
square root: a few 1e-6 relative) and of the rotation's two products, which
dominate when they cancel: |err| <= ulp_bf16(result) + 3e-5 (|y0| + |y1|), y the
normalised pair."""
import numpy as np
import pytest
import torch

import synthetic
from oracle import reference as ref
from tests.gpu_util import from_dev_bf16, to_dev_bf16, watchdog_clear

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import spacetime_attention_vdit_b200 as v  # noqa: F401
    yield
    watchdog_clear()


def _weights(group, seed):
    g = np.random.default_rng(seed)
    return (g.standard_normal(group) * 0.5 + 1.0).astype(np.float32)


def _check(B, grid, heads, D, split, group, eps=1e-6, weighted=True, tokens=None, seed=5, inplace=False):
    import spacetime_attention_vdit_b200 as v
    L = grid[0] * grid[1] * grid[2]
    q, k, _ = synthetic.qkv_bf16(B, L, heads, D, seed=seed, q_scale=3.0)
    wq = _weights(group, seed + 1) if weighted else None
    wk = _weights(group, seed + 2) if weighted else None
    qd, kd = to_dev_bf16(q), to_dev_bf16(k)
    wqd = None if wq is None else torch.from_numpy(wq).cuda()
    wkd = None if wk is None else torch.from_numpy(wk).cuda()
    qo, ko = v.qk_norm_rope_3d(qd, kd, grid, group, wqd, wkd, eps=eps, split=split, inplace=inplace)
    if inplace:
        assert qo.data_ptr() == qd.data_ptr() and ko.data_ptr() == kd.data_ptr()
    toks = np.arange(L) if tokens is None else tokens
    for bits, w, out in ((q, wq, qo), (k, wk, ko)):
        got = synthetic.bf16_bits_to_f64(from_dev_bf16(out)[:, toks])
        x = synthetic.bf16_bits_to_f64(bits[:, toks])
        w64 = None if w is None else w.astype(np.float64)
        y = ref.rms_norm(x, group, w64, eps)
        exp = ref.rope_3d(y, grid, split, tokens=toks)
        assert np.all(np.isfinite(got))
        mag = np.maximum(np.abs(exp), np.abs(got)).astype(np.float32)
        ulp = np.spacing(mag).astype(np.float64) * 2.0 ** 16
        pair = (np.abs(y[..., 0::2]) + np.abs(y[..., 1::2])).repeat(2, axis=-1)
        err = np.abs(got - exp)
        assert np.all(err <= ulp + 3e-5 * pair), f"max excess {(err - ulp - 3e-5 * pair).max():.3e}"


@pytest.mark.parametrize("B,grid,heads,D,split,group", [
    (1, (8, 8, 8), 2, 32, (12, 10, 10), 32),      # the tiny clip, per head
    (1, (8, 8, 8), 2, 32, (12, 10, 10), 64),      # the tiny clip, per token
    (2, (3, 4, 5), 3, 64, (22, 20, 22), 64),      # per head, odd head count
    (2, (3, 4, 5), 3, 64, (22, 20, 22), 192),     # per token, 24 vectors
    (1, (1, 1, 1), 4, 128, (44, 42, 42), 128),    # one token: only the norm
    (1, (2, 3, 7), 2, 128, (44, 42, 42), 256),
    (2, (3, 5, 6), 2, 128, (0, 64, 64), 128),     # empty time segment: no time table
])
def test_qk_norm_rope_small(B, grid, heads, D, split, group):
    _check(B, grid, heads, D, split, group)


def test_qk_norm_rope_unweighted_large_eps_inplace():
    _check(1, (3, 5, 6), 4, 128, (44, 42, 42), 512, eps=0.75, weighted=False, inplace=True)


@pytest.mark.parametrize("group", [128, 1536])
def test_qk_norm_rope_480p_17_frames(group):
    """The page's own shape: 7,800 tokens (5x30x52), 12 heads x 128, per head and
    per token (1,536 channels)."""
    _check(1, (5, 30, 52), 12, 128, (44, 42, 42), group)


@pytest.mark.parametrize("group", [128, 5120])
def test_qk_norm_rope_480p_81_frames_cfg_pair_sampled(group):
    """32,760 tokens, 40 heads x 128, batch 2: 4,096 seeded tokens checked."""
    _check(2, (21, 30, 52), 40, 128, (44, 42, 42), group, tokens=synthetic.sample_rows(32760, 4096, seed=0))


@pytest.mark.parametrize("group", [128, 5120])
def test_qk_norm_rope_720p_81_frames_sampled(group):
    """75,600 tokens (21x45x80), 40 heads x 128, batch 1: 4,096 seeded tokens
    checked, per head and per token (5,120 channels)."""
    _check(1, (21, 45, 80), 40, 128, (44, 42, 42), group, tokens=synthetic.sample_rows(75600, 4096, seed=0))
