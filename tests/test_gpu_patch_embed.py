"""GPU parity of the patch embedding (a Conv3d whose stride equals its kernel:
cheatsheet "Tiny video DiT"; "How AI Generates Video: Inside Sora and Wan2.1 on
a Real GPU", section 4) and of unpatchify, against the float64 oracle.

Unpatchify moves values: bit exact.  The embedding runs on bf16 operands (the
latent rounded to bf16 nearest-even on both sides, the weight given in bf16),
accumulates 64 exact products in float32 and adds the float32 bias, then rounds
once to bf16: |err| <= ulp_bf16(result) + 2^-16 (sum_f |x_f w_f| + |b|)."""
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


@pytest.mark.parametrize("N,C,grid,patch", [
    (1, 4, (8, 8, 8), (1, 2, 2)),
    (2, 16, (5, 30, 52), (1, 2, 2)),      # 17 frames at 480p
    (1, 3, (2, 3, 7), (2, 2, 3)),
    (1, 16, (3, 4, 130), (1, 2, 2)),      # a brick row wider than one CTA's chunk
])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_unpatchify_bit_exact(N, C, grid, patch, dtype):
    import spacetime_attention_vdit_b200 as v
    pt, ph, pw = patch
    F = C * pt * ph * pw
    g = np.random.default_rng(sum(grid) + C)
    tok = g.standard_normal((N, grid[0] * grid[1] * grid[2], F)).astype(np.float32)
    if dtype == torch.bfloat16:
        tok = synthetic.bf16_bits_to_f32(synthetic.f32_to_bf16_bits(tok))
    td = torch.from_numpy(tok).cuda().to(dtype)
    got = v.unpatchify_3d(td, C, grid, patch).float().cpu().numpy()
    exp = ref.unpatchify(tok, C, grid, pt, ph, pw)
    assert np.array_equal(got.view(np.uint32), exp.view(np.uint32))
    # and the round trip through patchify
    back = v.patchify_3d(v.unpatchify_3d(td, C, grid, patch), patch)
    assert torch.equal(back, td)


def _embed_check(N, C, T, H, W, patch, dim, with_bias=True, tokens=None, seed=7):
    import spacetime_attention_vdit_b200 as v
    pt, ph, pw = patch
    F = C * pt * ph * pw
    g = np.random.default_rng(seed)
    lat = g.standard_normal((N, C, T, H, W)).astype(np.float32)
    w_bits = synthetic.f32_to_bf16_bits((g.standard_normal((dim, F)) / 8.0).astype(np.float32))
    b = g.standard_normal(dim).astype(np.float32) if with_bias else None
    out = v.patch_embed_3d(torch.from_numpy(lat).cuda(), to_dev_bf16(w_bits), patch,
                           None if b is None else torch.from_numpy(b).cuda())
    L = (T // pt) * (H // ph) * (W // pw)
    assert out.shape == (N, L, dim)
    lat_r = synthetic.bf16_bits_to_f64(synthetic.f32_to_bf16_bits(lat))     # the operand the kernel uses
    w64 = synthetic.bf16_bits_to_f64(w_bits)
    toks = np.arange(L) if tokens is None else tokens
    exp = ref.patch_embed(lat_r, w64, None if b is None else b.astype(np.float64), pt, ph, pw, tokens=toks)
    got = synthetic.bf16_bits_to_f64(from_dev_bf16(out)[:, toks])
    brick = np.abs(ref.patchify(lat_r, pt, ph, pw)[:, toks])
    mag_terms = brick @ np.abs(w64).T + (0.0 if b is None else np.abs(b.astype(np.float64)))
    mag = np.maximum(np.abs(exp), np.abs(got)).astype(np.float32)
    ulp = np.spacing(mag).astype(np.float64) * 2.0 ** 16
    err = np.abs(got - exp)
    assert np.all(err <= ulp + 2.0 ** -16 * mag_terms), f"max excess {(err - ulp - 2.0 ** -16 * mag_terms).max():.3e}"


@pytest.mark.parametrize("N,C,T,H,W,patch,dim,bias", [
    (1, 16, 4, 16, 16, (1, 2, 2), 256, True),      # 256 tokens: two full token tiles
    (1, 16, 3, 10, 14, (1, 2, 2), 512, True),      # 105 tokens: one ragged tile
    (2, 16, 3, 11, 15, (1, 2, 2), 768, False),     # floored extents, no bias
    (1, 8, 6, 10, 12, (2, 2, 2), 256, True),       # another brick with 64 features
    (1, 16, 3, 20, 22, (1, 2, 2), 1280, True),     # 5 N tiles: work groups of 2, 2 and 1
    (1, 16, 2, 18, 30, (1, 2, 2), 1792, False),    # 7 N tiles: work groups of 2, 2, 2 and 1
])
def test_patch_embed_small(N, C, T, H, W, patch, dim, bias):
    _embed_check(N, C, T, H, W, patch, dim, bias)


def test_patch_embed_480p_17_frames():
    """The page's shape: [1, 16, 5, 60, 104] -> 7,800 tokens of width 1,536."""
    _embed_check(1, 16, 5, 60, 104, (1, 2, 2), 1536)


def test_patch_embed_480p_81_frames_cfg_pair_sampled():
    """[2, 16, 21, 60, 104] -> 2 x 32,760 tokens of width 1,536 (4,096 seeded tokens checked)."""
    _embed_check(2, 16, 21, 60, 104, (1, 2, 2), 1536, tokens=synthetic.sample_rows(32760, 4096, seed=0))


def test_patch_embed_480p_81_frames_cfg_pair_width_5120_sampled():
    """The bench's shape: [2, 16, 21, 60, 104] -> 2 x 32,760 tokens of the 14B
    model's width 5,120 (40 heads x 128; aicassindra Step 2), 20 N tiles in four
    work groups of 5; 4,096 seeded tokens checked."""
    _embed_check(2, 16, 21, 60, 104, (1, 2, 2), 5120, tokens=synthetic.sample_rows(32760, 4096, seed=0))
