"""Remaining oracle checks: fp32-precision RoPE, row subsets, the probe, the
split rule, and the seeded input generator's rounding."""
import numpy as np
import pytest
import torch

import synthetic
from oracle import closed_forms as cf
from oracle import reference as ref


def test_split_rule():
    """The cheatsheet's rope_3d ValueError: widths must add up to the head width."""
    x = np.zeros((1, 8, 1, 128))
    with pytest.raises(ValueError):
        ref.rope_3d(x, (2, 2, 2), (44, 42, 40))
    with pytest.raises(ValueError):
        ref.rope_3d(x, (2, 2, 2), (43, 43, 42))
    ref.rope_3d(x, (2, 2, 2), (44, 42, 42))


def test_rope_fp32_close_to_fp64():
    """The page-precision restatement differs from float64 only by float32
    rounding: a few ulps of the larger operand."""
    g = np.random.default_rng(5)
    grid, split = (5, 6, 7), (44, 42, 42)
    x = synthetic.bf16_bits_to_f32(synthetic.f32_to_bf16_bits(
        g.standard_normal((1, 210, 4, 128)).astype(np.float32)))
    r64 = ref.rope_3d(x.astype(np.float64), grid, split)
    r32 = ref.rope_3d_fp32(x, grid, split)
    mag = np.maximum(np.abs(x[..., 0::2]), np.abs(x[..., 1::2])).repeat(2, axis=-1)
    assert np.all(np.abs(r32 - r64) <= 4 * 2.0 ** -24 * mag + 1e-30)


def test_attention_row_subset():
    g = np.random.default_rng(6)
    q, k, v = (g.standard_normal((2, 50, 3, 16)) for _ in range(3))
    full, lse = ref.attention(q, k, v)
    rows = np.array([0, 7, 8, 49])
    sub, lse_s = ref.attention(q, k, v, rows=rows)
    assert np.allclose(sub, full[:, rows], atol=1e-14) and np.allclose(lse_s, lse[:, :, rows], atol=1e-14)
    # row blocking bounds memory only: any block size gives the same rows (BLAS
    # may round the last bit differently for different block shapes)
    blk, _ = ref.attention(q, k, v, row_block=7)
    assert np.allclose(blk, full, atol=1e-14)


def test_space_frame_subset():
    g = np.random.default_rng(7)
    T, HW = 4, 5
    q, k, v = (g.standard_normal((1, T * HW, 2, 8)) for _ in range(3))
    full, lse = ref.divided_space(q, k, v, T, HW)
    sub, lse_s = ref.divided_space(q, k, v, T, HW, frames=[1, 3])
    toks = np.r_[5:10, 15:20]
    assert np.allclose(sub, full[:, toks], atol=1e-14) and np.allclose(lse_s, lse[:, :, toks], atol=1e-14)


def test_divided_lse_against_masked_full():
    g = np.random.default_rng(8)
    T, HW = 3, 4
    q, k, v = (g.standard_normal((1, T * HW, 2, 8)) for _ in range(3))
    _, lt = ref.divided_time(q, k, v, T, HW)
    _, lm = ref.attention(q, k, v, mask=ref.time_mask(T, HW))
    assert np.allclose(lt, lm, atol=1e-13)
    _, ls = ref.divided_space(q, k, v, T, HW)
    _, lm = ref.attention(q, k, v, mask=ref.space_mask(T, HW))
    assert np.allclose(ls, lm, atol=1e-13)


def test_probe_slice_mass():
    """The towardsai section-7 probe: slice masses of one softmax row sum to one,
    and a query whose keys all sit in one slice puts all mass there."""
    g = np.random.default_rng(9)
    grid = (5, 3, 4)
    L = 60
    q = g.standard_normal((1, L, 2, 16))
    k = g.standard_normal((1, L, 2, 16))
    m = ref.slice_mass(q, k, 0, 1, cf.flat_index(2, 1, 1, grid), grid)
    assert m.shape == (5,) and abs(m.sum() - 1) < 1e-13
    k2 = np.zeros_like(k)
    k2[0, 24:36, 0] = 50 * q[0, 5, 0]   # slice t'=2 holds keys aligned with query 5
    m2 = ref.slice_mass(q, k2, 0, 0, 5, grid)
    assert m2[2] > 1 - 1e-9


def test_bf16_rounding_matches_torch():
    g = np.random.default_rng(10)
    x = np.concatenate([g.standard_normal(100000).astype(np.float32),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.5, 0.0, 3.0e38], np.float32)])
    ours = synthetic.f32_to_bf16_bits(x)
    theirs = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)
    back = synthetic.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_f64_to_bf16_direct():
    """Direct float64 rounding agrees with float32 rounding whenever the value is
    a float32, and avoids the double rounding of an f64->f32->bf16 detour."""
    g = np.random.default_rng(11)
    x = g.standard_normal(10000).astype(np.float32)
    assert np.array_equal(synthetic.f64_to_bf16_bits(x.astype(np.float64)), synthetic.f32_to_bf16_bits(x))
    # 1 + 2^-8 + 2^-30: float32 rounds it to the tie 1 + 2^-8 (then to even -> 1.0);
    # the exact value is above the tie and must round up to 1 + 2^-7.
    y = np.array([1.0 + 2.0 ** -8 + 2.0 ** -30])
    assert synthetic.bf16_bits_to_f64(synthetic.f64_to_bf16_bits(y))[0] == 1.0 + 2.0 ** -7


def test_generator_blocking_invariant():
    """Blockwise draws equal one draw, so big tensors do not depend on block size."""
    a = synthetic.normal_f32((3, 1000), 0, 2)
    b = synthetic.rng_for(0, 2).standard_normal(3000, dtype=np.float32).reshape(3, 1000)
    assert np.array_equal(a, b)
    old = synthetic._BLOCK
    try:
        synthetic._BLOCK = 7
        c = synthetic.normal_f32((3, 1000), 0, 2)
    finally:
        synthetic._BLOCK = old
    assert np.array_equal(a, c)


def test_divided_rows_match_full_passes():
    g = np.random.default_rng(12)
    T, HW = 5, 7
    q, k, v = (g.standard_normal((2, T * HW, 3, 8)) for _ in range(3))
    rows = np.array([0, 3, 7, 20, 34])
    ft, lt = ref.divided_time(q, k, v, T, HW)
    rt, rl = ref.divided_time_rows(q, k, v, T, HW, rows)
    assert np.allclose(rt, ft[:, rows], atol=1e-14) and np.allclose(rl, lt[:, :, rows], atol=1e-13)
    fs, ls = ref.divided_space(q, k, v, T, HW)
    rs, rsl = ref.divided_space_rows(q, k, v, T, HW, rows)
    assert np.allclose(rs, fs[:, rows], atol=1e-14) and np.allclose(rsl, ls[:, :, rows], atol=1e-13)


def test_rope_token_subset():
    g = np.random.default_rng(13)
    grid, split = (3, 4, 5), (12, 10, 10)
    x = g.standard_normal((2, 60, 2, 32))
    toks = np.array([0, 5, 19, 33, 59])
    full = ref.rope_3d(x, grid, split)
    assert np.array_equal(ref.rope_3d(x[:, toks], grid, split, tokens=toks), full[:, toks])
    x32 = x.astype(np.float32)
    assert np.array_equal(ref.rope_3d_fp32(x32[:, toks], grid, split, tokens=toks),
                          ref.rope_3d_fp32(x32, grid, split)[:, toks])


def test_patch_embed_token_subset_is_those_rows_of_torch_conv3d():
    """The oracle's token selection (used at full size, where only sampled tokens
    are checked) returns exactly those rows of torch's float64 conv3d."""
    import torch
    from oracle import reference as ref
    g = np.random.default_rng(54)
    N, C, T, H, W, dim = 2, 4, 3, 6, 8, 24
    x = g.standard_normal((N, C, T, H, W))
    w = g.standard_normal((dim, C * 4))
    b = g.standard_normal(dim)
    sel = np.array([0, 5, 17, 35])
    got = ref.patch_embed(x, w, b, 1, 2, 2, tokens=sel)
    y = torch.nn.functional.conv3d(torch.from_numpy(x), torch.from_numpy(w.reshape(dim, C, 1, 2, 2)),
                                   torch.from_numpy(b), stride=(1, 2, 2)).numpy()
    exp = y.reshape(N, dim, -1).transpose(0, 2, 1)[:, sel]
    assert got.shape == (N, sel.size, dim)
    assert np.allclose(got, exp, atol=1e-12)
