"""GPU parity of the two gather steps against the oracle: patchify bit for bit,
RoPE bit for bit against the page-precision restatement and within one bf16
ulp of the float64 definition."""
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
    import spacetime_attention_vdit_b200 as v  # noqa: F401  (fails loudly if the library is missing)
    yield
    watchdog_clear()


# --------------------------------------------------------------------------- patchify

@pytest.mark.parametrize("shape,patch", [
    ((1, 4, 8, 16, 16), (1, 2, 2)),       # the tiny clip
    ((2, 3, 5, 7, 9), (2, 2, 2)),         # ragged: every extent leaves a remainder
    ((1, 16, 5, 60, 104), (1, 2, 2)),     # 17 frames at 480p
    ((2, 5, 3, 4, 6), (1, 1, 1)),         # identity permutation
    ((1, 2, 4, 6, 500), (2, 3, 4)),       # rows longer than one CTA chunk
])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_patchify_bit_exact(shape, patch, dtype):
    import spacetime_attention_vdit_b200 as v
    lat = synthetic.latent_f32(*shape, seed=1)
    if dtype == "f32":
        exp = ref.patchify(lat, *patch)
        got = v.patchify_3d(torch.from_numpy(lat).cuda(), patch).cpu().numpy()
        assert got.dtype == np.float32 and np.array_equal(got.view(np.uint32), exp.view(np.uint32))
    else:
        bits = synthetic.f32_to_bf16_bits(lat)
        exp = ref.patchify(bits, *patch)
        got = from_dev_bf16(v.patchify_3d(to_dev_bf16(bits), patch))
        assert np.array_equal(got, exp)


@pytest.mark.parametrize("shape", [(2, 16, 21, 60, 104), (1, 16, 21, 90, 160)])
def test_patchify_full_size(shape):
    """The 81-frame 480p pair (batch 2) and the 720p clip, every element."""
    import spacetime_attention_vdit_b200 as v
    lat = synthetic.latent_f32(*shape, seed=0)
    got = v.patchify_3d(torch.from_numpy(lat).cuda(), (1, 2, 2)).cpu().numpy()
    exp = ref.patchify(lat, 1, 2, 2)
    assert got.shape == (shape[0], 21 * (shape[3] // 2) * (shape[4] // 2), 64)
    assert np.array_equal(got.view(np.uint32), exp.view(np.uint32))


# --------------------------------------------------------------------------- RoPE

def _rope_check(B, grid, heads, D, split, seed=3, tokens=None, scale=1.0):
    import spacetime_attention_vdit_b200 as v
    L = grid[0] * grid[1] * grid[2]
    q, k, _ = synthetic.qkv_bf16(B, L, heads, D, seed=seed, q_scale=scale)
    qd, kd = to_dev_bf16(q), to_dev_bf16(k)
    qo, ko = v.rope_3d(qd, kd, grid, split)
    toks = np.arange(L) if tokens is None else tokens
    for bits, out in ((q, qo), (k, ko)):
        got = from_dev_bf16(out)[:, toks]
        x32 = synthetic.bf16_bits_to_f32(bits[:, toks])
        exp32 = synthetic.f32_to_bf16_bits(ref.rope_3d_fp32(x32, grid, split, tokens=toks))
        assert np.array_equal(got, exp32), "not bit-identical to the page-precision rotation"
        # and within one bf16 ulp of the float64 definition, plus the float32
        # rounding of the two products (which dominates when they cancel):
        # |err| <= ulp_bf16(result) + 2^-22 * (|x0| + |x1|)
        exp64 = ref.rope_3d(x32.astype(np.float64), grid, split, tokens=toks)
        gotf = synthetic.bf16_bits_to_f64(got)
        mag = np.maximum(np.abs(exp64), np.abs(gotf)).astype(np.float32)
        ulp = np.spacing(mag).astype(np.float64) * 2.0 ** 16
        pair = (np.abs(x32[..., 0::2]) + np.abs(x32[..., 1::2])).astype(np.float64).repeat(2, axis=-1)
        assert np.all(np.abs(gotf - exp64) <= ulp + 2.0 ** -22 * pair)
    return qd, kd, qo, ko


@pytest.mark.parametrize("B,grid,heads,D,split", [
    (1, (3, 4, 5), 3, 128, (44, 42, 42)),
    (2, (8, 8, 8), 2, 32, (12, 10, 10)),
    (1, (2, 3, 7), 1, 64, (22, 20, 22)),
    (1, (1, 1, 1), 2, 128, (44, 42, 42)),     # a single token: identity
    (3, (5, 6, 7), 5, 128, (0, 64, 64)),      # empty time segment
])
def test_rope_small(B, grid, heads, D, split):
    _rope_check(B, grid, heads, D, split)


def test_rope_position_coded():
    """One-hot inputs: every pair of every token lands on its own closed-form
    angle, so a mis-paired, mis-positioned or mis-segmented index shows."""
    import spacetime_attention_vdit_b200 as v
    grid, D, split = (4, 5, 6), 128, (44, 42, 42)
    L = 120
    x = np.zeros((1, L, D // 2, D), dtype=np.float32)      # "head" p carries a one on pair p
    for p in range(D // 2):
        x[0, :, p, 2 * p] = 1.0
    bits = synthetic.f32_to_bf16_bits(x)
    qo, _ = v.rope_3d(to_dev_bf16(bits), to_dev_bf16(bits), grid, split)
    got = synthetic.bf16_bits_to_f64(from_dev_bf16(qo))
    ang = ref.rope_tables(grid, split)                       # [L, D/2]
    for p in range(D // 2):
        assert np.allclose(got[0, :, p, 2 * p], np.cos(ang[:, p]), atol=2 ** -8)
        assert np.allclose(got[0, :, p, 2 * p + 1], np.sin(ang[:, p]), atol=2 ** -8)
        others = np.delete(got[0, :, p, :], [2 * p, 2 * p + 1], axis=1)
        assert not others.any()


def test_rope_in_place():
    import spacetime_attention_vdit_b200 as v
    grid = (5, 6, 7)
    q, k, _ = synthetic.qkv_bf16(2, 210, 4, 128, seed=4)
    qo, ko = v.rope_3d(to_dev_bf16(q), to_dev_bf16(k), grid)
    qi, ki = to_dev_bf16(q), to_dev_bf16(k)
    r = v.rope_3d(qi, ki, grid, inplace=True)
    assert r[0].data_ptr() == qi.data_ptr()
    assert torch.equal(qi, qo) and torch.equal(ki, ko)


def test_rope_480p_17_frames():
    """The 7,800-token grid of a 17-frame 480p clip, 12 heads, every element."""
    _rope_check(1, (5, 30, 52), 12, 128, (44, 42, 42), seed=0)


@pytest.mark.parametrize("B,grid", [(2, (21, 30, 52)), (1, (21, 45, 80))])
def test_rope_full_size_sampled(B, grid):
    """81-frame 480p (batch 2) and 720p at 40 heads: 4,096 seeded tokens."""
    L = grid[0] * grid[1] * grid[2]
    toks = synthetic.sample_rows(L, 4096, seed=0)
    _rope_check(B, grid, 40, 128, (44, 42, 42), seed=0, tokens=toks)


@pytest.mark.parametrize("shape", [(1, 5, 3, 6, 1028), (1, 4, 2, 5, 2056), (2, 3, 2, 4, 12), (1, 16, 2, 4, 8)])
def test_patchify_122_fast_path_edges(shape):
    """(1,2,2) float32 shapes that exercise the fast path's chunking: several
    W-chunks (odd channel count, even chunk width), odd H (a floored row), and
    rows of a single vector."""
    import spacetime_attention_vdit_b200 as v
    lat = synthetic.latent_f32(*shape, seed=2)
    got = v.patchify_3d(torch.from_numpy(lat).cuda(), (1, 2, 2)).cpu().numpy()
    exp = ref.patchify(lat, 1, 2, 2)
    assert np.array_equal(got.view(np.uint32), exp.view(np.uint32))
