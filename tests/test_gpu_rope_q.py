"""GPU parity of Q's normalisation and 3D rotation inside the attention kernel
("How AI Generates Video: Inside Sora and Wan2.1 on a Real GPU", section 5,
Sub-Layer 1: RMSNorm on Q and K, then the 3D RoPE of section 4, then
attention), of the per-axis phasor table it reads, and of the K-only forms of
the stand-alone RoPE passes, against the float64 oracle.

The oracle side of the attention comparison rounds the rotated Q and K to
bfloat16 as the path stores them: without a norm, the page-precision rotation
(float64 angles, float32 phasors and products: ``rope_3d_fp32``), with which the
kernels agree bit for bit; with a per-head norm, the float64 norm and rotation.
Attention then uses the tolerance of every other attention test
(``tests/gpu_util.py``).  The one-step path is also checked to give the same
bits as the two-step path (rotate Q and K in a pass, then attend), which is
what the header promises."""
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


def _weights(n, seed):
    g = np.random.default_rng(seed)
    return (g.standard_normal(n) * 0.5 + 1.0).astype(np.float32)


@pytest.mark.parametrize("grid,D,split", [((21, 30, 52), 128, (44, 42, 42)),
                                          ((21, 45, 80), 128, (44, 42, 42)),
                                          ((5, 6, 9), 64, (24, 20, 20)),
                                          ((3, 4, 5), 32, (12, 10, 10)),
                                          ((7, 3, 11), 128, (0, 64, 64))])
def test_rope_table_bit_exact(grid, D, split):
    """Every (cos, sin) entry equals the float64 phasor rounded once to float32."""
    import spacetime_attention_vdit_b200 as v
    got = v.rope_3d_table(grid, D, split).cpu().numpy()
    exp = ref.rope_axis_phasors(grid, split).astype(np.float32)
    assert got.shape == exp.shape
    assert np.array_equal(got.view(np.uint32), exp.view(np.uint32))


def test_k_only_rope_bit_exact():
    """K rotated alone equals K rotated beside Q, and the page-precision oracle."""
    import spacetime_attention_vdit_b200 as v
    grid, split = (3, 7, 13), (44, 42, 42)
    q, k, _ = synthetic.qkv_bf16(2, 273, 3, 128, seed=31)
    qd, kd = to_dev_bf16(q), to_dev_bf16(k)
    none, ko = v.rope_3d(None, kd, grid, split)
    assert none is None
    _, ko2 = v.rope_3d(qd, kd, grid, split)
    assert torch.equal(ko.view(torch.int16), ko2.view(torch.int16))
    exp = synthetic.f32_to_bf16_bits(ref.rope_3d_fp32(synthetic.bf16_bits_to_f32(k), grid, split))
    assert np.array_equal(from_dev_bf16(ko), exp)
    _, kin = v.rope_3d(None, kd.clone(), grid, split, inplace=True)
    assert torch.equal(kin.view(torch.int16), ko.view(torch.int16))


@pytest.mark.parametrize("group", [128, 384])
def test_k_only_norm_rope_matches_pair(group):
    """K normalised and rotated alone (per head, and over the token's 3 x 128
    channels) equals the K of the Q-and-K pass, bit for bit."""
    import spacetime_attention_vdit_b200 as v
    grid, split = (3, 7, 13), (44, 42, 42)
    q, k, _ = synthetic.qkv_bf16(1, 273, 3, 128, seed=32, q_scale=3.0)
    wk = torch.from_numpy(_weights(group, 33)).cuda()
    wq = torch.from_numpy(_weights(group, 34)).cuda()
    qd, kd = to_dev_bf16(q), to_dev_bf16(k)
    _, ko = v.qk_norm_rope_3d(None, kd, grid, group, None, wk, split=split)
    _, ko2 = v.qk_norm_rope_3d(qd, kd, grid, group, wq, wk, split=split)
    assert torch.equal(ko.view(torch.int16), ko2.view(torch.int16))


def _oracle_rotated(bits, grid, split, norm, w):
    """The rotated tensor as the path stores it (bf16 bits)."""
    if norm:
        y = ref.qk_norm_rope_3d(synthetic.bf16_bits_to_f64(bits), grid, split, norm,
                                None if w is None else w.astype(np.float64))
        return synthetic.f64_to_bf16_bits(y)
    return synthetic.f32_to_bf16_bits(ref.rope_3d_fp32(synthetic.bf16_bits_to_f32(bits), grid, split))


def _run(v, qd, kd, vd, grid, split, norm, wq, wk):
    """One-step path (K rotated alone, Q in the attention prologue) and the
    two-step path (Q and K rotated in a pass, then attention)."""
    D = qd.shape[-1]
    table = v.rope_3d_table(grid, D, split)
    if norm:
        _, kr = v.qk_norm_rope_3d(None, kd, grid, norm, None, wk, split=split)
        qr2, kr2 = v.qk_norm_rope_3d(qd, kd, grid, norm, wq, wk, split=split)
    else:
        _, kr = v.rope_3d(None, kd, grid, split)
        qr2, kr2 = v.rope_3d(qd, kd, grid, split)
    o, lse = v.attn_full_rope_q(qd, kr, vd, grid, table, split, wq=wq, norm_group=norm, lse=True)
    o2, lse2 = v.attn_full(qr2, kr2, vd, lse=True)
    return o, lse, o2, lse2


@pytest.mark.parametrize("B,grid,heads,D,norm", [
    (1, (3, 7, 13), 2, 128, 0),       # 273 tokens: a second query block with one 17-row tile
    (2, (2, 9, 16), 2, 64, 64),       # per-head norm, 288 tokens
    (1, (4, 5, 9), 3, 32, 0),         # one query block, second tile ragged
    (1, (4, 5, 9), 3, 32, 32),
    (1, (7, 3, 11), 2, 128, 128),     # no time segment: split (0, 64, 64)
    (1, (5, 30, 52), 2, 128, 128),    # the 17-frame 480p grid, 7,800 tokens
])
def test_attn_full_rope_q_matches_oracle(B, grid, heads, D, norm):
    import spacetime_attention_vdit_b200 as v
    split = (0, 64, 64) if grid == (7, 3, 11) else v.default_split(D)
    L = grid[0] * grid[1] * grid[2]
    q, k, vv = synthetic.qkv_bf16(B, L, heads, D, seed=35 + D + norm)
    wq = _weights(D, 36) if norm else None
    wk = _weights(D, 37) if norm else None
    qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(vv)
    wqd = None if wq is None else torch.from_numpy(wq).cuda()
    wkd = None if wk is None else torch.from_numpy(wk).cuda()
    o, lse, o2, lse2 = _run(v, qd, kd, vd, grid, split, norm, wqd, wkd)
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), o2.view(torch.int16)), "one-step and two-step O differ"
    assert torch.equal(lse, lse2), "one-step and two-step LSE differ"
    qr = synthetic.bf16_bits_to_f64(_oracle_rotated(q, grid, split, norm, wq))
    kr = synthetic.bf16_bits_to_f64(_oracle_rotated(k, grid, split, norm, wk))
    rows = None if L <= 2048 else synthetic.sample_rows(L, 1024, seed=38)
    eo, lse_ref = ref.attention(qr, kr, synthetic.bf16_bits_to_f64(vv), rows=rows)
    got = dev_f64(o)
    glse = lse.cpu().numpy()
    if rows is not None:
        got, glse = got[:, rows], glse[:, :, rows]
    assert_attention_close(got, eo, glse, lse_ref, what=f"rope-q {grid} D={D} norm={norm}")


def test_attn_full_rope_q_480p_cfg_pair_sampled():
    """The benched configuration (81-frame 480p CFG pair: batch 2, 32,760 tokens,
    40 heads x 128, no norm): the same launch the bench times, sampled rows of
    three heads against the oracle, and every element against the two-step path."""
    import spacetime_attention_vdit_b200 as v
    grid, split = (21, 30, 52), (44, 42, 42)
    B, L, H, D = 2, 32760, 40, 128
    q, k, vv = synthetic.qkv_bf16(B, L, H, D, seed=39)
    qd, kd, vd = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(vv)
    o, lse, o2, lse2 = _run(v, qd, kd, vd, grid, split, 0, None, None)
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16), o2.view(torch.int16)), "one-step and two-step O differ"
    assert torch.equal(lse, lse2), "one-step and two-step LSE differ"
    rows = synthetic.sample_rows(L, 384, seed=40)
    got = dev_f64(o[:, torch.from_numpy(rows).cuda()])      # [B, rows, H, D]
    glse = lse.cpu().numpy()
    for h in (0, 17, 39):
        k32 = synthetic.bf16_bits_to_f32(k[:, :, h:h + 1])
        q32 = synthetic.bf16_bits_to_f32(q[:, rows, h:h + 1])
        kr = synthetic.bf16_bits_to_f64(synthetic.f32_to_bf16_bits(ref.rope_3d_fp32(k32, grid, split)))
        qr = synthetic.bf16_bits_to_f64(
            synthetic.f32_to_bf16_bits(ref.rope_3d_fp32(q32, grid, split, tokens=rows)))
        eo, lse_ref = ref.attention(qr, kr, synthetic.bf16_bits_to_f64(vv[:, :, h:h + 1]))
        assert_attention_close(got[:, :, h:h + 1], eo, glse[:, h:h + 1, rows], lse_ref, what=f"480p head {h}")
