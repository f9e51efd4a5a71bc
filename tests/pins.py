"""Pin checks for the oracle, written as functions of the implementation under test.

Each ``pin_*`` returns None when the implementation passes and raises
AssertionError otherwise.  ``test_oracle_pins.py`` runs every pin on the real
oracle (must pass) and on copies with a planted mistake (must fail), which
shows that the pins can see the mistakes one would plausibly make.

None of these checks retypes the oracle's own formula: each compares against
a library routine (``torch.nn.functional.conv3d``,
``scaled_dot_product_attention``, complex multiplication), a closed form, an
invariant the pages state, or a scalar brute force.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import brute
from oracle import closed_forms as cf

# ----------------------------------------------------------------------------
# Patchify  (towardsai section 4; cheatsheet "Tiny video DiT": a Conv3d whose
# stride equals its kernel)
# ----------------------------------------------------------------------------


def pin_patchify_conv3d(patchify):
    """patchify followed by a linear map equals conv3d with stride = kernel."""
    g = np.random.default_rng(11)
    for (N, C, T, H, W), (pt, ph, pw) in (((2, 3, 5, 6, 7), (2, 2, 3)),
                                          ((1, 4, 8, 16, 16), (1, 2, 2)),
                                          ((1, 2, 3, 4, 4), (1, 1, 1))):
        x = g.standard_normal((N, C, T, H, W))
        E = 5
        w = g.standard_normal((E, C, pt, ph, pw))
        tok = patchify(x, pt, ph, pw)                       # [N, L, C*pt*ph*pw]
        lin = tok @ w.reshape(E, -1).T                      # [N, L, E]
        conv = torch.nn.functional.conv3d(torch.from_numpy(x), torch.from_numpy(w),
                                          stride=(pt, ph, pw))  # [N, E, Tg, Hg, Wg]
        conv = conv.flatten(2).transpose(1, 2).numpy()     # [N, L, E] time-major
        assert lin.shape == conv.shape
        assert np.allclose(lin, conv, rtol=1e-12, atol=1e-12)


def pin_patchify_brute(patchify):
    g = np.random.default_rng(12)
    x = g.standard_normal((2, 3, 5, 5, 7))
    for p in ((1, 2, 2), (2, 2, 3), (1, 1, 1), (5, 1, 7)):
        got = patchify(x, *p)
        exp = np.array(brute.patchify(x.tolist(), *p))
        assert got.shape == exp.shape and np.array_equal(got, exp)


def pin_patchify_identity(patchify):
    """With 1x1x1 patches patchify is the transposition NCTHW -> N(THW)C."""
    g = np.random.default_rng(13)
    x = g.standard_normal((2, 3, 4, 5, 6)).astype(np.float32)
    exp = np.moveaxis(x, 1, -1).reshape(2, 4 * 5 * 6, 3)
    got = patchify(x, 1, 1, 1)
    assert got.dtype == np.float32 and np.array_equal(got, exp)


def pin_patchify_flat_index(patchify):
    """Token 4082 of the 17-frame 480p grid (towardsai section 7) is the brick at
    t' = 2, h = 18, w = 26: latent rows 36-37, columns 52-53."""
    T, H, W = 5, 60, 104
    t, h, w = np.meshgrid(np.arange(T), np.arange(H), np.arange(W), indexing="ij")
    code = (t * 1_000_000 + h * 1000 + w).astype(np.float64)[None, None]
    tok = patchify(code, 1, 2, 2)
    idx = cf.flat_index(2, 18, 26, (5, 30, 52))
    assert idx == 4082
    assert list(tok[0, idx]) == [2_036_052, 2_036_053, 2_037_052, 2_037_053]


PATCHIFY_PINS = [pin_patchify_conv3d, pin_patchify_brute, pin_patchify_identity,
                 pin_patchify_flat_index]

# ----------------------------------------------------------------------------
# 3D RoPE  (towardsai section 4)
# ----------------------------------------------------------------------------


def _grid_pos(grid):
    return np.stack(np.meshgrid(*(np.arange(n) for n in grid), indexing="ij"), -1).reshape(-1, 3)


def pin_rope_onehot(rope):
    """Closed-form angles: a unit vector on pair i of axis a at position p comes
    back as (cos(p*f), sin(p*f)) with f = 10000^(-2i/d_a) from the axis width."""
    grid, split, D = (3, 4, 5), (44, 42, 42), 128
    L = 60
    pos = _grid_pos(grid)
    offs = (0, 44, 86)
    for a, i in ((0, 0), (0, 1), (0, 21), (1, 0), (1, 3), (1, 20), (2, 0), (2, 7), (2, 20)):
        x = np.zeros((1, L, 1, D))
        x[:, :, :, offs[a] + 2 * i] = 1.0
        out = rope(x, grid, split)
        f = 10000.0 ** (-2.0 * i / split[a])
        for n in (0, 1, 7, 33, 59):
            ang = pos[n, a] * f
            exp = np.zeros(D)
            exp[offs[a] + 2 * i] = math.cos(ang)
            exp[offs[a] + 2 * i + 1] = math.sin(ang)
            assert np.allclose(out[0, n, 0], exp, atol=1e-13), (a, i, n)


def pin_rope_complex(rope):
    """Against complex multiplication by unit phasors (torch complex128), with the
    positions laid out time-major over the grid."""
    g = np.random.default_rng(21)
    grid, split = (2, 3, 4), (12, 10, 10)
    D = 32
    x = g.standard_normal((2, 24, 3, D))
    pos = _grid_pos(grid)
    ang = []
    for a, d in enumerate(split):
        f = torch.tensor([10000.0 ** (-(2.0 * j) / d) for j in range(d // 2)], dtype=torch.float64)
        ang.append(torch.outer(torch.from_numpy(pos[:, a]).double(), f))
    ang = torch.cat(ang, 1)                                     # [L, D/2]
    ph = torch.polar(torch.ones_like(ang), ang)[None, :, None, :]
    xc = torch.view_as_complex(torch.from_numpy(x).reshape(2, 24, 3, D // 2, 2).contiguous())
    exp = torch.view_as_real(xc * ph).reshape(2, 24, 3, D).numpy()
    assert np.allclose(rope(x, grid, split), exp, atol=1e-12)


def pin_rope_relative(rope):
    """q.k after RoPE depends only on the 3D displacement (towardsai section 4's
    demo: (1,10,20)->(3,12,25) and (2,15,30)->(4,17,35) share delta (2,2,5))."""
    g = np.random.default_rng(22)
    grid, split = (5, 18, 36), (44, 42, 42)
    L = 5 * 18 * 36
    qb, kb = g.standard_normal(128), g.standard_normal(128)
    x = np.zeros((1, L, 2, 128))
    x[0, :, 0] = qb
    x[0, :, 1] = kb
    r = rope(x, grid, split)

    def dot(pq, pk):
        return r[0, cf.flat_index(*pq, grid), 0] @ r[0, cf.flat_index(*pk, grid), 1]

    a = dot((1, 10, 20), (3, 12, 25))
    b = dot((2, 15, 30), (4, 17, 35))
    c = dot((0, 0, 0), (2, 2, 5))
    assert abs(a - b) < 1e-10 and abs(a - c) < 1e-10
    # and a different displacement gives a different score
    assert abs(dot((0, 0, 0), (2, 5, 2)) - c) > 1e-3


def pin_rope_norm_identity(rope):
    """Each pair keeps its length; the token at (0,0,0) is unchanged."""
    g = np.random.default_rng(23)
    grid, split = (3, 4, 5), (12, 10, 10)
    x = g.standard_normal((2, 60, 3, 32))
    r = rope(x, grid, split)
    n_in = np.hypot(x[..., 0::2], x[..., 1::2])
    n_out = np.hypot(r[..., 0::2], r[..., 1::2])
    assert np.allclose(n_in, n_out, rtol=1e-13)
    assert np.array_equal(r[:, 0], x[:, 0])


def pin_rope_brute(rope):
    g = np.random.default_rng(24)
    grid, split = (2, 3, 2), (12, 10, 10)
    x = g.standard_normal((1, 12, 2, 32))
    r = rope(x, grid, split)
    pos = _grid_pos(grid)
    for n in range(12):
        for h in range(2):
            exp = brute.rope_vector(list(x[0, n, h]), tuple(int(p) for p in pos[n]), split)
            assert np.allclose(r[0, n, h], exp, atol=1e-13)


ROPE_PINS = [pin_rope_onehot, pin_rope_complex, pin_rope_relative, pin_rope_norm_identity,
             pin_rope_brute]


# The per-axis phasor cache (towardsai section 4: one frequency table per axis,
# each token's angles looked up by its t, h and w).

def _phasor_index(grid, split, axis, pos, i):
    """Row of the per-axis table: time block, then height, then width; within a
    block pair-major (entry i * extent + pos)."""
    start = sum(grid[a] * (split[a] // 2) for a in range(axis))
    return start + i * grid[axis] + pos


def pin_phasors_brute(phasors):
    """Each entry is what the brute-force rotation does to a unit vector on that
    pair at that position (pure-Python loops, one token at a time)."""
    grid, split = (3, 4, 5), (12, 10, 10)
    tab = phasors(grid, split)
    assert tab.shape == (3 * 6 + 4 * 5 + 5 * 5, 2)
    off = (0, 12, 22)
    for axis in range(3):
        for pos in range(grid[axis]):
            for i in range(split[axis] // 2):
                x = [0.0] * 32
                x[off[axis] + 2 * i] = 1.0
                where = [0, 0, 0]
                where[axis] = pos
                r = brute.rope_vector(x, tuple(where), split)
                got = tab[_phasor_index(grid, split, axis, pos, i)]
                assert abs(got[0] - r[off[axis] + 2 * i]) < 1e-14 and abs(got[1] - r[off[axis] + 2 * i + 1]) < 1e-14


def pin_phasors_page_counts(phasors):
    """The 81-frame 480p grid [21, 30, 52] with the pairs per axis the page prints
    (towardsai section 4: 22 for time, 21 each for height and width, from the
    golden fixture): 21*22 + 30*21 + 52*21 entries; position 0 of every axis
    block is the identity phasor (1, 0)."""
    from tests.conftest import golden
    page = golden("page_numbers.txt")
    pairs = [int(page[k][0]) for k in ("rope_pairs_t", "rope_pairs_h", "rope_pairs_w")]
    grid, split = (21, 30, 52), (44, 42, 42)
    tab = phasors(grid, split)
    assert tab.shape == (21 * pairs[0] + 30 * pairs[1] + 52 * pairs[2], 2)
    for axis in range(3):
        for i in range(split[axis] // 2):
            assert tuple(tab[_phasor_index(grid, split, axis, 0, i)]) == (1.0, 0.0)


def pin_phasors_group(phasors):
    """Angles grow linearly with the position: entry(p) = entry(1)^p as complex
    numbers (torch complex128 powers), and every entry has modulus 1."""
    grid, split = (6, 7, 9), (44, 42, 42)
    tab = phasors(grid, split)
    z = torch.complex(torch.from_numpy(tab[:, 0].copy()), torch.from_numpy(tab[:, 1].copy()))
    assert torch.allclose(z.abs(), torch.ones_like(z.abs()), atol=1e-14)
    for axis in range(3):
        for i in range(split[axis] // 2):
            z1 = z[_phasor_index(grid, split, axis, 1, i)]
            for pos in range(grid[axis]):
                zp = z[_phasor_index(grid, split, axis, pos, i)]
                assert abs(complex(zp) - complex(z1) ** pos) < 1e-12, (axis, pos, i)


PHASOR_PINS = [pin_phasors_brute, pin_phasors_page_counts, pin_phasors_group]

# ----------------------------------------------------------------------------
# Patch embedding and unpatchify  (cheatsheet "Tiny video DiT": a Conv3d whose
# stride equals its kernel; towardsai section 4: bricks to model-width tokens)
# ----------------------------------------------------------------------------


def _onehot_brick_weight(C, pt, ph, pw):
    """Conv weight [F, C, pt, ph, pw] with weight[f, c, dt, dh, dw] = 1 iff f is the
    brick feature index of (c, dt, dh, dw)."""
    F = C * pt * ph * pw
    w = np.zeros((F, C, pt, ph, pw))
    for c in range(C):
        for dt in range(pt):
            for dh in range(ph):
                for dw in range(pw):
                    w[((c * pt + dt) * ph + dh) * pw + dw, c, dt, dh, dw] = 1.0
    return w


def pin_embed_conv3d(patch_embed):
    """torch's conv3d in float64, stride = kernel, then channels-last tokens."""
    g = np.random.default_rng(51)
    for (N, C, T, H, W), (pt, ph, pw), dim in (((2, 4, 3, 6, 8), (1, 2, 2), 24), ((1, 2, 4, 5, 7), (2, 2, 3), 10)):
        x = g.standard_normal((N, C, T, H, W))
        w = g.standard_normal((dim, C * pt * ph * pw))
        b = g.standard_normal(dim)
        got = patch_embed(x, w, b, pt, ph, pw)
        y = torch.nn.functional.conv3d(torch.from_numpy(x), torch.from_numpy(w.reshape(dim, C, pt, ph, pw)),
                                       torch.from_numpy(b), stride=(pt, ph, pw)).numpy()
        exp = y.reshape(N, dim, -1).transpose(0, 2, 1)
        assert np.allclose(got, exp, atol=1e-12)


def pin_embed_identity_and_brute(patch_embed):
    """The one-hot weight turns the embedding into patchify itself; scalar loops
    agree on a tiny clip with a bias."""
    g = np.random.default_rng(52)
    x = g.standard_normal((1, 3, 2, 4, 4))
    F = 3 * 1 * 2 * 2
    eye = np.eye(F)
    assert np.array_equal(patch_embed(x, eye, None, 1, 2, 2), brute_tokens(x, 1, 2, 2))
    w = g.standard_normal((5, F))
    b = g.standard_normal(5)
    got = patch_embed(x, w, b, 1, 2, 2)
    tok = brute.patchify(x.tolist(), 1, 2, 2)
    for l in range(len(tok[0])):
        for o in range(5):
            assert abs(got[0, l, o] - (sum(tok[0][l][f] * w[o, f] for f in range(F)) + b[o])) < 1e-12


def brute_tokens(x, pt, ph, pw):
    return np.array(brute.patchify(x.tolist(), pt, ph, pw))


def pin_unpatchify(unpatchify):
    """The inverse of patchify (exactly), torch's conv_transpose3d with the one-hot
    brick weight in float64, and scalar loops."""
    g = np.random.default_rng(53)
    for (N, C, T, H, W), (pt, ph, pw) in (((2, 3, 4, 6, 8), (1, 2, 2)), ((1, 2, 4, 6, 6), (2, 3, 2))):
        x = g.standard_normal((N, C, T, H, W))
        grid = (T // pt, H // ph, W // pw)
        tok = brute_tokens(x, pt, ph, pw)
        assert np.array_equal(unpatchify(tok, C, grid, pt, ph, pw), x)
        y = torch.nn.functional.conv_transpose3d(
            torch.from_numpy(tok.transpose(0, 2, 1).reshape(N, -1, *grid)),
            torch.from_numpy(_onehot_brick_weight(C, pt, ph, pw)), stride=(pt, ph, pw)).numpy()
        assert np.allclose(unpatchify(tok, C, grid, pt, ph, pw), y, atol=0)
    tok = g.standard_normal((1, 2 * 2 * 3, 8))
    assert np.array_equal(unpatchify(tok, 2, (2, 2, 3), 1, 2, 2),
                          np.array(brute.unpatchify(tok.tolist(), 2, (2, 2, 3), 1, 2, 2)))


EMBED_PINS = [pin_embed_conv3d, pin_embed_identity_and_brute]
UNPATCHIFY_PINS = [pin_unpatchify]

# ----------------------------------------------------------------------------
# Q/K RMSNorm before the 3D RoPE  (towardsai section 5, Sub-Layer 1)
# ----------------------------------------------------------------------------


def pin_norm_torch(qk_norm_rope):
    """With the rotation switched off (all positions 0: a (1,1,1) grid), the
    result is torch's own rms_norm in float64, per head and per token."""
    g = np.random.default_rng(41)
    x = g.standard_normal((2, 1, 3, 16)) * 3.0
    for group in (16, 48):
        w = g.standard_normal(group)
        for eps in (1e-6, 0.5):
            got = qk_norm_rope(x, (1, 1, 1), (6, 4, 6), group, w, eps)
            t = torch.from_numpy(x.reshape(2, 1, 48 // group, group))
            exp = torch.nn.functional.rms_norm(t, (group,), torch.from_numpy(w), eps).numpy().reshape(x.shape)
            assert np.allclose(got, exp, atol=1e-12, rtol=1e-12)


def pin_norm_closed(qk_norm_rope):
    """A constant group c gives c / sqrt(c^2 + eps) * w; with eps = 0 and w = 1
    every group has mean square 1 and scaling x does not change the result."""
    x = np.full((1, 1, 2, 8), 3.0)
    w = np.arange(1, 9, dtype=np.float64)
    got = qk_norm_rope(x, (1, 1, 1), (4, 2, 2), 8, w, 0.25)
    assert np.allclose(got[0, 0, 0], 3.0 / math.sqrt(9.25) * w, atol=1e-14)
    g = np.random.default_rng(42)
    x = g.standard_normal((1, 4, 2, 8))
    y = qk_norm_rope(x, (1, 2, 2), (4, 2, 2), 16, None, 0.0)
    assert np.allclose((y.reshape(1, 4, 16) ** 2).mean(axis=-1), 1.0, atol=1e-13)
    assert np.allclose(qk_norm_rope(7.5 * x, (1, 2, 2), (4, 2, 2), 16, None, 0.0), y, atol=1e-13)


def pin_norm_brute(qk_norm_rope):
    """Scalar loops in the page's order: normalise the group, then rotate each
    head's pairs (brute.rope_vector), with weights that do not commute with the
    rotation."""
    g = np.random.default_rng(43)
    grid, split = (2, 3, 2), (4, 2, 2)
    x = g.standard_normal((1, 12, 2, 8))
    w = g.standard_normal(16) + 2.0
    got = qk_norm_rope(x, grid, split, 16, w, 1e-3)
    for l in range(12):
        pos = (l // 6, (l // 2) % 3, l % 2)
        y = brute.rms_norm(list(x[0, l].reshape(16)), list(w), 1e-3)
        for hh in range(2):
            exp = brute.rope_vector(y[hh * 8:(hh + 1) * 8], pos, split)
            assert np.allclose(got[0, l, hh], exp, atol=1e-13)


NORM_PINS = [pin_norm_torch, pin_norm_closed, pin_norm_brute]

# ----------------------------------------------------------------------------
# Attention  (towardsai sections 5 and 7)
# ----------------------------------------------------------------------------


def _sdpa(q, k, v, scale, mask=None):
    """torch's scaled_dot_product_attention in float64 on [B, L, H, D] arrays."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).permute(0, 2, 1, 3)
    m = None if mask is None else torch.from_numpy(mask)
    o = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


def pin_attention_sdpa(attention):
    g = np.random.default_rng(31)
    for B, L, H, D in ((1, 130, 2, 32), (2, 64, 3, 16)):
        q, k, v = (g.standard_normal((B, L, H, D)) for _ in range(3))
        q *= 3.0  # a peaked softmax so that errors in the scale or the max show
        o, lse = attention(q, k, v, None)
        assert np.allclose(o, _sdpa(q, k, v, 1.0 / math.sqrt(D)), atol=1e-12)
        o2, _ = attention(q, k, v, 0.3)
        assert np.allclose(o2, _sdpa(q, k, v, 0.3), atol=1e-12)


def pin_attention_brute(attention):
    g = np.random.default_rng(32)
    q, k, v = (g.standard_normal((1, 17, 1, 8)) for _ in range(3))
    o, lse = attention(q, k, v, 0.5)
    bo, bl = brute.attention(q[0, :, 0].tolist(), k[0, :, 0].tolist(), v[0, :, 0].tolist(), 0.5)
    assert np.allclose(o[0, :, 0], bo, atol=1e-13)
    assert np.allclose(lse[0, 0], bl, atol=1e-13)


def pin_attention_special(attention):
    """A single key returns its value exactly; identical keys return the mean of
    the values; every softmax row sums to one (exp(s - lse) adds up to 1)."""
    g = np.random.default_rng(33)
    q, k, v = (g.standard_normal((1, 1, 2, 16)) for _ in range(3))
    o, lse = attention(q, k, v, None)
    assert np.array_equal(o, v)
    q = g.standard_normal((1, 9, 2, 16))
    k = np.repeat(g.standard_normal((1, 1, 2, 16)), 9, axis=1)
    v = g.standard_normal((1, 9, 2, 16))
    o, _ = attention(q, k, v, None)
    assert np.allclose(o, v.mean(axis=1, keepdims=True).repeat(9, axis=1), atol=1e-14)
    q, k = (g.standard_normal((1, 40, 1, 16)) * 2 for _ in range(2))
    v = g.standard_normal((1, 40, 1, 16))
    _, lse = attention(q, k, v, None)
    s = (q[0, :, 0] @ k[0, :, 0].T) / 4.0
    assert np.allclose(np.exp(s - lse[0, 0][:, None]).sum(axis=1), 1.0, atol=1e-13)


def pin_attention_cross(attention):
    """Cross-attention (towardsai section 5, Sub-Layer 2: the video tokens supply
    the queries, the text tokens the keys and values): Lq != Lk, against torch
    sdpa in float64 and brute force, with more queries than keys and fewer."""
    g = np.random.default_rng(34)
    for Lq, Lk in ((37, 11), (5, 23)):
        q = g.standard_normal((2, Lq, 2, 16)) * 2.0
        k, v = (g.standard_normal((2, Lk, 2, 16)) for _ in range(2))
        o, lse = attention(q, k, v, None)
        assert o.shape == (2, Lq, 2, 16) and lse.shape == (2, 2, Lq)
        assert np.allclose(o, _sdpa(q, k, v, 0.25), atol=1e-12)
        bo, bl = brute.attention(q[1, :, 1].tolist(), k[1, :, 1].tolist(), v[1, :, 1].tolist(), 0.25)
        assert np.allclose(o[1, :, 1], bo, atol=1e-13)
        assert np.allclose(lse[1, 1], bl, atol=1e-13)


ATTENTION_PINS = [pin_attention_sdpa, pin_attention_brute, pin_attention_special, pin_attention_cross]

# ----------------------------------------------------------------------------
# Divided attention  (cheatsheet "Tiny video DiT"; "Video as a 3D signal",
# "Patches and attention")
# ----------------------------------------------------------------------------


def pin_divided_time(divided_time):
    """The time pass equals full attention restricted to pairs at the same spatial
    site (torch sdpa with that boolean mask)."""
    g = np.random.default_rng(41)
    T, HW = 5, 6
    q, k, v = (g.standard_normal((2, T * HW, 2, 8)) for _ in range(3))
    site = np.arange(T * HW) % HW
    mask = site[:, None] == site[None, :]
    o, _ = divided_time(q, k, v, T, HW, None)
    assert np.allclose(o, _sdpa(q, k, v, 1 / math.sqrt(8), mask), atol=1e-12)


def pin_divided_space(divided_space):
    """The space pass equals full attention restricted to pairs in the same frame."""
    g = np.random.default_rng(42)
    T, HW = 4, 7
    q, k, v = (g.standard_normal((2, T * HW, 2, 8)) for _ in range(3))
    frame = np.arange(T * HW) // HW
    mask = frame[:, None] == frame[None, :]
    o, _ = divided_space(q, k, v, T, HW, None)
    assert np.allclose(o, _sdpa(q, k, v, 1 / math.sqrt(8), mask), atol=1e-12)


def pin_divided_degenerate(divided_time, divided_space):
    """T = 1: the time pass sees one key per site and returns V exactly; HW = 1:
    the space pass does the same."""
    g = np.random.default_rng(43)
    q, k, v = (g.standard_normal((1, 6, 2, 8)) for _ in range(3))
    o, _ = divided_time(q, k, v, 1, 6, None)
    assert np.array_equal(o, v)
    o, _ = divided_space(q, k, v, 6, 1, None)
    assert np.array_equal(o, v)
