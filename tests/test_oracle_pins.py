"""The oracle passes every pin; copies with a planted mistake fail at least one.

Planted mistakes live only here, in CPU code, on the oracle side."""
import numpy as np
import pytest

from oracle import reference as ref
from tests import pins

# ----------------------------------------------------------------------------
# the real oracle passes
# ----------------------------------------------------------------------------


@pytest.mark.parametrize("pin", pins.PATCHIFY_PINS, ids=lambda p: p.__name__)
def test_patchify_pins(pin):
    pin(ref.patchify)


@pytest.mark.parametrize("pin", pins.ROPE_PINS, ids=lambda p: p.__name__)
def test_rope_pins(pin):
    pin(ref.rope_3d)


@pytest.mark.parametrize("pin", pins.ATTENTION_PINS, ids=lambda p: p.__name__)
def test_attention_pins(pin):
    pin(lambda q, k, v, scale: ref.attention(q, k, v, scale))


@pytest.mark.parametrize("pin", pins.NORM_PINS, ids=lambda p: p.__name__)
def test_norm_pins(pin):
    pin(ref.qk_norm_rope_3d)


@pytest.mark.parametrize("pin", pins.EMBED_PINS, ids=lambda p: p.__name__)
def test_embed_pins(pin):
    pin(ref.patch_embed)


def test_unpatchify_pins():
    for pin in pins.UNPATCHIFY_PINS:
        pin(ref.unpatchify)


@pytest.mark.parametrize("pin", pins.PHASOR_PINS, ids=lambda p: p.__name__)
def test_phasor_pins(pin):
    pin(ref.rope_axis_phasors)


def test_divided_pins():
    pins.pin_divided_time(ref.divided_time)
    pins.pin_divided_space(ref.divided_space)
    pins.pin_divided_degenerate(ref.divided_time, ref.divided_space)


# ----------------------------------------------------------------------------
# planted mistakes are caught
# ----------------------------------------------------------------------------


def _fails(pin_list, fn):
    caught = 0
    for pin in pin_list:
        try:
            pin(fn)
        except (AssertionError, ValueError, IndexError):
            caught += 1
    return caught


def patchify_feature_order_swapped(latent, pt, ph, pw):
    """Mistake: brick features ordered (dt, dh, dw, c) instead of (c, dt, dh, dw)."""
    N, C, T, H, W = latent.shape
    Tg, Hg, Wg = T // pt, H // ph, W // pw
    x = latent[:, :, :Tg * pt, :Hg * ph, :Wg * pw].reshape(N, C, Tg, pt, Hg, ph, Wg, pw)
    return x.transpose(0, 2, 4, 6, 3, 5, 7, 1).reshape(N, Tg * Hg * Wg, -1)


def patchify_token_order_swapped(latent, pt, ph, pw):
    """Mistake: tokens flattened width-major instead of time-major."""
    N, C, T, H, W = latent.shape
    Tg, Hg, Wg = T // pt, H // ph, W // pw
    x = latent[:, :, :Tg * pt, :Hg * ph, :Wg * pw].reshape(N, C, Tg, pt, Hg, ph, Wg, pw)
    return x.transpose(0, 6, 4, 2, 1, 3, 5, 7).reshape(N, Tg * Hg * Wg, -1)


@pytest.mark.parametrize("bad", [patchify_feature_order_swapped, patchify_token_order_swapped])
def test_patchify_mistakes_caught(bad):
    assert _fails(pins.PATCHIFY_PINS, bad) >= 1


def _rope_variant(x, grid, split, theta=10000.0, freq_width=None, pairing="adjacent",
                  sign=1.0, axis_order=(0, 1, 2)):
    B, L, Hh, D = x.shape
    ref.check_split(D, split)
    Tg, Hg, Wg = grid
    idx = np.arange(L)
    pos = [idx // (Hg * Wg), (idx // Wg) % Hg, idx % Wg]
    angs = []
    for a, d in enumerate(split):
        w = d if freq_width is None else freq_width
        f = 1.0 / theta ** (np.arange(0, d, 2) / w)
        angs.append(np.outer(pos[axis_order[a]], f))
    ang = np.concatenate(angs, 1)
    c, s = np.cos(ang)[None, :, None], np.sin(ang)[None, :, None]
    out = np.empty_like(x)
    if pairing == "adjacent":
        i0, i1 = np.arange(0, D, 2), np.arange(1, D, 2)
    else:  # rotate-half within each axis segment
        i0, i1, off = [], [], 0
        for d in split:
            i0 += list(range(off, off + d // 2))
            i1 += list(range(off + d // 2, off + d))
            off += d
        i0, i1 = np.array(i0), np.array(i1)
    x0, x1 = x[..., i0], x[..., i1]
    out[..., i0] = x0 * c - sign * x1 * s
    out[..., i1] = sign * x0 * s + x1 * c
    return out


def attention_keys_cut_to_queries(q, k, v, scale):
    """Mistake: the key loop runs over the query length (a self-attention
    assumption that breaks cross-attention)."""
    Lq, Lk = q.shape[1], k.shape[1]
    n = min(Lq, Lk)
    return ref.attention(q, k[:, :n], v[:, :n], scale)


def test_cross_attention_mistake_caught():
    assert _fails([pins.pin_attention_cross], attention_keys_cut_to_queries) == 1


@pytest.mark.parametrize("kw", [
    dict(freq_width=128),            # frequencies from the head width, not the axis width
    dict(pairing="half"),            # rotate-half pairs instead of adjacent pairs
    dict(sign=-1.0),                 # rotation in the wrong direction
    dict(axis_order=(2, 1, 0)),      # width position on the time segment
], ids=["head-width-freq", "rotate-half", "sign", "axis-order"])
def test_rope_mistakes_caught(kw):
    # the unmodified variant passes, so a failure below is the planted mistake
    for pin in pins.ROPE_PINS:
        pin(lambda x, g, s: _rope_variant(x, g, s))
    bad = lambda x, g, s: _rope_variant(x, g, s, **kw)
    assert _fails(pins.ROPE_PINS, bad) >= 1


def _attention_variant(q, k, v, scale, no_scale=False, no_norm=False, drop_last_key=False):
    B, L, H, D = q.shape
    if scale is None or scale <= 0:
        scale = 1.0 / np.sqrt(D)
    if no_scale:
        scale = 1.0
    o = np.empty((B, L, H, v.shape[-1]))
    lse = np.empty((B, H, L))
    for b in range(B):
        for h in range(H):
            kk = k[b, :, h][:-1] if (drop_last_key and k.shape[1] > 1) else k[b, :, h]
            vv = v[b, :, h][:-1] if (drop_last_key and k.shape[1] > 1) else v[b, :, h]
            s = q[b, :, h] @ kk.T * scale
            m = s.max(1, keepdims=True)
            p = np.exp(s - m)
            l = p.sum(1, keepdims=True)
            o[b, :, h] = p @ vv if no_norm else (p @ vv) / l
            lse[b, h] = (m + np.log(l))[:, 0]
    return o, lse


@pytest.mark.parametrize("kw", [dict(no_scale=True), dict(no_norm=True), dict(drop_last_key=True)],
                         ids=["no-scale", "no-normalise", "ragged-tail-dropped"])
def test_attention_mistakes_caught(kw):
    for pin in pins.ATTENTION_PINS:
        pin(_attention_variant)
    bad = lambda q, k, v, s: _attention_variant(q, k, v, s, **kw)
    assert _fails(pins.ATTENTION_PINS, bad) >= 1


def test_divided_mistakes_caught():
    # time pass that groups by frame (it is the space pass), and the reverse
    with pytest.raises(AssertionError):
        pins.pin_divided_time(lambda q, k, v, T, HW, s: ref.divided_space(q, k, v, T, HW, s))
    with pytest.raises(AssertionError):
        pins.pin_divided_space(lambda q, k, v, T, HW, s: ref.divided_time(q, k, v, T, HW, s))


# ---- Q/K RMSNorm + RoPE: planted mistakes


def _norm_variant(x, grid, split, group, weight=None, eps=1e-6, rope_first=False, eps_outside=False,
                  sum_not_mean=False, per_head_group=False):
    x = np.asarray(x, dtype=np.float64)
    B, L, H, D = x.shape
    gsz = D if per_head_group else group
    w = np.ones(group) if weight is None else np.asarray(weight, dtype=np.float64)
    if gsz != group:
        w = np.resize(w, gsz)
    y = ref.rope_3d(x, grid, split) if rope_first else x
    g = y.reshape(B, L, (H * D) // gsz, gsz)
    ms = (g * g).sum(axis=-1, keepdims=True) if sum_not_mean else (g * g).mean(axis=-1, keepdims=True)
    r = (np.sqrt(ms) + eps) if eps_outside else np.sqrt(ms + eps)
    y = (g / r * w).reshape(B, L, H, D)
    return y if rope_first else ref.rope_3d(y, grid, split)


@pytest.mark.parametrize("kw", [dict(rope_first=True), dict(eps_outside=True), dict(sum_not_mean=True),
                                dict(per_head_group=True)],
                         ids=["rope-before-norm", "eps-outside-sqrt", "sum-not-mean", "group-per-head"])
def test_norm_mistakes_caught(kw):
    for pin in pins.NORM_PINS:
        pin(_norm_variant)
    bad = lambda *a, **k: _norm_variant(*a, **k, **kw)
    assert _fails(pins.NORM_PINS, bad) >= 1


# ---- patch embedding and unpatchify: planted mistakes


def embed_feature_order_swapped(latent, weight, bias, pt, ph, pw):
    """Mistake: brick features (dt, dh, dw, c) against a (c, dt, dh, dw) weight."""
    return patchify_feature_order_swapped(latent, pt, ph, pw) @ np.asarray(weight).T + (0 if bias is None else bias)


def embed_bias_dropped(latent, weight, bias, pt, ph, pw):
    return ref.patch_embed(latent, weight, None, pt, ph, pw)


def unpatchify_spatial_swapped(tokens, C, grid, pt, ph, pw):
    """Mistake: brick rows and columns exchanged on the way back."""
    N = tokens.shape[0]
    Tg, Hg, Wg = grid
    x = tokens.reshape(N, Tg, Hg, Wg, C, pt, ph, pw).transpose(0, 4, 1, 5, 2, 7, 3, 6)
    return np.ascontiguousarray(x.reshape(N, C, Tg * pt, Hg * pw, Wg * ph))


@pytest.mark.parametrize("bad", [embed_feature_order_swapped, embed_bias_dropped], ids=lambda f: f.__name__)
def test_embed_mistakes_caught(bad):
    assert _fails(pins.EMBED_PINS, bad) >= 1


def test_unpatchify_mistake_caught():
    assert _fails(pins.UNPATCHIFY_PINS, unpatchify_spatial_swapped) == 1


def _phasor_variant(grid, split, theta=10000.0, axis_order=(0, 1, 2), swap=False, head_width=None, start=0,
                    pos_major=False):
    parts = []
    for a in axis_order:
        n, d = grid[a], split[a]
        j = np.arange(0, d, 2, dtype=np.float64)
        f = 1.0 / (theta ** (j / (head_width or d)))
        ang = np.outer(f, np.arange(start, start + n, dtype=np.float64))
        if pos_major:
            ang = ang.T
        c, s_ = np.cos(ang), np.sin(ang)
        parts.append(np.stack([s_, c] if swap else [c, s_], axis=-1).reshape(-1, 2))
    return np.concatenate(parts, axis=0)


@pytest.mark.parametrize("kw", [
    dict(axis_order=(1, 0, 2)),      # height block before the time block
    dict(swap=True),                 # (sin, cos) instead of (cos, sin)
    dict(head_width=128),            # frequencies from the head width
    dict(start=1),                   # positions counted from 1
    dict(pos_major=True),            # position-major within an axis
], ids=["axis-order", "sin-cos", "head-width-freq", "one-based", "pos-major"])
def test_phasor_mistakes_caught(kw):
    for pin in pins.PHASOR_PINS:
        pin(_phasor_variant)
    bad = lambda g, s: _phasor_variant(g, s, **kw)
    assert _fails(pins.PHASOR_PINS, bad) >= 1
