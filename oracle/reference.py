"""Float64 definitions of the hot path: patchify, factorised 3D RoPE, attention.

TEST INFRASTRUCTURE: imported only by tests, the smoke check and the CPU
baseline of the bench.  Shares no code with the CUDA library.

Layouts follow the library's boundary so that tests compare element by element:

* latent clip ``[N, C, T, H, W]``;
* tokens ``[N, L, C*pt*ph*pw]`` with L flattened time-major, then rows, then
  columns;
* per-head Q/K/V/O ``[B, L, heads, head_dim]``.

Sources (page title, section):

* Patchify - "How AI Generates Video: Inside Sora and Wan2.1 on a Real GPU",
  section 4 (1x2x2 spacetime bricks of 16*1*2*2 = 64 floats, [5,30,52] grid);
  "Video and 3D Generation" cheatsheet, "Tiny video DiT" (patch embedding is a
  Conv3d whose stride equals its kernel); token order from section 7 of the
  towardsai article (flat index t*H'W' + h*W' + w).
* RoPE - towardsai section 4 (axes_dim [44, 42, 42] for time, height, width;
  per-axis frequencies theta^(-2i/d_axis) with theta = 10000 built in float64;
  adjacent pairs (x[2i], x[2i+1]) viewed as one complex number and multiplied
  by the unit phasor of angle pos * frequency).  The cheatsheet's
  "Troubleshooting" row: the three widths must add up to the head width.
* Attention - towardsai sections 5 and 7 (every token attends to every token;
  logits scaled by 1/sqrt(head_dim), then softmax, then the value average);
  aicassindra "Step 3: the diffusion transformer" (tiled kernels compute the
  same result).  Divided attention - cheatsheet "Tiny video DiT" and "Formulas
  and numbers"; "Video as a 3D signal", "Patches and attention" (a time pass
  over the T tokens at each spatial site, a space pass over the HW tokens of
  each frame).
* Q/K normalisation - towardsai section 5, "Sub-Layer 1": the projected Q and
  K are RMS-normalised, then rotated by the 3D RoPE.  RMSNorm here is the
  textbook one: each group of G consecutive channels of a token is divided by
  sqrt(mean of its squares + eps) and multiplied by a per-channel weight.  The
  page names neither the group nor eps: G is an argument (head_dim: per head;
  heads*head_dim: the token's whole projected vector).
"""
from __future__ import annotations

import math

import numpy as np

from .closed_forms import grid_position, token_grid

# ----------------------------------------------------------------------------
# Patchify
# ----------------------------------------------------------------------------


def patchify(latent: np.ndarray, pt: int, ph: int, pw: int) -> np.ndarray:
    """Cut ``[N, C, T, H, W]`` into (pt, ph, pw) bricks, one token per brick.

    Token (t', h', w') sits at row t'*H'*W' + h'*W' + w'; its features are the
    brick's values ordered channel first, then dt, dh, dw (the flattening of a
    Conv3d weight [out, C, pt, ph, pw]).  Extents that do not divide are
    floored; the leftover voxels are not read.  The dtype is preserved: this is
    a permutation of values, not arithmetic.
    """
    N, C, T, H, W = latent.shape
    Tg, Hg, Wg = token_grid(T, H, W, pt, ph, pw)
    x = latent[:, :, :Tg * pt, :Hg * ph, :Wg * pw]
    x = x.reshape(N, C, Tg, pt, Hg, ph, Wg, pw)
    # -> N, Tg, Hg, Wg, C, pt, ph, pw
    x = x.transpose(0, 2, 4, 6, 1, 3, 5, 7)
    return np.ascontiguousarray(x.reshape(N, Tg * Hg * Wg, C * pt * ph * pw))


def unpatchify(tokens: np.ndarray, C: int, grid, pt: int, ph: int, pw: int) -> np.ndarray:
    """Put every token's brick back: ``[N, Tg*Hg*Wg, C*pt*ph*pw]`` ->
    ``[N, C, Tg*pt, Hg*ph, Wg*pw]``, the inverse of ``patchify`` (the last step
    of the transformer maps its tokens back to the latent clip the same way the
    first cut it; same feature order)."""
    N, L, F = tokens.shape
    Tg, Hg, Wg = grid
    if L != Tg * Hg * Wg or F != C * pt * ph * pw:
        raise ValueError("tokens do not match the grid and brick")
    x = tokens.reshape(N, Tg, Hg, Wg, C, pt, ph, pw)
    # -> N, C, Tg, pt, Hg, ph, Wg, pw
    x = x.transpose(0, 4, 1, 5, 2, 6, 3, 7)
    return np.ascontiguousarray(x.reshape(N, C, Tg * pt, Hg * ph, Wg * pw))


def patch_embed(latent: np.ndarray, weight: np.ndarray, bias, pt: int, ph: int, pw: int,
                tokens=None) -> np.ndarray:
    """The patch embedding: a Conv3d whose stride equals its kernel (cheatsheet
    "Tiny video DiT"; towardsai section 4: each 1x2x2 brick of 16 latent channels
    becomes one model-width token), i.e. patchify then a matrix product, in
    float64.  ``weight`` is the Conv3d weight [dim, C, pt, ph, pw] flattened to
    [dim, C*pt*ph*pw]; ``bias`` is [dim] or None.  ``tokens`` optionally keeps
    only those token rows (each row is its own product, so a subset is exactly
    those rows of the full result).  Returns [N, L or len(tokens), dim]."""
    tok = patchify(np.asarray(latent, dtype=np.float64), pt, ph, pw)
    if tokens is not None:
        tok = tok[:, np.asarray(tokens)]
    w = np.asarray(weight, dtype=np.float64)
    y = tok @ w.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)
    return y


# ----------------------------------------------------------------------------
# 3D rotary position embedding
# ----------------------------------------------------------------------------


def check_split(head_dim: int, split) -> None:
    """The cheatsheet's rule: the time, height and width widths must add up to
    the head width (a ValueError otherwise).  Each width must also be even,
    since it is consumed as complex pairs."""
    d_t, d_h, d_w = split
    if d_t + d_h + d_w != head_dim:
        raise ValueError(f"rope split {split} does not add up to head_dim {head_dim}")
    if d_t % 2 or d_h % 2 or d_w % 2 or min(split) < 0:
        raise ValueError(f"rope split {split} must be non-negative and even")


def default_split(head_dim: int):
    """Time gets the remainder, height and width 2*floor(D/6) each: (44, 42, 42)
    for D = 128 as the towardsai article states; (12, 10, 10) for D = 32."""
    s = 2 * (head_dim // 6)
    return (head_dim - 2 * s, s, s)


def rope_inv_freq(d_axis: int, theta: float = 10000.0) -> np.ndarray:
    """Per-axis frequencies 1 / theta^(j/d_axis), j = 0, 2, ..., d_axis-2, in float64
    (towardsai section 4: each axis uses its own width, not the head width)."""
    j = np.arange(0, d_axis, 2, dtype=np.float64)
    return 1.0 / (theta ** (j / d_axis))


def rope_tables(grid, split, theta: float = 10000.0, tokens=None):
    """Per-token angles for every pair of the head: array [L, D/2] float64.

    Pair i < d_t/2 turns by t'*f_t[i]; the next d_h/2 pairs by h*f_h[i]; the last
    d_w/2 pairs by w*f_w[i]; positions are patch-grid indices.  ``tokens``
    restricts the rows to those sequence positions."""
    Tg, Hg, Wg = grid
    L = Tg * Hg * Wg
    idx = np.arange(L) if tokens is None else np.asarray(tokens)
    t, h, w = grid_position(idx, grid)
    parts = []
    for pos, d in zip((t, h, w), split):
        parts.append(np.outer(pos.astype(np.float64), rope_inv_freq(d, theta)))
    return np.concatenate(parts, axis=1)


def rope_axis_phasors(grid, split, theta: float = 10000.0) -> np.ndarray:
    """The RoPE's unit phasors per axis position, float64 [n, 2] of (cos, sin):
    the d_t/2 x Tg time entries (pair-major: entry i*Tg + t'), then d_h/2 x Hg
    height entries, then d_w/2 x Wg width entries.  The towardsai snippet builds
    one frequency table per axis and looks each token's angles up by its t, h
    and w (section 4); this is that per-axis cache, before the lookup.  The
    order of entries is the library's layout, which the pages do not fix."""
    parts = []
    for n, d in zip(grid, split):
        ang = np.outer(rope_inv_freq(d, theta), np.arange(n, dtype=np.float64))   # [d/2, n]
        parts.append(np.stack([np.cos(ang), np.sin(ang)], axis=-1).reshape(-1, 2))
    return np.concatenate(parts, axis=0)


def rope_3d(x: np.ndarray, grid, split, theta: float = 10000.0, tokens=None) -> np.ndarray:
    """Rotate Q or K ``[B, L, heads, D]`` in float64.

    For pair p = (x[2p], x[2p+1]) with angle a: (x0*cos a - x1*sin a,
    x0*sin a + x1*cos a), i.e. the complex product (x0 + i x1) * e^{ia}.
    ``tokens`` gives the sequence positions of x's rows when x holds a subset."""
    B, L, Hh, D = x.shape
    check_split(D, split)
    if tokens is None and L != grid[0] * grid[1] * grid[2]:
        raise ValueError("sequence length does not match the token grid")
    ang = rope_tables(grid, split, theta, tokens)    # [L, D/2]
    c = np.cos(ang)[None, :, None, :]
    s = np.sin(ang)[None, :, None, :]
    x = np.asarray(x, dtype=np.float64)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def rms_norm(x: np.ndarray, group: int, weight=None, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm of ``[B, L, heads, D]`` in float64 over groups of ``group``
    consecutive channels of each token's heads*D channels:
    y = x / sqrt(mean(x^2 over the group) + eps) * weight[channel mod group]."""
    x = np.asarray(x, dtype=np.float64)
    B, L, Hh, D = x.shape
    if group <= 0 or (Hh * D) % group != 0:
        raise ValueError("group must divide heads * head_dim")
    w = np.ones(group) if weight is None else np.asarray(weight, dtype=np.float64)
    if w.shape != (group,):
        raise ValueError("weight must have one entry per channel of a group")
    g = x.reshape(B, L, (Hh * D) // group, group)
    ms = (g * g).mean(axis=-1, keepdims=True)
    return (g / np.sqrt(ms + eps) * w).reshape(B, L, Hh, D)


def qk_norm_rope_3d(x: np.ndarray, grid, split, group: int, weight=None, eps: float = 1e-6,
                    theta: float = 10000.0, tokens=None) -> np.ndarray:
    """RMSNorm (``rms_norm``) then the 3D rotation (``rope_3d``), both in float64:
    what attn1 does to Q and to K before the scores (towardsai section 5)."""
    return rope_3d(rms_norm(x, group, weight, eps), grid, split, theta, tokens)


def rope_3d_fp32(x32: np.ndarray, grid, split, theta: float = 10000.0, tokens=None) -> np.ndarray:
    """The same rotation at the towardsai snippet's own precision.

    The snippet builds angles in float64 and stores the phasors as complex64,
    so cos and sin are the float64 values rounded once to float32; the vector
    is float32 and the complex product is evaluated in float32.  Here every
    product and every sum is rounded to float32 on its own (no fused
    multiply-add):  re = fl(fl(x0*c) - fl(x1*s)),  im = fl(fl(x0*s) + fl(x1*c)).
    """
    B, L, Hh, D = x32.shape
    check_split(D, split)
    ang = rope_tables(grid, split, theta, tokens)
    c = np.cos(ang).astype(np.float32)[None, :, None, :]
    s = np.sin(ang).astype(np.float32)[None, :, None, :]
    x32 = np.asarray(x32, dtype=np.float32)
    x0 = x32[..., 0::2]
    x1 = x32[..., 1::2]
    out = np.empty_like(x32)
    out[..., 0::2] = (x0 * c) - (x1 * s)
    out[..., 1::2] = (x0 * s) + (x1 * c)
    return out


# ----------------------------------------------------------------------------
# Attention
# ----------------------------------------------------------------------------


def default_scale(head_dim: int) -> float:
    """Logit scale 1/sqrt(head_dim) (towardsai section 7)."""
    return 1.0 / math.sqrt(head_dim)


def _attend_rows(qr, kh, vh, scale, allowed=None):
    """softmax(scale * q k^T) v for a block of query rows of one (batch, head).

    Two passes over each row: the row maximum, then the exponentials, their sum
    and the weighted sum of values.  Returns (out, lse) with lse = m + log(sum)."""
    s = (qr @ kh.T) * scale
    if allowed is not None:
        s = np.where(allowed, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p @ vh) / l
    return o, (m + np.log(l))[:, 0]


def attention(q, k, v, scale=None, mask=None, rows=None, row_block: int = 1024):
    """O = softmax(scale * Q K^T) V per (batch, head), non-causal, in float64.

    q: [B, Lq, H, D]; k, v: [B, Lk, H, D].  ``mask`` is an optional boolean
    [Lq, Lk] array of allowed pairs.  ``rows`` restricts the computation to the
    given query rows (every row is an independent softmax, so a subset is
    exactly those rows of the full result).  Query rows are processed
    ``row_block`` at a time only to bound memory.

    Returns (o, lse): o [B, R, H, D] and lse [B, H, R] (natural log), where R is
    Lq or len(rows).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Lq, Hh, D = q.shape
    if scale is None or scale <= 0:
        scale = default_scale(D)
    sel = np.arange(Lq) if rows is None else np.asarray(rows)
    R = sel.size
    o = np.empty((B, R, Hh, v.shape[-1]), dtype=np.float64)
    lse = np.empty((B, Hh, R), dtype=np.float64)
    for b in range(B):
        for h in range(Hh):
            kh = k[b, :, h, :]
            vh = v[b, :, h, :]
            for r0 in range(0, R, row_block):
                rr = sel[r0:r0 + row_block]
                allowed = None if mask is None else mask[rr]
                ob, lb = _attend_rows(q[b, rr, h, :], kh, vh, scale, allowed)
                o[b, r0:r0 + rr.size, h, :] = ob
                lse[b, h, r0:r0 + rr.size] = lb
    return o, lse


def attention_probs_row(q, k, b: int, h: int, i: int, scale=None) -> np.ndarray:
    """The softmax row of query i for (batch b, head h): probabilities over all keys."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    if scale is None or scale <= 0:
        scale = default_scale(q.shape[-1])
    s = (k[b, :, h, :] @ q[b, i, h, :]) * scale
    p = np.exp(s - s.max())
    return p / p.sum()


def slice_mass(q, k, b: int, h: int, i: int, grid, scale=None) -> np.ndarray:
    """Attention mass of query i summed over each time slice t' (the probe of
    towardsai section 7): the softmax row reshaped to the token grid and summed
    over rows and columns.  Entries sum to one."""
    p = attention_probs_row(q, k, b, h, i, scale)
    return p.reshape(grid).sum(axis=(1, 2))


# ----------------------------------------------------------------------------
# Divided attention: a time pass, then a space pass
# ----------------------------------------------------------------------------


def divided_time(q, k, v, T: int, HW: int, scale=None):
    """Time pass: for each batch, spatial site s and head, attention over the T
    tokens {t*HW + s}.  Inputs and output [B, T*HW, H, D].  Returns (o, lse)
    with lse [B, H, T*HW] in the tokens' own positions."""
    q = np.asarray(q, dtype=np.float64)
    B, L, Hh, D = q.shape
    if L != T * HW:
        raise ValueError("L must equal T*HW")

    def to_seq(x):  # [B, T, HW, H, D] -> [B*HW, T, H, D]
        x = np.asarray(x, dtype=np.float64).reshape(B, T, HW, Hh, -1)
        return x.transpose(0, 2, 1, 3, 4).reshape(B * HW, T, Hh, -1)

    o, lse = attention(to_seq(q), to_seq(k), to_seq(v), scale)
    o = o.reshape(B, HW, T, Hh, -1).transpose(0, 2, 1, 3, 4).reshape(B, L, Hh, -1)
    lse = lse.reshape(B, HW, Hh, T).transpose(0, 2, 3, 1).reshape(B, Hh, L)
    return o, lse


def divided_space(q, k, v, T: int, HW: int, scale=None, frames=None):
    """Space pass: for each batch, frame t and head, attention over the HW tokens
    of frame t (a contiguous run of the sequence).  ``frames`` optionally limits
    the computation to some frames; the result then holds only those frames'
    tokens, in order.  Returns (o, lse), lse [B, H, tokens]."""
    q = np.asarray(q, dtype=np.float64)
    B, L, Hh, D = q.shape
    if L != T * HW:
        raise ValueError("L must equal T*HW")
    fr = np.arange(T) if frames is None else np.asarray(frames)

    def to_seq(x):  # selected frames -> [B*F, HW, H, D]
        x = np.asarray(x, dtype=np.float64).reshape(B, T, HW, Hh, -1)[:, fr]
        return x.reshape(B * fr.size, HW, Hh, -1)

    o, lse = attention(to_seq(q), to_seq(k), to_seq(v), scale)
    o = o.reshape(B, fr.size * HW, Hh, -1)
    lse = lse.reshape(B, fr.size, Hh, HW).transpose(0, 2, 1, 3).reshape(B, Hh, fr.size * HW)
    return o, lse


def divided_time_rows(q, k, v, T: int, HW: int, rows, scale=None):
    """Selected query rows of the time pass: the row at sequence position r
    attends over the T tokens {t*HW + r % HW} of its site.  q, k, v
    [B, T*HW, H, D]; returns (o [B, R, H, D], lse [B, H, R])."""
    rows = np.asarray(rows)
    B, L, Hh, D = np.shape(q)
    if scale is None or scale <= 0:
        scale = default_scale(D)
    keys = np.arange(T)[None, :] * HW + (rows % HW)[:, None]      # [R, T]
    o = np.empty((B, rows.size, Hh, np.shape(v)[-1]))
    lse = np.empty((B, Hh, rows.size))
    for b in range(B):
        for h in range(Hh):
            qr = np.asarray(q[b, rows, h, :], dtype=np.float64)           # [R, D]
            kr = np.asarray(k[b, keys, h, :], dtype=np.float64)           # [R, T, D]
            vr = np.asarray(v[b, keys, h, :], dtype=np.float64)
            s = np.einsum("rd,rtd->rt", qr, kr) * scale
            m = s.max(axis=1, keepdims=True)
            p = np.exp(s - m)
            l = p.sum(axis=1, keepdims=True)
            o[b, :, h, :] = np.einsum("rt,rtd->rd", p, vr) / l
            lse[b, h] = (m + np.log(l))[:, 0]
    return o, lse


def divided_space_rows(q, k, v, T: int, HW: int, rows, scale=None):
    """Selected query rows of the space pass: the row at position r attends over
    the HW tokens of its frame r // HW.  Returns (o [B, R, H, D], lse [B, H, R])."""
    rows = np.asarray(rows)
    B, L, Hh, D = np.shape(q)
    o = np.empty((B, rows.size, Hh, np.shape(v)[-1]))
    lse = np.empty((B, Hh, rows.size))
    frame = rows // HW
    for f in np.unique(frame):
        sel = np.nonzero(frame == f)[0]
        sl = slice(f * HW, (f + 1) * HW)
        of, lf = attention(q[:, sl], k[:, sl], v[:, sl], scale, rows=rows[sel] - f * HW)
        o[:, sel] = of
        lse[:, :, sel] = lf
    return o, lse


def time_mask(T: int, HW: int) -> np.ndarray:
    """Allowed pairs of the time pass within the full sequence: same spatial site."""
    site = np.arange(T * HW) % HW
    return site[:, None] == site[None, :]


def space_mask(T: int, HW: int) -> np.ndarray:
    """Allowed pairs of the space pass within the full sequence: same frame."""
    frame = np.arange(T * HW) // HW
    return frame[:, None] == frame[None, :]


# ----------------------------------------------------------------------------
# Harness set-up for the tiny clip (not a step of the hot path)
# ----------------------------------------------------------------------------


def project_tiny(tokens: np.ndarray, w_embed: np.ndarray, w_qkv: np.ndarray, heads: int):
    """Turn the tiny clip's tokens into Q, K, V in float64: x = tokens @ w_embed,
    [q|k|v] = x @ w_qkv, each split into ``heads`` heads.  The projection weights
    are random (no trained model is used); this only builds attention inputs of
    the tiny clip's shape.  Returns three [N, L, heads, width/heads] arrays."""
    x = np.asarray(tokens, dtype=np.float64) @ w_embed
    qkv = x @ w_qkv
    N, L, three_w = qkv.shape
    w = three_w // 3
    hd = w // heads
    q, k, v = (qkv[..., i * w:(i + 1) * w].reshape(N, L, heads, hd) for i in range(3))
    return q, k, v
