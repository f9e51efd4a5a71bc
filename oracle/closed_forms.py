"""Closed forms the pages state for clip sizes, token counts and costs.

Sources (page title, section):

* "How AI Generates Video: Inside Sora and Wan2.1 on a Real GPU"
  (towardsai.com), sections 2 "The 4D Data Explosion and the 1.046 Quadrillion
  Attention Wall", 3 "Inside the 3D Causal VAE", 4 "Spacetime Tubes and 3D
  Factorized RoPE" and 7 "Probing the [7800 x 7800] Matrix".
* "Video Diffusion Models, in depth" (aicassindra.com), "Step 1: compress with
  a causal 3D VAE", "Step 2: patchify into spacetime tokens" (token counter and
  FLOP estimator), "Training: flow matching on long sequences" (activation size).
* "Video and 3D Generation" cheatsheet (aiengineeringfromscratch.com),
  "Formulas and numbers": video tokens and divided attention.
* "Video as a 3D signal" (denimpatel.github.io), "Patches and attention" and
  "The token budget": factorised cost as a sum of two quadratics.
"""
from __future__ import annotations


def latent_frames(frames: int, t_stride: int = 4) -> int:
    """Latent length of a causal video VAE: frame 0 is kept alone, then every
    ``t_stride`` frames become one latent frame, T' = 1 + (T-1)/t_stride
    (towardsai, section 3; aicassindra, Step 1).  Integer division as in the
    aicassindra token counter."""
    return 1 + (frames - 1) // t_stride


def token_grid(T: int, H: int, W: int, pt: int, ph: int, pw: int):
    """Patch grid (T/pt, H/ph, W/pw), flooring like a stride-equals-kernel
    convolution (cheatsheet "Video tokens"; aicassindra Step 2 uses ``//``)."""
    return (T // pt, H // ph, W // pw)


def video_tokens(frames: int, height: int, width: int,
                 vae_stride=(4, 8, 8), patch=(1, 2, 2)) -> int:
    """Tokens per clip from pixel sizes: causal-VAE latent, then (1,2,2) patches
    (aicassindra, Step 2)."""
    t_lat = latent_frames(frames, vae_stride[0])
    h_lat, w_lat = height // vae_stride[1], width // vae_stride[2]
    tg, hg, wg = token_grid(t_lat, h_lat, w_lat, *patch)
    return tg * hg * wg


def flat_index(t: int, h: int, w: int, grid) -> int:
    """Sequence position of token (t', h, w): time-major, then rows, then columns
    (towardsai, section 7: 2*1560 + 18*52 + 26 = 4082 for grid (5, 30, 52))."""
    _, hg, wg = grid
    return t * hg * wg + h * wg + w


def grid_position(idx: int, grid):
    """Inverse of :func:`flat_index`."""
    _, hg, wg = grid
    return idx // (hg * wg), (idx // wg) % hg, idx % wg


def full_pairs(T: int, HW: int) -> int:
    """Query-key pairs of full 3D attention, (T*HW)^2 (cheatsheet "Divided attention")."""
    return (T * HW) ** 2


def divided_pairs(T: int, HW: int) -> int:
    """Pairs of divided attention: a length-T pass at each of HW sites plus a
    length-HW pass in each of T frames, HW*T^2 + T*HW^2 (cheatsheet "Divided
    attention"; "Video as a 3D signal", "Patches and attention")."""
    return HW * T * T + T * HW * HW


def attention_flops(B: int, heads: int, Lq: int, Lk: int, head_dim: int) -> int:
    """Algorithmic FLOPs of softmax(QK^T)V: 2*Lq*Lk*D for QK^T plus 2*Lq*Lk*D for
    PV per (batch, head) - the estimator's 4*tokens^2*dim (aicassindra, Step 2)."""
    return 4 * B * heads * Lq * Lk * head_dim


def estimator(tokens: int, params: float = 14e9, layers: int = 40, dim: int = 5120):
    """The order-of-magnitude forward estimator of aicassindra, Step 2: dense FLOPs
    2*params*tokens and attention FLOPs 4*tokens^2*dim*layers."""
    dense = 2 * params * tokens
    attn = 4 * tokens * tokens * dim * layers
    return dense, attn

