"""Python binding of libvdit.so: spacetime self-attention over video-DiT tokens.

A thin ctypes layer: it checks that tensors are CUDA, contiguous and of the
right dtype and shape, passes their device pointers, sizes and the current
CUDA stream to the C ABI declared in ``include/vdit.h``, and raises
:class:`VditError` on a nonzero status.  Every step of the path runs in the
library's kernels; there is no fallback.  PyTorch is used only for device
memory and streams (outputs are allocated with ``torch.empty`` when the caller
passes none).

Calls (see ``include/vdit.h`` for the exact definitions and sources):

* :func:`patchify_3d`         latent [N, C, T, H, W] -> tokens [N, L, C*pt*ph*pw]
* :func:`patch_embed_3d`      the Conv3d patch embedding: tokens @ weight^T + bias
* :func:`unpatchify_3d`       tokens [N, L, C*pt*ph*pw] -> latent [N, C, T, H, W]
* :func:`rope_3d`             3D rotary positions on Q and K [B, L, heads, D]
* :func:`qk_norm_rope_3d`     RMSNorm of Q and K, then the 3D rotation, in one pass
* :func:`rope_3d_table`       the 3D RoPE's (cos, sin) pairs per axis position
* :func:`attn_full`           full 3D self-attention
* :func:`attn_full_rope_q`    full 3D self-attention that normalises and rotates Q itself
* :func:`attn_divided_time`   attention over the T tokens of each spatial site
* :func:`attn_divided_space`  attention over the HW tokens of each frame
* :func:`attn_cross`          video tokens attending to a separate key/value sequence
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["VditError", "lib", "patchify_3d", "patch_embed_3d", "unpatchify_3d", "rope_3d",
           "qk_norm_rope_3d", "rope_3d_table", "attn_full", "attn_full_rope_q", "attn_divided_time", "attn_divided_space", "attn_cross",
           "device_status", "watchdog_selftest", "status_string", "default_split", "LIB_PATH"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libvdit.so")

F32, BF16 = 0, 1
_STATUS = {0: "VDIT_OK", 1: "VDIT_ERR_NULL", 2: "VDIT_ERR_SHAPE", 3: "VDIT_ERR_ALIGN",
           4: "VDIT_ERR_UNSUPPORTED", 5: "VDIT_ERR_CUDA", 6: "VDIT_ERR_TIMEOUT"}


class VditError(RuntimeError):
    """A libvdit call returned a nonzero status."""

    def __init__(self, call: str, status: int):
        self.status = status
        super().__init__(f"{call}: {_STATUS.get(status, status)} ({status_string(status)})")


_lib = None

_P, _I, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
_SIGNATURES = {
    "vdit_patchify_3d": [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P],
    "vdit_rope_3d": [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P],
    "vdit_attn_full": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _P],
    "vdit_rope_3d_table": [_P, _I, _I, _I, _I, _I, _I, _I, _F, _P],
    "vdit_attn_full_rope_q": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _I, _I, _I, _P, _P, _I, _F, _P],
    "vdit_patch_embed_3d": [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P],
    "vdit_unpatchify_3d": [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _I, _P],
    "vdit_qk_norm_rope_3d": [_P, _P, _P, _P, _P, _P, _I, _F, _I, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P],
    "vdit_attn_divided_time": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P],
    "vdit_attn_divided_space": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P],
    "vdit_attn_cross": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P],
    "vdit_device_status": [ctypes.POINTER(ctypes.c_uint)],
    "vdit_watchdog_selftest": [_I, _P],
    "vdit_version": [],
}


def lib() -> ctypes.CDLL:
    """The loaded library; raises if libvdit.so has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libvdit.so not built at {LIB_PATH}: run "
                              "`python -m spacetime_attention_vdit_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        L.vdit_rope_3d_table_entries.argtypes = [_I] * 7
        L.vdit_rope_3d_table_entries.restype = ctypes.c_longlong
        L.vdit_status_string.argtypes = [ctypes.c_int]
        L.vdit_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().vdit_status_string(int(status)).decode()


def _check(call: str, rc: int) -> None:
    if rc != 0:
        raise VditError(call, rc)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, name: str, dtype=None) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def default_split(head_dim: int):
    """(44, 42, 42) for head_dim 128: time takes the remainder, height and width
    2*floor(head_dim/6) each."""
    s = 2 * (head_dim // 6)
    return (head_dim - 2 * s, s, s)


def patchify_3d(latent: torch.Tensor, patch=(1, 2, 2), out: torch.Tensor | None = None, stream=None):
    """Cut ``latent`` [N, C, T, H, W] (float32 or bfloat16) into (pt, ph, pw) bricks;
    returns tokens [N, Tg*Hg*Wg, C*pt*ph*pw] of the same dtype."""
    if latent.dim() != 5:
        raise ValueError("latent must be [N, C, T, H, W]")
    dt = {torch.float32: F32, torch.bfloat16: BF16}.get(latent.dtype)
    if dt is None:
        raise ValueError("latent must be float32 or bfloat16")
    N, C, T, H, W = latent.shape
    pt, ph, pw = patch
    L = (T // pt) * (H // ph) * (W // pw)
    F = C * pt * ph * pw
    if out is None:
        out = torch.empty((N, L, F), dtype=latent.dtype, device=latent.device)
    elif tuple(out.shape) != (N, L, F):
        raise ValueError(f"out must be {(N, L, F)}")
    _check("vdit_patchify_3d", lib().vdit_patchify_3d(
        _dev(latent, "latent"), _dev(out, "out", latent.dtype), dt, N, C, T, H, W, pt, ph, pw, _stream(stream)))
    return out


def _q_and_out(q, k, q_out, inplace):
    """Q's input and output pointers; both None when only K is rotated."""
    if q is None:
        return None, None, None
    if q.dim() != 4 or q.shape != k.shape:
        raise ValueError("q and k must both be [B, L, heads, head_dim]")
    if inplace:
        q_out = q
    q_out = torch.empty_like(q) if q_out is None else q_out
    return _dev(q, "q", torch.bfloat16), _dev(q_out, "q_out", torch.bfloat16), q_out


def rope_3d(q: torch.Tensor | None, k: torch.Tensor, grid, split=None, theta: float = 10000.0,
            q_out: torch.Tensor | None = None, k_out: torch.Tensor | None = None, inplace: bool = False,
            stream=None):
    """Rotate Q and K ([B, L, heads, D] bfloat16, L = Tg*Hg*Wg) by their 3D grid
    positions.  ``split`` = (d_t, d_h, d_w), default :func:`default_split`.
    Returns (q_out, k_out); with ``inplace`` the inputs are overwritten.  With
    ``q=None`` only K is rotated (for :func:`attn_full_rope_q`) and q_out is None."""
    if k.dim() != 4:
        raise ValueError("k must be [B, L, heads, head_dim]")
    B, L, Hh, D = k.shape
    Tg, Hg, Wg = grid
    if Tg * Hg * Wg != L:
        raise ValueError("grid does not match the sequence length")
    d_t, d_h, d_w = default_split(D) if split is None else split
    qp, qop, q_out = _q_and_out(q, k, q_out, inplace)
    if inplace:
        k_out = k
    k_out = torch.empty_like(k) if k_out is None else k_out
    _check("vdit_rope_3d", lib().vdit_rope_3d(
        qp, _dev(k, "k", torch.bfloat16), qop, _dev(k_out, "k_out", torch.bfloat16),
        B, Tg, Hg, Wg, Hh, D, d_t, d_h, d_w, float(theta), _stream(stream)))
    return q_out, k_out


def rope_3d_table(grid, head_dim: int, split=None, theta: float = 10000.0, out=None, device=None, stream=None):
    """The 3D RoPE's (cos, sin) pairs per axis position, float32 [n, 2] on the
    device, pair-major within each axis: time [d_t/2][Tg], then height
    [d_h/2][Hg], then width [d_w/2][Wg] (the layout ``include/vdit.h`` gives for
    vdit_rope_3d_table).  The input of
    :func:`attn_full_rope_q`; it depends only on the grid, the split and theta."""
    Tg, Hg, Wg = grid
    d_t, d_h, d_w = default_split(head_dim) if split is None else split
    n = lib().vdit_rope_3d_table_entries(Tg, Hg, Wg, head_dim, d_t, d_h, d_w)
    if n < 0:
        raise ValueError("bad grid or split")
    if out is None:
        out = torch.empty((max(n, 1), 2), dtype=torch.float32,
                          device=device if device is not None else torch.device("cuda", torch.cuda.current_device()))
    elif out.dtype != torch.float32 or out.numel() < 2 * n:
        raise ValueError(f"out must be float32 with at least {2 * n} elements")
    _check("vdit_rope_3d_table", lib().vdit_rope_3d_table(
        _dev(out, "out", torch.float32), Tg, Hg, Wg, head_dim, d_t, d_h, d_w, float(theta), _stream(stream)))
    return out[:n]


def patch_embed_3d(latent: torch.Tensor, weight: torch.Tensor, patch=(1, 2, 2), bias=None, out=None,
                   stream=None):
    """The Conv3d patch embedding on the tensor cores: latent float32 [N, C, T, H, W],
    weight bfloat16 [dim, C*pt*ph*pw] (or the Conv3d's [dim, C, pt, ph, pw]),
    bias float32 [dim] or None -> bfloat16 [N, L, dim]."""
    if latent.dim() != 5:
        raise ValueError("latent must be [N, C, T, H, W]")
    N, C, T, H, W = latent.shape
    pt, ph, pw = patch
    w = weight.reshape(weight.shape[0], -1)
    dim = w.shape[0]
    L = (T // pt) * (H // ph) * (W // pw)
    if out is None:
        out = torch.empty((N, L, dim), dtype=torch.bfloat16, device=latent.device)
    elif tuple(out.shape) != (N, L, dim):
        raise ValueError(f"out must be {(N, L, dim)}")
    _check("vdit_patch_embed_3d", lib().vdit_patch_embed_3d(
        _dev(latent, "latent", torch.float32), _dev(w, "weight", torch.bfloat16),
        None if bias is None else _dev(bias, "bias", torch.float32), _dev(out, "out", torch.bfloat16),
        N, C, T, H, W, pt, ph, pw, dim, _stream(stream)))
    return out


def unpatchify_3d(tokens: torch.Tensor, C: int, grid, patch=(1, 2, 2), out=None, stream=None):
    """Tokens [N, Tg*Hg*Wg, C*pt*ph*pw] (float32 or bfloat16) back to the latent
    [N, C, Tg*pt, Hg*ph, Wg*pw]: the inverse of :func:`patchify_3d`."""
    if tokens.dim() != 3:
        raise ValueError("tokens must be [N, L, features]")
    N, L, F = tokens.shape
    Tg, Hg, Wg = grid
    pt, ph, pw = patch
    if L != Tg * Hg * Wg or F != C * pt * ph * pw:
        raise ValueError("tokens do not match the grid and the brick")
    dt = {torch.float32: 0, torch.bfloat16: 1}.get(tokens.dtype)
    if dt is None:
        raise ValueError("tokens must be float32 or bfloat16")
    shape = (N, C, Tg * pt, Hg * ph, Wg * pw)
    if out is None:
        out = torch.empty(shape, dtype=tokens.dtype, device=tokens.device)
    elif tuple(out.shape) != shape:
        raise ValueError(f"out must be {shape}")
    _check("vdit_unpatchify_3d", lib().vdit_unpatchify_3d(
        _dev(tokens, "tokens", tokens.dtype), _dev(out, "out", tokens.dtype), dt, N, C, Tg, Hg, Wg, pt, ph, pw,
        _stream(stream)))
    return out


def qk_norm_rope_3d(q: torch.Tensor | None, k: torch.Tensor, grid, norm_group: int, wq=None, wk=None,
                    eps: float = 1e-6, split=None, theta: float = 10000.0, q_out=None, k_out=None,
                    inplace: bool = False, stream=None):
    """RMSNorm of Q and K over groups of ``norm_group`` channels of each token
    (head_dim: per head; heads*head_dim: the whole token), weights ``wq``/``wk``
    (float32 [norm_group] on the device, or None for 1), then the 3D rotation of
    :func:`rope_3d`, in one pass.  Returns (q_out, k_out); ``q=None``: K only."""
    if k.dim() != 4:
        raise ValueError("k must be [B, L, heads, head_dim]")
    B, L, Hh, D = k.shape
    Tg, Hg, Wg = grid
    if Tg * Hg * Wg != L:
        raise ValueError("grid does not match the sequence length")
    d_t, d_h, d_w = default_split(D) if split is None else split
    qp, qop, q_out = _q_and_out(q, k, q_out, inplace)
    if inplace:
        k_out = k
    k_out = torch.empty_like(k) if k_out is None else k_out
    w_ptrs = []
    for w, name in ((wq, "wq"), (wk, "wk")):
        if w is None:
            w_ptrs.append(None)
        else:
            if tuple(w.shape) != (norm_group,):
                raise ValueError(f"{name} must have norm_group entries")
            w_ptrs.append(_dev(w, name, torch.float32))
    _check("vdit_qk_norm_rope_3d", lib().vdit_qk_norm_rope_3d(
        qp, _dev(k, "k", torch.bfloat16), qop,
        _dev(k_out, "k_out", torch.bfloat16), w_ptrs[0], w_ptrs[1], int(norm_group), float(eps),
        B, Tg, Hg, Wg, Hh, D, d_t, d_h, d_w, float(theta), _stream(stream)))
    return q_out, k_out


def _attn_io(q, k, v, out, lse, cross=False):
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape:
        raise ValueError("q, k and v must be [B, L, heads, head_dim], k and v of one shape")
    if (q.shape != k.shape) if not cross else (q.shape[0] != k.shape[0] or q.shape[2:] != k.shape[2:]):
        raise ValueError("q and k must agree in batch, heads and head_dim" if cross
                         else "q, k and v must all be [B, L, heads, head_dim]")
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _dev(t, n, torch.bfloat16)
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape:
        raise ValueError("out must have q's shape")
    B, L, Hh, D = q.shape
    lse_t = None
    if lse is True:
        lse_t = torch.empty((B, Hh, L), dtype=torch.float32, device=q.device)
    elif isinstance(lse, torch.Tensor):
        if tuple(lse.shape) != (B, Hh, L):
            raise ValueError(f"lse must be {(B, Hh, L)}")
        lse_t = lse
    lse_p = None if lse_t is None else _dev(lse_t, "lse", torch.float32)
    return out, lse_t, lse_p


def attn_full(q, k, v, out=None, lse=None, scale: float = 0.0, stream=None):
    """O = softmax(scale Q K^T) V over all L tokens of each (batch, head).
    ``lse=True`` also returns the float32 [B, heads, L] log-sum-exp."""
    out, lse_t, lse_p = _attn_io(q, k, v, out, lse)
    B, L, Hh, D = q.shape
    _check("vdit_attn_full", lib().vdit_attn_full(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), _dev(out, "out", torch.bfloat16), lse_p, B, L, Hh, D,
        float(scale), _stream(stream)))
    return out if lse_t is None else (out, lse_t)


def attn_full_rope_q(q, k, v, grid, table, split=None, wq=None, norm_group: int = 0, eps: float = 1e-6,
                     out=None, lse=None, scale: float = 0.0, stream=None):
    """Full 3D self-attention with Q as projected: the kernel applies the per-head
    RMSNorm (``norm_group`` = head_dim, weight ``wq`` float32 [head_dim] or None;
    0: no norm) and the 3D rotation to Q in its prologue, with the pairs of
    ``table`` (:func:`rope_3d_table` of the same grid and split).  K must already
    be normalised and rotated (:func:`rope_3d` / :func:`qk_norm_rope_3d` with
    ``q=None``).  ``lse=True`` also returns [B, heads, L]."""
    Tg, Hg, Wg = grid
    if q.dim() != 4 or Tg * Hg * Wg != q.shape[1]:
        raise ValueError("grid does not match the sequence length")
    out, lse_t, lse_p = _attn_io(q, k, v, out, lse)
    B, L, Hh, D = q.shape
    d_t, d_h, d_w = default_split(D) if split is None else split
    wp = None
    if wq is not None:
        if tuple(wq.shape) != (D,):
            raise ValueError("wq must have head_dim entries")
        wp = _dev(wq, "wq", torch.float32)
    _check("vdit_attn_full_rope_q", lib().vdit_attn_full_rope_q(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), _dev(out, "out", torch.bfloat16), lse_p, B, Tg, Hg, Wg, Hh, D,
        float(scale), d_t, d_h, d_w, _dev(table, "table", torch.float32), wp, int(norm_group), float(eps),
        _stream(stream)))
    return out if lse_t is None else (out, lse_t)


def attn_cross(q, k, v, out=None, lse=None, scale: float = 0.0, stream=None):
    """Cross-attention: q [B, Lq, heads, D] over k, v [B, Lk, heads, D] (the video
    tokens attending to the text tokens).  ``lse=True`` also returns [B, heads, Lq]."""
    out, lse_t, lse_p = _attn_io(q, k, v, out, lse, cross=True)
    B, Lq, Hh, D = q.shape
    Lk = k.shape[1]
    _check("vdit_attn_cross", lib().vdit_attn_cross(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), _dev(out, "out", torch.bfloat16), lse_p, B, Lq, Lk, Hh, D,
        float(scale), _stream(stream)))
    return out if lse_t is None else (out, lse_t)


def _divided(name, q, k, v, T, HW, out, lse, scale, stream):
    out, lse_t, lse_p = _attn_io(q, k, v, out, lse)
    B, L, Hh, D = q.shape
    if T * HW != L:
        raise ValueError("L must equal T * HW")
    _check(name, getattr(lib(), name)(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), _dev(out, "out", torch.bfloat16), lse_p, B, T, HW, Hh, D,
        float(scale), _stream(stream)))
    return out if lse_t is None else (out, lse_t)


def attn_divided_time(q, k, v, T: int, HW: int, out=None, lse=None, scale: float = 0.0, stream=None):
    """Time pass: attention over the T tokens {t*HW + s} of each site s."""
    return _divided("vdit_attn_divided_time", q, k, v, T, HW, out, lse, scale, stream)


def attn_divided_space(q, k, v, T: int, HW: int, out=None, lse=None, scale: float = 0.0, stream=None):
    """Space pass: attention over the HW tokens of each frame t."""
    return _divided("vdit_attn_divided_space", q, k, v, T, HW, out, lse, scale, stream)


def device_status():
    """(status, flags) of the kernels' bounded waits since the last call; synchronises."""
    flags = ctypes.c_uint(0)
    rc = lib().vdit_device_status(ctypes.byref(flags))
    return rc, flags.value


def watchdog_selftest(site: int = 99) -> None:
    """Enqueue the library's failure-detection self-check on the current CUDA
    stream: a kernel whose one bounded wait can never complete runs out after
    the 2-second limit and records ``site`` in the device flags, which the next
    :func:`device_status` reports (VDIT_ERR_TIMEOUT) and clears."""
    rc = lib().vdit_watchdog_selftest(int(site), _stream(None))
    if rc != 0:
        raise VditError("vdit_watchdog_selftest", rc)
