"""GPU parity of full and divided attention against the float64 oracle.

Small cases are compared on every row; the 81-frame 480p and 720p clips on
4,096 seeded query rows per (batch, head).  Tolerances: tests/gpu_util.py."""
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


def f64(bits):
    return synthetic.bf16_bits_to_f64(bits)


# --------------------------------------------------------------------------- the tiny clip

def tiny_qkv():
    """latent [1,4,8,16,16] seed 0 -> (1,2,2) patches (512 tokens of 16) ->
    random projection to width 64 -> 2 heads of 32 -> bf16 Q, K, V."""
    lat = synthetic.latent_f32(1, 4, 8, 16, 16, seed=0)
    tok = ref.patchify(lat, 1, 2, 2)
    we, wq = synthetic.tiny_weights(16, 64, seed=0)
    q, k, v = ref.project_tiny(tok, we, wq, heads=2)
    return tuple(synthetic.f64_to_bf16_bits(x) for x in (q, k, v))


def test_tiny_full():
    import spacetime_attention_vdit_b200 as v_
    q, k, v = tiny_qkv()
    o, lse = v_.attn_full(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), lse=True)
    eo, el = ref.attention(f64(q), f64(k), f64(v))
    assert_attention_close(dev_f64(o), eo, lse.cpu().numpy(), el, "tiny full")


def test_tiny_time_pass():
    import spacetime_attention_vdit_b200 as v_
    q, k, v = tiny_qkv()
    o, lse = v_.attn_divided_time(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), 8, 64, lse=True)
    eo, el = ref.divided_time(f64(q), f64(k), f64(v), 8, 64)
    assert_attention_close(dev_f64(o), eo, lse.cpu().numpy(), el, "tiny time")


def test_tiny_space_pass():
    import spacetime_attention_vdit_b200 as v_
    q, k, v = tiny_qkv()
    o, lse = v_.attn_divided_space(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), 8, 64, lse=True)
    eo, el = ref.divided_space(f64(q), f64(k), f64(v), 8, 64)
    assert_attention_close(dev_f64(o), eo, lse.cpu().numpy(), el, "tiny space")


def test_tiny_divided_equals_masked_full():
    """The GPU time pass matches the oracle's full attention under the same-site
    mask, and the space pass under the same-frame mask."""
    import spacetime_attention_vdit_b200 as v_
    q, k, v = tiny_qkv()
    Q, K, V = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    for fn, mask in ((v_.attn_divided_time, ref.time_mask(8, 64)), (v_.attn_divided_space, ref.space_mask(8, 64))):
        o = fn(Q, K, V, 8, 64)
        eo, _ = ref.attention(f64(q), f64(k), f64(v), mask=mask)
        assert_attention_close(dev_f64(o), eo, what=fn.__name__)


# --------------------------------------------------------------------------- edge cases

@pytest.mark.parametrize("B,L,H,D", [
    (2, 1, 2, 128),        # a single key: O = V
    (1, 127, 2, 128),      # one short tile
    (1, 128, 1, 128),      # exactly one tile
    (1, 129, 3, 64),       # one row into the second tile
    (2, 200, 2, 32),
    (1, 300, 1, 128),
    (1, 1000, 2, 128),     # several tiles and a ragged tail
    (1, 2048, 1, 128),     # 16 key tiles: the last length whose O is staged for TMA stores
    (1, 2100, 1, 64),      # 17 key tiles: per-row stores
])
def test_full_ragged(B, L, H, D):
    import spacetime_attention_vdit_b200 as v_
    q, k, v = synthetic.qkv_bf16(B, L, H, D, seed=L)
    o, lse = v_.attn_full(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), lse=True)
    eo, el = ref.attention(f64(q), f64(k), f64(v))
    assert_attention_close(dev_f64(o), eo, lse.cpu().numpy(), el, f"full {B, L, H, D}")
    if L == 1:
        assert np.array_equal(from_dev_bf16(o), v)


@pytest.mark.parametrize("q_scale", [4.0, 12.0])
def test_full_sharp(q_scale):
    """Q scaled up: peaked softmax rows, max that moves between tiles (rescaling path)."""
    import spacetime_attention_vdit_b200 as v_
    q, k, v = synthetic.qkv_bf16(1, 1000, 2, 128, seed=7, q_scale=q_scale)
    o, lse = v_.attn_full(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), lse=True)
    eo, el = ref.attention(f64(q), f64(k), f64(v))
    assert_attention_close(dev_f64(o), eo, lse.cpu().numpy(), el, f"sharp x{q_scale}")


def test_full_explicit_scale():
    import spacetime_attention_vdit_b200 as v_
    q, k, v = synthetic.qkv_bf16(1, 300, 2, 64, seed=8)
    o = v_.attn_full(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), scale=0.3)
    eo, _ = ref.attention(f64(q), f64(k), f64(v), scale=0.3)
    assert_attention_close(dev_f64(o), eo, what="scale 0.3")


def test_full_constant_keys():
    """Identical keys: every output row is the mean of V."""
    import spacetime_attention_vdit_b200 as v_
    q, _, v = synthetic.qkv_bf16(1, 260, 2, 128, seed=9)
    k = np.repeat(synthetic.qkv_bf16(1, 1, 2, 128, seed=10)[1], 260, axis=1)
    o = v_.attn_full(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v))
    mean = f64(v).mean(axis=1, keepdims=True).repeat(260, axis=1)
    assert_attention_close(dev_f64(o), mean, what="constant keys")


@pytest.mark.parametrize("T,HW,H,D", [
    (1, 5, 2, 128),        # one frame: the time pass returns V
    (8, 64, 2, 32),
    (16, 9, 2, 128),
    (17, 7, 3, 128),
    (21, 13, 2, 128),      # the 81-frame latent length (24-row boxes)
    (21, 6, 1, 64),
    (23, 4, 2, 32),
    (24, 5, 2, 128),
    (25, 3, 2, 64),
    (32, 5, 2, 128),
    (33, 4, 2, 128),       # 48-row boxes, three m-tiles
    (40, 3, 2, 64),
    (48, 3, 1, 128),
    (64, 3, 1, 32),
    (65, 3, 2, 128),       # long clip: tensor-core kernel over a strided view
    (150, 2, 1, 128),
])
def test_time_pass_shapes(T, HW, H, D):
    import spacetime_attention_vdit_b200 as v_
    q, k, v = synthetic.qkv_bf16(2, T * HW, H, D, seed=T * 100 + HW)
    o, lse = v_.attn_divided_time(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), T, HW, lse=True)
    eo, el = ref.divided_time(f64(q), f64(k), f64(v), T, HW)
    assert_attention_close(dev_f64(o), eo, lse.cpu().numpy(), el, f"time {T, HW, H, D}")
    if T == 1:
        assert np.array_equal(from_dev_bf16(o), v)


@pytest.mark.parametrize("T,HW,H,D", [
    (5, 1, 2, 128),        # one site per frame: the space pass returns V
    (8, 64, 2, 32),
    (3, 130, 2, 128),
    (4, 300, 1, 64),
])
def test_space_pass_shapes(T, HW, H, D):
    import spacetime_attention_vdit_b200 as v_
    q, k, v = synthetic.qkv_bf16(2, T * HW, H, D, seed=T * 1000 + HW)
    o, lse = v_.attn_divided_space(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v), T, HW, lse=True)
    eo, el = ref.divided_space(f64(q), f64(k), f64(v), T, HW)
    assert_attention_close(dev_f64(o), eo, lse.cpu().numpy(), el, f"space {T, HW, H, D}")
    if HW == 1:
        assert np.array_equal(from_dev_bf16(o), v)


# --------------------------------------------------------------------------- 17 frames at 480p

def roped(bits, grid, tokens=None):
    """The oracle's RoPE at the page's precision, stored as bf16 like the path does."""
    x32 = synthetic.bf16_bits_to_f32(bits)
    return synthetic.f32_to_bf16_bits(ref.rope_3d_fp32(x32, grid, ref.default_split(bits.shape[-1]),
                                                       tokens=tokens))


def test_480p_17_frames_rope_full_attention():
    """7,800 tokens (grid 5x30x52), 12 heads x 128: RoPE then full attention, every row."""
    import spacetime_attention_vdit_b200 as v_
    grid = (5, 30, 52)
    q, k, v = synthetic.qkv_bf16(1, 7800, 12, 128, seed=0)
    qd, kd = v_.rope_3d(to_dev_bf16(q), to_dev_bf16(k), grid)
    o, lse = v_.attn_full(qd, kd, to_dev_bf16(v), lse=True)
    eo, el = ref.attention(f64(roped(q, grid)), f64(roped(k, grid)), f64(v))
    assert_attention_close(dev_f64(o), eo, lse.cpu().numpy(), el, "480p 17 frames")


# --------------------------------------------------------------------------- full-size clips

def _sampled_full(B, grid, H, seed=0, rows_per_head=4096):
    import spacetime_attention_vdit_b200 as v_
    L = grid[0] * grid[1] * grid[2]
    q, k, v = synthetic.qkv_bf16(B, L, H, 128, seed=seed)
    qd, kd = v_.rope_3d(to_dev_bf16(q), to_dev_bf16(k), grid, inplace=True)
    o, lse = v_.attn_full(qd, kd, to_dev_bf16(v), lse=True)
    rows = synthetic.sample_rows(L, rows_per_head, seed=seed)
    og = from_dev_bf16(o[:, rows])
    lg = lse[:, :, rows].cpu().numpy()
    del o, lse, qd, kd
    worst = (0.0, 0.0, 0.0)
    for h in range(H):
        kh = f64(roped(k[:, :, h:h + 1], grid))
        qh = f64(roped(q[:, rows, h:h + 1], grid, tokens=rows))
        eo, el = ref.attention(qh, kh, f64(v[:, :, h:h + 1]), rows=None)
        r = assert_attention_close(f64(og[:, :, h:h + 1]), eo, lg[:, h:h + 1], el, f"head {h}")
        worst = tuple(max(a, b) for a, b in zip(worst, r))
    return worst


def test_480p_81_frames_cfg_pair_sampled():
    """32,760 tokens (21x30x52), 40 heads x 128, batch 2: 4,096 rows per (batch, head)."""
    _sampled_full(2, (21, 30, 52), 40)


def test_720p_81_frames_sampled():
    """75,600 tokens (21x45x80), 40 heads x 128: 4,096 rows per head."""
    _sampled_full(1, (21, 45, 80), 40)


def _sampled_divided(B, T, HW, H, seed=0, rows_per_head=4096):
    """Both divided passes on [B, T*HW, H, 128] seeded inputs, compared with the
    oracle on `rows_per_head` seeded rows of every (batch, head)."""
    import spacetime_attention_vdit_b200 as v_
    q, k, v = synthetic.qkv_bf16(B, T * HW, H, 128, seed=seed)
    Q, K, V = to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(v)
    ot, lt = v_.attn_divided_time(Q, K, V, T, HW, lse=True)
    os_, ls = v_.attn_divided_space(Q, K, V, T, HW, lse=True)
    rows = synthetic.sample_rows(T * HW, rows_per_head, seed=seed)
    ot_g, lt_g = from_dev_bf16(ot[:, rows]), lt[:, :, rows].cpu().numpy()
    os_g, ls_g = from_dev_bf16(os_[:, rows]), ls[:, :, rows].cpu().numpy()
    del Q, K, V, ot, lt, os_, ls
    for h in range(H):
        qh, kh, vh = f64(q[:, :, h:h + 1]), f64(k[:, :, h:h + 1]), f64(v[:, :, h:h + 1])
        eo, el = ref.divided_time_rows(qh, kh, vh, T, HW, rows)
        assert_attention_close(f64(ot_g[:, :, h:h + 1]), eo, lt_g[:, h:h + 1], el, f"time head {h}")
        eo, el = ref.divided_space_rows(qh, kh, vh, T, HW, rows)
        assert_attention_close(f64(os_g[:, :, h:h + 1]), eo, ls_g[:, h:h + 1], el, f"space head {h}")


def test_720p_divided_sampled():
    """Divided attention at 720p: time pass (3,600 sites x 21 frames) and space pass
    (21 frames x 3,600 sites), 40 heads, 4,096 rows per head each."""
    _sampled_divided(1, 21, 3600, 40)


def test_480p_81_frames_cfg_pair_divided_sampled():
    """The divided passes at the shape the bench times: batch 2 (CFG pair), 21
    frames of 1,560 sites (30x52), 40 heads x 128; 4,096 rows per (batch, head).
    The space pass sweeps 13 key tiles per frame, so it runs the variant that
    stages O for TMA stores; the time pass uses 24-row boxes."""
    _sampled_divided(2, 21, 1560, 40)
