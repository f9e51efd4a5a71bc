"""Pins of oracle/closed_forms.py against the numbers the pages print."""
import numpy as np
import pytest

from oracle import closed_forms as cf
from oracle import reference as ref


def val(page_numbers, key, cast=int):
    return cast(page_numbers[key][0])


def test_latent_frames(page_numbers):
    assert cf.latent_frames(81) == val(page_numbers, "latent_frames_81")
    assert cf.latent_frames(17) == val(page_numbers, "latent_frames_17")
    # every 4k+1 length maps to k+1 latent frames
    for k in range(0, 40):
        assert cf.latent_frames(4 * k + 1) == k + 1


def test_latent_float_counts(page_numbers):
    assert 16 * cf.latent_frames(81) * (480 // 8) * (832 // 8) == val(page_numbers, "latent_floats_81")
    assert 16 * cf.latent_frames(17) * (480 // 8) * (832 // 8) == val(page_numbers, "latent_floats_17")
    assert 81 * 832 * 480 == val(page_numbers, "pixels_81_480p")


def test_token_counts(page_numbers):
    assert cf.video_tokens(17, 480, 832) == val(page_numbers, "tokens_17_480p")
    assert cf.video_tokens(81, 480, 832) == val(page_numbers, "tokens_81_480p")
    assert cf.video_tokens(81, 720, 1280) == val(page_numbers, "tokens_81_720p")
    g = cf.token_grid(21, 60, 104, 1, 2, 2)
    assert g == (21, 30, 52)
    assert g[1] * g[2] == val(page_numbers, "tokens_per_slice_480p")
    assert cf.token_grid(21, 90, 160, 1, 2, 2) == (21, 45, 80)


def test_tokens_agree_with_patchify(page_numbers):
    """The counter and the patchify gather agree on shapes (the grid the tiny
    model prints, and the brick size of the Wan2.1 latents)."""
    tiny = ref.patchify(np.zeros((1, 4, 8, 16, 16)), 2, 2, 2)
    assert tiny.shape == (1, val(page_numbers, "tiny_tokens"), val(page_numbers, "tiny_brick"))
    assert cf.token_grid(8, 16, 16, 2, 2, 2) == tuple(int(x) for x in page_numbers["tiny_grid"][0].split(","))
    wan = ref.patchify(np.zeros((1, 16, 5, 60, 104), dtype=np.float32), 1, 2, 2)
    assert wan.shape == (1, val(page_numbers, "tokens_17_480p"), val(page_numbers, "brick_floats"))


def test_flat_index(page_numbers):
    grid = (5, 30, 52)
    assert cf.flat_index(2, 18, 26, grid) == val(page_numbers, "flat_index_2_18_26")
    for idx in (0, 1, 51, 52, 1559, 1560, 4082, 7799):
        assert cf.flat_index(*cf.grid_position(idx, grid), grid) == idx


def test_pair_counts(page_numbers):
    assert cf.full_pairs(21, 1560) == val(page_numbers, "pairs_32760")
    raw = val(page_numbers, "pixels_81_480p") ** 2
    assert raw == val(page_numbers, "pairs_raw_81_480p")
    ratio = raw / cf.full_pairs(21, 1560)
    assert round(ratio, 1) == val(page_numbers, "pair_reduction", float)
    assert cf.full_pairs(5, 1560) == val(page_numbers, "links_per_head_7800")


def test_rope_split_pairs(page_numbers):
    d_t, d_h, d_w = ref.default_split(128)
    assert (d_t // 2, d_h // 2, d_w // 2) == (val(page_numbers, "rope_pairs_t"),
                                              val(page_numbers, "rope_pairs_h"),
                                              val(page_numbers, "rope_pairs_w"))
    assert ref.default_split(32) == (12, 10, 10)


def test_estimator_shares(page_numbers):
    for key, (f, h, w) in {"480p": (81, 480, 832), "720p": (81, 720, 1280)}.items():
        n = cf.video_tokens(f, h, w)
        dense, attn = cf.estimator(n)
        share = round(100 * attn / (dense + attn))
        assert share == val(page_numbers, f"attn_share_{key}")
        total = 100 * (dense + attn)
        assert float(f"{total:.1e}") == val(page_numbers, f"flops_clip_{key}", float)
    # attention term is the same 4 * L^2 * D count as attention_flops for one layer
    n = 32760
    assert cf.estimator(n, layers=1)[1] == cf.attention_flops(1, 1, n, n, 5120)


def test_activation_size(page_numbers):
    mb = 75600 * 5120 * 2 / 1e6
    assert abs(mb - val(page_numbers, "activation_mb_720p")) / mb < 0.01


def test_divided_cost_matches_masks():
    """HW*T^2 + T*HW^2 is the number of pairs the two passes' masks allow."""
    for T, HW in ((8, 64), (3, 5), (21, 7), (1, 9), (4, 1)):
        n_time = int(ref.time_mask(T, HW).sum())
        n_space = int(ref.space_mask(T, HW).sum())
        assert n_time == HW * T * T
        assert n_space == T * HW * HW
        assert cf.divided_pairs(T, HW) == n_time + n_space
        assert cf.full_pairs(T, HW) == (T * HW) ** 2


def test_divided_ratio_720p():
    # 720p token grid: 21 frames x 3600 sites per frame
    full, div = cf.full_pairs(21, 3600), cf.divided_pairs(21, 3600)
    assert div == 3600 * 441 + 21 * 3600 ** 2
    assert 20.8 < full / div < 20.9


def test_attention_flops():
    assert cf.attention_flops(2, 40, 32760, 32760, 128) == 4 * 2 * 40 * 32760 ** 2 * 128
    # 12 heads x 60,840,000 links x 128 dims x 4
    assert cf.attention_flops(1, 12, 7800, 7800, 128) == 373_800_960_000
