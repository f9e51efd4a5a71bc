"""Host check of the attention kernel's softmax schedule (no GPU): a float
emulation of one query row's sweep over 128-key tiles, with the kernel's rules
— the first tile's max, exponentials against the max in use afterwards, the
tile's max recomputed only when the tile's sum of P reaches 2^7, a move of the
max (with P taken again) only when a tile raises it by more than 8 in log2
units, one pair in 32 exponentiated by the FMA-pipe cubic (saturating near 2^8),
P rounded to bf16 for P.V — gives what the max-first schedule gives, and stays
within the attention tolerance of the float64 oracle on sharp softmax rows,
where the max moves often.  The same emulation with the sum test at 2^8 (the
cubic's saturated value sits just below it) misses a score above the max in use
and fails, which is why the test is at 2^7."""
import numpy as np

import synthetic
from oracle import reference as ref
from tests.test_exp2_fma_host import ex2_fma_emulated

BN = 128


def _bf16(x):
    return synthetic.bf16_bits_to_f64(synthetic.f64_to_bf16_bits(np.asarray(x, dtype=np.float64)))


def _exps(x):
    x = x.astype(np.float32)
    p = np.exp2(x.astype(np.float64))
    poly = ((np.arange(BN) // 2) % 32) == 31          # one pair in 32 on the FMA pipe
    p[poly] = ex2_fma_emulated(x[poly]).astype(np.float64)
    return p


def _row(s_row, v, start, lazy, threshold):
    """One query row: scores s_row [Lk] float32, values v [Lk, D]."""
    n = (len(s_row) + BN - 1) // BN
    sc = np.float32(1.0 / np.sqrt(v.shape[1]) * np.log2(np.e))
    m, l, o = -np.inf, 0.0, np.zeros(v.shape[1])
    for jj in range(n):
        t = (jj + start) % n
        s = np.full(BN, -np.inf, dtype=np.float32)
        seg = s_row[t * BN:(t + 1) * BN]
        s[:len(seg)] = seg
        vt = np.zeros((BN, v.shape[1]))
        vt[:len(seg)] = v[t * BN:(t + 1) * BN]
        alpha = 1.0
        if jj == 0:
            m = float(s.max() * sc)
            p = _exps(s * sc - np.float32(m))
        elif not lazy:
            mn = float(s.max() * sc)
            if mn > m + 8:
                alpha, m = 2.0 ** (m - mn), mn
            p = _exps(s * sc - np.float32(m))
        else:
            p = _exps(s * sc - np.float32(m))
            if not (p.sum() < threshold):
                mn = float(s.max() * sc)
                if mn > m + 8:
                    alpha, m = 2.0 ** (m - mn), mn
                    p = _exps(s * sc - np.float32(m))
        l = l * alpha + p.sum()
        o = o * alpha + _bf16(p) @ vt
    return _bf16(o / l)


def _attend(q, k, v, lazy, threshold=128.0):
    """All rows of one head, each 256-row query block starting its sweep at
    tile (block mod tiles), as the kernel's CTAs do."""
    S = (q @ k.T).astype(np.float32)
    n = (k.shape[0] + BN - 1) // BN
    return np.stack([_row(S[r], v, (r // 256) % n, lazy, threshold) for r in range(q.shape[0])])


def _case():
    q, k, v = synthetic.qkv_bf16(1, 600, 1, 128, seed=7, q_scale=12.0)
    f = synthetic.bf16_bits_to_f64
    qh, kh, vh = f(q)[0, :, 0], f(k)[0, :, 0], f(v)[0, :, 0]
    eo, _ = ref.attention(f(q), f(k), f(v))
    return qh, kh, vh, eo[0, :, 0]


def test_lazy_max_matches_max_first_on_sharp_rows():
    qh, kh, vh, eo = _case()
    lazy = _attend(qh, kh, vh, lazy=True)
    first = _attend(qh, kh, vh, lazy=False)
    assert np.abs(lazy - eo).max() <= 2e-2
    assert np.abs(lazy - first).max() <= 2e-2
    assert np.abs(lazy - eo).max() <= np.abs(first - eo).max() + 1e-3


def test_a_sum_test_at_two_to_the_eight_misses_the_saturated_cubic():
    qh, kh, vh, eo = _case()
    bad = _attend(qh, kh, vh, lazy=True, threshold=256.0)
    assert np.abs(bad - eo).max() > 2e-2
