"""Helpers shared by the GPU parity tests: moving bf16 bit patterns to and from
the device, and the attention tolerance check.

Attention tolerances (floating point; bf16 inputs, float32 arithmetic, bf16 P and O):
* contract: max |gpu - oracle| <= 2e-2 and mean |gpu - oracle| <= 2e-3;
* derived from the arithmetic: P and O are each rounded once to bf16 (relative
  2^-9 ~ 2e-3 per element, independent across terms), so the relative L2 error
  of O is a few 1e-3; we require ||gpu - oracle||_2 <= 1e-2 ||oracle||_2, which
  catches a wrong tile, a dropped rescale or a missing key that the absolute
  contract bound (loose next to |O| ~ 1/sqrt(L) for flat softmax rows) cannot;
* log-sum-exp: scores are exact products of bf16 values summed in float32 and
  exponentials are ex2.approx (relative 2^-22), so |lse - oracle| <= 1e-3.
"""
from __future__ import annotations

import numpy as np
import torch

import synthetic

MAX_ABS = 2e-2
MEAN_ABS = 2e-3
REL_L2 = 1e-2
LSE_ABS = 1e-3


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def from_dev_bf16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev_f64(t: torch.Tensor) -> np.ndarray:
    return synthetic.bf16_bits_to_f64(from_dev_bf16(t))


def attn_errors(got: np.ndarray, ref: np.ndarray):
    d = np.abs(got - ref)
    return float(d.max()), float(d.mean()), float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def assert_attention_close(got: np.ndarray, ref: np.ndarray, lse_got=None, lse_ref=None, what=""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, mean, rel = attn_errors(got, ref)
    assert mx <= MAX_ABS, f"{what}: max abs {mx:.3e}"
    assert mean <= MEAN_ABS, f"{what}: mean abs {mean:.3e}"
    assert rel <= REL_L2, f"{what}: relative L2 {rel:.3e}"
    if lse_got is not None:
        le = float(np.abs(lse_got - lse_ref).max())
        assert le <= LSE_ABS, f"{what}: lse max abs {le:.3e}"
    return mx, mean, rel


def watchdog_clear():
    import spacetime_attention_vdit_b200 as v
    rc, flags = v.device_status()
    assert rc == 0, f"device status {rc}, watchdog flags {flags:#x}"
