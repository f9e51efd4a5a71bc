"""Failure detection on the GPU without a fault: the library's self-check kernel
waits on an mbarrier that nothing arrives on, its bounded wait runs out after the
2-second limit every wait in the library has, and the host reads the timeout and
the wait site through vdit_device_status, which clears them; the next call then
computes normally (the context stayed usable)."""
import numpy as np
import pytest
import torch

import synthetic
from oracle import reference as ref
from tests.gpu_util import assert_attention_close, dev_f64, to_dev_bf16

pytestmark = pytest.mark.gpu

TIMEOUT = 6                     # VDIT_ERR_TIMEOUT


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    yield
    import spacetime_attention_vdit_b200 as v
    v.device_status()                          # never leave a flag set for later tests


def f64(bits):
    return synthetic.bf16_bits_to_f64(bits)


def test_bounded_wait_runs_out_and_is_reported():
    import time
    import spacetime_attention_vdit_b200 as v
    rc, flags = v.device_status()
    assert rc == 0 and flags == 0, f"flags left set before the test: {flags:#x}"
    t0 = time.monotonic()
    v.watchdog_selftest(site=77)
    rc, flags = v.device_status()              # synchronises
    waited = time.monotonic() - t0
    assert rc == TIMEOUT, rc
    assert flags & 1 and (flags >> 8) & 0xff == 77, f"{flags:#x}"
    assert 1.5 < waited < 30.0, waited          # the 2 s limit, not an endless wait
    rc, flags = v.device_status()              # cleared by the read above
    assert rc == 0 and flags == 0


def test_context_usable_after_a_timeout():
    import spacetime_attention_vdit_b200 as v
    v.watchdog_selftest(site=5)
    assert v.device_status()[0] == TIMEOUT
    q, k, vv = synthetic.qkv_bf16(1, 300, 2, 128, seed=3)
    o, lse = v.attn_full(to_dev_bf16(q), to_dev_bf16(k), to_dev_bf16(vv), lse=True)
    assert v.device_status() == (0, 0)
    eo, el = ref.attention(f64(q), f64(k), f64(vv))
    assert_attention_close(dev_f64(o), eo, lse.cpu().numpy(), el, "after a timeout")
    assert np.isfinite(lse.cpu().numpy()).all()


def test_site_out_of_range_is_refused():
    import spacetime_attention_vdit_b200 as v
    with pytest.raises(v.VditError):
        v.watchdog_selftest(site=0)
    with pytest.raises(v.VditError):
        v.watchdog_selftest(site=256)
    assert v.device_status() == (0, 0)
