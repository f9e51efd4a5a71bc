"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/vdit.h declares, and rejects bad arguments with the
documented status before touching CUDA."""
import ctypes
import os
import re

import pytest
import torch

from tests.conftest import ROOT

OK, NULL, SHAPE, ALIGN, UNSUP = 0, 1, 2, 3, 4
FAKE = 0x7f0000000000          # 16-byte aligned, never dereferenced: every call below returns first
MIS = FAKE + 8                 # 8-byte aligned only


@pytest.fixture(scope="module")
def L():
    import spacetime_attention_vdit_b200 as v
    if not os.path.exists(v.LIB_PATH):
        v_build = __import__("spacetime_attention_vdit_b200.build", fromlist=["build"])
        v_build.build()
    return v.lib()


def declared_functions():
    with open(os.path.join(ROOT, "include", "vdit.h")) as fh:
        text = fh.read()
    return sorted(set(re.findall(r"^(?:int|long long|const char\*)\s+(vdit_\w+)\s*\(", text, flags=re.M)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert {"vdit_patchify_3d", "vdit_rope_3d", "vdit_attn_full", "vdit_attn_divided_time",
            "vdit_attn_divided_space", "vdit_status_string", "vdit_device_status", "vdit_version",
            "vdit_rope_3d_table", "vdit_rope_3d_table_entries", "vdit_attn_full_rope_q"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_version_and_strings(L):
    assert L.vdit_version() == 10100
    for s in range(7):
        assert len(L.vdit_status_string(s)) > 0
    assert L.vdit_status_string(99) == b"unknown status"


def patchify(L, latent=FAKE, tokens=FAKE, dtype=0, N=1, C=4, T=8, H=16, W=16, pt=1, ph=2, pw=2):
    return L.vdit_patchify_3d(latent, tokens, dtype, N, C, T, H, W, pt, ph, pw, None)


def test_patchify_validation(L):
    assert patchify(L, latent=None) == NULL
    assert patchify(L, tokens=None) == NULL
    assert patchify(L, dtype=7) == UNSUP
    assert patchify(L, N=0) == SHAPE
    assert patchify(L, pw=-1) == SHAPE
    assert patchify(L, T=1, pt=2) == SHAPE            # no whole brick along time
    assert patchify(L, C=100000, pt=4, ph=4, pw=4) == UNSUP   # one brick beyond the staging buffer


def rope(L, q=FAKE, k=FAKE, qo=FAKE, ko=FAKE, B=1, Tg=2, Hg=3, Wg=4, heads=2, D=128, split=(44, 42, 42),
         theta=10000.0):
    return L.vdit_rope_3d(q, k, qo, ko, B, Tg, Hg, Wg, heads, D, *split, ctypes.c_float(theta), None)


def test_rope_validation(L):
    assert rope(L, q=None) == NULL
    assert rope(L, ko=None) == NULL
    # the cheatsheet's rope_3d ValueError: widths must add up to the head width
    assert rope(L, split=(44, 42, 40)) == SHAPE
    assert rope(L, split=(43, 43, 42)) == SHAPE
    assert rope(L, split=(-2, 66, 64)) == SHAPE
    assert rope(L, Hg=0) == SHAPE
    assert rope(L, theta=0.0) == SHAPE
    assert rope(L, D=36, split=(12, 12, 12)) == UNSUP  # not a multiple of 8
    assert rope(L, q=MIS) == ALIGN
    assert rope(L, ko=MIS) == ALIGN


def test_rope_k_only_form(L):
    """Q's pointers both NULL rotate K alone; only one of them NULL is an error."""
    assert rope(L, q=None, qo=None, k=None) == NULL
    assert rope(L, qo=None) == NULL
    assert rope(L, q=None, qo=None, split=(44, 42, 40)) == SHAPE
    assert rope(L, q=None, qo=None, ko=MIS) == ALIGN
    assert norm_rope(L, q=None, qo=None, k=None) == NULL
    assert norm_rope(L, q=None) == NULL
    assert norm_rope(L, q=None, qo=None, group=96) == SHAPE
    assert norm_rope(L, q=None, qo=None, ko=MIS) == ALIGN


def table(L, t=FAKE, Tg=21, Hg=30, Wg=52, D=128, split=(44, 42, 42), theta=10000.0):
    return L.vdit_rope_3d_table(t, Tg, Hg, Wg, D, *split, ctypes.c_float(theta), None)


def test_rope_table_validation(L):
    assert L.vdit_rope_3d_table_entries(21, 30, 52, 128, 44, 42, 42) == 21 * 22 + 30 * 21 + 52 * 21
    assert L.vdit_rope_3d_table_entries(21, 30, 52, 128, 0, 64, 64) == 30 * 32 + 52 * 32
    assert L.vdit_rope_3d_table_entries(21, 30, 52, 128, 44, 42, 40) == -1
    assert L.vdit_rope_3d_table_entries(0, 30, 52, 128, 44, 42, 42) == -1
    assert table(L, t=None) == NULL
    assert table(L, split=(43, 43, 42)) == SHAPE
    assert table(L, Wg=0) == SHAPE
    assert table(L, theta=-1.0) == SHAPE
    assert table(L, t=MIS) == ALIGN


def attn_rope(L, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, B=1, grid=(3, 8, 12), heads=2, D=128,
              split=(44, 42, 42), tab=FAKE, wq=None, group=0, eps=1e-6):
    return L.vdit_attn_full_rope_q(q, k, v, o, lse, B, *grid, heads, D, ctypes.c_float(0.0), *split, tab, wq,
                                   group, ctypes.c_float(eps), None)


def test_attn_full_rope_q_validation(L):
    assert attn_rope(L, tab=None) == NULL
    assert attn_rope(L, q=None) == NULL
    assert attn_rope(L, grid=(3, 0, 12)) == SHAPE
    assert attn_rope(L, B=0) == SHAPE
    assert attn_rope(L, split=(44, 42, 40)) == SHAPE
    assert attn_rope(L, D=48, split=(16, 16, 16)) == UNSUP
    assert attn_rope(L, group=256) == UNSUP           # a token-wide group needs every head
    assert attn_rope(L, group=64) == UNSUP
    assert attn_rope(L, group=128, eps=-1.0) == SHAPE
    assert attn_rope(L, tab=MIS) == ALIGN
    assert attn_rope(L, group=128, wq=MIS) == ALIGN
    assert attn_rope(L, k=MIS) == ALIGN
    # the table and the weights are staged in one K/V stage: 8 n + 4 D <= 256 D
    # bytes, 4,032 pairs at D = 128 (a call that passed every check would
    # launch, so only the refused side is called here)
    assert L.vdit_rope_3d_table_entries(182, 1, 1, 128, 44, 42, 42) == 4046
    assert attn_rope(L, grid=(182, 1, 1), split=(44, 42, 42), B=1) == UNSUP


def norm_rope(L, q=FAKE, k=FAKE, qo=FAKE, ko=FAKE, wq=None, wk=None, group=128, eps=1e-6, B=1, Tg=2, Hg=3,
              Wg=4, heads=2, D=128, split=(44, 42, 42), theta=10000.0):
    return L.vdit_qk_norm_rope_3d(q, k, qo, ko, wq, wk, group, ctypes.c_float(eps), B, Tg, Hg, Wg, heads, D,
                                  *split, ctypes.c_float(theta), None)


def test_qk_norm_rope_validation(L):
    assert norm_rope(L, q=None) == NULL
    assert norm_rope(L, group=0) == SHAPE
    assert norm_rope(L, group=96) == SHAPE            # does not divide heads * head_dim = 256
    assert norm_rope(L, eps=-1.0) == SHAPE
    assert norm_rope(L, split=(44, 42, 40)) == SHAPE
    assert norm_rope(L, group=12, D=24, split=(8, 8, 8)) == UNSUP        # not a multiple of 8
    assert norm_rope(L, heads=3, D=32, split=(12, 10, 10), group=48) == UNSUP   # 6 vectors, not the token
    assert norm_rope(L, heads=72, D=128) == UNSUP   # 9,216 channels per token
    assert norm_rope(L, wq=MIS) == ALIGN
    assert norm_rope(L, ko=MIS) == ALIGN


def attn(L, fn="vdit_attn_full", q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=None, dims=(1, 256, 2, 128)):
    f = getattr(L, fn)
    return f(q, k, v, o, lse, *dims, ctypes.c_float(0.0), None)


@pytest.mark.parametrize("fn,dims", [("vdit_attn_full", (1, 256, 2, 128)),
                                     ("vdit_attn_divided_time", (1, 8, 64, 2, 32)),
                                     ("vdit_attn_divided_space", (1, 8, 64, 2, 32)),
                                     ("vdit_attn_cross", (1, 256, 77, 2, 128))])
def test_attention_validation(L, fn, dims):
    assert attn(L, fn, dims=dims, q=None) == NULL
    assert attn(L, fn, dims=dims, o=None) == NULL
    assert attn(L, fn, dims=dims, v=MIS) == ALIGN
    assert attn(L, fn, dims=dims, lse=FAKE + 2) == ALIGN
    bad_d = dims[:-1] + (48,)
    assert attn(L, fn, dims=bad_d) == UNSUP
    zero = (0,) + dims[1:]
    assert attn(L, fn, dims=zero) == SHAPE
    neg = dims[:1] + (-5,) + dims[2:]
    assert attn(L, fn, dims=neg) == SHAPE


def test_watchdog_selftest_site_checked(L):
    assert L.vdit_watchdog_selftest(0, None) == SHAPE
    assert L.vdit_watchdog_selftest(256, None) == SHAPE
    assert L.vdit_watchdog_selftest(-1, None) == SHAPE


def test_cross_key_length_checked(L):
    assert attn(L, "vdit_attn_cross", dims=(1, 256, 0, 2, 128)) == SHAPE
    assert attn(L, "vdit_attn_cross", dims=(1, 256, -3, 2, 128)) == SHAPE


def embed(L, latent=FAKE, w=FAKE, b=None, out=FAKE, N=1, C=16, T=5, H=6, W=8, pt=1, ph=2, pw=2, dim=512):
    return L.vdit_patch_embed_3d(latent, w, b, out, N, C, T, H, W, pt, ph, pw, dim, None)


def test_patch_embed_validation(L):
    assert embed(L, latent=None) == NULL
    assert embed(L, w=None) == NULL
    assert embed(L, N=0) == SHAPE
    assert embed(L, H=1) == SHAPE                       # no whole brick along h
    assert embed(L, C=8) == UNSUP                       # 32 features per brick
    assert embed(L, dim=384) == UNSUP                   # not a multiple of 256
    assert embed(L, w=MIS) == ALIGN
    assert embed(L, b=MIS) == ALIGN
    assert embed(L, latent=FAKE + 2) == ALIGN


def test_unpatchify_validation(L):
    f = lambda **kw: L.vdit_unpatchify_3d(kw.get("t", FAKE), kw.get("o", FAKE), kw.get("dt", 0), 1, 4, 2, 3, 4,
                                          1, 2, 2, None)
    assert f(t=None) == NULL
    assert f(o=None) == NULL
    assert f(dt=3) == UNSUP
    assert L.vdit_unpatchify_3d(FAKE, FAKE, 0, 1, 4, 0, 3, 4, 1, 2, 2, None) == SHAPE
    assert L.vdit_unpatchify_3d(FAKE, FAKE, 0, 1, 4096, 2, 3, 4, 1, 2, 2, None) == UNSUP   # 64 KB tokens


def test_binding_refuses_cpu_tensors(L):
    """The product path has no CPU fallback: host tensors are refused."""
    import spacetime_attention_vdit_b200 as v
    q = torch.zeros((1, 8, 1, 32), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        v.attn_full(q, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        v.patchify_3d(torch.zeros((1, 1, 1, 2, 2)))
    with pytest.raises(ValueError, match="CUDA"):
        v.rope_3d(None, q, (1, 2, 4), (12, 10, 10))
    tab = torch.zeros((1 * 6 + 2 * 5 + 4 * 5, 2), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        v.attn_full_rope_q(q, q, q, (1, 2, 4), tab, (12, 10, 10))
    with pytest.raises(ValueError, match="grid"):
        v.attn_full_rope_q(q, q, q, (1, 2, 5), tab, (12, 10, 10))


def test_build_command_targets_sm100a():
    from spacetime_attention_vdit_b200 import build
    cmd = build.command()
    assert "arch=compute_100a,code=sm_100a" in cmd
    assert "-lineinfo" in cmd


def test_register_budget_fits_each_sm_subpartition(tmp_path):
    """Every kernel's registers x the warps one SM sub-partition receives fit its
    16,384 registers (warps of a CTA are spread round-robin over 4 sub-partitions),
    so no launch can fail for lack of registers.  Uses ptxas's own report."""
    import shutil
    import subprocess
    from spacetime_attention_vdit_b200 import build
    if shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"):
        pytest.skip("nvcc not available")
    out = str(tmp_path / "vdit_regcheck.so")
    res = subprocess.run(build.command(ptxas_verbose=True, out=out), capture_output=True, text=True)
    assert res.returncode == 0, res.stderr[-2000:]
    regs = {}
    name = None
    for line in res.stderr.splitlines():
        m = re.search(r"Compiling entry function '(\w+)'", line)
        if m:
            name = m.group(1)
        m = re.search(r"Used (\d+) registers", line)
        if m and name:
            regs[name] = int(m.group(1))
    threads = {"attn_fwd_tcgen05": 384, "rope3d_table_kernel": 256, "rope3d_kernel": 256, "patchify3d_kernel": 256,
               "patchify122_f32_kernel": 128, "qk_norm_rope3d_kernel": 256, "patch_embed_kernel": 320,
               "unpatchify3d_kernel": 256, "watchdog_selftest_kernel": 32}

    def block_of(kname):
        for key, t in threads.items():
            if key in kname:
                return t
        m = re.search(r"attn_time_short_kernelILi(\d+)ELi(\d+)", kname)
        D, TB = int(m.group(1)), int(m.group(2))       # head dim, box rows
        tp = (TB + 15) // 16 * 16
        wpu = 2 if tp >= 32 else 1
        stage = 3 * TB * D * 2
        nstage = min((231424 // (stage + 16)) & ~1, 16, 2 * ((10 if D >= 128 else 16) // wpu))
        assert 1024 + nstage * (stage + 16) <= 232448
        return 32 * (1 + (nstage // 2) * wpu)
    assert regs, "no ptxas report"
    # the attention kernel splits its launch registers between warpgroups
    # (setmaxnreg): two softmax warpgroups take 216 each, the control warpgroup
    # keeps 56, which needs exactly 168 per thread at launch (384 threads)
    src = open(os.path.join(os.path.dirname(build.__file__), "csrc", "attn_tcgen05.cuh")).read()
    m = re.search(r"REGS_LAUNCH = (\d+), REGS_SOFTMAX = (\d+), REGS_CONTROL = (\d+)", src)
    launch, soft, ctrl = (int(x) for x in m.groups())
    assert 2 * 128 * soft + 128 * ctrl <= 384 * launch
    assert 32 * (2 * soft + ctrl) <= 16384              # one warp of each warpgroup per sub-partition
    for kname, r in regs.items():
        if "attn_fwd_tcgen05" in kname:
            assert r == launch, (kname, r)
        warps = block_of(kname) // 32
        per_sub = -(-warps // 4)                  # warps on the fullest sub-partition
        alloc = -(-r // 8) * 8                    # registers are granted in multiples of 8
        assert per_sub * 32 * alloc <= 16384, (kname, r, block_of(kname))
