"""Benchmark of the spacetime-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step runs every step of the path once on one batch of seeded synthetic
input resident in HBM:

    patchify (latent -> tokens) -> 3D RoPE on Q, K -> full 3D attention
                                                   -> time pass + space pass

The default workload is the 81-frame 832x480 clip as a CFG pair: latent
[2, 16, 21, 60, 104] fp32, patch (1, 2, 2) -> 32,760 tokens, Q/K/V
[2, 32760, 40, 128] bf16 ~ N(0, 1) (seed 0; the projection that would produce
them needs trained weights and is not part of the path).  The metric is
attention TFLOP/s over the step (4*L_q*L_k*D per head for every attention
call; patchify and RoPE add time, no FLOPs) and ms per step (one layer).

Multi-GPU: one process per GPU.  Under torchrun every rank runs its own clip
pair (the path has no exchange step, so there is no data-path collective); the
reported time is the max over ranks and the value counts the work of all ranks
("scaling": "weak").  ``--gpus N`` with N > 1 outside torchrun starts the N
local ranks itself (torch.distributed.run on 127.0.0.1); a world size that
differs from ``--gpus`` is an error.

After the main step the line carries ``workloads``: the other clips of the
pages, timed on their own - full attention at 75,600 tokens (81 frames at
1280x720), divided attention at 720p against that full-attention time (the
pages' 20.88x pair ratio beside the measured ratio), and the 17-frame 480p
clip (7,800 tokens, 12 heads).

``--impl reference`` times the float64 CPU oracle on bounded samples of the
same workload (rank 0 only) and prints the same JSON line with "impl":
"reference".  The CPU baseline inside the default run does the same once.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention TFLOP/s and ms/layer at 32,760 tokens; % of B200 dense BF16 peak"

TEXT_TOKENS = 512          # prompt tokens the video tokens cross-attend to (towardsai section 5)
E2E_SETS = 3               # device buffer sets the end-to-end pipeline rotates through
E2E_MIN_STEPS = 64         # end-to-end steps timed at least (fill and drain included)

WORKLOADS = {
    # name: (B, T latent frames, H latent, W latent, heads, head_dim, description)
    "480p81_cfg_pair": (2, 21, 60, 104, 40, 128,
                        "81-frame 832x480 clip, CFG pair: 2 x 21x30x52 = 32,760 tokens, 40 heads x 128"),
    "480p81": (1, 21, 60, 104, 40, 128, "81-frame 832x480 clip: 21x30x52 = 32,760 tokens, 40 heads x 128"),
    "720p81": (1, 21, 90, 160, 40, 128, "81-frame 1280x720 clip: 21x45x80 = 75,600 tokens, 40 heads x 128"),
    "480p17": (1, 5, 60, 104, 12, 128, "17-frame 832x480 clip: 5x30x52 = 7,800 tokens, 12 heads x 128"),
}
DEFAULT_WORKLOAD = "480p81_cfg_pair"
LATENT_C = 16
PATCH = (1, 2, 2)


def workload_dims(name):
    B, T, H, W, heads, D, desc = WORKLOADS[name]
    Tg, Hg, Wg = T // PATCH[0], H // PATCH[1], W // PATCH[2]
    return dict(B=B, T=T, H=H, W=W, heads=heads, D=D, Tg=Tg, Hg=Hg, Wg=Wg, L=Tg * Hg * Wg, HW=Hg * Wg, desc=desc)


def step_flops(d):
    """Algorithmic FLOPs of one step: 4*Lq*Lk*D per (batch, head) for full
    attention, the time pass (HW sites x T^2) and the space pass (T frames x HW^2)."""
    B, H, D, L, T, HW = d["B"], d["heads"], d["D"], d["L"], d["Tg"], d["HW"]
    full = 4 * B * H * L * L * D
    tpass = 4 * B * H * D * HW * T * T
    spass = 4 * B * H * D * T * HW * HW
    return full, tpass, spass


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def code_only(src):
    """C++ source without its comments and blank lines, each line stripped: what
    the compiler sees, so that editing a comment does not change the hash."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    lines = (re.sub(r"//.*", "", ln).strip() for ln in src.splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_source_hash():
    """Hash of the attention kernel's code (comments excluded): a stored ncu
    traffic figure is used only while it still describes the kernel that runs."""
    h = hashlib.sha256()
    for f in ("attn_tcgen05.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "spacetime_attention_vdit_b200", "csrc", f), encoding="utf-8") as fh:
            h.update(code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def stored_traffic(workload):
    """DRAM bytes per launch of the full-attention kernel from a committed ncu
    summary, or None when absent or taken on other kernel source."""
    try:
        with open(os.path.join(ROOT, "profiles", "attn_full_traffic.json")) as f:
            rec = json.load(f)
    except OSError:
        return None
    ent = rec.get(workload)
    if not ent or ent.get("source_hash") != kernel_source_hash():
        return None
    return ent.get("dram_bytes_per_launch")


ATTN_KERNEL = "attn_fwd_tcgen05_kernel<128, false>"


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples taken while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.dev)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self):
        rows = []
        for line in (getattr(self, "out", "") or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]) if parts[3] not in ("[N/A]", "") else 0.0,
                             parts[5], parts[6], parts[7], parts[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        loaded = [r for r in rows if r[2] > 200.0] or rows
        reasons = set()
        for r in loaded:
            for name, val in zip(("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"),
                                 r[3:]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": max(r[2] for r in rows)}


# ----------------------------------------------------------------------------- CPU oracle legs

def oracle_sample(d, budget_s, seed=0):
    """Time the float64 oracle on a bounded sample of the step: query rows of full
    attention of one (batch, head), plus the same rows of the space and time
    passes.  Returns (FLOPs done, seconds, description, query rows done)."""
    import synthetic
    from oracle import reference as ref

    L, D, T, HW = d["L"], d["D"], d["Tg"], d["HW"]
    q, k, v = synthetic.qkv_bf16(1, L, 1, D, seed=seed)
    qf, kf, vf = (synthetic.bf16_bits_to_f64(x) for x in (q, k, v))
    rows = 64
    flops = 0
    t0 = time.perf_counter()
    done_rows = 0
    while True:
        sel = synthetic.sample_rows(L, rows, seed=seed + done_rows)
        ref.attention(qf, kf, vf, rows=sel)
        ref.divided_space_rows(qf, kf, vf, T, HW, sel)
        ref.divided_time_rows(qf, kf, vf, T, HW, sel)
        flops += 4 * rows * L * D + 4 * rows * HW * D + 4 * rows * T * D
        done_rows += rows
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
        # the next chunk: at most double, and no longer than the time left at the
        # rate just measured, so a step stays close to its budget
        per_row = el / done_rows
        rows = int(max(16, min(4096, rows * 2, (budget_s - el) / per_row + 1)))
    return flops, el, f"{done_rows} query rows of one (batch, head): full attention over all {L} keys, " \
                      f"space pass over {HW} keys and time pass over {T} keys, float64 NumPy", done_rows


def oracle_full_small(seed=0):
    """Time the float64 oracle's full attention over every query row of the
    17-frame 480p clip (7,800 tokens x 12 heads x 128): small enough to run whole."""
    import synthetic
    from oracle import reference as ref

    B, T, H, W, heads, D, _ = WORKLOADS["480p17"]
    L = T * (H // PATCH[1]) * (W // PATCH[2])
    q, k, v = synthetic.qkv_bf16(B, L, heads, D, seed=seed)
    qf, kf, vf = (synthetic.bf16_bits_to_f64(x) for x in (q, k, v))
    t0 = time.perf_counter()
    ref.attention(qf, kf, vf)
    el = time.perf_counter() - t0
    flops = 4 * B * heads * L * L * D
    return {"workload": "480p17", "what": f"full attention, every one of {L} rows x {heads} heads, float64 NumPy",
            "s": el, "tflops": flops / el / 1e12}


def oracle_rates(d, flops, seconds, rows):
    """Measured oracle rows per second, and the time a whole step would take at the
    measured FLOP rate (extrapolated: the oracle never runs a whole step)."""
    return {"rows_per_s": rows / seconds,
            "extrapolated_step_s": sum(step_flops(d)) / (flops / seconds)}


def rank_seed(rank: int) -> int:
    """Each rank processes its own clip pair (independent problems, weak scaling)."""
    return 1000 * rank


def reduce_max(x: float, world: int, device) -> float:
    """Max of x over all ranks (the timing rule: the slowest rank sets the time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, flops_per_rank_step: float, steps: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: the work of every rank over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (max_ms * 1e-3) / 1e12


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def free_port() -> int:
    import socket
    with socket.socket() as sock:
        sock.bind(("127.0.0.1", 0))
        return sock.getsockname()[1]


def launch_command(gpus: int, argv, port: int):
    """The torch.distributed.run command that starts `gpus` local ranks of this
    script with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr", "127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + list(argv)


def maybe_launch_ranks(gpus: int, argv):
    """With --gpus N > 1 outside torchrun, run the N ranks as children and return
    their exit status; None when this process is already a rank (or N == 1)."""
    if gpus <= 1 or "WORLD_SIZE" in os.environ:
        return None
    return subprocess.call(launch_command(gpus, argv, free_port()))


def check_world(gpus: int) -> int:
    """The world size torchrun gave this process; it must equal --gpus."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != gpus:
        raise SystemExit(f"bench.py: --gpus {gpus} but the world size is {world}")
    return world


def run_launcher_check(gpus: int) -> int:
    """Host-only check of the multi-rank plumbing (no GPU, no timing): every rank
    joins a gloo group and is counted; rank 0 prints how many ranks it saw."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    world = check_world(gpus)
    rank = int(os.environ.get("RANK", "0"))
    if world > 1:
        dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    seen = torch.ones(1)
    if world > 1:
        dist.all_reduce(seen)
        dist.barrier()
    if rank == 0:
        print(json.dumps({"launcher_check": True, "world": world, "ranks_seen": int(seen.item())}), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_reference(args, d):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    steps, warmup = args.steps, args.warmup
    per_step_budget = max(1.0, min(20.0, 150.0 / max(1, steps + warmup)))
    for _ in range(warmup):
        oracle_sample(d, per_step_budget / 4)
    tot_f, tot_s, tot_r, desc = 0, 0.0, 0, ""
    for _ in range(steps):
        f, s, desc, r = oracle_sample(d, per_step_budget)
        tot_f += f
        tot_s += s
        tot_r += r
    val = tot_f / tot_s / 1e12
    line = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": steps, "warmup": warmup, "ms_per_step": 1e3 * tot_s / steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "description": d["desc"], "batch": d["B"], "tokens": d["L"],
                       "heads": d["heads"], "head_dim": d["D"]},
            "cpu_baseline": {"kind": "oracle", "value": val, "unit": "TFLOP/s", "cores": cpu_cores(),
                             "sample": f"per step: {desc}", **oracle_rates(d, tot_f, tot_s, tot_r)},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm

def time_launches(fn, reps, stream, flush=None):
    """Mean CUDA-event time (ms) of `fn` over `reps` launches on `stream`, each
    bracketed by its own events; `flush` (untimed) runs before every launch."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    for a, b in evs:
        if flush is not None:
            flush()
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs)


def rope_q_row(vd, q, k, v, qr, kr, o, grid, stream, dev, peaks, rounds=3):
    """Q's 3D rotation in the attention prologue against the two-step path
    (towardsai section 5, Sub-Layer 1, then attention): rotate K alone, then
    attention that rotates Q itself, against rotating Q and K in a pass, then
    attention.  The two are timed in alternation, each pass and attention
    launch with its own events, so that both see the same clock."""
    import torch
    B, L, Hh, D = q.shape
    table = vd.rope_3d_table(grid, D)
    flops = 4.0 * B * Hh * L * L * D

    def two(ev):
        ev[0].record(stream)
        vd.rope_3d(q, k, grid, q_out=qr, k_out=kr)
        ev[1].record(stream)
        vd.attn_full(qr, kr, v, out=o)
        ev[2].record(stream)

    def one(ev):
        ev[0].record(stream)
        vd.rope_3d(None, k, grid, k_out=kr)
        ev[1].record(stream)
        vd.attn_full_rope_q(q, kr, v, grid, table, out=o)
        ev[2].record(stream)

    for fn in (two, one):
        fn([torch.cuda.Event(enable_timing=True) for _ in range(3)])
    evs = {"two": [], "one": []}
    for _ in range(rounds):
        for name, fn in (("two", two), ("one", one)):
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            fn(e)
            evs[name].append(e)
    torch.cuda.synchronize(dev)

    def mean(name, a, b):
        return statistics.mean(e[a].elapsed_time(e[b]) for e in evs[name])
    a_ms = mean("one", 1, 2)
    return {"two_step_ms": mean("two", 0, 2), "one_step_ms": mean("one", 0, 2),
            "rope_qk_ms": mean("two", 0, 1), "rope_k_ms": mean("one", 0, 1),
            "attn_ms": mean("two", 1, 2), "attn_rope_q_ms": a_ms,
            "attn_rope_q_tflops": flops / (a_ms * 1e-3) / 1e12,
            "attn_rope_q_frac_of_burst": flops / (a_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "rounds": rounds}


def other_workloads(vd, dev, stream, peaks):
    """The pages' other clips, each timed on its own after 3 warm-up launches.

    * 720p81_full: 81 frames at 1280x720, 21x45x80 = 75,600 tokens, 40 heads x
      128, batch 1: RoPE then full 3D attention (aicassindra Step 2).
    * 720p81_divided: the time pass (3,600 sites x 21 frames) and the space pass
      (21 frames x 3,600 sites) on the same Q, K, V, and the full-attention time
      over their sum beside the pages' pair ratio HW*T^2 + T*HW^2 against
      (T*HW)^2 = 20.88 (cheatsheet "Formulas and numbers").
    * 480p17: 17 frames at 832x480, 5x30x52 = 7,800 tokens, 12 heads x 128:
      patchify, RoPE and full attention; its inputs fit in L2, so L2 is flushed
      (a 512 MB write) before every timed launch.

    Inputs are device-drawn N(0, 1) values (torch generator, seeded), rounded to
    bf16: the values do not change the work; the parity tests use the seeded
    host generators.  The 720p inputs (774 MB per tensor) are larger than L2."""
    import torch
    peak, hbm = peaks["bf16_tflops"], peaks["hbm_gbs"]
    gen = torch.Generator(device=dev)
    out = {}

    def normal(shape, seed):
        gen.manual_seed(seed)
        return torch.randn(shape, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)

    # ---- 720p: full attention (config of 75,600 tokens) and divided attention
    T, Hg, Wg, H, D = 21, 45, 80, 40, 128
    L, HW = T * Hg * Wg, Hg * Wg
    q, k, v = normal((1, L, H, D), 40), normal((1, L, H, D), 41), normal((1, L, H, D), 42)
    o = torch.empty_like(q)
    rope = lambda: vd.rope_3d(q, k, (T, Hg, Wg), inplace=True)
    for _ in range(3):
        rope()
    rope_ms = time_launches(rope, 5, stream)
    full = lambda: vd.attn_full(q, k, v, out=o)
    for _ in range(3):
        full()
    full_ms = time_launches(full, 5, stream)
    full_f = 4.0 * H * L * L * D
    out["720p81_full"] = {"tokens": L, "heads": H, "head_dim": D, "batch": 1, "attn_ms": full_ms,
                          "tflops": full_f / (full_ms * 1e-3) / 1e12,
                          "frac_of_burst": full_f / (full_ms * 1e-3) / 1e12 / peak,
                          "rope_ms": rope_ms, "rope_gb_s": 4 * q.numel() * 2 / (rope_ms * 1e-3) / 1e9,
                          "rope_frac_hbm": 4 * q.numel() * 2 / (rope_ms * 1e-3) / 1e9 / hbm}
    tpass = lambda: vd.attn_divided_time(q, k, v, T, HW, out=o)
    spass = lambda: vd.attn_divided_space(q, k, v, T, HW, out=o)
    for _ in range(3):
        tpass()
        spass()
    t_ms = time_launches(tpass, 10, stream)
    s_ms = time_launches(spass, 10, stream)
    s_f = 4.0 * H * D * T * HW * HW
    out["720p81_divided"] = {
        "time_pass": {"sequences": HW * H, "length": T, "ms": t_ms,
                      "gb_s": 4 * q.numel() * 2 / (t_ms * 1e-3) / 1e9,
                      "frac_hbm": 4 * q.numel() * 2 / (t_ms * 1e-3) / 1e9 / hbm},
        "space_pass": {"sequences": T * H, "length": HW, "ms": s_ms, "tflops": s_f / (s_ms * 1e-3) / 1e12,
                       "frac_of_burst": s_f / (s_ms * 1e-3) / 1e12 / peak},
        "pair_ratio": (L * L) / (HW * T * T + T * HW * HW),
        "time_ratio_full_over_divided": full_ms / (t_ms + s_ms)}
    del q, k, v, o

    # ---- 17 frames at 480p (7,800 tokens, 12 heads): L2 flushed before each launch
    T, Hl, Wl, H = 5, 60, 104, 12
    grid = (T, Hl // 2, Wl // 2)
    L = grid[0] * grid[1] * grid[2]
    lat = torch.randn((1, LATENT_C, T, Hl, Wl), generator=gen.manual_seed(43), device=dev)
    tok = torch.empty((1, L, LATENT_C * 4), dtype=torch.float32, device=dev)
    q, k, v = normal((1, L, H, D), 44), normal((1, L, H, D), 45), normal((1, L, H, D), 46)
    qr, kr, o = torch.empty_like(q), torch.empty_like(k), torch.empty_like(q)
    scrub = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    flush = lambda: scrub.zero_()
    steps = {"patchify": lambda: vd.patchify_3d(lat, PATCH, out=tok),
             "rope": lambda: vd.rope_3d(q, k, grid, q_out=qr, k_out=kr),
             "attn_full": lambda: vd.attn_full(qr, kr, v, out=o)}
    ms = {}
    for name, fn in steps.items():
        for _ in range(3):
            fn()
        ms[name] = time_launches(fn, 10, stream, flush)
    full_f = 4.0 * H * L * L * D
    out["480p17"] = {"tokens": L, "heads": H, "head_dim": D, "batch": 1, "l2": "flushed before every launch",
                     "attn_ms": ms["attn_full"], "tflops": full_f / (ms["attn_full"] * 1e-3) / 1e12,
                     "frac_of_burst": full_f / (ms["attn_full"] * 1e-3) / 1e12 / peak,
                     "rope_ms": ms["rope"], "patchify_ms": ms["patchify"]}
    del scrub, lat, tok, q, k, v, qr, kr, o
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-aux", action="store_true", help="skip the large-batch patchify measurement")
    ap.add_argument("--no-workloads", action="store_true", help="skip the other clips (720p, 17-frame 480p)")
    ap.add_argument("--launcher-check", action="store_true",
                    help="only start the ranks and count them (host-side test of --gpus)")
    args = ap.parse_args()
    d = workload_dims(args.workload)
    if args.warmup < 3:
        ap.error("at least 3 warm-up steps")
    launched = maybe_launch_ranks(args.gpus, sys.argv[1:])
    if launched is not None:
        return launched
    if args.launcher_check:
        return run_launcher_check(args.gpus)
    check_world(args.gpus)
    if args.impl == "reference":
        return run_reference(args, d)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    import spacetime_attention_vdit_b200 as vd
    import synthetic

    B, L, Hh, D, Tg, HW = d["B"], d["L"], d["heads"], d["D"], d["Tg"], d["HW"]
    grid = (d["Tg"], d["Hg"], d["Wg"])
    seed = rank_seed(rank)
    lat_h = torch.from_numpy(synthetic.latent_f32(B, LATENT_C, d["T"], d["H"], d["W"], seed=seed)).pin_memory()
    qb, kb, vb = synthetic.qkv_bf16(B, L, Hh, D, seed=seed)

    def pinned_bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()

    q_h, k_h, v_h = pinned_bf16(qb), pinned_bf16(kb), pinned_bf16(vb)
    del qb, kb, vb
    lat = lat_h.to(dev)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    tok = torch.empty((B, L, LATENT_C * PATCH[0] * PATCH[1] * PATCH[2]), dtype=torch.float32, device=dev)
    qr, kr = torch.empty_like(q), torch.empty_like(k)
    o_full, o_time, o_space = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)

    names = ("patchify", "rope", "attn_full", "attn_time", "attn_space")
    launches_per_step = len(names)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        vd.patchify_3d(lat, PATCH, out=tok)
        if ev is not None:
            ev[1].record(stream)
        vd.rope_3d(q, k, grid, q_out=qr, k_out=kr)
        if ev is not None:
            ev[2].record(stream)
        vd.attn_full(qr, kr, v, out=o_full)
        if ev is not None:
            ev[3].record(stream)
        vd.attn_divided_time(qr, kr, v, Tg, HW, out=o_time)
        if ev is not None:
            ev[4].record(stream)
        vd.attn_divided_space(qr, kr, v, Tg, HW, out=o_space)
        if ev is not None:
            ev[5].record(stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def max_over_ranks(x):
        return reduce_max(x, world, dev)

    for _ in range(args.warmup):
        step()
    rc, flags = vd.device_status()
    if rc != 0:
        raise RuntimeError(f"kernel watchdog tripped during warm-up: flags {flags:#x}")

    # ---- device-resident timed region
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        time.sleep(0.5)          # nvidia-smi is sampling before the timed region starts
        barrier()
        start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        stop.record(stream)
        barrier()
    clocks = clk.summary()
    ms_local = start.elapsed_time(stop)
    ms = max_over_ranks(ms_local)
    per_row = {n: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j, n in enumerate(names)}
    rc, flags = vd.device_status()
    if rc != 0:
        raise RuntimeError(f"kernel watchdog tripped in the timed region: flags {flags:#x}")

    full_f, time_f, space_f = step_flops(d)
    flops_step = full_f + time_f + space_f
    value = job_throughput(world, flops_step, args.steps, ms)

    # ---- end to end through the public API with host buffers
    # Every step copies its inputs in from pinned host memory and its results
    # back out.  The copies of one step overlap the compute of its neighbours:
    # three streams (host->device, compute, device->host) and three device
    # buffer sets, as a serving loop would run them (a step's input copy may
    # start once the step three back has been computed, so a late copy does not
    # stall the compute stream); the timed region spans the first input copy to
    # the last output copy, pipeline fill and drain included.
    e2e = None
    if not args.no_e2e:
        sets = [dict(lat=lat, q=q, k=k, v=v, tok=tok, qr=qr, kr=kr, o_full=o_full, o_time=o_time,
                     o_space=o_space)]
        for _ in range(E2E_SETS - 1):
            sets.append({n: torch.empty_like(t) for n, t in sets[0].items()})
        out_names = ("tok", "o_full", "o_time", "o_space")
        outs_h = [[torch.empty(sets[0][n].shape, dtype=sets[0][n].dtype).pin_memory() for n in out_names]
                  for _ in range(E2E_SETS)]
        h2d = sum(t.numel() * t.element_size() for t in (lat_h, q_h, k_h, v_h))
        d2h = sum(sets[0][n].numel() * sets[0][n].element_size() for n in out_names)
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        s_comp = stream

        def set_step(bs):
            vd.patchify_3d(bs["lat"], PATCH, out=bs["tok"])
            vd.rope_3d(bs["q"], bs["k"], grid, q_out=bs["qr"], k_out=bs["kr"])
            vd.attn_full(bs["qr"], bs["kr"], bs["v"], out=bs["o_full"])
            vd.attn_divided_time(bs["qr"], bs["kr"], bs["v"], Tg, HW, out=bs["o_time"])
            vd.attn_divided_space(bs["qr"], bs["kr"], bs["v"], Tg, HW, out=bs["o_space"])

        def run_pipeline(n_steps, first=None, last=None):
            ev_in, ev_comp, ev_out = {}, {}, {}
            for t in range(n_steps):
                bs, oh = sets[t % E2E_SETS], outs_h[t % E2E_SETS]
                with torch.cuda.stream(s_in):
                    if t == 0 and first is not None:
                        first.record(s_in)
                    if t >= E2E_SETS:
                        s_in.wait_event(ev_comp[t - E2E_SETS])  # the set's inputs are consumed
                    for name, hsrc in (("lat", lat_h), ("q", q_h), ("k", k_h), ("v", v_h)):
                        bs[name].copy_(hsrc, non_blocking=True)
                    ev_in[t] = torch.cuda.Event()
                    ev_in[t].record(s_in)
                with torch.cuda.stream(s_comp):
                    s_comp.wait_event(ev_in[t])
                    if t >= E2E_SETS:
                        s_comp.wait_event(ev_out[t - E2E_SETS])  # the set's outputs are read out
                    set_step(bs)
                    ev_comp[t] = torch.cuda.Event()
                    ev_comp[t].record(s_comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_comp[t])
                    for hbuf, name in zip(oh, out_names):
                        hbuf.copy_(bs[name], non_blocking=True)
                    ev_out[t] = torch.cuda.Event()
                    ev_out[t].record(s_out)
            if last is not None:
                last.record(s_out)

        run_pipeline(E2E_SETS)
        # a serving loop runs without end: enough steps that the fill and drain
        # (one step's input copy and one step's output copy) weigh little
        e_steps = min(max(args.steps, E2E_MIN_STEPS), 4 * E2E_MIN_STEPS)
        barrier()
        torch.cuda.synchronize(dev)
        s2, t2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        run_pipeline(e_steps, first=s2, last=t2)
        torch.cuda.synchronize(dev)
        barrier()
        e_ms = max_over_ranks(s2.elapsed_time(t2))
        rc, flags = vd.device_status()
        if rc != 0:
            raise RuntimeError(f"kernel watchdog tripped in the end-to-end leg: flags {flags:#x}")
        # each direction's copies alone, on an idle device: the rate the
        # pipeline cannot beat when the copies take longer than the kernels
        copy_ms = {}
        for direction in ("h2d", "d2h"):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(s_in):
                a.record(s_in)
                if direction == "h2d":
                    for name, hsrc in (("lat", lat_h), ("q", q_h), ("k", k_h), ("v", v_h)):
                        sets[1][name].copy_(hsrc, non_blocking=True)
                else:
                    for hbuf, name in zip(outs_h[1], out_names):
                        hbuf.copy_(sets[1][name], non_blocking=True)
                b.record(s_in)
            torch.cuda.synchronize(dev)
            copy_ms[direction] = max_over_ranks(a.elapsed_time(b))
        e2e = {"value": job_throughput(world, flops_step, e_steps, e_ms), "unit": "TFLOP/s",
               "ms_per_step": e_ms / e_steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": e_steps,
               "h2d_ms_alone": copy_ms["h2d"], "d2h_ms_alone": copy_ms["d2h"],
               "h2d_gb_s": h2d / (copy_ms["h2d"] * 1e-3) / 1e9, "d2h_gb_s": d2h / (copy_ms["d2h"] * 1e-3) / 1e9,
               "pipelined": (f"host->device, compute and device->host on three streams, {E2E_SETS} device "
                             "buffer sets; fill and drain inside the timed region")}
        del sets[1:]

    # ---- roofline of the dominant kernel (full attention)
    peaks, peaks_kind = measured_peaks()
    full_ms = per_row["attn_full"]
    achieved = full_f / (full_ms * 1e-3) / 1e12
    # the record denominator is the measured burst bf16 GEMM rate; the step is
    # tens of ms and the timed region about a second, not a seconds-long run
    peak = peaks["bf16_tflops"]
    sustained = peaks.get("bf16_tflops_sustained")
    roofline = {"bound": "tensor", "kernel": ATTN_KERNEL, "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": stored_traffic(args.workload),
                "peak_kind": f"{peaks_kind} bf16 burst (cuBLAS-class GEMM, best of 10)",
                "frac_of_sustained": achieved / sustained if sustained else None,
                "flops_per_launch": full_f, "avg_launch_ms": full_ms}

    hbm = peaks["hbm_gbs"]
    tok_bytes = tok.numel() * 4
    row_bytes = {
        "patchify": lat.numel() * 4 + tok_bytes,
        "rope": 4 * q.numel() * 2,
        "attn_time": 4 * q.numel() * 2,
    }
    rows = {}
    for n in names:
        r = {"ms": per_row[n]}
        if n in row_bytes:
            r["gb_s"] = row_bytes[n] / (per_row[n] * 1e-3) / 1e9
            r["frac_hbm"] = r["gb_s"] / hbm
        if n == "attn_full":
            r["tflops"] = achieved
        if n == "attn_space":
            r["tflops"] = space_f / (per_row[n] * 1e-3) / 1e12
        rows[n] = r
    # divided attention against full attention: the pages' count of attended
    # pairs, L^2 / (HW*T^2 + T*HW^2) (20.88 at 720p), beside the measured time ratio
    pairs_full = d["L"] * d["L"]
    pairs_div = d["HW"] * d["Tg"] * d["Tg"] + d["Tg"] * d["HW"] * d["HW"]
    divided = {"pair_ratio": pairs_full / pairs_div,
               "time_ratio": per_row["attn_full"] / (per_row["attn_time"] + per_row["attn_space"])}

    # ---- auxiliary: patchify at a size where bandwidth, not launch latency, shows
    aux = None
    if not args.no_aux:
        big = torch.empty((64, LATENT_C, 21, 90, 160), dtype=torch.float32, device=dev).normal_()
        big_tok = torch.empty((64, 21 * 45 * 80, LATENT_C * 4), dtype=torch.float32, device=dev)
        for _ in range(3):
            vd.patchify_3d(big, PATCH, out=big_tok)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 5
        a.record(stream)
        for _ in range(reps):
            vd.patchify_3d(big, PATCH, out=big_tok)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        pms = a.elapsed_time(b_) / reps
        pbytes = 2 * big.numel() * 4
        aux = {"patchify_64_clips_720p": {"latent": [64, LATENT_C, 21, 90, 160], "ms": pms,
                                          "gb_s": pbytes / (pms * 1e-3) / 1e9,
                                          "frac_hbm": pbytes / (pms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                          "bytes": pbytes}}
        del big, big_tok

    # ---- next row: text cross-attention, the video tokens of this workload against
    # 512 prompt tokens (towardsai section 5, Sub-Layer 2); timed on its own
    cross = None
    if not args.no_aux:
        Lk = TEXT_TOKENS
        kt = torch.empty((d["B"], Lk, Hh, D), dtype=torch.bfloat16, device=dev).normal_()
        vt = torch.empty_like(kt).normal_()
        oc = torch.empty_like(q)
        for _ in range(3):
            vd.attn_cross(q, kt, vt, out=oc)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        a.record(stream)
        for _ in range(reps):
            vd.attn_cross(q, kt, vt, out=oc)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        cms = a.elapsed_time(b_) / reps
        cflops = 4.0 * d["B"] * Hh * L * Lk * D
        cross = {"attn_cross_512": {"Lq": L, "Lk": Lk, "ms": cms, "tflops": cflops / (cms * 1e-3) / 1e12,
                                    "frac_of_burst": cflops / (cms * 1e-3) / 1e12 / peaks["bf16_tflops"]}}
        del kt, vt, oc
        # next row: Q/K RMSNorm fused with the 3D RoPE (towardsai section 5,
        # Sub-Layer 1), over each token's whole heads*D vector, weights 1
        qn, kn = torch.empty_like(q), torch.empty_like(k)
        width = Hh * D
        for _ in range(3):
            vd.qk_norm_rope_3d(q, k, grid, width, q_out=qn, k_out=kn)
        a.record(stream)
        for _ in range(reps):
            vd.qk_norm_rope_3d(q, k, grid, width, q_out=qn, k_out=kn)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        nms = a.elapsed_time(b_) / reps
        nbytes = 4 * q.numel() * 2
        cross["qk_norm_rope"] = {"norm_group": width, "ms": nms, "gb_s": nbytes / (nms * 1e-3) / 1e9,
                                 "frac_hbm": nbytes / (nms * 1e-3) / 1e9 / peaks["hbm_gbs"], "bytes": nbytes}
        del qn, kn
        cross["rope_q_in_attention"] = rope_q_row(vd, q, k, v, qr, kr, o_full, grid, stream, dev, peaks)
        # next row: the patch embedding (patchify and the Conv3d weight on the tensor
        # cores) to the model width heads*D of this workload
        dim = Hh * D
        wemb = (torch.randn(dim, LATENT_C * PATCH[0] * PATCH[1] * PATCH[2], device=dev) / 8).to(torch.bfloat16)
        bemb = torch.randn(dim, device=dev)
        emb = torch.empty((d["B"], L, dim), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            vd.patch_embed_3d(lat, wemb, PATCH, bemb, out=emb)
        a.record(stream)
        for _ in range(reps):
            vd.patch_embed_3d(lat, wemb, PATCH, bemb, out=emb)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        ems = a.elapsed_time(b_) / reps
        ebytes = lat.numel() * 4 + wemb.numel() * 2 + dim * 4 + emb.numel() * 2
        cross["patch_embed"] = {"dim": dim, "ms": ems, "gb_s": ebytes / (ems * 1e-3) / 1e9,
                                "frac_hbm": ebytes / (ems * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                "tflops": 2.0 * emb.numel() * wemb.shape[1] / (ems * 1e-3) / 1e12, "bytes": ebytes}
        del wemb, bemb, emb
        # next row: unpatchify, measured where bandwidth shows (64 clips at 720p)
        big_tok = torch.empty((64, 21 * 45 * 80, LATENT_C * 4), dtype=torch.float32, device=dev).normal_()
        big = torch.empty((64, LATENT_C, 21, 90, 160), dtype=torch.float32, device=dev)
        for _ in range(3):
            vd.unpatchify_3d(big_tok, LATENT_C, (21, 45, 80), PATCH, out=big)
        a.record(stream)
        for _ in range(5):
            vd.unpatchify_3d(big_tok, LATENT_C, (21, 45, 80), PATCH, out=big)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        ums = a.elapsed_time(b_) / 5
        ubytes = 2 * big.numel() * 4
        cross["unpatchify_64_clips_720p"] = {"ms": ums, "gb_s": ubytes / (ums * 1e-3) / 1e9,
                                             "frac_hbm": ubytes / (ums * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                             "bytes": ubytes}
        del big_tok, big

    workloads = None
    if not args.no_workloads:
        workloads = other_workloads(vd, dev, stream, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        f, s, desc, r = oracle_sample(d, 15.0)
        cpu = {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": desc + f"; {s:.1f} s", **oracle_rates(d, f, s, r),
               "whole_small_clip": oracle_full_small()}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": args.workload, "description": d["desc"], "batch": d["B"],
                           "tokens": L, "heads": Hh, "head_dim": D, "grid": list(grid), "patch": list(PATCH),
                           "latent": [d["B"], LATENT_C, d["T"], d["H"], d["W"]],
                           "step": "patchify + rope + full attention + time pass + space pass",
                           "flops_per_step_per_gpu": flops_step,
                           "l2": "inputs larger than L2: %.2f GB of Q/K/V per step" % (3 * q.numel() * 2 / 1e9),
                           "parallelism": f"replicas x{world}"},
                "roofline": roofline, "rows": rows, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps, "clocks": clocks, "aux": aux,
                "divided_vs_full": divided, "next_rows": cross, "workloads": workloads,
                "frac_of_nominal_dense_bf16": achieved / 2250.0}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
