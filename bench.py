#!/usr/bin/env python
"""Benchmark of the Krea 2 attention core at the 4 MP shape (dense / band / scanline).

One step = the three attention variants over one batch of synthetic inputs at
the Krea 2 4 MP shape (512 text tokens + a 128 x 128 token grid, 48 q heads /
12 kv heads, head_dim 128):
  * dense: the CFG pair (batch 2), bf16, sigmoid gate, queries in 4096-token slices;
  * band:  TileMix band, fp16, smooth_k, band +-2 key blocks, 50% of the left-over
           image-image tiles INT8 (quantiser included);
  * scanline: bf16, window 11, tile_aligned, text padded to 512.
FLOPs = 4 * B * Hq * d * (admitted query-key pairs); value = FLOPs / device time.

python bench.py [--gpus N --steps K --warmup W] [--impl reference]
Under torchrun every rank runs the same step on its own GPU (independent
problems, no collective on the data path); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention TFLOP/s at Krea 2 4 MP shape (dense/band/scanline), % of tensor peak"
WORKLOAD = ("krea2_4mp_attention_step: dense CFG pair B=2 bf16+gate sliced 4096 | TileMix band p=0.5 "
            "fp16 smooth_k | scanline w11 tile_aligned bf16; 48/12 heads, d=128, 512 text + 128x128 grid")
TILE = 128


def roofline_traffic():
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary,
    or None once the kernel source differs from the one the counters came from."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "attn_fwd_roofline.json")
    src = os.path.join(ROOT, "diffusion_transformer_attention_bidirectional_b200", "csrc", "attn_sm100.cu")
    try:
        rec = json.load(open(path))
        digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except (OSError, ValueError):
        return None, None
    if rec.get("kernel_source_sha256") != digest:
        return None, rec
    return rec.get("dram_bytes_per_launch"), rec


DATASHEET_BF16 = 2250.0  # TFLOP/s, dense FP16/BF16 (NVIDIA's B200 figure without sparsity)
DATASHEET_INT8 = 4500.0  # TOP/s, dense INT8


def measure_int8_peak(device, n: int = 8192, reps: int = 10) -> float:
    """Dense INT8 tensor throughput of this GPU in TOP/s: torch._int_mm (a library
    INT8 GEMM, s8 x s8 -> s32) at n^3, best of `reps` after warm-up. Used only as the
    INT8 denominator of the TileMix blended peak, never on the measured path."""
    g = torch.Generator(device).manual_seed(0)
    a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device, generator=g)
    b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device, generator=g).t()
    for _ in range(3):
        torch._int_mm(a, b)
    torch.cuda.synchronize(device)
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize(device)
        best = min(best, e0.elapsed_time(e1))
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"bf16": p["bf16_tflops"], "bf16_sustained": p["bf16_tflops_sustained"],
                "hbm_gbs": p["hbm_gbs"], "source": "measured"}
    return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


# ----------------------------------------------------------------------------- workload
ONLY_CASE = None  # --case: run one workload alone (for profiling)


def step_cases():
    from synth import inputs as S

    if ONLY_CASE:
        extra = {c.name: c for c in _step_cases_all()}
        if ONLY_CASE in extra:
            return [extra[ONLY_CASE]]
        return [S.ALL_CASES[ONLY_CASE]()]
    return _step_cases_all()


def _step_cases_all():
    from synth import inputs as S

    dense = S.cfg_pair_4mp_sliced()
    band = S.tilemix_band_4mp()
    scan = S.Case("scanline_4mp", 1, 48, 12, 128, 512, 128, 128, dtype="bf16", mode="scanline", seed=3,
                  window=11, tile_aligned=True, text_pad=512)
    return [dense, band, scan]


def admitted_pairs(case, K) -> int:
    """Admitted (query, key) pairs per (batch, q head), from the library's tile map.
    Dense / TileMix: every pair of real tokens. Scanline with tile_aligned: every
    pair of real tokens inside an active tile."""
    L = case.seq_len
    if case.mode != "scanline":
        return L * L
    T, H, W = case.text_len, case.grid_h, case.grid_w
    if not case.tile_aligned:
        # token rule: text queries see all L keys, image queries the T text keys and
        # the W keys of every row within window // 2 of their own
        half = case.window // 2
        rows = sum(min(H - 1, r + half) - max(0, r - half) + 1 for r in range(H))
        return T * L + H * W * T + rows * W * W
    rp, col, _ = K.get_map("scanline", case.text_len, case.grid_h, case.grid_w, window=case.window,
                           tile_aligned=True, text_pad=case.text_pad)
    T, N = case.text_len, case.grid_h * case.grid_w
    Pt = case.text_pad or max(512, -(-T // TILE) * TILE)

    def valid_in_tile(t):
        s0, s1 = t * TILE, t * TILE + TILE
        return max(0, min(s1, T) - s0) + max(0, min(s1, Pt + N) - max(s0, Pt))

    vt = [valid_in_tile(t) for t in range(len(rp) - 1)]
    total = 0
    for a in range(len(rp) - 1):
        total += vt[a] * sum(vt[b] for b in col[rp[a]:rp[a + 1]])
    return total


def case_flops(case, K) -> float:
    return 4.0 * case.batch * case.q_heads * case.head_dim * admitted_pairs(case, K)


def make_call(case, K, bufs, ws, status):
    """Closures that launch one variant (all its kernels) on the current stream."""
    q, k, v, g, out = bufs
    opts = dict(text_len=case.text_len, grid_h=case.grid_h, grid_w=case.grid_w, mode=case.mode, out=out,
                pattern=case.pattern, percentage=case.percentage, band_blocks=case.band_blocks,
                smooth_k=case.smooth_k, window=case.window, tile_aligned=case.tile_aligned,
                text_pad=case.text_pad, qk_fp32_accumulate=case.qk_fp32_accumulate, status=status)
    if ws is not None:
        opts["workspace"] = ws
    L = case.seq_len
    if case.q_len:
        slices = [(s, min(case.q_len, L - s)) for s in range(0, L, case.q_len)]
    else:
        slices = [(0, 0)]
    launches = []
    for i, (s, n) in enumerate(slices):
        # the query slices are independent (each writes only its own rows): every slice
        # after the first may start while the one before it finishes its last wave
        launches.append(lambda s=s, n=n, ov=i > 0: K.attention(q, k, v, g, q_start=s, q_len=n,
                                                                 overlap_previous=ov, **opts))
    n_kernels = len(slices) + (4 if case.mode == "tilemix" else 0)  # quantiser: 2 mean + 2 quant kernels
    return launches, n_kernels


def median_ms(fns, stream, flush, reps: int = 8, skip: int = 3) -> float:
    """Median CUDA-event time of running `fns` in order on `stream`, L2 flushed
    before each repetition; the first `skip` repetitions are warm-up."""
    times = []
    for it in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for fn in fns:
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        if it >= skip:
            times.append(a.elapsed_time(b))
    return sorted(times)[len(times) // 2]


def time_fused_prologue(K, device, stream, flush, P):
    """The dense 1 MP call on raw q/k projections: the QK prologue as its own pass
    on q and k, then the core, against the prologue on k and the query half fused
    into the core (krea_attn_fwd_rope_q), where q skips one HBM round trip."""
    from synth import inputs as S

    dc = S.dense_1mp()
    qd1, kd1, vd1, gd1 = (t.to(device) for t in S.make_inputs(dc))
    o1 = torch.empty(qd1.shape, dtype=torch.float32, device=device)
    table = K.rope_table(K.rope_positions(dc.text_len, dc.grid_h, dc.grid_w, device))
    qn1, kn1 = torch.empty_like(qd1), torch.empty_like(kd1)
    geo = dict(text_len=dc.text_len, grid_h=dc.grid_h, grid_w=dc.grid_w, out=o1)

    def chained():
        K.qk_prologue(qd1, table, out=qn1)
        K.qk_prologue(kd1, table, out=kn1)
        K.attention(qn1, kn1, vd1, gd1, **geo)

    def fused():
        K.qk_prologue(kd1, table, out=kn1)
        K.attention_rope_q(qd1, kn1, vd1, gd1, table, **geo)

    t_ch, t_fu = median_ms([chained], stream, flush), median_ms([fused], stream, flush)
    return {"prologue_then_attention_ms": round(t_ch, 4), "fused_q_prologue_ms": round(t_fu, 4),
            "speedup": round(t_ch / t_fu, 4), "hbm_bytes_saved": 2 * qd1.numel() * qd1.element_size(),
            "workload": "dense 1 MP on raw q/k projections: qk_prologue(q), qk_prologue(k), attention vs "
                        "qk_prologue(k), attention_rope_q"}


def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest value of x over all ranks (timings are reported as the max)."""
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_rank: float, world: int, ms: float) -> float:
    """Whole-job TFLOP/s: every rank runs the same step (weak scaling), time is the max."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and clock-event reasons sampled DURING the timed region. Reads only:
    NVML queries from a background thread every ~10 ms (so that a timed region of
    a fraction of a second still gets dozens of samples), else `nvidia-smi -lms`.
    start() returns once the first sample is in."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device):
        self.device = device
        self.idx = device.index if device.index is not None else 0
        self.proc = None
        self.file = None
        self.thread = None
        self.samples = []  # (sm_mhz, max_mhz, set of reasons)
        self.source = None

    def _nvml_handle(self):
        import pynvml

        pynvml.nvmlInit()
        try:
            uuid = str(torch.cuda.get_device_properties(self.device).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
        except Exception:  # noqa: BLE001 - fall back to the ordinal
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.idx)

    def start(self):
        try:
            nv, h = self._nvml_handle()
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.stop_flag = threading.Event()

            def poll():
                while not self.stop_flag.is_set():
                    try:
                        sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                        r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                        self.samples.append((sm, mx, {n for n, b in bits.items() if r & b}))
                    except Exception:  # noqa: BLE001 - a failed read is a missing sample
                        pass
                    self.stop_flag.wait(0.01)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
            self.source = "nvml"
        except Exception:  # noqa: BLE001 - no NVML: nvidia-smi
            try:
                self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
                self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.QUERY}",
                                              "--format=csv,noheader,nounits", "-lms", "50"],
                                             stdout=self.file, stderr=subprocess.DEVNULL)
                self.source = "nvidia-smi"
            except (OSError, FileNotFoundError):
                self.proc = None
        t0 = time.time()
        while time.time() - t0 < 5.0 and not self._have_sample():
            time.sleep(0.01)

    def _have_sample(self):
        if self.thread is not None:
            return len(self.samples) > 0
        if self.file is not None:
            return os.path.getsize(self.file.name) > 0
        return True

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            rows = list(self.samples)
        elif self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.file.flush()
            self.file.seek(0)
            rows = []
            for r in (x.split(",") for x in self.file.read().strip().splitlines() if x.strip()):
                if len(r) < 9:
                    continue
                try:
                    rows.append((float(r[1]), float(r[2]),
                                 {n for n, v in zip(self.NAMES, r[5:9]) if "Active" in v and "Not" not in v}))
                except ValueError:
                    continue
            os.unlink(self.file.name)
        else:
            return None
        if not rows:
            return None
        reasons = set().union(*(r[2] for r in rows))
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows), "source": self.source}


# ----------------------------------------------------------------------------- our arm
def clean_flush(flush, clean):
    """Evict L2 for an HBM-bound timing: write `flush` (larger than L2), then read
    `clean` (also larger), so the lines left in L2 are clean and no write-back of
    the flush lands inside the timed region."""
    flush.zero_()
    clean.sum()


CLEAN_L2 = "flushed before each pass: 256 MB written, then another 256 MB read (no dirty lines left)"


def time_prologue(K, device, stream, flush, P, reps: int = 8):
    """The QK prologue (RMSNorm + 3-axis RoPE, one HBM pass) at the 4 MP shape, bound
    by HBM: algorithmic bytes = every q and k row read once and written once."""
    from synth import inputs as S

    pc = S.Case("prologue_4mp", 1, 48, 12, 128, 512, 128, 128, dtype="bf16", mode="dense", seed=91, prologue=True)
    q_raw, k_raw, _, _ = S.make_inputs(pc)
    qd, kd = q_raw.to(device), k_raw.to(device)
    qo, ko_ = torch.empty_like(qd), torch.empty_like(kd)
    table = K.rope_table(K.rope_positions(pc.text_len, pc.grid_h, pc.grid_w, device))
    clean = torch.empty_like(flush)
    times = []
    for it in range(reps):
        clean_flush(flush, clean)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        K.qk_prologue(qd, table, out=qo)
        K.qk_prologue(kd, table, out=ko_)
        b.record(stream)
        torch.cuda.synchronize(device)
        if it >= 3:
            times.append(a.elapsed_time(b))
    ms = sorted(times)[len(times) // 2]
    nbytes = 2 * (qd.numel() + kd.numel()) * qd.element_size()
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"kernel": "prologue_kernel<bf16, 128> (q then k)", "ms": round(ms, 4), "algorithmic_bytes": nbytes,
            "achieved_gbs": round(gbs, 1), "peak_gbs": P["hbm_gbs"], "frac": round(gbs / P["hbm_gbs"], 4),
            "bound": "hbm", "peak_source": f"{P['source']} copy bandwidth", "l2": CLEAN_L2}


def time_exchange(K, device, stream, flush, P, world: int = 4, reps: int = 8):
    """The sequence <-> head exchange at the 4 MP shape with `world` ranks emulated
    on this GPU (every destination in its own HBM): q through the QK prologue
    into the head shards, gate copied into them, the fp32 output copied back to
    the token shards. Bound by HBM here (by NVLink on real peers); algorithmic
    bytes = every row read once and written once."""
    from diffusion_transformer_attention_bidirectional_b200 import seqpar
    from synth import inputs as S

    pc = S.Case("exchange_4mp", 1, 48, 12, 128, 512, 128, 128, dtype="bf16", mode="dense", seed=93, gate=True,
                prologue=True)
    q_raw, _, _, g = S.make_inputs(pc)
    qd, gd = q_raw.to(device), g.to(device)
    B, L, Hq, d = qd.shape
    Ls = L // world
    table = K.rope_table(K.rope_positions(pc.text_len, pc.grid_h, pc.grid_w, device))
    qh = [torch.empty(B, L, Hq // world, d, dtype=qd.dtype, device=device) for _ in range(world)]
    gh = [torch.empty_like(x) for x in qh]
    oh = [torch.empty(B, L, Hq // world, d, dtype=torch.float32, device=device) for _ in range(world)]
    os_ = [torch.empty(B, Ls, Hq, d, dtype=torch.float32, device=device) for _ in range(world)]
    dq, dg, do = seqpar.Destinations.of(qh), seqpar.Destinations.of(gh), seqpar.Destinations.of(os_)

    clean = torch.empty_like(flush)

    def timed(fn):
        times = []
        for it in range(reps):
            clean_flush(flush, clean)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for r in range(world):
                fn(r)
            b.record(stream)
            torch.cuda.synchronize(device)
            if it >= 3:
                times.append(a.elapsed_time(b))
        return sorted(times)[len(times) // 2]

    res = {"world_emulated": world, "peak_gbs": P["hbm_gbs"], "bound": "hbm",
           "peak_source": f"{P['source']} copy bandwidth", "l2": CLEAN_L2}
    legs = {
        "qk_prologue_to_heads": (lambda r: seqpar.qk_prologue_to_heads(qd[:, r * Ls:(r + 1) * Ls], table, dq, r),
                                 2 * qd.numel() * qd.element_size()),
        "seq_to_heads(gate)": (lambda r: seqpar.seq_to_heads(gd[:, r * Ls:(r + 1) * Ls], dg, r),
                               2 * gd.numel() * gd.element_size()),
        "heads_to_seq(out fp32)": (lambda r: seqpar.heads_to_seq(oh[r], do, r), 2 * B * L * Hq * d * 4),
    }
    for name, (fn, nbytes) in legs.items():
        ms = timed(fn)
        gbs = nbytes / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 4), "algorithmic_bytes": nbytes, "achieved_gbs": round(gbs, 1),
                     "frac": round(gbs / P["hbm_gbs"], 4)}
    return res


def time_backward(K, device, stream, flush, P, reps: int = 6):
    """The backward (prep + dq/dk/dv kernel) on the dense 1 MP shape: 48/12 heads,
    d 128, bf16, gate. Algorithmic FLOPs: five products of 2 d per admitted pair
    (S, dP, dV, dK, dQ), i.e. 10 d per pair per query head."""
    from synth import inputs as S

    c = S.dense_1mp()
    q, k, v, g = (t.to(device) for t in S.make_inputs(c))
    lse = torch.empty(c.batch, c.q_heads, c.seq_len, dtype=torch.float32, device=device)
    out = K.attention(q, k, v, g, text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w, lse=lse)
    dout = torch.randn(out.shape, dtype=torch.float32, device=device, generator=torch.Generator(device).manual_seed(7))
    grads = (torch.empty(out.shape, dtype=torch.float32, device=device),
             torch.empty(k.shape, dtype=torch.float32, device=device),
             torch.empty(v.shape, dtype=torch.float32, device=device),
             torch.empty(out.shape, dtype=torch.float32, device=device))
    p = K.make_params(c.batch, c.q_heads, c.kv_heads, c.head_dim, c.text_len, c.grid_h, c.grid_w, in_dtype=c.dtype)
    scratch = torch.empty(K.bwd_scratch_bytes(c.text_len, c.grid_h, c.grid_w, p), dtype=torch.uint8, device=device)
    times = []
    for it in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        K.attention_backward(q, k, v, g, out, dout, lse, text_len=c.text_len, grid_h=c.grid_h, grid_w=c.grid_w,
                             scratch=scratch, grads=grads)
        b.record(stream)
        torch.cuda.synchronize(device)
        if it >= 2:
            times.append(a.elapsed_time(b))
    ms = sorted(times)[len(times) // 2]
    flops = 10.0 * c.batch * c.q_heads * c.head_dim * c.seq_len * c.seq_len
    return {"workload": "dense 1 MP backward: B=1, 48/12 heads, d=128, 512 text + 64x64, bf16, gate",
            "ms": round(ms, 4), "tflops": round(flops / (ms * 1e-3) / 1e12, 1),
            "frac_of_peak": round(flops / (ms * 1e-3) / 1e12 / P["bf16"], 4),
            "note": "one krea_attn_bwd call: the prep pass (dO, D, dgate; dq zeroed) and the gradient kernel; "
                    "scratch and gradient buffers allocated before the timed region"}


def run_ours(args, rank, world, device):
    import diffusion_transformer_attention_bidirectional_b200 as K
    from synth import inputs as S

    K._lib.lib()
    cases = step_cases()
    P = peaks()
    torch.cuda.set_device(device)
    P["int8"] = measure_int8_peak(device)
    stream = torch.cuda.current_stream(device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    host, dev_bufs, calls, flops, kernels, workspaces = [], [], [], [], 0, []
    for c in cases:
        q, k, v, g = S.make_inputs(c)
        hb = [t.pin_memory() if t is not None else None for t in (q, k, v, g)]
        db = [t.to(device) if t is not None else None for t in hb]
        out = torch.empty(q.shape, dtype=torch.float32, device=device)
        ws = None
        if c.mode == "tilemix":
            p = K.make_params(c.batch, c.q_heads, c.kv_heads, c.head_dim, c.text_len, c.grid_h, c.grid_w,
                              in_dtype=c.dtype, smooth_k=c.smooth_k)
            ws = torch.empty(K.workspace_bytes("tilemix", c.text_len, c.grid_h, c.grid_w, p), dtype=torch.uint8,
                             device=device)
        launches, nk = make_call(c, K, (*db, out), ws, status)
        workspaces.append(ws)
        host.append((hb, torch.empty(out.shape, dtype=out.dtype, pin_memory=True)))
        dev_bufs.append((db, out))
        calls.append(launches)
        flops.append(case_flops(c, K))
        kernels += nk
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)  # 256 MB > 126 MB L2

    def step(timed_events=None):
        # one event pair per variant, around all its launches (an event between two
        # launches would also keep a query slice from overlapping the one before it)
        for vi, launches in enumerate(calls):
            if timed_events is not None:
                timed_events[vi][0].record(stream)
            for fn in launches:
                fn()
            if timed_events is not None:
                timed_events[vi][1].record(stream)

    # the first call of each variant with a cold tile-map cache: the host map build and
    # its upload are inside (the pages' "first render stalls" while masks are built)
    K.clear_cache()
    torch.cuda.synchronize(device)
    first_ms = []
    for launches in calls:
        t0 = time.perf_counter()
        for fn in launches:
            fn()
        torch.cuda.synchronize(device)
        first_ms.append((time.perf_counter() - t0) * 1e3)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during warm-up")

    sampler = ClockSampler(device)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    sampler.start()
    per_step = []
    var_ms = [0.0] * len(calls)
    var_min = [float("inf")] * len(calls)
    for _ in range(args.steps):
        flush.zero_()  # evict L2 between steps, outside the timed span
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in calls]
        step(ev)
        torch.cuda.synchronize(device)
        tot = 0.0
        for vi, (a, b) in enumerate(ev):
            ms = a.elapsed_time(b)
            var_ms[vi] += ms
            var_min[vi] = min(var_min[vi], ms)
            tot += ms
        per_step.append(tot)
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during timing")
    step_ms = max_over_ranks(sum(per_step) / len(per_step), world, device)
    total_flops = sum(flops)
    value = job_throughput(total_flops, world, step_ms)

    # e2e through the public API with host buffers: pinned H2D of every input,
    # the step, D2H of every output, all inside the timed span. Copies run on
    # their own streams so that variant i+1's inputs upload and variant i's
    # output downloads while variant i computes (what a caller streaming
    # requests does); events keep every buffer's reads before its next write.
    e2e_steps = max(1, min(args.steps, 3))
    h2d = sum(t.numel() * t.element_size() for hb, _ in host for t in hb if t is not None)
    d2h = sum(o.numel() * o.element_size() for _, o in host)
    s_in, s_out, s_comp = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    nv = len(calls)
    ev_in = [torch.cuda.Event() for _ in range(nv)]
    ev_done = [torch.cuda.Event() for _ in range(nv)]
    ev_out = [torch.cuda.Event() for _ in range(nv)]
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for si in range(e2e_steps):
        for vi, ((hb, hout), (db, dout)) in enumerate(zip(host, dev_bufs)):
            with torch.cuda.stream(s_in):
                if si > 0:
                    s_in.wait_event(ev_done[vi])  # the previous step finished reading these inputs
                for h_, d_ in zip(hb, db):
                    if h_ is not None:
                        d_.copy_(h_, non_blocking=True)
                ev_in[vi].record(s_in)
            s_comp.wait_event(ev_in[vi])
            if si > 0:
                s_comp.wait_event(ev_out[vi])  # the previous output left the device
            with torch.cuda.stream(s_comp):
                for fn in calls[vi]:
                    fn()
            ev_done[vi].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[vi])
                hout.copy_(dout, non_blocking=True)
                ev_out[vi].record(s_out)
    s_out.wait_event(ev_out[nv - 1])
    e1.record(s_out)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, device)
    e2e_value = job_throughput(total_flops, world, e2e_ms)

    # Checks of the pages' claims, outside the timed step (median of 5, L2 flushed):
    # TileMix band against the same call with every tile FP16 (pattern "zero"),
    # beside the speedup the map predicts when INT8 halves the QK^T half of a tile.
    comparisons = {}
    for i, c in enumerate(cases):
        if c.mode != "tilemix" or c.pattern == "zero" or args.no_comparisons:
            continue
        db, dout = dev_bufs[i]
        zero_calls, _ = make_call(dataclasses.replace(c, pattern="zero"), K, (*db, dout), workspaces[i], status)
        times = {"band": [], "zero": []}
        for _ in range(5):
            for name, fns in (("band", calls[i]), ("zero", zero_calls)):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for fn in fns:
                    fn()
                b.record(stream)
                torch.cuda.synchronize(device)
                times[name].append(a.elapsed_time(b))
        med = {k: sorted(v)[len(v) // 2] for k, v in times.items()}
        rp, col, kind = K.get_map("tilemix", c.text_len, c.grid_h, c.grid_w, pattern=c.pattern,
                                  percentage=c.percentage, band_blocks=c.band_blocks)
        n8 = int(((kind & 2) > 0).sum())
        comparisons[f"{c.name}_vs_pattern_zero"] = {
            "band_ms": round(med["band"], 4), "zero_ms": round(med["zero"], 4),
            "speedup": round(med["zero"] / med["band"], 4),
            "modelled_speedup": round(2 * len(kind) / (2 * (len(kind) - n8) + 1.5 * n8), 4)}
    # Scanline token rule (tile_aligned off) against tile-aligned at 1 MP, where the
    # 64-token rows put two rows in a tile and the two rules differ.
    if not args.no_comparisons:
        from synth import inputs as S

        base = S.scanline_1mp()
        q1, k1, v1, _ = (t.to(device) if t is not None else None for t in S.make_inputs(base))
        o1 = torch.empty(q1.shape, dtype=torch.float32, device=device)
        rec = {}
        for name, ta in (("tile_aligned", True), ("token_rule", False)):
            c = dataclasses.replace(base, tile_aligned=ta)
            fns, _ = make_call(c, K, (q1, k1, v1, None, o1), None, status)
            times = []
            for it in range(8):
                flush.zero_()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for fn in fns:
                    fn()
                b.record(stream)
                torch.cuda.synchronize(device)
                if it >= 3:
                    times.append(a.elapsed_time(b))
            ms = sorted(times)[len(times) // 2]
            pairs = admitted_pairs(c, K)
            rec[name] = {"ms": round(ms, 4), "admitted_pairs": pairs,
                         "tflops": round(case_flops(c, K) / (ms * 1e-3) / 1e12, 1)}
        comparisons["scanline_1mp_token_rule_vs_tile_aligned"] = rec
        # the dense 1 MP forward (48/12 heads, bf16, gate) on the same grid: the scanline
        # mask admits 37.35 % of its pairs, so proportional speed is a time ratio 0.3735
        dc = S.dense_1mp()
        qd1, kd1, vd1, gd1 = (t.to(device) for t in S.make_inputs(dc))
        fns, _ = make_call(dc, K, (qd1, kd1, vd1, gd1, o1), None, status)
        times = []
        for it in range(8):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for fn in fns:
                fn()
            b.record(stream)
            torch.cuda.synchronize(device)
            if it >= 3:
                times.append(a.elapsed_time(b))
        ms = sorted(times)[len(times) // 2]
        comparisons["dense_1mp"] = {"ms": round(ms, 4), "tflops": round(case_flops(dc, K) / (ms * 1e-3) / 1e12, 1),
                                    "workload": "B=1, 48/12 heads, d=128, 512 text + 64x64, bf16, gate"}
        comparisons["scanline_1mp_time_vs_dense_1mp"] = {
            "ratio": round(rec["tile_aligned"]["ms"] / ms, 4),
            "admitted_pair_ratio": round(rec["tile_aligned"]["admitted_pairs"] / (dc.seq_len ** 2), 4)}
        comparisons["qk_prologue_fused_1mp"] = time_fused_prologue(K, device, stream, flush, P)
        del q1, k1, v1, o1, qd1, kd1, vd1, gd1
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} during the comparisons")

    prologue = None if args.no_comparisons else time_prologue(K, device, stream, flush, P)
    backward = None if args.no_comparisons else time_backward(K, device, stream, flush, P)

    # roofline of the dominant kernel: the attention kernel on the dense variant (its
    # launches are attention kernels only, the query slices overlapping), algorithmic
    # FLOPs / event time of the whole variant: the mean launch is that time / slices
    dense_attn_ms = var_ms[0] / args.steps
    achieved = flops[0] / (dense_attn_ms * 1e-3) / 1e12
    traffic, traffic_rec = roofline_traffic()
    names = [c.name for c in cases]
    variants = {}
    for i, c in enumerate(cases):
        ms = var_ms[i] / args.steps
        tf = flops[i] / (ms * 1e-3) / 1e12
        pk = P["bf16"]
        if c.mode == "tilemix":
            # blended peak: the QK^T half of the INT8 tiles' FLOPs at the measured INT8
            # peak, everything else at the measured 16-bit peak
            rp, col, kind = K.get_map("tilemix", c.text_len, c.grid_h, c.grid_w, pattern=c.pattern,
                                      percentage=c.percentage, band_blocks=c.band_blocks)
            n8 = int(((kind & 2) > 0).sum())
            f8 = flops[i] * (n8 / len(kind)) / 2
            pk = flops[i] / ((flops[i] - f8) / P["bf16"] + f8 / P["int8"])
        pks = pk * P["bf16_sustained"] / P["bf16"]
        # the datasheet's dense peaks (2250 TFLOP/s 16-bit, 4500 TOPS INT8), blended the same way
        pkd = DATASHEET_BF16
        if c.mode == "tilemix":
            pkd = flops[i] / ((flops[i] - f8) / DATASHEET_BF16 + f8 / DATASHEET_INT8)
        variants[names[i]] = {"ms": round(ms, 4), "min_ms": round(var_min[i], 4), "tflops": round(tf, 1),
                              "peak_tflops": round(pk, 1), "frac_of_peak": round(tf / pk, 4),
                              "frac_of_sustained_peak": round(tf / pks, 4),
                              "frac_of_datasheet_peak": round(tf / pkd, 4), "gflop": round(flops[i] / 1e9, 1),
                              "first_call_cold_map_ms": round(first_ms[i], 3)}
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "global_batch": world * 4, "seq_len": cases[0].seq_len,
                   "parallelism": f"replicas{world}", "l2": "flushed between steps (256 MB write)"},
        # the timed loop lasts well under a second: the burst bf16 peak is the
        # denominator, the sustained one's fraction is reported beside it
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": P["bf16"],
                     "unit": "TFLOP/s", "frac": round(achieved / P["bf16"], 4),
                     "frac_of_sustained_peak": round(achieved / P["bf16_sustained"], 4),
                     "frac_of_datasheet_peak": round(achieved / DATASHEET_BF16, 4), "traffic": traffic,
                     "kernel": "attn_fwd_kernel<bf16> (dense CFG pair, 5 slices)",
                     "launches": len(calls[0]), "mean_launch_ms": round(dense_attn_ms / len(calls[0]), 4),
                     "timing": "event pair around the variant's launches (later slices overlap the one "
                               "before them): mean launch = that time / launches",
                     "traffic_source": (traffic_rec or {}).get("launch"),
                     "peak_source": f"{P['source']} bf16 burst (sustained {P['bf16_sustained']})",
                     "int8_peak_tops": round(P["int8"], 1), "int8_peak_source": "torch._int_mm 8192^3, best of 10"},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": kernels * args.steps,
        "variants": variants,
        "comparisons": comparisons,
    }
    if prologue is not None:
        res["prologue"] = prologue
    if backward is not None:
        res["backward"] = backward
    dense_tf = next((v["tflops"] for n, v in variants.items() if "cfg_pair" in n), None)
    for n, v in variants.items():
        if dense_tf and n.startswith("scanline"):
            # scanline visits only active tiles: at dense efficiency its time would
            # scale with its admitted pairs, i.e. this ratio would be 1
            comparisons[f"{n}_efficiency_vs_dense"] = round(v["tflops"] / dense_tf, 4)
    if clocks:
        res["clocks"] = clocks
    return res


# ----------------------------------------------------------------------------- oracle (CPU)
def _oracle_admitted_keys(ko, c, rows):
    """Admitted keys of each sampled query row, counted from the oracle's own tile
    map and token rule (dense / TileMix: every key)."""
    L = c.seq_len
    if c.mode != "scanline":
        return [L] * len(rows)
    phys = ko.logical_layout(c.text_len, c.grid_h, c.grid_w, "scanline", c.text_pad)
    slot_of = np.empty(L, dtype=np.int64)
    slot_of[phys[phys >= 0]] = np.nonzero(phys >= 0)[0]
    tile_of = slot_of // TILE
    kind = ko.tile_map(c).kind
    keys = np.arange(L)
    counts = []
    for t in rows:
        adm = kind[tile_of[t], tile_of] >= 0
        if not c.tile_aligned:
            adm &= ko.scanline_token_rule(np.int64(t), keys, c.text_len, c.grid_w, c.window)
        counts.append(int(adm.sum()))
    return counts


_SAMPLE_INPUTS = {}


def oracle_sample(rows_per_tile: int = 4, tile_stride: int = 8):
    """Time the fp64 oracle, as it stands, on a bounded sample of the same workload:
    `rows_per_tile` query rows from every `tile_stride`-th query tile (the last
    tile too), so text and image queries are both sampled; all heads, batch 0.
    FLOPs count each sampled row's own admitted keys. The oracle's per-call work
    that does not scale with the sampled rows (tile map, key centring and INT8
    codes of whole tensors) is timed apart, on a call for one row and one head,
    and taken out of the sampled call's time (seconds = sampled call - that call);
    it is returned beside it. An untimed one-row call comes first, so that both
    timed calls find numpy's large allocations in the same (warm) state; a case
    whose one-row call still takes longer than its sampled call keeps its whole
    time. Returns (flops, seconds, fixed_seconds, rows)."""
    from oracle import krea_oracle as ko
    from synth import inputs as S

    cases = step_cases()
    t_total, t_fixed, f_total, n_rows = 0.0, 0.0, 0.0, 0
    for c in cases:
        key = repr(c)  # the same seeded inputs every call: generated once per case
        if key not in _SAMPLE_INPUTS:
            _SAMPLE_INPUTS[key] = S.make_inputs(c)
        q, k, v, g = _SAMPLE_INPUTS[key]
        L = c.seq_len
        nt = -(-L // TILE)
        tiles = sorted(set(range(0, nt, tile_stride)) | {nt - 1})
        rows = np.array([t * TILE + i for t in tiles for i in range(rows_per_tile) if t * TILE + i < L])
        ko.attention(c, q, k, v, g, rows=rows[:1], batches=[0], heads=[0])  # untimed: warm allocations
        t0 = time.perf_counter()
        ko.attention(c, q, k, v, g, rows=rows[:1], batches=[0], heads=[0])
        t_one = time.perf_counter() - t0
        t0 = time.perf_counter()
        ko.attention(c, q, k, v, g, rows=rows, batches=[0])
        t_call = time.perf_counter() - t0
        if t_one < t_call:
            t_fixed += t_one
            t_total += t_call - t_one
        else:
            t_total += t_call
        f_total += 4.0 * c.q_heads * c.head_dim * sum(_oracle_admitted_keys(ko, c, rows))
        n_rows += len(rows)
    return f_total, t_total, t_fixed, n_rows


def cpu_cores():
    try:
        import threadpoolctl

        info = threadpoolctl.threadpool_info()
        n = max((i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"), default=None)
        if n:
            return n
    except Exception:
        pass
    return os.cpu_count()


def run_reference(args):
    oracle_sample(rows_per_tile=1, tile_stride=64)  # untimed warm-up of numpy / BLAS
    for _ in range(args.warmup):
        oracle_sample(rows_per_tile=1, tile_stride=32)
    runs = [oracle_sample(rows_per_tile=2) for _ in range(args.steps)]
    f = sum(r[0] for r in runs)
    t = sum(r[1] for r in runs)
    fixed = sum(r[2] for r in runs) / len(runs)
    value = f / t / 1e12
    sample = (f"{runs[0][3]} query rows (2 from every 8th query tile and the last) of each variant, all 48 heads, "
              f"batch 0, fp64 numpy oracle; time = sampled call minus a one-row one-head call, whose "
              f"whole-tensor work (map, key centring, INT8 codes) took {fixed:.2f} s per step")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / max(1, args.steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--prologue-only", action="store_true",
                    help="time only the QK prologue at the 4 MP shape (profiling)")
    ap.add_argument("--exchange-only", action="store_true",
                    help="time only the sequence <-> head exchange (ranks emulated on one GPU)")
    ap.add_argument("--fused-prologue-only", action="store_true",
                    help="time only the dense 1 MP call with the query prologue fused, against the chained one")
    ap.add_argument("--backward-only", action="store_true",
                    help="time only the backward at the dense 1 MP shape (profiling)")
    ap.add_argument("--no-comparisons", action="store_true",
                    help="skip the band-vs-zero timing after the timed steps (launch-list captures)")
    ap.add_argument("--case", default=None,
                    help="profile one workload alone (a synth.inputs case or a step variant name)")
    args = ap.parse_args()
    global ONLY_CASE
    ONLY_CASE = args.case
    if args.case:
        args.no_cpu_baseline = True
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    if args.prologue_only or args.backward_only or args.exchange_only or args.fused_prologue_only:
        import diffusion_transformer_attention_bidirectional_b200 as K

        torch.cuda.set_device(device)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        fn = (time_prologue if args.prologue_only else time_exchange if args.exchange_only else
              time_fused_prologue if args.fused_prologue_only else time_backward)
        print(json.dumps(fn(K, device, torch.cuda.current_stream(device), flush, peaks())), flush=True)
        return
    try:
        res = run_ours(args, rank, world, device)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            f, t, fixed, n = oracle_sample(rows_per_tile=16)  # about 10 s of fp64 work on 16 host cores
            res["cpu_baseline"] = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(),
                                   "kind": "oracle",
                                   "sample": f"{n} query rows (16 from every 8th query tile and the last) over the "
                                             f"three variants, all 48 heads, batch 0; {t:.1f} s of fp64 numpy = sampled "
                                             f"calls minus one-row one-head calls, whose whole-tensor work (map, "
                                             f"key centring, INT8 codes: {fixed:.2f} s) is left out"}
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
