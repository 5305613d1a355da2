"""Benchmark of the fused grouped-KV attention forward on B200.

One step = one pass of the hot path over synthetic inputs resident in HBM:
  * prefill: attn_fwd on the Llama-3-8B-shaped causal GQA workload
    (B=1, S=4096, 32 query / 8 KV heads, head dim 128) -- the headline;
  * decode: attn_decode on the GQA decode workload (B=32, cache lengths
    ~U[1024, 32768], 32/8 heads, head dim 128), split-KV + combine;
  * MLA decode: attn_decode on the latent cache (B=64, 4096 rows of 576,
    128 heads, value = first 512 columns).
`value` is prefill TFLOP/s (algorithmic FLOPs: causal pairs only); the
decode regime is reported in HBM GB/s (algorithmic bytes: the K/V rows below
each sequence's length, plus q, o and lse) under "regimes". Each kernel is
timed with CUDA events on its launching stream; L2 (126 MB) is flushed
before every timed launch by writing a 512 MB buffer and then reading a
256 MB one (so the flush's dirty lines are not written back inside the
timed launch).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Multi-GPU: launched by torchrun, one rank per GPU; every rank runs its own
replica of the workload (independent problems, weak scaling), time is the max
over ranks, value the sum of all ranks' work over that time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "prefill TFLOP/s & decode HBM GB/s (fraction of B200 peak), 1 GPU"
HEADLINE = "llama3_8b_prefill"
DECODE = "gqa_decode"
MLA = "mla_decode"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------
# algorithmic work
# ----------------------------------------------------------------------------
def prefill_flops(w) -> float:
    """4 * d per visible (query, key) pair per head: 2d for Q.K^T, 2d for P.V."""
    if w.causal:
        off = w.Skv - w.Sq
        pairs = sum(min(w.Skv, i + off + 1) for i in range(w.Sq))
    else:
        pairs = w.Sq * w.Skv
    return float(w.B * w.n_q * pairs * 2 * (w.d_qk + w.d_v))


def prefill_bytes(w) -> float:
    return float(2 * (w.B * w.n_q * w.Sq * (w.d_qk + w.d_v) + w.B * w.n_kv * w.Skv * (w.d_qk + w.d_v))
                 + 4 * w.B * w.n_q * w.Sq)


def decode_bytes(w, seqlens, cache_elem_bytes=2) -> float:
    """K and V rows below each sequence's length (2 bytes per element, or 1
    for an FP8 cache), q, o (bf16) and lse (fp32)."""
    total_keys = float(sum(int(x) for x in seqlens))
    kv = total_keys * w.n_kv * (w.d_qk + w.d_v) * cache_elem_bytes
    return kv + w.B * w.n_q * (w.d_qk * 2 + w.d_v * 2 + 4)


def decode_flops(w, seqlens) -> float:
    return float(sum(int(x) for x in seqlens)) * w.n_q * 2 * (w.d_qk + w.d_v)


def mla_bytes(w, seqlens) -> float:
    """Each latent row is read once (it is both key and value), plus q, o, lse."""
    rows = float(sum(int(x) for x in seqlens))
    return rows * w.d_qk * 2 + w.B * w.n_q * (w.d_qk * 2 + w.d_v * 2 + 4)


# ----------------------------------------------------------------------------
# measurement helpers
# ----------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """SM clocks and throttle reasons sampled during the timed region.

    Polls NVML every ~2 ms from a thread (the timed region can be a few
    milliseconds); falls back to `nvidia-smi -lms 100` if NVML is missing."""

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
               "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int):
        self.idx = device_index
        self.samples = []          # (sm_mhz, max_mhz, reasons_mask)
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.idx)
            self._max = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._poll, daemon=True)
            self._thread.start()
        except Exception:
            self._nvml = None
        return self

    def _poll(self):
        p = self._nvml
        while not self._stop.is_set():
            try:
                sm = p.nvmlDeviceGetClockInfo(self._h, p.NVML_CLOCK_SM)
                rs = p.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((float(sm), float(self._max), int(rs)))
            except Exception:
                pass
            time.sleep(0.002)

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "source": "none"}
        reasons = sorted({n for (_, _, m) in self.samples for n, bit in self.REASONS.items() if m & bit})
        return {"sm_mhz": statistics.median(s for s, _, _ in self.samples),
                "sm_max_mhz": self.samples[-1][1], "reasons": reasons, "samples": len(self.samples),
                "source": "nvml"}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def aggregate(values: dict, world_size: int):
    """Reduce per-rank numbers: max of times, sum of work. `values` holds
    'time_s' (max-reduced) and 'work' (sum-reduced)."""
    if world_size <= 1:
        return dict(values)
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([values["time_s"]], dtype=torch.float64, device=dev)
    w = torch.tensor([values["work"]], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return {"time_s": float(t.item()), "work": float(w.item())}


# ----------------------------------------------------------------------------
# the CPU oracle leg (reported baseline; also the --impl reference arm)
# ----------------------------------------------------------------------------
def oracle_sample(w, q, k, v, n_rows, seed):
    """Time the fp64 oracle on a seeded sample of query rows of the workload.
    Returns (seconds, algorithmic FLOPs of those rows, threads)."""
    import numpy as np
    import oracle
    from mqa_attention_attn_b200 import inputs
    rows = inputs.sample_rows(n_rows, w.B, w.n_q, w.Sq, seed)[:n_rows]
    rb, rh, ri = rows[:, 0].long(), rows[:, 1].long(), rows[:, 2].long()
    q_rows = q[rb, rh, ri]
    threads = os.cpu_count() or 1
    kd = oracle._f64(k)
    vd = oracle._f64(v)
    off = w.Skv - w.Sq
    flops = float(sum((min(w.Skv, int(i) + off + 1) if w.causal else w.Skv) for i in ri)) * 2 * (w.d_qk + w.d_v)
    t0 = time.perf_counter()
    oracle.sdpa_rows(q_rows, rows.numpy(), kd, vd, w.B, w.n_q, w.Sq, w.causal, w.scale, nthreads=threads)
    dt = time.perf_counter() - t0
    return dt, flops, threads


def oracle_full(w, q, k, v):
    """Time the fp64 oracle on the whole workload (every query row).
    Returns (seconds, algorithmic FLOPs, threads)."""
    import oracle
    threads = os.cpu_count() or 1
    qd, kd, vd = oracle._f64(q), oracle._f64(k), oracle._f64(v)
    t0 = time.perf_counter()
    oracle.sdpa(qd, kd, vd, w.causal, w.scale, nthreads=threads)
    dt = time.perf_counter() - t0
    return dt, prefill_flops(w), threads


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    import torch
    from mqa_attention_attn_b200 import inputs
    w = inputs.WORKLOADS[HEADLINE]
    q, k, v = inputs.make(w, device="cpu")
    n_rows = args.ref_rows
    for i in range(args.warmup):
        oracle_sample(w, q, k, v, n_rows, 1000 + i)
    times, flops = [], []
    threads = os.cpu_count() or 1
    for i in range(args.steps):
        dt, fl, threads = oracle_sample(w, q, k, v, n_rows, 2000 + i)
        times.append(dt)
        flops.append(fl)
    value = sum(flops) / sum(times) / 1e12
    ms = 1e3 * sum(times) / len(times)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "S": w.Sq, "n_q": w.n_q, "n_kv": w.n_kv, "d": w.d_qk,
                   "causal": w.causal, "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"{n_rows} seeded query rows of {w.name} per step (fp64 plain "
                                   f"definition, OpenMP over rows)"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# the CUDA arm
# ----------------------------------------------------------------------------
def run_ours(args):
    import torch
    ws, rank, local = _dist()
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    from mqa_attention_attn_b200 import binding, build, inputs
    build.build_library()
    binding.lib()

    w = inputs.WORKLOADS[HEADLINE]
    wd = inputs.WORKLOADS[DECODE]
    gen_seed_shift = 1000 * rank
    q, k, v = inputs.prefill_inputs(w.B, w.Sq, w.Skv, w.n_q, w.n_kv, w.d_qk, w.d_v, w.seed + gen_seed_shift,
                                    device=dev)
    o = torch.empty((w.B, w.n_q, w.Sq, w.d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.n_q, w.Sq), dtype=torch.float32, device=dev)
    seqlens, qd, kc, vc = inputs.decode_inputs(wd.B, wd.n_q, wd.n_kv, wd.d_qk, wd.d_v, wd.Skv, wd.seqlen_range,
                                               wd.seed + gen_seed_shift, device=dev)
    sl_dev = seqlens.to(dev)
    od = torch.empty((wd.B, wd.n_q, wd.d_v), dtype=torch.bfloat16, device=dev)
    ld = torch.empty((wd.B, wd.n_q), dtype=torch.float32, device=dev)
    wsz = binding.decode_workspace_bytes(wd.B, wd.n_q, wd.n_kv, wd.d_qk, wd.d_v, wd.Skv)
    work = torch.empty(wsz, dtype=torch.uint8, device=dev)
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)

    def cold_l2(val):
        """Write 512 MB (evicts every line of the 126 MB L2), then read 256 MB so
        that the written lines are back in HBM before the timed launch instead of
        being written back while it runs."""
        flush.fill_(val)
        torch.sum(flush_rd, dim=0, out=flush_sum)
    wm = inputs.WORKLOADS[MLA]
    slm, qm, cm = inputs.mla_inputs(wm.B, wm.n_q, wm.d_qk, wm.Skv, wm.seqlen_range, wm.seed + gen_seed_shift,
                                    device=dev)
    cm4 = cm[:, None]
    slm_dev = slm.to(dev)
    om = torch.empty((wm.B, wm.n_q, wm.d_v), dtype=torch.bfloat16, device=dev)
    lm = torch.empty((wm.B, wm.n_q), dtype=torch.float32, device=dev)
    by_m = mla_bytes(wm, slm)
    fl_m = decode_flops(wm, slm)

    stream = torch.cuda.current_stream(dev)
    fl_p = prefill_flops(w)
    by_p = prefill_bytes(w)
    by_d = decode_bytes(wd, seqlens)
    fl_d = decode_flops(wd, seqlens)

    do_p = args.only in ("all", "prefill")
    do_d = args.only in ("all", "decode")
    do_m = args.only in ("all", "mla")
    do_g = args.only in ("all", "paged")
    do_f = args.only in ("all", "fp8")
    do_r = args.only in ("all", "rope")

    # rotary position embedding on the prefill and decode workloads (tables
    # for the Llama-3 base 500000): prefill takes q, k unrotated, decode a
    # cache that holds rotated keys
    ROPE_BASE = 500000.0
    if do_r:
        cos_p, sin_p = binding.rope_tables(w.Skv, w.d_qk, ROPE_BASE, device=dev)
        cos_d, sin_d = binding.rope_tables(wd.Skv, wd.d_qk, ROPE_BASE, device=dev)
        k_rot = torch.empty_like(k)
        o_r, lse_r = torch.empty_like(o), torch.empty_like(lse)
        od_r, ld_r = torch.empty_like(od), torch.empty_like(ld)

    # the GQA decode workload with its cache in e4m3, one scale per KV head
    if do_f:
        def to_e4m3(x):
            amax = x.float().abs().amax(dim=(0, 2, 3)).clamp_min(1e-6)
            sc = (amax / 448.0).float()
            return (x.float() / sc[None, :, None, None]).to(torch.float8_e4m3fn), sc.contiguous()
        k8, ks8 = to_e4m3(kc)
        v8, vs8 = to_e4m3(vc)
        of8 = torch.empty_like(od)
        lf8 = torch.empty_like(ld)
        work8 = torch.empty(binding.decode_fp8_workspace_bytes(wd.B, wd.n_q, wd.n_kv, wd.Skv), dtype=torch.uint8,
                            device=dev)
        by_f = decode_bytes(wd, seqlens, cache_elem_bytes=1)

    # the GQA decode workload again, its cache cut into 64-token pages placed
    # in a pool in a seeded random order (the paged-cache serving layout)
    PAGE = 64
    if do_g:
        P = wd.Skv // PAGE
        npg = (seqlens.long() + PAGE - 1) // PAGE
        b_idx = torch.repeat_interleave(torch.arange(wd.B), npg)
        p_idx = torch.cat([torch.arange(int(n)) for n in npg])
        perm = torch.randperm(len(b_idx), generator=torch.Generator().manual_seed(wd.seed + 77))
        table = torch.zeros(wd.B, P, dtype=torch.int32)
        table[b_idx, p_idx] = perm.to(torch.int32)
        table_dev = table.to(dev)
        pool_k = torch.empty(len(b_idx), PAGE, wd.n_kv, wd.d_qk, dtype=torch.bfloat16, device=dev)
        pool_v = torch.empty_like(pool_k)
        kview = kc.view(wd.B, wd.n_kv, P, PAGE, wd.d_qk).permute(0, 2, 3, 1, 4)
        vview = vc.view(wd.B, wd.n_kv, P, PAGE, wd.d_v).permute(0, 2, 3, 1, 4)
        pid_dev, b_dev, p_dev = perm.to(dev), b_idx.to(dev), p_idx.to(dev)
        pool_k[pid_dev] = kview[b_dev, p_dev]
        pool_v[pid_dev] = vview[b_dev, p_dev]
        del pid_dev, b_dev, p_dev
        og = torch.empty_like(od)
        lg = torch.empty_like(ld)

    # One step of the hot path = prefill, GQA decode, MLA decode (`core`); the
    # regimes of the rows built beyond it (paged, FP8, RoPE: `nxt`) are timed
    # in a loop of their own after it, so that they do not disturb the
    # headline numbers.
    def step(times_p, times_d, times_m=None, times_g=None, times_f=None, times_rp=None, times_rd=None,
             core=True, nxt=True):
        if do_p and core:
            cold_l2(1.0)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            binding.attn_fwd(q, k, v, w.causal, w.scale, o=o, lse=lse, stream=stream)
            e1.record(stream)
            if times_p is not None:
                times_p.append((e0, e1))
        if do_d and core:
            cold_l2(2.0)
            e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e2.record(stream)
            binding.attn_decode(qd, kc, vc, sl_dev, wd.scale, o=od, lse=ld, workspace=work, stream=stream)
            e3.record(stream)
            if times_d is not None:
                times_d.append((e2, e3))
        if do_m and core:
            cold_l2(3.0)
            e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e4.record(stream)
            binding.attn_decode(qm, cm4, cm4, slm_dev, wm.scale, d_v=wm.d_v, o=om, lse=lm, stream=stream)
            e5.record(stream)
            if times_m is not None:
                times_m.append((e4, e5))
        if do_g and nxt:
            cold_l2(4.0)
            e6, e7 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e6.record(stream)
            binding.attn_decode_paged(qd, pool_k, pool_v, table_dev, sl_dev, wd.scale, o=og, lse=lg,
                                      workspace=work, stream=stream)
            e7.record(stream)
            if times_g is not None:
                times_g.append((e6, e7))
        if do_f and nxt:
            cold_l2(5.0)
            e8, e9 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e8.record(stream)
            binding.attn_decode_fp8(qd, k8, v8, ks8, vs8, sl_dev, wd.scale, o=of8, lse=lf8, workspace=work8,
                                    stream=stream)
            e9.record(stream)
            if times_f is not None:
                times_f.append((e8, e9))
        if do_r and nxt:
            cold_l2(6.0)
            e10, e11 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e10.record(stream)
            binding.attn_fwd_rope(q, k, v, w.causal, w.scale, cos_p, sin_p, k_rot=k_rot, o=o_r, lse=lse_r,
                                  stream=stream)
            e11.record(stream)
            if times_rp is not None:
                times_rp.append((e10, e11))
            cold_l2(7.0)
            e12, e13 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e12.record(stream)
            binding.attn_decode_rope(qd, kc, vc, sl_dev, wd.scale, cos_d, sin_d, o=od_r, lse=ld_r, workspace=work,
                                     stream=stream)
            e13.record(stream)
            if times_rd is not None:
                times_rd.append((e12, e13))

    def barrier():
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    tp, td, tm, tg, tf, trp, trd = [], [], [], [], [], [], []
    t_wall = 0.0
    with ClockSampler(torch.cuda.current_device()) as clocks:
        for core, nxt in ((True, False), (False, True)):
            if not ((core and (do_p or do_d or do_m)) or (nxt and (do_g or do_f or do_r))):
                continue
            for _ in range(max(3, args.warmup)):
                step(None, None, core=core, nxt=nxt)
            barrier()
            assert binding.device_status(stream) == 0, "device status not clean after warm-up"
            t_wall0 = time.perf_counter()
            for _ in range(args.steps):
                step(tp, td, tm, tg, tf, trp, trd, core=core, nxt=nxt)
            barrier()
            t_wall += time.perf_counter() - t_wall0
    st = binding.device_status(stream)
    assert st == 0, f"device status {st}"
    ms_p = [a.elapsed_time(b) for a, b in tp] or [float("nan")]
    ms_d = [a.elapsed_time(b) for a, b in td] or [float("nan")]
    ms_m = [a.elapsed_time(b) for a, b in tm] or [float("nan")]
    ms_g = [a.elapsed_time(b) for a, b in tg] or [float("nan")]
    mean_g = sum(ms_g) / len(ms_g)
    ms_f = [a.elapsed_time(b) for a, b in tf] or [float("nan")]
    mean_f = sum(ms_f) / len(ms_f)
    mean_m = sum(ms_m) / len(ms_m)
    mean_p = sum(ms_p) / len(ms_p)
    mean_d = sum(ms_d) / len(ms_d)
    ms_rp = [a.elapsed_time(b) for a, b in trp] or [float("nan")]
    ms_rd = [a.elapsed_time(b) for a, b in trd] or [float("nan")]
    mean_rp = sum(ms_rp) / len(ms_rp)
    mean_rd = sum(ms_rd) / len(ms_rd)

    agg_p = aggregate({"time_s": sum(ms_p) / 1e3, "work": fl_p * args.steps}, ws)
    agg_d = aggregate({"time_s": sum(ms_d) / 1e3, "work": by_d * args.steps}, ws)
    value = agg_p["work"] / agg_p["time_s"] / 1e12
    dec_gbs = agg_d["work"] / agg_d["time_s"] / 1e9

    # ---- end to end through the public API with host buffers: every step
    # copies its q, k, v from pinned host memory and reads O and LSE back.
    # Steps are pipelined over three streams with two device buffer sets
    # (host-to-device copies of step i+1 and the device-to-host read of step
    # i-1 overlap the attention of step i), the way a serving loop would run.
    e2e = None
    if not args.no_e2e and do_p:
        qh, kh, vh = (t.cpu().pin_memory() for t in (q, k, v))
        NB = 2
        dev_in = [tuple(torch.empty_like(t) for t in (q, k, v)) for _ in range(NB)]
        dev_out = [(torch.empty_like(o), torch.empty_like(lse)) for _ in range(NB)]
        host_out = [(torch.empty(o.shape, dtype=o.dtype).pin_memory(),
                     torch.empty(lse.shape, dtype=lse.dtype).pin_memory()) for _ in range(NB)]
        h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh))
        d2h = o.numel() * o.element_size() + lse.numel() * lse.element_size()
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_free = [None] * NB     # attention of the buffer's previous step has read its inputs
        out_free = [None] * NB    # its outputs have been read back

        def e2e_step(i):
            bi = i % NB
            qx, kx, vx = dev_in[bi]
            ox, lx = dev_out[bi]
            oh, lh = host_out[bi]
            if in_free[bi] is not None:
                s_in.wait_event(in_free[bi])
            with torch.cuda.stream(s_in):
                qx.copy_(qh, non_blocking=True)
                kx.copy_(kh, non_blocking=True)
                vx.copy_(vh, non_blocking=True)
            loaded = torch.cuda.Event()
            loaded.record(s_in)
            stream.wait_event(loaded)
            if out_free[bi] is not None:
                stream.wait_event(out_free[bi])
            binding.attn_fwd(qx, kx, vx, w.causal, w.scale, o=ox, lse=lx, stream=stream)
            done = torch.cuda.Event()
            done.record(stream)
            in_free[bi] = done
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                oh.copy_(ox, non_blocking=True)
                lh.copy_(lx, non_blocking=True)
            read = torch.cuda.Event()
            read.record(s_out)
            out_free[bi] = read

        for i in range(3):
            e2e_step(i)
        barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(s_in)
        for i in range(args.steps):
            e2e_step(i)
        s1.record(s_out)
        barrier()
        e2e_ms = s0.elapsed_time(s1) / args.steps
        agg_e = aggregate({"time_s": e2e_ms / 1e3, "work": fl_p}, ws)
        e2e = {"value": agg_e["work"] / agg_e["time_s"] / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "pipelined": "3 streams, 2 buffer sets: copies of neighbouring steps overlap the attention"}

    peaks, peak_src = load_peaks()
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_bw = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    achieved_tf = fl_p / (mean_p / 1e3) / 1e12
    traffic = load_traffic()
    roofline = {"bound": "tensor", "achieved": achieved_tf, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": achieved_tf / peak_tf, "traffic": traffic.get("prefill_kernel_128"),
                "kernel": "attn::pf::prefill_kernel<128>", "peak_source": f"{peak_src} bf16_tflops (burst)",
                "algorithmic_flops_per_launch": fl_p}
    dec_achieved = by_d / (mean_d / 1e3) / 1e9
    regimes = {
        "prefill": {"workload": w.name, "ms": mean_p, "tflops": achieved_tf,
                    "frac_of_peak": achieved_tf / peak_tf, "frac_of_nominal_2250": achieved_tf / 2250.0,
                    "algorithmic_flops": fl_p, "algorithmic_bytes": by_p},
        "decode": {"workload": wd.name, "ms": mean_d, "gbs": dec_achieved, "aggregate_gbs": dec_gbs,
                   "frac_of_peak": dec_achieved / peak_bw, "frac_of_nominal_8000": dec_achieved / 8000.0,
                   "algorithmic_bytes": by_d, "algorithmic_flops": fl_d,
                   "kernels": "attn::dec::decode_split_kernel<4> + decode_combine_kernel",
                   "peak": peak_bw, "peak_source": f"{peak_src} hbm_gbs",
                   "roofline": {"bound": "hbm", "achieved": dec_achieved, "peak": peak_bw, "unit": "GB/s",
                                "frac": dec_achieved / peak_bw, "traffic": traffic.get("decode_split_kernel_4"),
                                "note": "achieved over split + merge launches; traffic of the split kernel"}},
        "mla_decode": {"workload": wm.name, "ms": mean_m, "gbs": by_m / (mean_m / 1e3) / 1e9,
                       "tflops": fl_m / (mean_m / 1e3) / 1e12,
                       "frac_of_peak_hbm": by_m / (mean_m / 1e3) / 1e9 / peak_bw,
                       "roofline_frac": max(by_m / (peak_bw * 1e9), fl_m / (peak_tf * 1e12)) / (mean_m / 1e3),
                       "algorithmic_bytes": by_m, "algorithmic_flops": fl_m,
                       "kernel": "attn::mla::mla_decode_kernel (2-CTA cluster)",
                       "roofline": {"bound": "hbm", "achieved": by_m / (mean_m / 1e3) / 1e9, "peak": peak_bw,
                                    "unit": "GB/s", "frac": by_m / (mean_m / 1e3) / 1e9 / peak_bw,
                                    "traffic": traffic.get("mla_decode_kernel"),
                                    "tensor_frac": fl_m / (mean_m / 1e3) / 1e12 / peak_tf}},
        "paged_decode": {"workload": f"{wd.name}, {PAGE}-token pages in a shuffled pool", "ms": mean_g,
                         "gbs": by_d / (mean_g / 1e3) / 1e9, "frac_of_peak": by_d / (mean_g / 1e3) / 1e9 / peak_bw,
                         "algorithmic_bytes": by_d,
                         "kernels": "attn::dec::decode_split_kernel<4, paged> + decode_combine_kernel"},
        "fp8_decode": {"workload": f"{wd.name}, e4m3 cache with one scale per KV head", "ms": mean_f,
                       "gbs": (by_f / (mean_f / 1e3) / 1e9) if do_f else None,
                       "frac_of_peak": (by_f / (mean_f / 1e3) / 1e9 / peak_bw) if do_f else None,
                       "speedup_vs_bf16_cache": (mean_d / mean_f) if (do_f and do_d) else None,
                       "algorithmic_bytes": by_f if do_f else None,
                       "kernels": "attn::dec::decode_split_kernel<4, fp8> + decode_combine_kernel",
                       "roofline": ({"bound": "hbm", "achieved": by_f / (mean_f / 1e3) / 1e9, "peak": peak_bw,
                                     "unit": "GB/s", "frac": by_f / (mean_f / 1e3) / 1e9 / peak_bw,
                                     "traffic": traffic.get("decode_split_kernel_4_fp8"),
                                     "note": "achieved over split + merge launches; traffic of the split kernel"}
                                    if do_f else None)},
        "rope_prefill": {"workload": f"{w.name}, RoPE base {ROPE_BASE:g} on q and k", "ms": mean_rp,
                         "tflops": (fl_p / (mean_rp / 1e3) / 1e12) if do_r else None,
                         "frac_of_peak": (fl_p / (mean_rp / 1e3) / 1e12 / peak_tf) if do_r else None,
                         "overhead_vs_attn_fwd": (mean_rp / mean_p - 1.0) if (do_r and do_p) else None,
                         "kernels": "attn::rope::rope_apply_kernel (keys, once) + attn::pf::prefill_kernel<128, rope> "
                                    "(queries rotated in shared memory)",
                         "roofline": ({"bound": "tensor", "achieved": fl_p / (mean_rp / 1e3) / 1e12, "peak": peak_tf,
                                       "unit": "TFLOP/s", "frac": fl_p / (mean_rp / 1e3) / 1e12 / peak_tf,
                                       "traffic": traffic.get("prefill_kernel_128_rope"),
                                       "note": "achieved over both launches; traffic of the attention kernel"}
                                      if do_r else None)},
        "rope_decode": {"workload": f"{wd.name}, query rotated at seqlen - 1, cache of rotated keys",
                        "ms": mean_rd, "gbs": (by_d / (mean_rd / 1e3) / 1e9) if do_r else None,
                        "frac_of_peak": (by_d / (mean_rd / 1e3) / 1e9 / peak_bw) if do_r else None,
                        "kernels": "attn::dec::decode_split_kernel<4> (query rotated in the MMA warp) + "
                                   "decode_combine_kernel"},
    }

    cpu_baseline = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline and do_p:
        qc, kc_, vc_ = q.cpu(), k.cpu(), v.cpu()
        dt, fl, threads = oracle_full(w, qc, kc_, vc_)
        cpu_baseline = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                        "sample": f"the whole {w.name} workload, all {w.B * w.n_q * w.Sq} query rows "
                                  f"(fp64 plain definition, OpenMP over rows), {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sum(x for x in (mean_p, mean_d, mean_m) if x == x),
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "S": w.Sq, "n_q": w.n_q, "n_kv": w.n_kv, "d": w.d_qk,
                       "causal": w.causal, "decode_workload": wd.name,
                       "l2": "flushed before every timed launch (512 MB write, then 256 MB read)",
                       "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"},
            "roofline": roofline,
            "regimes": regimes,
            "cpu_baseline": cpu_baseline,
            "e2e": e2e,
            "clocks": clocks.summary(),
            "gpu_launches": (int(do_p) + 2 * int(do_d) + int(do_m) + 2 * int(do_g) + 2 * int(do_f) + 4 * int(do_r)) *
                            args.steps,
            "wall_s_timed_region": t_wall,
        }
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def load_traffic():
    """Per-launch DRAM bytes of the kernels, from the committed ncu summary."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f)
    return {}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-rows", type=int, default=16384,
                    help="query rows of the headline workload per reference-arm step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--only", default="all", choices=["all", "prefill", "decode", "mla", "paged", "fp8", "rope"],
                    help="time one regime only (used for profiling captures)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
