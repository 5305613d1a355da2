"""Benchmark of the fused grouped-KV attention forward on B200.

One step = one pass of the hot path over synthetic inputs resident in HBM:
  * prefill: attn_fwd on the Llama-3-8B-shaped causal GQA workload
    (B=1, S=4096, 32 query / 8 KV heads, head dim 128) -- the headline;
  * decode: attn_decode on the GQA decode workload (B=32, cache lengths
    ~U[1024, 32768], 32/8 heads, head dim 128), split-KV + combine;
  * MLA decode: attn_decode on the latent cache (B=64, 4096 rows of 576,
    128 heads, value = first 512 columns).
The other configurations are timed after the step, each in a loop of its
own: the 70B-shaped long prefill (B=1, S=32768, 64 / 8 heads), the tiny
causal forward (B=1, S=64, 4 / 2 heads, head dim 32, a latency), two
small-batch GQA decodes (B=1 at 32768 keys, B=4 at 8192) and two small-batch
MLA decodes (B=1 and B=4 at 4096 keys); so are the rows built beyond the
path (paged prefill and decode, FP8 and RoPE forms).
`value` is prefill TFLOP/s (algorithmic FLOPs: causal pairs only); the
decode regimes are reported in HBM GB/s (algorithmic bytes: the K/V rows
below each sequence's length, plus q, o and lse) under "regimes". Each kernel
is timed with CUDA events on its launching stream; L2 (126 MB) is flushed
before every timed launch by writing a 512 MB buffer and then reading a
256 MB one (so the flush's dirty lines are not written back inside the
timed launch).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Multi-GPU: one rank per GPU (torchrun; `--gpus N` without it starts the N
ranks itself); every rank runs its own replica of the workload (independent
problems, weak scaling), time is the max over ranks, value the sum of all
ranks' work over that time.
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
LONG = "llama3_70b_long_prefill"
TINY = "tiny_prefill"
# the MLA decode: kernel name, launches per call, key of its per-launch DRAM traffic
MLA_KERNEL = "attn::mla::mla_decode_kernel (2-CTA cluster)"
MLA_LAUNCHES = 1
MLA_TRAFFIC_KEY = "mla_decode_kernel"
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


def prefill_fp8_bytes(w) -> float:
    """e4m3 q, k, v (one byte per element) and their fp32 tile scales, the
    bf16 output and the fp32 LSE."""
    tq, tk = -(-w.Sq // 128), -(-w.Skv // 128)
    return float(w.B * w.n_q * w.Sq * w.d_qk + w.B * w.n_kv * w.Skv * (w.d_qk + w.d_v)
                 + 4 * (w.B * w.n_q * tq + 2 * w.B * w.n_kv * tk)
                 + 2 * w.B * w.n_q * w.Sq * w.d_v + 4 * w.B * w.n_q * w.Sq)


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
    milliseconds). Without NVML there is no sample: the summary then reports
    `samples: 0` and no clock."""

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
class Regime:
    """One timed launch sequence of the benchmark: `launch()` enqueues the
    library call(s) on the bench stream; `launches` is how many of this
    library's kernels one call runs; `group` is the timed loop it belongs to
    ("core": the hot-path step; "configs": the other configurations;
    "next": the rows built beyond the path)."""

    def __init__(self, name, group, launches, launch):
        self.name, self.group, self.launches, self.launch = name, group, launches, launch
        self.events = []

    def ms(self):
        return [a.elapsed_time(b) for a, b in self.events]

    def mean_ms(self):
        ms = self.ms()
        return sum(ms) / len(ms) if ms else float("nan")


def _oracle_decode_sample(wd, seqlens, qd, kc, vc, n_seq, d_v=None, cache_bytes=None):
    """The fp64 oracle on the first `n_seq` sequences of a decode workload
    (every (b, h) row of those, the cache trimmed to their longest length;
    the tensors may live on the device, only that slice is copied to the
    host). Returns (seconds, algorithmic bytes of those sequences, threads)."""
    import oracle
    threads = os.cpu_count() or 1
    n_seq = min(n_seq, wd.B)
    sl = seqlens[:n_seq]
    L = int(sl.max())
    qx = oracle._f64(qd[:n_seq, :, None, :])
    kx = oracle._f64(kc[:n_seq, :, :L])
    vx = kx if vc is kc else oracle._f64(vc[:n_seq, :, :L])
    t0 = time.perf_counter()
    oracle.sdpa(qx, kx, vx, False, wd.scale, seqlens=sl.numpy(), d_v=d_v, nthreads=threads)
    dt = time.perf_counter() - t0
    rows = float(sl.long().sum())
    per_row = cache_bytes if cache_bytes is not None else wd.n_kv * (wd.d_qk + wd.d_v) * 2
    nbytes = rows * per_row + n_seq * wd.n_q * (wd.d_qk * 2 + wd.d_v * 2 + 4)
    return dt, nbytes, threads


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
    stream = torch.cuda.current_stream(dev)
    gen_seed_shift = 1000 * rank
    sel = lambda *names: args.only == "all" or args.only in names

    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.zeros(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    flush_sum = torch.empty((), dtype=torch.float32, device=dev)

    def cold_l2(val):
        """Write 512 MB (evicts every line of the 126 MB L2), then read 256 MB so
        that the written lines are back in HBM before the timed launch instead of
        being written back while it runs."""
        flush.fill_(val)
        torch.sum(flush_rd, dim=0, out=flush_sum)

    regimes = {}

    def add(name, group, launches, fn):
        regimes[name] = Regime(name, group, launches, fn)

    # ---- the hot-path step: prefill (headline), GQA decode, MLA decode
    w = inputs.WORKLOADS[HEADLINE]
    wd = inputs.WORKLOADS[DECODE]
    wm = inputs.WORKLOADS[MLA]
    q, k, v = inputs.prefill_inputs(w.B, w.Sq, w.Skv, w.n_q, w.n_kv, w.d_qk, w.d_v, w.seed + gen_seed_shift,
                                    device=dev)
    o = torch.empty((w.B, w.n_q, w.Sq, w.d_v), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.n_q, w.Sq), dtype=torch.float32, device=dev)
    fl_p, by_p = prefill_flops(w), prefill_bytes(w)
    if sel("prefill"):
        add("prefill", "core", 1, lambda: binding.attn_fwd(q, k, v, w.causal, w.scale, o=o, lse=lse, stream=stream))

    seqlens, qd, kc, vc = inputs.decode_inputs(wd.B, wd.n_q, wd.n_kv, wd.d_qk, wd.d_v, wd.Skv, wd.seqlen_range,
                                               wd.seed + gen_seed_shift, device=dev)
    sl_dev = seqlens.to(dev)
    od = torch.empty((wd.B, wd.n_q, wd.d_v), dtype=torch.bfloat16, device=dev)
    ld = torch.empty((wd.B, wd.n_q), dtype=torch.float32, device=dev)
    work = torch.empty(binding.decode_workspace_bytes(wd.B, wd.n_q, wd.n_kv, wd.d_qk, wd.d_v, wd.Skv),
                       dtype=torch.uint8, device=dev)
    by_d, fl_d = decode_bytes(wd, seqlens), decode_flops(wd, seqlens)
    if sel("decode"):
        add("decode", "core", 2, lambda: binding.attn_decode(qd, kc, vc, sl_dev, wd.scale, o=od, lse=ld,
                                                             workspace=work, stream=stream))

    slm, qm, cm = inputs.mla_inputs(wm.B, wm.n_q, wm.d_qk, wm.Skv, wm.seqlen_range, wm.seed + gen_seed_shift,
                                    device=dev)
    cm4 = cm[:, None]
    slm_dev = slm.to(dev)
    om = torch.empty((wm.B, wm.n_q, wm.d_v), dtype=torch.bfloat16, device=dev)
    lm = torch.empty((wm.B, wm.n_q), dtype=torch.float32, device=dev)
    by_m, fl_m = mla_bytes(wm, slm), decode_flops(wm, slm)
    mla_ws_n = binding.decode_workspace_bytes(wm.B, wm.n_q, wm.n_kv, wm.d_qk, wm.d_v, wm.Skv)
    work_m = torch.empty(max(mla_ws_n, 1), dtype=torch.uint8, device=dev)
    if sel("mla"):
        add("mla_decode", "core", MLA_LAUNCHES, lambda: binding.attn_decode(
            qm, cm4, cm4, slm_dev, wm.scale, d_v=wm.d_v, o=om, lse=lm, workspace=work_m, stream=stream))

    # ---- the other configurations: the 70B-shaped long prefill and the tiny one
    if sel("long"):
        wl = inputs.WORKLOADS[LONG]
        ql, kl, vl = inputs.prefill_inputs(wl.B, wl.Sq, wl.Skv, wl.n_q, wl.n_kv, wl.d_qk, wl.d_v,
                                           wl.seed + gen_seed_shift, device=dev)
        ol = torch.empty((wl.B, wl.n_q, wl.Sq, wl.d_v), dtype=torch.bfloat16, device=dev)
        lsel = torch.empty((wl.B, wl.n_q, wl.Sq), dtype=torch.float32, device=dev)
        add("long_prefill", "configs", 1,
            lambda: binding.attn_fwd(ql, kl, vl, wl.causal, wl.scale, o=ol, lse=lsel, stream=stream))
    if sel("tiny"):
        wt = inputs.WORKLOADS[TINY]
        qt, kt, vt = inputs.prefill_inputs(wt.B, wt.Sq, wt.Skv, wt.n_q, wt.n_kv, wt.d_qk, wt.d_v,
                                           wt.seed + gen_seed_shift, device=dev)
        ot = torch.empty((wt.B, wt.n_q, wt.Sq, wt.d_v), dtype=torch.bfloat16, device=dev)
        lset = torch.empty((wt.B, wt.n_q, wt.Sq), dtype=torch.float32, device=dev)
        add("tiny_prefill", "configs", 1,
            lambda: binding.attn_fwd(qt, kt, vt, wt.causal, wt.scale, o=ot, lse=lset, stream=stream))

    # small-batch GQA decode (Llama-3-8B heads, full-length caches): one
    # sequence of 32768 keys and four of 8192, where the split-KV plan must
    # cut the keys finely enough to reach every SM
    small_decode = {"decode_b1_32k": (1, 32768), "decode_b4_8k": (4, 8192)}
    sd = {}
    if sel("small_decode"):
        for name, (Bs, Ls) in small_decode.items():
            sl_s, q_s, k_s, v_s = inputs.decode_inputs(Bs, wd.n_q, wd.n_kv, wd.d_qk, wd.d_v, Ls, (Ls, Ls),
                                                       wd.seed + 100 + Bs + gen_seed_shift, device=dev)
            ws_s = torch.empty(binding.decode_workspace_bytes(Bs, wd.n_q, wd.n_kv, wd.d_qk, wd.d_v, Ls),
                               dtype=torch.uint8, device=dev)
            o_s = torch.empty((Bs, wd.n_q, wd.d_v), dtype=torch.bfloat16, device=dev)
            l_s = torch.empty((Bs, wd.n_q), dtype=torch.float32, device=dev)
            sd[name] = (sl_s, decode_bytes(inputs.Workload(name, "decode", B=Bs, n_q=wd.n_q, n_kv=wd.n_kv,
                                                           d_qk=wd.d_qk, d_v=wd.d_v, seed=0), sl_s))
            sl_s_dev = sl_s.to(dev)
            add(name, "configs", 2, (lambda q_s=q_s, k_s=k_s, v_s=v_s, sl_s_dev=sl_s_dev, ws_s=ws_s, o_s=o_s, l_s=l_s:
                                     binding.attn_decode(q_s, k_s, v_s, sl_s_dev, wd.scale, o=o_s, lse=l_s,
                                                         workspace=ws_s, stream=stream)))

    # small-batch MLA decode (the MLA workload's shape with 1 and 4
    # sequences): the keys of each sequence are cut into chunks over the SMs
    small_mla = {"mla_decode_b1": 1, "mla_decode_b4": 4}
    smla = {}
    if sel("small_decode"):
        for name, Bm in small_mla.items():
            sl_m, q_m, c_m = inputs.mla_inputs(Bm, wm.n_q, wm.d_qk, wm.Skv, (wm.Skv, wm.Skv),
                                               wm.seed + 100 + Bm + gen_seed_shift, device=dev)
            nws = binding.decode_workspace_bytes(Bm, wm.n_q, wm.n_kv, wm.d_qk, wm.d_v, wm.Skv)
            ws_m = torch.empty(max(nws, 1), dtype=torch.uint8, device=dev)
            o_m = torch.empty((Bm, wm.n_q, wm.d_v), dtype=torch.bfloat16, device=dev)
            l_m = torch.empty((Bm, wm.n_q), dtype=torch.float32, device=dev)
            smla[name] = (mla_bytes(inputs.Workload(name, "mla_decode", B=Bm, n_q=wm.n_q, n_kv=1, d_qk=wm.d_qk,
                                                    d_v=wm.d_v, seed=0), sl_m),
                          decode_flops(inputs.Workload(name, "mla_decode", B=Bm, n_q=wm.n_q, n_kv=1, d_qk=wm.d_qk,
                                                       d_v=wm.d_v, seed=0), sl_m), nws > 0)
            c_m4, sl_m_dev = c_m[:, None], sl_m.to(dev)
            add(name, "configs", 2 if nws > 0 else 1,
                (lambda q_m=q_m, c_m4=c_m4, sl_m_dev=sl_m_dev, ws_m=ws_m, o_m=o_m, l_m=l_m:
                 binding.attn_decode(q_m, c_m4, c_m4, sl_m_dev, wm.scale, d_v=wm.d_v, o=o_m, lse=l_m, workspace=ws_m,
                                     stream=stream)))

    # ---- the rows built beyond the path, on the same workloads
    # rotary position embedding (Llama-3 base 500000): prefill takes q, k
    # unrotated, decode a cache that holds rotated keys
    ROPE_BASE = 500000.0
    if sel("rope"):
        cos_p, sin_p = binding.rope_tables(w.Skv, w.d_qk, ROPE_BASE, device=dev)
        cos_d, sin_d = binding.rope_tables(wd.Skv, wd.d_qk, ROPE_BASE, device=dev)
        k_rot = torch.empty_like(k)
        o_r, lse_r = torch.empty_like(o), torch.empty_like(lse)
        od_r, ld_r = torch.empty_like(od), torch.empty_like(ld)
        add("rope_prefill", "next", 2, lambda: binding.attn_fwd_rope(
            q, k, v, w.causal, w.scale, cos_p, sin_p, k_rot=k_rot, o=o_r, lse=lse_r, stream=stream))
        add("rope_decode", "next", 2, lambda: binding.attn_decode_rope(
            qd, kc, vc, sl_dev, wd.scale, cos_d, sin_d, o=od_r, lse=ld_r, workspace=work, stream=stream))

    # the GQA decode workload with its cache in e4m3, one scale per KV head
    if sel("fp8"):
        def to_e4m3(x):
            amax = x.float().abs().amax(dim=(0, 2, 3)).clamp_min(1e-6)
            sc = (amax / 448.0).float()
            return (x.float() / sc[None, :, None, None]).to(torch.float8_e4m3fn), sc.contiguous()
        k8, ks8 = to_e4m3(kc)
        v8, vs8 = to_e4m3(vc)
        of8, lf8 = torch.empty_like(od), torch.empty_like(ld)
        work8 = torch.empty(binding.decode_fp8_workspace_bytes(wd.B, wd.n_q, wd.n_kv, wd.Skv), dtype=torch.uint8,
                            device=dev)
        by_f = decode_bytes(wd, seqlens, cache_elem_bytes=1)
        add("fp8_decode", "next", 2, lambda: binding.attn_decode_fp8(
            qd, k8, v8, ks8, vs8, sl_dev, wd.scale, o=of8, lse=lf8, workspace=work8, stream=stream))
        # the same cache quantised with one scale per 128-key tile of each
        # (sequence, KV head)
        def to_e4m3_tiles(x):
            Bx, nk, S, d = x.shape
            nt = (S + 127) // 128
            xp = torch.nn.functional.pad(x.float(), (0, 0, 0, nt * 128 - S)).view(Bx, nk, nt, 128, d)
            sc = (xp.abs().amax(dim=(3, 4)).clamp_min(1e-6) / 448.0).float().contiguous()
            q8 = (xp / sc[..., None, None]).view(Bx, nk, nt * 128, d)[:, :, :S].to(torch.float8_e4m3fn)
            return q8.contiguous(), sc
        k8t, kst = to_e4m3_tiles(kc)
        v8t, vst = to_e4m3_tiles(vc)
        of8t, lf8t = torch.empty_like(od), torch.empty_like(ld)
        add("fp8_decode_tiles", "next", 2, lambda: binding.attn_decode_fp8_tiles(
            qd, k8t, v8t, kst, vst, sl_dev, wd.scale, o=of8t, lse=lf8t, workspace=work8, stream=stream))
        # the Llama-3-8B prefill with Q, K and V in e4m3, one scale per 128-row
        # tile of each (sequence, head): the widening pass and the attention
        q8p, qsp = to_e4m3_tiles(q)
        k8p, ksp = to_e4m3_tiles(k)
        v8p, vsp = to_e4m3_tiles(v)
        o_f8p, lse_f8p = torch.empty_like(o), torch.empty_like(lse)
        work_f8p = torch.empty(binding.fwd_fp8_workspace_bytes(w.B, w.Sq, w.Skv, w.n_q, w.n_kv, w.d_qk),
                               dtype=torch.uint8, device=dev)
        add("fp8_prefill", "next", 2, lambda: binding.attn_fwd_fp8(
            q8p, k8p, v8p, qsp, ksp, vsp, w.causal, w.scale, o=o_f8p, lse=lse_f8p, workspace=work_f8p,
            stream=stream))

    # the Llama-3-8B prefill with its keys and values in 64-token pages placed
    # in a pool in a seeded random order (chunked-prefill serving layout)
    if sel("paged"):
        PPAGE = 64
        Pp = w.Skv // PPAGE
        perm_p = torch.randperm(Pp, generator=torch.Generator().manual_seed(w.seed + 78)).to(torch.int32)
        table_p = perm_p[None].to(dev)
        kd_p = k[0].permute(1, 0, 2).reshape(Pp, PPAGE, w.n_kv, w.d_qk)
        vd_p = v[0].permute(1, 0, 2).reshape(Pp, PPAGE, w.n_kv, w.d_v)
        pool_kp, pool_vp = torch.empty_like(kd_p), torch.empty_like(vd_p)
        pool_kp[perm_p.long().to(dev)] = kd_p
        pool_vp[perm_p.long().to(dev)] = vd_p
        del kd_p, vd_p
        q_packed = q[0].permute(1, 0, 2).contiguous()
        cu_qp = torch.tensor([0, w.Sq], dtype=torch.int32, device=dev)
        sk_p = torch.tensor([w.Skv], dtype=torch.int32, device=dev)
        o_pp = torch.empty_like(q_packed)
        l_pp = torch.empty((w.n_q, w.Sq), dtype=torch.float32, device=dev)
        add("paged_prefill", "next", 1, lambda: binding.attn_fwd_paged(
            q_packed, pool_kp, pool_vp, table_p, cu_qp, sk_p, w.Sq, w.causal, w.scale, o=o_pp, lse=l_pp, stream=stream))

    # the GQA decode workload again, its cache cut into 64-token pages placed
    # in a pool in a seeded random order (the paged-cache serving layout)
    PAGE = 64
    if sel("paged"):
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
        og, lg = torch.empty_like(od), torch.empty_like(ld)
        add("paged_decode", "next", 2, lambda: binding.attn_decode_paged(
            qd, pool_k, pool_v, table_dev, sl_dev, wd.scale, o=og, lse=lg, workspace=work, stream=stream))

    def barrier():
        if ws > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    # The step (the hot path's regimes, one after another) is warmed up and
    # timed in a loop of its own; every other regime gets a loop of its own
    # too, so that neither disturbs the headline nor the others (power and
    # clock state carry over from one kernel to the next). Every timed launch
    # follows an L2 flush and has its own events.
    t_wall = 0.0
    loops = [[r for r in regimes.values() if r.group == "core"]]
    loops += [[r] for g in ("configs", "next") for r in regimes.values() if r.group == g and r.name != "long_prefill"]
    # the long prefill (about 0.4 s of full tensor load) last: the power
    # state it leaves behind would slow whatever ran after it
    loops += [[r] for r in regimes.values() if r.name == "long_prefill"]
    with ClockSampler(torch.cuda.current_device()) as clocks:
        for rs in loops:
            if not rs:
                continue

            def one_step(timed):
                for i, r in enumerate(rs):
                    cold_l2(float(i + 1))
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    r.launch()
                    e1.record(stream)
                    if timed:
                        r.events.append((e0, e1))

            for _ in range(max(3, args.warmup)):
                one_step(False)
            barrier()
            assert binding.device_status(stream) == 0, "device status not clean after warm-up"
            t_wall0 = time.perf_counter()
            for _ in range(args.steps):
                one_step(True)
            barrier()
            t_wall += time.perf_counter() - t_wall0
    st = binding.device_status(stream)
    assert st == 0, f"device status {st}"
    mean = {n: r.mean_ms() for n, r in regimes.items()}
    nan = float("nan")

    # ---- end to end through the public API with host buffers: every step
    # copies its q, k, v from pinned host memory and reads O and LSE back.
    # Steps are pipelined over three streams with two device buffer sets
    # (host-to-device copies of step i+1 and the device-to-host read of step
    # i-1 overlap the attention of step i), the way a serving loop would run.
    e2e = None
    if not args.no_e2e and "prefill" in regimes:
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
    traffic = load_traffic()

    def tf(flops, ms):
        return flops / (ms / 1e3) / 1e12

    def gbs(nbytes, ms):
        return nbytes / (ms / 1e3) / 1e9

    def tensor_roofline(flops, ms, kernel, traffic_key, note=None):
        a = tf(flops, ms)
        r = {"bound": "tensor", "achieved": a, "peak": peak_tf, "unit": "TFLOP/s", "frac": a / peak_tf,
             "traffic": traffic.get(traffic_key), "kernel": kernel,
             "peak_source": f"{peak_src} bf16_tflops (burst)", "algorithmic_flops_per_launch": flops}
        if note:
            r["note"] = note
        return r

    def hbm_roofline(nbytes, ms, kernel, traffic_key, note=None):
        a = gbs(nbytes, ms)
        r = {"bound": "hbm", "achieved": a, "peak": peak_bw, "unit": "GB/s", "frac": a / peak_bw,
             "traffic": traffic.get(traffic_key), "kernel": kernel, "peak_source": f"{peak_src} hbm_gbs",
             "algorithmic_bytes_per_launch": nbytes}
        if note:
            r["note"] = note
        return r

    # ---- the oracle on the host cores, per regime (rank 0 of a 1-GPU run only)
    do_cpu = rank == 0 and ws == 1 and not args.no_cpu_baseline
    cpu = {}
    if do_cpu and "prefill" in regimes:
        dt, fl, threads = oracle_full(w, q.cpu(), k.cpu(), v.cpu())
        cpu["prefill"] = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                          "sample": f"the whole {w.name} workload, all {w.B * w.n_q * w.Sq} query rows "
                                    f"(fp64 plain definition, OpenMP over rows), {dt:.1f} s"}
    if do_cpu and "decode" in regimes:
        n_seq = 8
        dt, nb, threads = _oracle_decode_sample(wd, seqlens, qd, kc, vc, n_seq)
        cpu["decode"] = {"value": nb / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": f"the first {n_seq} of the {wd.B} sequences of {wd.name}, every (b, h) row, "
                                   f"{nb / 1e9:.2f} GB of algorithmic bytes in {dt:.1f} s"}
    if do_cpu and "mla_decode" in regimes:
        n_seq = 16
        dt, nb, threads = _oracle_decode_sample(wm, slm, qm, cm4, cm4, n_seq, d_v=wm.d_v,
                                                cache_bytes=wm.d_qk * 2)
        cpu["mla_decode"] = {"value": nb / dt / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": f"the first {n_seq} of the {wm.B} sequences of {wm.name}, every (b, h) "
                                       f"row, {nb / 1e6:.0f} MB of algorithmic bytes in {dt:.1f} s"}
    if do_cpu and "long_prefill" in regimes:
        n_rows = 2048
        dt, fl, threads = oracle_sample(wl, ql.cpu(), kl.cpu(), vl.cpu(), n_rows, 4242)
        rate = fl / dt
        cpu["long_prefill"] = {"value": rate / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                               "sample": f"{n_rows} seeded query rows of {wl.name} ({dt:.1f} s); the whole "
                                         f"workload extrapolated at that rate: {prefill_flops(wl) / rate:.0f} s",
                               "extrapolated": True}

    # ---- the JSON line
    ms_p, ms_d, ms_m = mean.get("prefill", nan), mean.get("decode", nan), mean.get("mla_decode", nan)
    value = nan
    if "prefill" in regimes:
        agg_p = aggregate({"time_s": sum(regimes["prefill"].ms()) / 1e3, "work": fl_p * args.steps}, ws)
        value = agg_p["work"] / agg_p["time_s"] / 1e12
    out = {}
    if "prefill" in regimes:
        out["prefill"] = {"workload": w.name, "ms": ms_p, "tflops": tf(fl_p, ms_p),
                          "frac_of_peak": tf(fl_p, ms_p) / peak_tf, "frac_of_nominal_2250": tf(fl_p, ms_p) / 2250.0,
                          "algorithmic_flops": fl_p, "algorithmic_bytes": by_p, "cpu_baseline": cpu.get("prefill")}
    if "decode" in regimes:
        agg_d = aggregate({"time_s": sum(regimes["decode"].ms()) / 1e3, "work": by_d * args.steps}, ws)
        out["decode"] = {"workload": wd.name, "ms": ms_d, "gbs": gbs(by_d, ms_d),
                         "aggregate_gbs": agg_d["work"] / agg_d["time_s"] / 1e9,
                         "frac_of_peak": gbs(by_d, ms_d) / peak_bw, "frac_of_nominal_8000": gbs(by_d, ms_d) / 8000.0,
                         "algorithmic_bytes": by_d, "algorithmic_flops": fl_d,
                         "kernels": "attn::dec::decode_split_kernel<4> + decode_combine_kernel",
                         "roofline": hbm_roofline(by_d, ms_d, "attn::dec::decode_split_kernel<4>",
                                                  "decode_split_kernel_4",
                                                  "achieved over split + merge launches; traffic of the split kernel"),
                         "cpu_baseline": cpu.get("decode")}
    if "mla_decode" in regimes:
        t_hbm, t_tc = by_m / (peak_bw * 1e9), fl_m / (peak_tf * 1e12)
        out["mla_decode"] = {"workload": wm.name, "ms": ms_m, "gbs": gbs(by_m, ms_m), "tflops": tf(fl_m, ms_m),
                             "frac_of_peak_hbm": gbs(by_m, ms_m) / peak_bw,
                             "roofline_frac": max(t_hbm, t_tc) / (ms_m / 1e3),
                             "algorithmic_bytes": by_m, "algorithmic_flops": fl_m, "kernel": MLA_KERNEL,
                             "roofline": dict(hbm_roofline(by_m, ms_m, MLA_KERNEL, MLA_TRAFFIC_KEY),
                                              tensor_frac=tf(fl_m, ms_m) / peak_tf),
                             "cpu_baseline": cpu.get("mla_decode")}
    if "long_prefill" in regimes:
        ms_l = mean["long_prefill"]
        fl_l = prefill_flops(wl)
        out["long_prefill"] = {"workload": wl.name, "ms": ms_l, "tflops": tf(fl_l, ms_l),
                               "frac_of_peak": tf(fl_l, ms_l) / peak_tf,
                               "frac_of_nominal_2250": tf(fl_l, ms_l) / 2250.0,
                               "algorithmic_flops": fl_l, "algorithmic_bytes": prefill_bytes(wl),
                               "roofline": tensor_roofline(fl_l, ms_l, "attn::pf::prefill_kernel<128>",
                                                           "prefill_kernel_128_long"),
                               "cpu_baseline": cpu.get("long_prefill")}
    if "tiny_prefill" in regimes:
        ms_t = mean["tiny_prefill"]
        fl_t = prefill_flops(wt)
        lat = sorted(regimes["tiny_prefill"].ms())
        out["tiny_prefill"] = {"workload": wt.name, "ms": ms_t, "latency_us": 1e3 * ms_t,
                               "latency_us_median": 1e3 * lat[len(lat) // 2], "tflops": tf(fl_t, ms_t),
                               "algorithmic_flops": fl_t, "bound": "launch latency (one CTA, one key tile)"}
    for name in small_decode:
        if name not in regimes:
            continue
        ms_s = mean[name]
        sl_s, by_s = sd[name]
        Bs, Ls = small_decode[name]
        out[name] = {"workload": f"GQA decode, B={Bs}, every cache length {Ls}, n_q={wd.n_q} n_kv={wd.n_kv} d=128",
                     "ms": ms_s, "gbs": gbs(by_s, ms_s), "frac_of_peak": gbs(by_s, ms_s) / peak_bw,
                     "algorithmic_bytes": by_s,
                     "roofline": hbm_roofline(by_s, ms_s, "attn::dec::decode_split_kernel<4>", None,
                                              "achieved over split + merge launches")}
    for name, Bm in small_mla.items():
        if name not in regimes:
            continue
        ms_s = mean[name]
        by_s, fl_s, split = smla[name]
        t_hbm, t_tc = by_s / (peak_bw * 1e9), fl_s / (peak_tf * 1e12)
        out[name] = {"workload": f"MLA absorbed decode, B={Bm}, S=4096, 128 heads, key 576 / value 512",
                     "ms": ms_s, "gbs": gbs(by_s, ms_s), "tflops": tf(fl_s, ms_s),
                     "roofline_frac": max(t_hbm, t_tc) / (ms_s / 1e3), "split_kv": split,
                     "algorithmic_bytes": by_s, "algorithmic_flops": fl_s,
                     "roofline": dict(hbm_roofline(by_s, ms_s, MLA_KERNEL, None,
                                                   "achieved over split + merge launches" if split else None),
                                      tensor_frac=tf(fl_s, ms_s) / peak_tf)}
    if "paged_decode" in regimes:
        ms_g = mean["paged_decode"]
        out["paged_decode"] = {"workload": f"{wd.name}, {PAGE}-token pages in a shuffled pool", "ms": ms_g,
                               "gbs": gbs(by_d, ms_g), "frac_of_peak": gbs(by_d, ms_g) / peak_bw,
                               "algorithmic_bytes": by_d,
                               "kernels": "attn::dec::decode_split_kernel<4, paged> + decode_combine_kernel"}
    if "paged_prefill" in regimes:
        ms_pp = mean["paged_prefill"]
        out["paged_prefill"] = {"workload": f"{w.name}, keys and values in 64-token pages in a shuffled pool",
                                "ms": ms_pp, "tflops": tf(fl_p, ms_pp), "frac_of_peak": tf(fl_p, ms_pp) / peak_tf,
                                "kernel": "attn::pf::prefill_kernel<128, paged>",
                                "roofline": tensor_roofline(fl_p, ms_pp, "attn::pf::prefill_kernel<128, paged>",
                                                            "prefill_kernel_128_paged")}
    if "fp8_decode" in regimes:
        ms_f = mean["fp8_decode"]
        out["fp8_decode"] = {"workload": f"{wd.name}, e4m3 cache with one scale per KV head", "ms": ms_f,
                             "gbs": gbs(by_f, ms_f), "frac_of_peak": gbs(by_f, ms_f) / peak_bw,
                             "speedup_vs_bf16_cache": (ms_d / ms_f) if "decode" in regimes else None,
                             "algorithmic_bytes": by_f,
                             "kernels": "attn::dec::decode_split_kernel<4, fp8> + decode_combine_kernel",
                             "roofline": hbm_roofline(by_f, ms_f, "attn::dec::decode_split_kernel<4, fp8>",
                                                      "decode_split_kernel_4_fp8",
                                                      "achieved over split + merge launches; traffic of the "
                                                      "split kernel")}
    if "fp8_decode_tiles" in regimes:
        ms_ft = mean["fp8_decode_tiles"]
        # plus the key and value scales of the tiles below each length
        by_ft = by_f + sum(wd.n_kv * ((int(L) + 127) // 128) * 2 * 4 for L in seqlens.tolist())
        out["fp8_decode_tiles"] = {"workload": f"{wd.name}, e4m3 cache with one scale per 128-key tile",
                                   "ms": ms_ft, "gbs": gbs(by_ft, ms_ft), "frac_of_peak": gbs(by_ft, ms_ft) / peak_bw,
                                   "algorithmic_bytes": by_ft,
                                   "kernels": "attn::dec::decode_split_kernel<4, fp8> (tile scales) + "
                                              "decode_combine_kernel",
                                   "roofline": hbm_roofline(by_ft, ms_ft, "attn::dec::decode_split_kernel<4, fp8>",
                                                            None, "achieved over split + merge launches")}
    if "fp8_prefill" in regimes:
        ms_fp = mean["fp8_prefill"]
        out["fp8_prefill"] = {"workload": f"{w.name}, e4m3 q, k, v with one scale per 128-row tile",
                              "ms": ms_fp, "tflops": tf(fl_p, ms_fp), "frac_of_peak": tf(fl_p, ms_fp) / peak_tf,
                              "algorithmic_flops": fl_p, "algorithmic_bytes": prefill_fp8_bytes(w),
                              "kernels": "attn::f8::widen_e4m3_kernel (keys and values, e4m3 -> bf16) + "
                                         "attn::pf::prefill_kernel<128, fp8> (queries widened in shared memory, "
                                         "tile scales folded in)",
                              "roofline": tensor_roofline(fl_p, ms_fp, "attn::pf::prefill_kernel<128, fp8>",
                                                          "prefill_kernel_128_fp8",
                                                          "achieved over both launches; traffic of the attention "
                                                          "kernel")}
    if "rope_prefill" in regimes:
        ms_rp, ms_rd = mean["rope_prefill"], mean["rope_decode"]
        out["rope_prefill"] = {"workload": f"{w.name}, RoPE base {ROPE_BASE:g} on q and k", "ms": ms_rp,
                               "tflops": tf(fl_p, ms_rp), "frac_of_peak": tf(fl_p, ms_rp) / peak_tf,
                               "overhead_vs_attn_fwd": (ms_rp / ms_p - 1.0) if "prefill" in regimes else None,
                               "kernels": "attn::rope::rope_apply_kernel (keys, once) + "
                                          "attn::pf::prefill_kernel<128, rope> (queries rotated in shared memory)",
                               "roofline": tensor_roofline(fl_p, ms_rp, "attn::pf::prefill_kernel<128, rope>",
                                                           "prefill_kernel_128_rope",
                                                           "achieved over both launches; traffic of the attention "
                                                           "kernel")}
        out["rope_decode"] = {"workload": f"{wd.name}, query rotated at seqlen - 1, cache of rotated keys",
                              "ms": ms_rd, "gbs": gbs(by_d, ms_rd), "frac_of_peak": gbs(by_d, ms_rd) / peak_bw,
                              "kernels": "attn::dec::decode_split_kernel<4> (query rotated in the MMA warp) + "
                                         "decode_combine_kernel"}

    if rank == 0:
        roofline = (tensor_roofline(fl_p, ms_p, "attn::pf::prefill_kernel<128>", "prefill_kernel_128")
                    if "prefill" in regimes else None)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sum(x for x in (ms_p, ms_d, ms_m) if x == x),
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "S": w.Sq, "n_q": w.n_q, "n_kv": w.n_kv, "d": w.d_qk,
                       "causal": w.causal, "decode_workload": wd.name, "mla_workload": wm.name,
                       "l2": "flushed before every timed launch (512 MB write, then 256 MB read)",
                       "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU"},
            "roofline": roofline,
            "regimes": out,
            "cpu_baseline": cpu.get("prefill"),
            "e2e": e2e,
            "clocks": clocks.summary(),
            "gpu_launches": sum(r.launches * len(r.events) for r in regimes.values()) +
                            (args.steps if e2e is not None else 0),
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


def relaunch_ranks(args) -> int:
    """`--gpus N` (N > 1) outside a distributed launch: start N ranks on this
    node with torch.distributed.run (one process per GPU, rendezvous on
    127.0.0.1) running this same command, and return their exit status."""
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


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
    ap.add_argument("--only", default="all",
                    choices=["all", "prefill", "decode", "mla", "long", "tiny", "small_decode", "paged", "fp8", "rope"],
                    help="time one regime only (used for profiling captures)")
    args = ap.parse_args()
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if "WORLD_SIZE" in os.environ:
        ws = int(os.environ["WORLD_SIZE"])
        if ws != args.gpus:
            print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={ws}: launch one rank per GPU", file=sys.stderr)
            return 2
    elif args.gpus > 1:
        return relaunch_ranks(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
