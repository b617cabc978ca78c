"""Benchmark of one absorbed MLA decode step (one layer) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]
                    [--workload NAME] [--num-splits S]

A step is the whole hot path over one batch: mla_absorb_q -> mla_decode ->
mla_combine (when split) -> mla_up_proj, through the C ABI. The default
workload is the DeepSeek-V3 decode shape (B=64, H=128, Q=1, Dn=128, Dr=64,
Vd=128, Ckv=512, Lk=4096, bf16 storage, contiguous cache). Inputs are
seeded synthetic data resident in HBM before timing; L2 is flushed (a
256 MiB write) before every timed step, outside the step's events.

Reported (one JSON line from rank 0):
  value        decode tokens/s over all ranks (B*Q*N / max-over-ranks step time)
  roofline     the decode kernel (the dominant launch): algorithmic bytes per
               launch / its mean CUDA-event duration, against measured HBM peak
  step         whole-step bytes, flops, TB/s, TFLOP/s and fraction of
               max(bytes/HBM peak, flops/bf16 peak)
  e2e          the same metric with per-step H2D of q_nope/q_pe from pinned host
               memory and D2H of the output inside the timed region
  cpu_baseline the fp64 oracle timed on the host cores on a bounded sample

With N > 1 (torchrun), each rank decodes its own batch of the same shape
(data-parallel over sequences; no collective on the data path) and the
step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/s and achieved HBM TB/s (% of roofline) per MLA layer, 1×B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the datasheet figures, reported beside the measured-peak fractions
SPEC_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}


def spec_fraction(achieved: float, unit: str) -> float:
    """achieved / the datasheet peak of its unit (HBM GB/s or dense bf16 TFLOP/s)."""
    return achieved / (SPEC_PEAKS["hbm_gbs"] if unit == "GB/s" else SPEC_PEAKS["bf16_tflops"])


L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def make_workload(name: str, rank: int):
    from latent_kv_decode_b200 import workloads as wl
    m = re.fullmatch(r"dsv3_b(\d+)_lk(\d+)", name)
    if m:
        return wl.dsv3(B=int(m.group(1)), Lk=int(m.group(2)), seed=1 + 1000 * rank)
    if name == "longctx_b4_lk131072":
        return wl.longctx(seed=3 + 1000 * rank)
    if name == "ragged_paged_b128_q2":
        return wl.ragged_paged(seed=2 + 1000 * rank)
    if name == "v41_fp4_sink_h64":
        return wl.v41_shared_latent(seed=4 + 1000 * rank)
    raise SystemExit(f"unknown workload {name}")


def max_over_ranks(values, dist=None, device=None):
    """Element-wise max of per-rank floats across the process group (every
    rank gets the result); identity without a group."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tokens_per_s(B: int, Q: int, world: int, step_ms: float) -> float:
    """Whole-job throughput: every rank decodes its own B*Q query rows per step
    (weak scaling), so the job does B*Q*world rows per max-over-ranks step."""
    return B * Q * world / (step_ms * 1e-3)


def workload_desc(w) -> dict:
    if w.q is not None:
        return dict(workload=f"{w.name}: B={w.B} H={w.H} Q={w.Q} Ckv={w.Ckv} Lk={w.Lk}, shared latent "
                             f"(K = V), FP4 E2M1 with an E4M3 scale per 16 (288 B/token), sink, "
                             f"inverse RoPE on the last {w.rope_tail} dims, bf16 q and x",
                    B=w.B, H=w.H, Q=w.Q, Lk=w.Lk, Ckv=w.Ckv, cache="contiguous FP4 entries",
                    l2="flushed before every timed step (256 MiB write)")
    d = dict(workload=f"{w.name}: B={w.B} H={w.H} Q={w.Q} Dn={w.Dn} Dr={w.Dr} Vd={w.Vd} "
                      f"Ckv={w.Ckv} Lk={w.Lk}{' ragged paged' if w.block_table is not None else ''}"
                      f", {w.dtype} storage, fp32 accumulate",
             B=w.B, H=w.H, Q=w.Q, Lk=w.Lk, Dn=w.Dn, Dr=w.Dr, Vd=w.Vd, Ckv=w.Ckv,
             cache="paged 64-token pages" if w.block_table is not None else "contiguous",
             l2="flushed before every timed step (256 MiB write); cache larger than L2")
    return d


def algorithmic(w):
    """Algorithmic bytes / flops of one step and of the decode launch.

    Decode launch: every cache row once (Ckv+Dr elements), q_lat and q_pe
    read once, x written once. Step: cache rows, wkv_b (W_UK and W_UV), q_nope,
    q_pe and out, each once (340,787,200 B for B=64, Lk=4096). Flops: 2*H*Q*(Ckv+Dr) per
    visible token for the scores and 2*H*Q*Ckv for the aggregation, plus the
    two projections 2*B*Q*H*Ckv*(Dn+Vd).
    """
    es = 4 if w.dtype == "f32" else 2
    L = w.lens()
    if w.q is not None:
        # shared latent (K = V = the FP4 latent, 288 B per token): the step is
        # the decode alone (q in, x out); scores and aggregation both Ckv wide
        entry = w.Ckv // 2 + w.Ckv // 16
        HQ = w.H * w.Q
        vis = float(L.sum())
        b = vis * entry + w.B * HQ * w.Ckv * es * 2
        fl = vis * w.Q * w.H * 2 * (2 * w.Ckv)
        return dict(decode_bytes=b, decode_flops=fl, step_bytes=b, step_flops=fl)
    if w.causal:
        vis_rows = sum(int(l) - w.Q + 1 + q for l in L for q in range(w.Q)) / w.Q
    else:
        vis_rows = float(L.sum())
    rows_read = float(L.sum())
    HQ = w.H * w.Q
    dec_bytes = rows_read * (w.Ckv + w.Dr) * es + w.B * HQ * (w.Ckv + w.Dr) * es + w.B * HQ * w.Ckv * es
    dec_flops = vis_rows * w.Q * w.H * 2 * ((w.Ckv + w.Dr) + w.Ckv)
    # the step's unavoidable traffic: cache rows, wkv_b, the queries and the output
    # (q_lat and x are intermediates a fused step would not write)
    step_bytes = (rows_read * (w.Ckv + w.Dr) * es + w.H * (w.Dn + w.Vd) * w.Ckv * es
                  + w.B * HQ * (w.Dn + w.Dr) * es + w.B * HQ * w.Vd * es)
    proj_flops = 2 * w.B * HQ * w.Ckv * (w.Dn + w.Vd)
    return dict(decode_bytes=dec_bytes, decode_flops=dec_flops,
                step_bytes=step_bytes, step_flops=dec_flops + proj_flops)


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons while the timed region runs.

    Read-only NVML queries every 10 ms from a thread (nvidia-smi at 100 ms when
    NVML is unavailable). Nothing here changes a GPU setting.
    """

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4))

    def __init__(self, index: int, period_s: float = 0.01):
        self.index = index
        self.period = period_s
        self.proc = None
        self.nvml = None
        self.lines = []
        self.samples = []          # (sm_mhz, max_mhz, reason bits) from NVML
        self.stop = threading.Event()

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.nvml = (pynvml, h)
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
            return self
        except Exception:
            self.nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _poll(self):
        nv, h = self.nvml
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        while not self.stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(mx), int(bits)))
            except Exception:
                pass
            self.stop.wait(self.period)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        self.stop.set()
        if self.nvml is not None:
            self.t.join(timeout=5)
            try:
                self.nvml[0].nvmlShutdown()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        for s_mhz, m_mhz, bits in self.samples:
            sm.append(s_mhz)
            mx.append(m_mhz)
            reasons.update(n for n, b in self.REASONS if bits & b)
        names = [n for n, _ in self.REASONS]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvml" if self.samples else "nvidia-smi"}


def _code_only(text: str) -> str:
    """C/C++/CUDA source with comments removed and whitespace runs collapsed, so
    that documentation edits do not count as a change of the profiled code.
    String and character literals are kept as they are."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash(files) -> str:
    """Hash of the code (comments stripped) of the named csrc files: the
    profiled kernel's own sources."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "latent_kv_decode_b200", "csrc")
    for f in sorted(files):
        h.update(_code_only(open(os.path.join(csrc, f), encoding="utf-8").read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if the
    summary's kernel sources still hash to the value it was captured with."""
    p = os.path.join(ROOT, "profiles", f"decode_{workload}.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m_files = re.search(r"kernel sources:\s*(.+)", txt)
    m_hash = re.search(r"kernel source hash:\s*`?([0-9a-f]{16})", txt)
    m_bytes = re.search(r"dram bytes per launch:\s*([0-9.eE+]+)", txt)
    if not m_files or not m_hash or not m_bytes:
        return None
    files = m_files.group(1).replace("`", "").split()
    try:
        if m_hash.group(1) != kernel_source_hash(files):
            return None
    except OSError:
        return None
    return float(m_bytes.group(1))


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    from latent_kv_decode_b200 import ops

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = make_workload(args.workload, rank)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def up(a, dtype=dt):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).to(dev)

    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    shared = w.q is not None
    if shared:
        # shared-latent variant (FP4 latent, sink, inverse RoPE): the step is
        # the decode (+ combine); q in, x out
        from latent_kv_decode_b200 import workloads as wlmod
        q = up(w.q)
        kv = torch.from_numpy(wlmod.fp4_random_entries(w.B, w.Lk, w.Ckv)).to(dev)
        sinks = torch.from_numpy(w.sinks.astype(np.float32)).to(dev)
        call = ops.make_decode_args(q, None, kv, None, w.softmax_scale, sinks=sinks,
                                    rope_tail=w.rope_tail, rope_theta=w.rope_theta,
                                    num_splits=args.num_splits, Lk=w.Lk)
        h2d = [q]
        out = call.x
    else:
        q_nope, q_pe, wkv_b = up(w.q_nope), up(w.q_pe), up(w.wkv_b)
        if w.block_table is not None:
            kv, pe = up(w.kv_pool), up(w.pe_pool)
            bt = torch.from_numpy(w.block_table).to(dev)
        else:
            kv, pe = up(w.kv_cache), up(w.pe_cache)
            bt = None
        seq_lens = torch.from_numpy(w.seq_lens).to(dev) if w.seq_lens is not None else None
        q_lat = torch.empty((w.B, w.H, w.Q, w.Ckv), dtype=dt, device=dev)
        out = torch.empty((w.B, w.H, w.Q, w.Vd), dtype=dt, device=dev)
        call = ops.make_decode_args(q_lat, q_pe, kv, pe, w.softmax_scale, seq_lens=seq_lens,
                                    block_table=bt, page_size=w.page_size, causal=w.causal,
                                    num_splits=args.num_splits,
                                    Lk=w.Lk if bt is None else None)
        h2d = [q_nope, q_pe]
    need = ops.workspace_bytes(call)
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    split = call.num_splits > 1
    launches_per_step = (1 if shared else 3) + (1 if split else 0)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        if not shared:
            ops.mla_absorb_q(q_nope, wkv_b, q_lat, stream=stream)
        if evs:
            evs[1].record(stream)
        ops.launch_decode(call, ws, stream=stream)
        if evs:
            evs[2].record(stream)
        if split:
            ops.mla_combine(call, stream=stream)
        if evs:
            evs[3].record(stream)
        if not shared:
            ops.mla_up_proj(call.x, wkv_b, w.Dn, out, stream=stream)
        if evs:
            evs[4].record(stream)

    for _ in range(args.warmup):
        flush.fill_(1.0)
        step()
    torch.cuda.synchronize()

    dist = None
    if world > 1:
        import torch.distributed as dist
    K = args.steps
    # timed steps: events only at the step's ends, so consecutive kernels keep
    # their programmatic (overlapped-prologue) launch edges
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        for i in range(K):
            flush.fill_(float(i))
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    mean_step = sum(step_ms) / K
    # per-kernel breakdown (and the decode launch's own duration for its
    # roofline): a separate pass with an event between every two kernels
    KB = min(K, 100)
    bevs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(KB)]
    for i in range(KB):
        flush.fill_(float(i))
        step(bevs[i])
    torch.cuda.synchronize()
    dec_ms = [e[1].elapsed_time(e[2]) for e in bevs]
    comb_ms = [e[2].elapsed_time(e[3]) for e in bevs]
    abs_ms = [e[0].elapsed_time(e[1]) for e in bevs]
    up_ms = [e[3].elapsed_time(e[4]) for e in bevs]
    mean_dec = sum(dec_ms) / KB

    # end to end: H2D of this step's queries from pinned memory, the calls, D2H of out
    h_in = [t.cpu().pin_memory() for t in h2d]
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for _ in range(3):
        for d_t, h_t in zip(h2d, h_in):
            d_t.copy_(h_t, non_blocking=True)
        step()
        h_out.copy_(out, non_blocking=True)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    for i in range(K):
        flush.fill_(float(i))
        e2e_ev[i][0].record(stream)
        for d_t, h_t in zip(h2d, h_in):
            d_t.copy_(h_t, non_blocking=True)
        step()
        h_out.copy_(out, non_blocking=True)
        e2e_ev[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_mean = sum(e[0].elapsed_time(e[1]) for e in e2e_ev) / K

    mean_step, mean_dec, e2e_mean = max_over_ranks([mean_step, mean_dec, e2e_mean], dist, dev)
    if rank != 0:
        return None

    peaks, psrc = load_peaks()
    hbm = peaks["hbm_gbs"]
    tflops = peaks["bf16_tflops"]
    alg = algorithmic(w)
    dec_gbs = alg["decode_bytes"] / (mean_dec * 1e-3) / 1e9
    step_gbs = alg["step_bytes"] / (mean_step * 1e-3) / 1e9
    step_tf = alg["step_flops"] / (mean_step * 1e-3) / 1e12
    roof_s = max(alg["step_bytes"] / (hbm * 1e9), alg["step_flops"] / (tflops * 1e12))
    tokens = w.B * w.Q * world
    value = job_tokens_per_s(w.B, w.Q, world, mean_step)
    pct = lambda xs, q: float(np.percentile(np.asarray(xs), q))
    res = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(mean_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded N(0,1) inputs, wkv_b N(0,1)/sqrt(512), no trained weights)",
        "config": dict(workload_desc(w), parallelism=f"dp{world}" if world > 1 else "single GPU",
                       num_splits=call.num_splits),
        "roofline": (
            {
                "kernel": "mla_decode (decode kernel, one launch per step)",
                "bound": "hbm",
                "achieved": round(dec_gbs, 1),
                "peak": hbm,
                "unit": "GB/s",
                "frac": round(dec_gbs / hbm, 4),
                "traffic": profiled_traffic(args.workload),
                "peak_source": f"hbm_gbs of {psrc}",
                "algorithmic_bytes_per_launch": int(alg["decode_bytes"]),
            }
            if alg["decode_bytes"] / (hbm * 1e9) >= alg["decode_flops"] / (tflops * 1e12) else
            {
                "kernel": "mla_decode (decode kernel, one launch per step)",
                "bound": "tensor",
                "achieved": round(alg["decode_flops"] / (mean_dec * 1e-3) / 1e12, 2),
                "peak": tflops,
                "unit": "TFLOP/s",
                "frac": round(alg["decode_flops"] / (mean_dec * 1e-3) / 1e12 / tflops, 4),
                "traffic": profiled_traffic(args.workload),
                "peak_source": f"bf16_tflops of {psrc} (dense bf16 MMA; the FP4 cache is dequantised to bf16)",
                "algorithmic_flops_per_launch": int(alg["decode_flops"]),
                "algorithmic_bytes_per_launch": int(alg["decode_bytes"]),
            }
        ),
        "step": {
            "bytes": int(alg["step_bytes"]), "flops": int(alg["step_flops"]),
            "roofline_frac_of_spec": round(
                max(alg["step_bytes"] / (SPEC_PEAKS["hbm_gbs"] * 1e9),
                    alg["step_flops"] / (SPEC_PEAKS["bf16_tflops"] * 1e12)) / (mean_step * 1e-3), 4),
            "TB_per_s": round(step_gbs / 1e3, 4), "TFLOP_per_s": round(step_tf, 2),
            "roofline_us": round(roof_s * 1e6, 2),
            "roofline_frac": round(roof_s / (mean_step * 1e-3), 4),
            "roofline_basis": f"max(bytes/{hbm} GB/s, flops/{tflops} TFLOP/s) of {psrc}",
            "p50_ms": round(pct(step_ms, 50), 5), "p95_ms": round(pct(step_ms, 95), 5),
            "p99_ms": round(pct(step_ms, 99), 5),
            "kernel_ms": {"absorb": round(sum(abs_ms) / KB, 5), "decode": round(mean_dec, 5),
                          "combine": round(sum(comb_ms) / KB, 5), "up_proj": round(sum(up_ms) / KB, 5),
                          "basis": f"separate pass of {KB} steps with an event between kernels"},
        },
        "e2e": {
            "value": round(job_tokens_per_s(w.B, w.Q, world, e2e_mean), 1), "unit": "tokens/s",
            "ms_per_step": round(e2e_mean, 5),
            "h2d_bytes_per_step": int(sum(t.numel() * t.element_size() for t in h2d)),
            "d2h_bytes_per_step": int(out.numel() * out.element_size()),
            "path": ("pinned host q -> mla_decode -> mla_combine -> pinned host x, one stream"
                     if shared else
                     "pinned host q_nope/q_pe -> mla_absorb_q -> mla_decode -> mla_combine -> "
                     "mla_up_proj -> pinned host out, one stream"),
        },
        "gpu_launches": launches_per_step * K,
        "clocks": clk.summary(),
        "peaks": {"hbm_gbs": hbm, "bf16_tflops": tflops, "source": psrc},
    }
    r = res["roofline"]
    r["frac_of_spec"] = round(spec_fraction(r["achieved"], r["unit"]), 4)
    return res


# ---------------------------------------------------------------------------
# oracle timing (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------

def time_oracle(w, budget_s: float = 12.0, min_seqs: int = 1):
    """Run the fp64 oracle sequence by sequence until ``budget_s`` passes.

    Returns (tokens/s, seconds, sequences, cores). BLAS is held to one thread
    (einsum's own loops are single-threaded), so cores = 1.
    """
    from threadpoolctl import threadpool_limits

    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from harness import oracle_step

    done, t0 = 0, time.perf_counter()
    with threadpool_limits(limits=1):
        while done < w.B and (done < min_seqs or time.perf_counter() - t0 < budget_s):
            oracle_step(w, batch=[done])
            done += 1
    el = time.perf_counter() - t0
    return done * w.Q / el, el, done, 1


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return None
    w = make_workload(args.workload, 0)
    per_step = []
    seqs_done = 0
    for _ in range(args.warmup + args.steps):
        tps, el, n, cores = time_oracle(w, budget_s=args.ref_budget)
        per_step.append(el / (n * w.Q))
        seqs_done = n
    sec_per_token = sum(per_step[args.warmup:]) / max(1, args.steps)
    value = 1.0 / sec_per_token
    res = {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(sec_per_token * w.B * w.Q * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) inputs, wkv_b N(0,1)/sqrt(512), no trained weights)",
        "config": dict(workload_desc(w), parallelism="host cores"),
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": f"{seqs_done} of {w.B} sequences per step (whole step "
                                   f"scaled by token count), fp64 NumPy, 1 thread"},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    return res


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="dsv3_b64_lk4096")
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--ref-budget", type=float, default=4.0,
                    help="seconds of oracle work per reference step")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, rank, world, local_rank)
        if res is not None:
            if world == 1 and not args.no_cpu_baseline:
                w = make_workload(args.workload, 0)
                tps, el, n, cores = time_oracle(w, budget_s=15.0)
                res["cpu_baseline"] = {"value": round(tps, 3), "unit": "tokens/s", "cores": cores,
                                       "kind": "oracle",
                                       "sample": f"{n} of {w.B} sequences of the same workload, "
                                                 f"fp64 NumPy oracle, {el:.1f} s, 1 thread"}
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
