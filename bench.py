#!/usr/bin/env python
"""Benchmark of the tiled attention hot path on B200.

One step is one pass of the whole path over one batch of synthetic input:
  * fa_fwd on the Llama-2-7B-shaped causal prefill (B=32, H=32, L=4096,
    head_dim=128, K scaled by 2), and
  * fa_decode_splitkv on 64 sequences (Hq=32, Hkv=8, head_dim=128, KV lengths
    uniform in [512, 32768], 8 splits) followed by its LSE combine.
Inputs are generated once by the seeded generator and stay resident in HBM;
they are far larger than L2 (3.2 GB prefill, 8.6 GB KV cache), so no flush is
needed between steps.

Reported:
  value    attention TFLOP/s over the whole step (prefill FLOPs by the metric's
           convention 4*B*H*L*L*D/2, plus decode FLOPs 4*Hq*D*sum(len)), summed
           over ranks and divided by the slowest rank's time;
  roofline the prefill kernel (the dominant one) against the measured bf16 peak;
  decode   achieved KV GB/s of the split-KV decode against the measured HBM peak;
  e2e      the same metric through the public API with pinned host buffers,
           host->device copies of every input and device->host copies of every
           output inside the timed region;
  cpu_baseline  the fp64 oracle timed on this host's cores on a bounded sample.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
For N > 1 launch with torch.distributed.run (one process per GPU): every rank
runs its own independent problems (weak scaling, no collective on the data path).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from tiled_attention_23_b200 import synthetic as syn  # noqa: E402

METRIC = "attn fwd TFLOP/s (bf16, causal) & decode KV GB/s, as % of B200 roofline"
UNIT = "TFLOP/s"
PREFILL = syn.LLAMA_PREFILL
DECODE = syn.DECODE
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


# ----------------------------------------------------------------------------
# host-side helpers (unit-tested on CPU)
# ----------------------------------------------------------------------------
def load_peaks(path=os.path.join(ROOT, "MEASURED_PEAKS.json")):
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def decode_flops(seqlens, w=DECODE) -> float:
    """QK^T and PV over every valid key: 4 * Hq * D per key."""
    return 4.0 * w.Hq * w.D * float(np.sum(np.asarray(seqlens, dtype=np.int64)))


def step_flops(seqlens) -> float:
    return PREFILL.flops + decode_flops(seqlens)


CLOCK_FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
                "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
                "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
REASON_NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


def parse_clocks(text: str, index: int | None = None):
    """Summarise nvidia-smi CSV samples: median SM MHz, max MHz, active reasons."""
    sm, mx, reasons = [], [], set()
    for line in text.splitlines():
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < len(CLOCK_FIELDS) or not parts[0].isdigit():
            continue
        if index is not None and int(parts[0]) != index:
            continue
        try:
            sm.append(float(parts[1].split()[0]))
            mx.append(float(parts[2].split()[0]))
        except ValueError:
            continue
        for name, val in zip(REASON_NAMES, parts[5:9]):
            if val.lower() == "active":
                reasons.add(name)
    if not sm:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
    return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
            "samples": len(sm)}


def gpu_smi_id(device_index: int) -> str:
    """nvidia-smi --id for a torch device (its UUID, robust to CUDA_VISIBLE_DEVICES)."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(device_index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:  # pragma: no cover
        return str(device_index)


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""

    def __init__(self, smi_id: str, interval_ms: int = 50):
        self.index, self.interval_ms, self.proc, self.path = smi_id, interval_ms, None, None

    def __enter__(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", "--query-gpu=" + ",".join(CLOCK_FIELDS),
                 "--format=csv,noheader", f"-lms={self.interval_ms}"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        try:
            with open(self.path) as f:
                text = f.read()
            os.unlink(self.path)
        except OSError:
            text = ""
        return parse_clocks(text)


def max_over_ranks(value: float) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def oracle_sample(budget_s: float, prefill_inputs, decode_inputs, nthreads: int, seed: int = 0):
    """Time the fp64 oracle as it stands on a bounded random sample of the step.

    Random prefill query rows, with one random decode (sequence, head) row per
    64 of them, are processed in batches until ``budget_s`` seconds have
    elapsed.  FLOPs are counted by the metric's convention (a
    prefill row counts 4*Lk*D/2, a decode row 4*len*D).
    Returns (TFLOP/s, description, seconds).
    """
    import oracle
    q, k, v = prefill_inputs
    dq, dkc, dvc, lens = decode_inputs
    rng = np.random.default_rng(seed)
    w, d = PREFILL, DECODE
    n_pre_rows = w.B * w.Hq * w.Lq
    flops = 0.0
    rows_p = rows_d = 0
    t0 = time.perf_counter()
    batch = max(64, nthreads * 16)
    while True:
        rp = rng.integers(0, n_pre_rows, size=batch, dtype=np.int64)
        oracle.attention(q, k, v, w.scale, w.causal, rows=rp, nthreads=nthreads)
        flops += batch * 4.0 * w.Lk * w.D / 2
        rows_p += batch
        nd = max(1, batch // 64)
        rd = rng.integers(0, d.B * d.Hq, size=nd, dtype=np.int64)
        oracle.decode(dq, dkc, dvc, lens, d.scale, rows=rd, nthreads=nthreads)
        flops += 4.0 * d.D * float(np.sum(lens[rd // d.Hq].astype(np.int64)))
        rows_d += nd
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    desc = (f"{rows_p} random query rows of {w.name} and {rows_d} random (sequence, head) rows of "
            f"{d.name}, fp64, {nthreads} threads, {el:.1f} s")
    return flops / el / 1e12, desc, el


def _code_only(text: str) -> str:
    """C++ source without comments and blank space, so that comment edits keep the hash."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def prefill_source_hash() -> str:
    """Hash of the prefill kernel's code (comments ignored): ncu traffic counts apply only to this version."""
    import hashlib
    h = hashlib.sha256()
    for name in ("fa_fwd_sm100.cu", "ptx.cuh"):
        with open(os.path.join(ROOT, "tiled_attention_23_b200", "csrc", name), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per full prefill launch from the committed ncu summary, or None
    when the kernel sources changed since the counters were taken."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            tr = json.load(f)
    except (OSError, ValueError):
        return None
    if tr.get("source_hash") != prefill_source_hash():
        return None
    return tr.get("fa_fwd_per_launch_bytes")


def json_line(d: dict) -> str:
    return json.dumps(d, separators=(", ", ": "))


# ----------------------------------------------------------------------------
# reference arm: the fp64 CPU oracle as it stands
# ----------------------------------------------------------------------------
def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    nthreads = host_cores()
    pre = PREFILL.inputs(seed_offset=0)
    dec = DECODE.inputs(seed_offset=0)
    per_step = args.ref_step_seconds
    times, vals, descs = [], [], []
    for i in range(args.warmup + args.steps):
        val, desc, el = oracle_sample(per_step, pre, dec, nthreads, seed=i)
        if i >= args.warmup:
            times.append(el)
            vals.append(val)
            descs.append(desc)
    value = float(np.mean(vals))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * float(np.mean(times)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": config_dict(world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                         "sample": descs[-1] if descs else ""},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json_line(line), flush=True)


def config_dict(world: int) -> dict:
    w, d = PREFILL, DECODE
    return {
        "workload": f"{w.name} + {d.name}",
        "prefill": {"B": w.B, "Lq": w.Lq, "Lk": w.Lk, "Hq": w.Hq, "Hkv": w.Hkv, "D": w.D, "causal": w.causal,
                    "k_scale": 2 ** w.k_pow2, "scale": "1/sqrt(D)"},
        "decode": {"B": d.B, "Hq": d.Hq, "Hkv": d.Hkv, "D": d.D, "len": [d.len_lo, d.len_hi],
                   "max_seqlen": d.Lmax, "num_splits": d.num_splits},
        "l2": "no flush: inputs larger than L2 (3.2 GB prefill Q/K/V, 8.6 GB KV cache)",
        "parallelism": f"replicas x{world} (independent problems per rank)",
    }


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
def run_ours(args, rank: int, world: int, local_rank: int):
    import torch
    from tiled_attention_23_b200 import attention as A

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device; the CUDA path has no fallback")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    A.lib()  # load (and fail loudly) before any timing
    peaks, peak_src = load_peaks()

    # Inputs: independent problems per rank (rank-dependent seed).
    q, k, v = PREFILL.inputs(seed_offset=rank)
    dq_h, dkc_h, dvc_h, lens_h = DECODE.inputs(seed_offset=rank)
    to_dev = A.to_device_bf16
    gq, gk, gv = to_dev(q, dev), to_dev(k, dev), to_dev(v, dev)
    go = torch.empty_like(gq)
    glse = torch.empty((PREFILL.B, PREFILL.Hq, PREFILL.Lq), dtype=torch.float32, device=dev)
    dq, dkc, dvc = to_dev(dq_h, dev), to_dev(dkc_h, dev), to_dev(dvc_h, dev)
    dlens = torch.from_numpy(lens_h).to(dev)
    do = torch.empty_like(dq)
    dlse = torch.empty((DECODE.B, DECODE.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty((A.decode_workspace_bytes(DECODE.B, DECODE.Hq, DECODE.D, DECODE.num_splits),),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize(dev)

    kv_bytes = DECODE.kv_bytes(lens_h)
    flops = step_flops(lens_h)
    launches_per_step = 3   # fa_fwd kernel, decode split kernel, decode combine kernel

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        A.fwd(gq, gk, gv, causal=PREFILL.causal, scale=PREFILL.scale, o=go, lse=glse, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        A.decode_splitkv(dq, dkc, dvc, dlens, DECODE.num_splits, scale=DECODE.scale, o=do, lse=dlse,
                         workspace=ws, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if A.device_status() != A.FA_OK:
        raise SystemExit("bench.py: a kernel reported a timed-out wait during warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(gpu_smi_id(local_rank)) as clk:
        start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        stop.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    clocks = clk.summary()
    if A.device_status() != A.FA_OK:
        raise SystemExit("bench.py: a kernel reported a timed-out wait")
    ms_local = start.elapsed_time(stop)
    ms = max_over_ranks(ms_local)
    pre_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[1].elapsed_time(e[2]) for e in evs]
    pre_avg = max_over_ranks(float(np.mean(pre_ms)))
    dec_avg = max_over_ranks(float(np.mean(dec_ms)))
    ms_per_step = ms / args.steps
    value = world * flops * args.steps / (ms * 1e-3) / 1e12

    prefill_tflops = PREFILL.flops / (pre_avg * 1e-3) / 1e12
    decode_gbs = kv_bytes / (dec_avg * 1e-3) / 1e9
    traffic = profiled_traffic()

    # ------------------------------------------- next-row kernels (outside the timed step)
    extra = {}
    if not args.no_extra:
        extra = run_extra(args, A, dev, stream, (dq, dkc, dvc, dlens), (dq_h, dkc_h, dvc_h, lens_h), ws, peaks,
                          peak_src, (gq, gk, gv, go, glse), rank)

    # ---------------------------------------------------------------- e2e
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, A, dev, stream, (q, k, v), (dq_h, dkc_h, dvc_h, lens_h), flops, world)

    # ---------------------------------------------------------------- cpu baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        nthreads = host_cores()
        val, desc, _ = oracle_sample(args.cpu_seconds, (q, k, v), (dq_h, dkc_h, dvc_h, lens_h), nthreads)
        cpu = {"value": val, "unit": UNIT, "cores": nthreads, "kind": "oracle", "sample": desc}

    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_dict(world),
        # The timed region is short (K steps of a few ms each, well under the
        # seconds it takes the power cap to pull the clock down), so the
        # denominator is the burst bf16 figure; the sustained one is beside it.
        "roofline": {"bound": "tensor", "kernel": "fa_fwd_pair_kernel<128, causal>",
                     "achieved": prefill_tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": prefill_tflops / peaks["bf16_tflops"], "traffic": traffic,
                     "peak_source": f"{peak_src} bf16 burst (cuBLAS GEMM, best of 10)",
                     "frac_of_sustained": prefill_tflops / peaks["bf16_tflops_sustained"],
                     "ms_per_launch": pre_avg, "ms_per_launch_sd": float(np.std(pre_ms)),
                     "ms_per_launch_min": float(np.min(pre_ms))},
        "decode": {"bound": "hbm", "kernel": "fa_decode_split_kernel<128> + combine",
                   "achieved": decode_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                   "frac": decode_gbs / peaks["hbm_gbs"], "kv_bytes": kv_bytes, "ms_per_call": dec_avg,
                   "ms_per_call_sd": float(np.std(dec_ms)),
                   "peak_source": f"{peak_src} copy"},
        **extra,
        "e2e": e2e,
        "cpu_baseline": cpu,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    print(json_line(line), flush=True)


def time_calls(fn, stream, reps: int, warmup: int = 3) -> float:
    """Mean device time (ms) of ``fn`` over ``reps`` back-to-back calls on ``stream``."""
    import torch
    for _ in range(warmup):
        fn()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    torch.cuda.synchronize()
    ev[0].record(stream)
    for _ in range(reps):
        fn()
    ev[1].record(stream)
    torch.cuda.synchronize()
    return ev[0].elapsed_time(ev[1]) / reps


def run_extra(args, A, dev, stream, decode_dev, decode_host, ws, peaks, peak_src, prefill_dev, rank):
    """Kernels of the rows beyond the step, each against its own roofline.

    decode_paged: the decode workload with its KV cache laid out in 64-key
    pages in a seeded random order (same keys, same algorithmic bytes).
    decode_int8: the decode workload with K and V quantised to int8 (one fp32
    scale per token and head); algorithmic bytes are the codes plus scales.
    prefill_varlen: a packed batch of 32 causal sequences of seeded lengths in
    [256, 8192] with the Llama-shaped heads (FLOPs by the causal convention,
    per sequence).
    prefill_fp8: fa_fwd_fp8 on the Llama-shaped prefill with Q, K, V quantised
    per head to e4m3 by fa_quantize_fp8 (same FLOPs; peak = twice the bf16
    peak, the nominal fp8/bf16 ratio); quantize_fp8: the quantiser on Q.
    prefill_long_gqa: the long-context head_dim-256 causal prefill (B2 Hq32
    L8192) for GQA groups 1/2/4/8; prefill_fp8_long_gqa: its FP8 form at G = 4.
    backward: fa_bwd on the Llama-shaped prefill (its O and lse from the timed
    forward, a seeded upstream gradient); algorithmic FLOPs 2.5x the forward's
    (five products of the same size), halved when causal.
    """
    import torch
    dq, dkc, dvc, dlens = decode_dev
    q_h, kc_h, vc_h, lens_h = decode_host
    out = {}
    kp, vp, table = syn.paginate(kc_h, vc_h, lens_h, syn.DECODE_PAGE_SIZE, seed=7, spare_pages=16)
    dkp, dvp = A.to_device_bf16(kp, dev), A.to_device_bf16(vp, dev)
    dtab = torch.from_numpy(table).to(dev)
    del kp, vp
    do = torch.empty_like(dq)
    dlse = torch.empty((DECODE.B, DECODE.Hq), dtype=torch.float32, device=dev)

    def paged():
        A.decode_paged(dq, dkp, dvp, dtab, dlens, DECODE.num_splits, scale=DECODE.scale, o=do, lse=dlse,
                       workspace=ws, stream=stream)
    ms = time_calls(paged, stream, reps=max(10, args.steps // 2))
    if A.device_status() != A.FA_OK:
        raise SystemExit("bench.py: a kernel reported a timed-out wait")
    gbs = DECODE.kv_bytes(lens_h) / (ms * 1e-3) / 1e9
    out["decode_paged"] = {"bound": "hbm", "kernel": "fa_decode_split_kernel<128, paged> + combine",
                           "page_size": syn.DECODE_PAGE_SIZE, "achieved": gbs, "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "ms_per_call": ms,
                           "peak_source": f"{peak_src} copy"}
    del dkp, dvp
    torch.cuda.empty_cache()

    # int8 KV cache (K and V int8), quantised on the device by the library
    kq, ks = A.quantize_kv_int8(dkc)
    vq, vs = A.quantize_kv_int8(dvc)

    def int8():
        A.decode_int8(dq, kq, ks, vq, vs, dlens, DECODE.num_splits, scale=DECODE.scale, o=do, lse=dlse,
                      workspace=ws, stream=stream)
    ms = time_calls(int8, stream, reps=max(10, args.steps // 2))
    if A.device_status() != A.FA_OK:
        raise SystemExit("bench.py: a kernel reported a timed-out wait")
    i8_bytes = int(np.sum(lens_h.astype(np.int64))) * DECODE.Hkv * (2 * DECODE.D + 2 * 4)
    gbs = i8_bytes / (ms * 1e-3) / 1e9
    out["decode_int8"] = {"bound": "hbm", "kernel": "fa_decode_split_i8_kernel<128, v_int8> + combine",
                          "kv_bytes": i8_bytes, "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                          "frac": gbs / peaks["hbm_gbs"], "ms_per_call": ms,
                          "peak_source": f"{peak_src} copy"}
    del kq, ks, vq, vs
    torch.cuda.empty_cache()

    # packed variable-length causal prefill (block-diagonal), tensor-bound
    vw = syn.VARLEN_PREFILL
    vq, vk, vv, cu = vw.inputs()
    lens = np.diff(cu)
    gq, gk, gv = (A.to_device_bf16(x, dev) for x in (vq, vk, vv))
    gcu = torch.from_numpy(cu).to(dev)
    del vq, vk, vv
    go = torch.empty_like(gq)
    glse = torch.empty((vw.Hq, gq.shape[0]), dtype=torch.float32, device=dev)
    max_q = int(lens.max())

    def varlen():
        A.fwd_varlen(gq, gk, gv, gcu, gcu, max_q, causal=vw.causal, scale=vw.scale, o=go, lse=glse, stream=stream)
    ms = time_calls(varlen, stream, reps=max(5, args.steps // 4))
    if A.device_status() != A.FA_OK:
        raise SystemExit("bench.py: a kernel reported a timed-out wait")
    tf = vw.flops(lens) / (ms * 1e-3) / 1e12
    out["prefill_varlen"] = {"bound": "tensor", "kernel": "fa_fwd_pair_kernel<128, causal, varlen>",
                             "workload": vw.name, "tokens": int(cu[-1]), "achieved": tf,
                             "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": tf / peaks["bf16_tflops"], "ms_per_call": ms,
                             "frac_of_sustained": tf / peaks["bf16_tflops_sustained"],
                             "peak_source": f"{peak_src} bf16 burst"}
    del gq, gk, gv, go, glse
    torch.cuda.empty_cache()

    # FP8 (e4m3) forward of the Llama-shaped causal prefill: Q, K, V quantised
    # per head on the device by the library (timed separately), then attended
    pq, pk, pv, po, plse = prefill_dev
    q8, qd = A.quantize_fp8(pq, stream=stream)
    k8, kd = A.quantize_fp8(pk, stream=stream)
    v8, vd = A.quantize_fp8(pv, stream=stream)
    o8 = torch.empty_like(po)
    lse8 = torch.empty_like(plse)

    def fp8():
        A.fwd_fp8(q8, k8, v8, qd, kd, vd, causal=PREFILL.causal, scale=PREFILL.scale, o=o8, lse=lse8,
                  stream=stream)
    ms = time_calls(fp8, stream, reps=max(5, args.steps // 4))
    if A.device_status() != A.FA_OK:
        raise SystemExit("bench.py: a kernel reported a timed-out wait")
    tf = PREFILL.flops / (ms * 1e-3) / 1e12
    fp8_peak = 2.0 * peaks["bf16_tflops"]
    out["prefill_fp8"] = {"bound": "tensor", "kernel": "fa_fwd_pair_kernel<128, causal, fp8>",
                          "workload": PREFILL.name, "achieved": tf, "peak": fp8_peak, "unit": "TFLOP/s",
                          "frac": tf / fp8_peak, "ms_per_call": ms,
                          "frac_of_bf16_peak": tf / peaks["bf16_tflops"],
                          "peak_source": f"{peak_src} bf16 burst x 2 (nominal fp8/bf16 ratio 4.5/2.25)"}

    def quant():
        A.quantize_fp8(pq, out=q8, descale=qd, stream=stream)
    ms = time_calls(quant, stream, reps=max(5, args.steps // 4))
    n_el = pq.numel()
    gbs = 3.0 * n_el / (ms * 1e-3) / 1e9
    out["quantize_fp8"] = {"bound": "hbm", "kernels": "amax_kernel<128> + quantize_kernel<128> + finalize",
                           "tensor": "Q of " + PREFILL.name, "achieved": gbs, "peak": peaks["hbm_gbs"],
                           "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "ms_per_call": ms,
                           "bytes_convention": "3 B per element (bf16 read + e4m3 write); the two passes "
                                               "move 5 B per element",
                           "peak_source": f"{peak_src} copy"}
    del q8, k8, v8, qd, kd, vd, o8, lse8
    torch.cuda.empty_cache()

    # long-context GQA prefill (head_dim 256), per group size, and its FP8 form at G = 4
    per_g = {}
    for g in (1, 2, 4, 8):
        lw = syn.LONG_GQA[g]
        lq, lk, lv = (A.to_device_bf16(x, dev) for x in lw.inputs(seed_offset=rank))
        lo = torch.empty_like(lq)
        llse = torch.empty((lw.B, lw.Hq, lw.Lq), dtype=torch.float32, device=dev)

        def long_fwd():
            A.fwd(lq, lk, lv, causal=lw.causal, scale=lw.scale, o=lo, lse=llse, stream=stream)
        ms = time_calls(long_fwd, stream, reps=max(5, args.steps // 4))
        tf = lw.flops / (ms * 1e-3) / 1e12
        per_g[str(g)] = {"workload": lw.name, "achieved": tf, "ms_per_call": ms}
        if g == 4:
            l8 = [A.quantize_fp8(x, stream=stream) for x in (lq, lk, lv)]

            def long_fp8():
                A.fwd_fp8(l8[0][0], l8[1][0], l8[2][0], l8[0][1], l8[1][1], l8[2][1], causal=lw.causal,
                          scale=lw.scale, o=lo, lse=llse, stream=stream)
            ms8 = time_calls(long_fp8, stream, reps=max(5, args.steps // 4))
            tf8 = lw.flops / (ms8 * 1e-3) / 1e12
            out["prefill_fp8_long_gqa"] = {"bound": "tensor", "kernel": "fa_fwd_single_kernel<256, 64, causal, fp8>",
                                           "workload": lw.name, "achieved": tf8, "peak": fp8_peak,
                                           "unit": "TFLOP/s", "frac": tf8 / fp8_peak, "ms_per_call": ms8,
                                           "peak_source": f"{peak_src} bf16 burst x 2"}
            del l8
        del lq, lk, lv, lo, llse
        torch.cuda.empty_cache()
    if A.device_status() != A.FA_OK:
        raise SystemExit("bench.py: a kernel reported a timed-out wait")
    worst = min(v["achieved"] for v in per_g.values())
    out["prefill_long_gqa"] = {"bound": "tensor", "kernel": "fa_fwd_single_kernel<256, 64, causal>",
                               "per_group": per_g, "achieved": worst, "peak": peaks["bf16_tflops"],
                               "unit": "TFLOP/s", "frac": worst / peaks["bf16_tflops"],
                               "frac_of_sustained": worst / peaks["bf16_tflops_sustained"],
                               "note": "achieved = the slowest group size",
                               "peak_source": f"{peak_src} bf16 burst"}

    # backward of the Llama-shaped causal prefill
    dout = A.to_device_bf16(syn.normal_bf16((PREFILL.B, PREFILL.Lq, PREFILL.Hq, PREFILL.D), PREFILL.seed + rank,
                                            syn.STREAM_Q + 10), dev)
    gdq, gdk, gdv = torch.empty_like(pq), torch.empty_like(pk), torch.empty_like(pv)
    bws = torch.empty((A.lib().fa_bwd_workspace_bytes(PREFILL.B, PREFILL.Hq, PREFILL.Lq),), dtype=torch.uint8,
                      device=dev)

    def backward():
        A.bwd(pq, pk, pv, po, plse, dout, causal=PREFILL.causal, scale=PREFILL.scale, dq=gdq, dk=gdk, dv=gdv,
              workspace=bws, stream=stream)
    ms = time_calls(backward, stream, reps=max(3, args.steps // 10))
    if A.device_status() != A.FA_OK:
        raise SystemExit("bench.py: a kernel reported a timed-out wait")
    tf = 2.5 * PREFILL.flops / (ms * 1e-3) / 1e12
    out["backward"] = {"bound": "tensor", "kernels": "fa_bwd_delta + fa_bwd_dq_kernel<128, causal> + "
                       "fa_bwd_dkdv_kernel<128, causal>", "workload": PREFILL.name, "achieved": tf,
                       "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                       "frac": tf / peaks["bf16_tflops"], "ms_per_call": ms,
                       "frac_of_sustained": tf / peaks["bf16_tflops_sustained"],
                       "flops_convention": "2.5 x forward (5 products), halved when causal",
                       "peak_source": f"{peak_src} bf16 burst"}
    del dout, gdq, gdk, gdv, bws
    torch.cuda.empty_cache()

    # backward at head_dim 256: the long-context GQA prefill (G = 4)
    lw = syn.LONG_GQA[4]
    lq, lk, lv = (A.to_device_bf16(x, dev) for x in lw.inputs(seed_offset=rank))
    lo, llse = A.fwd(lq, lk, lv, causal=lw.causal, scale=lw.scale, stream=stream)
    ldo = A.to_device_bf16(syn.normal_bf16((lw.B, lw.Lq, lw.Hq, lw.D), lw.seed + rank, syn.STREAM_Q + 10), dev)
    ldq, ldk, ldv = torch.empty_like(lq), torch.empty_like(lk), torch.empty_like(lv)
    lws = torch.empty((A.lib().fa_bwd_workspace_bytes(lw.B, lw.Hq, lw.Lq),), dtype=torch.uint8, device=dev)

    def backward_long():
        A.bwd(lq, lk, lv, lo, llse, ldo, causal=lw.causal, scale=lw.scale, dq=ldq, dk=ldk, dv=ldv,
              workspace=lws, stream=stream)
    ms = time_calls(backward_long, stream, reps=max(3, args.steps // 10))
    if A.device_status() != A.FA_OK:
        raise SystemExit("bench.py: a kernel reported a timed-out wait")
    tf = 2.5 * lw.flops / (ms * 1e-3) / 1e12
    out["backward_long_gqa"] = {"bound": "tensor", "kernels": "fa_bwd_delta + fa_bwd_dq_kernel<256, 64, causal> + "
                                "fa_bwd_dkdv_kernel<256, 64, dV pass> + fa_bwd_dkdv_kernel<256, 64, dK pass>",
                                "workload": lw.name, "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                "frac": tf / peaks["bf16_tflops"], "ms_per_call": ms,
                                "frac_of_sustained": tf / peaks["bf16_tflops_sustained"],
                                "flops_convention": "2.5 x forward (5 products), halved when causal",
                                "peak_source": f"{peak_src} bf16 burst"}
    del lq, lk, lv, lo, llse, ldo, ldq, ldk, ldv, lws
    torch.cuda.empty_cache()
    return out


def run_e2e(args, A, dev, stream, prefill_host, decode_host, flops, world):
    """Same step through the public API with pinned host buffers: copies in, compute, copies out.

    The decode cache is copied as each sequence's valid rows (one copy per
    sequence for K and for V: rows [0, len_b) of sequence b are contiguous);
    the rows past a sequence's length are never read by the kernel, so they
    are not an input of the step.
    """
    import torch
    q, k, v = prefill_host
    dq_h, dkc_h, dvc_h, lens_h = decode_host

    def pinned(a):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if a.dtype == np.uint16 else a)
        return t.pin_memory()

    hq, hk, hv = pinned(q), pinned(k), pinned(v)
    hdq, hdk, hdv, hlens = pinned(dq_h), pinned(dkc_h), pinned(dvc_h), pinned(lens_h)
    ho = torch.empty(hq.shape, dtype=torch.int16).pin_memory()
    hlse = torch.empty((PREFILL.B, PREFILL.Hq, PREFILL.Lq), dtype=torch.float32).pin_memory()
    hdo = torch.empty(hdq.shape, dtype=torch.int16).pin_memory()
    hdlse = torch.empty((DECODE.B, DECODE.Hq), dtype=torch.float32).pin_memory()
    lens_list = [int(x) for x in lens_h]
    row_bytes = DECODE.Hkv * DECODE.D * 2
    h2d = (sum(t.numel() * t.element_size() for t in (hq, hk, hv, hdq, hlens))
           + 2 * row_bytes * sum(lens_list))
    d2h = sum(t.numel() * t.element_size() for t in (ho, hlse, hdo, hdlse))
    ws = torch.empty((A.decode_workspace_bytes(DECODE.B, DECODE.Hq, DECODE.D, DECODE.num_splits),),
                     dtype=torch.uint8, device=dev)
    # device buffers the copies land in
    gq = torch.empty(hq.shape, dtype=torch.bfloat16, device=dev)
    gk = torch.empty(hk.shape, dtype=torch.bfloat16, device=dev)
    gv = torch.empty(hv.shape, dtype=torch.bfloat16, device=dev)
    gdq = torch.empty(hdq.shape, dtype=torch.bfloat16, device=dev)
    gdk = torch.empty(hdk.shape, dtype=torch.bfloat16, device=dev)
    gdv = torch.empty(hdv.shape, dtype=torch.bfloat16, device=dev)
    glens = torch.empty(hlens.shape, dtype=torch.int32, device=dev)

    def step():
        gq.view(torch.int16).copy_(hq, non_blocking=True)
        gk.view(torch.int16).copy_(hk, non_blocking=True)
        gv.view(torch.int16).copy_(hv, non_blocking=True)
        gdq.view(torch.int16).copy_(hdq, non_blocking=True)
        for b, n in enumerate(lens_list):
            gdk[b, :n].view(torch.int16).copy_(hdk[b, :n], non_blocking=True)
            gdv[b, :n].view(torch.int16).copy_(hdv[b, :n], non_blocking=True)
        glens.copy_(hlens, non_blocking=True)
        o, lse = A.fwd(gq, gk, gv, causal=PREFILL.causal, scale=PREFILL.scale, stream=stream)
        do, dlse = A.decode_splitkv(gdq, gdk, gdv, glens, DECODE.num_splits, scale=DECODE.scale,
                                    workspace=ws, stream=stream)
        ho.copy_(o.view(torch.int16), non_blocking=True)
        hlse.copy_(lse, non_blocking=True)
        hdo.copy_(do.view(torch.int16), non_blocking=True)
        hdlse.copy_(dlse, non_blocking=True)

    steps = max(1, min(args.steps, args.e2e_steps))
    for _ in range(max(1, min(args.warmup, 2))):
        step()
    torch.cuda.synchronize(dev)
    barrier()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        step()
    stop.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ms = max_over_ranks(start.elapsed_time(stop))
    return {"value": world * flops * steps / (ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "ms_per_step": ms / steps}


def run_profile_case(args):
    """A small case of one kernel for ncu: a few warm-up launches then one more.

    prefill:      the Llama-shaped prefill at batch 4 (537 MB of Q/K/V, over 4x L2);
    decode:       the decode workload at batch 16 (about 1.2 GB of valid K/V rows);
    decode_paged: the same in shuffled 64-key pages;
    decode_int8:  the same quantised to int8 K and V (codes and scales);
    varlen:       the first 8 sequences of the packed variable-length workload;
    prefill_fp8:  the Llama-shaped prefill at batch 4 quantised to e4m3;
    prefill_fp8_long: the long GQA prefill (head_dim 256, G = 4) quantised to e4m3;
    prefill_long: the long GQA prefill (head_dim 256, G = 4) in bf16;
    backward:     fa_bwd of the Llama-shaped prefill at batch 2;
    backward_long: fa_bwd of the long GQA prefill (head_dim 256, G = 4).
    """
    import torch
    from tiled_attention_23_b200 import attention as A
    torch.cuda.set_device(0)
    n = args.warmup + 1
    if args.profile == "prefill":
        w = PREFILL.with_(B=4)
        q, k, v = (A.to_device_bf16(x) for x in w.inputs())
        for _ in range(n):
            A.fwd(q, k, v, causal=w.causal, scale=w.scale)
    elif args.profile == "prefill_fp8":
        w = PREFILL.with_(B=4)
        q8, k8, v8 = (A.quantize_fp8(A.to_device_bf16(x)) for x in w.inputs())
        for _ in range(n):
            A.fwd_fp8(q8[0], k8[0], v8[0], q8[1], k8[1], v8[1], causal=w.causal, scale=w.scale)
    elif args.profile == "prefill_long":
        w = syn.LONG_GQA[4]
        q, k, v = (A.to_device_bf16(x) for x in w.inputs())
        for _ in range(n):
            A.fwd(q, k, v, causal=w.causal, scale=w.scale)
    elif args.profile == "prefill_fp8_long":
        w = syn.LONG_GQA[4]
        q8, k8, v8 = (A.quantize_fp8(A.to_device_bf16(x)) for x in w.inputs())
        for _ in range(n):
            A.fwd_fp8(q8[0], k8[0], v8[0], q8[1], k8[1], v8[1], causal=w.causal, scale=w.scale)
    elif args.profile == "backward":
        w = PREFILL.with_(B=2)
        q, k, v = (A.to_device_bf16(x) for x in w.inputs())
        do = A.to_device_bf16(syn.normal_bf16((w.B, w.Lq, w.Hq, w.D), 1, syn.STREAM_Q + 10))
        o, lse = A.fwd(q, k, v, causal=w.causal, scale=w.scale)
        for _ in range(n):
            A.bwd(q, k, v, o, lse, do, causal=w.causal, scale=w.scale)
    elif args.profile == "backward_long":
        w = syn.LONG_GQA[4]
        q, k, v = (A.to_device_bf16(x) for x in w.inputs())
        do = A.to_device_bf16(syn.normal_bf16((w.B, w.Lq, w.Hq, w.D), 1, syn.STREAM_Q + 10))
        o, lse = A.fwd(q, k, v, causal=w.causal, scale=w.scale)
        for _ in range(n):
            A.bwd(q, k, v, o, lse, do, causal=w.causal, scale=w.scale)
    elif args.profile == "varlen":
        w = syn.VARLEN_PREFILL.with_(B=8)
        q, k, v, cu = w.inputs()
        q, k, v = (A.to_device_bf16(x) for x in (q, k, v))
        gcu = torch.from_numpy(cu).cuda()
        for _ in range(n):
            A.fwd_varlen(q, k, v, gcu, gcu, int(np.diff(cu).max()), causal=w.causal, scale=w.scale)
    else:
        d = DECODE.with_(B=16)
        q, kc, vc, lens = d.inputs()
        glens = torch.from_numpy(lens).cuda()
        gq = A.to_device_bf16(q)
        if args.profile == "decode":
            gk, gv = A.to_device_bf16(kc), A.to_device_bf16(vc)
            for _ in range(n):
                A.decode_splitkv(gq, gk, gv, glens, d.num_splits, scale=d.scale)
        elif args.profile == "decode_paged":
            kp, vp, table = syn.paginate(kc, vc, lens, syn.DECODE_PAGE_SIZE, seed=7, spare_pages=16)
            gk, gv = A.to_device_bf16(kp), A.to_device_bf16(vp)
            gt = torch.from_numpy(table).cuda()
            for _ in range(n):
                A.decode_paged(gq, gk, gv, gt, glens, d.num_splits, scale=d.scale)
        else:   # decode_int8
            kq, ks = A.quantize_kv_int8(A.to_device_bf16(kc))
            vq, vs = A.quantize_kv_int8(A.to_device_bf16(vc))
            for _ in range(n):
                A.decode_int8(gq, kq, ks, vq, vs, glens, d.num_splits, scale=d.scale)
    torch.cuda.synchronize()
    if A.device_status() != A.FA_OK:
        raise SystemExit("profile case: a kernel reported a timed-out wait")
    print(f"profile case {args.profile} done")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the next-row kernels (paged decode, ...)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--ref-step-seconds", type=float, default=4.0)
    ap.add_argument("--profile", choices=["prefill", "decode", "decode_paged", "decode_int8", "varlen", "prefill_fp8",
                                          "prefill_fp8_long", "prefill_long", "backward", "backward_long"],
                    default=None,
                    help="run a small single-kernel case for ncu instead of the benchmark")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be at least 3")
    if a.steps < 1:
        ap.error("--steps must be positive")
    return a


def main(argv=None):
    args = parse_args(argv)
    if args.profile:
        run_profile_case(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    if world > 1 and args.impl == "ours":
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            if dist.is_initialized():
                dist.destroy_process_group()


if __name__ == "__main__":
    main()
