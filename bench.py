#!/usr/bin/env python
"""Benchmark of the exact-attention hot path on B200; prints one JSON line on rank 0.

A step is one pass over both entry points of the hot path:
  * prefill: attn_fwd on the long non-causal workload B=2, H=16, N=8192, d=128 (bf16, scale
             1/sqrt(d)), the configuration the >=60 % tensor-core gate is stated on;
  * decode:  attn_decode_splitkv (split kernel + combine) on B=8, Hq=32, Hkv=8, d=128 with KV
             lengths drawn uniformly from [1024, 131072].
`value` is the prefill throughput in TFLOP/s (4*B*H*N^2*d); the decode half of the metric is
reported under "decode" in GB/s of algorithmic HBM bytes. Both are timed with CUDA events on the
launching stream; the step's inputs (0.2 GB prefill + 4.3 GB decode) exceed the 126 MB L2, and the
decode pass evicts the prefill inputs before the next step. "gates" times the other prefill
workloads (causal N=2048, causal and GQA N=8192, the head-dim sweep) one launch at a time with a
256 MiB L2 flush before each.

`--impl reference` times the CPU oracle instead, on a bounded sample of the same workloads.
Multi-GPU (torchrun): every rank runs the same step on its own GPU (independent problems, no
collective on the data path); `value` counts the work of all ranks over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "attn fwd TFLOP/s & % of BF16 peak (prefill); decode HBM GB/s & % of peak"
NOMINAL_BF16_TFLOPS = 2250.0
NOMINAL_HBM_GBS = 8000.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
LONG_REGION_MS = 1000.0  # a timed region at least this long is measured against the sustained peak


# DRAM traffic per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum; summaries and commands
# in profiles/), per workload, keyed to the sha256 of the kernel source it was measured on: once
# that file changes, the figure is stale and the bench line reports null until it is measured again.
PREFILL_SRC = "exact_io_aware_41_b200/csrc/attn_fwd.cu"
DECODE_SRC = "exact_io_aware_41_b200/csrc/attn_decode.cu"
PREFILL_SHA = "63b6180f1f6afe9c54d540d7fed48ed998708272751ad149f087cb68eb2d9625"  # sha256 of PREFILL_SRC when the prefill figures were taken
BACKWARD_SRC = "exact_io_aware_41_b200/csrc/attn_bwd.cu"
BACKWARD_SHA = "7491f9ddae8c644559ef9b6c2c8b785dd6d0e2b6edefb74273e7b734d4d89e0d"
NCU_TRAFFIC = {
    # attn_fwd_kernel<128>: 350.77 MB read + 52.83 MB written
    synth.LONG_8K.name: (PREFILL_SRC, PREFILL_SHA, 403_600_640.0),
    # attn_fwd_kernel<128>: 128.36 MB read + 13.21 MB written
    synth.CAUSAL_2K.name: (PREFILL_SRC, PREFILL_SHA, 141_571_328.0),
    # attn_fwd_kernel<128>: 213.84 MB read + 50.57 MB written
    synth.LONG_8K_CAUSAL.name: (PREFILL_SRC, PREFILL_SHA, 264_412_160.0),
    # attn_fwd_kernel<128>: 369.63 MB read + 106.79 MB written
    synth.LONG_8K_GQA.name: (PREFILL_SRC, PREFILL_SHA, 476_417_024.0),
    # attn_fwd_kernel<128>: 373.41 MB read + 101.96 MB written
    synth.LONG_8K_GQA_CAUSAL.name: (PREFILL_SRC, PREFILL_SHA, 475_375_616.0),
    # attn_fwd_kernel<32>: 50.40 MB read + 1.50 MB written
    synth.SWEEP[0].name: (PREFILL_SRC, PREFILL_SHA, 51_898_624.0),
    # attn_fwd_kernel<64>: 114.14 MB read + 22.27 MB written
    synth.SWEEP[1].name: (PREFILL_SRC, PREFILL_SHA, 136_412_928.0),
    # attn_fwd_kernel<128>: 345.82 MB read + 53.71 MB written
    synth.SWEEP[2].name: (PREFILL_SRC, PREFILL_SHA, 399_529_984.0),
    # attn_fwd_kernel<256> on CTA pairs: 743.03 MB read + 118.83 MB written
    synth.SWEEP[3].name: (PREFILL_SRC, PREFILL_SHA, 861_856_512.0),
    # attn_fwd_kernel<128, 8-bit> on the long non-causal workload: 138.46 MB read + 42.28 MB written
    "fp8 " + synth.LONG_8K.name: (PREFILL_SRC, PREFILL_SHA, 180_734_720.0),
    # attn_bwd_kernel on the causal N2048 workload: 425.18 MB read + 215.12 MB written
    "backward " + synth.CAUSAL_2K.name: (BACKWARD_SRC, BACKWARD_SHA, 657_230_848.0),
    # decode_split_tc_kernel<128,4> (2123.81 MB read + 7.59 MB written) + decode_combine_kernel<128>
    # (4.29 MB read) on the full decode workload
    synth.DECODE.name: (DECODE_SRC, "eaf4990882bbcba5d723de8f5b505ab0c1520f88553cb35fa7ee6758aa501c3a", 2_135_693_824.0),
}


def ncu_traffic(name: str):
    import hashlib

    if name not in NCU_TRAFFIC:
        return None
    path, digest, nbytes = NCU_TRAFFIC[name]
    try:
        with open(os.path.join(ROOT, path), "rb") as f:
            return nbytes if hashlib.sha256(f.read()).hexdigest() == digest else None
    except OSError:
        return None


def step_tensor_peak(peaks: dict, timed_ms: float):
    """The bf16 tensor peak for a kernel timed inside the step loop: over a timed region of a second
    or more the GPU settles at its power-capped clock, so the sustained GEMM figure; over a short one
    (a few tens of steps) the burst figure. Returns (peak, long_region)."""
    long_region = timed_ms >= LONG_REGION_MS
    key = "bf16_tflops_sustained" if long_region else "bf16_tflops"
    return peaks.get(key, FALLBACK[key]), long_region


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK), "fallback"


# ------------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], 0.0, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = max(smax, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": smax, "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# distributed plumbing
# ------------------------------------------------------------------------------------------------
def dist_setup(n_gpus: int):
    """Rank, world and the process group from the torchrun environment (NCCL on GPUs, gloo on CPUs).

    The group carries only the barrier around the timed region and the max-over-ranks reduction of
    the timings: every rank runs an independent problem, nothing on the data path is exchanged.
    """
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return world, rank, local, pg


def max_over_ranks(values, dist, device=None):
    """Element-wise maximum of a list of floats over all ranks (the slowest rank's times)."""
    if dist is None:
        return list(values)
    import torch

    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def physical_gpu(local: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x for x in vis.split(",") if x.strip()]
        if local < len(ids) and ids[local].strip().isdigit():
            return int(ids[local])
    return local


# ------------------------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ------------------------------------------------------------------------------------------------
def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def _head_inputs(w: synth.Prefill, b: int, h: int):
    g = h // (w.Hq // w.Hkv)
    dq = np.arange(w.d, dtype=np.int64)
    tq = np.arange(w.Nq, dtype=np.int64)[:, None]
    tk = np.arange(w.Nkv, dtype=np.int64)[:, None]
    q = synth.normal_bf16_at(w.seed, synth.STREAM_Q, (((b * w.Nq + tq) * w.Hq + h) * w.d + dq).reshape(-1))
    kidx = (((b * w.Nkv + tk) * w.Hkv + g) * w.d + dq).reshape(-1)
    k = synth.normal_bf16_at(w.seed, synth.STREAM_K, kidx)
    v = synth.normal_bf16_at(w.seed, synth.STREAM_V, kidx)
    f = synth.bf16_bits_to_f64
    return (f(q).reshape(1, w.Nq, 1, w.d), f(k).reshape(1, w.Nkv, 1, w.d), f(v).reshape(1, w.Nkv, 1, w.d))


def cpu_prefill(w: synth.Prefill, budget_s: float):
    import oracle

    heads, flops, spent = 0, 0.0, 0.0
    per_head = w.flops / (w.B * w.Hq)
    while spent < budget_s and heads < w.B * w.Hq:
        b, h = divmod(heads, w.Hq)
        q, k, v = _head_inputs(w, b, h)
        t0 = time.perf_counter()
        oracle.attention(q, k, v, w.scale, w.causal)
        spent += time.perf_counter() - t0
        flops += per_head
        heads += 1
    return flops / spent / 1e12, f"{heads} of {w.B * w.Hq} (b, h) heads of {w.name}, {spent:.1f} s", spent


def cpu_decode(w: synth.Decode, budget_s: float, tokens: int = 2048):
    """Oracle decode on all B sequences and all query heads, each sequence truncated to its first
    `tokens` KV tokens (host draws of the same seeded cache), repeated until the budget is spent."""
    import oracle

    lens = np.minimum(w.lengths(), tokens)
    cap = int(lens.max())
    shape = (w.B, cap, w.Hkv, w.d)
    q = synth.bf16_bits_to_f64(synth.normal_bf16(w.seed, synth.STREAM_Q, (w.B, w.Hq, w.d)))
    # the first `cap` tokens of the full cache [B, Nkv_cap, Hkv, d]: draw those rows of each sequence
    row = np.arange(cap * w.Hkv * w.d, dtype=np.int64)
    flat = (np.arange(w.B, dtype=np.int64)[:, None] * (w.cap * w.Hkv * w.d) + row[None, :]).reshape(-1)
    k = synth.bf16_bits_to_f64(synth.normal_bf16_at(w.seed, synth.STREAM_K, flat)).reshape(shape)
    v = synth.bf16_bits_to_f64(synth.normal_bf16_at(w.seed, synth.STREAM_V, flat)).reshape(shape)
    per_rep = int(lens.astype(np.int64).sum()) * w.Hkv * w.d * 2 * 2
    byts, spent, reps = 0.0, 0.0, 0
    while spent < budget_s:
        t0 = time.perf_counter()
        oracle.decode(q, k, v, lens, w.scale)
        spent += time.perf_counter() - t0
        byts += per_rep
        reps += 1
    return byts / spent / 1e9, (f"{reps} x (all {w.B} sequences truncated to their first {tokens} KV tokens, "
                                f"all {w.Hq} query heads) of {w.name}"), spent


# ------------------------------------------------------------------------------------------------
# GPU arm
# ------------------------------------------------------------------------------------------------
def run_ours(args, world, rank, local, dist):
    import torch

    import exact_io_aware_41_b200 as lib

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    peaks, peak_src = _peaks()

    P = synth.LONG_8K
    Dw = synth.DECODE
    q = synth.normal_bf16_torch(P.seed, synth.STREAM_Q, (P.B, P.Nq, P.Hq, P.d), dev)
    k = synth.normal_bf16_torch(P.seed, synth.STREAM_K, (P.B, P.Nkv, P.Hkv, P.d), dev)
    v = synth.normal_bf16_torch(P.seed, synth.STREAM_V, (P.B, P.Nkv, P.Hkv, P.d), dev)
    o = torch.empty_like(q)
    lse = torch.empty((P.B, P.Hq, P.Nq), dtype=torch.float32, device=dev)

    cap = Dw.cap
    lens_np = Dw.lengths()
    dq = synth.normal_bf16_torch(Dw.seed, synth.STREAM_Q, (Dw.B, Dw.Hq, Dw.d), dev)
    kc = synth.normal_bf16_torch(Dw.seed, synth.STREAM_K, (Dw.B, cap, Dw.Hkv, Dw.d), dev)
    vc = synth.normal_bf16_torch(Dw.seed, synth.STREAM_V, (Dw.B, cap, Dw.Hkv, Dw.d), dev)
    lens = torch.from_numpy(lens_np).to(dev)
    do = torch.empty_like(dq)
    dlse = torch.empty((Dw.B, Dw.Hq), dtype=torch.float32, device=dev)
    ws = torch.empty(lib.attn_decode_workspace_bytes(Dw.B, Dw.Hq, Dw.Hkv, Dw.d, cap, 0), dtype=torch.uint8,
                     device=dev)
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    K, W = args.steps, args.warmup
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]

    def step(e=None):
        if e is not None:
            e[0].record(stream)
        lib.attn_fwd(q, k, v, scale=P.scale, causal=P.causal, out=o, lse=lse)
        if e is not None:
            e[1].record(stream)
        lib.attn_decode_splitkv(dq, kc, vc, lens, scale=Dw.scale, workspace=ws, out=do, lse=dlse)
        if e is not None:
            e[2].record(stream)

    for _ in range(W):
        step()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    sampler = ClockSampler(physical_gpu(local))
    sampler.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(K):
        step(ev[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    total_ms = t_start.elapsed_time(t_end)
    pf_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    dec_ms = sum(e[1].elapsed_time(e[2]) for e in ev)
    total_ms, pf_ms, dec_ms = max_over_ranks([total_ms, pf_ms, dec_ms], dist, dev)
    err = lib.attn_get_last_error()
    if err != lib.ATTN_OK:
        raise SystemExit(f"device error word after the timed region: {lib.status_string(err)}")

    pf_flops = P.flops
    dec_bytes = Dw.algorithmic_bytes()
    value = world * K * pf_flops / (pf_ms * 1e-3) / 1e12
    pf_avg_s = pf_ms * 1e-3 / K
    dec_avg_s = dec_ms * 1e-3 / K
    pf_tflops_1 = pf_flops / pf_avg_s / 1e12
    dec_gbs_1 = dec_bytes / dec_avg_s / 1e9
    dec_value = world * K * dec_bytes / (dec_ms * 1e-3) / 1e9

    # ---- gates: the other prefill workloads, one launch at a time after an L2 flush (not in `value`)
    gates = {}
    if not args.no_gates:
        for w in GATES:
            gates[w.name] = time_prefill(lib, w, dev, stream, peaks)
            torch.cuda.empty_cache()
        gates["fp8 " + P.name] = time_prefill_fp8(lib, P, dev, stream, peaks)
        torch.cuda.empty_cache()
        gates["backward " + synth.CAUSAL_2K.name] = time_backward(lib, synth.CAUSAL_2K, dev, stream, peaks)
        torch.cuda.empty_cache()

    # ---- end to end through the public API with pinned host buffers
    e2e = e2e_prefill(lib, P, q, k, v, stream, max(3, min(K, 50)))
    dec_e2e = e2e_decode(lib, Dw, dq, kc, vc, lens_np, stream, 2) if not args.no_e2e_decode else None
    e2e["ms"], dms = max_over_ranks([e2e["ms"], (dec_e2e or {}).get("ms", 0.0)], dist, dev)
    if dec_e2e:
        dec_e2e["ms"] = dms

    if rank != 0:
        return None

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        v_cpu, sample, _ = cpu_prefill(P, args.cpu_budget)
        cpu = {"value": v_cpu, "unit": "TFLOP/s", "cores": _blas_threads(), "kind": "oracle", "sample": sample}
        dv, dsample, _ = cpu_decode(Dw, args.cpu_budget / 2)
        cpu["decode"] = {"value": dv, "unit": "GB/s", "sample": dsample}

    meas_tf, long_region = step_tensor_peak(peaks, total_ms)
    meas_bw = peaks.get("hbm_gbs", FALLBACK["hbm_gbs"])
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": total_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: seeded i.i.d. N(0,1) rounded to bf16 (splitmix64 + Box-Muller), decode lengths U[1024,131072]",
        "config": {
            "workload": P.name,
            "decode_workload": Dw.name,
            "decode_kv_tokens": int(lens_np.sum()),
            "parallelism": f"replica x{world} (independent problems, no collective)",
            "l2": "inputs larger than L2: the step reads 4.5 GB (prefill 0.2 GB); the decode pass evicts the "
                  "prefill inputs; gates flush L2 (256 MiB write) before every launch",
        },
        "frac_of_nominal_bf16": pf_tflops_1 / NOMINAL_BF16_TFLOPS,
        "roofline": {"bound": "tensor", "kernel": "attn::attn_fwd_kernel<128, false, false>",
                     "achieved": pf_tflops_1, "peak": meas_tf, "unit": "TFLOP/s", "frac": pf_tflops_1 / meas_tf,
                     "peak_source": f"{peak_src} bf16 {'sustained' if long_region else 'burst'} (cuBLAS; timed "
                                    f"region {total_ms / 1e3:.2f} s)",
                     "traffic": ncu_traffic(P.name), "traffic_source": "ncu dram__bytes_read.sum + "
                     "dram__bytes_write.sum of one launch on this workload (null: not measured on this source)"},
        "decode": {
            "value": dec_value, "unit": "GB/s", "ms_per_call": dec_avg_s * 1e3,
            "algorithmic_bytes_per_call": dec_bytes,
            "frac_of_nominal_hbm": dec_gbs_1 / NOMINAL_HBM_GBS,
            "roofline": {"bound": "hbm", "kernel": "decode_split_tc_kernel<128,4> + decode_combine_kernel<128>",
                         "achieved": dec_gbs_1, "peak": meas_bw, "unit": "GB/s", "frac": dec_gbs_1 / meas_bw,
                         "peak_source": f"{peak_src} copy bandwidth",
                         "traffic": ncu_traffic(Dw.name)},
            "e2e": dec_e2e and {
                "value": world * dec_bytes / (dec_e2e["ms"] * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": dec_e2e["h2d"], "d2h_bytes_per_step": dec_e2e["d2h"]},
        },
        "e2e": {"value": world * pf_flops / (e2e["ms"] * 1e-3) / 1e12, "unit": "TFLOP/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]},
        "gates": gates,
        "gpu_launches": 3 * K,  # per step: the prefill kernel, the decode split kernel, the combine kernel
        "kernels": {"prefill": lib.kernel_name(0), "decode": [lib.kernel_name(1), lib.kernel_name(2)]},
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    return line


GATES = (synth.CAUSAL_2K, synth.LONG_8K_CAUSAL, synth.LONG_8K_GQA, synth.LONG_8K_GQA_CAUSAL, *synth.SWEEP)


def prefill_bytes(w) -> int:
    """Algorithmic HBM bytes of one prefill launch: Q, K, V read once, O and LSE written once."""
    return (2 * w.B * w.Nq * w.Hq * w.d + 2 * 2 * w.B * w.Nkv * w.Hkv * w.d + 2 * w.B * w.Nq * w.Hq * w.d
            + 4 * w.B * w.Hq * w.Nq)


def time_prefill(lib, w, dev, stream, peaks, reps=20, warm=5):
    import torch

    q = synth.normal_bf16_torch(w.seed, synth.STREAM_Q, (w.B, w.Nq, w.Hq, w.d), dev)
    k = synth.normal_bf16_torch(w.seed, synth.STREAM_K, (w.B, w.Nkv, w.Hkv, w.d), dev)
    v = synth.normal_bf16_torch(w.seed, synth.STREAM_V, (w.B, w.Nkv, w.Hkv, w.d), dev)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(warm):
        lib.attn_fwd(q, k, v, scale=w.scale, causal=w.causal, out=o, lse=lse)
    ms = []
    for _ in range(reps):
        flush.fill_(1)  # 256 MiB write: L2 holds none of the inputs when the kernel starts
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        lib.attn_fwd(q, k, v, scale=w.scale, causal=w.causal, out=o, lse=lse)
        b.record(stream)
        b.synchronize()
        ms.append(a.elapsed_time(b))
    med = float(np.median(ms))
    tf = w.flops / (med * 1e-3) / 1e12
    pk = peaks.get("bf16_tflops", FALLBACK["bf16_tflops"])
    return {"ms": med, "tflops": tf, "frac_of_measured": tf / pk, "frac_of_nominal": tf / NOMINAL_BF16_TFLOPS,
            "roofline": {"bound": "tensor", "kernel": f"attn::attn_fwd_kernel<{w.d}, false, {'true' if w.d == 256 else 'false'}>", "achieved": tf, "peak": pk,
                         "unit": "TFLOP/s", "frac": tf / pk, "traffic": ncu_traffic(w.name),
                         "algorithmic_bytes": prefill_bytes(w)}}


FP8_SIGNS_SEED = 4242


def fp8_signs(d: int, device):
    """The rotation's sign vector: +-1 from a seeded generator (an input of the method)."""
    import torch

    u = np.random.default_rng(FP8_SIGNS_SEED).random(d)
    return torch.from_numpy(np.where(u < 0.5, -1.0, 1.0).astype(np.float32)).to(device)


def time_prefill_fp8(lib, w, dev, stream, peaks, reps=20, warm=5):
    """attn_fwd_fp8 on the workload's inputs quantized once (rotation + e4m3, not timed), one launch
    at a time after an L2 flush; TFLOP/s against the fp8 dense peak (2x the measured bf16 peak, the
    nominal fp8 / bf16 ratio)."""
    import torch

    q = synth.normal_bf16_torch(w.seed, synth.STREAM_Q, (w.B, w.Nq, w.Hq, w.d), dev)
    k = synth.normal_bf16_torch(w.seed, synth.STREAM_K, (w.B, w.Nkv, w.Hkv, w.d), dev)
    v = synth.normal_bf16_torch(w.seed, synth.STREAM_V, (w.B, w.Nkv, w.Hkv, w.d), dev)
    sg = fp8_signs(w.d, dev)
    q8, aq = lib.attn_fp8_quantize(q, sg)
    k8, ak = lib.attn_fp8_quantize(k, sg)
    vt8, av = lib.attn_fp8_quantize(v, None, transpose=True)
    del q, k, v
    o = torch.empty((w.B, w.Nq, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def call():
        lib.attn_fwd_fp8(q8, k8, vt8, aq, ak, av, scale=w.scale, causal=w.causal, out=o, lse=lse)
    for _ in range(warm):
        call()
    ms = []
    for _ in range(reps):
        flush.fill_(1)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call()
        b.record(stream)
        b.synchronize()
        ms.append(a.elapsed_time(b))
    med = float(np.median(ms))
    tf = w.flops / (med * 1e-3) / 1e12
    pk = 2.0 * peaks.get("bf16_tflops", FALLBACK["bf16_tflops"])
    return {"ms": med, "tflops": tf, "dtype": "e4m3 operands, fp32 accumulate",
            "roofline": {"bound": "tensor", "kernel": "attn::attn_fwd_kernel<128, true, false>", "achieved": tf, "peak": pk,
                         "unit": "TFLOP/s", "frac": tf / pk, "peak_source": "2 x bf16 peak (nominal fp8/bf16 ratio)",
                         "traffic": ncu_traffic("fp8 " + w.name)}}


def time_backward(lib, w, dev, stream, peaks, reps=20, warm=5):
    """attn_bwd (pre-pass, main kernel, dQ conversion) after an L2 flush, on the forward's O and LSE.
    FLOPs = 2.5 x the forward's (five products of the forward's size against two)."""
    import torch

    q = synth.normal_bf16_torch(w.seed, synth.STREAM_Q, (w.B, w.Nq, w.Hq, w.d), dev)
    k = synth.normal_bf16_torch(w.seed, synth.STREAM_K, (w.B, w.Nkv, w.Hkv, w.d), dev)
    v = synth.normal_bf16_torch(w.seed, synth.STREAM_V, (w.B, w.Nkv, w.Hkv, w.d), dev)
    do = synth.normal_bf16_torch(w.seed, 5, (w.B, w.Nq, w.Hq, w.d), dev)
    o, lse = lib.attn_fwd(q, k, v, scale=w.scale, causal=w.causal)
    ws = torch.empty(lib.attn_bwd_workspace_bytes(w.B, w.Hq, w.Nq, w.d), dtype=torch.uint8, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def call():
        lib.attn_bwd(q, k, v, o, lse, do, scale=w.scale, causal=w.causal, workspace=ws, dq=dq, dk=dk, dv=dv)
    for _ in range(warm):
        call()
    ms = []
    for _ in range(reps):
        flush.fill_(1)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        call()
        b.record(stream)
        b.synchronize()
        ms.append(a.elapsed_time(b))
    med = float(np.median(ms))
    tf = 2.5 * w.flops / (med * 1e-3) / 1e12
    pk = peaks.get("bf16_tflops", FALLBACK["bf16_tflops"])
    return {"ms": med, "tflops": tf, "flops": 2.5 * w.flops,
            "roofline": {"bound": "tensor", "kernel": "attn::attn_bwd_kernel (+ pre and post passes)", "achieved": tf,
                         "peak": pk, "unit": "TFLOP/s", "frac": tf / pk, "traffic": ncu_traffic("backward " + w.name)}}


def e2e_prefill(lib, P, q, k, v, stream, n):
    """Per step: host (pinned) -> device copies of that step's Q, K, V, attn_fwd, and device -> host
    copies of its O and LSE. Steps are pipelined the way a serving loop would run them: three
    streams (copy in, compute, copy out) and two buffer sets, so step i+1's inputs cross PCIe while
    step i computes and step i-1's result comes back (the link is full duplex)."""
    import torch

    hq = q.cpu().pin_memory()
    hk = k.cpu().pin_memory()
    hv = v.cpu().pin_memory()
    dev_in = [tuple(torch.empty_like(t) for t in (q, k, v)) for _ in range(2)]
    dev_out = [(torch.empty_like(q), torch.empty((P.B, P.Hq, P.Nq), dtype=torch.float32, device=q.device))
               for _ in range(2)]
    ho = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(2)]
    hl = [torch.empty((P.B, P.Hq, P.Nq), dtype=torch.float32).pin_memory() for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    s_cmp = stream
    # per buffer set: inputs landed, inputs consumed, outputs written, outputs read back
    ev = [{name: torch.cuda.Event() for name in ("in_done", "in_free", "out_done", "out_free")} for _ in range(2)]
    used = [False, False]

    def one(i):
        b = i & 1
        e = ev[b]
        dq, dk, dv = dev_in[b]
        o, lse = dev_out[b]
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(e["in_free"])
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            e["in_done"].record(s_in)
        s_cmp.wait_event(e["in_done"])
        if used[b]:
            s_cmp.wait_event(e["out_free"])
        lib.attn_fwd(dq, dk, dv, scale=P.scale, causal=P.causal, out=o, lse=lse, stream=s_cmp)
        e["in_free"].record(s_cmp)
        e["out_done"].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(e["out_done"])
            ho[b].copy_(o, non_blocking=True)
            hl[b].copy_(lse, non_blocking=True)
            e["out_free"].record(s_out)
        used[b] = True

    for i in range(2):
        one(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_in)  # every timed copy and launch is ordered after it through the events above
    s_cmp.wait_event(start)
    s_out.wait_event(start)
    for i in range(n):
        one(i)
    end_cmp = torch.cuda.Event()
    end_cmp.record(s_cmp)
    s_out.wait_event(end_cmp)
    with torch.cuda.stream(s_out):
        s_out.wait_stream(s_in)
        end.record(s_out)
    end.synchronize()
    h2d = 3 * q.numel() * 2
    d2h = q.numel() * 2 + P.B * P.Hq * P.Nq * 4
    return {"ms": start.elapsed_time(end) / n, "h2d": h2d, "d2h": d2h}


def e2e_decode(lib, Dw, dq, kc, vc, lens_np, stream, n):
    """The decode call with its whole KV cache copied from pinned host memory every step."""
    import torch

    try:
        hq = dq.cpu().pin_memory()
        hk = kc.cpu().pin_memory()
        hv = vc.cpu().pin_memory()
    except RuntimeError:
        return None
    hl = torch.from_numpy(lens_np).pin_memory()
    d_q, d_k, d_v = torch.empty_like(dq), torch.empty_like(kc), torch.empty_like(vc)
    d_l = torch.empty(len(lens_np), dtype=torch.int32, device=dq.device)
    ho = torch.empty(dq.shape, dtype=dq.dtype).pin_memory()
    hls = torch.empty((Dw.B, Dw.Hq), dtype=torch.float32).pin_memory()

    def one():
        d_q.copy_(hq, non_blocking=True)
        d_k.copy_(hk, non_blocking=True)
        d_v.copy_(hv, non_blocking=True)
        d_l.copy_(hl, non_blocking=True)
        o, lse = lib.attn_decode_splitkv(d_q, d_k, d_v, d_l, scale=Dw.scale)
        ho.copy_(o, non_blocking=True)
        hls.copy_(lse, non_blocking=True)

    one()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        one()
    b.record(stream)
    b.synchronize()
    h2d = (dq.numel() + kc.numel() + vc.numel()) * 2 + len(lens_np) * 4
    d2h = dq.numel() * 2 + Dw.B * Dw.Hq * 4
    out = {"ms": a.elapsed_time(b) / n, "h2d": h2d, "d2h": d2h}
    del hk, hv, d_k, d_v
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------------------------------------
# reference arm: the CPU oracle, timed as it stands
# ------------------------------------------------------------------------------------------------
_HEAD_CACHE = {}


def _rows_inputs(w: synth.Prefill, b: int, h: int, i0: int, m: int):
    """Query rows [i0, i0+m) of head (b, h) and the keys they can see (all keys when not causal)."""
    if (b, h) not in _HEAD_CACHE:
        _HEAD_CACHE[(b, h)] = _head_inputs(w, b, h)
    q, k, v = _HEAD_CACHE[(b, h)]
    nk = min(w.Nkv, i0 + m + (w.Nkv - w.Nq)) if w.causal else w.Nkv
    # with Nq = m and Nkv = nk, the bottom-right causal mask gives row r the keys j <= r + i0 + (Nkv - Nq)
    flops = 4.0 * w.d * (sum(min(nk, i + 1 + (w.Nkv - w.Nq)) for i in range(i0, i0 + m)) if w.causal else m * nk)
    return q[:, i0:i0 + m], k[:, :nk], v[:, :nk], flops


def run_reference(args, world, rank):
    """The CPU oracle as it stands, on bounded samples of the GPU arm's workloads, rank 0 only."""
    import oracle

    if rank != 0:
        return None
    P, Dw = synth.LONG_8K, synth.DECODE
    m = 64
    blocks = [(b, h, i0) for (b, h) in ((0, 0), (1, 5), (0, 10), (1, 15)) for i0 in range(0, P.Nq, m)]
    per_step = min(1.0, 100.0 / max(1, args.steps))  # keeps K steps within a couple of minutes
    cursor = 0

    def one_step():
        nonlocal cursor
        fl, sp, n = 0.0, 0.0, 0
        while n == 0 or sp < per_step:
            b, h, i0 = blocks[(cursor * 7919) % len(blocks)]
            cursor += 1
            q, k, v, f = _rows_inputs(P, b, h, i0, m)
            t0 = time.perf_counter()
            oracle.attention(q, k, v, P.scale, P.causal)
            sp += time.perf_counter() - t0
            fl += f
            n += 1
        return fl, sp, n

    for _ in range(args.warmup):
        one_step()
    flops, spent, nblk = 0.0, 0.0, 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        f, sp, n = one_step()
        flops += f
        spent += sp
        nblk += n
    wall = time.perf_counter() - t0
    value = flops / spent / 1e12
    dv, dsample, _ = cpu_decode(Dw, min(8.0, max(2.0, args.cpu_budget / 2)))
    cores = _blas_threads()
    sample = (f"{nblk} blocks of {m} query rows (with the keys they see) of {P.name}, "
              f"{spent:.1f} s of oracle time over {args.steps} steps")
    return {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": wall * 1e3 / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: seeded i.i.d. N(0,1) rounded to bf16",
        "config": {"workload": P.name, "decode_workload": Dw.name,
                   "parallelism": "CPU oracle on rank 0 only", "l2": "n/a (CPU)"},
        "decode": {"value": dv, "unit": "GB/s", "sample": dsample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
        "gpu_launches": 0,
    }


def run_only(args):
    """One kernel on one workload, K timed launches (for profiling runs and per-workload numbers)."""
    import torch

    import exact_io_aware_41_b200 as lib

    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    peaks, src = _peaks()
    if args.only == "backward":
        w = synth.CAUSAL_2K
        q = synth.normal_bf16_torch(w.seed, synth.STREAM_Q, (w.B, w.Nq, w.Hq, w.d), dev)
        k = synth.normal_bf16_torch(w.seed, synth.STREAM_K, (w.B, w.Nkv, w.Hkv, w.d), dev)
        v = synth.normal_bf16_torch(w.seed, synth.STREAM_V, (w.B, w.Nkv, w.Hkv, w.d), dev)
        do = synth.normal_bf16_torch(w.seed, 5, (w.B, w.Nq, w.Hq, w.d), dev)
        o, lse = lib.attn_fwd(q, k, v, scale=w.scale, causal=w.causal)
        ws = torch.empty(lib.attn_bwd_workspace_bytes(w.B, w.Hq, w.Nq, w.d), dtype=torch.uint8, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)

        def call():
            lib.attn_bwd(q, k, v, o, lse, do, scale=w.scale, causal=w.causal, workspace=ws, dq=dq, dk=dk, dv=dv)
        work, unit, name = 2.5 * w.flops / 1e12, "TFLOP/s", "backward " + w.name
    elif args.only == "prefill_fp8":
        w = synth.LONG_8K
        q = synth.normal_bf16_torch(w.seed, synth.STREAM_Q, (w.B, w.Nq, w.Hq, w.d), dev)
        k = synth.normal_bf16_torch(w.seed, synth.STREAM_K, (w.B, w.Nkv, w.Hkv, w.d), dev)
        v = synth.normal_bf16_torch(w.seed, synth.STREAM_V, (w.B, w.Nkv, w.Hkv, w.d), dev)
        sg = fp8_signs(w.d, dev)
        q8, aq = lib.attn_fp8_quantize(q, sg)
        k8, ak = lib.attn_fp8_quantize(k, sg)
        vt8, av = lib.attn_fp8_quantize(v, None, transpose=True)
        del q, k, v
        o = torch.empty((w.B, w.Nq, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)

        def call():
            lib.attn_fwd_fp8(q8, k8, vt8, aq, ak, av, scale=w.scale, causal=w.causal, out=o, lse=lse)
        work, unit, name = w.flops / 1e12, "TFLOP/s", "fp8 " + w.name
    elif args.only == "prefill":
        table = {w.name: w for w in synth.PREFILL_WORKLOADS}
        w = table[args.workload] if args.workload else synth.LONG_8K
        q = synth.normal_bf16_torch(w.seed, synth.STREAM_Q, (w.B, w.Nq, w.Hq, w.d), dev)
        k = synth.normal_bf16_torch(w.seed, synth.STREAM_K, (w.B, w.Nkv, w.Hkv, w.d), dev)
        v = synth.normal_bf16_torch(w.seed, synth.STREAM_V, (w.B, w.Nkv, w.Hkv, w.d), dev)
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)

        def call():
            lib.attn_fwd(q, k, v, scale=w.scale, causal=w.causal, out=o, lse=lse)
        work, unit, name = w.flops / 1e12, "TFLOP/s", w.name
    else:
        w = synth.DECODE
        lens_np = np.minimum(w.lengths(), args.decode_cap) if args.decode_cap else w.lengths()
        cap = int(args.decode_cap or w.cap)
        dq = synth.normal_bf16_torch(w.seed, synth.STREAM_Q, (w.B, w.Hq, w.d), dev)
        kc = synth.normal_bf16_torch(w.seed, synth.STREAM_K, (w.B, cap, w.Hkv, w.d), dev)
        vc = synth.normal_bf16_torch(w.seed, synth.STREAM_V, (w.B, cap, w.Hkv, w.d), dev)
        lens = torch.from_numpy(lens_np.astype(np.int32)).to(dev)
        do = torch.empty_like(dq)
        dl = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
        ws = torch.empty(lib.attn_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.d, cap, args.chunk), dtype=torch.uint8,
                         device=dev)

        def call():
            lib.attn_decode_splitkv(dq, kc, vc, lens, scale=w.scale, chunk=args.chunk, workspace=ws, out=do, lse=dl)
        byts = int(lens_np.astype(np.int64).sum()) * w.Hkv * w.d * 4 + w.B * w.Hq * (w.d * 4 + 4)
        work, unit, name = byts / 1e9, "GB/s", f"{w.name} (lengths capped at {cap})"
    torch.cuda.synchronize()
    torch.cuda.empty_cache()  # drop the generator's temporaries: only the workload stays on the device
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for a, b in evs:
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in evs]
    med = float(np.median(ms))
    err = lib.attn_get_last_error()
    print(json.dumps({"only": args.only, "workload": name, "median_ms": med, "value": work / (med * 1e-3),
                      "unit": unit, "steps": args.steps, "warmup": args.warmup, "device_error": err}), flush=True)
    if err != lib.ATTN_OK:
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-gates", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e-decode", action="store_true")
    ap.add_argument("--only", choices=("prefill", "prefill_fp8", "backward", "decode"), default=None,
                    help="time one kernel on one workload (profiling and per-workload numbers)")
    ap.add_argument("--workload", default=None, help="prefill workload name for --only prefill")
    ap.add_argument("--decode-cap", type=int, default=0, help="cap decode lengths/cache for --only decode")
    ap.add_argument("--chunk", type=int, default=0, help="decode chunk for --only decode (0 = automatic)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.only:
        run_only(args)
        return
    world, rank, local, dist = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            line = run_reference(args, world, rank)
        else:
            line = run_ours(args, world, rank, local, dist)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if dist:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
