#!/usr/bin/env python
"""Benchmark of the Parallax forward pass (decode + causal prefill) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--sweep] [--no-decode-configs] [--small]

One step = one pass of the whole hot path over one batch of synthetic input:
  * decode: one plx_decode call on a Qwen3-0.6B-shaped layer, B=64, context
    4096 (equal seqlens), Hq=16, Hkv=8, d=128, bf16 KV cache;
  * prefill: one plx_fwd call at the pretraining shape B=8, N=4096, Hq=16,
    Hkv=8, d=128, causal, returning out and lse.
`value` is the decode throughput in GB/s of algorithmic bytes (every cached
key/value row read once, q/r/out once, lse), summed over all ranks; the
prefill TFLOP/s and both kernels' roofline fractions ride along.

Multi-GPU (torchrun, one rank per GPU): every rank runs the same per-GPU
workload on its own GPU with no collective on the data path (weak scaling);
the timed region is bracketed by a barrier + synchronize on both sides and
the max over ranks is taken.

--impl reference times the fp64 CPU oracle (the only reference there is) on
a bounded sample of the same decode workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode attn HBM GB/s & µs/step; prefill TFLOP/s; % of B200 roofline"

DEC = dict(B=64, Hq=16, Hkv=8, S=4096, d=128)
PRE = dict(B=8, Hq=16, Hkv=8, N=4096, d=128)
L2_BYTES = 126 * 1024 * 1024

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ work counts
def decode_bytes(B, Hq, Hkv, d, seqlens):
    """Algorithmic bytes of one decode step: each cached K and V row of the
    live context once (bf16), q, r and out once (bf16), lse (fp32)."""
    kv = sum(int(s) for s in seqlens) * Hkv * 2 * d * 2
    return kv + 3 * B * Hq * d * 2 + 4 * B * Hq


def decode_flops(Hq, d, seqlens):
    """8d per (query head, key): q.k, rho.k, p v, p s v (2d each)."""
    return 8 * d * Hq * sum(int(s) for s in seqlens)


def prefill_flops(B, Hq, N, d, causal=True):
    """8d per unmasked (query, key) pair: QK^T, RK^T, PV, (P*S)V."""
    pairs = N * (N + 1) // 2 if causal else N * N
    return 8 * d * pairs * B * Hq


def backward_flops(B, Hq, N, d, causal=True):
    """16d per unmasked (query, key) pair: the products the gradient needs once
    each -- QK^T and RK^T (recomputed scores), dO V^T, W_hat^T dO, dA^T Q and
    dS^T R (dK), dA K (dQ) and dS K (dR), 2d each."""
    pairs = N * (N + 1) // 2 if causal else N * N
    return 16 * d * pairs * B * Hq


def prefill_bytes(B, Hq, Hkv, N, d):
    return (3 * B * Hq + 2 * B * Hkv) * N * d * 2 + 4 * B * Hq * N


# ------------------------------------------------------------------ environment
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


KERNEL_SOURCES = {
    "prefill": ("plx_fwd.cuh", "plx_tcgen05.cuh", "plx_ptx.cuh"),
    "decode": ("plx_decode.cuh", "plx_ptx.cuh"),
    "backward": ("plx_bwd.cuh", "plx_tcgen05.cuh", "plx_ptx.cuh"),
    "projection": ("plx_proj.cuh", "plx_tcgen05.cuh", "plx_ptx.cuh"),
}


def source_hash(kernel_key):
    """Hash of the source files that make up one kernel."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "parameterized_local_linear_plx_b200", "csrc")
    for name in KERNEL_SOURCES[kernel_key]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (profiles/ncu_traffic.json); else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
    except Exception:
        return None
    e = t.get(kernel_key)
    if not e or e.get("source_hash") != source_hash(kernel_key):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled while timing.

    Polls NVML (the library nvidia-smi reads) from a thread every ~2 ms, so
    even a short timed region gets samples; falls back to `nvidia-smi -lms 50`.
    """

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, cuda_index):
        self.cuda_index = cuda_index
        self.gpu = str(cuda_index)  # nvidia-smi -i: the device UUID when known
        self.uuid = None
        try:
            import torch
            u = str(torch.cuda.get_device_properties(cuda_index).uuid)
            self.uuid = u if u.startswith("GPU-") else "GPU-" + u
            self.gpu = self.uuid
        except Exception:
            pass
        self.samples = []  # (sm_mhz, max_mhz, reasons_mask)
        self._stop = None
        self._thread = None
        self._proc = None

    def _poll_nvml(self, handle, nvml):
        import time as _t
        while not self._stop.is_set():
            try:
                sm = nvml.nvmlDeviceGetClockInfo(handle, nvml.NVML_CLOCK_SM)
                mx = nvml.nvmlDeviceGetMaxClockInfo(handle, nvml.NVML_CLOCK_SM)
                try:
                    rs = nvml.nvmlDeviceGetCurrentClocksEventReasons(handle)
                except Exception:
                    rs = nvml.nvmlDeviceGetCurrentClocksThrottleReasons(handle)
                self.samples.append((float(sm), float(mx), int(rs)))
            except Exception:
                pass
            _t.sleep(0.002)

    def __enter__(self):
        import threading
        try:
            import pynvml as nvml
            nvml.nvmlInit()
            # NVML numbers GPUs ignoring CUDA_VISIBLE_DEVICES: find ours by UUID
            handle = (nvml.nvmlDeviceGetHandleByUUID(self.uuid.encode()) if self.uuid
                      else nvml.nvmlDeviceGetHandleByIndex(self.cuda_index))
            self._stop = threading.Event()
            self._thread = threading.Thread(target=self._poll_nvml, args=(handle, nvml), daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
            try:
                self._proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=clocks.sm,clocks.max.sm,"
                     "clocks_event_reasons.active", "--format=csv,noheader,nounits", "-lms", "50"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                self._proc = None
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self._proc is not None:
            self._proc.terminate()
            try:
                out, _ = self._proc.communicate(timeout=5)
            except Exception:
                self._proc.kill()
                out, _ = self._proc.communicate()
            for ln in out.splitlines():
                parts = [x.strip() for x in ln.split(",")]
                try:
                    self.samples.append((float(parts[0]), float(parts[1]), int(parts[2], 16)))
                except Exception:
                    continue
        return False

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        reasons = set()
        for _, _, mask in self.samples:
            for bit, name in self.REASONS.items():
                if mask & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[0] for s in self.samples),
                "sm_max_mhz": max(s[1] for s in self.samples), "reasons": sorted(reasons),
                "samples": len(self.samples), "source": "nvml" if self._thread is not None else "nvidia-smi"}


# ------------------------------------------------------------------ distributed
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x, world, device=None):
    """Max of a float over all ranks (used only outside the timed region)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world, device=None):
    if world == 1:
        return
    import torch.distributed as dist
    if device is not None and device.type == "cuda":
        dist.barrier(device_ids=[device.index])
    else:
        dist.barrier()


# ------------------------------------------------------------------ CPU oracle timing
def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_decode_sample(q, r, kc, vc, sl, budget_s=10.0, max_entries=None):
    """Run the oracle's effective-weight decode on batch entries one at a time
    (cycling over them) until ~budget_s of wall time is used or max_entries
    are done.  Returns (entries, seconds, bytes)."""
    import oracle
    B, Hq, d = q.shape
    Hkv = kc.shape[1]
    done, t0, nbytes = 0, time.perf_counter(), 0
    limit = max_entries or 1 << 30
    while done < limit:
        b = done % B  # cycle over the entries until the budget is used
        oracle.decode_effective(q[b:b + 1], r[b:b + 1], kc[b:b + 1], vc[b:b + 1], sl[b:b + 1])
        nbytes += decode_bytes(1, Hq, Hkv, d, sl[b:b + 1].tolist())
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return done, time.perf_counter() - t0, nbytes


def oracle_explicit_tiny():
    """Seconds the explicit-Sigma oracle takes on the tiny prefill (B=1, H=1,
    N=256, d=64, causal, fp32 draws rounded to bf16)."""
    import torch
    import oracle
    from parameterized_local_linear_plx_b200 import inputs
    q, k, v, r = inputs.prefill_inputs(1, 1, 1, 256, 64, seed=0, dtype=torch.float32)
    q, k, v, r = (t.bfloat16() for t in (q, k, v, r))
    t0 = time.perf_counter()
    oracle.prefill_explicit(q, k, v, r, causal=True)
    return time.perf_counter() - t0


def bench_config(world):
    """The `config` object of the JSON line, identical in both arms."""
    return {
        "workload": f"decode: Qwen3-0.6B-shaped layer B={DEC['B']} ctx={DEC['S']} (equal seqlens) Hq=16 Hkv=8 "
                    f"d=128 bf16 KV cache; prefill: B={PRE['B']} N={PRE['N']} Hq=16 Hkv=8 d=128 causal bf16, out+lse",
        "l2": f"inputs larger than L2 (decode {decode_bytes(DEC['B'], DEC['Hq'], DEC['Hkv'], DEC['d'], [DEC['S']] * DEC['B']) / 1e9:.2f} GB, "
              f"prefill {prefill_bytes(**PRE) / 1e9:.2f} GB per step; L2 126 MB)",
        "parallelism": f"replicas x{world}, no collective on the data path",
    }


def run_reference(args, world, rank):
    """--impl reference: the fp64 CPU oracle on a bounded sample per step."""
    if rank != 0:
        return 0
    import torch
    from parameterized_local_linear_plx_b200 import inputs
    q, kc, vc, r, sl = inputs.decode_inputs(4, DEC["Hq"], DEC["Hkv"], DEC["S"], DEC["d"], seed=0)
    per_step = 2  # batch entries of the B=64 decode step per timed step
    for _ in range(args.warmup):
        oracle_decode_sample(q, r, kc, vc, sl, budget_s=1e9, max_entries=1)
    times, nbytes = [], 0
    for _ in range(args.steps):
        n, t, b = oracle_decode_sample(q, r, kc, vc, sl, budget_s=1e9, max_entries=per_step)
        times.append(t)
        nbytes += b
    total = sum(times)
    value = nbytes / total / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": bench_config(world),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cpu_threads(), "nproc": os.cpu_count(), "kind": "oracle",
                         "sample": f"decode only: {per_step} of the {DEC['B']} batch entries (x {DEC['Hq']} heads x "
                                   f"{DEC['S']} keys) per step, effective-weight fp64 form"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, world, rank, local):
    import torch
    import torch.distributed as dist
    from parameterized_local_linear_plx_b200 import build, inputs
    if rank == 0:
        build.build()
    if world > 1:
        barrier(world)  # wait for rank 0's build (CPU barrier before CUDA init)
    from parameterized_local_linear_plx_b200 import plx

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)

    # ---- inputs, resident in HBM (generated on the device, seeded per rank)
    q, kc, vc, r, sl = inputs.decode_inputs(DEC["B"], DEC["Hq"], DEC["Hkv"], DEC["S"], DEC["d"],
                                            seed=rank, device=dev)
    seqlens = [DEC["S"]] * DEC["B"]
    ws_bytes = plx.plx_decode_workspace_size(DEC["B"], DEC["Hq"], DEC["Hkv"], DEC["S"], DEC["d"], 0)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    dout = torch.empty_like(q)
    dlse = torch.empty(DEC["B"], DEC["Hq"], dtype=torch.float32, device=dev)
    pq, pk, pv, pr = inputs.prefill_inputs(PRE["B"], PRE["Hq"], PRE["Hkv"], PRE["N"], PRE["d"], seed=100 + rank,
                                           device=dev)
    pout = torch.empty_like(pq)
    plse = torch.empty(PRE["B"], PRE["Hq"], PRE["N"], dtype=torch.float32, device=dev)
    n_splits = plx.plx_decode_num_splits(DEC["B"], DEC["Hq"], DEC["Hkv"], DEC["S"], DEC["d"])
    launches_per_step = 2 + 1  # decode split + combine, prefill

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        plx.plx_decode(q, kc, vc, sl, r, out=dout, lse=dlse, workspace=ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        plx.plx_fwd(pq, pk, pv, pr, causal=True, out=pout, lse=plse, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st = plx.plx_check_device_status(stream)
    if st != plx.PLX_OK:
        raise RuntimeError(f"device status after warm-up: {plx.plx_status_string(st)}")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    total_ms = t_start.elapsed_time(t_end)
    dec_ms = [e[0].elapsed_time(e[1]) for e in evs]
    pre_ms = [e[1].elapsed_time(e[2]) for e in evs]
    st = plx.plx_check_device_status(stream)
    if st != plx.PLX_OK:
        raise RuntimeError(f"device status after timing: {plx.plx_status_string(st)}")

    total_ms_max = max_over_ranks(total_ms, world, dev)
    dec_avg = max_over_ranks(sum(dec_ms) / len(dec_ms), world, dev)
    pre_avg = max_over_ranks(sum(pre_ms) / len(pre_ms), world, dev)

    d_bytes = decode_bytes(DEC["B"], DEC["Hq"], DEC["Hkv"], DEC["d"], seqlens)
    d_flops = decode_flops(DEC["Hq"], DEC["d"], seqlens)
    p_flops = prefill_flops(PRE["B"], PRE["Hq"], PRE["N"], PRE["d"], True)
    # whole-job decode throughput: bytes of all ranks over the slowest rank's decode time
    value = world * d_bytes / (dec_avg * 1e-3) / 1e9
    prefill_tflops = world * p_flops / (pre_avg * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    long_region = total_ms > 1000.0
    tf_key = "bf16_tflops_sustained" if long_region else "bf16_tflops"
    tf_peak = float(peaks.get(tf_key, FALLBACK_PEAKS[tf_key]))
    dec_achieved = d_bytes / (dec_avg * 1e-3) / 1e9
    pre_achieved = p_flops / (pre_avg * 1e-3) / 1e12
    roof_dec = {"bound": "hbm", "achieved": dec_achieved, "peak": hbm, "unit": "GB/s",
                "frac": dec_achieved / hbm, "traffic": load_traffic("decode"),
                "traffic_note": "scaled x4 from a B=16 ncu capture of the decode kernel",
                "kernel": "plx_decode (split + combine), per call",
                "peak_source": f"{peak_src} hbm_gbs"}
    roof_pre = {"bound": "tensor", "achieved": pre_achieved, "peak": tf_peak, "unit": "TFLOP/s",
                "frac": pre_achieved / tf_peak, "traffic": load_traffic("prefill"),
                "traffic_note": "scaled x4 from a B=2 ncu capture; a lower bound (the last writes are still "
                                "in L2 when the capture ends)",
                "kernel": "plx_fwd_kernel<128,true>", "peak_source": f"{peak_src} {tf_key}"}

    # ---- end to end through the public API: pinned host buffers, copies timed
    e2e = run_e2e(plx, args, dev, stream, world, q, kc, vc, r, sl, d_bytes)

    # ---- the same decode step on a paged cache (block tables), timed on its own
    paged = run_paged(plx, args, dev, stream, world, local, d_bytes, hbm, peak_src)

    # ---- context-parallel decode, ranks emulated as slices on this GPU (timed on its own)
    cpd = run_cp(plx, args, dev, stream, world, q, kc, vc, r, sl, d_bytes)

    # ---- context-parallel prefill, the last rank emulated on this GPU (timed on its own)
    cpp = run_cp_prefill(plx, args, dev, stream, local, tf_peak, peak_src)

    # ---- packed variable-length prefill with the same token count (timed on its own)
    varlen = run_varlen(plx, args, dev, stream, world, local, tf_peak, peak_src, tf_key)

    # ---- host cost of one small decode call
    host = run_host_overhead(plx, dev, stream)

    # ---- prefill end to end: inputs from pinned host memory, out and lse back
    e2e_pre = run_e2e_prefill(plx, args, dev, stream, world, pq, pk, pv, pr)

    # ---- the q/k/v/rho projection in front of the attention (timed on its own)
    proj = run_projection(plx, args, dev, stream, world, tf_peak, f"{peak_src} {tf_key}")

    # ---- training backward of the prefill shape (timed on its own; not part of the step)
    bwd = run_backward(plx, args, dev, stream, world, local, pq, pk, pv, pr, peaks, peak_src)

    # ---- every decode configuration (sweep, B=1/16, compute-matched), timed on its own, rank 0 at N=1
    dcfg = None
    if world == 1 and not args.no_decode_configs:
        torch.cuda.empty_cache()
        dcfg = decode_configs(plx, args, dev, hbm)
    # ---- CPU baseline: the oracle on this host, rank 0, N=1 only
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        qh, kh, vh, rh, slh = (t.cpu() for t in (q, kc, vc, r, sl))
        n, secs, nb = oracle_decode_sample(qh, rh, kh, vh, slh, budget_s=10.0)
        cpu = {"value": nb / secs / 1e9, "unit": "GB/s", "cores": cpu_threads(), "nproc": os.cpu_count(), "kind": "oracle",
               "sample": f"{n} (b) entries of the B={DEC['B']} decode step, cycling (each: all {DEC['Hq']} "
                         f"heads x {DEC['S']} keys), effective-weight fp64 form, {secs:.1f} s",
               "explicit_tiny_prefill_s": oracle_explicit_tiny()}

    clocks = clk.summary()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": bench_config(world),
            "decode": {"gbs": value, "us_per_step": dec_avg * 1e3, "us_median": statistics.median(dec_ms) * 1e3,
                       "bytes_per_step": d_bytes, "partitions": n_splits,
                       "tflops": world * d_flops / (dec_avg * 1e-3) / 1e12},
            "prefill": {"tflops": prefill_tflops, "ms_per_step": pre_avg, "ms_median": statistics.median(pre_ms),
                        "flops_per_step": p_flops,
                        "gbs_io": world * prefill_bytes(**PRE) / (pre_avg * 1e-3) / 1e9,
                        "roofline": roof_pre},
            # the dominant kernel of the step by time is the prefill kernel
            "roofline": roof_pre,
            "roofline_decode": roof_dec,
            "e2e": e2e,
            "e2e_prefill": e2e_pre,
            "decode_host_overhead": host,
            "projection": proj,
            "decode_paged": paged,
            "prefill_varlen": varlen,
            "decode_cp_emulated": cpd,
            "prefill_cp_emulated": cpp,
            "backward": bwd,
            "decode_configs": dcfg,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    return 0


def run_paged(plx, args, dev, stream, world, local, d_bytes, hbm, peak_src):
    """plx_decode_paged on the decode workload (B=64, context 4096, equal
    seqlens) with pages of 16 and of 64 keys, slots assigned to pool pages by
    a random permutation; CUDA events per call, max over ranks."""
    import torch
    res = {}
    for ps in (64, 16):
        q, kp, vp, r, table, sl = inputs_mod().paged_decode_inputs(
            DEC["B"], DEC["Hq"], DEC["Hkv"], DEC["S"] // ps, ps, DEC["d"], seed=200 + local, seqlens="equal",
            device=dev)
        out = torch.empty_like(q)
        lse = torch.empty(DEC["B"], DEC["Hq"], dtype=torch.float32, device=dev)
        need = plx.plx_decode_workspace_size(DEC["B"], DEC["Hq"], DEC["Hkv"], DEC["S"], DEC["d"], 0)
        ws = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
        for _ in range(max(3, args.warmup)):
            plx.plx_decode_paged(q, kp, vp, table, sl, r, out=out, lse=lse, workspace=ws, stream=stream)
        steps = max(1, min(args.steps, 50))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(steps):
            plx.plx_decode_paged(q, kp, vp, table, sl, r, out=out, lse=lse, workspace=ws, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        st = plx.plx_check_device_status(stream)
        if st != plx.PLX_OK:
            raise RuntimeError(f"device status after the paged decode: {plx.plx_status_string(st)}")
        us = max_over_ranks(e0.elapsed_time(e1) / steps * 1e3, world, dev)
        gbs = d_bytes / (us * 1e-6) / 1e9
        res[f"page_{ps}"] = {"gbs": world * gbs, "us_per_step": us, "frac_of_hbm": gbs / hbm}
        del q, kp, vp, r, table, sl, out, lse, ws
    res["workload"] = (f"decode B={DEC['B']} ctx={DEC['S']} Hq={DEC['Hq']} Hkv={DEC['Hkv']} d={DEC['d']} on page "
                       f"pools [pages, Hkv, page_size, d], random page assignment")
    res["peak_source"] = f"{peak_src} hbm_gbs"
    return res


def run_cp(plx, args, dev, stream, world, q, kc, vc, r, sl, d_bytes, ranks=8):
    """The per-rank costs of context-parallel decode for the decode workload
    split over `ranks` ranks along the sequence, measured on this one GPU:
    one rank's plx_decode_partial on its 4096/ranks-key slice, the merge of
    all ranks' partials, and the bytes each rank sends in the all-gather."""
    import torch
    L = DEC["S"] // ranks
    ks = kc[:, :, :L].contiguous()
    vs = vc[:, :, :L].contiguous()
    part = plx.plx_decode_partial(q, ks, vs, sl, r, key_offset=0, stream=stream)
    gathered = torch.stack([part] * ranks)
    out = torch.empty_like(q)
    lse = torch.empty(DEC["B"], DEC["Hq"], dtype=torch.float32, device=dev)

    def timed(fn, n):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n * 1e3

    n = max(1, min(args.steps, 50))
    t_part = timed(lambda: plx.plx_decode_partial(q, ks, vs, sl, r, key_offset=0, partial=part, stream=stream), n)
    t_merge = timed(lambda: plx.plx_decode_merge(gathered, out=out, lse=lse, stream=stream), n)
    st = plx.plx_check_device_status(stream)
    if st != plx.PLX_OK:
        raise RuntimeError(f"device status after the context-parallel legs: {plx.plx_status_string(st)}")
    slice_bytes = d_bytes // ranks
    return {"workload": f"decode B={DEC['B']} ctx={DEC['S']} split over {ranks} ranks along the sequence "
                        f"({L} keys per rank); ranks emulated on one GPU",
            "ranks": ranks, "partial_us_per_rank": t_part, "merge_us": t_merge,
            "slice_gbs": slice_bytes / (t_part * 1e-6) / 1e9,
            "exchange_bytes_per_rank": part.numel() * 4,
            "note": "per-rank step time = partial + all-gather of exchange_bytes_per_rank + merge; the "
                    "all-gather is not measured (one GPU per run)"}


def run_cp_prefill(plx, args, dev, stream, local, tf_peak, peak_src, ranks=4):
    """The per-rank costs of context-parallel prefill for the prefill workload
    cut into `ranks` chunks along the sequence, measured on this one GPU for
    the last rank, which has the most blocks: its queries against its own
    chunk (causal) and every earlier chunk (in full), then the merge."""
    import torch
    B, Hq, Hkv, d = PRE["B"], PRE["Hq"], PRE["Hkv"], PRE["d"]
    C = PRE["N"] // ranks
    g = torch.Generator(device=dev).manual_seed(400 + local)
    q = torch.randn(B, Hq, C, d, generator=g, device=dev).bfloat16()
    r = (0.1 * torch.randn(B, Hq, C, d, generator=g, device=dev)).bfloat16()
    ks = torch.randn(ranks, B, Hkv, C, d, generator=g, device=dev).bfloat16()
    vs = torch.randn(ranks, B, Hkv, C, d, generator=g, device=dev).bfloat16()
    parts = torch.empty(ranks, B, Hq, C, 2 * d + 4, dtype=torch.float32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, C, dtype=torch.float32, device=dev)
    last = ranks - 1

    def blocks():
        for j in range(ranks):
            plx.plx_fwd_partial(q, ks[j], vs[j], r, causal=(j == last), partial=parts[j], stream=stream)

    def timed(fn, n):
        for _ in range(3):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / n

    n = max(1, min(args.steps, 20))
    t_blocks = timed(blocks, n)
    t_merge = timed(lambda: plx.plx_fwd_merge(parts, out=out, lse=lse, stream=stream), n)

    # the zig-zag layout: 2 * ranks chunks of c = N / (2 ranks), rank r holds
    # chunks r and 2 ranks - 1 - r; every rank's blocks and merges, timed rank by rank
    from parameterized_local_linear_plx_b200 import cp as cpm
    c = PRE["N"] // (2 * ranks)
    zq = torch.randn(B, Hq, 2 * c, d, generator=g, device=dev).bfloat16()
    zr = (0.1 * torch.randn(B, Hq, 2 * c, d, generator=g, device=dev)).bfloat16()
    zk = torch.randn(2 * ranks, B, Hkv, c, d, generator=g, device=dev).bfloat16()
    zv = torch.randn(2 * ranks, B, Hkv, c, d, generator=g, device=dev).bfloat16()
    zq_h = [zq[:, :, :c].contiguous(), zq[:, :, c:].contiguous()]
    zr_h = [zr[:, :, :c].contiguous(), zr[:, :, c:].contiguous()]
    # slots 0 .. ranks - 1 for the early chunk's blocks (at most ranks), ranks .. 3 ranks - 1 for the late one's
    zparts = torch.empty(3 * ranks, B, Hq, c, 2 * d + 4, dtype=torch.float32, device=dev)
    zout = torch.empty(B, Hq, c, d, dtype=torch.bfloat16, device=dev)
    zlse = torch.empty(B, Hq, c, dtype=torch.float32, device=dev)
    zz = []
    for rk in range(ranks):
        local, remote = cpm.zigzag_blocks(rk, ranks)
        a, b_ = cpm.zigzag_chunks(rk, ranks)

        def zig(local=local, remote=remote, a=a, b_=b_):
            used = {a: 0, b_: ranks}
            for qc, kc, causal in local + remote:
                h = 0 if qc == a else 1
                plx.plx_fwd_partial(zq_h[h], zk[kc], zv[kc], zr_h[h], causal=causal, partial=zparts[used[qc]],
                                    stream=stream)
                used[qc] += 1
            plx.plx_fwd_merge(zparts[:used[a]], out=zout, lse=zlse, stream=stream)
            plx.plx_fwd_merge(zparts[ranks:used[b_]], out=zout, lse=zlse, stream=stream)

        zz.append(timed(zig, n))
    zflops = 8 * d * (2 * (c * (c + 1) // 2) + (2 * ranks - 1) * c * c) * B * Hq  # every rank's pairs
    st = plx.plx_check_device_status(stream)
    if st != plx.PLX_OK:
        raise RuntimeError(f"device status after the context-parallel prefill legs: {plx.plx_status_string(st)}")
    flops = 8 * d * (C * (C + 1) // 2 + last * C * C) * B * Hq  # the last rank's (query, key) pairs
    return {"workload": f"causal prefill B={B} N={PRE['N']} Hq={Hq} Hkv={Hkv} d={d} cut into {ranks} chunks of {C} "
                        f"(one per rank); the last rank (most blocks) emulated on one GPU",
            "ranks": ranks, "blocks_ms_last_rank": t_blocks, "merge_ms": t_merge,
            "tflops_blocks": flops / (t_blocks * 1e-3) / 1e12, "frac_of_peak": flops / (t_blocks * 1e-3) / 1e12 / tf_peak,
            "peak_source": peak_src,
            "exchange_bytes_per_rank": 2 * B * Hkv * C * d * 2,
            "note": "per-rank step time = all-gather of the key / value chunks + blocks + merge; the all-gather "
                    "is not measured (one GPU per run); earlier ranks have fewer blocks",
            "zigzag": {"layout": f"{2 * ranks} chunks of {c}; rank r holds chunks r and {2 * ranks - 1} - r: "
                                 f"{2 * ranks + 1} blocks (2 causal) and 2 merges per rank",
                       "ms_per_rank": zz, "max_over_min": max(zz) / min(zz),
                       "tflops_slowest_rank": zflops / (max(zz) * 1e-3) / 1e12,
                       "note": "blocks + merges per rank; the all-gather overlaps the three local blocks"}}


VARLEN_LENS = [4096, 1, 2048, 777, 1024, 3000, 64, 65, 512, 1500, 4000, 129, 333, 2500, 100, 900,
               4096, 2048, 1200, 3100]  # 31,493 tokens in 20 sequences of 1 .. 4096


def run_varlen(plx, args, dev, stream, world, local, tf_peak, peak_src, tf_key):
    """plx_fwd_varlen on 20 packed causal sequences of 1 .. 4096 tokens
    (31,493 tokens, about the prefill step's 32,768), Hq=16, Hkv=8, d=128."""
    import torch
    lens = VARLEN_LENS if not args.small else VARLEN_LENS[:5]
    total = sum(lens)
    g = torch.Generator(device=dev).manual_seed(300 + local)
    mk = lambda h: (torch.randn(total, h, PRE["d"], generator=g, device=dev)).bfloat16()
    q, k, v = mk(PRE["Hq"]), mk(PRE["Hkv"]), mk(PRE["Hkv"])
    r = (0.1 * torch.randn(total, PRE["Hq"], PRE["d"], generator=g, device=dev)).bfloat16()
    cu = torch.tensor([0] + list(torch.cumsum(torch.tensor(lens), 0)), dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(PRE["Hq"], total, dtype=torch.float32, device=dev)
    for _ in range(max(3, args.warmup)):
        plx.plx_fwd_varlen(q, k, v, cu, max(lens), r, out=out, lse=lse, stream=stream)
    steps = max(1, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for _ in range(steps):
        plx.plx_fwd_varlen(q, k, v, cu, max(lens), r, out=out, lse=lse, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    st = plx.plx_check_device_status(stream)
    if st != plx.PLX_OK:
        raise RuntimeError(f"device status after the packed prefill: {plx.plx_status_string(st)}")
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, world, dev)
    flops = sum(8 * PRE["d"] * (n * (n + 1) // 2) * PRE["Hq"] for n in lens)
    achieved = flops / (ms * 1e-3) / 1e12
    return {"workload": f"{len(lens)} packed causal sequences of 1..{max(lens)} tokens ({total} tokens), "
                        f"Hq={PRE['Hq']} Hkv={PRE['Hkv']} d={PRE['d']}, out+lse",
            "tflops": world * achieved, "ms_per_step": ms, "flops_per_step": flops,
            "frac_of_peak": achieved / tf_peak, "peak_source": f"{peak_src} {tf_key}"}


def inputs_mod():
    from parameterized_local_linear_plx_b200 import inputs
    return inputs


def run_backward(plx, args, dev, stream, world, local, pq, pk, pv, pr, peaks, peak_src):
    """plx_fwd_train then plx_bwd at the prefill shape (B=8, N=4096, causal),
    dO ~ N(0, 1) bf16; CUDA events around each call, max over ranks."""
    import torch
    g = torch.Generator(device=dev).manual_seed(7 + local)
    dout = torch.randn(pq.shape, generator=g, device=dev).bfloat16()
    out = torch.empty_like(pq)
    obar = torch.empty_like(pq)
    lse = torch.empty(PRE["B"], PRE["Hq"], PRE["N"], dtype=torch.float32, device=dev)
    sbar = torch.empty_like(lse)
    dq, dr, dk, dv = torch.empty_like(pq), torch.empty_like(pq), torch.empty_like(pk), torch.empty_like(pv)
    ws = torch.empty(plx.plx_bwd_workspace_size(PRE["B"], PRE["Hq"], PRE["Hkv"], PRE["N"], PRE["d"]),
                     dtype=torch.uint8, device=dev)

    def one(ev=None):
        if ev is not None:
            ev[0].record(stream)
        plx.plx_fwd_train(pq, pk, pv, pr, causal=True, out=out, lse=lse, obar=obar, sbar=sbar, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        plx.plx_bwd(pq, pk, pv, pr, out, dout, lse, obar, sbar, causal=True, dq=dq, dk=dk, dv=dv, dr=dr,
                    workspace=ws, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(max(3, args.warmup)):
        one()
    torch.cuda.synchronize(dev)
    steps = max(1, min(args.steps, 20))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    barrier(world, dev)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        for i in range(steps):
            one(evs[i])
        torch.cuda.synchronize(dev)
    barrier(world, dev)
    st = plx.plx_check_device_status(stream)
    if st != plx.PLX_OK:
        raise RuntimeError(f"device status after the backward: {plx.plx_status_string(st)}")
    fwd_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in evs) / steps, world, dev)
    bwd_ms = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in evs) / steps, world, dev)
    b_flops = backward_flops(PRE["B"], PRE["Hq"], PRE["N"], PRE["d"], True)
    f_flops = prefill_flops(PRE["B"], PRE["Hq"], PRE["N"], PRE["d"], True)
    tf_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    achieved = b_flops / (bwd_ms * 1e-3) / 1e12
    return {
        "workload": f"training backward of the prefill shape B={PRE['B']} N={PRE['N']} Hq={PRE['Hq']} "
                    f"Hkv={PRE['Hkv']} d={PRE['d']} causal; dO ~ N(0,1) bf16",
        "tflops": world * achieved, "ms_per_step": bwd_ms, "flops_per_step": b_flops,
        "fwd_train_ms": fwd_ms, "fwd_train_tflops": world * f_flops / (fwd_ms * 1e-3) / 1e12,
        "steps": steps, "launches_per_step": 4,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": tf_peak, "unit": "TFLOP/s",
                     "frac": achieved / tf_peak, "traffic": load_traffic("backward"),
                     "kernel": "plx_bwd (pre + q-side + kv-side), per call",
                     "peak_source": f"{peak_src} bf16_tflops"},
        "clocks": clk.summary(),
    }


PROJ = dict(d_model=1024)  # Qwen3-0.6B hidden size


def run_projection(plx, args, dev, stream, world, tf_peak, peak_src):
    """plx_qkvr_proj at the prefill shape (tokens B*N = 32768, d_model = 1024,
    W = [W_Q; W_K; W_V; W_R] of 6144 rows) and plx_qkvr_proj_decode at the
    decode shape (B = 64 new tokens, k and v appended into a context-4096
    cache); CUDA events around each call, max over ranks."""
    import torch
    B, N, Hq, Hkv, d = PRE["B"], PRE["N"], PRE["Hq"], PRE["Hkv"], PRE["d"]
    dm = PROJ["d_model"]
    nout = (2 * Hq + 2 * Hkv) * d
    g = torch.Generator(device=dev).manual_seed(500)
    x = torch.randn(B * N, dm, generator=g, device=dev).bfloat16()
    w = (torch.randn(nout, dm, generator=g, device=dev) / dm ** 0.5).bfloat16()
    q = torch.empty(B, Hq, N, d, dtype=torch.bfloat16, device=dev)
    r = torch.empty_like(q)
    k = torch.empty(B, Hkv, N, d, dtype=torch.bfloat16, device=dev)
    v = torch.empty_like(k)

    def timed(fn, n):
        for _ in range(3):
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        barrier(world, dev)
        torch.cuda.synchronize(dev)
        for a, b in evs:
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world, dev)
        return max_over_ranks(sum(a.elapsed_time(b) for a, b in evs) / n, world, dev)

    n = max(1, min(args.steps, 20))
    ms = timed(lambda: plx.plx_qkvr_proj(x, w, B, N, Hq, Hkv, d, q=q, k=k, v=v, r=r, stream=stream), n)
    flops = 2 * B * N * dm * nout
    achieved = flops / (ms * 1e-3) / 1e12
    # decode step: 64 new tokens appended into a [64, 8, 4096, 128] cache at row 4000
    Bd, S = DEC["B"], DEC["S"]
    xd = torch.randn(Bd, dm, generator=g, device=dev).bfloat16()
    kc = torch.zeros(Bd, Hkv, S, d, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    sl = torch.full((Bd,), S - 96, dtype=torch.int32, device=dev)
    sl2 = torch.empty_like(sl)
    qd = torch.empty(Bd, Hq, d, dtype=torch.bfloat16, device=dev)
    rd = torch.empty_like(qd)
    us_dec = 1e3 * timed(lambda: plx.plx_qkvr_proj_decode(xd, w, kc, vc, sl, Hq, seqlens_out=sl2, q=qd, r=rd,
                                                          stream=stream), n)
    st = plx.plx_check_device_status(stream)
    if st != plx.PLX_OK:
        raise RuntimeError(f"device status after the projection: {plx.plx_status_string(st)}")
    w_bytes = nout * dm * 2
    return {"workload": f"q/k/v/rho projection x W^T, x [{B * N}, {dm}], W [{nout}, {dm}] ([W_Q; W_K; W_V; W_R]), "
                        f"outputs scattered to [B, H, N, d]; decode: {Bd} tokens, k/v appended into the cache",
            "tflops": world * achieved, "ms_per_step": ms, "flops_per_step": flops,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": tf_peak, "unit": "TFLOP/s",
                         "frac": achieved / tf_peak, "traffic": load_traffic("projection"),
                         "traffic_note": "scaled x4 from a 2 x 4096-token ncu capture", "peak_source": peak_src},
            "decode_us": us_dec,
            "decode_gbs_weights": w_bytes / (us_dec * 1e-6) / 1e9,
            "decode_note": "at 64 tokens the step is bound by reading W once (HBM); gbs counts the weight bytes"}


def run_host_overhead(plx, dev, stream):
    """Host time per decode call at B=1 (context 4096): the Python binding
    (argument checks, ctypes) and the raw C ABI through ctypes, each over 200
    calls enqueued without synchronising (the GPU keeps up at this size, so
    the loop measures the host's enqueue cost: checks, cached tensor maps, two
    kernel launches)."""
    import ctypes
    import torch
    q, kc, vc, r, sl = inputs_mod().decode_inputs(1, DEC["Hq"], DEC["Hkv"], DEC["S"], DEC["d"], seed=9, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(1, DEC["Hq"], dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, plx.plx_decode_workspace_size(1, DEC["Hq"], DEC["Hkv"], DEC["S"], DEC["d"], 0)),
                     dtype=torch.uint8, device=dev)
    P = ctypes.c_void_p
    args_c = (P(q.data_ptr()), P(r.data_ptr()), P(kc.data_ptr()), P(vc.data_ptr()), P(sl.data_ptr()),
              P(out.data_ptr()), P(lse.data_ptr()), 1, DEC["Hq"], DEC["Hkv"], DEC["S"], DEC["d"],
              DEC["d"] ** -0.5, 0, P(ws.data_ptr()), ws.numel(), P(stream.cuda_stream))
    res = {}
    for name, fn in (("binding", lambda: plx.plx_decode(q, kc, vc, sl, r, out=out, lse=lse, workspace=ws,
                                                       stream=stream)),
                     ("c_abi", lambda: plx.lib.plx_decode(*args_c))):
        for _ in range(20):
            fn()
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for _ in range(200):
            fn()
        res[f"{name}_us_per_call"] = (time.perf_counter() - t0) / 200 * 1e6
        torch.cuda.synchronize(dev)
    st = plx.plx_check_device_status(stream)
    if st != plx.PLX_OK:
        raise RuntimeError(f"device status after the host-overhead leg: {plx.plx_status_string(st)}")
    res["workload"] = f"plx_decode B=1 ctx={DEC['S']} Hq={DEC['Hq']} Hkv={DEC['Hkv']} d={DEC['d']}, 200 calls"
    return res


def run_e2e_prefill(plx, args, dev, stream, world, pq, pk, pv, pr):
    """plx_fwd measured with the step's q, k, v, r copied from pinned host
    memory and out, lse copied back, all inside the timed region (one H2D
    and one D2H copy per step, of packed buffers)."""
    import torch
    nq, nk = pq.numel() * 2, pk.numel() * 2
    nout = pq.numel() * 2
    nlse = PRE["B"] * PRE["Hq"] * PRE["N"] * 4
    h_in = torch.empty(2 * nq + 2 * nk, dtype=torch.uint8).pin_memory()
    offs = [0, nq, nq + nk, nq + 2 * nk]
    for t, o, nb in ((pq, offs[0], nq), (pk, offs[1], nk), (pv, offs[2], nk), (pr, offs[3], nq)):
        h_in[o:o + nb].view(torch.bfloat16).view(t.shape).copy_(t.cpu())
    d_in = torch.empty_like(h_in, device=dev)
    dq = d_in[offs[0]:offs[0] + nq].view(torch.bfloat16).view(pq.shape)
    dk = d_in[offs[1]:offs[1] + nk].view(torch.bfloat16).view(pk.shape)
    dv = d_in[offs[2]:offs[2] + nk].view(torch.bfloat16).view(pv.shape)
    dr = d_in[offs[3]:offs[3] + nq].view(torch.bfloat16).view(pq.shape)
    d_res = torch.empty(nout + nlse, dtype=torch.uint8, device=dev)
    dout = d_res[:nout].view(torch.bfloat16).view(pq.shape)
    dlse = d_res[nout:].view(torch.float32).view(PRE["B"], PRE["Hq"], PRE["N"])
    h_res = torch.empty(nout + nlse, dtype=torch.uint8).pin_memory()

    def one():
        d_in.copy_(h_in, non_blocking=True)
        plx.plx_fwd(dq, dk, dv, dr, causal=True, out=dout, lse=dlse, stream=stream)
        h_res.copy_(d_res, non_blocking=True)

    for _ in range(3):
        one()
    torch.cuda.synchronize(dev)
    steps = max(1, min(args.steps, 10))
    barrier(world, dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(steps):
        one()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    flops = prefill_flops(PRE["B"], PRE["Hq"], PRE["N"], PRE["d"], True)
    return {"value": world * flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h_in.numel(),
            "d2h_bytes_per_step": h_res.numel(), "ms_per_step": ms}


def run_e2e(plx, args, dev, stream, world, q, kc, vc, r, sl, d_bytes):
    """Decode measured through plx_decode with the step's inputs (q, r,
    seqlens) copied from pinned host memory and its result (out, lse) read
    back, all inside the timed region.  The inputs travel packed in one
    buffer and the results in another (one H2D and one D2H copy per step);
    the KV cache is the engine's resident state and is not re-sent."""
    import torch
    B, Hq, d = q.shape
    nq, nsl = q.numel() * 2, sl.numel() * 4
    nout, nlse = q.numel() * 2, B * Hq * 4
    h_in = torch.empty(2 * nq + nsl, dtype=torch.uint8).pin_memory()
    h_in[:nq].view(torch.bfloat16).view(q.shape).copy_(q.cpu())
    h_in[nq:2 * nq].view(torch.bfloat16).view(q.shape).copy_(r.cpu())
    h_in[2 * nq:].view(torch.int32).copy_(sl.cpu())
    d_in = torch.empty_like(h_in, device=dev)
    dq = d_in[:nq].view(torch.bfloat16).view(q.shape)
    dr = d_in[nq:2 * nq].view(torch.bfloat16).view(q.shape)
    dsl = d_in[2 * nq:].view(torch.int32)
    d_res = torch.empty(nout + nlse, dtype=torch.uint8, device=dev)
    dout = d_res[:nout].view(torch.bfloat16).view(q.shape)
    dlse = d_res[nout:].view(torch.float32).view(B, Hq)
    h_res = torch.empty(nout + nlse, dtype=torch.uint8).pin_memory()
    ws = torch.empty(max(16, plx.plx_decode_workspace_size(B, Hq, kc.shape[1], kc.shape[2], d, 0)),
                     dtype=torch.uint8, device=dev)

    def one():
        d_in.copy_(h_in, non_blocking=True)
        plx.plx_decode(dq, kc, vc, dsl, dr, out=dout, lse=dlse, workspace=ws, stream=stream)
        h_res.copy_(d_res, non_blocking=True)

    for _ in range(max(3, args.warmup)):
        one()
    torch.cuda.synchronize(dev)
    barrier(world, dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        one()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, world, dev)
    return {"value": world * d_bytes / (ms * 1e-3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h_in.numel(),
            "d2h_bytes_per_step": h_res.numel(), "us_per_step": ms * 1e3}


# ------------------------------------------------------------------ decode configurations
SWEEP_B = (1, 8, 64, 256, 1024, 2048)
SWEEP_CTX = (128, 1024, 4096, 16384, 32768)
SWEEP_CAP = 150e9  # bytes of KV cache above which a sweep point is skipped


def time_decode_point(plx, torch, dev, pool_k, pool_v, B, ctx, d, seqlens_mode, seed, use_r=True, iters=10):
    """Per-call time of plx_decode (split + combine, or chunk + merge) on a
    [B, 8, ctx, d] cache viewed from the pools; q, r ~ N(0,1), N(0, 0.1^2);
    seqlens "equal" or "ragged" (uniform in [ctx/2, ctx]).

    us: calls enqueued back to back between one pair of CUDA events (three
    rounds, the median), each call on its own copy of the cache, rotating
    over enough copies (adjacent views of the pools) that at least twice the
    L2's size of other cache bytes is read between two uses of a copy; a
    cache of 2x L2 or more is its own rotation.  This is the steady per-call
    cost of a stream of decode calls from HBM.
    us_single: one call between its own pair of events after the L2 was
    emptied (a read of twice its size) -- the cold single-call latency; each
    timing event costs the GPU ~2.6 us before the next kernel starts, which
    this figure carries."""
    Hq, Hkv = 16, 8
    n = B * Hkv * ctx * d
    alloc = 2 * n * 2
    copies = 1 if alloc >= 2 * L2_BYTES else -(-2 * L2_BYTES // alloc) + 1
    copies = max(1, min(copies, pool_k.numel() // n))
    rotate_ok = copies * alloc >= 2 * L2_BYTES or alloc >= 2 * L2_BYTES
    views = [(pool_k[i * n:(i + 1) * n].view(B, Hkv, ctx, d), pool_v[i * n:(i + 1) * n].view(B, Hkv, ctx, d))
             for i in range(copies)]
    kc, vc = views[0]
    g = torch.Generator(device=dev).manual_seed(seed)
    q = torch.randn(B, Hq, d, generator=g, device=dev).bfloat16()
    r = (0.1 * torch.randn(B, Hq, d, generator=g, device=dev)).bfloat16() if use_r else None
    if seqlens_mode == "equal":
        sl = torch.full((B,), ctx, dtype=torch.int32, device=dev)
    else:
        sl = torch.randint(ctx // 2, ctx + 1, (B,), generator=g, device=dev, dtype=torch.int32)
    ws = torch.empty(max(16, plx.plx_decode_workspace_size(B, Hq, Hkv, ctx, d, 0)), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=dev)
    for i in range(max(5, copies)):
        kv = views[i % copies]
        plx.plx_decode(q, kv[0], kv[1], sl, r, out=out, lse=lse, workspace=ws)
    # back to back over the rotation
    calls = copies * max(1, -(-max(iters, 20) // copies))
    per_call = []
    for _ in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for i in range(calls):
            kv = views[i % copies]
            plx.plx_decode(q, kv[0], kv[1], sl, r, out=out, lse=lse, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        per_call.append(a.elapsed_time(b) / calls)
    # single calls after emptying the L2 by READING a buffer twice its size
    # (writing one would leave dirty lines whose write-back then competes
    # with the call being timed); caches of at least 2x L2 need no flush
    flush_src = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if alloc < 2 * L2_BYTES else None
    flush_dst = torch.empty((), dtype=torch.float32, device=dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    torch.cuda.synchronize()
    for a, b in evs:
        if flush_src is not None:
            torch.sum(flush_src, dim=0, out=flush_dst)
        a.record()
        plx.plx_decode(q, kc, vc, sl, r, out=out, lse=lse, workspace=ws)
        b.record()
    torch.cuda.synchronize()
    st = plx.plx_check_device_status()
    if st != plx.PLX_OK:
        raise RuntimeError(f"device status after decode point ({B}, {ctx}): {plx.plx_status_string(st)}")
    ms_single = statistics.median(a.elapsed_time(b) for a, b in evs)
    ms = statistics.median(per_call) if rotate_ok else ms_single
    nb = decode_bytes(B, Hq, Hkv, d, sl.tolist())
    return {"B": B, "ctx": ctx, "d": d, "seqlens": seqlens_mode, "us": ms * 1e3, "bytes": nb,
            "gbs": nb / (ms * 1e-3) / 1e9, "us_single": ms_single * 1e3,
            "gbs_single": nb / (ms_single * 1e-3) / 1e9, "kv_alloc_gb": alloc / 1e9,
            "rotation_copies": copies if rotate_ok else None, "flushed_l2_single": flush_src is not None}


def decode_configs(plx, args, dev, hbm):
    """Every decode configuration of the workload list, timed on this GPU:
    the Qwen3-0.6B-shaped layer at B = 1 and 16 (B = 64 is the bench's own
    decode), the sweep B x context with ragged lengths (points whose KV cache
    exceeds 150 GB skipped), and the compute-matched pair (Parallax at d = 64
    against the softmax-only path at d = 128, B = 128, context 32768).  One
    pair of K/V pools sized for the largest point is drawn once and viewed
    for every point."""
    import torch
    elems = 0
    for B in SWEEP_B:
        for ctx in SWEEP_CTX:
            if B * ctx * 8 * 2 * 128 * 2 <= SWEEP_CAP:
                elems = max(elems, B * 8 * ctx * 128)
    free, _ = torch.cuda.mem_get_info(dev)
    if 2 * elems * 2 > free - (4 << 30):
        return {"skipped": f"needs {4 * elems / 1e9:.0f} GB of free device memory, {free / 1e9:.0f} GB free"}
    pool_k = torch.empty(elems, dtype=torch.bfloat16, device=dev)
    pool_v = torch.empty(elems, dtype=torch.bfloat16, device=dev)
    g = torch.Generator(device=dev).manual_seed(1234)
    step = 1 << 28
    for pool in (pool_k, pool_v):
        for i0 in range(0, elems, step):
            i1 = min(elems, i0 + step)
            pool[i0:i1].copy_(torch.randn(i1 - i0, generator=g, device=dev))
    iters = 10 if not args.small else 3
    res = {"peak_hbm_gbs": hbm, "spec_hbm_gbs": 8000.0,
           "timing": "us: per call, calls enqueued back to back between one pair of CUDA events (median of 3 "
                     "rounds of >= 20 calls), each call on its own copy of the KV cache, rotating over enough "
                     "copies that >= 2x L2 of other cache bytes is read between two uses of a copy (a cache of "
                     "2x L2 or more is its own rotation); us_single: one call between its own events after a "
                     "2x-L2 read emptied the L2 (median of the calls), which includes the ~2.6 us a timing "
                     "event costs the GPU before the next kernel"}
    res["config2"] = []
    for B in (1, 16):
        pt = time_decode_point(plx, torch, dev, pool_k, pool_v, B, 4096, 128, "equal", seed=B, iters=iters)
        pt["frac_of_hbm"] = pt["gbs"] / hbm
        pt["frac_of_spec"] = pt["gbs"] / 8000.0
        res["config2"].append(pt)
    res["sweep"] = []
    for B in SWEEP_B:
        for ctx in SWEEP_CTX:
            if B * ctx * 8 * 2 * 128 * 2 > SWEEP_CAP:
                res["sweep"].append({"B": B, "ctx": ctx, "skipped": "KV cache above 150 GB"})
                continue
            pt = time_decode_point(plx, torch, dev, pool_k, pool_v, B, ctx, 128, "ragged", seed=B * 7 + ctx,
                                   iters=iters)
            pt["frac_of_hbm"] = pt["gbs"] / hbm
            pt["frac_of_spec"] = pt["gbs"] / 8000.0
            pt["bar_applies"] = pt["bytes"] >= 100e6  # ~100 MB and up: not launch-bound
            res["sweep"].append(pt)
    cm = {}
    for name, d, use_r in (("parallax_d64", 64, True), ("softmax_d128", 128, False)):
        cm[name] = time_decode_point(plx, torch, dev, pool_k, pool_v, 128, 32768, d, "equal", seed=5, use_r=use_r,
                                     iters=iters)
    cm["speedup_parallax_d64_over_softmax_d128"] = cm["softmax_d128"]["us"] / cm["parallax_d64"]["us"]
    res["compute_matched"] = cm
    big = [p for p in res["sweep"] if p.get("bar_applies")]
    res["sweep_min_frac_of_spec_at_100MB_and_up"] = min(p["frac_of_spec"] for p in big) if big else None
    del pool_k, pool_v
    torch.cuda.empty_cache()
    return res


def run_sweep(args):
    """--sweep: the decode configurations as one JSON line."""
    import torch
    from parameterized_local_linear_plx_b200 import build
    build.build()
    from parameterized_local_linear_plx_b200 import plx
    dev = torch.device("cuda", 0)
    peaks, _ = load_peaks()
    print(json.dumps({"decode_configs": decode_configs(plx, args, dev, float(peaks.get("hbm_gbs", 6650.0)))}),
          flush=True)


def run_profile_small(args):
    """--profile-small: one call of each small case the ncu summaries in
    profiles/ capture (decode in its three plans, the projection in both
    forms), then exit; inputs larger than L2 but a few GB at most."""
    import torch
    from parameterized_local_linear_plx_b200 import build, inputs
    build.build()
    from parameterized_local_linear_plx_b200 import plx
    dev = torch.device("cuda", 0)
    # decode, balanced plan: B=1, context 32768, Hq=16, Hkv=8, d=128 (134 MB of KV)
    q, kc, vc, r, sl = inputs.decode_inputs(1, 16, 8, 32768, 128, seed=0, device=dev)
    plx.plx_decode(q, kc, vc, sl, r)
    del kc, vc
    # decode, chunked plan: B=64, context 4096 (1.07 GB of KV)
    q, kc, vc, r, sl = inputs.decode_inputs(64, 16, 8, 4096, 128, seed=0, device=dev)
    plx.plx_decode(q, kc, vc, sl, r)
    del kc, vc
    # decode, segment plan: B=1024, context 128, lengths uniform in [64, 128] (537 MB of KV allocated)
    q, kc, vc, r, sl = inputs.decode_inputs(1024, 16, 8, 128, 128, seed=0, seqlens="ragged", device=dev)
    plx.plx_decode(q, kc, vc, sl, r)
    del kc, vc
    # projection, prefill form: 2 x 4096 tokens, d_model 1024, W [6144, 1024]
    g = torch.Generator(device=dev).manual_seed(1)
    x = torch.randn(8192, 1024, generator=g, device=dev).bfloat16()
    w = (torch.randn(6144, 1024, generator=g, device=dev) / 32).bfloat16()
    plx.plx_qkvr_proj(x, w, 2, 4096, 16, 8, 128)
    # projection, decode form: 64 tokens appended into a [64, 8, 4096, 128] cache
    kc = torch.zeros(64, 8, 4096, 128, dtype=torch.bfloat16, device=dev)
    vc = torch.zeros_like(kc)
    s = torch.full((64,), 4000, dtype=torch.int32, device=dev)
    plx.plx_qkvr_proj_decode(x[:64].contiguous(), w, kc, vc, s, 16)
    torch.cuda.synchronize()
    st = plx.plx_check_device_status()
    if st != plx.PLX_OK:
        raise RuntimeError(f"device status: {plx.plx_status_string(st)}")
    print(json.dumps({"profile_small": "ok"}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["plx", "reference"], default="plx")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--small", action="store_true",
                    help="profiling-size workload: decode B=16, prefill B=2 (both still larger than L2)")
    ap.add_argument("--sweep", action="store_true", help="only the decode configurations (sweep, B=1/16, "
                    "compute-matched) as one JSON line")
    ap.add_argument("--no-decode-configs", action="store_true", help="leave the decode configurations out of the "
                    "bench line")
    ap.add_argument("--profile-small", action="store_true", help="one call of each small case the ncu summaries "
                    "capture (decode in its three plans, the projection in both forms), then exit")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.small:
        DEC["B"] = 16
        PRE["B"] = 2
    world, rank, local = dist_setup()
    if args.gpus != world and world > 1:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.sweep:
        return run_sweep(args)
    if args.profile_small:
        return run_profile_small(args)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        return run_gpu(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
