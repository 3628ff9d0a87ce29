#!/usr/bin/env python
"""Benchmark of the bifocal attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (``value``): bifocal prefill TFLOP/s at L = 131072 with Qwen3-8B attention heads
(Hq 32, Hkv 8, D 128), w_pretrained 32768 (G = 4), w0 4096, frequency interpolation,
counted as 2 * 2 * (L^2 / 2) * D * Hq FLOP per prefill. One step = one full prefill
(RoPE pass + fused attention) over inputs already resident in HBM (1.5 GB, larger than
L2). The same run also times: the attention kernel alone (roofline), the plain causal
RoPE comparator (overhead), the 200-step decode across the G = 4 -> 5 change (us/step and
GB/s vs HBM), the end-to-end call with host buffers, and the fp64 CPU oracle on a bounded
sample of the same workload (cpu_baseline). Multi-GPU runs are replicas (weak scaling):
each rank runs the same workload; value = all ranks' FLOPs / the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "bifocal prefill TFLOP/s at 128K (frac of BF16 peak); decode µs/step vs HBM"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of the dominant kernel,
# from one single-pass ncu capture of a full-size launch (L = 131072, the bench workload), keyed
# by the SHA-256 of the kernel's sources at capture time: when the sources no longer match, the
# kernel has changed since the counters were taken and traffic is null.
TRAFFIC = {
    "prefill_attention": {
        "bytes_per_launch": 4.99e9 + 1.07e9,
        "sources": ["common.cuh", "prefill_tc.cuh", "prefill_tc2.cuh", "rope_loads.cuh"],
        "sha256": "106d9b5065b65889cceba8fcd35e1efe2d8acb7fa1ffd87c2a35f5119e62651f",
    },
}


def measured_traffic(name):
    import hashlib
    t = TRAFFIC.get(name)
    if t is None:
        return None
    h = hashlib.sha256()
    try:
        for f in t["sources"]:
            with open(os.path.join(ROOT, "rope_context_extension_bifocal_b200", "csrc", f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    return t["bytes_per_launch"] if h.hexdigest() == t["sha256"] else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ distributed plumbing
class Dist:
    def __init__(self, want_pg: bool):
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False
        if want_pg and self.world > 1:
            import datetime

            import torch
            import torch.distributed as dist
            backend = "nccl" if torch.cuda.is_available() else "gloo"
            dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
            self.pg = True

    def barrier(self):
        if self.pg:
            import torch.distributed as dist
            dist.barrier()

    def max(self, x: float) -> float:
        if not self.pg:
            return x
        import torch
        import torch.distributed as dist
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            import torch.distributed as dist
            dist.destroy_process_group()


# ------------------------------------------------------------------ clocks sampler
class Clocks:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            cmd += ["-i", uuid if uuid.startswith("GPU-") else "GPU-" + uuid]
        except Exception:
            pass
        self.cmd = cmd

    def start(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, parts[3:7]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ timing helpers
class nvtx_range:
    """An NVTX range around one phase of the run (visible in a profiler's timeline); a no-op where
    NVTX is unavailable. Host-side markers only: nothing is added on the device."""

    def __init__(self, torch, name):
        self.torch, self.name, self.on = torch, name, False

    def __enter__(self):
        try:
            self.torch.cuda.nvtx.range_push(self.name)
            self.on = True
        except Exception:
            self.on = False
        return self

    def __exit__(self, *exc):
        if self.on:
            try:
                self.torch.cuda.nvtx.range_pop()
            except Exception:
                pass
        return False


def time_loop(fn, steps, warmup, dist, torch):
    """Device time of `steps` calls of fn (CUDA events on the current stream), max over ranks."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(steps):
        fn()
    e.record()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    return dist.max(s.elapsed_time(e))


def cpu_info():
    try:
        cores = len(os.sched_getaffinity(0))
    except Exception:
        cores = os.cpu_count() or 1
    threads = cores
    try:
        from threadpoolctl import threadpool_info
        ti = [x for x in threadpool_info() if x.get("user_api") == "blas"]
        if ti:
            threads = int(ti[0].get("num_threads", cores))
    except Exception:
        pass
    return cores, threads


def oracle_sample(q, k, v, w, rows, heads):
    """Time the fp64 oracle on (rows x heads) of the prefill workload; returns (seconds, counted FLOPs)."""
    import numpy as np

    import oracle.bifocal_ref as R
    g = w.hq // w.hkv
    t0 = time.perf_counter()
    for h in heads:
        qh = q[:, :, h:h + 1].float().double().numpy()
        kh = k[:, :, h // g:h // g + 1].float().double().numpy()
        vh = v[:, :, h // g:h // g + 1].float().double().numpy()
        R.bifocal_attention(qh, kh, vh, w.w0, w.w_pretrained, w.theta, w.mode, rows=np.asarray(rows))
    dt = time.perf_counter() - t0
    flops = sum(4.0 * w.head_dim * (r + 1) for r in rows) * len(heads)
    return dt, flops


def cpu_baseline_measure(q, k, v, w):
    """The fp64 oracle on a bounded sample of the prefill workload, on the host cores, with the
    rate it reached and, labelled as extrapolated, the time it would take for the 512-row-per-head
    sample of the parity tests and for the whole prefill (cost per row = its causal key count),
    plus the decode oracle's seconds per step at the decode workload's length."""
    import numpy as np

    import oracle.bifocal_ref as R
    import seeded_inputs as si
    rows512 = si.sample_rows(w.seed, w.L, w.w0, w.w_pretrained, 512)
    rows = rows512[::43]  # 12 rows spread over the sequence, both branches over all their keys
    dt, fl = oracle_sample(q, k, v, w, [int(r) for r in rows], list(range(w.hq)))
    keys = float(sum(int(r) + 1 for r in rows)) * w.hq
    rate = keys / dt
    out = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "kind": "oracle",
           "sample": f"query rows {', '.join(str(int(r)) for r in rows)} (every 43rd row of the 512-row parity "
                     f"sample) x all {w.hq} heads of the same workload, fp64 NumPy, {dt:.1f} s",
           "sample_s": dt, "rows_per_s": len(rows) * w.hq / dt, "causal_keys_per_s": rate,
           "extrapolated_512_row_sample_s": float(sum(int(r) + 1 for r in rows512)) * w.hq / rate,
           "extrapolated_full_prefill_s": w.L * (w.L + 1) / 2.0 * w.hq / rate}
    # decode: the oracle's step at the decode workload's length (cache 131000 + 1), one step timed
    dw = si.DECODE_128K
    stream = si.DecodeStream(dw)
    kp, vp = stream.cache_prefix()
    qd, kn, vn = stream.step()
    L = dw.prefix_len + 1
    kc = np.zeros((L, dw.hkv, dw.head_dim))
    vc = np.zeros((L, dw.hkv, dw.head_dim))
    kc[:L - 1] = kp.float().double().numpy()
    vc[:L - 1] = vp.float().double().numpy()
    kc[L - 1] = R.rope_keys_for_cache(kn[None].float().double().numpy(), dw.theta, start=L - 1)[0]
    vc[L - 1] = vn.float().double().numpy()
    t0 = time.perf_counter()
    R.bifocal_decode_reference(qd.float().double().numpy(), kc, vc, L, dw.w0, dw.w_pretrained, dw.theta, dw.mode)
    out["decode_s_per_step"] = time.perf_counter() - t0
    out["decode_note"] = f"bifocal_decode_reference at L = {L}, Hq {dw.hq}, Hkv {dw.hkv}, one step"
    return out


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    """The fp64 CPU oracle as the reference arm, on bounded samples of the same workload."""
    import seeded_inputs as si
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = si.qwen3_8b_128k(args.w0)
    q, k, v = si.prefill_inputs(w)
    rows = [w.L - 1]
    heads = list(range(8))
    times, flops = [], 0.0
    for i in range(args.warmup + args.steps):
        dt, fl = oracle_sample(q, k, v, w, rows, heads)
        if i >= args.warmup:
            times.append(dt)
            flops = fl
    ms = 1000.0 * statistics.mean(times)
    value = flops / (ms / 1000.0) / 1e12
    cores, threads = cpu_info()
    sample = f"query row {rows[0]} of query heads 0-7 per step (fp64 NumPy oracle, both RoPE branches over all keys)"
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w):
    G = max(1, -(-w.L // w.w_pretrained))  # for the record only; the library computes its own
    return {"workload": w.name, "batch": 1, "L": w.L, "hq": w.hq, "hkv": w.hkv, "head_dim": w.head_dim, "w0": w.w0,
            "w_pretrained": w.w_pretrained, "G": G, "mode": w.mode, "theta": w.theta, "seed": w.seed,
            "l2": "inputs larger than L2 (q+k+v 1.5 GB bf16)", "parallelism": "replicas"}


# ------------------------------------------------------------------ our arm
def roof(bound, achieved, peak, unit, kernel, scope, peak_kind, **extra):
    """A roofline entry for a secondary line: achieved / peak, what was timed, against which peak."""
    r = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
         "kernel": kernel, "scope": scope, "traffic": None,
         "peak_kind": f"{peak_kind} {'bf16 dense burst' if unit == 'TFLOP/s' else 'HBM copy'}"}
    r.update(extra)
    return r


def run_ours(args):
    import torch

    import rope_context_extension_bifocal_b200 as bfl
    import seeded_inputs as si

    dist = Dist(want_pg=True)
    torch.cuda.set_device(dist.local)
    dev = torch.device("cuda", dist.local)
    peaks, peak_kind = load_peaks()
    launches = 0

    w = si.qwen3_8b_128k(args.w0)
    q_h, k_h, v_h = si.prefill_inputs(w)
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    params = bfl.make_params(w.hq, w.hkv, w.head_dim, w.w0, w.w_pretrained, w.theta, w.mode)
    ws = torch.empty(bfl.prefill_workspace_size(bfl.DTYPE_BF16, 1, w.L, params), dtype=torch.uint8, device=dev)
    out = torch.empty(1, w.L, w.hq, w.head_dim, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(1, w.hq, w.L, dtype=torch.float32, device=dev)
    flops = w.causal_flops

    def step_rope():
        bfl.bifocal_prefill_rope(q, k, v, params, ws)

    def step_attn():
        bfl.bifocal_prefill_attention(v, params, ws, out, lse)

    # ---- headline: K full prefills, per-kernel events inside the timed region
    for _ in range(args.warmup):
        step_rope()
        step_attn()
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = Clocks(dist.local)
    clocks.start()
    time.sleep(0.3)
    with nvtx_range(torch, "headline: 128K prefill steps"):
        for i in range(args.steps):
            ev[i][0].record()
            step_rope()
            ev[i][1].record()
            step_attn()
            ev[i][2].record()
            launches += 2
    torch.cuda.synchronize()
    clk = clocks.stop()
    dist.barrier()
    total_ms = dist.max(ev[0][0].elapsed_time(ev[-1][2]))
    attn_ms = dist.max(statistics.mean(e[1].elapsed_time(e[2]) for e in ev))
    rope_ms = dist.max(statistics.mean(e[0].elapsed_time(e[1]) for e in ev))
    ms_per_step = total_ms / args.steps
    value = flops * dist.world / (ms_per_step / 1e3) / 1e12
    attn_tflops = flops / (attn_ms / 1e3) / 1e12
    peak_t = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    roofline = {"bound": "tensor", "achieved": attn_tflops, "peak": peak_t, "unit": "TFLOP/s",
                "frac": attn_tflops / peak_t, "frac_of_sustained_peak": attn_tflops / peak_sus,
                "sustained_peak": peak_sus, "traffic": measured_traffic("prefill_attention"),
                "traffic_unit": "bytes per launch (DRAM read + write, ncu)", "kernel": "bifocal attention (prefill)",
                "peak_kind": f"{peak_kind} bf16 dense burst", "kernel_ms": attn_ms, "rope_pass_ms": rope_ms}

    # ---- the fused-load kernel (RoPE and correction inside the tile loads, no workspace): A/B
    fused = None
    if not args.no_fused:
        pf = bfl.make_params(w.hq, w.hkv, w.head_dim, w.w0, w.w_pretrained, w.theta, w.mode, None,
                             bfl.FLAG_FUSED_ROPE)

        def step_fused():
            bfl._prefill("bifocal_prefill", q, k, v, pf, True, False, out, ws, None)

        n_f = max(3, args.steps)
        f_ms = time_loop(step_fused, n_f, 1, dist, torch) / n_f
        f_t = flops / (f_ms / 1e3) / 1e12
        fused = {"ms": f_ms, "tflops": f_t, "frac_of_peak": f_t / peak_t, "steps": n_f,
                 "vs_rope_pass_step": ms_per_step / f_ms,
                 "note": "bifocal_prefill with BF_FLAG_FUSED_ROPE: one launch, raw q/k tiles rotated in shared "
                         "memory, empty workspace (the headline step is RoPE pass + attention)"}

    # ---- plain comparator (same shapes, original RoPE only)
    def step_plain():
        bfl.rope_causal_prefill(q, k, v, theta=w.theta, out=out, workspace=ws)

    plain_ms = time_loop(step_plain, max(2, args.steps // 2), 1, dist, torch) / max(2, args.steps // 2)
    overhead_prefill = ms_per_step / plain_ms - 1.0

    # ---- w0 sweep of the 128K config (short)
    sweep = {}
    if not args.no_sweep:
        for w0 in si.QWEN3_8B_128K_W0:
            p2 = bfl.make_params(w.hq, w.hkv, w.head_dim, w0, w.w_pretrained, w.theta, w.mode)

            # the headline's step count, with the attention kernel timed on its own as well
            bfl.bifocal_prefill_rope(q, k, v, p2, ws)
            bfl.bifocal_prefill_attention(v, p2, ws, out, lse)
            torch.cuda.synchronize()
            dist.barrier()
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
            for e3 in evs:
                e3[0].record()
                bfl.bifocal_prefill_rope(q, k, v, p2, ws)
                e3[1].record()
                bfl.bifocal_prefill_attention(v, p2, ws, out, lse)
                e3[2].record()
            torch.cuda.synchronize()
            dist.barrier()
            ms = dist.max(evs[0][0].elapsed_time(evs[-1][2])) / args.steps
            k_ms = dist.max(statistics.mean(e3[1].elapsed_time(e3[2]) for e3 in evs))
            k_t = flops / (k_ms / 1e3) / 1e12
            sweep[str(w0)] = {"ms": ms, "tflops": flops / (ms / 1e3) / 1e12, "steps": args.steps,
                              "roofline": roof("tensor", k_t, peak_t, "TFLOP/s", "bifocal attention (prefill)",
                                               "attention kernel alone", peak_kind, kernel_ms=k_ms)}

    # ---- end to end through the public call with host buffers
    e2e = None
    if not args.no_e2e:
        qp, kp, vp = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()

        def step_e2e():
            q.copy_(qp, non_blocking=True)
            k.copy_(kp, non_blocking=True)
            v.copy_(vp, non_blocking=True)
            bfl.bifocal_prefill(q, k, v, w0=w.w0, w_pretrained=w.w_pretrained, theta=w.theta, mode=w.mode, out=out,
                                workspace=ws)
            out_h.copy_(out, non_blocking=True)
            lse_h.copy_(lse, non_blocking=True)

        n_e2e = max(2, args.steps // 2)
        e2e_ms = time_loop(step_e2e, n_e2e, 1, dist, torch) / n_e2e
        h2d = sum(t.numel() * t.element_size() for t in (q, k, v))
        d2h = out.numel() * out.element_size() + lse.numel() * lse.element_size()
        e2e = {"value": flops * dist.world / (e2e_ms / 1e3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
        del qp, kp, vp, out_h, lse_h

    # ---- chunked prefill over a cache: a 4096-token chunk after 126976 cached tokens
    chunk = None
    if not args.no_chunk:
        C = 4096
        P0 = w.L - C
        kc_all = torch.empty(w.L, w.hkv, w.head_dim, dtype=torch.bfloat16, device=dev)
        vc_all = torch.empty_like(kc_all)
        bfl.bifocal_prefill_rope(q, k, v, params, ws, kcache=kc_all, vcache=vc_all)  # original-RoPE keys of all rows
        wsc = torch.empty(bfl.prefill_chunk_workspace_size(P0, C, params), dtype=torch.uint8, device=dev)
        qc, kc_, vc_ = q[0, P0:], k[0, P0:], v[0, P0:]
        outc = torch.empty(C, w.hq, w.head_dim, dtype=torch.bfloat16, device=dev)

        def step_chunk(flags=0):
            bfl.bifocal_prefill_chunk(qc, kc_, vc_, kc_all, vc_all, P0, w0=w.w0, w_pretrained=w.w_pretrained,
                                      theta=w.theta, mode=w.mode, want_lse=False, out=outc, workspace=wsc,
                                      flags=flags)

        n_chunk = max(3, args.steps)
        chunk_ms = time_loop(step_chunk, n_chunk, 1, dist, torch) / n_chunk
        chunk_flops = 4.0 * w.head_dim * w.hq * (C * P0 + C * (C + 1) / 2)
        chunk_tflops = chunk_flops / (chunk_ms / 1e3) / 1e12
        fchunk_ms = time_loop(lambda: step_chunk(bfl.FLAG_FUSED_ROPE), n_chunk, 1, dist, torch) / n_chunk
        fchunk_tflops = chunk_flops / (fchunk_ms / 1e3) / 1e12
        pfc = bfl.make_params(w.hq, w.hkv, w.head_dim, w.w0, w.w_pretrained, w.theta, w.mode, None,
                              bfl.FLAG_FUSED_ROPE)
        chunk = {"workload": f"qwen3_8b_chunk_after_{P0}_cached_C{C}_w{w.w0}", "P0": P0, "C": C,
                 "G": bfl.bifocal_factor(w.L, w.w_pretrained), "ms": chunk_ms, "tflops": chunk_tflops,
                 "frac_of_peak": chunk_tflops / peak_t, "workspace_bytes": wsc.numel(),
                 "roofline": roof("tensor", chunk_tflops, peak_t, "TFLOP/s", "chunked prefill",
                                  "whole call (re-phase + RoPE pass + attention)", peak_kind),
                 "note": "one call = cache re-phase pass + chunk RoPE pass + attention (3 launches); "
                         "FLOPs counted over the chunk's causal pairs",
                 "fused": {"ms": fchunk_ms, "tflops": fchunk_tflops, "frac_of_peak": fchunk_tflops / peak_t,
                           "workspace_bytes": bfl.prefill_chunk_workspace_size(P0, C, pfc),
                           "note": "BF_FLAG_FUSED_ROPE: chunk rows written to the cache, then one attention "
                                   "launch that re-phases cached keys in its tile loads (2 launches)"}}
        del kc_all, vc_all, wsc, outc

    # ---- sliding-window prefill (the local layers of a hybrid model), window = w0
    window = None
    if not args.no_window:
        pw = bfl.make_params(w.hq, w.hkv, w.head_dim, w.w0, w.w_pretrained, w.theta, w.mode, None, bfl.FLAG_WINDOW)

        def step_window():
            bfl.bifocal_prefill_rope(q, k, v, pw, ws)
            bfl.bifocal_prefill_attention(v, pw, ws, out, lse)

        n_win = max(3, args.steps)
        win_ms = time_loop(step_window, n_win, 1, dist, torch) / n_win
        Wn = min(w.w0, w.L)
        pairs = Wn * (Wn + 1) / 2 + (w.L - Wn) * Wn  # causal pairs with i - j < w0
        win_tflops = 4.0 * w.head_dim * w.hq * pairs / (win_ms / 1e3) / 1e12
        window = {"workload": f"qwen3_8b_L{w.L}_window{Wn}", "window": Wn, "ms": win_ms, "tflops": win_tflops,
                  "frac_of_peak": win_tflops / peak_t,
                  "roofline": roof("tensor", win_tflops, peak_t, "TFLOP/s", "sliding-window prefill",
                                   "whole step (RoPE pass + attention)", peak_kind),
                  "note": "BF_FLAG_WINDOW prefill (RoPE pass + attention); FLOPs counted over the window's pairs"}

    # ---- decode: 200 steps across the G = 4 -> 5 change
    decode = None
    if not args.no_decode:
        del ws
        torch.cuda.empty_cache()
        with nvtx_range(torch, "decode sessions"):
            decode = run_decode(args, torch, bfl, si, dev, peaks, peak_kind)

    paged = None
    if not args.no_paged:
        torch.cuda.empty_cache()
        with nvtx_range(torch, "batched paged decode"):
            paged = run_paged(args, torch, bfl, si, dev, peaks, peak_kind)

    chunk_paged = None
    if not args.no_chunk_paged:
        torch.cuda.empty_cache()
        with nvtx_range(torch, "batched paged chunked prefill"):
            chunk_paged = run_chunk_paged(args, torch, bfl, si, dev, peak_t, peak_kind, dist)

    # ---- CPU baseline: the oracle on a bounded sample, rank 0, N = 1 only
    cpu = None
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        cores, threads = cpu_info()
        cpu = cpu_baseline_measure(q_h, k_h, v_h, w)
        cpu["cores"] = threads
        cpu["sample"] += f"; host has {cores} usable cores"

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": dist.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "precision": {"inputs": "bf16", "qk_operands": "f16", "pv_operands": "bf16", "accumulate": "f32"},
        "data": "synthetic: q/k/v iid N(0,1) bf16, torch CPU generator seed 3 (Qwen3-8B attention shapes)",
        "config": workload_config(w),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clk,
        "gpu_launches": launches,
        "overhead_vs_plain": {"prefill": overhead_prefill, "prefill_plain_ms": plain_ms,
                              "decode": decode["overhead_vs_plain"] if decode else None},
        "w0_sweep": sweep,
        "fused_prefill": fused,
        "decode": decode,
        "chunked_prefill": chunk,
        "window_prefill": window,
        "paged_decode": paged,
        "chunk_paged": chunk_paged,
        "build": bfl.build_info(),
    }
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    dist.close()
    return 0


def run_decode(args, torch, bfl, si, dev, peaks, peak_kind):
    w = si.DECODE_128K
    stream = si.DecodeStream(w)
    kp, vp = stream.cache_prefix()
    kcache = torch.zeros(w.capacity, w.hkv, w.head_dim, dtype=torch.bfloat16, device=dev)
    vcache = torch.zeros_like(kcache)
    kcache[:w.prefix_len] = kp.to(dev)
    vcache[:w.prefix_len] = vp.to(dev)
    del kp, vp
    steps = [tuple(t.to(dev) for t in stream.step()) for _ in range(args.decode_steps)]
    params = bfl.make_params(w.hq, w.hkv, w.head_dim, w.w0, w.w_pretrained, w.theta, w.mode)
    ws = torch.empty(bfl.decode_workspace_size(w.capacity, params), dtype=torch.uint8, device=dev)
    out = torch.empty(w.hq, w.head_dim, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(w.hq, dtype=torch.float32, device=dev)

    def session(fn):
        for t in range(min(args.warmup, len(steps))):  # warm-up rewrites the same rows the session writes
            fn(t)
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in steps]
        for t in range(len(steps)):
            ev[t][0].record()
            fn(t)
            ev[t][1].record()
        torch.cuda.synchronize()
        return [a.elapsed_time(b) * 1e3 for a, b in ev]  # us

    def bif(t):
        q, kn, vn = steps[t]
        bfl.bifocal_decode(q, kn, vn, kcache, vcache, w.prefix_len + t + 1, w0=w.w0, w_pretrained=w.w_pretrained,
                           theta=w.theta, mode=w.mode, out=out, workspace=ws)

    def plain(t):
        q, kn, vn = steps[t]
        bfl.rope_causal_decode(q, kn, vn, kcache, vcache, w.prefix_len + t + 1, theta=w.theta, out=out,
                               workspace=ws)

    def window(t):  # the local layers of a hybrid model: keys L - w0 .. L - 1 only
        q, kn, vn = steps[t]
        bfl.bifocal_decode(q, kn, vn, kcache, vcache, w.prefix_len + t + 1, w0=w.w0, w_pretrained=w.w_pretrained,
                           theta=w.theta, mode=w.mode, flags=bfl.FLAG_WINDOW, out=out, workspace=ws)

    us = session(bif)
    us_plain = session(plain)
    us_window = session(window)
    gbs = [w.cache_bytes(w.prefix_len + t + 1) / (u * 1e-6) / 1e9 for t, u in enumerate(us)]
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    med = statistics.median(us)
    med_gbs = statistics.median(gbs)
    srt = sorted(us)
    return {
        "workload": w.name, "steps": len(us), "us_mean": statistics.mean(us), "us_median": med,
        "us_p95": srt[min(len(srt) - 1, int(0.95 * len(srt)))], "us_min": srt[0],
        "gbs_median": med_gbs, "us_steps_70_75": us[70:76], "G_steps_70_75": [
            bfl.bifocal_factor(w.prefix_len + t + 1, w.w_pretrained) for t in range(70, 76)],
        "overhead_vs_plain": statistics.median(us) / statistics.median(us_plain) - 1.0,
        "plain_us_median": statistics.median(us_plain),
        "roofline": {"bound": "hbm", "achieved": med_gbs, "peak": hbm, "unit": "GB/s", "frac": med_gbs / hbm,
                     "traffic": None, "kernel": "decode step (append + split-KV partial + combine)",
                     "peak_kind": f"{peak_kind} HBM copy",
                     "bytes_per_step_at_131072": w.cache_bytes(131072)},
        "gpu_launches": 3 * len(us),
        "window": {"w0": w.w0, "us_median": statistics.median(us_window),
                   "bytes_per_step": 4 * w.hkv * w.head_dim * w.w0,
                   "note": "sliding-window decode (BF_FLAG_WINDOW): reads the last w0 cached tokens"},
    }


def run_paged(args, torch, bfl, si, dev, peaks, peak_kind):
    """Batched decode over a paged cache: 8 sequences of ~16K tokens (Qwen3-8B heads), page 64."""
    B, page, hq, hkv, D, w0, wp = 8, 64, 32, 8, 128, 4096, 4096
    lens = [16384 + 97 * b for b in range(B)]  # G = 4 or 5 per sequence
    max_len = max(lens) + 1
    max_pages = (max_len + page - 1) // page
    g = si.generator(404)
    pool_pages = B * max_pages
    table = torch.randperm(pool_pages, generator=g).to(torch.int32).reshape(B, max_pages).to(dev)
    kpool = torch.randn(pool_pages * page, hkv, D, device=dev).to(torch.bfloat16)
    vpool = torch.randn(pool_pages * page, hkv, D, device=dev).to(torch.bfloat16)
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    q = torch.randn(B, hq, D, device=dev).to(torch.bfloat16)
    kn = torch.randn(B, hkv, D, device=dev).to(torch.bfloat16)
    vn = torch.randn(B, hkv, D, device=dev).to(torch.bfloat16)
    prm = bfl.make_params(hq, hkv, D, w0, wp, 1e6)
    ws = torch.empty(bfl.decode_paged_workspace_size(B, max_len, prm), dtype=torch.uint8, device=dev)
    out = torch.empty(B, hq, D, dtype=torch.bfloat16, device=dev)

    def step():
        bfl.bifocal_decode_paged(q, kn, vn, kpool, vpool, page, table, seq, max_len, w0=w0, w_pretrained=wp,
                                 theta=1e6, want_lse=False, out=out, workspace=ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(30)]
    for a, b_ in ev:
        a.record()
        step()
        b_.record()
    torch.cuda.synchronize()
    us = statistics.median(a.elapsed_time(b_) * 1e3 for a, b_ in ev)
    nbytes = sum(4 * hkv * D * L for L in lens)
    gbs = nbytes / (us * 1e-6) / 1e9
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    return {"workload": f"qwen3_8b_paged_decode_B{B}_L{lens[0]}-{lens[-1]}_page{page}", "us_median": us,
            "gbs": gbs, "frac_of_hbm": gbs / hbm, "bytes_per_step": nbytes,
            "roofline": roof("hbm", gbs, hbm, "GB/s", "batched paged decode",
                             "whole step (append + split-KV partial + combine)", peak_kind),
            "G": [bfl.bifocal_factor(L, wp) for L in lens]}


def run_chunk_paged(args, torch, bfl, si, dev, peak_t, peak_kind, dist):
    """Chunked prefill for a batch over a paged cache: 8 sequences of 16K-23K cached tokens, chunks of
    512-2048 tokens (Qwen3-8B heads), page 64, G 5-7 per sequence."""
    B, page, hq, hkv, D, w0, wp = 8, 64, 32, 8, 128, 4096, 4096
    cached = [16384 + 1024 * b for b in range(B)]
    chunks = [2048, 1024, 2048, 512, 2048, 1536, 2048, 768]
    lens = [p0 + c for p0, c in zip(cached, chunks)]
    max_pages = (max(lens) + page - 1) // page
    g = si.generator(505)
    pool_pages = B * max_pages
    table = torch.randperm(pool_pages, generator=g).to(torch.int32).reshape(B, max_pages).to(dev)
    kpool = torch.randn(pool_pages * page, hkv, D, device=dev).to(torch.bfloat16)
    vpool = torch.randn(pool_pages * page, hkv, D, device=dev).to(torch.bfloat16)
    T = sum(chunks)
    q = torch.randn(T, hq, D, device=dev).to(torch.bfloat16)
    k = torch.randn(T, hkv, D, device=dev).to(torch.bfloat16)
    v = torch.randn(T, hkv, D, device=dev).to(torch.bfloat16)
    out = torch.empty(T, hq, D, dtype=torch.bfloat16, device=dev)

    def step():
        bfl.bifocal_prefill_chunk_paged(q, k, v, chunks, cached, kpool, vpool, page, table, w0=w0, w_pretrained=wp,
                                        theta=1e6, want_lse=False, out=out)

    n = max(3, args.steps)
    ms = time_loop(step, n, 1, dist, torch) / n
    flops = sum(4.0 * D * hq * (c * p0 + c * (c + 1) / 2) for p0, c in zip(cached, chunks))
    tflops = flops / (ms / 1e3) / 1e12
    return {"workload": f"qwen3_8b_paged_chunks_B{B}_P0_{cached[0]}-{cached[-1]}_C{min(chunks)}-{max(chunks)}_page{page}",
            "ms": ms, "tflops": tflops, "frac_of_peak": tflops / peak_t, "workspace_bytes": 0,
            "roofline": roof("tensor", tflops, peak_t, "TFLOP/s", "batched paged chunked prefill",
                             "whole call (pool writes + fused attention)", peak_kind),
            "G": [bfl.bifocal_factor(L, wp) for L in lens],
            "note": "bifocal_prefill_chunk_paged: chunk keys/values into their pages, then one fused attention launch "
                    "over all chunks (2 launches); FLOPs counted over each chunk's causal pairs"}


def run_case(args):
    """One named case, `--reps` timed calls after an untimed one, on cuda:0 (for ncu captures and
    quick timing). Inputs follow the seeded recipe (iid N(0,1) bf16)."""
    import torch

    import rope_context_extension_bifocal_b200 as bfl
    import seeded_inputs as si

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    a = args
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if a.case.startswith("prefill"):
        q, k, v = (t.to(dev) for t in si.random_qkv(3, 1, a.L, a.hq, a.hkv, a.D, "bf16"))
        p = bfl.make_params(a.hq, a.hkv, a.D, a.w0, a.w_pretrained, a.theta, a.mode, None, a.flags)
        ws = torch.empty(bfl.prefill_workspace_size(bfl.DTYPE_BF16, 1, a.L, p), dtype=torch.uint8, device=dev)
        out = torch.empty(1, a.L, a.hq, a.D, dtype=torch.bfloat16, device=dev)

        def call():
            if a.case == "prefill":
                bfl.bifocal_prefill(q, k, v, w0=a.w0, w_pretrained=a.w_pretrained, theta=a.theta, mode=a.mode,
                                    flags=a.flags, out=out, workspace=ws)
            else:
                bfl.rope_causal_prefill(q, k, v, theta=a.theta, out=out, workspace=ws)
        work, unit = 4.0 * a.L * a.L / 2 * a.D * a.hq, "TFLOP/s"
    else:
        cap = a.L + 16
        kc = torch.randn(cap, a.hkv, a.D, device=dev).to(torch.bfloat16)
        vc = torch.randn(cap, a.hkv, a.D, device=dev).to(torch.bfloat16)
        q = torch.randn(a.hq, a.D, device=dev).to(torch.bfloat16)
        kn = torch.randn(a.hkv, a.D, device=dev).to(torch.bfloat16)
        vn = torch.randn(a.hkv, a.D, device=dev).to(torch.bfloat16)
        p = bfl.make_params(a.hq, a.hkv, a.D, a.w0, a.w_pretrained, a.theta, a.mode, None, a.flags)
        ws = torch.empty(bfl.decode_workspace_size(cap, p), dtype=torch.uint8, device=dev)
        out = torch.empty(a.hq, a.D, dtype=torch.bfloat16, device=dev)

        def call():
            if a.case == "decode":
                bfl.bifocal_decode(q, kn, vn, kc, vc, a.L, w0=a.w0, w_pretrained=a.w_pretrained, theta=a.theta,
                                   mode=a.mode, flags=a.flags, out=out, workspace=ws)
            else:
                bfl.rope_causal_decode(q, kn, vn, kc, vc, a.L, theta=a.theta, out=out, workspace=ws)
        work, unit = 2.0 * 2 * a.L * a.hkv * a.D, "GB/s"  # cache bytes read
    call()
    torch.cuda.synchronize()
    s.record()
    for _ in range(a.reps):
        call()
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / a.reps
    word = bfl.device_status_word()
    rate = work / (ms / 1e3) / (1e12 if unit == "TFLOP/s" else 1e9)
    print(json.dumps({"case": a.case, "L": a.L, "hq": a.hq, "hkv": a.hkv, "D": a.D, "w0": a.w0,
                      "w_pretrained": a.w_pretrained, "ms_per_call": ms, "rate": rate, "unit": unit,
                      "status_word": word}), flush=True)
    return 0 if word == 0 else 1


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--w0", type=int, default=4096)
    ap.add_argument("--decode-steps", type=int, default=200)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-chunk", action="store_true")
    ap.add_argument("--no-chunk-paged", action="store_true")
    ap.add_argument("--no-window", action="store_true")
    ap.add_argument("--no-paged", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-fused", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    g = ap.add_argument_group("single case (--case): one kernel path timed alone, e.g. for an ncu capture")
    g.add_argument("--case", choices=["prefill", "prefill_plain", "decode", "decode_plain"])
    g.add_argument("--L", type=int, default=32768)
    g.add_argument("--hq", type=int, default=32)
    g.add_argument("--hkv", type=int, default=8)
    g.add_argument("--D", type=int, default=128)
    g.add_argument("--w-pretrained", type=int, default=8192)
    g.add_argument("--theta", type=float, default=1e6)
    g.add_argument("--mode", default="freq_interp", choices=["freq_interp", "pos_alias"])
    g.add_argument("--reps", type=int, default=3)
    g.add_argument("--flags", type=int, default=0, help="BF_FLAG_* bits")
    args = ap.parse_args()
    if args.case:
        return run_case(args)
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
