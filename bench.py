#!/usr/bin/env python
"""Benchmark of the Gemma 3 5:1 block attention on B200.

One step = one 5:1 block (five local layers, one global layer) of prefill on
the 27B-shaped 8K-token workload, through g3attn_prefill.  The same run also
times one decode block step on the 64-sequence, 4K-128K-token workload (six
g3attn_decode calls) and reports it under "decode".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl g3attn|reference]

Under torchrun each rank runs the whole workload on its own GPU (the units
are independent, no data-path collective): weak scaling, value = all ranks'
FLOPs / the slowest rank's time.  `--impl reference` times the float64 CPU
oracle on bounded samples of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import inputs  # noqa: E402
from global_gqa_b200 import metrics, shard  # noqa: E402

METRIC = "prefill attn TFLOP/s (unmasked FLOPs, 5:1 block) & decode KV GB/s, 1 B200"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_PATH = os.path.join(ROOT, "profiles", "prefill_attention_traffic.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# B200 data-sheet figures (dense bf16, HBM3e), reported beside the measured peaks.
NOMINAL = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0}


def fractions(value: float, measured: float, nominal: float) -> dict:
    """A block-level rate as a fraction of the measured peak and of the data-sheet peak."""
    return {"of_measured": value / measured if measured else None, "of_nominal": value / nominal}


def peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK), "fallback"


DECODE_TRAFFIC_PATH = os.path.join(ROOT, "profiles", "decode_split_traffic.json")


# The library's per-kernel trace brackets each launch with CUDA events; an event
# between two kernels keeps the next launch from starting until the previous one
# has drained (~5.7 us per kernel boundary, ~4 % of a traced 8K block step).  So
# the timed loops carry the trace on every TRACE_EVERY-th step only (the first
# one included: two of the default 20 steps), and a kernel's average duration
# comes from those steps' launches.
TRACE_EVERY = 10


def n_traced(steps: int) -> int:
    """Timed steps that carry the trace: 0, TRACE_EVERY, 2*TRACE_EVERY, ..."""
    return (steps + TRACE_EVERY - 1) // TRACE_EVERY


def launches_in_timed_region(trace: dict, steps: int, untraced_per_step: int = 0) -> int:
    """All launches of the timed loop: the traced steps' launches per step times the steps, plus
    the launches the library does not trace (each prefill call's device-error reset kernel)."""
    per_step = sum(v[0] for v in trace.values()) // max(n_traced(steps), 1)
    return (per_step + untraced_per_step) * steps


def kernel_source_hash(files=("prefill.cu", "sm100_ptx.cuh", "tmem_wide.cuh", "g3_internal.h")) -> str:
    """Hash of the sources a committed ncu traffic figure was taken on."""
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "global_gqa_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


# ------------------------------------------------------------- clock sampler
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, torch_dev_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            h = None
            try:
                import torch
                uuid = str(torch.cuda.get_device_properties(torch_dev_index).uuid)
                h = nv.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
                idx = int(vis.split(",")[torch_dev_index]) if vis and vis.split(",")[0].isdigit() else torch_dev_index
                h = nv.nvmlDeviceGetHandleByIndex(idx)
            self._h = h
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        except Exception:
            self._h = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)  # the 20-step block region lasts ~32 ms

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if self._h is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def block_config(cfg, world: int, block_flops: float) -> dict:
    """The `config` object of a block-prefill line; both arms print this one."""
    return {"workload": cfg.name, "batch": cfg.B, "seq_len": cfg.S, "q_heads": cfg.Hq, "kv_heads": cfg.Hkv,
            "head_dim": cfg.D, "block": "5 local (W=1024, base 1e4) + 1 global (base 1e6, interp 8)",
            "unmasked_flops_per_step": block_flops,
            "l2": "inputs larger than L2: each layer reads 128 MiB of q/k/v and writes 64 MiB",
            "parallelism": f"independent replicas x{world}"}


# ------------------------------------------------------- multi-rank helpers
def max_over_ranks(value: float, device) -> float:
    """The largest of every rank's value (the slowest rank's time)."""
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist = torch.distributed
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank_step: float, steps: int, world: int, ms_max: float) -> float:
    """Units per second of the whole job: every rank does the same work."""
    return units_per_rank_step * steps * world / (ms_max * 1e-3)


# ------------------------------------------------------------ CPU baselines
def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


_ORACLE_INPUTS = {}


def oracle_prefill_sample(cfg, budget_s: float, seed: int = 0):
    """Time the oracle on sampled query rows of every layer of the block.

    Returns (flops, seconds, n_rows).  Rows come from a seeded permutation and
    are processed in groups of 64 until the time budget is spent (at least one
    group per layer).
    """
    from oracle import attention as O
    blk = cfg.block()
    rng = np.random.default_rng(seed)
    flops, secs, nrows = 0.0, 0.0, 0
    key = (cfg.name, len(blk))
    if key not in _ORACLE_INPUTS:
        _ORACLE_INPUTS[key] = [inputs.config_layer_inputs(cfg, li) for li in range(len(blk))]
    xs = _ORACLE_INPUTS[key]
    order = rng.permutation(cfg.S)
    g = 0
    while True:
        for li, L in enumerate(blk):
            rows = np.sort(order[(g * 64) % cfg.S:(g * 64) % cfg.S + 64])
            x = xs[li]
            lo, hi = metrics.row_intervals(cfg.S, L.kind, L.window)
            t0 = time.perf_counter()
            O.prefill_rows(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], L.kind,
                           L.window, L.rope_base, L.interp, x["spans"], rows=rows)
            secs += time.perf_counter() - t0
            flops += 4.0 * cfg.D * cfg.Hq * cfg.B * float(np.sum(hi[rows] - lo[rows] + 1))
            nrows += rows.size
        g += 1
        if secs >= budget_s:
            return flops, secs, nrows


def decode_traffic_per_launch(alg_bytes_per_launch: float):
    """DRAM bytes per decode_split launch: the committed capture of a smaller
    decode (8 sequences of 16K-32K tokens, larger than L2) scaled by algorithmic
    KV bytes, while the decode sources are the ones it was taken on."""
    try:
        with open(DECODE_TRAFFIC_PATH) as f:
            tr = json.load(f)
        if tr.get("source_hash") == kernel_source_hash(("decode.cu", "sm100_ptx.cuh", "g3_internal.h")):
            return tr["bytes_per_algorithmic_byte"] * alg_bytes_per_launch
    except (OSError, ValueError, KeyError):
        pass
    return None


def oracle_extras_baselines(line: dict, budget_s: float) -> None:
    """The oracles of the backward, of decode and of the soft tokens, timed as
    they stand on bounded samples of the same workloads (rank 0, N = 1)."""
    from oracle import backward as BW
    from oracle import projector as PJ
    cfg = inputs.BLOCK_8K
    if line.get("backward"):
        L = cfg.block()[0]
        S1 = 2048  # the oracle's cost grows as S^2: the first 2048 tokens of the layer
        x = inputs.prefill_backward_inputs(cfg.B, S1, cfg.Hq, cfg.Hkv, cfg.D, seed=cfg.seed, layer=0)
        G = cfg.Hq // cfg.Hkv
        t0 = time.perf_counter()
        BW.prefill_backward(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], L.kind, L.window,
                            L.rope_base, L.interp, x["dout"], None, kv_heads=[0])
        secs = time.perf_counter() - t0
        flops = 2.5 * metrics.layer_flops(cfg.B, S1, cfg.Hq, cfg.D, L.kind, L.window) * G / cfg.Hq
        line["backward"]["cpu_baseline"] = {
            "value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "seconds": secs, "sample": f"gradients of kv head 0 and its {G} query heads over the first {S1} tokens "
                                       f"of a local layer (W={L.window}) of {cfg.name} (algorithmic FLOPs), "
                                       f"float64 numpy"}
    if line.get("decode"):
        # One local (ring) and the global layer of the first sequences of the
        # 64-sequence batch, until about half the budget is spent.
        from oracle import attention as OA
        dc = inputs.DECODE_B64
        blk = dc.block()
        lens = inputs.decode_lengths(dc.B, dc.len_lo, dc.len_hi, dc.seed)
        nbytes, secs, n_seq = 0, 0.0, 0
        for b in range(dc.B):
            for li in (0, len(blk) - 1):
                L = blk[li]
                Lb = int(lens[b])
                n_hist = (Lb - 1) if L.kind == 1 else min(Lb, L.window) - 1
                hist = inputs.cache_history(n_hist, dc.Hkv, dc.D, seed=dc.seed, layer=li, batch=b)
                st = inputs.decode_step_inputs(1, dc.Hq, dc.Hkv, dc.D, seed=dc.seed, layer=li)
                t0 = time.perf_counter()
                OA.decode(st["q"], st["k_new"], st["v_new"], st["q_gamma"], st["k_gamma"], np.array([Lb]),
                          [hist["k"]], [hist["v"]], np.array([Lb - 1 - n_hist]), L.kind, L.window, L.rope_base,
                          L.interp)
                secs += time.perf_counter() - t0
                nbytes += metrics.decode_kv_bytes([Lb], dc.Hkv, dc.D, L.kind, L.window)
            n_seq += 1
            if secs > budget_s / 2:
                break
        line["decode"]["cpu_baseline"] = {
            "value": nbytes / secs / 1e9, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
            "seconds": secs, "sample": f"the first {n_seq} of the {dc.B} sequences of {dc.name}, one ring layer "
                                       f"and the global layer each (KV bytes counted as the GPU metric counts "
                                       f"them), float64 numpy"}
    if line.get("soft_tokens"):
        Bi, gh, F = 8, 64, 1152
        px = np.random.default_rng(17).standard_normal((Bi, gh * gh, F)).astype(np.float32)
        gam = np.ones(F)
        t0 = time.perf_counter()
        PJ.soft_tokens(px, gam, gh, gh, 4)
        secs = time.perf_counter() - t0
        nbytes = (Bi * gh * gh * F + Bi * (gh // 4) ** 2 * F) * 2 + F * 4
        line["soft_tokens"]["cpu_baseline"] = {
            "value": nbytes / secs / 1e9, "unit": "GB/s", "cores": blas_threads(), "kind": "oracle", "seconds": secs,
            "sample": f"{Bi} of the 64 images (64x64 patches x 1152 features, bytes counted as bf16 like the GPU "
                      f"metric), float64 numpy"}


# ---------------------------------------------------------------- GPU arm
def run_gpu(args, rank, world, local_rank):
    import torch
    import global_gqa_b200 as g3

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    g3.lib()
    pk, pk_kind = peaks()
    cfg = inputs.BLOCK_8K
    blk = cfg.block()

    # ---- prefill block inputs, resident in HBM (one set per layer); under
    # torchrun every rank takes a sequence of its own (seeded by rank)
    layers = []
    for li, L in enumerate(blk):
        x = inputs.prefill_layer_inputs(cfg.B, cfg.S, cfg.Hq, cfg.Hkv, cfg.D, seed=cfg.seed + rank, layer=li,
                                        n_spans=cfg.n_spans)
        xd = {k: (None if v is None else v.to(dev)) for k, v in x.items()}
        xd["out"] = torch.empty_like(xd["q"])
        layers.append((L, xd))
    ws = torch.empty(g3.prefill_workspace_size(cfg.B, cfg.S, cfg.Hq, cfg.Hkv, cfg.D), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    block_flops = metrics.block_flops(cfg.B, cfg.S, cfg.Hq, cfg.D, blk)

    def prefill_step():
        for L, x in layers:
            g3.prefill(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], L.kind, L.window,
                       L.rope_base, L.interp, x["spans"], out=x["out"], ws=ws, stream=stream)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        prefill_step()
    if g3.check_device_error(ws) != 0:
        raise RuntimeError("device error during warm-up")
    sampler = ClockSampler(local_rank)
    g3.trace_collect()
    barrier()
    with sampler:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            g3.trace_enable(i % TRACE_EVERY == 0)
            prefill_step()
        g3.trace_enable(False)
        e1.record(stream)
        barrier()
    ms = e0.elapsed_time(e1)
    trace = g3.trace_collect()
    if g3.check_device_error(ws) != 0:
        raise RuntimeError("device error in the timed region")
    ms_max = max_over_ranks(ms, dev)
    value = weak_scaling_rate(block_flops, args.steps, world, ms_max) / 1e12

    n_attn, attn_ms = trace.get("prefill_attention", (0, 0.0))
    achieved = block_flops * n_traced(args.steps) / (attn_ms * 1e-3) / 1e12 if attn_ms > 0 else None
    traffic = None
    try:
        with open(TRAFFIC_PATH) as f:
            tr = json.load(f)
        if tr.get("source_hash") == kernel_source_hash():
            traffic = tr.get("bytes_per_launch")
    except (OSError, ValueError):
        pass
    peak_tf = pk["bf16_tflops"]
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                "frac": (achieved / peak_tf) if achieved else None,
                "frac_of_nominal": (achieved / NOMINAL["bf16_tflops"]) if achieved else None, "traffic": traffic,
                "kernel": "prefill_attention", "peak_kind": f"{pk_kind} dense bf16 burst",
                "launches": n_attn, "avg_launch_ms": attn_ms / max(n_attn, 1),
                "traced_steps": n_traced(args.steps)}
    # Launches and time of the traced steps (every TRACE_EVERY-th timed step).
    kernels = {k: {"launches": v[0], "ms": v[1], "share": v[1] / max(sum(x[1] for x in trace.values()), 1e-9)}
               for k, v in trace.items()}

    # ---- per layer kind (outside the timed region): one local and the global layer
    layer_kinds = {}
    for li in (0, len(blk) - 1):
        L, x = layers[li]
        f = metrics.layer_flops(cfg.B, cfg.S, cfg.Hq, cfg.D, L.kind, L.window)
        g3.trace_collect()
        barrier()
        g3.trace_enable(True)
        for _ in range(max(args.steps, 5)):
            g3.prefill(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], L.kind, L.window,
                       L.rope_base, L.interp, x["spans"], out=x["out"], ws=ws, stream=stream)
        barrier()
        g3.trace_enable(False)
        tr = g3.trace_collect()
        na, ma = tr.get("prefill_attention", (1, 0.0))
        npro, mpro = tr.get("prefill_prologue", (1, 0.0))
        layer_kinds["local" if L.kind == 0 else "global"] = {
            "flops": f, "attention_us": 1e3 * ma / na, "attention_tflops": f / (ma / na * 1e-3) / 1e12,
            "prologue_us": 1e3 * mpro / npro}

    # ---- chunked prefill (outside the timed region): the same block, each layer's
    # 8192-token prompt taken as four 2048-token chunks onto its KV cache
    chunked = None
    if args.extras:
        C = 2048
        cws = None
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        caches = []
        for L, x in layers:
            cap = L.window if L.kind == 0 else cfg.S
            caches.append((torch.empty(cfg.B, cfg.Hkv, cap, cfg.D, dtype=torch.bfloat16, device=dev),
                           torch.empty(cfg.B, cfg.Hkv, cap, cfg.D, dtype=torch.bfloat16, device=dev)))
        need = max(g3.prefill_chunk_workspace_size(cfg.B, C, cfg.Hq, cfg.Hkv, cfg.D, a, L.kind, L.window)
                   for L, _ in layers for a in range(0, cfg.S, C))
        cws = torch.empty(need, dtype=torch.uint8, device=dev)
        pieces = [[{k: x[k][:, a:a + C].contiguous() for k in ("q", "k", "v", "positions")}
                   for a in range(0, cfg.S, C)] for _, x in layers]

        def chunked_block():
            for (L, x), (kc, vc), ps in zip(layers, caches, pieces):
                for i, pc in enumerate(ps):
                    g3.prefill_chunk(pc["q"], pc["k"], pc["v"], x["q_gamma"], x["k_gamma"], pc["positions"], kc, vc,
                                     i * C, L.kind, L.window, L.rope_base, L.interp, None, ws=cws, stream=stream)

        for _ in range(2):
            chunked_block()
        barrier()
        reps = max(args.steps // 2, 3)
        ev0.record(stream)
        for _ in range(reps):
            chunked_block()
        ev1.record(stream)
        barrier()
        cms = ev0.elapsed_time(ev1) / reps
        chunked = {"workload": f"{cfg.name} as {cfg.S // C} chunks of {C} tokens per layer (no image spans)",
                   "ms_per_block": cms, "tflops": block_flops / (cms * 1e-3) / 1e12}
        del caches, cws, pieces

    # ---- Gemma 3 1B attention shapes (outside the timed region): one local and
    # one global layer of 32768 tokens, 4 query heads, 1 kv head, head dim 256
    shapes_1b = None
    if args.extras:
        S1, Hq1, Hkv1, D1 = 32768, 4, 1, 256
        x1 = {k: v.to(dev) for k, v in inputs.prefill_layer_inputs(1, S1, Hq1, Hkv1, D1, seed=0, layer=0).items()
              if v is not None}
        out1 = torch.empty_like(x1["q"])
        ws1 = torch.empty(g3.prefill_workspace_size(1, S1, Hq1, Hkv1, D1), dtype=torch.uint8, device=dev)
        bws1 = torch.empty(g3.prefill_backward_workspace_size(1, S1, Hq1, Hkv1, D1), dtype=torch.uint8, device=dev)
        shapes_1b = {"workload": "B1 S32768 Hq4 Hkv1 D256 (Gemma 3 1B shapes)"}
        for kind, W, base, interp, name in ((0, 1024, 1e4, 1.0, "local"), (1, S1, 1e6, 8.0, "global")):
            f = metrics.layer_flops(1, S1, Hq1, D1, kind, W)
            for _ in range(2):
                g3.prefill(x1["q"], x1["k"], x1["v"], x1["q_gamma"], x1["k_gamma"], x1["positions"], kind, W, base,
                           interp, out=out1, ws=ws1, stream=stream)
            g3.trace_collect()
            barrier()
            g3.trace_enable(True)
            for _ in range(5):
                g3.prefill(x1["q"], x1["k"], x1["v"], x1["q_gamma"], x1["k_gamma"], x1["positions"], kind, W, base,
                           interp, out=out1, ws=ws1, stream=stream)
            barrier()
            g3.trace_enable(False)
            tr = g3.trace_collect()
            na, ma = tr.get("prefill_attention", (1, 0.0))
            npro, mpro = tr.get("prefill_prologue", (1, 0.0))
            shapes_1b[name] = {"flops": f, "attention_us": 1e3 * ma / na,
                               "attention_tflops": f / (ma / na * 1e-3) / 1e12, "prologue_us": 1e3 * mpro / npro}
            # The backward of the same layer, from its out / lse and a random dout.
            o1, l1 = g3.prefill(x1["q"], x1["k"], x1["v"], x1["q_gamma"], x1["k_gamma"], x1["positions"], kind, W,
                                base, interp, return_lse=True, ws=ws1, stream=stream)
            do1 = torch.empty_like(o1)
            inputs.device_fill_normal_bf16(do1, seed=200 + kind)
            g1 = {"dq": torch.empty_like(x1["q"]), "dk": torch.empty_like(x1["k"]), "dv": torch.empty_like(x1["v"]),
                  "dq_gamma": torch.empty(D1, dtype=torch.float32, device=dev),
                  "dk_gamma": torch.empty(D1, dtype=torch.float32, device=dev)}

            def backward_1b():
                g3.prefill_backward(x1["q"], x1["k"], x1["v"], x1["q_gamma"], x1["k_gamma"], x1["positions"], kind,
                                    W, base, interp, None, o1, l1, do1, grads=g1, ws=bws1, stream=stream)

            for _ in range(2):
                backward_1b()
            if g3.check_device_error(bws1) != 0:
                raise RuntimeError("device error in the head-dim-256 backward warm-up")
            g3.trace_collect()
            barrier()
            g3.trace_enable(True)
            e0g = torch.cuda.Event(enable_timing=True)
            e1g = torch.cuda.Event(enable_timing=True)
            e0g.record(stream)
            for _ in range(3):
                backward_1b()
            e1g.record(stream)
            barrier()
            g3.trace_enable(False)
            tr = g3.trace_collect()
            bms = e0g.elapsed_time(e1g) / 3
            shapes_1b[name]["backward"] = {
                "ms": bms, "tflops_algorithmic": 2.5 * f / (bms * 1e-3) / 1e12,
                "kernels_us": {k: 1e3 * m / n for k, (n, m) in tr.items() if n > 0},
                "note": "dV, dK and dQ kernels of head dim 256 (64-row streamed sub-tiles); trace on every call"}
            del o1, l1, do1, g1
        del x1, out1, ws1, bws1

    # ---- image soft tokens (outside the timed region): 64 images, 64x64 patch
    # grid of 1152 features each, 4x4 pool -> 256 tokens; HBM-bound
    soft = None
    if args.extras:
        Bi, gh, F = 64, 64, 1152
        px = torch.empty(Bi, gh * gh, F, dtype=torch.bfloat16, device=dev)
        inputs.device_fill_normal_bf16(px, seed=17)
        gam = torch.ones(F, dtype=torch.float32, device=dev)
        so = torch.empty(Bi, (gh // 4) ** 2, F, dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            g3.soft_tokens(px, gam, gh, gh, 4, out=so, stream=stream)
        e0s = torch.cuda.Event(enable_timing=True)
        e1s = torch.cuda.Event(enable_timing=True)
        barrier()
        e0s.record(stream)
        for _ in range(20):
            g3.soft_tokens(px, gam, gh, gh, 4, out=so, stream=stream)
        e1s.record(stream)
        barrier()
        sms = e0s.elapsed_time(e1s) / 20
        sbytes = (px.numel() + so.numel()) * 2 + F * 4
        gbs = sbytes / (sms * 1e-3) / 1e9
        soft = {"workload": "64 images, 64x64 patches x 1152 features, 4x4 pool -> 256 tokens",
                "us": sms * 1e3, "bytes": sbytes, "GB/s": gbs, "frac_of_measured_hbm": gbs / pk["hbm_gbs"],
                "note": "inputs 604 MB > L2, re-read each call"}
        del px, so

    # ---- backward of the block (outside the timed region): every layer's
    # gradients from its forward out / lse and a random dout
    backward = None
    if args.extras:
        bws = torch.empty(g3.prefill_backward_workspace_size(cfg.B, cfg.S, cfg.Hq, cfg.Hkv, cfg.D),
                          dtype=torch.uint8, device=dev)
        fwd = []
        for li, (L, x) in enumerate(layers):
            o, lse = g3.prefill(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], L.kind,
                                L.window, L.rope_base, L.interp, x["spans"], return_lse=True, ws=ws, stream=stream)
            do = torch.empty_like(o)
            inputs.device_fill_normal_bf16(do, seed=100 + li)
            fwd.append((o, lse, do))
        grads = {"dq": torch.empty_like(layers[0][1]["q"]), "dk": torch.empty_like(layers[0][1]["k"]),
                 "dv": torch.empty_like(layers[0][1]["v"]),
                 "dq_gamma": torch.empty(cfg.D, dtype=torch.float32, device=dev),
                 "dk_gamma": torch.empty(cfg.D, dtype=torch.float32, device=dev)}

        def backward_block():
            for (L, x), (o, lse, do) in zip(layers, fwd):
                g3.prefill_backward(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], L.kind,
                                    L.window, L.rope_base, L.interp, x["spans"], o, lse, do, grads=grads, ws=bws,
                                    stream=stream)

        for _ in range(3):
            backward_block()
        if g3.check_device_error(bws) != 0:
            raise RuntimeError("device error in the backward warm-up")
        reps = max(args.steps // 2, 5)
        g3.trace_collect()
        barrier()
        e0b = torch.cuda.Event(enable_timing=True)
        e1b = torch.cuda.Event(enable_timing=True)
        e0b.record(stream)
        for i in range(reps):
            g3.trace_enable(i % TRACE_EVERY == 0)
            backward_block()
        g3.trace_enable(False)
        e1b.record(stream)
        barrier()
        tr = g3.trace_collect()
        if g3.check_device_error(bws) != 0:
            raise RuntimeError("device error in the backward timing")
        bms = e0b.elapsed_time(e1b) / reps
        # Algorithmic FLOPs: five products per visible pair (S, dP, dV, dK, dQ)
        # = 2.5 x the forward's two.  The dK/dV kernel executes four of them
        # (S^T, dP^T, dV, dK) and the dQ kernel three (S, dP, dQ).
        alg = 2.5 * block_flops
        ker = {}
        for name, mult in (("backward_dkdv", 2.0), ("backward_dq", 1.5)):
            n_k, m_k = tr.get(name, (0, 0.0))
            tf = mult * block_flops * n_traced(reps) / (m_k * 1e-3) / 1e12 if m_k > 0 else None
            ker[name] = {"launches": n_k, "ms": m_k, "tflops_executed": tf,
                         "frac_of_measured_peak": tf / peak_tf if tf else None}
        for name in ("prefill_prologue", "backward_prep", "backward_norm_rope"):
            n_k, m_k = tr.get(name, (0, 0.0))
            ker[name] = {"launches": n_k, "ms": m_k}
        kinds = {}
        for li in (0, len(blk) - 1):
            (L, x), (o, lse, do) = layers[li], fwd[li]
            f = metrics.layer_flops(cfg.B, cfg.S, cfg.Hq, cfg.D, L.kind, L.window)
            g3.trace_collect()
            barrier()
            g3.trace_enable(True)
            for _ in range(5):
                g3.prefill_backward(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], L.kind,
                                    L.window, L.rope_base, L.interp, x["spans"], o, lse, do, grads=grads, ws=bws,
                                    stream=stream)
            barrier()
            g3.trace_enable(False)
            tl = g3.trace_collect()
            row = {}
            for name, mult in (("backward_dkdv", 2.0), ("backward_dq", 1.5)):
                n_k, m_k = tl.get(name, (1, 0.0))
                row[name] = {"us": 1e3 * m_k / n_k, "tflops_executed": mult * f / (m_k / n_k * 1e-3) / 1e12}
            for name in ("prefill_prologue", "backward_prep", "backward_norm_rope"):
                n_k, m_k = tl.get(name, (1, 0.0))
                row[name] = {"us": 1e3 * m_k / n_k}
            kinds["local" if L.kind == 0 else "global"] = row
        backward = {"workload": f"{cfg.name}: gradients of all six layers (dq, dk, dv, both gains)",
                    "ms_per_block": bms, "tflops": alg / (bms * 1e-3) / 1e12,
                    "flops_per_block": alg, "flops_note": "algorithmic: 2.5 x the forward's unmasked FLOPs",
                    "kernels": ker, "layer_kinds": kinds}
        del bws, fwd, grads

    # ---- end to end through the public API from pinned host memory
    host = []
    for L, x in layers:
        hx = {k: (v.cpu().pin_memory() if v is not None and k != "out" else None) for k, v in x.items()}
        hx["out"] = torch.empty(x["out"].shape, dtype=x["out"].dtype).pin_memory()
        host.append((L, hx))
    h2d = sum(v.numel() * v.element_size() for _, hx in host for k, v in hx.items() if v is not None and k != "out")
    d2h = sum(hx["out"].numel() * hx["out"].element_size() for _, hx in host)

    # Uploads, layers and downloads on three streams ordered by events, so a
    # layer's download overlaps the next layer's upload (the host link is full
    # duplex) and both overlap the kernels.  A layer's input buffers are
    # overwritten only after its previous prefill read them, and its output
    # only after its previous download.
    h2d_st = torch.cuda.Stream(dev)
    d2h_st = torch.cuda.Stream(dev)
    ev_c = [None] * len(layers)
    ev_d = [None] * len(layers)

    def e2e_step():
        for i, ((L, hx), (_, x)) in enumerate(zip(host, layers)):
            with torch.cuda.stream(h2d_st):
                if ev_c[i] is not None:
                    h2d_st.wait_event(ev_c[i])
                for k in ("q", "k", "v", "q_gamma", "k_gamma", "positions"):
                    x[k].copy_(hx[k], non_blocking=True)
                eh = torch.cuda.Event()
                eh.record(h2d_st)
            stream.wait_event(eh)
            if ev_d[i] is not None:
                stream.wait_event(ev_d[i])
            g3.prefill(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], L.kind, L.window,
                       L.rope_base, L.interp, x["spans"], out=x["out"], ws=ws, stream=stream)
            ec = torch.cuda.Event()
            ec.record(stream)
            ev_c[i] = ec
            with torch.cuda.stream(d2h_st):
                d2h_st.wait_event(ec)
                hx["out"].copy_(x["out"], non_blocking=True)
                ed = torch.cuda.Event()
                ed.record(d2h_st)
                ev_d[i] = ed

    e2e_steps = max(1, min(args.steps, 20))
    e2e_step()
    barrier()
    w0 = time.perf_counter()
    e0.record(stream)
    h2d_st.wait_event(e0)
    for _ in range(e2e_steps):
        e2e_step()
    for ed in ev_d:
        stream.wait_event(ed)
    e1.record(stream)
    barrier()
    wall = time.perf_counter() - w0
    e2e_ms = max_over_ranks(max(e0.elapsed_time(e1), wall * 1e3), dev)
    e2e_value = weak_scaling_rate(block_flops, e2e_steps, world, e2e_ms) / 1e12
    del host

    # ---- decode block step on the 64 x (4K..128K) workload
    decode = None
    if not args.no_decode:
        decode = run_decode(args, dev, stream, rank, world, pk, pk_kind)

    # ---- mixed text+image 2 x 32K block and 128K block
    long_blocks = None
    if args.extras:
        long_blocks = run_long_blocks(args, dev, stream, rank, world, pk, pk_kind)

    clocks = sampler.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": block_config(cfg, world, block_flops),
        "value_frac": fractions(value / max(world, 1), peak_tf, NOMINAL["bf16_tflops"]),
        "roofline": roofline,
        "kernels": kernels,
        "layer_kinds": layer_kinds,
        "chunked_prefill": chunked,
        "shapes_1b": shapes_1b,
        "soft_tokens": soft,
        "backward": backward,
        "gpu_launches": launches_in_timed_region(trace, args.steps, untraced_per_step=len(blk)),
        "clocks": clocks,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps},
        "decode": decode,
        "long_blocks": long_blocks,
    }
    return line


def run_decode(args, dev, stream, rank, world, pk, pk_kind):
    """Six g3attn_decode calls on the 64-sequence batch; under torchrun the
    batch is split by sequence (shard.sequence_shard) and the rate counts the
    whole batch's bytes over the slowest rank's time (strong scaling)."""
    import torch
    import global_gqa_b200 as g3
    cfg = inputs.DECODE_B64
    blk = cfg.block()
    lens_all = inputs.decode_lengths(cfg.B, cfg.len_lo, cfg.len_hi, cfg.seed)
    b0, b1 = shard.sequence_shard(cfg.B, world, rank)
    B = b1 - b0
    lens = lens_all[b0:b1]
    sl = lens.to(dev)
    caches = []
    for li, L in enumerate(blk):
        if L.kind == 0:
            kc = torch.empty(B, cfg.Hkv, cfg.window, cfg.D, dtype=torch.bfloat16, device=dev)
        else:
            kc = torch.empty(B, cfg.Hkv, cfg.global_capacity, cfg.D, dtype=torch.bfloat16, device=dev)
        vc = torch.empty_like(kc)
        inputs.device_fill_normal_bf16(kc, inputs.seed_for(cfg.seed, li, inputs.T_KC) + b0)
        inputs.device_fill_normal_bf16(vc, inputs.seed_for(cfg.seed, li, inputs.T_VC) + b0)
        step_in = inputs.decode_step_inputs(cfg.B, cfg.Hq, cfg.Hkv, cfg.D, seed=cfg.seed, layer=li)
        x = {k: (v[b0:b1] if v.dim() == 3 else v).contiguous().to(dev) for k, v in step_in.items()}
        x["out"] = torch.empty_like(x["q"])
        caches.append((L, kc, vc, x))
    ws = torch.empty(g3.decode_workspace_size(B, cfg.Hq, cfg.Hkv, cfg.D, cfg.len_hi), dtype=torch.uint8,
                     device=dev)
    step_bytes = sum(metrics.decode_kv_bytes(lens.numpy(), cfg.Hkv, cfg.D, L.kind, L.window) for L in blk)
    all_bytes = sum(metrics.decode_kv_bytes(lens_all.numpy(), cfg.Hkv, cfg.D, L.kind, L.window) for L in blk)

    def step():
        for L, kc, vc, x in caches:
            g3.decode(x["q"], x["k_new"], x["v_new"], x["q_gamma"], x["k_gamma"], kc, vc, sl, cfg.len_hi, L.kind,
                      L.window, L.rope_base, L.interp, out=x["out"], ws=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    if g3.check_device_error(ws) != 0:
        raise RuntimeError("device error in decode warm-up")
    g3.trace_collect()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        g3.trace_enable(i % TRACE_EVERY == 0)
        step()
    g3.trace_enable(False)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    trace = g3.trace_collect()
    ms = max_over_ranks(e0.elapsed_time(e1), dev)
    gbs = all_bytes * args.steps / (ms * 1e-3) / 1e9
    n_split, split_ms = trace.get("decode_split", (0, 0.0))
    ach = step_bytes * n_traced(args.steps) / (split_ms * 1e-3) / 1e9 if split_ms > 0 else None
    del caches
    torch.cuda.empty_cache()
    return {
        "metric": "decode KV GB/s (5:1 block)", "value": gbs, "unit": "GB/s", "ms_per_step": ms / args.steps,
        "config": {"workload": cfg.name, "batch": cfg.B, "context": f"U[{cfg.len_lo},{cfg.len_hi}]",
                   "kv_bytes_per_step": all_bytes, "l2": "inputs larger than L2 (~38 GB of cache read per step)",
                   "parallelism": f"batch split by sequence over {world} rank(s)", "sequences_per_rank": B},
        "scaling": "strong",
        "value_frac": fractions(gbs / max(world, 1), pk["hbm_gbs"], NOMINAL["hbm_gbs"]),
        "roofline": {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": (ach / pk["hbm_gbs"]) if ach else None,
                     "frac_of_nominal": (ach / NOMINAL["hbm_gbs"]) if ach else None,
                     "traffic": decode_traffic_per_launch(step_bytes / len(blk)), "kernel": "decode_split",
                     "peak_kind": f"{pk_kind} copy bandwidth", "launches": n_split,
                     "traced_steps": n_traced(args.steps)},
        "kernels": {k: {"launches": v[0], "ms": v[1]} for k, v in trace.items()},
        "gpu_launches": launches_in_timed_region(trace, args.steps),
    }


# ------------------------------------------- mixed text+image and 128K blocks
LONG_CONFIGS = (inputs.MIXED_32K, inputs.LONG_128K)


def long_block_spans(cfg):
    """Image spans of the workload: one set per sequence, the same in every
    layer of the block (images sit at fixed token positions)."""
    return inputs.image_spans(cfg.B, cfg.S, cfg.n_spans, cfg.seed, 0)


def run_long_blocks(args, dev, stream, rank, world, pk, pk_kind):
    """Times the six g3attn_prefill calls of the mixed text+image block (2 x
    32768 tokens, 8 images of 256 tokens per sequence) and of the 128K block,
    each outside the headline timed region; inputs are generated on the device.
    Under torchrun the kv heads are split over the ranks (shard.kv_head_shard)
    and the rate counts the whole block over the slowest rank (strong scaling)."""
    import torch
    import global_gqa_b200 as g3
    res = {}
    for cfg_all in LONG_CONFIGS:
        G = cfg_all.Hq // cfg_all.Hkv
        sh = shard.kv_head_shard(cfg_all.Hkv, G, world, rank)
        Hkv_r = sh["kv"][1] - sh["kv"][0]
        if Hkv_r == 0:
            # a rank without kv heads still takes the same collective steps
            torch.distributed.barrier()
            max_over_ranks(0.0, dev)
            torch.distributed.barrier()
            continue
        cfg = inputs.PrefillConfig(cfg_all.name, cfg_all.B, cfg_all.S, Hkv_r * G, Hkv_r, cfg_all.D, cfg_all.n_spans,
                                   cfg_all.global_interp, cfg_all.seed + 7919 * sh["kv"][0])
        blk = cfg.block()
        spans = long_block_spans(cfg)
        spans_d = None if spans is None else spans.to(dev)
        layers = []
        for li, L in enumerate(blk):
            x = {}
            for name, shape, tid in (("q", (cfg.B, cfg.S, cfg.Hq, cfg.D), inputs.T_Q),
                                     ("k", (cfg.B, cfg.S, cfg.Hkv, cfg.D), inputs.T_K),
                                     ("v", (cfg.B, cfg.S, cfg.Hkv, cfg.D), inputs.T_V)):
                x[name] = inputs.device_fill_normal_bf16(torch.empty(shape, dtype=torch.bfloat16, device=dev),
                                                         inputs.seed_for(cfg.seed, li, tid))
            x["q_gamma"] = inputs.gamma(cfg.D, cfg.seed, li, inputs.T_QG).to(dev)
            x["k_gamma"] = inputs.gamma(cfg.D, cfg.seed, li, inputs.T_KG).to(dev)
            x["positions"] = inputs.positions(cfg.B, cfg.S).to(dev)
            x["out"] = torch.empty_like(x["q"])
            layers.append((L, x))
        ws = torch.empty(g3.prefill_workspace_size(cfg.B, cfg.S, cfg.Hq, cfg.Hkv, cfg.D), dtype=torch.uint8,
                         device=dev)
        flops = metrics.block_flops(cfg.B, cfg.S, cfg.Hq, cfg.D, blk,
                                    None if spans is None else spans.numpy())
        flops_all = flops * cfg_all.Hq / cfg.Hq

        def call(L, x):
            g3.prefill(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], L.kind, L.window,
                       L.rope_base, L.interp, spans_d, out=x["out"], ws=ws, stream=stream)

        for L, x in layers:  # warm-up block
            call(L, x)
        if g3.check_device_error(ws) != 0:
            raise RuntimeError(f"device error in the {cfg.name} warm-up")
        reps = 3 if cfg.S > 65536 else 5
        g3.trace_collect()
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        sampler = ClockSampler(dev.index)
        with sampler:
            e0.record(stream)
            for i in range(reps):
                g3.trace_enable(i == 0)  # the first block carries the kernel trace
                for L, x in layers:
                    call(L, x)
            g3.trace_enable(False)
            e1.record(stream)
            torch.cuda.synchronize(dev)
        tr = g3.trace_collect()
        if g3.check_device_error(ws) != 0:
            raise RuntimeError(f"device error in the {cfg.name} timing")
        ms = max_over_ranks(e0.elapsed_time(e1) / reps, dev)
        if world > 1:
            torch.distributed.barrier()
        n_attn, attn_ms = tr.get("prefill_attention", (0, 0.0))
        ach = flops / (attn_ms * 1e-3) / 1e12 if attn_ms > 0 else None
        # per layer kind: one local and the global layer, traced alone
        kinds = {}
        for li in (0, len(blk) - 1):
            L, x = layers[li]
            f = metrics.layer_flops(cfg.B, cfg.S, cfg.Hq, cfg.D, L.kind, L.window,
                                    None if spans is None else spans.numpy())
            call(L, x)  # warm-up: a layer's first call after the other kind runs slower
            g3.trace_collect()
            g3.trace_enable(True)
            for _ in range(2):
                call(L, x)
            g3.trace_enable(False)
            t = g3.trace_collect()
            na, ma = t.get("prefill_attention", (1, 0.0))
            npro, mpro = t.get("prefill_prologue", (1, 0.0))
            kinds["local" if L.kind == 0 else "global"] = {
                "flops": f, "attention_us": 1e3 * ma / na, "attention_tflops": f / (ma / na * 1e-3) / 1e12,
                "prologue_us": 1e3 * mpro / npro}
        res[cfg.name] = {
            "workload": cfg.name,
            "config": {"batch": cfg.B, "seq_len": cfg.S, "q_heads": cfg_all.Hq, "kv_heads": cfg_all.Hkv,
                       "head_dim": cfg.D, "image_spans_per_sequence": cfg.n_spans,
                       "global_interp": cfg.global_interp, "unmasked_flops_per_block": flops_all,
                       "l2": "inputs far larger than L2", "inputs": "N(0,1) bf16 generated on the device",
                       "parallelism": f"kv heads split over {world} rank(s)", "kv_heads_per_rank": cfg.Hkv},
            "scaling": "strong",
            "ms_per_block": ms, "tflops": flops_all / (ms * 1e-3) / 1e12, "blocks_timed": reps,
            "value_frac": fractions(flops_all / (ms * 1e-3) / 1e12 / max(world, 1), pk["bf16_tflops_sustained"],
                                    NOMINAL["bf16_tflops"]),
            # Blocks of 27-180 ms run for seconds back to back: the GPU settles at
            # its power-capped clock, so the peak is the sustained matmul figure.
            "roofline": {"bound": "tensor", "achieved": ach, "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                         "frac": (ach / pk["bf16_tflops_sustained"]) if ach else None,
                         "frac_of_burst": (ach / pk["bf16_tflops"]) if ach else None,
                         "frac_of_nominal": (ach / NOMINAL["bf16_tflops"]) if ach else None, "traffic": None,
                         "kernel": "prefill_attention",
                         "peak_kind": f"{pk_kind} dense bf16 sustained (seconds-long, under the power cap)",
                         "launches": n_attn, "avg_launch_ms": attn_ms / max(n_attn, 1)},
            "clocks": sampler.summary(),
            "kernels": {k: {"launches": v[0], "ms": v[1]} for k, v in tr.items()},
            "layer_kinds": kinds,
            "gpu_launches": (sum(v[0] for v in tr.values()) + len(blk)) * reps,  # + the untraced error resets
        }
        del layers, ws, x
        torch.cuda.empty_cache()
    return res


def oracle_long_baselines(long_res: dict, budget_s: float) -> None:
    """The oracle timed as it stands on sampled query rows of every layer of the
    mixed and 128K blocks, on one GQA group (2 query heads, 1 kv head) of the
    same sequences and spans; its FLOP rate is extrapolated to the whole block
    by the unmasked-pair count."""
    from oracle import attention as O
    for cfg in LONG_CONFIGS:
        r = long_res.get(cfg.name) if long_res else None
        if not r:
            continue
        blk = cfg.block()
        spans = long_block_spans(cfg)
        sp = None if spans is None else spans.numpy()
        rng = np.random.default_rng(5)
        flops, secs, nrows, li = 0.0, 0.0, 0, 0
        per_layer = max(budget_s / len(blk), 0.5)
        for li, L in enumerate(blk):
            x = inputs.prefill_layer_inputs(cfg.B, cfg.S, 2, 1, cfg.D, seed=cfg.seed, layer=li)
            lo, hi = [], []
            for b in range(cfg.B):
                a, c = metrics.row_intervals(cfg.S, L.kind, L.window, None if sp is None else sp[b])
                lo.append(a)
                hi.append(c)
            t_layer = 0.0
            while t_layer < per_layer:
                rows = np.sort(rng.choice(cfg.S, 128, replace=False))
                t0 = time.perf_counter()
                O.prefill_rows(x["q"], x["k"], x["v"], x["q_gamma"], x["k_gamma"], x["positions"], L.kind,
                               L.window, L.rope_base, L.interp, spans, rows=rows)
                dt = time.perf_counter() - t0
                t_layer += dt
                secs += dt
                flops += 4.0 * cfg.D * 2 * sum(float(np.sum(hi[b][rows] - lo[b][rows] + 1)) for b in range(cfg.B))
                nrows += rows.size * cfg.B
        rate = flops / secs
        r["cpu_baseline"] = {
            "value": rate / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle", "seconds": secs,
            "extrapolated_s_per_block": r["config"]["unmasked_flops_per_block"] / rate,
            "sample": f"{nrows} query rows (groups of 128, every layer) of one GQA group (2 query heads, 1 kv head) "
                      f"of the {cfg.name} sequences, float64 numpy; the block time is extrapolated by "
                      f"unmasked-pair count"}


# ---------------------------------------------------------- reference arm
def run_reference(args):
    cfg = inputs.BLOCK_8K
    cores = blas_threads()
    for _ in range(args.warmup):
        oracle_prefill_sample(cfg, 0.0, seed=1)
    flops, secs, rows = 0.0, 0.0, 0
    for s in range(args.steps):
        f, t, r = oracle_prefill_sample(cfg, 0.0, seed=100 + s)
        flops, secs, rows = flops + f, secs + t, rows + r
    value = flops / secs / 1e12
    sample = f"{rows} query rows (64 per layer per step, all 32 heads) of the {cfg.name} block"
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": block_config(cfg, int(os.environ.get("WORLD_SIZE", "1")),
                                   metrics.block_flops(cfg.B, cfg.S, cfg.Hq, cfg.D, cfg.block())),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_probe_layer(kind_name: str, S: int) -> dict:
    """One 27B-shaped attention layer (B 1, 32 query / 16 kv heads, D 128) of S
    tokens, run twice (the second call is the one a profiler captures with
    `-s` skipping the first launches); prints its traced attention time."""
    import torch
    import global_gqa_b200 as g3
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    kind = 0 if kind_name == "local" else 1
    base, interp = (1e4, 1.0) if kind == 0 else (1e6, 8.0)
    x = {}
    for name, H, tid in (("q", 32, inputs.T_Q), ("k", 16, inputs.T_K), ("v", 16, inputs.T_V)):
        x[name] = inputs.device_fill_normal_bf16(torch.empty(1, S, H, 128, dtype=torch.bfloat16, device=dev),
                                                 inputs.seed_for(0, kind, tid))
    qg, kg = inputs.gamma(128, 0, kind, inputs.T_QG).to(dev), inputs.gamma(128, 0, kind, inputs.T_KG).to(dev)
    pos = inputs.positions(1, S).to(dev)
    out = torch.empty_like(x["q"])
    ws = torch.empty(g3.prefill_workspace_size(1, S, 32, 16, 128), dtype=torch.uint8, device=dev)
    for i in range(2):
        g3.trace_enable(i == 1)
        g3.prefill(x["q"], x["k"], x["v"], qg, kg, pos, kind, 1024, base, interp, out=out, ws=ws)
    torch.cuda.synchronize(dev)
    g3.trace_enable(False)
    if g3.check_device_error(ws) != 0:
        raise RuntimeError("device error in the probe layer")
    n, ms = g3.trace_collect()["prefill_attention"]
    f = metrics.layer_flops(1, S, 32, 128, kind, 1024)
    return {"probe_layer": kind_name, "seq_len": S, "attention_us": 1e3 * ms / n,
            "attention_tflops": f / (ms / n * 1e-3) / 1e12}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="g3attn", choices=["g3attn", "reference"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-extras", dest="extras", action="store_false",
                    help="skip the chunked-prefill and 1B-shape measurements")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--probe-layer", choices=["local", "global"],
                    help="only run one 27B-shaped layer of --probe-seq tokens twice (for profiler captures)")
    ap.add_argument("--probe-seq", type=int, default=32768)
    args = ap.parse_args()
    if args.probe_layer:
        print(json.dumps(run_probe_layer(args.probe_layer, args.probe_seq)), flush=True)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        # Every rank runs the same work between collectives, so a rank that
        # stalls or dies shows as a collective timing out well within this.
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                             device_id=torch.device("cuda", local_rank))
    line = run_gpu(args, rank, world, local_rank)
    if rank == 0 and world == 1:
        f, s, r = oracle_prefill_sample(inputs.BLOCK_8K, args.cpu_budget)
        line["cpu_baseline"] = {"value": f / s / 1e12, "unit": "TFLOP/s", "cores": blas_threads(),
                                "kind": "oracle", "seconds": s,
                                "sample": f"{r} query rows (groups of 64 per layer, all 32 heads) of the "
                                          f"{inputs.BLOCK_8K.name} block, float64 numpy"}
        if args.extras and args.cpu_budget > 0:
            oracle_extras_baselines(line, args.cpu_budget)
            oracle_long_baselines(line.get("long_blocks"), args.cpu_budget / 2)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
