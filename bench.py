#!/usr/bin/env python
"""Throughput of the TokenGate gated-prefill hot path on B200.

One step = the whole path over one synthetic batch: gate-MLP score of every token ->
top-K with the question tail -> gather of the kept rows -> token-gated causal attention
(one above-L layer), each through the C ABI of libtokengate. Default workload: N=32768
tokens, question tail 128, K=2048 (2176 kept rows), d=2048, gate 2048->256->1, 16 query /
8 KV heads, head_dim 128, bf16 (Qwen3-1.7B shapes; seeded synthetic data).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tokengate|reference]

Prints ONE JSON line on rank 0. With N > 1 (torchrun) every rank runs an independent
replica of the workload (the path needs no exchange between GPUs) and value = tokens of
all ranks / max-over-ranks time. ``--impl reference`` times the CPU oracle instead, on a
bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "gated-prefill tokens/s at N=32K,K=2K; gated-attn TFLOP/s and % of bf16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="tokengate", choices=["tokengate", "reference"])
    ap.add_argument("--workload", default="qwen3_32k")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-full-ref", action="store_true")
    ap.add_argument("--no-other", action="store_true", help="skip the other configurations' throughput")
    ap.add_argument("--no-bw", action="store_true", help="skip the byte-heavy select/gather instances")
    ap.add_argument("--bw-only", action="store_true", help="run only the byte-heavy select/gather instances")
    ap.add_argument("--bw-reps", type=int, default=20)
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read-only) every 5 ms."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int):
        self.samples = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - depends on the box
            self.error = repr(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(0.005)

    def start(self):
        if self._h is not None:
            self._t.start()
        return self

    def stop(self):
        self._stop.set()
        if self._t.is_alive():
            self._t.join()
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "nvml", "note": getattr(self, "error", "no samples")}
        busy = [m for m, r in self.samples if not (r & 0x1)] or [m for m, _ in self.samples]
        seen = 0
        for _, r in self.samples:
            seen |= r
        names = [k for k, v in self.REASONS.items() if seen & v and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples), "source": "nvml 5 ms"}


# --------------------------------------------------------------------------- oracle timing


def oracle_step(wl, H, W1, b1, w2, b2, layers):
    """One whole step of the CPU oracle on the workload, timed (wall clock, host cores).

    The step starts from the stored input bytes (bf16 bits widened exactly to float64, as the
    oracle consumes them): gate-MLP scores of every token, top-K with the question tail on those
    scores, gather, and gated attention over every kept query row, every head and every above-L
    layer. Returns (seconds, description)."""
    import numpy as np

    import tg_inputs as ti
    from oracle import tg_oracle as orc

    t0 = time.perf_counter()
    s = orc.gate_scores(ti.widen(H, wl.dtype), ti.widen(W1, wl.dtype), b1, ti.widen(w2, wl.dtype), b2)
    kept, cu = orc.topk_select(s, wl.seqlens, wl.q_len, wl.k)
    _, pos, _, lg = orc.gather(H, s, kept, wl.seqlens, wl.q_len, cu)
    for (Q, K, V) in layers:
        orc.gated_attention(ti.widen(Q, wl.dtype), ti.widen(K, wl.dtype), ti.widen(V, wl.dtype), lg, pos, cu,
                            wl.Hq, wl.Hkv, 1.0 / math.sqrt(wl.D))
    dt = time.perf_counter() - t0
    m = int(np.asarray(cu)[-1])
    desc = (f"full step: scores of all {wl.n_tok} tokens, select, gather, attention over all {m} kept rows x "
            f"{wl.Hq} heads x {len(layers)} layer(s), float64 NumPy from the stored input bytes")
    return dt, desc


def blas_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# --------------------------------------------------------------------------- main


KERNEL_SRC = {"score": "tg_score_tc.cu", "select": "tg_select.cu", "gather": "tg_gather.cu",
              "gated_attn": "tg_attn_tc.cu"}


def kernel_hash(kernel_key):
    """Hash of the sources a kernel is built from (its .cu and the shared device headers);
    DRAM counters recorded under profiles/ apply only while this hash is unchanged."""
    h = hashlib.sha256()
    for n in (KERNEL_SRC[kernel_key], "tg_sm100.cuh", "tg_internal.cuh"):
        p = os.path.join(ROOT, "learned_token_pruning_02_b200", "csrc", n)
        if not os.path.exists(p):
            return ""
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_from_profile(kernel_key, src_hash):
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d.get(kernel_key)
        if isinstance(e, dict) and e.get("source_hash") == src_hash:
            return e.get("bytes_per_launch")
    except Exception:
        pass
    return None


def bandwidth_instances(tg, torch, dev, peak_gbs, reps):
    """Select and gather on byte-heavy shapes, with the same kernels and entry points, to show
    their bandwidth where the bench workload is latency-bound: select over 64 sequences of
    131072 seeded N(0,1) scores (question tail 256, K=4096 each; 33.5 MB read) and a gather of
    65536 of 131072 rows of d=2048 bf16 (537 MB moved). L2 is flushed before every launch; each
    launch is timed alone with CUDA events on its stream. The select runs both as one cluster per
    sequence (tg_topk_select) and as the four-kernel stream over all SMs (tg_topk_select_stream)."""
    gen = torch.Generator(device=dev)
    gen.manual_seed(20260)
    stream = torch.cuda.current_stream()
    flush = L2Flush(torch, dev)

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            flush()
            torch.cuda._sleep(100_000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) / 1e3)
        return sum(ts) / len(ts)

    out = {"l2": "flushed before every launch (512 MiB memset, then a 256 MiB read sweep)", "peak_gbs": peak_gbs}
    B, N, q, K = 64, 131072, 256, 4096
    seqlens, q_len, k = (N,) * B, (q,) * B, (K,) * B
    sc = torch.randn(B * N, device=dev, generator=gen, dtype=torch.float32)
    m_tot = tg.tg_kept_counts(seqlens, q_len, k)[-1]
    kept = torch.empty(m_tot, device=dev, dtype=torch.int32)
    cu_dev = torch.empty(B + 1, device=dev, dtype=torch.int32)
    t = timed(lambda: tg.tg_topk_select(sc, seqlens, q_len, k, kept_idx=kept, cu_kept_dev=cu_dev))
    byts = B * (N - q) * 4 + m_tot * 4
    out["select"] = {"shape": f"{B} sequences x {N} tokens, question tail {q}, K={K}", "bytes": byts,
                     "us": t * 1e6, "gbs": byts / t / 1e9, "frac": byts / t / 1e9 / peak_gbs}
    ws = torch.empty(tg.tg_topk_select_stream_workspace_size(seqlens, q_len, k), device=dev, dtype=torch.uint8)
    t = timed(lambda: tg.tg_topk_select_stream(sc, seqlens, q_len, k, kept_idx=kept, cu_kept_dev=cu_dev, ws=ws))
    out["select_stream"] = {"shape": out["select"]["shape"], "bytes": byts, "us": t * 1e6, "gbs": byts / t / 1e9,
                            "frac": byts / t / 1e9 / peak_gbs,
                            "note": "tg_topk_select_stream: histogram, candidates, threshold, compaction over all SMs"}
    del sc, kept, ws
    N, d, q = 131072, 2048, 256
    K = 65536 - q
    H = torch.randn(N, d, device=dev, generator=gen, dtype=torch.float32).to(torch.bfloat16)
    s1 = torch.randn(N, device=dev, generator=gen, dtype=torch.float32)
    kept, _ = tg.tg_topk_select(s1, (N,), (q,), (K,))
    M = kept.numel()
    Hk = torch.empty(M, d, device=dev, dtype=torch.bfloat16)
    pos = torch.empty(M, device=dev, dtype=torch.int32)
    g = torch.empty(M, device=dev, dtype=torch.float32)
    lg = torch.empty(M, device=dev, dtype=torch.float32)
    t = timed(lambda: tg.tg_gather(H, s1, kept, (N,), (q,), (K,), H_kept=Hk, pos=pos, g=g, logg=lg))
    byts = 2 * M * d * 2 + 16 * M
    out["gather"] = {"shape": f"{M} of {N} rows, d={d} bf16", "bytes": byts, "us": t * 1e6,
                     "gbs": byts / t / 1e9, "frac": byts / t / 1e9 / peak_gbs}
    return out


def qkv_rope_time(tg, torch, dev, Hk, pos, Hq, Hkv, D, peak_tflops, reps):
    """Projection of the bench workload's kept rows to Q/K/V with rotary embedding at their
    original positions (a seeded N(0, 1/d) stacked projection, theta 1e6), L2 flushed before
    every launch."""
    gen = torch.Generator(device=dev)
    gen.manual_seed(20262)
    M, d = Hk.shape
    N = (Hq + 2 * Hkv) * D
    W = (torch.randn(N, d, device=dev, generator=gen) / d ** 0.5).to(torch.bfloat16)
    Q = torch.empty(M, Hq, D, device=dev, dtype=torch.bfloat16)
    K = torch.empty(M, Hkv, D, device=dev, dtype=torch.bfloat16)
    V = torch.empty(M, Hkv, D, device=dev, dtype=torch.bfloat16)
    flush = L2Flush(torch, dev)
    stream = torch.cuda.current_stream()
    run = lambda: tg.tg_qkv_rope(Hk, W, pos, Hq, Hkv, D, 1.0e6, Q=Q, K=K, V=V)
    run()
    torch.cuda.synchronize()
    tot = 0.0
    for _ in range(reps):
        flush()
        torch.cuda._sleep(100_000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1) / 1e3
    t = tot / reps
    flops = 2.0 * M * N * d
    return {"shape": f"M={M} kept rows x d={d} -> {Hq}/{Hkv} heads x D={D}, rotary at original positions",
            "us": t * 1e6, "tflops": flops / t / 1e12, "frac": flops / t / 1e12 / peak_tflops}


def attn_bwd_time(tg, torch, dev, Q, K, V, logg, pos, cu, scale, peak_tflops, reps):
    """Gradients of the gated attention for the bench workload's kept set (one above-L layer's
    Q/K/V, the chain's own log g and positions, a seeded N(0, 1) upstream dO): the forward gives
    O and lse, then the backward's four kernels are timed together, L2 flushed before each run.
    Algorithmic work: the five products of the backward (S recomputed, dP, dV, dK, dQ), each
    2 D flop per visible (query, key) pair and head."""
    gen = torch.Generator(device=dev)
    gen.manual_seed(20263)
    Hq, D = Q.shape[1], Q.shape[2]
    m = cu[-1]
    O, lse = tg.tg_gated_attn_fwd(Q, K, V, logg, pos, cu, scale)
    dO = torch.randn(Q.shape, device=dev, generator=gen).to(torch.bfloat16)
    bufs = dict(dQ=torch.empty(Q.shape, device=dev), dK=torch.empty(K.shape, device=dev),
                dV=torch.empty(V.shape, device=dev), dlogg=torch.empty(m, device=dev),
                dscore=torch.empty(m, device=dev))
    flush = L2Flush(torch, dev)
    stream = torch.cuda.current_stream()
    run = lambda: tg.tg_gated_attn_bwd(Q, K, V, logg, pos, cu, O, lse, dO, scale, want_dscore=True, **bufs)
    run()
    torch.cuda.synchronize()
    tot = 0.0
    for _ in range(reps):
        flush()
        torch.cuda._sleep(100_000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run()
        e1.record(stream)
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1) / 1e3
    t = tot / reps
    pairs = sum((b - a) * (b - a + 1) // 2 for a, b in zip(cu[:-1], cu[1:]))
    flops = 10.0 * Hq * D * pairs
    return {"shape": f"M={m} kept rows in {len(cu) - 1} sequence(s), {Hq}/{K.shape[1]} heads, D={D}, bf16 in, f32 gradients",
            "us": t * 1e6, "tflops": flops / t / 1e12, "bound": "tensor", "peak": peak_tflops,
            "frac": flops / t / 1e12 / peak_tflops,
            "note": "tcgen05 kernels: rowsum(dO*O) pre-pass, dK/dV per (128-key tile, KV head) cluster, d log g sum, dQ per (128-query tile, head)"}


def projected_chain_time(tg, torch, dev, cb, flush, reps):
    """The path with the above-L layer's own projection (tg_prefill_projected): score, top-K, kept
    rows, Q/K/V with rotary embedding at original positions into a kept-only K/V cache (a seeded
    N(0, 1/d) stacked projection, theta 1e6), gated attention; L2 flushed before each step."""
    wl = cb.wl
    gen = torch.Generator(device=dev)
    gen.manual_seed(20264)
    W = (torch.randn((wl.Hq + 2 * wl.Hkv) * wl.D, wl.d, device=dev, generator=gen) / wl.d ** 0.5).to(torch.bfloat16)
    run = lambda o: tg.tg_prefill_projected(cb.H, cb.W1, cb.b1, cb.w2, cb.b2, wl.seqlens, wl.q_len, wl.k, [W], 1.0e6,
                                            wl.Hq, wl.Hkv, wl.D, cb.scale, out=o)
    out = run(None)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ts = []
    for _ in range(reps):
        flush()
        torch.cuda._sleep(200_000)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        run(out)
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    ms = sum(ts) / len(ts)
    return {"value": wl.n_tok / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
            "note": "score + select + kept-row copy + Q/K/V projection with rotary embedding + gated attention, "
                    "one above-L layer, through tg_prefill_projected (bound Python call per step)"}


def gate_bwd_time(tg, torch, dev, cb, reps):
    """Gradients of the gate network from d score of the bench workload's kept rows (seeded
    N(0, 0.01) d score): two tcgen05 products (z split over d, then u^T H split over the kept rows),
    the GELU' pass between them and an ordered reduction. `us` is the device time per call, from
    `reps` calls captured once into a CUDA graph and replayed; `eager_us` times the same calls
    launched one by one (the host's launch work per call is longer than the GPU's)."""
    gen = torch.Generator(device=dev)
    gen.manual_seed(20265)
    Hk = cb.out["H_kept"]
    M, d = Hk.shape
    dg = cb.W1.shape[0]
    ds = torch.randn(M, device=dev, generator=gen) * 0.01
    bufs = dict(dW1=torch.empty(dg, d, device=dev), db1=torch.empty(dg, device=dev), dw2=torch.empty(dg, device=dev),
                db2=torch.empty(1, device=dev),
                ws=torch.empty(tg.lib().tg_gate_mlp_bwd_workspace_size(M, d, dg), device=dev, dtype=torch.uint8))
    run = lambda: tg.tg_gate_mlp_bwd(Hk, cb.W1, cb.b1, cb.w2, ds, **bufs)
    run()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    t_eager = e0.elapsed_time(e1) / reps / 1e3
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        run()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(reps):
            run()
    graph.replay()
    torch.cuda.synchronize()
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / reps / 1e3
    del graph
    flops = 4.0 * M * d * dg
    return {"shape": f"M={M} kept rows, d={d}, dg={dg}", "us": t * 1e6, "tflops": flops / t / 1e12,
            "eager_us": t_eager * 1e6,
            "note": "tcgen05 z = H W1^T (K split), GELU' pass, tcgen05 dW1 = u^T H (row splits), ordered "
                    "reduction; device time per call from a CUDA graph of back-to-back calls, L2 warm"}


def split_select_times(tg, torch, dev, reps):
    """The sequence-split selection's two device steps for one 131072-token sequence cut into 8
    blocks, K=4096: one rank's top-k candidates of its 16352-token block, and the merge of the
    8 x 4096 gathered candidates (the all-gather between devices is not part of this run)."""
    from learned_token_pruning_02_b200 import split

    gen = torch.Generator(device=dev)
    gen.manual_seed(20261)
    world, n_ctx, q, k = 8, 131072 - 256, 256, 4096
    s = torch.randn(n_ctx + q, device=dev, generator=gen, dtype=torch.float32)
    lo, hi = split.block_bounds(n_ctx, world, 0)
    counts = split.candidate_counts(n_ctx, world, k)
    cs = torch.empty(world * k, device=dev, dtype=torch.float32)
    ci = torch.empty(world * k, device=dev, dtype=torch.int32)
    for r in range(world):
        a, b = split.block_bounds(n_ctx, world, r)
        tg.tg_topk_candidates(s[a:b], k, base=a, cand_score=cs[r * k:(r + 1) * k], cand_idx=ci[r * k:(r + 1) * k])
    kept = torch.empty(k + q, device=dev, dtype=torch.int32)
    stream = torch.cuda.current_stream()

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(reps):
            torch.cuda._sleep(100_000)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            tot += e0.elapsed_time(e1) * 1e3
        return tot / reps

    c_us = timed(lambda: tg.tg_topk_candidates(s[lo:hi], k, base=lo, cand_score=cs[:k], cand_idx=ci[:k]))
    m_us = timed(lambda: tg.tg_topk_merge(cs, ci, k, n_ctx, q, kept_idx=kept))
    whole, _ = tg.tg_topk_select(s, (n_ctx + q,), (q,), (k,))
    torch.cuda.synchronize()
    return {"shape": f"{n_ctx + q} tokens (question tail {q}) over {world} blocks, K={k}",
            "candidates_us": c_us, "merge_us": m_us, "equals_whole_sequence_select": bool(torch.equal(kept, whole))}


def run_reference(args, wl):
    """The oracle arm: whole oracle steps on the host cores (rank 0 only). Warm-up and timed
    steps are full steps; if the requested count would run past about three minutes, fewer steps
    are timed and the line says how many (the per-step time is measured, never extrapolated)."""
    import tg_inputs as ti

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    H = ti.hidden_states(wl)
    W1, b1, w2, b2 = ti.gate_weights(wl)
    layers = [ti.qkv(wl, l) for l in range(wl.n_layers)]
    t_first, desc = oracle_step(wl, H, W1, b1, w2, b2, layers)  # the first warm-up step sizes the run
    budget = 180.0
    fit = max(1, int((budget - t_first) / max(t_first, 1e-3)))
    warm = min(max(args.warmup - 1, 0), max(0, fit - args.steps))
    steps = max(1, min(args.steps, fit - warm))
    for _ in range(warm):
        oracle_step(wl, H, W1, b1, w2, b2, layers)
    ts = [oracle_step(wl, H, W1, b1, w2, b2, layers)[0] for _ in range(steps)]
    t_step = sum(ts) / len(ts)
    value = wl.n_tok / t_step
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": steps, "warmup": 1 + warm, "ms_per_step": t_step * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    if steps != args.steps or 1 + warm != args.warmup:
        line["note"] = (f"{args.steps} steps after {args.warmup} warm-up steps were asked for; {steps} full steps "
                        f"after {1 + warm} warm-up step(s) fit the time budget and were timed")
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl):
    return {
        "workload": f"{wl.name}: N={'+'.join(map(str, wl.seqlens))}, question tail {'+'.join(map(str, wl.q_len))}, "
                    f"K={'+'.join(map(str, wl.k))}, d={wl.d}, gate {wl.d}->{wl.dg}->1 GELU, {wl.Hq}/{wl.Hkv} heads, "
                    f"head_dim {wl.D}, {wl.n_layers} above-L layer(s), {wl.dtype}",
        "global_batch": wl.B, "seq_len": max(wl.seqlens), "kept_rows": wl.m_tot,
        "parallelism": "replicas (one independent workload per GPU)",
        "l2": "flushed between timed steps (512 MiB memset, then a 256 MiB read sweep that evicts its dirty lines)",
    }


class L2Flush:
    """Leaves L2 holding only clean lines of an unrelated buffer: a 512 MiB memset, then a read of
    256 MiB more (a reduction), so the next kernel's reads neither hit in L2 nor wait behind the
    write-back of dirty lines."""

    def __init__(self, torch, dev):
        self.w = torch.empty(512 << 20, device=dev, dtype=torch.uint8)
        self.r = torch.zeros(64 << 20, device=dev, dtype=torch.float32)
        self.acc = torch.zeros((), device=dev, dtype=torch.float32)

    def __call__(self):
        self.w.zero_()
        self.acc.add_(self.r.sum())


class ChainBench:
    """Device buffers and the prepared C-ABI arguments of one workload's whole chain."""

    def __init__(self, tg, torch, np, dev, wl, stream):
        import tg_inputs as ti

        def bf(a):
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)

        self.wl = wl
        self.Hn = ti.hidden_states(wl)
        self.W1n, self.b1n, self.w2n, self.b2 = ti.gate_weights(wl)
        self.lay = [ti.qkv(wl, l) for l in range(wl.n_layers)]
        self.H_host = bf(self.Hn).pin_memory()
        self.qkv_host = [tuple(bf(x).pin_memory() for x in L) for L in self.lay]
        self.H = self.H_host.to(dev)
        self.W1, self.b1, self.w2 = bf(self.W1n).to(dev), torch.from_numpy(self.b1n).to(dev), bf(self.w2n).to(dev)
        self.layers = [tuple(x.to(dev) for x in L) for L in self.qkv_host]
        self.cu = tg.tg_kept_counts(wl.seqlens, wl.q_len, wl.k)
        M = self.M = self.cu[-1]
        self.scale = 1.0 / math.sqrt(wl.D)
        f32, i32 = torch.float32, torch.int32
        self.out = {"score": torch.empty(wl.n_tok, device=dev, dtype=f32),
                    "kept_idx": torch.empty(M, device=dev, dtype=i32),
                    "cu_kept_dev": torch.empty(wl.B + 1, device=dev, dtype=i32),
                    "H_kept": torch.empty(M, wl.d, device=dev, dtype=torch.bfloat16),
                    "pos": torch.empty(M, device=dev, dtype=i32), "g": torch.empty(M, device=dev, dtype=f32),
                    "logg": torch.empty(M, device=dev, dtype=f32),
                    "O": [torch.empty_like(L[0]) for L in self.layers], "lse": [None] * len(self.layers)}
        self.status = torch.zeros(1, device=dev, dtype=i32)
        self.stream = stream
        self.chain = tg.PreparedChain(self.H, self.W1, self.b1, self.w2, self.b2, wl.seqlens, wl.q_len, wl.k,
                                      self.layers, self.scale, self.out, dev_status=self.status, stream=stream)

    def stages(self, ev=None):
        """The four stage entry points one after another, with an event between kernels."""
        c, st = self.chain, self.stream
        if ev:
            ev[0].record(st)
        c.score()
        if ev:
            ev[1].record(st)
        c.select()
        if ev:
            ev[2].record(st)
        c.gather()
        if ev:
            ev[3].record(st)
        for li in range(len(self.layers)):
            c.attention(li)
        if ev:
            ev[4].record(st)

    def measure(self, torch, np, steps, warmup, flush, barrier):
        """Region A: whole steps through tg_prefill_above_L, events at step boundaries only (the
        metric). Region B: the stage entry points with events between kernels (per-kernel times)."""
        for _ in range(warmup):
            flush()
            self.stages()
            flush()
            self.chain.prefill()
        torch.cuda.synchronize()
        st = self.stream
        ev_a = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        barrier()
        torch.cuda.synchronize()
        for i in range(steps):
            flush()  # outside the timed events
            torch.cuda._sleep(200_000)  # keeps the host's launches ahead of the GPU (no idle gaps timed)
            ev_a[i][0].record(st)
            self.chain.prefill()
            ev_a[i][1].record(st)
        torch.cuda.synchronize()
        barrier()
        step_ms = np.array([e[0].elapsed_time(e[1]) for e in ev_a])
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
        barrier()
        torch.cuda.synchronize()
        for i in range(steps):
            flush()
            torch.cuda._sleep(200_000)
            self.stages(evs[i])
        torch.cuda.synchronize()
        barrier()
        st_ms = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(4)] for i in range(steps)])
        return step_ms, st_ms.mean(axis=0)

    def per_kernel(self, np, stage_ms, pk):
        wl, cu, M = self.wl, self.cu, self.M
        flops_attn = 4.0 * wl.Hq * wl.D * sum(m * (m + 1) / 2 for m in np.diff(cu))
        bytes_score = wl.n_tok * wl.d * 2 + wl.n_tok * 4 + wl.dg * wl.d * 2
        bytes_gather = M * wl.d * 2 * 2 + M * 4 * 4
        bytes_select = (wl.n_tok - sum(wl.q_len)) * 4 + M * 4
        out = {}
        for i, nm in enumerate(("score", "select", "gather", "gated_attn")):
            t_s = stage_ms[i] / 1e3 / (wl.n_layers if nm == "gated_attn" else 1)
            if nm == "gated_attn":
                e = {"bound": "tensor", "achieved": flops_attn / t_s / 1e12, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "algorithmic": flops_attn}
            else:
                byts = {"score": bytes_score, "select": bytes_select, "gather": bytes_gather}[nm]
                e = {"bound": "hbm", "achieved": byts / t_s / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "algorithmic": byts}
            e["frac"] = e["achieved"] / e["peak"]
            e["us"] = t_s * 1e6
            out[nm] = e
        return out


def other_workload(tg, torch, np, dev, name, steps, warmup, flush, pk):
    """Throughput of another configuration through the same entry point (rank 0 only)."""
    import tg_inputs as ti

    wl = ti.WORKLOADS[name]
    cb = ChainBench(tg, torch, np, dev, wl, torch.cuda.current_stream())
    step_ms, stage_ms = cb.measure(torch, np, steps, warmup, flush, lambda: None)
    ms = float(step_ms.mean())
    kern = cb.per_kernel(np, stage_ms, pk)
    res = {"config": workload_config(wl)["workload"], "steps": steps, "warmup": warmup, "ms_per_step": ms,
           "value": wl.n_tok / (ms / 1e3), "unit": "tokens/s",
           "stages_us": {n: float(x * 1e3) for n, x in zip(("score", "select", "gather", "gated_attn"), stage_ms)},
           "kernels": {k: {kk: v[kk] for kk in ("achieved", "unit", "frac", "us")} for k, v in kern.items()},
           "device_status": int(cb.status.item())}
    del cb
    torch.cuda.empty_cache()
    return res


def main():
    args = parse()
    import tg_inputs as ti

    wl = ti.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)

    import numpy as np
    import torch
    import torch.distributed as dist

    import learned_token_pruning_02_b200 as tg
    from learned_token_pruning_02_b200 import replicas

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    if args.bw_only:
        pk, _ = peaks()
        bw = bandwidth_instances(tg, torch, dev, pk["hbm_gbs"], args.bw_reps)
        if rank == 0:
            print(json.dumps({"bandwidth_instances": bw}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0

    # ---------------- inputs (seeded, identical on every rank: weak-scaling replicas)
    stream = torch.cuda.current_stream()
    cb = ChainBench(tg, torch, np, dev, wl, stream)
    flush = L2Flush(torch, dev)
    H, W1, b1, w2, b2, layers, out = cb.H, cb.W1, cb.b1, cb.w2, cb.b2, cb.layers, cb.out
    M, cu, scale, status = cb.M, cb.cu, cb.scale, cb.status
    launches_per_step = 4 + (wl.n_layers - 1)  # score, select, gather, attention per layer

    clocks = ClockSampler(local).start()
    step_ms, stage_ms = cb.measure(torch, np, args.steps, args.warmup, flush, barrier)
    clk = clocks.stop()
    t_total = replicas.max_over_ranks(float(step_ms.sum()), device=dev)
    ms_per_step = t_total / args.steps
    value = wl.n_tok * world * args.steps / (t_total / 1e3)
    dev_status = int(status.item())

    # ---------------- roofline of the dominant kernel
    pk, pk_src = peaks()
    per_kernel = cb.per_kernel(np, stage_ms, pk)
    names = ["score", "select", "gather", "gated_attn"]
    for nm in names:
        per_kernel[nm]["traffic"] = traffic_from_profile(nm, kernel_hash(nm))
    attn_tflops = per_kernel["gated_attn"]["achieved"]
    score_gbs = per_kernel["score"]["achieved"]
    dominant = names[int(np.argmax(stage_ms))]
    roof = {"kernel": dominant}
    roof.update({k: per_kernel[dominant][k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")})
    roof["peak_source"] = f"{pk_src} ({'burst' if roof['bound'] == 'tensor' else 'copy'})"

    # ---------------- end to end through the public API, host buffers in and out
    e2e = None
    if args.e2e_steps > 0:
        Os = out["O"]
        kept = out["kept_idx"]
        O_host = [torch.empty(L[0].shape, dtype=torch.bfloat16).pin_memory() for L in layers]
        kept_host = torch.empty(M, dtype=torch.int32).pin_memory()

        def e2e_step():
            H.copy_(cb.H_host, non_blocking=True)
            for (q, k, v), (qh, kh, vh) in zip(layers, cb.qkv_host):
                q.copy_(qh, non_blocking=True)
                k.copy_(kh, non_blocking=True)
                v.copy_(vh, non_blocking=True)
            tg.tg_prefill_above_L(H, W1, b1, w2, b2, wl.seqlens, wl.q_len, wl.k, layers, scale, out=out,
                                  dev_status=status)
            for o, oh in zip(Os, O_host):
                oh.copy_(o, non_blocking=True)
            kept_host.copy_(kept, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        t = replicas.max_over_ranks(e0.elapsed_time(e1), device=dev)
        h2d = H.numel() * 2 + sum(x.numel() * 2 for L in layers for x in L)
        d2h = sum(o.numel() * 2 for o in Os) + M * 4
        e2e = {"value": wl.n_tok * world * args.e2e_steps / (t / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": t / args.e2e_steps, "api": "tg_prefill_above_L", "steps": args.e2e_steps}

    # ---------------- unpruned causal attention at the full length (reference point)
    full_ref = None
    if not args.no_full_ref and rank == 0:
        n = max(wl.seqlens)
        gq = torch.Generator(device=dev).manual_seed(7)
        q = (torch.randn(n, wl.Hq, wl.D, device=dev, generator=gq) / math.sqrt(128)).to(torch.bfloat16)
        k = (torch.randn(n, wl.Hkv, wl.D, device=dev, generator=gq) / math.sqrt(128)).to(torch.bfloat16)
        v = (torch.randn(n, wl.Hkv, wl.D, device=dev, generator=gq) / math.sqrt(128)).to(torch.bfloat16)
        p = torch.arange(n, device=dev, dtype=torch.int32)
        o = torch.empty_like(q)
        reps = 3
        tg.tg_gated_attn_fwd(q, k, v, None, p, [0, n], scale, O=o, want_lse=False)
        torch.cuda.synchronize()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(reps):
            tg.tg_gated_attn_fwd(q, k, v, None, p, [0, n], scale, O=o, want_lse=False)
        a1.record(stream)
        torch.cuda.synchronize()
        ms = a0.elapsed_time(a1) / reps
        fl = 4.0 * wl.Hq * wl.D * n * (n + 1) / 2
        full_ref = {"n": n, "ms": ms, "tflops": fl / (ms / 1e3) / 1e12,
                    "note": "unpruned causal attention over all N tokens (g == 1), same kernel"}
        del q, k, v, o

    # ---------------- the same chain replayed from a CUDA graph (captured once, launch edges kept)
    graph = None
    try:
        g_stream = torch.cuda.Stream(device=dev)
        g_chain = tg.PreparedChain(H, W1, b1, w2, b2, wl.seqlens, wl.q_len, wl.k, layers, scale, out,
                                   dev_status=status, stream=g_stream)
        cg = torch.cuda.CUDAGraph()
        g_stream.wait_stream(stream)
        with torch.cuda.stream(g_stream):
            g_chain.prefill()  # warm the capture stream's path once outside the graph
            torch.cuda.synchronize()
            with torch.cuda.graph(cg, stream=g_stream):
                g_chain.prefill()
        torch.cuda.synchronize()
        for _ in range(args.warmup):
            flush()
            cg.replay()
        torch.cuda.synchronize()
        ev_g = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
        for i in range(args.steps):
            flush()
            torch.cuda._sleep(200_000)
            ev_g[i][0].record(stream)
            cg.replay()
            ev_g[i][1].record(stream)
        torch.cuda.synchronize()
        g_local = float(sum(e[0].elapsed_time(e[1]) for e in ev_g))
        del cg
    except Exception as ex:  # capture is optional evidence; the metric above does not depend on it
        g_local = float("inf")
        graph = {"value": None, "error": f"{type(ex).__name__}: {ex}"[:200]}
    # every rank takes this collective whether or not its capture worked
    barrier()
    g_ms = replicas.max_over_ranks(g_local, device=dev) / args.steps
    if graph is None and g_ms != float("inf"):
        graph = {"value": wl.n_tok * world / (g_ms / 1e3), "unit": "tokens/s", "ms_per_step": g_ms,
                 "note": "tg_prefill_above_L captured once into a CUDA graph and replayed per step"}
    elif graph is None:
        graph = {"value": None, "error": "capture failed on another rank"}

    # ---------------- byte-heavy select/gather instances (bandwidth evidence)
    bw = None
    if not args.no_bw:
        barrier()
        bw = bandwidth_instances(tg, torch, dev, pk["hbm_gbs"], args.bw_reps)

    split_t = split_select_times(tg, torch, dev, 20) if not args.no_bw else None
    qkv_t = (qkv_rope_time(tg, torch, dev, out["H_kept"], out["pos"], wl.Hq, wl.Hkv, wl.D, pk["bf16_tflops"], 20)
             if not args.no_bw else None)
    bwd_t = (attn_bwd_time(tg, torch, dev, *layers[0], out["logg"], out["pos"], list(cu), scale, pk["bf16_tflops"], 5)
             if not args.no_bw else None)

    proj_t = projected_chain_time(tg, torch, dev, cb, flush, 20) if not args.no_bw else None
    gbwd_t = gate_bwd_time(tg, torch, dev, cb, 20) if not args.no_bw else None

    # ---------------- the other configurations, through the same entry point (rank 0)
    others = None
    if rank == 0 and not args.no_other:
        others = {}
        for name in ("qwen3_8k", "qwen3_128k", "ragged4"):
            if name != wl.name:
                others[name] = other_workload(tg, torch, np, dev, name, 20, 3, flush, pk)

    # ---------------- CPU oracle baseline (rank 0, N = 1 only): one whole oracle step
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t_cpu, desc = oracle_step(wl, cb.Hn, cb.W1n, cb.b1n, cb.w2n, cb.b2, cb.lay)
        cpu = {"value": wl.n_tok / t_cpu, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
               "sample": desc, "seconds": t_cpu, "host_cpus": os.cpu_count()}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; Qwen3-1.7B shapes)",
            "config": workload_config(wl),
            "stages_us": {n: float(x * 1e3) for n, x in zip(names, stage_ms)},
            "gated_attn_tflops": attn_tflops,
            "gated_attn_frac_of_bf16_peak": attn_tflops / pk["bf16_tflops"],
            "score_hbm_gbs": score_gbs,
            "roofline": roof,
            "kernels": per_kernel,
            "cpu_baseline": cpu,
            "e2e": e2e,
            # timed regions A, B and the graph replays together
            "gpu_launches": (3 if graph.get("value") else 2) * launches_per_step * args.steps,
            "stages_sum_us": float(stage_ms.sum() * 1e3),
            "clocks": clk,
            "full_attention_reference": full_ref,
            "other_workloads": others,
            "bandwidth_instances": bw,
            "graph_replay": graph,
            "split_select": split_t,
            "qkv_rope": qkv_t,
            "gated_attn_bwd": bwd_t,
            "projected_chain": proj_t,
            "gate_mlp_bwd": gbwd_t,
            "device_status": dev_status,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
