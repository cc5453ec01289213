#!/usr/bin/env python
"""Routed-decode benchmark of the Memory Sparse Attention hot path on one B200.

One step = one routing layer's whole hot path for one decode token over the
100M-token memory: route (prep, Kr scan over all 1.56M pooled chunks, Top-k,
certified fp64 re-scoring) -> fetch of the selected documents' pooled K/V from
pinned host memory -> sparse GQA decode over [pooled K/V ++ 4097 local
tokens].  Consecutive steps stand for consecutive routing layers with their
own queries, issued on two alternating streams: step s+1's route runs while
step s's fetch crosses the host link, as the pages describe ("content K/V ...
fetched asynchronously when selected"), and step s's latency-bound Top-k,
re-scoring and decode run beside step s+1's bandwidth-bound Kr scan.  The
end-to-end figure ("e2e") runs the same pipelined steps through host
buffers (per-step copies in and out), timed by the host clock.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference]

Prints one JSON line (rank 0).  With N > 1 (torchrun), every rank runs an
independent replica on its own GPU ("replicas only": the path has no
cross-GPU exchange) and the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import BY_NAME, MEM_100M, gen  # noqa: E402

METRIC = "Kr routing scan GB/s + routed decode tokens/s at 16M/100M-token memory"
# memories whose scan and decode rooflines every default run reports
STAGE_WORKLOADS = ("16m-bf16-lognormal-65536docs", "100m-bf16-390625x256-hosttier", "16m-bf16-lognormal-batch32",
                   "1m-bf16-4096x256-T64")
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="msa", choices=["msa", "reference"])
    ap.add_argument("--workload", default=MEM_100M.name, choices=sorted(BY_NAME))
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-stage-rooflines", action="store_true",
                    help="skip the per-kernel rooflines at the 16M, 100M and batch-32 memories")
    ap.add_argument("--stage", default="step",
                    choices=["step", "encode", "route", "decode", "loop", "interleave", "stream_encode", "train"],
                    help="step: the whole hot path (default); otherwise one stage alone; loop: several "
                         "routing layers per generated token through runtime.RoutedDecodeLoop")
    ap.add_argument("--layers", type=int, default=2, help="routing layers of --stage loop")
    ap.add_argument("--docs", type=int, default=0,
                    help="stage runs only: the first N documents of the workload (e.g. a small bank for a profile)")
    ap.add_argument("--batch-tokens", type=int, default=262144, help="tokens per push, --stage stream_encode")
    ap.add_argument("--rounds", type=int, default=4, help="retrieval rounds per question, --stage interleave")
    ap.add_argument("--per-round", type=int, default=8, help="documents added per round, --stage interleave")
    ap.add_argument("--round-tokens", type=int, default=4, help="tokens generated per round, --stage interleave")
    return ap.parse_args()


# ------------------------------------------------------------------ replicas

def replica_env():
    """(rank, world size, local rank) as torchrun sets them; (0, 1, 0) alone."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, world: int, device) -> float:
    """The job's time is the slowest replica's: max of x over all ranks (every
    rank takes part and gets the result); x itself when alone."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ helpers

def peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            v = float(json.load(open(p))["hbm_gbs"])
            return v, "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


def peak_bf16_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            return float(json.load(open(p))["bf16_tflops"]), "measured"
        except Exception:
            pass
    return 1590.0, "fallback"


# source files each kernel is built from: an ncu traffic record counts only
# while their hash matches the one it was taken on
KERNEL_SOURCES = {
    "kr_scan_kernel": ("route.cuh", "msa_common.cuh"),
    "kr_scan_mma_kernel": ("route_mma.cuh", "msa_common.cuh"),
    "decode_mma_kernel": ("decode_mma.cuh", "decode.cuh", "msa_common.cuh"),
    "decode_tc_kernel": ("decode_tc.cuh", "decode_mma.cuh", "decode.cuh", "route_mma.cuh", "msa_common.cuh"),
}


def decode_kernel_name(w) -> str:
    """The decode kernel the library's plan picks for workload `w`: bf16 banks
    with head_dim 128 and more than 64 query rows per kv head (whole tokens of
    a group size of at least 4 that divides 128) run on tcgen05, other bf16
    banks on mma.sync, fp32 banks on the CUDA cores."""
    if w.dtype != "bf16":
        return "decode_kernel"
    G = w.n_q_heads // w.n_kv_heads
    if w.head_dim == 128 and G * w.T > 64 and G >= 4 and 128 % G == 0:
        return "decode_tc_kernel"
    return "decode_mma_kernel"


def kernel_source_sha(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "routed_sparse_attention_b200", "csrc", f), "rb").read())
    return h.hexdigest()


def kernel_traffic(kernel: str, workload: str):
    """ncu DRAM bytes (read + write) per launch of `kernel` on `workload`, from
    profiles/traffic.json, if taken on the kernel's current source; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(kernel)
    if not rec or rec.get("source_sha256") != kernel_source_sha(kernel):
        return None
    by = rec.get("bytes_per_launch", {})
    return by.get(workload)


def scan_traffic():
    """ncu DRAM bytes per scan launch on the 100M bank (see kernel_traffic)."""
    return kernel_traffic("kr_scan_kernel", MEM_100M.name)


class Clocks:
    """nvidia-smi samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: str):
        self.path = tempfile.mktemp(suffix=".csv")
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def workload_config(w, world: int) -> dict:
    """The `config` of both arms' JSON lines, from the workload alone."""
    L = gen.doc_lengths(w)
    loc = gen.local_lengths(w)
    return {"workload": w.name, "memory_tokens": int(L.sum()), "docs": w.n_docs,
            "pooled_chunks": int(((L + w.chunk - 1) // w.chunk).sum()), "batch": w.B, "T": w.T,
            "top_k": w.top_k, "local_ctx": int(loc.max()) if w.B == 1 else [int(loc.min()), int(loc.max())],
            "kv_tier": "pinned host" if w.kv_on_host else "hbm", "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2: the whole Kr bank is streamed every step"}


# ------------------------------------------------------------------ the oracle baseline

def cpu_baseline(w, kr_first_docs, seconds: float, one_thread: bool = True):
    """Time the fp64 oracle (as it stands) on the host cores on a bounded
    sample: routing over the first docs of the bank, scaled to the whole bank
    by chunk count, plus one full decode step; with one_thread, also on a
    single thread.  kr_first_docs(n) returns the pooled router keys of the
    bank's first n documents (host tensor)."""
    import oracle
    L = gen.doc_lengths(w)
    tok = gen.offsets(L)
    coff = oracle.chunk_offsets(tok, w.chunk)
    qs = gen.make_queries(w.replace(B=1), "cpu")
    # calibrate: route over a small slice, then size the sample to ~seconds
    def route_slice(n_docs):
        c = int(coff[n_docs])
        kr = kr_first_docs(n_docs)
        t0 = time.perf_counter()
        oracle.route(qs["qr"], coff[:n_docs + 1], kr, min(w.top_k, n_docs), w.n_kv_heads)
        return time.perf_counter() - t0, c
    probe = max(w.top_k, min(w.n_docs, 2048))
    t, c = route_slice(probe)
    n = int(min(w.n_docs, max(probe, probe * seconds * 0.8 / max(t, 1e-3))))
    t, c = route_slice(n)
    t_route = t * (int(coff[-1]) / c)
    # one decode step on the full local context against the sampled docs
    sel = np.arange(w.top_k, dtype=np.int32)[None]
    kv = gen.make_memory(w.replace(n_docs=w.top_k, n_needles=0), qs["qr"], "cpu")
    lk, lv = qs["local_k"][: int(qs["local_off"][1]) * w.n_kv_heads * w.head_dim], \
        qs["local_v"][: int(qs["local_off"][1]) * w.n_kv_heads * w.head_dim]
    kcoff = oracle.chunk_offsets(kv["doc_tok_off"], w.chunk)
    t0 = time.perf_counter()
    oracle.decode(qs["q"][:1], sel, kcoff, kv["k_pool"], kv["v_pool"], qs["local_off"][:2], lk, lv,
                  w.top_k, w.rope_theta, w.n_kv_heads)
    t_dec = time.perf_counter() - t0
    step = t_route + t_dec
    cores = oracle.threads()
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            model = next((ln.split(":", 1)[1].strip() for ln in f if ln.startswith("model name")), None)
    except OSError:
        pass
    res = {"value": w.T / step, "unit": "tokens/s", "cores": cores, "kind": "oracle", "cpu_model": model,
           "sample": (f"routing over the first {n} of {w.n_docs} documents ({c} of {int(coff[-1])} "
                      f"pooled chunks) in {t:.2f} s, scaled by chunk count; one full decode "
                      f"step ({t_dec * 1e3:.1f} ms); 1 query token"),
           "seconds_per_step": step}
    if not one_thread:
        return res
    # the same kind of sample on one thread, sized to about a quarter of the time
    oracle.set_threads(1)
    try:
        t1, c1 = route_slice(probe)
        n1 = int(min(w.n_docs, max(probe, probe * seconds * 0.25 / max(t1, 1e-3))))
        if n1 != probe:
            t1, c1 = route_slice(n1)
        t0 = time.perf_counter()
        oracle.decode(qs["q"][:1], sel, kcoff, kv["k_pool"], kv["v_pool"], qs["local_off"][:2], lk, lv,
                      w.top_k, w.rope_theta, w.n_kv_heads)
        t_dec1 = time.perf_counter() - t0
    finally:
        oracle.set_threads(cores)
    step1 = t1 * (int(coff[-1]) / c1) + t_dec1
    res.update({"value_1thread": w.T / step1, "seconds_per_step_1thread": step1,
                "sample_1thread": (f"routing over the first {n1} documents ({c1} pooled chunks) in {t1:.2f} s "
                                   f"on one thread, scaled by chunk count; one decode step "
                                   f"({t_dec1 * 1e3:.1f} ms)")})
    return res


def run_reference(args, rank):
    """The reference arm: the CPU oracle, timed as it stands on the host cores."""
    if rank != 0:
        return
    import oracle
    w = BY_NAME[args.workload]
    L = gen.doc_lengths(w)
    qr = gen.make_queries(w, "cpu")["qr"]

    def kr_rows(n_docs):
        sub = w.replace(n_docs=n_docs, kv_on_host=False, per_token=False,
                        n_needles=min(w.n_needles, n_docs))
        return gen.make_memory(sub, qr, "cpu")["kr_pool"]

    steps = []
    base = first = None
    for i in range(args.warmup + args.steps):
        b = cpu_baseline(w, kr_rows, args.cpu_seconds if i == 0 else min(args.cpu_seconds, 4.0), one_thread=i == 0)
        if i >= args.warmup:
            steps.append(b["seconds_per_step"])
        base = b
        first = first or b
    sec = float(np.mean(steps))
    val = w.B * w.T / sec
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args.gpus),
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": base["cores"],
                             "kind": "oracle", "sample": base["sample"], "cpu_model": base["cpu_model"],
                             "value_1thread": first["value_1thread"], "sample_1thread": first["sample_1thread"]},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ the GPU arm

def run_msa(args, rank, world):
    import routed_sparse_attention_b200 as msa
    from routed_sparse_attention_b200 import Layout
    from routed_sparse_attention_b200.runtime import Bank, Decoder, Router

    w = BY_NAME[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    x = gen.generate(w, device=dev, host_interleaved=w.kv_on_host)
    layout = Layout.of(w)
    bank = Bank(layout, x["doc_tok_off"], kr_pool=x.get("kr_pool"), k_pool=x.get("k_pool"),
                v_pool=x.get("v_pool"), host_kv=x.get("host_kv"), device=dev) if not w.per_token else \
        Bank(layout, x["doc_tok_off"], k_tok=x["k_tok"], v_tok=x["v_tok"], kr_tok=x["kr_tok"], device=dev)
    routers = [Router(bank, w.B, w.T, w.top_k, dev) for _ in range(2)]
    decoders = [Decoder(bank, w.B, w.T, w.top_k, x["local_off"], dev) for _ in range(2)]
    # two query sets so consecutive steps route different queries
    qsets = [(x["qr"], x["q"])]
    q2 = gen.make_queries(w.replace(seed=w.seed + 1), dev)
    qsets.append((q2["qr"], q2["q"]))
    lk, lv = x["local_k"], x["local_v"]
    # each stream's rotated key cache (global RoPE at top_k + j), built once
    # like a prefill; every step rotates only its T new tokens into it
    caches = [decoders[j].rotate_local(lk, torch.empty_like(lk)) for j in range(2)]
    s_main, s_fetch = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    torch.cuda.synchronize()

    def mk_event(timing=False):
        e = torch.cuda.Event(enable_timing=timing)
        e.record(s_main)
        return e

    ev_sel = [mk_event(), mk_event()]
    ev_fetch = [mk_event(), mk_event()]

    # Consecutive steps (routing layers) alternate between two compute
    # streams, so one layer's latency-bound Top-k, re-scoring and decode run
    # beside the next layer's bandwidth-bound Kr scan; each step's own kernels
    # stay in order on its stream.
    streams = [s_main, torch.cuda.Stream(dev)]

    def finish(i, j, q, dec_ev):
        st = streams[j]
        if bank.host_tier:
            decoders[j].fetch(routers[j].idx_host, ev_sel[j], s_fetch, ev_fetch[j])
            st.wait_event(ev_fetch[j])
        if dec_ev is not None:
            dec_ev[i][0].record(st)
        decoders[j].rotate_local(lk, caches[j], new_tokens=w.T, stream=st)
        decoders[j](q, caches[j], lv, routers[j].idx, stream=st)
        if dec_ev is not None:
            dec_ev[i][1].record(st)

    def pipeline(n, scan_ev, dec_ev=None):
        prev = None
        for i in range(n):
            j = i % 2
            qr, q = qsets[i % 2]
            msa.scan_events(*scan_ev[i])
            routers[j](qr, stream=streams[j])
            ev_sel[j].record(streams[j])
            if prev is not None:
                finish(*prev, dec_ev)
            prev = (i, j, q)
        if prev is not None:
            finish(*prev, dec_ev)
        msa.scan_events()
        s_main.wait_stream(streams[1])

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    # warm-up (untimed), then K timed steps
    pipeline(args.warmup, [(mk_event(True), mk_event(True)) for _ in range(args.warmup)])
    torch.cuda.synchronize()
    K = args.steps
    scan_ev = [(mk_event(True), mk_event(True)) for _ in range(K)]
    dec_ev = [(mk_event(True), mk_event(True)) for _ in range(K)]
    t0, t1 = mk_event(True), mk_event(True)
    torch.cuda.synchronize()
    visible = [v for v in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if v]
    clocks = Clocks(visible[dev.index] if dev.index < len(visible) else str(dev.index))
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record(s_main)
    pipeline(K, scan_ev, dec_ev)
    t1.record(s_main)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier()
    ms = t0.elapsed_time(t1)
    scan_ms = [a.elapsed_time(b) for a, b in scan_ev]
    # Consecutive scans overlap at their edges (two streams), so a launch's own
    # start-to-stop time counts the neighbour it shares the GPU with.  The time
    # per scan is the span from the first scan's start to the last scan's stop,
    # divided by K; scans cover that whole span back to back.
    scan_span_ms = max(scan_ev[0][0].elapsed_time(b) for _, b in scan_ev)
    dec_ms = [a.elapsed_time(b) for a, b in dec_ev]
    status = msa.device_status(s_main)
    ms = max_over_ranks(ms, world, dev)

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(w, bank, routers, decoders, x, caches, dev, streams, s_fetch, ev_sel, ev_fetch, max(4, K))

    # ---- the same layers without overlap between them
    dep = dependent_layers(w, bank, routers[0], decoders[0], x, caches[0], qsets[0][1], qsets[0][0], s_main,
                           s_fetch, max(4, K))
    if bank.host_tier:
        dep["device_fetch"] = dependent_layers(w, bank, routers[0], decoders[0], x, caches[0], qsets[0][1],
                                               qsets[0][0], s_main, s_fetch, max(4, K), device_fetch=True)

    # ---- each kernel on its own after an L2 flush: the scan and the decode at
    #      the 16M, 100M and batch-32 memories
    flush = L2Flush(dev)
    rooflines, stage_us = [], {}
    if not args.no_stage_rooflines:
        rl, us = kernel_rooflines(w, bank, x, dev, flush, K, args.warmup)
        rooflines += rl
        stage_us[w.name] = us
        for name in STAGE_WORKLOADS:
            if name == w.name:
                continue
            wo = BY_NAME[name]
            if wo.per_token:                   # the pooled bank of that shape, generated directly
                wo = wo.replace(per_token=False)
            xo = gen.generate(wo, device=dev, host_interleaved=wo.kv_on_host)
            bo = Bank(Layout.of(wo), xo["doc_tok_off"], kr_pool=xo["kr_pool"], k_pool=xo.get("k_pool"),
                      v_pool=xo.get("v_pool"), host_kv=xo.get("host_kv"), device=dev)
            rl, us = kernel_rooflines(wo, bo, xo, dev, flush, K, args.warmup)
            rooflines += rl
            stage_us[name] = us
            del xo, bo
            torch.cuda.empty_cache()

    C, D = bank.n_chunks, bank.n_docs
    esz = 2 if w.dtype == "bf16" else 4
    scan_bytes = C * w.n_kv_heads * w.router_dim * esz + D * 12   # Kr + CSR + doc scores
    avg_scan_s = scan_span_ms / K / 1e3
    peak, peak_kind = peak_hbm()
    achieved = scan_bytes / avg_scan_s / 1e9
    tokens = w.B * w.T * K * world
    value = tokens / (ms / 1e3)
    ltot = int(x["local_off"][1] - x["local_off"][0])
    cfg = workload_config(w, world)
    assert cfg["memory_tokens"] == int(x["doc_tok_off"][-1]) and cfg["pooled_chunks"] == C
    assert cfg["local_ctx"] == ltot - w.T
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": cfg,
        "value_is": ("consecutive routing layers pipelined on two streams (a layer's selection, fetch and "
                     "decode beside the next layer's scan); see dependent_step for layers without overlap"),
        "dependent_step": dep,
        "rooflines": rooflines, "stage_us": stage_us,
        "kr_scan_gbs": achieved, "kr_scan_us": avg_scan_s * 1e6,
        "kr_scan_us_per_launch_overlapped": float(np.mean(scan_ms)) * 1e3,
        "decode_us_overlapped": float(np.mean(dec_ms)) * 1e3,
        "roofline": {"kernel": "kr_scan_kernel", "bound": "hbm", "achieved": achieved, "peak": peak,
                     "unit": "GB/s", "frac": achieved / peak, "peak_kind": f"{peak_kind} (hbm_gbs)",
                     "traffic": scan_traffic(), "algorithmic_bytes_per_launch": scan_bytes},
        # per step: route_prep, kr_scan, topk_local, merge_band, rescore,
        # final_select, rope_local (the new token's key), decode
        "gpu_launches": 8 * K,
        "device_status": status,
        "e2e": e2e,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        def kr_rows(n_docs):
            return bank.kr[:int(bank.doc_chunk_off_host[n_docs])].cpu()
        line["cpu_baseline"] = cpu_baseline(w, kr_rows, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(w, bank, routers, decoders, x, caches, dev, streams, s_fetch, ev_sel, ev_fetch, steps):
    """End to end through the public API with host buffers, pipelined like
    the device step (consecutive routing layers alternate between two
    streams).  Per step: pinned host -> device copies of the router query,
    the decode query and the T new tokens' K/V (into that stream's local
    K/V), route, host-tier fetch (the host waits for that step's indices
    while the other stream routes the next layer), the new keys' rotation
    into the key cache, decode, and device -> host reads of the output and
    the selected documents.  Timed by the host clock from the first copy to
    the completion of the last read."""
    H, d, T, B = w.n_kv_heads, w.head_dim, w.T, w.B
    loff = x["local_off"]
    h_qr = x["qr"].cpu().pin_memory()
    h_q = x["q"].cpu().pin_memory()
    new_k = torch.empty(B, H, T, d, dtype=x["local_k"].dtype).pin_memory()
    new_v = torch.empty_like(new_k).pin_memory()
    for b in range(B):
        lt = int(loff[b + 1] - loff[b])
        new_k[b].copy_(x["local_k"][int(loff[b]) * H * d:int(loff[b + 1]) * H * d].view(H, lt, d)[:, lt - T:])
        new_v[b].copy_(x["local_v"][int(loff[b]) * H * d:int(loff[b + 1]) * H * d].view(H, lt, d)[:, lt - T:])
    per = []
    for j in range(2):
        raw_k, raw_v = x["local_k"].clone(), x["local_v"].clone()
        vk, vv = [], []
        for b in range(B):
            lt = int(loff[b + 1] - loff[b])
            a0, a1 = int(loff[b]) * H * d, int(loff[b + 1]) * H * d
            vk.append(raw_k[a0:a1].view(H, lt, d)[:, lt - T:])
            vv.append(raw_v[a0:a1].view(H, lt, d)[:, lt - T:])
        per.append(dict(d_qr=torch.empty_like(x["qr"]), d_q=torch.empty_like(x["q"]), raw_k=raw_k, raw_v=raw_v,
                        vk=vk, vv=vv,
                        out_h=torch.empty(decoders[j].out.shape, dtype=decoders[j].out.dtype).pin_memory(),
                        idx_h=torch.empty(B, w.top_k, dtype=torch.int32).pin_memory()))

    def route(j):
        st, p = streams[j], per[j]
        with torch.cuda.stream(st):
            p["d_qr"].copy_(h_qr, non_blocking=True)
            p["d_q"].copy_(h_q, non_blocking=True)
            for b in range(B):
                p["vk"][b].copy_(new_k[b], non_blocking=True)
                p["vv"][b].copy_(new_v[b], non_blocking=True)
        routers[j](p["d_qr"], stream=st)
        ev_sel[j].record(st)

    def finish(j):
        st, p = streams[j], per[j]
        if bank.host_tier:
            decoders[j].fetch(routers[j].idx_host, ev_sel[j], s_fetch, ev_fetch[j])
            st.wait_event(ev_fetch[j])
        decoders[j].rotate_local(p["raw_k"], caches[j], new_tokens=T, stream=st)
        out = decoders[j](p["d_q"], caches[j], p["raw_v"], routers[j].idx, stream=st)
        with torch.cuda.stream(st):
            p["out_h"].copy_(out, non_blocking=True)
            p["idx_h"].copy_(routers[j].idx, non_blocking=True)

    def run(n):
        prev = None
        for i in range(n):
            j = i % 2
            route(j)
            if prev is not None:
                finish(prev)
            prev = j
        if prev is not None:
            finish(prev)
        torch.cuda.synchronize()

    run(2)
    t0 = time.perf_counter()
    run(steps)
    wall = time.perf_counter() - t0
    h2d = (h_qr.numel() * h_qr.element_size() + h_q.numel() * h_q.element_size()
           + 2 * new_k.numel() * new_k.element_size())
    d2h = per[0]["out_h"].numel() * per[0]["out_h"].element_size() + per[0]["idx_h"].numel() * 4
    return {"value": B * T * steps / wall, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": steps, "timing": "host clock, pipelined over two streams",
            "fetch_h2d_bytes_per_step": int(2 * w.top_k * 4 * H * d * 2) if bank.host_tier else 0}

class L2Flush:
    """Before each timed run: write a buffer larger than L2, then read another
    one, so that L2 holds only clean lines of unrelated data (the write alone
    leaves 126 MB of dirty lines whose write-back the timed kernel would pay)."""

    def __init__(self, dev, mib: int = 256):
        self.w = torch.empty(mib << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones((mib << 20) // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.fill_(1)
        self.r.sum()


def iq_mean(xs) -> float:
    """Mean of the samples between the 25th and 75th percentiles.  CUDA
    events tick in about 0.5 us, so a median of microsecond launches sits on
    a tick; the interquartile mean keeps the median's indifference to stray
    samples and resolves below a tick."""
    v = np.sort(np.asarray(xs, dtype=np.float64))
    lo, hi = len(v) // 4, len(v) - len(v) // 4
    return float(v[lo:hi].mean()) if hi > lo else float(v.mean())


def launch_time(fn, flush, K: int, W: int, inner=None) -> tuple:
    """Interquartile mean (iq_mean) over K runs of fn() timed with CUDA
    events on the current stream, the L2 flushed (flush()) before each; with
    inner = (start, stop) events that fn records around one launch, also that
    launch's own time."""
    for _ in range(W):
        fn()
    ts, ti = [], []
    for _ in range(K):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b) / 1e3)
        if inner is not None:
            ti.append(inner[0].elapsed_time(inner[1]) / 1e3)
    return iq_mean(ts), (iq_mean(ti) if ti else None)


def decode_bytes(w, bank, sel: np.ndarray, local_off) -> int:
    """Algorithmic bytes of one decode call: every key and value row it must
    read (pooled rows of the selected documents' chunks, live local rows) plus
    the query and the output."""
    esz = 2 if w.dtype == "bf16" else 4
    coff = bank.doc_chunk_off_host.numpy()
    n_mem = np.array([sum(int(coff[d + 1] - coff[d]) for d in row) for row in sel])
    lens = np.diff(np.asarray(local_off))
    return int(((n_mem + lens) * 2 * w.head_dim * esz * w.n_kv_heads).sum()
               + 2 * w.B * w.T * w.n_q_heads * w.head_dim * esz)


def back_to_back_decode(dec, q, k_cache, v_cache, idx, reps: int = 5) -> tuple:
    """Seconds per decode when decodes run back to back: one call per local
    cache over R copies of the caches (R x their bytes > 2 x the 126 MB L2, so
    no call finds its predecessor's rows in L2), recorded in a CUDA graph and
    replayed `reps` times; returns (seconds per decode, R)."""
    cache_bytes = (k_cache.numel() * k_cache.element_size() + v_cache.numel() * v_cache.element_size())
    R = int(min(32, max(1, -(-2 * 126 * 2 ** 20 // max(cache_bytes, 1)))))
    ks = [k_cache] + [k_cache.clone() for _ in range(R - 1)]
    vs = [v_cache] + [v_cache.clone() for _ in range(R - 1)]
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for r in range(R):
            dec(q, ks[r], vs[r], idx)
    torch.cuda.current_stream().wait_stream(side)
    g.replay()                                           # warm-up
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        g.replay()
    b.record()
    b.synchronize()
    sec = a.elapsed_time(b) / 1e3 / (reps * R)
    del g, ks, vs
    torch.cuda.empty_cache()
    return sec, R


def decode_flops(w, bank, sel: np.ndarray, local_off) -> float:
    """Useful arithmetic of one decode call: S = q.k and O += p v, 2 d flops
    each, per visible (query row, key) pair; query token t of query b sees
    the selected documents' pooled rows and local keys j <= L_b + t."""
    coff = bank.doc_chunk_off_host.numpy()
    n_mem = np.array([sum(int(coff[d + 1] - coff[d]) for d in row) for row in sel])
    lens = np.diff(np.asarray(local_off))                    # live local rows L_b + T
    T = w.T
    pairs = sum(T * int(n_mem[b]) + sum(int(lens[b]) - T + t + 1 for t in range(T)) for b in range(w.B))
    return 4.0 * w.head_dim * w.n_q_heads * pairs


def kernel_rooflines(w, bank, x, dev, flush, K: int, W: int) -> tuple:
    """The routing scan and the sparse decode of workload w, each launched on
    its own after an L2 flush and timed with CUDA events (interquartile mean of K): one
    roofline entry per kernel, plus the route (scan + selection) time."""
    import routed_sparse_attention_b200 as msa
    from routed_sparse_attention_b200.runtime import Decoder, Router
    peak, peak_kind = peak_hbm()
    esz = 2 if w.dtype == "bf16" else 4
    router = Router(bank, w.B, w.T, w.top_k, dev)
    sev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    sev[0].record()          # torch creates an event's CUDA handle on its first record
    sev[1].record()

    def route():
        msa.scan_events(*sev)
        router(x["qr"])
        msa.scan_events()
    route_s, scan_s = launch_time(route, flush, K, W, inner=sev)
    nq = w.B * w.T
    scan_kernel = "kr_scan_mma_kernel" if (w.dtype == "bf16" and nq > 4) else "kr_scan_kernel"
    scan_bytes = bank.n_chunks * w.n_kv_heads * w.router_dim * esz + bank.n_docs * 12
    idx, _ = router(x["qr"])
    dec = Decoder(bank, w.B, w.T, w.top_k, x["local_off"], dev)
    if bank.host_tier:
        s = torch.cuda.current_stream()
        e1, e2 = torch.cuda.Event(), torch.cuda.Event()
        e1.record(s)
        e2.record(s)
        dec.fetch(router.idx_host, e1, s, e2)
    k_cache = dec.rotate_local(x["local_k"], torch.empty_like(x["local_k"]))
    torch.cuda.synchronize()
    dbytes = decode_bytes(w, bank, idx.cpu().numpy(), x["local_off"])
    dec_s, _ = launch_time(lambda: dec(x["q"], k_cache, x["local_v"], idx), flush, K, W)
    try:
        b2b_s, b2b_r = back_to_back_decode(dec, x["q"], k_cache, x["local_v"], idx)
        b2b_err = None
    except Exception as ex:  # reported in the line; the isolated figure stands on its own
        b2b_s, b2b_r, b2b_err = None, 0, f"{type(ex).__name__}: {ex}"[:200]
        torch.cuda.synchronize()
    dec_kernel = decode_kernel_name(w)
    # what one launch costs on this GPU under the same flush and events: a
    # one-element op, and a plain library read of the decode's bytes
    one = torch.zeros(1, dtype=torch.float32, device=dev)
    plain = torch.ones(dbytes // 2, dtype=torch.bfloat16, device=dev)
    empty_s, _ = launch_time(lambda: one.add_(1), flush, K, W)
    plain_s, _ = launch_time(lambda: plain.sum(), flush, K, W)
    del plain
    timing = ("CUDA events around the one launch; before each, 256 MiB written then 256 MiB of another "
              "buffer read (L2 holds no input); interquartile mean of K")
    out = []
    for kern, nbytes, sec, per in ((scan_kernel, scan_bytes, scan_s, "route call (all query rows)"),
                                   (dec_kernel, dbytes, dec_s,
                                    "decode call" + (" (with its split merge kernel)" if dec_kernel == "decode_tc_kernel"
                                                     else ""))):
        ach = nbytes / sec / 1e9
        out.append({"kernel": kern, "workload": w.name, "bound": "hbm", "algorithmic_bytes": nbytes,
                    "per": per, "us": sec * 1e6, "achieved": ach, "peak": peak, "unit": "GB/s",
                    "frac": ach / peak, "peak_kind": f"{peak_kind} (hbm_gbs)",
                    "traffic": kernel_traffic(kern, w.name), "timing": timing})
    if dec_kernel == "decode_tc_kernel":
        # many query rows per kv head (T = 64: ~260 flop per byte, near the
        # tensor ridge): the roof is the tensor pipe; the HBM fraction stays beside it
        fl = decode_flops(w, bank, idx.cpu().numpy(), x["local_off"])
        tpk, tkind = peak_bf16_tflops()
        e = out[-1]
        e["hbm"] = {"achieved": e["achieved"], "peak": e["peak"], "unit": "GB/s", "frac": e["frac"]}
        e.update({"bound": "tensor", "flops": fl, "achieved": fl / dec_s / 1e12, "peak": tpk, "unit": "TFLOP/s",
                  "frac": fl / dec_s / 1e12 / tpk, "peak_kind": f"{tkind} (bf16_tflops)"})
    e = out[-1]
    if b2b_s is None:
        e["back_to_back"] = {"error": b2b_err}
    else:
        e["back_to_back"] = {
            "us": b2b_s * 1e6, "replicas": b2b_r, "hbm_frac": dbytes / b2b_s / 1e9 / peak,
            "what": f"the same decode over {b2b_r} local caches (together more than twice the L2), recorded in one "
                    "CUDA graph and replayed; CUDA events around the replays, time per decode. A launch in a stream "
                    "of launches, without the per-call event and launch cost of the isolated figure above"}
        if dec_kernel == "decode_tc_kernel":
            e["back_to_back"]["tensor_frac"] = e["flops"] / b2b_s / 1e12 / e["peak"]
    out[-1]["same_flush_references"] = {
        "empty_op_us": empty_s * 1e6, "plain_read_us": plain_s * 1e6,
        "plain_read_frac": dbytes / plain_s / 1e9 / peak, "decode_over_plain_read": dec_s / plain_s,
        "what": "a one-element torch op, and torch.sum over a buffer of the decode's bytes, timed the same way"}
    return out, {"route_us": route_s * 1e6, "scan_us": scan_s * 1e6, "decode_us": dec_s * 1e6}


def dependent_layers(w, bank, router, decoder, x, cache, q, qr, st, s_fetch, n: int, device_fetch=False) -> dict:
    """Routing layers one after another on one stream, as a model whose next
    layer's router query depends on this layer's output would run them: route
    -> host-tier fetch -> rotation of the new token's key -> decode; no
    overlap between layers.  The fetch is the per-document copies (the host
    waits for the selection, then issues them) or, with device_fetch, one
    kernel reading the mapped host tier in stream order.  CUDA events on the
    stream from the first route to the last decode."""
    e_sel, e_fetch = torch.cuda.Event(), torch.cuda.Event()
    e_sel.record(st)
    e_fetch.record(st)

    def layer():
        router(qr, stream=st)
        if bank.host_tier and device_fetch:
            decoder.fetch_device(router.idx, stream=st)
        elif bank.host_tier:
            e_sel.record(st)
            decoder.fetch(router.idx_host, e_sel, s_fetch, e_fetch)
            st.wait_event(e_fetch)
        decoder.rotate_local(x["local_k"], cache, new_tokens=w.T, stream=st)
        decoder(q, cache, x["local_v"], router.idx, stream=st)
    for _ in range(3):
        layer()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(st)
    for _ in range(n):
        layer()
    b.record(st)
    b.synchronize()
    ms = a.elapsed_time(b) / n
    fetch = "none (K/V in HBM)" if not bank.host_tier else (
        "one kernel reading the mapped host tier" if device_fetch else "per-document cudaMemcpyAsync after a host wait")
    return {"ms_per_layer": ms, "tokens_per_s": w.B * w.T / (ms / 1e3), "layers": n, "fetch": fetch,
            "what": "one routing layer after another on one stream: route -> host-tier fetch -> "
                    "rotation of the new key -> decode, no overlap between layers"}


def run_loop(args):
    """Generated tokens/s of the multi-layer loop: per token and routing layer
    (each layer its own bank of the workload's shape), append the token's K/V,
    route (or reuse the first selection: route once per question), fetch from
    the host tier, decode.  Sequential host loop through the runtime API,
    timed with CUDA events; both routing modes are reported."""
    from routed_sparse_attention_b200 import Layout
    from routed_sparse_attention_b200.runtime import Bank, RoutedDecodeLoop

    w = BY_NAME[args.workload]
    assert not w.per_token, "the loop runs on pooled banks"
    dev = torch.device("cuda", torch.cuda.current_device())
    K, W, NL = args.steps, args.warmup, args.layers
    banks, xs = [], []
    for i in range(NL):
        wi = w.replace(mem_seed=w.mem_seed + 97 * i)
        x = gen.generate(wi, device=dev, host_interleaved=w.kv_on_host)
        banks.append(Bank(Layout.of(wi), x["doc_tok_off"], kr_pool=x["kr_pool"], k_pool=x.get("k_pool"),
                          v_pool=x.get("v_pool"), host_kv=x.get("host_kv"), device=dev))
        xs.append(x)
    loff = xs[0]["local_off"]
    prompt = torch.tensor([int(loff[b + 1] - loff[b]) - w.T for b in range(w.B)])
    H, d = w.n_kv_heads, w.head_dim
    res = {}
    for once in (False, True):
        loop = RoutedDecodeLoop(banks, w.B, w.top_k, prompt, prompt + 2 * (K + W), route_once=once, device=dev)
        for li, x in enumerate(xs):
            kp, vp = [], []
            for b in range(w.B):
                lt = int(loff[b + 1] - loff[b])
                a0 = int(loff[b]) * H * d
                kp.append(x["local_k"][a0:a0 + H * lt * d].view(H, lt, d)[:, :int(prompt[b])])
                vp.append(x["local_v"][a0:a0 + H * lt * d].view(H, lt, d)[:, :int(prompt[b])])
            loop.prefill(li, kp, vp)
        inputs = []
        for x in xs:
            kn = torch.stack([x["local_k"][int(loff[b]) * H * d:int(loff[b + 1]) * H * d]
                              .view(H, -1, d)[:, -1] for b in range(w.B)])
            vn = torch.stack([x["local_v"][int(loff[b]) * H * d:int(loff[b + 1]) * H * d]
                              .view(H, -1, d)[:, -1] for b in range(w.B)])
            inputs.append((x["qr"][:, :1].contiguous(), x["q"][:, :1].contiguous(), kn, vn))

        def token():
            for li in range(NL):
                loop.step(li, *inputs[li])
        for _ in range(W):
            token()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        a.record()
        for _ in range(K):
            token()
        b.record()
        b.synchronize()
        wall = time.perf_counter() - t0
        res["route_once" if once else "route_per_step"] = {
            "tokens_per_s": w.B * K / (a.elapsed_time(b) / 1e3), "ms_per_token": a.elapsed_time(b) / K,
            "wall_tokens_per_s": w.B * K / wall}
    # route once, then each token's appends and decodes on all layers as one CUDA graph replay
    loop = RoutedDecodeLoop(banks, w.B, w.top_k, prompt, prompt + 2 * (K + W), route_once=True, device=dev,
                            graph=True)
    for li, x in enumerate(xs):
        kp, vp = [], []
        for b in range(w.B):
            lt = int(loff[b + 1] - loff[b])
            a0 = int(loff[b]) * H * d
            kp.append(x["local_k"][a0:a0 + H * lt * d].view(H, lt, d)[:, :int(prompt[b])])
            vp.append(x["local_v"][a0:a0 + H * lt * d].view(H, lt, d)[:, :int(prompt[b])])
        loop.prefill(li, kp, vp)
    for li, (qr_i, q_i, kn_i, vn_i) in enumerate(inputs):
        loop.inputs[li]["q"].copy_(q_i)
        loop.inputs[li]["k_new"].copy_(kn_i)
        loop.inputs[li]["v_new"].copy_(vn_i)
    loop.token([inp[0] for inp in inputs])
    for _ in range(W):
        loop.token()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    a.record()
    for _ in range(K):
        loop.token()
    b.record()
    b.synchronize()
    wall = time.perf_counter() - t0
    res["route_once_graph"] = {"tokens_per_s": w.B * K / (a.elapsed_time(b) / 1e3), "ms_per_token": a.elapsed_time(b) / K,
                               "wall_tokens_per_s": w.B * K / wall}
    line = {"metric": f"routed decode tokens/s, {NL} routing layers per token", "stage": "loop",
            "value": res["route_per_step"]["tokens_per_s"], "unit": "tokens/s", "n_gpus": 1, "steps": K,
            "warmup": W, "higher_is_better": True, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "layers": NL, "batch": w.B, "top_k": w.top_k,
                       "prompt_tokens": int(prompt.max())},
            "modes": res, "device_status": __import__("routed_sparse_attention_b200").device_status()}
    print(json.dumps(line), flush=True)


def run_interleave(args):
    """Memory Interleave questions/s: per question, `rounds` rounds of
    (route for |S| + per_round documents, expand the set, fetch the host tier,
    rotate the local keys at the new offset, then generate `round_tokens`
    tokens).  Sequential host loop through the runtime API, timed with CUDA
    events."""
    from routed_sparse_attention_b200 import Layout, device_status
    from routed_sparse_attention_b200.runtime import Bank, MemoryInterleave

    w = BY_NAME[args.workload]
    assert not w.per_token, "interleave runs on a pooled bank"
    dev = torch.device("cuda", torch.cuda.current_device())
    K, W, R, p, G = args.steps, args.warmup, args.rounds, args.per_round, args.round_tokens
    x = gen.generate(w, device=dev, host_interleaved=w.kv_on_host)
    bank = Bank(Layout.of(w), x["doc_tok_off"], kr_pool=x["kr_pool"], k_pool=x.get("k_pool"),
                v_pool=x.get("v_pool"), host_kv=x.get("host_kv"), device=dev)
    loff = x["local_off"]
    H, d = w.n_kv_heads, w.head_dim
    prompt = torch.tensor([int(loff[b + 1] - loff[b]) - w.T for b in range(w.B)])
    mi = MemoryInterleave(bank, w.B, p, p * R, prompt, prompt + R * G, device=dev)
    kp, vp = [], []
    for b in range(w.B):
        lt = int(loff[b + 1] - loff[b])
        a0 = int(loff[b]) * H * d
        kp.append(x["local_k"][a0:a0 + H * lt * d].view(H, lt, d)[:, :int(prompt[b])])
        vp.append(x["local_v"][a0:a0 + H * lt * d].view(H, lt, d)[:, :int(prompt[b])])
    mi.prefill(kp, vp)
    gq = torch.Generator(device=dev).manual_seed(w.seed + 11)
    qr_rounds = [(x["qr"][:, :1] + 0.25 * torch.randn(x["qr"][:, :1].shape, generator=gq, device=dev)
                  .to(x["qr"].dtype)).contiguous() for _ in range(R)]
    q = x["q"][:, :1].contiguous()
    kn = torch.stack([x["local_k"][int(loff[b]) * H * d:int(loff[b + 1]) * H * d].view(H, -1, d)[:, -1]
                      for b in range(w.B)])
    vn = torch.stack([x["local_v"][int(loff[b]) * H * d:int(loff[b + 1]) * H * d].view(H, -1, d)[:, -1]
                      for b in range(w.B)])

    def question():
        mi.reset()
        for r in range(R):
            mi.expand(qr_rounds[r])
            for _ in range(G):
                mi.generate(q, kn, vn)
    for _ in range(W):
        question()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    a.record()
    for _ in range(K):
        question()
    b.record()
    b.synchronize()
    wall = time.perf_counter() - t0
    ms = a.elapsed_time(b) / K
    line = {"metric": "Memory Interleave questions/s", "stage": "interleave",
            "value": w.B * 1e3 / ms, "unit": "questions/s", "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_question": ms, "ms_per_round": ms / R, "generated_tokens_per_s": w.B * R * G * 1e3 / ms,
            "wall_questions_per_s": w.B * K / wall, "higher_is_better": True, "dtype": w.dtype,
            "data": "synthetic",
            "config": {"workload": w.name, "batch": w.B, "rounds": R, "per_round": p, "round_tokens": G,
                       "final_set": R * p, "prompt_tokens": int(prompt.max())},
            "device_status": device_status()}
    print(json.dumps(line), flush=True)


def run_stream_encode(args):
    """Streaming offline encode tokens/s: batches of whole documents of the
    workload's shape (per-token K, V, Kr in pinned host memory, two buffers
    reused in turn as a producer would) pushed through msa_encoder_* into a
    host-tier bank (Kr on the device, pooled K/V back in pinned memory).  The
    timed region is K pushes plus the final wait; its bound is the
    host-to-device copy of the per-token rows, measured here on the same
    pinned buffers for the roofline."""
    import routed_sparse_attention_b200 as msa
    from routed_sparse_attention_b200 import Layout

    w = BY_NAME[args.workload]
    dev = torch.device("cuda", torch.cuda.current_device())
    K, W = args.steps, args.warmup
    lay = Layout.of(w)
    H, d, dr, dt = w.n_kv_heads, w.head_dim, w.router_dim, lay.torch_dtype
    L = int(w.doc_len)
    docs = max(1, args.batch_tokens // L)
    ntok = docs * L
    rel = torch.arange(docs + 1, dtype=torch.int64) * L
    g = torch.Generator(device=dev).manual_seed(w.mem_seed)
    bufs = []
    for _ in range(2):
        bufs.append([torch.randn(ntok, H, dim, generator=g, device=dev).to(dt).cpu().pin_memory()
                     for dim in (d, d, dr)])
    ch = docs * ((L + w.chunk - 1) // w.chunk)
    cap = ch * (K + W)
    kr = torch.empty(cap, H, dr, dtype=dt, device=dev)
    host_kv = torch.empty(2 * cap, H, d, dtype=dt).pin_memory()
    enc = msa.StreamEncoder(lay, ntok, docs, L, cap, kr, host_kv_out=host_kv)
    for i in range(W):
        enc.push(rel, *bufs[i % 2])
    enc.finish()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    a.record()
    for i in range(K):
        enc.push(rel, *bufs[i % 2])
    enc.finish()
    b.record()
    b.synchronize()
    wall = time.perf_counter() - t0
    ms = a.elapsed_time(b)
    nd, nc, _, _ = enc.finish()
    enc.close()
    in_bytes = ntok * H * (2 * d + dr) * (2 if dt == torch.bfloat16 else 4)
    # the bound: a plain pinned host-to-device copy of the same buffers
    scratch = torch.empty(ntok * H * (2 * d + dr), dtype=dt, device=dev)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flat = [t.view(-1) for t in bufs[0]]
    for rep in range(4):
        if rep == 1:
            c0.record()
        at = 0
        for t in flat:
            scratch[at:at + t.numel()].copy_(t, non_blocking=True)
            at += t.numel()
    c1.record()
    c1.synchronize()
    h2d = in_bytes * 3 / (c0.elapsed_time(c1) / 1e3) / 1e9
    achieved = in_bytes * K / (ms / 1e3) / 1e9
    line = {"metric": "streaming offline encode tokens/s", "stage": "stream_encode",
            "value": ntok * K / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_batch": ms / K, "wall_tokens_per_s": ntok * K / wall, "higher_is_better": True,
            "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "batch_tokens": ntok, "batch_docs": docs, "doc_len": L,
                       "bytes_in_per_batch": in_bytes, "output": "host tier (Kr on device, K/V pinned host)"},
            "roofline": {"bound": "h2d", "achieved": achieved, "peak": h2d, "unit": "GB/s",
                         "frac": achieved / h2d, "peak_source": "pinned host-to-device copy of the same buffers"},
            "full_corpus_seconds": w.n_docs * L / (ntok * K / (ms / 1e3)),
            "device_status": msa.device_status()}
    print(json.dumps(line), flush=True)


def run_train(args):
    """Training-time routing layer, forward + backward per step: route (top-k),
    rotate the local keys, sparse attention with its log-sum-exp, the
    auxiliary routing loss, then the attention and loss gradients.  A
    training-sized shape: a 64K-token bank (256 documents x 256 tokens), 8
    queries of 64 tokens with 1984 prefix tokens each.  Reports tokens/s (the
    B*T query tokens per step) and the attention backward's arithmetic rate
    against the fp32 CUDA-core peak."""
    import routed_sparse_attention_b200 as msa
    from routed_sparse_attention_b200 import Layout
    from routed_sparse_attention_b200.runtime import Bank, TrainLayer

    from workloads import Workload
    w = Workload(name="train-64k-bank-8x64", dtype="bf16", n_docs=256, doc_len=256, lognormal_sigma=0.0,
                 len_clip=(256, 256), chunk=64, n_q_heads=32, n_kv_heads=8, head_dim=128, router_dim=128, T=64,
                 B=8, local_len=(1, 1), top_k=16, n_needles=0, per_token=False, kv_on_host=False, seed=940,
                 mem_seed=941)
    dev = torch.device("cuda", torch.cuda.current_device())
    K, W = args.steps, args.warmup
    B, T, Hq, Hkv, d, dr = w.B, w.T, w.n_q_heads, w.n_kv_heads, w.head_dim, w.router_dim
    prefix = 1984
    x = gen.generate(w.replace(per_token=False), device=dev)
    lay = Layout.of(w)
    bank = Bank(lay, x["doc_tok_off"], kr_pool=x["kr_pool"], k_pool=x["k_pool"], v_pool=x["v_pool"], device=dev)
    dt = lay.torch_dtype
    g = torch.Generator(device=dev).manual_seed(7)
    live = prefix + T
    loff = torch.arange(B + 1, dtype=torch.int64) * live
    q = torch.randn(B, T, Hq, d, generator=g, device=dev).to(dt)
    qr = torch.randn(B, T, Hq, dr, generator=g, device=dev).to(dt)
    lk = torch.randn(B * live * Hkv * d, generator=g, device=dev).to(dt)
    lv = torch.randn(B * live * Hkv * d, generator=g, device=dev).to(dt)
    dout = torch.randn(B, T, Hq, d, generator=g, device=dev).to(dt)
    dloss = torch.ones(B, dtype=torch.float32, device=dev)
    pos_off = torch.arange(B + 1, dtype=torch.int32, device=dev)
    pos_doc = torch.arange(B, dtype=torch.int32, device=dev) * 7
    layer = TrainLayer(bank, B, T, w.top_k, loff, tau=0.1, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    bwd_ms = []

    def step(timed=False):
        layer.forward(q, qr, lk, lv, pos_off, pos_doc)
        if timed:
            ev[2].record()
        layer.backward(dout, dloss)
        if timed:
            ev[3].record()
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    ev[0].record()
    for _ in range(K):
        step()
    ev[1].record()
    torch.cuda.synchronize()
    ms = ev[0].elapsed_time(ev[1]) / K
    for _ in range(3):
        step(timed=True)
        torch.cuda.synchronize()
        bwd_ms.append(ev[2].elapsed_time(ev[3]))
    bwd = min(bwd_ms)
    # the attention backward alone (prep, tile kernel, rotation), on buffers
    # zeroed outside the timed region, L2 flushed before each
    flush = L2Flush(dev)
    gb = layer.grad_buffers()
    attn_ms = []
    for i in range(max(K, 5)):
        for t in gb.values():
            t.zero_()
        flush()
        ev[2].record()
        layer.attention_backward(dout, gb)
        ev[3].record()
        torch.cuda.synchronize()
        if i > 0:
            attn_ms.append(ev[2].elapsed_time(ev[3]))
    attn = iq_mean(attn_ms)
    # useful arithmetic of the attention backward: five products (S, dP, dV, dK, dq)
    # of 2*d flops per visible (row, key) pair
    nmem = int(sum(int(bank.doc_chunk_off_host[s + 1] - bank.doc_chunk_off_host[s])
                   for s in layer.router.idx.cpu().reshape(-1).tolist()))
    pairs = Hkv * (Hq // Hkv) * (nmem * T + B * sum(prefix + t + 1 for t in range(T)))
    flops = 10.0 * d * pairs
    if w.dtype == "bf16":                      # the tensor-core backward
        peak, src = peak_bf16_tflops()
        bound, src = "tensor", f"{src} dense bf16 (cuBLAS GEMM)"
    else:                                      # fp32 on the CUDA cores
        sm_count = torch.cuda.get_device_properties(dev).multi_processor_count
        peak, bound = sm_count * 128 * 2 * 1965.0 * 1e6 / 1e12, "alu"
        src = "148 SMs x 128 fp32 lanes x 2 flops x 1965 MHz"
    line = {"metric": "training routing layer tokens/s (forward + backward)", "stage": "train",
            "value": B * T / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": W,
            "ms_per_step": ms, "backward_ms": bwd, "attention_backward_ms": attn, "higher_is_better": True,
            "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "bank_tokens": w.n_docs * w.doc_len, "batch": B, "T": T,
                       "prefix": prefix, "top_k": w.top_k},
            "roofline": {"kernel": "attention backward (prep + tile kernel + rotation)", "bound": bound,
                         "achieved": flops / (attn / 1e3) / 1e12, "peak": peak, "unit": "TFLOP/s",
                         "frac": flops / (attn / 1e3) / 1e12 / peak, "peak_source": src,
                         "flops": flops, "timing": "CUDA events around the attention backward call alone, "
                                                   "L2 flushed before each, interquartile mean; backward_ms is the "
                                                   "whole layer backward (gradient buffers, attention, routing loss)"},
            "device_status": msa.device_status()}
    print(json.dumps(line), flush=True)


def run_stage(args):
    """One stage of the path on its own (one GPU), timed with CUDA events:
    encode (per-token banks), route (Kr scan + selection) or decode.  Prints
    one JSON line with the stage's roofline; the default run is the step."""
    import routed_sparse_attention_b200 as msa
    from routed_sparse_attention_b200 import Layout
    from routed_sparse_attention_b200.runtime import Bank, Decoder, Router

    w = BY_NAME[args.workload]
    if args.docs:
        w = w.replace(name=f"{w.name}-first{args.docs}docs", n_docs=args.docs,
                      n_needles=min(w.n_needles, args.docs))
    dev = torch.device("cuda", torch.cuda.current_device())
    x = gen.generate(w, device=dev, host_interleaved=w.kv_on_host)
    lay = Layout.of(w)
    esz = 2 if w.dtype == "bf16" else 4
    peak, peak_kind = peak_hbm()
    flush = L2Flush(dev)
    K, W = args.steps, args.warmup

    def timed(fn):
        for _ in range(W):
            fn()
        ts = []
        for _ in range(K):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b) / 1e3)
        return iq_mean(ts)

    if args.stage == "encode":
        assert w.per_token, "encode runs on a per-token workload"
        bank = Bank(lay, x["doc_tok_off"], k_tok=x["k_tok"], v_tok=x["v_tok"], kr_tok=x["kr_tok"], device=dev)
        n_tok, C = int(x["doc_tok_off"][-1]), bank.n_chunks
        row = w.n_kv_heads * (2 * w.head_dim + w.router_dim) * esz
        nbytes = n_tok * row + C * row + 16 * (w.n_docs + 1)

        def fn():
            msa.encode_memory(lay, bank.doc_tok_off, bank.doc_chunk_off, C, int(bank.max_doc_len),
                              x["k_tok"], x["v_tok"], x["kr_tok"], bank.rope, bank.k, bank.v, bank.kr)
        sec = timed(fn)
        metric, value, unit, kern = "encode GB/s", nbytes / sec / 1e9, "GB/s", "encode_pool_kernel"
        extra = {"tokens": n_tok, "pooled_chunks": C, "encode_us": sec * 1e6}
    else:
        if w.per_token:
            bank = Bank(lay, x["doc_tok_off"], k_tok=x["k_tok"], v_tok=x["v_tok"], kr_tok=x["kr_tok"], device=dev)
        else:
            bank = Bank(lay, x["doc_tok_off"], kr_pool=x["kr_pool"], k_pool=x.get("k_pool"),
                        v_pool=x.get("v_pool"), host_kv=x.get("host_kv"), device=dev)
        router = Router(bank, w.B, w.T, w.top_k, dev)
        if args.stage == "route":
            ev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            ev[0].record(); ev[1].record()
            scan_s = []

            def fn():
                msa.scan_events(*ev)
                router(x["qr"])
                msa.scan_events()
            for _ in range(W):
                fn()
            ts = []
            for _ in range(K):
                flush()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(); fn(); b.record(); b.synchronize()
                ts.append(a.elapsed_time(b) / 1e3)
                scan_s.append(ev[0].elapsed_time(ev[1]) / 1e3)
            sec = iq_mean(ts)
            scan = iq_mean(scan_s)
            nbytes = bank.n_chunks * w.n_kv_heads * w.router_dim * esz + bank.n_docs * 12
            nq = w.B * w.T
            if w.dtype == "bf16" and nq > 4:     # tensor-core scan: 32, 64 or 128 rows per pass
                nqp = 32 if nq <= 32 else (64 if nq <= 64 else 128)
                n_pass = (nq + nqp - 1) // nqp
            else:                                 # CUDA-core scan: 1, 2 or 4 rows per pass
                n_pass = (nq + 3) // 4 if nq > 2 else 1
            kern = "kr_scan_mma_kernel" if (w.dtype == "bf16" and nq > 4) else "kr_scan_kernel"
            metric, value, unit = "route Kr scan GB/s", nbytes / scan / 1e9, "GB/s"
            extra = {"route_us": sec * 1e6, "scan_us": scan * 1e6, "query_rows": w.B * w.T,
                     "scan_passes": n_pass, "scan_bytes_all_passes": nbytes * n_pass}
        else:
            idx, _ = router(x["qr"])
            dec = Decoder(bank, w.B, w.T, w.top_k, x["local_off"], dev)
            if bank.host_tier:
                s = torch.cuda.current_stream()
                e1, e2 = torch.cuda.Event(), torch.cuda.Event()
                e1.record(s); e2.record(s)
                dec.fetch(router.idx_host, e1, s, e2)
            torch.cuda.synchronize()
            lens = np.diff(x["local_off"])
            sel = idx.cpu().numpy()
            coff = bank.doc_chunk_off_host.numpy()
            n_mem = np.array([sum(int(coff[d + 1] - coff[d]) for d in row) for row in sel])
            nbytes = int(((n_mem + lens) * 2 * w.head_dim * esz * w.n_kv_heads).sum()
                         + 2 * w.B * w.T * w.n_q_heads * w.head_dim * esz)

            k_cache = dec.rotate_local(x["local_k"], torch.empty_like(x["local_k"]))

            def fn():
                dec(x["q"], k_cache, x["local_v"], idx)
            sec = timed(fn)
            kern = decode_kernel_name(w)
            metric, value, unit = "sparse decode GB/s", nbytes / sec / 1e9, "GB/s"
            # a reference point for one launch reading this many bytes on this GPU:
            # a plain library reduction over a buffer of the same size, timed the same way
            plain = torch.ones(nbytes // 2, dtype=torch.bfloat16, device=dev)
            floor_s = timed(lambda: plain.sum())
            extra = {"decode_us": sec * 1e6, "decode_bytes": nbytes,
                     "tokens_per_s": w.B * w.T / sec,
                     "floor": {"plain_read_us": floor_s * 1e6,
                               "what": "torch.sum over a buffer of the decode's bytes, same L2 flush and events",
                               "frac_of_peak": nbytes / floor_s / 1e9 / peak}}
            if kern == "decode_tc_kernel":            # many query rows: the tensor roof
                fl = decode_flops(w, bank, sel, x["local_off"])
                tpk, tkind = peak_bf16_tflops()
                extra["tensor"] = {"flops": fl, "achieved": fl / sec / 1e12, "peak": tpk, "unit": "TFLOP/s",
                                   "frac": fl / sec / 1e12 / tpk, "peak_kind": f"{tkind} (bf16_tflops)"}
    line = {"metric": metric, "value": value, "unit": unit, "n_gpus": 1, "steps": K, "warmup": W,
            "higher_is_better": True, "dtype": w.dtype, "data": "synthetic", "stage": args.stage,
            "config": {"workload": w.name, "l2": "before every timed run 256 MiB written, then 256 MiB of another "
                                                 "buffer read (L2 holds no input)"},
            "roofline": {"kernel": kern, "bound": "hbm", "achieved": value, "peak": peak, "unit": "GB/s",
                         "frac": value / peak, "peak_kind": f"{peak_kind} (hbm_gbs)"},
            "device_status": msa.device_status()}
    line.update(extra)
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    rank, world, local = replica_env()
    if args.impl == "reference":
        run_reference(args, rank)
        return
    torch.cuda.set_device(local)
    if args.stage == "loop":
        run_loop(args)
        return
    if args.stage == "interleave":
        run_interleave(args)
        return
    if args.stage == "stream_encode":
        run_stream_encode(args)
        return
    if args.stage == "train":
        run_train(args)
        return
    if args.stage != "step":
        run_stage(args)
        return
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))
    try:
        run_msa(args, rank, world)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
