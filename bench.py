#!/usr/bin/env python
"""Benchmark of the HeadKV hot path on B200 (one JSON line on rank 0).

One step = one pass of the whole hot path over one batch: reset, prefill +
head grouping + compression for every layer, then every decode step
(fused append + decode attention per layer, one STE call), replayed as one
CUDA graph with the inputs resident in HBM.  value = decode image tokens/s
over the whole pass (prefill time included).  Inputs are far larger than L2
(the cache and the per-step inputs of all layers rotate through HBM).

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl reference]

Multi-GPU: one process per GPU (torchrun); every rank runs its own batch of
the workload (weak scaling, no data-path collective); the time is the max
over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "compressed decode image tokens/s and step µs; achieved HBM GB/s vs B200 peak"
UNIT = "image tokens/s"
# which sequences form a classifier-free-guidance pair (values of hkv_cfg_pairing)
PAIRINGS = {"untied": 0, "halves": 1, "adjacent": 2}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="lumina_mgpt_768",
                    help="the headline workload (default: the largest single-GPU shape)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-full", action="store_true", help="skip the full-cache comparator")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end arm")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--mode", default="headkv", choices=["headkv", "uniform"],
                    help="uniform: the same per-head budget for every head (a comparator)")
    ap.add_argument("--unstratified", action="store_true",
                    help="eviction over one pool instead of near/far strata (a comparator)")
    ap.add_argument("--cls-queries", type=int, default=1,
                    help="group heads by the last n prefill queries' per-distance weights")
    ap.add_argument("--cfg-pairing", default="untied", choices=list(PAIRINGS),
                    help="group the two streams of a CFG pair by their mean row")
    ap.add_argument("--no-decoder-layer", action="store_true",
                    help="skip whole decoder layers (projections + MLP on random weights "
                         "around each attention call), compressed and full cache")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the shorter runs of every other workload (all_configs)")
    ap.add_argument("--profile", action="store_true",
                    help="eager run of a reduced workload for ncu captures (no timing line)")
    ap.add_argument("--seqs", type=int, default=None,
                    help="override the workload's sequences (profile runs and reduced timings)")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the workload's layers (profile runs and reduced timings)")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline leg")
    ap.add_argument("--profile-steps", type=int, default=64)
    return ap.parse_args()


# ---------------------------------------------------------------------------
# CPU oracle timing (the reported CPU baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(w, seed, seconds, threads=None, opts=None):
    """Runs whole (sequence, layer) units of the workload through the CPU
    oracle on host threads for about `seconds`; returns (image tokens/s,
    threads, units done).  opts: the variant flags (mode, stratified,
    cls_queries, cfg_pairing)."""
    from concurrent.futures import ThreadPoolExecutor

    from kv_cache_compression_hkv_b200.inputs import generate_layer
    from oracle import hkv_oracle as O

    threads = threads or os.cpu_count() or 1
    opts = opts or {}
    pairing = opts.get("cfg_pairing", O.CFG_UNTIED)
    nq = opts.get("cls_queries", 1)
    prm = O.UnitParams(num_heads=w.num_heads, head_dim=w.head_dim, max_len=w.max_len,
                       prefill_len=w.prefill_len, local_window=w.local_window, ste_m=w.ste_m,
                       near_dist=w.near_dist, score_window=w.score_window, rho_num=w.rho[0],
                       rho_den=w.rho[1], mode=opts.get("mode", O.MODE_HEADKV),
                       stratified=opts.get("stratified", True), cls_queries=nq)
    n_seq = min(w.num_seqs, threads)
    if pairing != O.CFG_UNTIED:
        n_seq = max(2, n_seq - n_seq % 2)
    q, k, v = generate_layer(w, 0, seed, "cpu", num_seqs=n_seq)
    units = [tuple(x[s].double().numpy() for x in (q, k, v)) for s in range(n_seq)]
    O.build()
    done = [0]
    deadline = time.perf_counter() + seconds
    lock = threading.Lock()
    P = w.prefill_len

    def rows(s):
        qs, ks, vs = units[s]
        return np.stack([O.class_row(qs[h, :P], ks[h, :P], vs[h, :P], nq)
                         for h in range(w.num_heads)])

    def worker(i):
        n = 0
        while True:
            s = i % len(units)
            cls = None
            if pairing != O.CFG_UNTIED:
                # the sample pairs its own sequences: the same work as the
                # true partner's row
                cls = O.tied_rows(rows(s), rows(O.cfg_partner(s, n_seq, pairing)))
            O.run_unit(prm, *units[s], want_decode=True, cls_rows=cls)
            n += 1
            if time.perf_counter() > deadline:
                break
        with lock:
            done[0] += n

    t0 = time.perf_counter()
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(worker, range(threads)))
    el = time.perf_counter() - t0
    tokens_per_unit = w.images * w.decode_steps / (w.num_seqs * w.num_layers)
    return done[0] * tokens_per_unit / el, threads, done[0], el


def oracle_opts(args) -> dict:
    """The variant flags as oracle unit parameters."""
    return {"mode": 2 if args.mode == "uniform" else 0, "stratified": not args.unstratified,
            "cls_queries": args.cls_queries, "cfg_pairing": PAIRINGS[args.cfg_pairing]}


def planted_recovery(w, labels, seed) -> dict:
    """How the computed labels ([layers, S, H], 1 = Local) meet the heads
    the synthetic inputs planted Local: the share of planted Local heads
    labelled Local, and of planted Global heads labelled Local."""
    from kv_cache_compression_hkv_b200.inputs import planted_local_heads
    planted = np.stack([planted_local_heads(w, l, seed).numpy() for l in range(w.num_layers)])
    planted = np.broadcast_to(planted[:, None, :], labels.shape)
    local = labels == 1
    return {"local_as_local": float(local[planted].mean()) if planted.any() else None,
            "global_as_local": float(local[~planted].mean()) if (~planted).any() else None}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

def gpu_id(dev) -> str:
    """nvidia-smi id of a torch device (its UUID; indices may be remapped)."""
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev.index or 0)


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: str):
        self.index = index
        self.proc = None

    def __enter__(self):
        if self.index is None:  # not sampled
            return self
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = [r.split(",") for r in (self.out or "").strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if "Active" in r[5 + i]
                          and "Not" not in r[5 + i]})
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------

class Inputs:
    """Per-layer prefill blocks [S, H, P, d] and per-step decode inputs
    [steps, S, H, d], all resident in HBM."""

    def __init__(self, w, seed, dev):
        from kv_cache_compression_hkv_b200.inputs import generate_layer
        P = w.prefill_len
        self.pre, self.dec = [], []
        for l in range(w.num_layers):
            q, k, v = generate_layer(w, l, seed, dev)
            self.pre.append(tuple(x[:, :, :P].contiguous() for x in (q, k, v)))
            self.dec.append(tuple(x[:, :, P:].permute(2, 0, 1, 3).contiguous() for x in (q, k, v)))
            del q, k, v
        torch.cuda.synchronize()

    def nbytes(self):
        return sum(x.numel() * x.element_size() for t in self.pre + self.dec for x in t)


def run_pass(cache, w, inp, outs, evict=True, pre_out=None, hooks=None):
    """Enqueues one whole pass on the current stream (eagerly or under capture)."""
    if hooks:
        hooks("pass_begin", None, None)
    cache.reset()
    for l in range(w.num_layers):
        q, k, v = inp.pre[l]
        cache.prefill_classify(l, q, k, v, out=None if pre_out is None else pre_out[l])
    if hooks:
        hooks("decode_begin", None, None)
    for t in range(w.decode_steps):
        for l in range(w.num_layers):
            q, k, v = inp.dec[l]
            if hooks:
                hooks("pre_decode", t, l)
            cache.decode_step(l, q[t], k[t], v[t], outs[l])
            if hooks:
                hooks("post_decode", t, l)
        if evict:
            if hooks:
                hooks("pre_evict", t, None)
            cache.ste_evict()
            if hooks:
                hooks("post_evict", t, None)
    if hooks:
        hooks("decode_end", None, None)


def capture(fn):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def decode_tokens_per_launch(cache, w, inp, outs):
    """Eager pass that reads back every layer's cache lengths right after its
    decode launches: kv tokens each decode launch reads, [steps, layers]."""
    S, H = w.num_seqs, w.num_heads
    tok = np.zeros((w.decode_steps, w.num_layers), np.int64)
    cache.reset()
    for l in range(w.num_layers):
        cache.prefill_classify(l, *inp.pre[l])
    for t in range(w.decode_steps):
        for l in range(w.num_layers):
            q, k, v = inp.dec[l]
            cache.decode_step(l, q[t], k[t], v[t], outs[l])
        for l in range(w.num_layers):
            ln, _ = cache.lens(l)
            tok[t, l] = int(ln.sum())
        cache.ste_evict()
    torch.cuda.synchronize()
    return tok


def timed_replays(g, n):
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(s)
    for _ in range(n):
        g.replay()
    e1.record(s)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n  # ms per replay


# workloads on which the pages compare whole-model speed and memory with
# the full cache (LlamaGen-XL and Janus-Pro-7B at rho = 1/6): the
# decoder-layer arm runs on these
DECODER_LAYER_WORKLOADS = ("llamagen_xl", "janus_pro_7b_rho6")


def gpu_arm(args, rank, world, dev, w, lite=False):
    """The timed GPU arm on workload w.  lite: the shorter run of the sweep
    (one warm-up and two timed passes, the full-cache comparator on one
    timed pass, no end-to-end arm, no clock sampling).  The decoder-layer
    arm runs on DECODER_LAYER_WORKLOADS unless --no-decoder-layer."""
    import kv_cache_compression_hkv_b200 as hkv

    S, H, d, Ly = w.num_seqs, w.num_heads, w.head_dim, w.num_layers
    es = 2 if w.dtype == "bf16" else 4
    steps = w.decode_steps
    from kv_cache_compression_hkv_b200 import dist
    inp = Inputs(w, dist.rank_seed(args.seed, rank), dev)
    outs = [torch.empty(S, H, d, dtype=w.torch_dtype, device=dev) for _ in range(Ly)]
    pre_out = [torch.empty(S, H, w.prefill_len, d, dtype=w.torch_dtype, device=dev) for _ in range(Ly)]
    cfg = hkv.config_for(w, mode=hkv.MODE_UNIFORM if args.mode == "uniform" else hkv.MODE_HEADKV,
                         stratified=not args.unstratified, cls_queries=args.cls_queries,
                         cfg_pairing=PAIRINGS[args.cfg_pairing])
    cache = hkv.HeadKVCache(cfg, device=dev)

    # one eager pass: warms every kernel and yields the bytes each decode launch reads
    tokens = decode_tokens_per_launch(cache, w, inp, outs)
    labels = np.stack([cache.labels(l)[0] for l in range(Ly)])
    rc, detail = cache.check()
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail}) after the eager pass")

    # main graph: the whole pass
    # events of the last replay: pass start, decode start (prefill and
    # grouping of every layer done), decode end
    ev_pre = torch.cuda.Event(enable_timing=True, external=True)
    ev_dec = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]

    def hooks_main(what, t, l):
        if what == "pass_begin":
            ev_pre.record()
        elif what == "decode_begin":
            ev_dec[0].record()
        elif what == "decode_end":
            ev_dec[1].record()

    g_main = capture(lambda: run_pass(cache, w, inp, outs, pre_out=pre_out, hooks=hooks_main))
    for _ in range(1 if lite else args.warmup):
        g_main.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(None if lite else gpu_id(dev)) as clk:
        ms = timed_replays(g_main, 2 if lite else args.steps)
        decode_ms = ev_dec[0].elapsed_time(ev_dec[1])
        prefill_ms = ev_pre.elapsed_time(ev_dec[0])
    if world > 1:
        ms = dist.max_over_ranks(ms, dev)
        torch.distributed.barrier()
    rc, detail = cache.check()
    if rc != 0:
        raise RuntimeError(f"device status {rc} ({detail}) after the timed passes")

    # per step: the span of its Ly back-to-back decode launches (events only
    # around the run, so consecutive launches may overlap as they do in the
    # timed pass) and of its eviction; same stream as the kernels
    n_ev = steps * 2
    evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * n_ev)]

    def hooks_prof(what, t, l):
        if what == "pre_decode" and l == 0:
            evs[4 * t].record()
        elif what == "post_decode" and l == Ly - 1:
            evs[4 * t + 1].record()
        elif what == "pre_evict":
            evs[4 * t + 2].record()
        elif what == "post_evict":
            evs[4 * t + 3].record()

    g_prof = capture(lambda: run_pass(cache, w, inp, outs, pre_out=pre_out, hooks=hooks_prof))
    g_prof.replay()
    torch.cuda.synchronize()
    ev = cache.evict_stats()  # this pass's evictions (reset clears the counters)
    dur = np.array([evs[2 * i].elapsed_time(evs[2 * i + 1]) for i in range(n_ev)]).reshape(steps, 2)
    dec_us = np.repeat(dur[:, :1] * 1e3 / Ly, Ly, axis=1)  # average launch of each step
    evict_us = dur[:, 1] * 1e3
    kv_bytes = tokens * 2 * d * es                      # kept K + V read (new token included)
    io_bytes = S * H * d * es * 4                        # q read, o written, new k/v row stored
    alg = kv_bytes + io_bytes
    achieved = float(alg.sum() / (dec_us.sum() * 1e-6) / 1e9)
    del g_prof

    traffic_ratio = decode_traffic_ratio(w.name)
    peaks = {}
    pk = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk):
        peaks = json.load(open(pk))
    peak = peaks.get("hbm_gbs", 6650.0)
    peak_src = "measured" if "hbm_gbs" in peaks else "fallback"

    res = {
        "ms_per_step": ms,
        "decode_step_us": decode_ms * 1e3 / steps,
        "prefill_ms": prefill_ms,
        "tokens_per_s": w.images * steps / (ms * 1e-3) * world,
        "clocks": clk.summary(),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": (None if traffic_ratio is None
                                 else round(traffic_ratio * float(alg.mean()))),
                     "kernel": "decode_kernel (fused append + split-K decode attention)",
                     "peak_source": peak_src,
                     "bytes_per_launch_avg": float(alg.mean()),
                     "launch_us_avg": float(dec_us.mean())},
        "evict_us_avg": float(evict_us.mean()),
        "evict_us_max": float(evict_us.max()),
        # eviction over the pass: positions + r logits of every scored token,
        # K|V pairs of the moved rows read and written; time = the spans of
        # the steps' eviction calls (eviction kernel + next-step plan)
        "evict": {"heads": ev["heads"], "rows_moved": ev["rows_moved"],
                  "bytes": ev["tokens"] * (4 + 4 * w.score_window) + ev["rows_moved"] * 4 * d * es,
                  "call_us_total": float(evict_us.sum())},
        "labels_local_frac": float((labels == 1).mean()),
        "labels_planted": planted_recovery(w, labels, dist.rank_seed(args.seed, rank)),
        # per layer at prefill: attention, grouping, packing, plan; per
        # step: one decode launch per layer, the eviction, the plan
        "gpu_launches": args.steps * (4 * Ly + steps * (Ly + 2)),
        "kv_pool_bytes": cache.nbytes,
    }
    del g_main

    # full-cache comparator (same kernels, no compression)
    if not args.no_full:
        cache_f = hkv.HeadKVCache(hkv.config_for(w, mode=hkv.MODE_FULL), device=dev)
        g_full = capture(lambda: run_pass(cache_f, w, inp, outs, pre_out=pre_out,
                                          hooks=hooks_main))
        for _ in range(1 if lite else 2):
            g_full.replay()
        ms_f = timed_replays(g_full, 1 if lite else max(1, min(args.steps, 3)))
        dec_f = ev_dec[0].elapsed_time(ev_dec[1])
        res["full"] = {"ms_per_step": ms_f, "decode_step_us": dec_f * 1e3 / steps,
                       "kv_pool_bytes": cache_f.nbytes}
        res["speedup_decode_vs_full"] = dec_f / decode_ms
        res["speedup_pass_vs_full"] = ms_f / ms
        del g_full, cache_f
        torch.cuda.empty_cache()

    if not args.no_decoder_layer and w.name in DECODER_LAYER_WORKLOADS:
        res["decoder_layer"] = decoder_layer_arm(args, w, cache, inp, outs, pre_out, dev)

    # end to end through the C ABI from pinned host buffers
    if not lite and not args.no_e2e:
        try:
            res["e2e"] = e2e_arm(args, w, cache, inp, dev, world)
        except RuntimeError as e:  # e.g. the host cannot pin every step's inputs
            res["e2e"] = {"value": None, "unit": UNIT, "error": str(e)[:200]}
            torch.cuda.synchronize()
    return res


def sweep_arm(args, dev, skip):
    """Shorter runs of every workload but `skip` (one warm-up, two timed
    passes each, with the full-cache comparator): image tokens/s, decode
    step and launch, roofline fraction and speedup over full per workload."""
    from kv_cache_compression_hkv_b200.inputs import WORKLOADS
    out = {}
    for name, w in WORKLOADS.items():
        if name == skip:
            continue
        r = gpu_arm(args, 0, 1, dev, w, lite=True)
        out[name] = {
            "value": r["tokens_per_s"], "ms_per_step": r["ms_per_step"],
            "decode_step_us": r["decode_step_us"],
            "launch_us_avg": r["roofline"]["launch_us_avg"],
            "roofline_frac": r["roofline"]["frac"],
            "evict_us_avg": r["evict_us_avg"], "evict_us_max": r["evict_us_max"],
            "full_decode_step_us": (r.get("full") or {}).get("decode_step_us"),
            "speedup_decode_vs_full": r.get("speedup_decode_vs_full"),
            "kv_pool_bytes": r["kv_pool_bytes"],
            "full_kv_pool_bytes": (r.get("full") or {}).get("kv_pool_bytes"),
            "labels_local_frac": r["labels_local_frac"]}
        if r.get("decoder_layer"):
            out[name]["decoder_layer"] = r["decoder_layer"]
        torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------------------
# dense work of a decoder layer around each attention call (comparison harness)
# ---------------------------------------------------------------------------

class DecoderLayers:
    """The dense work of a LLaMA-style decoder layer around every attention
    call, on random weights: a QKV projection before it, the output
    projection, a SwiGLU MLP and the residual adds after it.  hidden = H * d;
    the MLP width is the LLaMA rule (the multiple of 256 at or above
    8/3 * hidden), which gives 3584 / 5632 / 11008 for hidden 1280 / 2048 /
    4096.  The projections run on cuBLAS (torch.matmul): a harness for
    whole-layer step times, not part of the compressed path.  The cache is
    still fed the workload's planted q, k, v, so that compression behaves as
    in the headline runs; the QKV projection's output is computed and left
    in a scratch buffer."""

    def __init__(self, w, dev, seed):
        S, Ly = w.num_seqs, w.num_layers
        self.hid = hid = w.num_heads * w.head_dim
        self.ffn = ffn = -(-(8 * hid) // (3 * 256)) * 256
        dt = w.torch_dtype
        g = torch.Generator(device=dev).manual_seed(seed * 31 + 5)

        def rnd(n_in, n_out):
            # small branch gain so 2 x layers residual adds stay finite
            return (torch.randn(n_in, n_out, generator=g, device=dev) * (0.1 / n_in ** 0.5)).to(dt)

        self.wqkv = [rnd(hid, 3 * hid) for _ in range(Ly)]
        self.wo = [rnd(hid, hid) for _ in range(Ly)]
        self.w13 = [rnd(hid, 2 * ffn) for _ in range(Ly)]
        self.w2 = [rnd(ffn, hid) for _ in range(Ly)]
        self.x0 = torch.randn(S, hid, generator=g, device=dev).to(dt)
        self.x = torch.empty_like(self.x0)
        self.qkv = torch.empty(S, 3 * hid, dtype=dt, device=dev)
        self.gu = torch.empty(S, 2 * ffn, dtype=dt, device=dev)
        self.act = torch.empty(S, ffn, dtype=dt, device=dev)
        self.y = torch.empty(S, hid, dtype=dt, device=dev)
        self.weight_bytes = sum(t.numel() * t.element_size()
                                for ts in (self.wqkv, self.wo, self.w13, self.w2) for t in ts)

    def flops_per_step(self, S, Ly):
        return 2 * S * Ly * self.hid * (3 * self.hid + self.hid + 3 * self.ffn)

    def pre(self, l):
        if l == 0:
            self.x.copy_(self.x0)  # the new token's embedding
        torch.matmul(self.x, self.wqkv[l], out=self.qkv)

    def post(self, l, o):
        torch.matmul(o.view(o.shape[0], -1), self.wo[l], out=self.y)
        self.x.add_(self.y)
        torch.matmul(self.x, self.w13[l], out=self.gu)
        gate, up = self.gu[:, : self.ffn], self.gu[:, self.ffn:]
        torch.mul(torch.nn.functional.silu(gate), up, out=self.act)
        torch.matmul(self.act, self.w2[l], out=self.y)
        self.x.add_(self.y)


def decoder_layer_arm(args, w, cache, inp, outs, pre_out, dev):
    """Whole-layer step times, compressed and full cache, with the dense
    work of DecoderLayers around every attention call."""
    import kv_cache_compression_hkv_b200 as hkv
    dense = DecoderLayers(w, dev, args.seed)
    # one eager round first: cuBLAS makes its handle and workspace on first
    # use, which a stream capture does not allow
    for l in range(w.num_layers):
        dense.pre(l)
        dense.post(l, outs[l])
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]

    def hooks(what, t, l):
        if what == "decode_begin":
            ev[0].record()
        elif what == "decode_end":
            ev[1].record()
        elif what == "pre_decode":
            dense.pre(l)
        elif what == "post_decode":
            dense.post(l, outs[l])

    def step_us(c):
        g = capture(lambda: run_pass(c, w, inp, outs, pre_out=pre_out, hooks=hooks))
        g.replay()
        timed_replays(g, max(1, min(args.steps, 2)))
        us = ev[0].elapsed_time(ev[1]) * 1e3 / w.decode_steps
        del g
        return us

    us = step_us(cache)
    cache_f = hkv.HeadKVCache(hkv.config_for(w, mode=hkv.MODE_FULL), device=dev)
    us_f = step_us(cache_f)
    out = {"hidden": dense.hid, "ffn": dense.ffn, "step_us": us, "full_step_us": us_f,
           "speedup": us_f / us, "weight_bytes": dense.weight_bytes,
           "kv_pool_bytes": cache.nbytes, "full_kv_pool_bytes": cache_f.nbytes,
           "memory_saving": 1.0 - (cache.nbytes + dense.weight_bytes)
                                  / (cache_f.nbytes + dense.weight_bytes),
           "dense_gflop_per_step": dense.flops_per_step(w.num_seqs, w.num_layers) / 1e9}
    del cache_f, dense
    torch.cuda.empty_cache()
    return out


def e2e_arm(args, w, cache, inp, dev, world):
    """Same pass with every input copied from pinned host memory inside the
    timed region (each layer's prefill q, k, v; each step's q_t, k_t, v_t of
    every layer) and each step's result (the last layer's output) copied
    back."""
    S, H, d, Ly, steps = w.num_seqs, w.num_heads, w.head_dim, w.num_layers, w.decode_steps
    host_pre = [tuple(torch.empty(x.shape, dtype=x.dtype).pin_memory() for x in t) for t in inp.pre]
    for hp, dp in zip(host_pre, inp.pre):
        for hx, dx in zip(hp, dp):
            hx.copy_(dx)
    # one contiguous block per step: [steps][Ly][q, k, v][S][H][d]
    host_dec = torch.empty(steps, Ly, 3, S, H, d, dtype=w.torch_dtype).pin_memory()
    for l in range(Ly):
        for j in range(3):
            host_dec[:, l, j].copy_(inp.dec[l][j])
    # the step's result read back: the last layer's attention output (what
    # the next token depends on); the other layers' outputs stay on the GPU
    host_out = torch.empty(steps, S, H, d, dtype=w.torch_dtype).pin_memory()
    dev_pre = [tuple(torch.empty_like(x) for x in t) for t in inp.pre]
    stage = [torch.empty(Ly, 3, S, H, d, dtype=w.torch_dtype, device=dev) for _ in range(2)]
    outs2 = [torch.empty(Ly, S, H, d, dtype=w.torch_dtype, device=dev) for _ in range(2)]
    h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(steps)]    # step t's inputs landed
    ev_done = [torch.cuda.Event() for _ in range(steps)]  # step t's kernels finished
    ev_out = [torch.cuda.Event() for _ in range(steps)]   # step t's outputs copied out

    def body():
        # step t+1's inputs go up and step t's outputs come down on two side
        # streams while step t computes; staging and outputs double-buffered
        main = torch.cuda.current_stream()
        cache.reset()
        for l in range(Ly):
            for hx, dx in zip(host_pre[l], dev_pre[l]):
                dx.copy_(hx, non_blocking=True)
            cache.prefill_classify(l, *dev_pre[l])
        h2d_s.wait_stream(main)
        d2h_s.wait_stream(main)

        def stage_in(t):
            with torch.cuda.stream(h2d_s):
                if t >= 2:
                    h2d_s.wait_event(ev_done[t - 2])
                stage[t & 1].copy_(host_dec[t], non_blocking=True)
                ev_in[t].record(h2d_s)

        stage_in(0)
        for t in range(steps):
            if t + 1 < steps:
                stage_in(t + 1)
            main.wait_event(ev_in[t])
            if t >= 2:
                main.wait_event(ev_out[t - 2])
            st, ot = stage[t & 1], outs2[t & 1]
            for l in range(Ly):
                cache.decode_step(l, st[l, 0], st[l, 1], st[l, 2], ot[l])
            cache.ste_evict()
            ev_done[t].record(main)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(ev_done[t])
                host_out[t].copy_(ot[Ly - 1], non_blocking=True)
                ev_out[t].record(d2h_s)
        main.wait_stream(h2d_s)
        main.wait_stream(d2h_s)

    g = capture(body)
    for _ in range(2):
        g.replay()
    ms = timed_replays(g, max(1, min(args.steps, 3)))
    if world > 1:
        from kv_cache_compression_hkv_b200 import dist
        ms = dist.max_over_ranks(ms, dev)
    h2d = sum(x.numel() * x.element_size() for t in host_pre for x in t) + \
        host_dec.numel() * host_dec.element_size()
    d2h = host_out.numel() * host_out.element_size()
    del g
    return {"value": w.images * steps / (ms * 1e-3) * world, "unit": UNIT,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "ms_per_step": ms}


def profile_run(args, w):
    """Eager prefill + decode steps of a reduced copy of the workload: the
    command ncu captures single launches of (nothing is timed here).  Prints
    the algorithmic bytes of every decode launch, in launch order, so that
    the DRAM bytes of a captured launch can be compared with them."""
    import kv_cache_compression_hkv_b200 as hkv
    dev = torch.device("cuda", 0)
    w = w.scaled(num_seqs=args.seqs or w.num_seqs, num_layers=args.layers or w.num_layers)
    inp = Inputs(w, args.seed, dev)
    outs = [torch.empty(w.num_seqs, w.num_heads, w.head_dim, dtype=w.torch_dtype, device=dev)
            for _ in range(w.num_layers)]
    cache = hkv.HeadKVCache(hkv.config_for(w), device=dev)
    es = 2 if w.dtype == "bf16" else 4
    for l in range(w.num_layers):
        cache.prefill_classify(l, *inp.pre[l])
    alg, evict_steps, evict_alg = [], [], []
    steps = min(args.profile_steps, w.decode_steps)
    for t in range(steps):
        for l in range(w.num_layers):
            q, k, v = inp.dec[l]
            cache.decode_step(l, q[t], k[t], v[t], outs[l])
            ln, _ = cache.lens(l)
            alg.append(int(ln.sum()) * 2 * w.head_dim * es + w.num_seqs * w.num_heads * w.head_dim * es * 4)
        st0 = cache.evict_stats()
        cache.ste_evict()
        st1 = cache.evict_stats()
        # algorithmic bytes of this step's eviction: per evicted head its
        # positions and r logits, and the rows it moved (K|V pair read + written)
        if st1["heads"] > st0["heads"]:
            evict_steps.append(t)
            evict_alg.append((st1["tokens"] - st0["tokens"]) * (4 + 4 * w.score_window) +
                             (st1["rows_moved"] - st0["rows_moved"]) * 2 * 2 * w.head_dim * es)
    torch.cuda.synchronize()
    rc, detail = cache.check()
    print(json.dumps({"profile_run": w.name, "seqs": w.num_seqs, "layers": w.num_layers,
                      "steps": steps, "status": rc, "decode_alg_bytes": alg,
                      "evict_steps": evict_steps, "evict_alg_bytes": evict_alg}))
    if rc != 0:
        raise SystemExit(f"device status {rc} ({detail})")


def decode_traffic_ratio(workload: str):
    """DRAM bytes per algorithmic byte of decode_kernel on this workload from
    the committed ncu summary, if it was taken on the decode source as it is
    now (else None)."""
    import hashlib
    import re
    path = os.path.join(ROOT, "profiles", f"decode_kernel_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    m_rat = re.search(r"dram_per_algorithmic_byte:\s*([0-9.]+)", text)
    if not (m_sha and m_rat):
        return None
    src = os.path.join(ROOT, "kv_cache_compression_hkv_b200", "csrc", "decode.cu")
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != m_sha.group(1):
        return None
    return float(m_rat.group(1))


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from kv_cache_compression_hkv_b200.inputs import WORKLOADS
    w = WORKLOADS[args.workload]
    if not args.profile and (args.seqs or args.layers):
        w = w.scaled(num_seqs=args.seqs or w.num_seqs, num_layers=args.layers or w.num_layers,
                     images=(args.seqs or w.num_seqs) * w.images // w.num_seqs)
    config = {"workload": w.name, "num_seqs": w.num_seqs, "images": w.images,
              "num_layers": w.num_layers, "num_heads": w.num_heads, "head_dim": w.head_dim,
              "max_len": w.max_len, "prefill_len": w.prefill_len, "decode_steps": w.decode_steps,
              "rho": f"{w.rho[0]}/{w.rho[1]}", "local_window": w.local_window, "ste_m": w.ste_m,
              "near_dist": w.near_dist, "l2": "inputs and cache larger than L2 (no flush needed)"}
    if args.mode != "headkv" or args.unstratified:
        config["budgets"] = args.mode
        config["strata"] = "pooled" if args.unstratified else "near/far"
    if args.cls_queries != 1 or args.cfg_pairing != "untied":
        config["grouping_queries"] = args.cls_queries
        config["cfg_pairing"] = args.cfg_pairing

    if args.impl == "reference":
        # the reference arm is the CPU oracle, on rank 0 only
        if rank != 0:
            return
        vals = []
        cores = 0
        per = max(2.0, min(args.cpu_seconds, 20.0))
        for i in range(args.warmup + args.steps):
            v, cores, n, el = oracle_sample(w, args.seed, per if i >= args.warmup else 1.0,
                                            opts=oracle_opts(args))
            if i >= args.warmup:
                vals.append(v)
        val = float(np.mean(vals))
        sample = f"whole (sequence, layer) units of {w.name} through the oracle, ~{per:.0f} s per step"
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            # a whole pass (every image token of the workload) at the sampled rate
            "ms_per_step": 1e3 * w.images * w.decode_steps / val,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config,
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}))
        return

    if args.profile:
        profile_run(args, w)
        return

    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    res = gpu_arm(args, rank, world, dev, w)
    torch.cuda.empty_cache()
    sweep = None
    if world == 1 and not args.no_sweep:
        sweep = sweep_arm(args, dev, w.name)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        v, cores, n, el = oracle_sample(w, args.seed, args.cpu_seconds, opts=oracle_opts(args))
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{n} whole (sequence, layer) units of {w.name} in {el:.1f} s "
                         f"(one unit = 1/{w.num_seqs * w.num_layers} of a pass)"}
        if cores > 1:
            v1, _, n1, el1 = oracle_sample(w, args.seed, max(1.0, args.cpu_seconds / 3),
                                           threads=1, opts=oracle_opts(args))
            cpu["single_core"] = {"value": v1, "unit": UNIT, "cores": 1,
                                  "sample": f"{n1} units in {el1:.1f} s"}
    if rank == 0:
        line = {
            "metric": METRIC, "value": res["tokens_per_s"], "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": res["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic (seeded planted-attention Q/K/V, shapes of the workload)",
            "config": config,
            "decode_step_us": res["decode_step_us"], "prefill_ms": res["prefill_ms"],
            "roofline": res["roofline"], "evict_us_avg": res["evict_us_avg"],
            "evict_us_max": res["evict_us_max"], "evict": res["evict"],
            "cpu_baseline": cpu, "e2e": res.get("e2e"), "gpu_launches": res["gpu_launches"],
            "clocks": res["clocks"], "full": res.get("full"),
            "speedup_decode_vs_full": res.get("speedup_decode_vs_full"),
            "speedup_pass_vs_full": res.get("speedup_pass_vs_full"),
            "kv_pool_bytes": res["kv_pool_bytes"], "labels_local_frac": res["labels_local_frac"],
            "labels_planted": res["labels_planted"],
            # whole decoder layers, compressed vs full cache, on the shapes the
            # pages compare end to end (the headline's own when it is one)
            "decoder_layer": res.get("decoder_layer") or
                {k: v["decoder_layer"] for k, v in (sweep or {}).items() if "decoder_layer" in v} or None,
            "all_configs": sweep,
        }
        print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
