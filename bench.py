#!/usr/bin/env python
"""LSA single-layer prefill throughput on B200, with the decode step rate.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lsa|reference]
                    [--workload prefill-1m|prefill-128k|prefill-4k|decode-32x1m|decode-4x10m]
                    [--mode flat|tree] [--agg mean|max] [--no-tree] [--no-decode]

The default line: a step is one whole LSA attention layer over a 2^20-token
prompt (key build: latents + Ward buckets; per query chunk: query latents,
centroid scoring, selection + assembly, sparse attention), flat search,
inputs already in HBM; `value` = tokens/s of the layer.  The same line
carries
  tree    the same layer with tree search (beam 2), timed on its own;
  decode  the batched decode step rate, 32 requests x 2^20 tokens, measured
          after the prefill buffers are freed, with its HBM fraction;
  e2e     the layer through the C-ABI call lsa_prefill_host from pinned host
          Q/K/V into pinned host O, the copies inside the timed region.
The timed region holds only the steps (no per-launch events, no
synchronisation between steps); per-kernel and per-stage times come from a
pass of their own after it.

With N GPUs (torchrun), each rank takes hkv / N kv-heads of the one layer
and their query heads (no collective inside the layer: strong scaling), and
decode splits the requests.

--impl reference times the CPU oracle (the method restated in plain fp64 C)
on a bounded sample of the same workload, extrapolated to the same metric.
"""
from __future__ import annotations

import argparse
import ctypes
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "LSA layer prefill tokens/s"
UNIT = "tokens/s"

# ncu DRAM bytes (read + write) per (query, kv-head) of the gather attention
# kernel, summed over the 56 launches of one whole step of the workload (the
# committed launch-list summary of the 1M line gives the command); reported as
# `traffic` only while the kernel's source (the text from its template header
# to its launcher, hashed) is the one that capture measured.
ATTN_TRAFFIC = {"kernel_sha256_prefix": "2e3df2e5bd8b2f99", "bytes_per_query_kvhead": 310348.7,
                "workload": "prefill-1m"}



def attn_kernel_hash():
    import hashlib
    src = open(os.path.join(ROOT, "clustered_key_indexing_b200/csrc/lsa_attn.cu")).read()
    a, b = src.find("template <int SPLIT>"), src.find("lsa_status launch_attn(")
    return hashlib.sha256(src[a:b].encode()).hexdigest()[:16] if a >= 0 and b > a else None


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="lsa", choices=["lsa", "reference"])
    p.add_argument("--workload", default="prefill-1m",
                   choices=["prefill-4k", "prefill-128k", "prefill-1m", "decode-32x1m", "decode-4x10m"])
    p.add_argument("--mode", default=None, choices=["flat", "tree"])
    p.add_argument("--agg", default=None, choices=["mean", "max"])
    p.add_argument("--chunk", type=int, default=16384)
    p.add_argument("--T", type=int, default=None, help="prefix length of the workload (profiling runs)")
    p.add_argument("--batch", type=int, default=None, help="decode requests (profiling runs)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
    p.add_argument("--no-tree", action="store_true", help="skip the tree-search timing on the prefill line")
    p.add_argument("--no-decode", action="store_true", help="skip the decode block on the 1M prefill line")
    p.add_argument("--fp8", action="store_true", help="decode: FP8 (e4m3) centroid cache for the flat scan")
    p.add_argument("--pca", action="store_true", help="time the training-free projection fit on the workload's keys")
    p.add_argument("--backward", action="store_true",
                   help="time the sparse-attention backward over the layer's saved index rows")
    return p.parse_args()


def workload_cfg(args):
    c = dict(synth.CONFIGS[args.workload])
    if args.T:
        c["T"] = args.T
    if args.batch and "batch" in c:
        c["batch"] = args.batch
    if args.mode:
        c["mode"] = 0 if args.mode == "flat" else 1
    if args.agg:
        c["agg"] = 0 if args.agg == "mean" else 1
    return c


def config_json(args, c, world, split="none"):
    par = {"none": "1 GPU", "heads": f"kv-heads split over {world} GPUs ({c['hkv'] // world} each, no collective)",
           "replicas": f"replicas x{world} (one layer per GPU)"}[split]
    return {
        "workload": args.workload, "T": c["T"], "hkv": c["hkv"], "hq": c["hq"], "d_head": c["d"],
        "d_latent": c["dl"], "k": c["k"], "sinks": c["sinks"], "window": c["window"],
        "search": "flat" if c["mode"] == 0 else f"tree(beam={c['beam']})",
        "query_score": "group-mean" if c["agg"] == 0 else "max-over-heads (native)",
        "parallelism": par,
        "l2": "no flush: per-step inputs (Q/K/V) are larger than L2",
        "inputs": "host-drawn (numpy PCG64)" if c["T"] <= 131072 else "device-drawn (torch Philox), same recipe",
    }


# --------------------------------------------------------------- helpers

class Clocks:
    """nvidia-smi samples during the timed region."""

    def __init__(self, dev_index: int):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                       "-lms", "200", "-i", str(dev_index)], stdout=self.f,
                                      stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self) -> dict:
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.p.terminate()
        self.p.wait()
        self.f.seek(0)
        rows = [r.split(",") for r in self.f.read().strip().splitlines() if r.count(",") >= 8]
        os.unlink(self.f.name)
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if "Active" in v and "Not" not in v})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def emit_json(line):
    """Print the result line; any non-JSON value (reported on stderr with its
    key) is printed as text."""
    def walk(o, path):
        if isinstance(o, dict):
            for k, v in o.items():
                walk(v, f"{path}.{k}")
        elif isinstance(o, (list, tuple)):
            for i, v in enumerate(o):
                walk(v, f"{path}[{i}]")
        elif not isinstance(o, (str, int, float, bool, type(None))):
            print(f"bench.py: non-JSON value at {path}: {type(o).__name__} {o!r:.80}", file=sys.stderr)
    walk(line, "line")
    print(json.dumps(line, default=lambda o: o.decode(errors="replace") if isinstance(o, bytes) else str(o)),
          flush=True)


def peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


# ------------------------------------------------------------ CPU oracle

def oracle_sample(inp, c, n_blocks=None, n_queries=32, seed=0, full=None):
    """Time the oracle on one kv-head: the build of `n_blocks` cluster blocks
    (all if None) and select + attention for `n_queries` stratified positions.
    `full`: an optional dict that keeps the whole head's cache (the query
    sample needs it) between calls on the same inputs; that build is not
    part of the timed sample.
    Returns (seconds per layer extrapolated to T x hkv, description)."""
    import oracle
    T, hkv = c["T"], c["hkv"]
    G = c["hq"] // hkv
    ocfg = oracle.Cfg(k=c["k"], sinks=c["sinks"], window=c["window"], beam=c["beam"],
                      mode=c["mode"], agg=c["agg"])
    Tb = T if n_blocks is None else min(T, 512 * n_blocks)
    K1 = np.ascontiguousarray(inp["K"][:, :1])
    t0 = time.perf_counter()
    U = oracle.key_latent_pool(K1[:Tb], inp["Wk"], 4)
    cache = oracle.build_cache(U, Tb, ocfg)
    tree = oracle.build_tree(cache) if c["mode"] == 1 else None
    t_build = time.perf_counter() - t0
    if Tb < T:  # the query sample needs the whole head's cache
        if full is not None and "cache" in full:
            cache, tree = full["cache"], full["tree"]
        else:
            U = oracle.key_latent_pool(K1, inp["Wk"], 4)
            cache = oracle.build_cache(U, T, ocfg)
            tree = oracle.build_tree(cache) if c["mode"] == 1 else None
            if full is not None:
                full["cache"], full["tree"] = cache, tree
    # stratified positions: one uniform draw inside each of n_queries equal
    # slices of [W + S, T) (the selection's cost grows with t)
    rng = np.random.default_rng(seed)
    lo = c["window"] + c["sinks"]
    edges = lo + (np.arange(n_queries + 1) * (T - lo)) // n_queries
    tpos = np.array([rng.integers(a, max(a + 1, b)) for a, b in zip(edges[:-1], edges[1:])], np.int64)
    Qs = np.ascontiguousarray(inp["Q"][tpos][:, :G])
    t1 = time.perf_counter()
    Y = oracle.query_latent(Qs, inp["Wq"], 1, c["agg"])
    idx, _, _ = oracle.select(cache, Y, tpos, ocfg, tree=tree, G=G)
    oracle.attention(Qs, K1, np.ascontiguousarray(inp["V"][:, :1]), idx)
    t_q = (time.perf_counter() - t1) / n_queries
    per_layer = t_build * (T / Tb) * hkv + t_q * T * hkv
    desc = (f"1 of {hkv} kv-heads: build of {Tb // 512} blocks ({Tb} keys) + select/attention of "
            f"{n_queries} stratified query positions (G={G} heads), extrapolated to T={T} x {hkv} heads")
    return per_layer, desc, t_build + t_q * n_queries


# ------------------------------------------------------------------ main

def bits_of(t):
    return t.contiguous().view(torch_int16()).numpy().view(np.uint16)


def torch_int16():
    import torch
    return torch.int16


def max_over_ranks(ms, world, dev=None):
    """The slowest rank's time: every rank takes this one collective, in the
    same place (weak scaling, one independent layer or batch per rank)."""
    if world == 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=dev if dev is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world, units_per_rank, ms_per_step):
    """Whole-job throughput: the units all ranks processed per second, timed
    by the slowest rank."""
    return world * units_per_rank / (ms_per_step / 1e3)


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    c = workload_cfg(args)
    # the sample reads one kv-head: draw one kv-head (and its query heads) of
    # the workload's recipe on the host
    inp = synth.layer_inputs(args.workload, seed=0, T=c["T"], parts=("Q", "K", "V"), hkv=1)
    vals = []
    desc = ""
    full = {}
    for i in range(args.warmup + args.steps):
        per_layer, desc, _ = oracle_sample(inp, c, n_blocks=8, n_queries=16, seed=i, full=full)
        if i >= args.warmup:
            vals.append(c["T"] / per_layer)
    v = statistics.median(vals)
    spread = {"min": min(vals), "max": max(vals), "steps": len(vals)}
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * c["T"] / v,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_json(args, c, 1),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
                         "spread_over_steps": spread},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    emit_json(line)


def l2_read_peak(dev):
    """Peak of the L2-to-SM read path on this GPU, measured live: the
    library's lsa_l2_read streams a 48 MiB buffer (resident in the 126 MB
    L2) 32 times from 4 CTAs per SM; best of 10 timed launches."""
    import torch
    from clustered_key_indexing_b200._lib import check, lib
    nbytes, passes = 48 << 20, 32
    ctas = 4 * torch.cuda.get_device_properties(dev).multi_processor_count
    buf = torch.ones(nbytes, dtype=torch.uint8, device=dev)
    sink = torch.empty(int(lib().lsa_l2_read_sink_bytes(ctas)), dtype=torch.uint8, device=dev)
    st = torch.cuda.current_stream()
    sp = ctypes_ptr(sink)

    def launch():
        check(lib().lsa_l2_read(ctypes_ptr(buf), nbytes, passes, ctas, sp, ctypes.c_void_p(st.cuda_stream)),
              "lsa_l2_read")

    for _ in range(3):
        launch()
    best = float("inf")
    for _ in range(10):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        launch()
        e1.record(st)
        e1.synchronize()
        best = min(best, e0.elapsed_time(e1))
    gbs = int(lib().lsa_l2_read_bytes(nbytes, passes)) / (best / 1e3) / 1e9
    return gbs, (f"lsa_l2_read: {nbytes >> 20} MiB buffer x {passes} passes, 16-byte L1-bypassing loads, "
                 f"{ctas} CTAs x 512 threads, best of 10 launches (CUDA events), measured in this run")


class Prefill:
    """One rank's share of a prefill layer on the device: its kv-heads' Q/K/V
    (and pinned host copies for the e2e leg), cache, tree, per-chunk buffers."""

    def __init__(self, args, c, world, rank, dev):
        import torch

        import clustered_key_indexing_b200 as lsa
        from clustered_key_indexing_b200.shard import head_range
        self.lsa = lsa
        T, hkv, hq = c["T"], c["hkv"], c["hq"]
        self.split = "heads" if world > 1 and hkv % world == 0 else ("replicas" if world > 1 else "none")
        if self.split == "heads":
            h0, h1, q0, q1 = head_range(hkv, hq, world, rank)
            seed = 0            # one layer, each rank its heads of it
        else:
            h0, h1, q0, q1 = 0, hkv, 0, hq
            seed = rank         # one whole layer per rank
        self.hkv, self.hq, self.T = h1 - h0, q1 - q0, T
        if T <= 131072:
            inp = synth.layer_inputs(args.workload, seed=seed, T=T)
            Qb, Kb, Vb = (np.ascontiguousarray(inp[x][:, a:b]) for x, a, b in (("Q", q0, q1), ("K", h0, h1),
                                                                              ("V", h0, h1)))

            def pinned(bits):
                return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()

            self.hQ, self.hK, self.hV = pinned(Qb), pinned(Kb), pinned(Vb)
            self.Q, self.K, self.V = self.hQ.to(dev), self.hK.to(dev), self.hV.to(dev)
            self.Wk_np, self.Wq_np = inp["Wk"], inp["Wq"]
            self.inp = dict(inp, Q=Qb, K=Kb, V=Vb)
        else:
            Q, K, V = synth.device_layer(c, seed, dev)
            if self.split == "heads":
                Q, K, V = Q[:, q0:q1].contiguous(), K[:, h0:h1].contiguous(), V[:, h0:h1].contiguous()
                torch.cuda.empty_cache()
            self.Q, self.K, self.V = Q, K, V
            self.hQ, self.hK, self.hV = (x.cpu().pin_memory() for x in (Q, K, V))
            self.Wk_np, self.Wq_np = synth.projections(seed, c["d"], c["dl"])
            self.inp = None
        self.Wk, self.Wq = torch.from_numpy(self.Wk_np).to(dev), torch.from_numpy(self.Wq_np).to(dev)
        self.dev = dev
        self.c = c
        self.O = torch.empty_like(self.Q)
        self.args = args
        self.configure(c["mode"])

    def configure(self, mode):
        """Cache, tree (tree mode) and chunk buffers for search mode `mode`."""
        import torch
        lsa, c = self.lsa, self.c
        self.cfg = lsa.Config(k=c["k"], sinks=c["sinks"], window=c["window"], beam=c["beam"], mode=mode,
                              agg=c["agg"])
        if not hasattr(self, "cache"):
            self.cache = lsa.Cache(self.hkv, self.T, self.cfg, device=self.dev)
        self.tree = lsa.Tree(self.cache, device=self.dev) if mode == 1 else None
        self.chunk = lsa.prefill_chunk(self.cfg, self.T, self.hq, self.hkv, self.args.chunk)
        self.idx = torch.empty((self.chunk, self.hkv, self.cfg.row), dtype=torch.int32, device=self.dev)
        self.sws = torch.empty(lsa.select_workspace_bytes(self.cfg, self.chunk, self.hq, self.cache) or 1,
                               dtype=torch.uint8, device=self.dev)
        self.aws = torch.empty(lsa.select_attn_workspace_bytes(self.chunk, self.hq) or 1, dtype=torch.uint8,
                               device=self.dev)
        self.chunks = [(t0, min(self.chunk, self.T - t0)) for t0 in range(0, self.T, self.chunk)]

    def step(self, stage_ev=None, stream=None):
        """One whole layer; stage_ev: optional (build, [select per chunk],
        [attention per chunk]) event pairs recorded on `stream`."""
        lsa, cfg = self.lsa, self.cfg
        if stage_ev:
            stage_ev[0][0].record(stream)
        lsa.build_buckets(self.K, self.Wk, cfg, self.cache)
        if self.tree is not None:
            lsa.build_tree(self.cache, cfg, self.tree)
        if stage_ev:
            stage_ev[0][1].record(stream)
        for ci, (t0, n) in enumerate(self.chunks):
            if stage_ev:
                stage_ev[1][ci][0].record(stream)
            lsa.select(self.Q[t0:t0 + n], t0, self.Wq, self.cache, cfg, tree=self.tree, idx=self.idx[:n],
                       ws=self.sws)
            if stage_ev:
                stage_ev[1][ci][1].record(stream)
                stage_ev[2][ci][0].record(stream)
            lsa.select_attn(self.Q[t0:t0 + n], self.K, self.V, self.idx[:n], t0, cfg, self.T,
                            O=self.O[t0:t0 + n], ws=self.aws)
            if stage_ev:
                stage_ev[2][ci][1].record(stream)

    def entries(self):
        """Valid index entries of one layer: (gathered: sinks + long range, window)."""
        lsa, cfg = self.lsa, self.cfg
        lsa.build_buckets(self.K, self.Wk, cfg, self.cache)
        if self.tree is not None:
            lsa.build_tree(self.cache, cfg, self.tree)
        ng = self.c["sinks"] + self.c["k"]
        vg = vw = 0
        for t0, n in self.chunks:
            lsa.select(self.Q[t0:t0 + n], t0, self.Wq, self.cache, cfg, tree=self.tree, idx=self.idx[:n],
                       ws=self.sws)
            vg += int((self.idx[:n, :, :ng] >= 0).sum().item())
            vw += int((self.idx[:n, :, ng:] >= 0).sum().item())
        lsa.check_device_error()
        return vg, vw


def timed_steps(fn, steps, world, dev):
    """Device time of `steps` calls of fn (ms), bracketed by a barrier and a
    synchronize on both sides, max over ranks; no event or synchronisation
    between the steps."""
    import torch
    import torch.distributed as dist
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    return max_over_ranks(e0.elapsed_time(e1), world, dev)


def kernel_pass(P, steps, names):
    """Per-kernel and per-stage times of `steps` more steps (a pass of its
    own, after the timed region: every launch bracketed by CUDA events)."""
    import torch
    stream = torch.cuda.current_stream()

    def ev():
        return torch.cuda.Event(enable_timing=True)

    stage_ev = ((ev(), ev()), [(ev(), ev()) for _ in P.chunks], [(ev(), ev()) for _ in P.chunks])
    kt = P.lsa.KernelTimer()
    build = sel = attn = 0.0
    with kt:
        for _ in range(steps):
            P.step(stage_ev, stream)
            torch.cuda.synchronize()
            build += stage_ev[0][0].elapsed_time(stage_ev[0][1])
            sel += sum(a.elapsed_time(b) for a, b in stage_ev[1])
            attn += sum(a.elapsed_time(b) for a, b in stage_ev[2])
    kernels = {}
    for name in names:
        kms, kn = kt.get(name)
        if kn:
            kernels[name] = {"ms_per_step": kms / steps, "launches_per_step": kn / steps, "ms_per_launch": kms / kn}
    total = build + sel + attn
    for kv in kernels.values():
        kv["share_of_step"] = kv["ms_per_step"] * steps / total if total > 0 else None
    return kernels, {"build": build / steps, "select": sel / steps, "attention": attn / steps}


PREFILL_KERNELS = ("attn_kernel", "band_attn_kernel", "flat_cand_kernel", "flat_sample_kernel",
                   "flat_resolve_kernel", "latent_kernel", "ward_kernel", "select_fallback_kernel",
                   "tree_select_kernel", "tree_level_kernel", "sample_gather_kernel", "meta_gather_kernel")


def run_lsa(args):
    import torch

    from clustered_key_indexing_b200._lib import lib

    world, rank, local = dist_setup(args)
    c = workload_cfg(args)
    T = c["T"]
    dev = torch.device("cuda", torch.cuda.current_device())
    P = Prefill(args, c, world, rank, dev)
    lsa, cfg = P.lsa, P.cfg
    hkv, hq = P.hkv, P.hq
    scaling = "strong" if P.split == "heads" else "weak"
    units = T if P.split == "heads" else world * T   # tokens of the job per step

    P.step()
    torch.cuda.synchronize()
    valid_g, valid_w = P.entries()

    for _ in range(args.warmup):
        P.step()
    clocks = Clocks(torch.cuda.current_device())
    n0 = lib().lsa_launch_count()
    lib().lsa_fallback_rows()  # reset the counter
    ms = timed_steps(P.step, args.steps, world, dev)
    clk = clocks.stop()
    launches = lib().lsa_launch_count() - n0
    fallback_rows = int(lib().lsa_fallback_rows())
    lsa.check_device_error()
    ms_step = ms / args.steps
    value = units / (ms_step / 1e3)
    # per-kernel times: a separate pass after the timed region
    kernels, stages = kernel_pass(P, min(args.steps, 2), PREFILL_KERNELS)

    # e2e: the whole-layer C-ABI call from pinned host buffers
    e2e = None
    if not args.no_e2e:
        hO = torch.empty_like(P.hQ).pin_memory()
        pws = torch.empty(lsa.prefill_workspace_bytes(cfg, T, hq, hkv, P.chunk), dtype=torch.uint8, device=dev)
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        stream = torch.cuda.current_stream()

        def e2e_step():
            # lsa_prefill_host: uploads, the layer and the copy back, overlapped
            lsa.prefill_host(P.hQ, P.hK, P.hV, P.Wk, P.Wq, cfg, hO=hO, dev_bufs=(P.Q, P.K, P.V, P.O),
                             cache=P.cache, tree=P.tree, chunk=P.chunk, ws=pws, stream=stream, h2d_stream=up,
                             d2h_stream=down)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        ems = timed_steps(e2e_step, args.steps, world, dev)
        e2e = {"value": units / (ems / args.steps / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": (P.hQ.numel() + P.hK.numel() + P.hV.numel()) * 2,
               "d2h_bytes_per_step": hO.numel() * 2,
               "path": "lsa_prefill_host (pinned host Q/K/V in, O out; copies overlapped with the layer)"}
        del pws, hO

    pk, src = peaks()
    # algorithmic work per step of the kernels with a roofline:
    #   attn_kernel: K and V rows of every gathered entry (2 x 256 B), its
    #     index entries (4 B), Q read, O write, the window partial (fp32 O and
    #     lse) read;
    #   band_attn_kernel: 4 x 128 FLOP per (window entry, query head);
    #   flat_cand_kernel / flat_sample_kernel: 2 x 64 FLOP per (row, scored
    #     centroid), every eligible / every 8th centroid -- tensor cores.
    G = hq // hkv
    rows_per_q = hq if cfg.agg else hkv
    NB = ((T + 3) // 4 + 127) // 128 * 64  # buckets per kv-head
    tt = np.arange(T, dtype=np.int64)
    lim = tt - c["window"]
    ncol = np.where(lim >= 0, np.minimum(NB, 64 * (np.maximum(lim, 0) // 512 + 1)), 0)
    work = {
        "attn_kernel": ("l2", valid_g * (2 * 256 + 4) + T * hq * (2 * 256 + 4 * 129)),
        "band_attn_kernel": ("tensor", valid_w * G * 4 * 128),
        "flat_cand_kernel": ("tensor", 2 * 64 * rows_per_q * int(ncol.sum())),
        "flat_sample_kernel": ("tensor", 2 * 64 * rows_per_q * int(((ncol + 7) // 8).sum())),
    }
    l2_gbs, l2_how = l2_read_peak(dev)

    def roof(name):
        bound, w = work[name]
        k = kernels.get(name)
        if not k:
            return None
        per_launch = w / k["launches_per_step"]
        sec = k["ms_per_launch"] / 1e3
        if bound == "l2":
            ach, peak, unit, psrc = per_launch / sec / 1e9, l2_gbs, "GB/s", l2_how
        else:
            ach, unit = per_launch / sec / 1e12, "TFLOP/s"
            peak = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
            psrc = src + " (sustained cuBLAS bf16: the kernel runs inside a seconds-long step)"
        r = {"kernel": name, "bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
             "traffic": None, "peak_source": psrc, "work_per_launch": per_launch,
             "ms_per_launch": k["ms_per_launch"], "share_of_step": k["share_of_step"]}
        if name == "attn_kernel":
            h = attn_kernel_hash()
            if (h and h == ATTN_TRAFFIC["kernel_sha256_prefix"] and args.workload == ATTN_TRAFFIC["workload"]
                    and ATTN_TRAFFIC["bytes_per_query_kvhead"]):
                r["traffic"] = ATTN_TRAFFIC["bytes_per_query_kvhead"] * T * hkv / k["launches_per_step"]
            # the same kernel against HBM: the bytes it must bring from DRAM at
            # least once (every K/V row of its heads, the index rows, Q, O, the
            # window partial) -- a lower bound on its DRAM traffic
            distinct = T * hkv * 2 * 256 + T * hkv * (c["sinks"] + c["k"]) * 4 + T * hq * (2 * 256 + 4 * 129)
            dl = distinct / k["launches_per_step"]
            r["hbm_view"] = {"achieved": dl / sec / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                             "frac": dl / sec / 1e9 / pk["hbm_gbs"], "peak_source": src,
                             "bytes": "distinct bytes per launch (each K/V row once, index rows, Q, O, partials)"}
            r["note"] = ("gathered K/V rows are re-read from L2 by many queries (one kv-head's K/V per wave of "
                         "warps), so the kernel's bound is the L2-to-SM read rate, measured live by lsa_l2_read; "
                         "achieved = 516 B per valid gathered entry + Q, O and the window partial")
        return r

    ranked = sorted((n for n in work if n in kernels), key=lambda n: -kernels[n]["ms_per_step"])
    roofline = roof(ranked[0]) if ranked else None
    roofline_scoring = roof("flat_cand_kernel")
    if roofline_scoring:
        roofline_scoring["note"] = ("tcgen05 scores of every eligible centroid; the epilogue appends the candidates "
                                    "(score >= tau, about 2k keys' buckets per row)")
    roofline_band = roof("band_attn_kernel")
    if roofline_band:
        roofline_band["note"] = ("tcgen05 window attention: S = Q K^T and O = P V in tensor memory; achieved = "
                                 "4 x 128 FLOP per valid (window entry, query head)")

    # tree search over the same layer, timed on its own
    tree_line = None
    if cfg.mode == 0 and not args.no_tree:
        P.configure(1)
        for _ in range(2):
            P.step()
        tms = timed_steps(P.step, max(2, min(args.steps, 3)), world, dev) / max(2, min(args.steps, 3))
        tk, tst = kernel_pass(P, 1, PREFILL_KERNELS)
        tree_line = {"value": units / (tms / 1e3), "unit": UNIT, "ms_per_step": tms,
                     "search": f"tree(beam={c['beam']})", "stages_ms_per_step": tst,
                     "kernels": {n: v["ms_per_step"] for n, v in tk.items()}}
        P.configure(0)
        lsa.check_device_error()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        if P.inp is None:  # the oracle sample reads head 0's K/V and the query rows
            inp = {"Wk": P.Wk_np, "Wq": P.Wq_np, "K": bits_of(P.hK[:, :1]), "V": bits_of(P.hV[:, :1]),
                   "Q": bits_of(P.hQ)}
        else:
            inp = P.inp
        # about 10-20 s of oracle work: 128K: head 0's whole build + 2048
        # positions; 1M: 512 blocks + 640 positions (the head's whole cache,
        # which the positions need, is built outside the timed sample)
        per_layer, desc, spent = oracle_sample(inp, dict(c, hkv=hkv, hq=hq), n_blocks=None if T <= 131072 else 512,
                                               n_queries=2048 if T <= 131072 else 640)
        cpu = {"value": T / per_layer, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
               "sample_seconds": spent}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": scaling,
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_json(args, c, world, P.split), "query_chunk": P.chunk, "clocks": clk, "e2e": e2e,
        "gpu_launches": int(launches), "roofline": roofline, "roofline_scoring": roofline_scoring,
        "roofline_band": roofline_band,
        "tree": tree_line, "kernels": kernels, "cpu_baseline": cpu,
        "stages_ms_per_step": stages, "select_fallback_rows_per_step": fallback_rows / args.steps,
    }
    del P
    torch.cuda.empty_cache()
    if not args.no_decode and args.workload == "prefill-1m":
        # the decode step rate, after the prefill buffers are freed
        dargs = argparse.Namespace(**vars(args))
        dargs.workload, dargs.steps, dargs.warmup, dargs.mode = "decode-32x1m", 512, 3, None
        line["decode"] = decode_measure(dargs, world, rank, dev)
    if rank == 0:
        emit_json(line)
    if world > 1:
        dist_teardown()


def dist_teardown():
    import torch.distributed as dist
    dist.barrier()
    dist.destroy_process_group()


def run_decode(args):
    """Batched decode on its own (`--workload decode-*`): one line."""
    import torch
    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    d = decode_measure(args, world, rank, dev)
    if rank == 0:
        emit_json(d)
    if world > 1:
        dist_teardown()


def decode_measure(args, world, rank, dev):
    """Batched decode: `batch` requests (split over the ranks) whose prompts
    (built with lsa_decode_load, outside the timing) end so that the middle
    timed step appends the last key of a 512-key block in every request: the
    timed steps include one streaming Ward pass per request (with 512 timed
    steps that is exactly the steady-state rate of one block per 512
    tokens).  Returns the decode line (steps/s of the whole batch)."""
    import torch

    import clustered_key_indexing_b200 as lsa
    from clustered_key_indexing_b200._lib import check, lib
    from clustered_key_indexing_b200.shard import request_range

    c = workload_cfg(args)
    r0, r1 = request_range(c["batch"], world, rank)
    B, hkv, hq, T = r1 - r0, c["hkv"], c["hq"], c["T"]
    cfg = lsa.Config(k=c["k"], sinks=c["sinks"], window=c["window"], beam=c["beam"],
                     mode=c["mode"], agg=c["agg"])
    n0, nsteps, cap = decode_plan(T, args.warmup, args.steps)
    Wk_np, Wq_np = synth.projections(rank, c["d"], c["dl"])
    Wk, Wq = torch.from_numpy(Wk_np).to(dev), torch.from_numpy(Wq_np).to(dev)
    ccfg = cfg.c()
    cw = dict(c, batch=B)
    fp8 = bool(getattr(args, "fp8", False)) and cfg.mode == 0
    if c.get("shared_prefix"):
        # one shared K/V for the prompt's whole blocks but the last, every
        # request's own tokens after it
        sl = 512 * ((n0 - 512) // 512)
        shared = synth.device_shared_prefix(cw, rank, dev, sl)
        dec = lsa.Decode(B, hkv, hq, cap, cfg, device=dev, shared=shared, fp8=fp8)
        q, kk, vv = synth.device_decode_tails(cw, rank, dev, sl, n0, nsteps, dec.K, dec.V)
    else:
        sl = 0
        dec = lsa.Decode(B, hkv, hq, cap, cfg, device=dev, fp8=fp8)
        q, kk, vv = synth.device_decode(cw, rank, dev, n0, nsteps, dec.K, dec.V)
    for r in range(B):
        check(lib().lsa_decode_load(ctypes_ref(dec.d), r, n0, ctypes_ptr(Wk), ctypes_ref(ccfg),
                                    ctypes_ptr(dec.ws), dec.ws.numel(), None), "lsa_decode_load")
    o = torch.empty((B, hq, c["d"]), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    for s_ in range(args.warmup):
        dec.step(q[s_], kk[s_], vv[s_], Wk, Wq, o=o)
    lens0 = dec.len
    clocks = Clocks(torch.cuda.current_device())
    nl0 = lib().lsa_launch_count()
    it = iter(range(args.warmup, args.warmup + args.steps))

    def one():
        s_ = next(it)
        dec.step(q[s_], kk[s_], vv[s_], Wk, Wq, o=o)

    ms = timed_steps(one, args.steps, world, dev)
    clk = clocks.stop()
    launches = lib().lsa_launch_count() - nl0
    lsa.check_device_error()
    ms_step = ms / args.steps
    # a pass of its own for the per-step split and the per-kernel times: the
    # next `steps` steps, each step and each launch bracketed by events
    s1 = args.warmup + args.steps
    sev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    kt = lsa.KernelTimer()
    with kt:
        sev[0].record(stream)
        for i, s_ in enumerate(range(s1, nsteps)):
            dec.step(q[s_], kk[s_], vv[s_], Wk, Wq, o=o)
            sev[i + 1].record(stream)
        torch.cuda.synchronize()
    step_ms = [sev[i].elapsed_time(sev[i + 1]) for i in range(args.steps)]
    # steps that append the last key of a block run the streaming Ward pass
    cl = [(n0 + s1 + i + 1) % 512 == 0 for i in range(args.steps)]
    plain = [m for m, f in zip(step_ms, cl) if not f]
    clus = [m for m, f in zip(step_ms, cl) if f]
    kernels = {}
    for name in ("decode_score_kernel", "decode_keep_kernel", "decode_resolve_kernel", "attn_kernel_split",
                 "decode_append_kernel", "latent_kernel", "ward_kernel", "tree_select_kernel"):
        kms, kn = kt.get(name)
        if kn:
            kernels[name] = {"ms_per_step": kms / args.steps, "launches_per_step": kn / args.steps}
    lsa.check_device_error()
    # algorithmic bytes per step: the centroids the search must read (128 B,
    # FP8 64 B, with a 4-byte record) -- flat: every eligible bucket; tree: the children
    # of the beam at every level above L* plus the B * 2^L* leaves under the
    # final beam -- the gathered K/V rows of every index entry (512 B), Q and O
    row = cfg.row
    if cfg.mode == 1:
        lstar = 0
        while c["beam"] * 8 * (1 << lstar) < c["k"]:
            lstar += 1
        tree_nodes = 2 * c["beam"] * (dec.tree.levels - 1 - lstar) + c["beam"] * (1 << lstar)
    byts = 0.0
    for t in lens0:
        for s_ in range(args.steps):
            pos = t + s_
            lim = pos - c["window"]
            nb = min(cap // 512 * 64, 64 * (lim // 512 + 1))
            nb = min(nb, 64 * ((pos + 1) // 512))
            if cfg.mode == 1:
                nb = min(nb, tree_nodes)
            byts += hkv * (nb * (68 if fp8 else 132) + row * 512) + 2 * hq * c["d"] * 2
    byts /= args.steps
    pk, src = peaks()
    achieved = byts / (ms_step / 1e3) / 1e9
    del dec, q, kk, vv, o
    torch.cuda.empty_cache()
    return {
        "metric": "LSA decode steps/s", "value": 1e3 / ms_step, "unit": "steps/s",
        "tokens_per_s": c["batch"] * 1e3 / ms_step, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "strong" if world > 1 else "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "batch": c["batch"], "context": T, "shared_prefix": sl, "hkv": hkv,
                   "hq": hq, "k": c["k"], "sinks": c["sinks"], "window": c["window"],
                   "search": "flat" if c["mode"] == 0 else f"tree(beam={c['beam']})",
                   "centroids": "fp8 e4m3 (64 B)" if fp8 else "bf16 (128 B)",
                   "parallelism": f"requests split over {world} GPU(s)" if world > 1 else "1 GPU",
                   "inputs": "device-drawn (torch Philox), same recipe as synth",
                   "l2": f"no flush: per-step centroid scan ({byts / 1e9:.1f} GB) is larger than L2"},
        "clocks": clk, "gpu_launches": int(launches), "kernels": kernels,
        "ms_per_step_without_clustering": float(np.mean(plain)) if plain else None,
        "ms_per_clustering_step": float(np.mean(clus)) if clus else None,
        "clustering_steps": len(clus),
        "roofline": {"kernel": "decode step (centroid scan + gather + attention)", "bound": "hbm",
                     "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / pk["hbm_gbs"], "traffic": None, "peak_source": src,
                     "bytes_per_step": byts},
    }


def decode_prompt_len(T, warmup, steps):
    """Prompt length after which step warmup + steps // 2 appends position
    T - 1 (T a multiple of 512: the last key of a cluster block)."""
    return T - 1 - warmup - steps // 2


def decode_plan(T, warmup, steps):
    """(prompt length n0, steps drawn, pool capacity) of a decode run: the
    warm-up steps, the timed steps, then as many again for the per-kernel
    pass."""
    n0 = decode_prompt_len(T, warmup, steps)
    nsteps = warmup + 2 * steps
    return n0, nsteps, -(-(n0 + nsteps) // 512) * 512


def run_pca(args):
    """The training-free projection (lsa_fit_pca) on the workload's keys: one
    step = one fit over all T * hkv keys (fp64 second moments + Jacobi)."""
    import torch

    import clustered_key_indexing_b200 as lsa

    world, rank, local = dist_setup(args)
    c = workload_cfg(args)
    dev = torch.device("cuda", torch.cuda.current_device())
    if c["T"] <= 131072:
        K = torch.from_numpy(synth.layer_inputs(args.workload, seed=rank, T=c["T"], parts=("K",))["K"]
                             .view(np.int16)).view(torch.bfloat16).to(dev)
    else:
        _, K, _ = synth.device_layer(dict(c, hq=c["hkv"]), rank, dev)
    N = K.shape[0] * K.shape[1]
    for _ in range(args.warmup):
        lsa.fit_pca(K)
    torch.cuda.synchronize()
    clocks = Clocks(torch.cuda.current_device())
    kt = lsa.KernelTimer()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with kt:
        e0.record(stream)
        for _ in range(args.steps):
            W, eig = lsa.fit_pca(K)
        e1.record(stream)
        torch.cuda.synchronize()
    clk = clocks.stop()
    lsa.check_device_error()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
    kms, kn = kt.get("pca_moments_kernel")
    jms, jn = kt.get("pca_jacobi_kernel")
    # algorithmic work of the moments: one fp64 FMA per key and per entry of
    # the symmetric 128 x 128 matrix's upper triangle; peak: 148 SMs x 64
    # fp64 FMA per clock x 2 FLOP x 1965 MHz
    flops = N * (128 * 129 // 2) * 2.0
    peak = 148 * 64 * 2 * 1.965e9 / 1e12
    mom_ms = kms / max(kn, 1)
    achieved = flops / (mom_ms / 1e3) / 1e12
    if rank == 0:
        emit_json({
            "metric": "LSA PCA projection fit keys/s", "value": job_rate(world, N, ms), "unit": "keys/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": args.workload, "T": c["T"], "hkv": c["hkv"], "keys": N,
                                            "d_latent": 64, "l2": "no flush: the keys are larger than L2"},
            "clocks": clk, "gpu_launches": 3 * args.steps,
            "kernels": {"pca_moments_kernel": mom_ms, "pca_jacobi_kernel": jms / max(jn, 1)},
            "roofline": {"kernel": "pca_moments_kernel", "bound": "alu", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                         "peak_source": "derived: 148 SMs x 64 fp64 FMA/clk x 2 x 1965 MHz",
                         "work_per_launch": flops},
            "eigenvalues_top4": [float(x) for x in eig[:4].cpu()],
        })


def oracle_backward_sample(inp, c, n_queries=16, seed=0):
    """Time the oracle's attention backward on one kv-head: rows of
    `n_queries` stratified positions from the oracle's own selection, O from
    the oracle's forward, then oracle.attention_backward over those rows.
    Returns (seconds per layer extrapolated to T x hkv, description)."""
    import oracle
    T, hkv = c["T"], c["hkv"]
    G = c["hq"] // hkv
    ocfg = oracle.Cfg(k=c["k"], sinks=c["sinks"], window=c["window"], beam=c["beam"],
                      mode=c["mode"], agg=c["agg"])
    K1 = np.ascontiguousarray(inp["K"][:, :1])
    V1 = np.ascontiguousarray(inp["V"][:, :1])
    cache = oracle.build_cache(oracle.key_latent_pool(K1, inp["Wk"], 4), T, ocfg)
    tree = oracle.build_tree(cache) if c["mode"] == 1 else None
    rng = np.random.default_rng(seed)
    lo = c["window"] + c["sinks"]
    tpos = np.sort(rng.choice(np.arange(lo, T), size=n_queries, replace=False))
    Qs = np.ascontiguousarray(inp["Q"][tpos][:, :G])
    Y = oracle.query_latent(Qs, inp["Wq"], 1, c["agg"])
    idx, _, _ = oracle.select(cache, Y, tpos, ocfg, tree=tree, G=G)
    dO = rng.standard_normal(Qs.shape)
    t0 = time.perf_counter()
    oracle.attention_backward(Qs, K1, V1, idx, dO)
    t_q = (time.perf_counter() - t0) / n_queries
    desc = (f"1 of {hkv} kv-heads: attention backward over the oracle's own rows at {n_queries} stratified "
            f"query positions (G={G} heads), extrapolated to T={T} x {hkv} heads")
    return t_q * T * hkv, desc


def run_backward(args):
    """The sparse-attention backward (lsa_attn_backward) over a prefill
    layer's saved index rows: one step = dQ, dK, dV of all T queries, with dK
    and dV zeroed first.  The rows and the forward output O come from the
    library's own selection and attention before the timed region."""
    import torch

    import clustered_key_indexing_b200 as lsa

    world, rank, local = dist_setup(args)
    c = workload_cfg(args)
    T, hkv, hq = c["T"], c["hkv"], c["hq"]
    cfg = lsa.Config(k=c["k"], sinks=c["sinks"], window=c["window"], beam=c["beam"],
                     mode=c["mode"], agg=c["agg"])
    dev = torch.device("cuda", torch.cuda.current_device())
    if T > 131072:
        raise SystemExit("--backward keeps every query's index row: use a workload of at most 131072 tokens")
    inp = synth.layer_inputs(args.workload, seed=rank, T=T)

    def on_dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)

    Q, K, V = on_dev(inp["Q"]), on_dev(inp["K"]), on_dev(inp["V"])
    Wk, Wq = torch.from_numpy(inp["Wk"]).to(dev), torch.from_numpy(inp["Wq"]).to(dev)
    cache = lsa.Cache(hkv, T, cfg, device=dev)
    tree = lsa.Tree(cache, device=dev) if cfg.mode == 1 else None
    lsa.build_buckets(K, Wk, cfg, cache)
    if tree is not None:
        lsa.build_tree(cache, cfg, tree)
    idx = torch.empty((T, hkv, cfg.row), dtype=torch.int32, device=dev)
    chunk = lsa.prefill_chunk(cfg, T, hq, hkv, args.chunk)
    for t0 in range(0, T, chunk):
        n = min(chunk, T - t0)
        lsa.select(Q[t0:t0 + n], t0, Wq, cache, cfg, tree=tree, idx=idx[t0:t0 + n])
    O = lsa.sparse_attn(Q, K, V, idx)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + rank)
    dO = torch.randn(Q.shape, generator=gen, device=dev, dtype=torch.float32).to(torch.bfloat16)
    dQ = torch.empty((T, hq, 128), dtype=torch.float32, device=dev)
    dK = torch.zeros((T, hkv, 128), dtype=torch.float32, device=dev)
    dV = torch.zeros_like(dK)
    stream = torch.cuda.current_stream()

    def step():
        dK.zero_()
        dV.zero_()
        lsa.attn_backward(Q, K, V, O, dO, idx, dK=dK, dV=dV)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    lsa.check_device_error()
    clocks = Clocks(torch.cuda.current_device())
    kt = lsa.KernelTimer()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with kt:
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        torch.cuda.synchronize()
    clk = clocks.stop()
    lsa.check_device_error()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
    bms, bn = kt.get("attn_bwd_kernel")
    bwd_ms = bms / max(bn, 1)
    # algorithmic bytes per valid index entry: the K row twice (statistics,
    # then gradients) and the V row once, 256 B each, plus the fp32 dK and dV
    # rows added to (2 x 512 B)
    n_valid = int((idx >= 0).sum())
    bytes_ = n_valid * (3 * 256 + 2 * 512.0)
    pk, src = peaks()
    achieved = bytes_ / (bwd_ms / 1e3) / 1e9
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        per_layer, desc = oracle_backward_sample(inp, c)
        cpu = {"value": T / per_layer, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": desc}
    if rank == 0:
        emit_json({
            "metric": "LSA attention backward tokens/s", "value": job_rate(world, T, ms), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": args.workload, "T": T, "hkv": hkv, "hq": hq, "k": c["k"], "sinks": c["sinks"],
                       "window": c["window"], "index_entries": n_valid,
                       "l2": "no flush: per-step K/V gathers and dK/dV (fp32) are larger than L2"},
            "clocks": clk, "gpu_launches": args.steps, "e2e": None,
            "kernels": {"attn_bwd_kernel": bwd_ms},
            "roofline": {"kernel": "attn_bwd_kernel", "bound": "hbm", "achieved": achieved,
                         "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": achieved / pk["hbm_gbs"],
                         "traffic": None, "peak_source": src, "bytes_per_launch": bytes_},
            "cpu_baseline": cpu,
        })


def ctypes_ref(x):
    import ctypes
    return ctypes.byref(x)


def ctypes_ptr(t):
    import ctypes
    return ctypes.c_void_p(t.data_ptr())


if __name__ == "__main__":
    a = parse()
    if a.impl == "reference":
        run_reference(a)
    elif a.pca:
        run_pca(a)
    elif a.backward:
        run_backward(a)
    elif a.workload.startswith("decode"):
        run_decode(a)
    else:
        run_lsa(a)
