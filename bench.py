#!/usr/bin/env python
"""LSA single-layer prefill throughput on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lsa|reference]
                    [--workload prefill-128k|prefill-4k|prefill-1m] [--mode flat|tree]
                    [--agg mean|max]

A step is one whole LSA attention layer over a T-token prompt (key build:
latents + Ward buckets; [tree]; per query chunk: query latents, centroid
scoring, selection + assembly, sparse attention), inputs already in HBM.
`value` = tokens/s summed over ranks (each rank runs its own layer: weak
scaling, no collective on the data path).  `e2e` repeats the measurement
through the whole-layer C-ABI call (lsa_prefill) from pinned host buffers,
with the Q/K/V upload and the O download inside the timed region.

--impl reference times the CPU oracle (the method restated in plain fp64 C)
on a bounded sample of the same workload, extrapolated to the same metric.
"""
from __future__ import annotations

import argparse
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
# kernel, averaged over the seven launches of one timed step of the workload
# (the committed ncu summary of attn_kernel gives the command); reported as
# `traffic` only while the kernel's source (the text from its template header
# to its launcher, hashed) is the one that capture measured.
ATTN_TRAFFIC = {"kernel_sha256_prefix": "d24e17fa489f0fb0", "bytes_per_query_kvhead": 19224.3,
                "workload": "prefill-128k"}


# Peak of the L2-to-SM read path on this machine's B200s, from ncu's
# l1tex__m_xbar2l1tex_read_bytes.sum.per_second (12.905 TB/s) and its
# pct_of_peak_sustained_elapsed (37.04%) for the gather attention kernel.
L2_TO_SM_PEAK_GBS = 12904.99 / 0.3703643


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
    p.add_argument("--workload", default="prefill-128k",
                   choices=["prefill-4k", "prefill-128k", "prefill-1m", "decode-32x1m", "decode-4x10m"])
    p.add_argument("--mode", default=None, choices=["flat", "tree"])
    p.add_argument("--agg", default=None, choices=["mean", "max"])
    p.add_argument("--chunk", type=int, default=16384)
    p.add_argument("--T", type=int, default=None, help="prefix length of the workload (profiling runs)")
    p.add_argument("--batch", type=int, default=None, help="decode requests (profiling runs)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu", action="store_true")
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


def config_json(args, c, world, chunk=None):
    return {
        "workload": args.workload, "T": c["T"], "hkv": c["hkv"], "hq": c["hq"], "d_head": c["d"],
        "d_latent": c["dl"], "k": c["k"], "sinks": c["sinks"], "window": c["window"],
        "search": "flat" if c["mode"] == 0 else f"tree(beam={c['beam']})",
        "query_score": "group-mean" if c["agg"] == 0 else "max-over-heads (native)",
        "query_chunk": chunk or args.chunk, "parallelism": f"replicas x{world} (one layer per GPU)",
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
    rng = np.random.default_rng(seed)
    lo = c["window"] + c["sinks"]
    tpos = np.sort(rng.choice(np.arange(lo, T), size=n_queries, replace=False))
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
    inp = synth.layer_inputs(args.workload, seed=0, T=c["T"], parts=("Q", "K", "V"))
    vals = []
    desc = ""
    full = {}
    for i in range(args.warmup + args.steps):
        per_layer, desc, _ = oracle_sample(inp, c, n_blocks=8, n_queries=16, seed=i, full=full)
        if i >= args.warmup:
            vals.append(c["T"] / per_layer)
    v = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * c["T"] / v,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_json(args, c, 1),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    emit_json(line)


def run_lsa(args):
    import torch

    import torch.distributed as dist

    import clustered_key_indexing_b200 as lsa
    from clustered_key_indexing_b200._lib import lib

    world, rank, local = dist_setup(args)
    c = workload_cfg(args)
    T, hkv, hq = c["T"], c["hkv"], c["hq"]
    cfg = lsa.Config(k=c["k"], sinks=c["sinks"], window=c["window"], beam=c["beam"],
                     mode=c["mode"], agg=c["agg"])
    dev = torch.device("cuda", torch.cuda.current_device())
    host_drawn = T <= 131072
    if host_drawn:
        inp = synth.layer_inputs(args.workload, seed=rank, T=T)

        def pinned(bits):
            return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory()

        hQ, hK, hV = pinned(inp["Q"]), pinned(inp["K"]), pinned(inp["V"])
        Q, K, V = hQ.to(dev), hK.to(dev), hV.to(dev)
        Wk_np, Wq_np = inp["Wk"], inp["Wq"]
    else:
        Q, K, V = synth.device_layer(c, rank, dev)
        hQ, hK, hV = (x.cpu().pin_memory() for x in (Q, K, V))
        Wk_np, Wq_np = synth.projections(rank, c["d"], c["dl"])
        inp = {"Wk": Wk_np, "Wq": Wq_np}
    Wk, Wq = torch.from_numpy(Wk_np).to(dev), torch.from_numpy(Wq_np).to(dev)
    cache = lsa.Cache(hkv, T, cfg, device=dev)
    tree = lsa.Tree(cache, device=dev) if cfg.mode == 1 else None
    O = torch.empty_like(Q)
    chunk = lsa.prefill_chunk(cfg, T, hq, hkv, args.chunk)
    row = cfg.row
    idx = torch.empty((chunk, hkv, row), dtype=torch.int32, device=dev)
    sws = torch.empty(lsa.select_workspace_bytes(cfg, chunk, hq, cache) or 1, dtype=torch.uint8, device=dev)
    aws = torch.empty(lsa.select_attn_workspace_bytes(chunk, hq) or 1, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    chunks = [(t0, min(chunk, T - t0)) for t0 in range(0, T, chunk)]
    def ev():
        return torch.cuda.Event(enable_timing=True)

    attn_ev = [(ev(), ev()) for _ in chunks]
    sel_ev = [(ev(), ev()) for _ in chunks]
    build_ev = (ev(), ev())

    def step(timed_attn=False):
        if timed_attn:
            build_ev[0].record(stream)
        lsa.build_buckets(K, Wk, cfg, cache)
        if tree is not None:
            lsa.build_tree(cache, cfg, tree)
        if timed_attn:
            build_ev[1].record(stream)
        for ci, (t0, n) in enumerate(chunks):
            if timed_attn:
                sel_ev[ci][0].record(stream)
            lsa.select(Q[t0:t0 + n], t0, Wq, cache, cfg, tree=tree, idx=idx[:n], ws=sws)
            if timed_attn:
                sel_ev[ci][1].record(stream)
                attn_ev[ci][0].record(stream)
            lsa.select_attn(Q[t0:t0 + n], K, V, idx[:n], t0, cfg, T, O=O[t0:t0 + n], ws=aws)
            if timed_attn:
                attn_ev[ci][1].record(stream)

    # index entries per step: gathered (sinks + long range) and window
    step()
    torch.cuda.synchronize()
    valid_g = valid_w = 0
    lsa.build_buckets(K, Wk, cfg, cache)
    if tree is not None:
        lsa.build_tree(cache, cfg, tree)
    ng = c["sinks"] + c["k"]
    for t0, n in chunks:
        lsa.select(Q[t0:t0 + n], t0, Wq, cache, cfg, tree=tree, idx=idx[:n], ws=sws)
        valid_g += int((idx[:n, :, :ng] >= 0).sum().item())
        valid_w += int((idx[:n, :, ng:] >= 0).sum().item())
    lsa.check_device_error()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = Clocks(torch.cuda.current_device())
    n0 = lib().lsa_launch_count()
    lib().lsa_fallback_rows()  # reset the counter
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    kt = lsa.KernelTimer()
    ev0.record(stream)
    attn_ms = sel_ms = build_ms = 0.0
    with kt:
        for _ in range(args.steps):
            step(timed_attn=True)
            torch.cuda.synchronize()  # read this step's stage events
            attn_ms += sum(a.elapsed_time(b) for a, b in attn_ev)
            sel_ms += sum(a.elapsed_time(b) for a, b in sel_ev)
            build_ms += build_ev[0].elapsed_time(build_ev[1])
        ev1.record(stream)
        torch.cuda.synchronize()
    kernels = {}
    for name in ("attn_kernel", "band_attn_kernel", "flat_cand_kernel", "flat_sample_kernel", "flat_resolve_kernel",
                 "latent_kernel", "ward_kernel", "select_fallback_kernel", "tree_select_kernel"):
        kms, kn = kt.get(name)
        if kn:
            kernels[name] = {"ms_per_step": kms / args.steps, "launches_per_step": kn / args.steps,
                             "ms_per_launch": kms / kn}
    clk = clocks.stop()
    launches = lib().lsa_launch_count() - n0
    fallback_rows = int(lib().lsa_fallback_rows())
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    if world > 1:
        dist.barrier()
    lsa.check_device_error()
    ms_step = ms / args.steps
    value = job_rate(world, T, ms_step)

    # e2e: the whole-layer C-ABI call from pinned host buffers
    e2e = None
    if not args.no_e2e:
        hO = torch.empty_like(hQ).pin_memory()
        pws = torch.empty(lsa.prefill_workspace_bytes(cfg, T, hq, hkv, chunk), dtype=torch.uint8, device=dev)
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

        def e2e_step():
            # lsa_prefill_host: uploads, the layer and the copy back, overlapped
            lsa.prefill_host(hQ, hK, hV, Wk, Wq, cfg, hO=hO, dev_bufs=(Q, K, V, O), cache=cache, tree=tree,
                             chunk=chunk, ws=pws, stream=stream, h2d_stream=up, d2h_stream=down)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), world, dev)
        e2e = {"value": job_rate(world, T, ems / args.steps), "unit": UNIT,
               "h2d_bytes_per_step": hQ.numel() * 2 + hK.numel() * 2 + hV.numel() * 2,
               "d2h_bytes_per_step": hO.numel() * 2}

    pk, src = peaks()
    for kv in kernels.values():
        kv["share_of_step"] = kv["ms_per_step"] / ms_step if ms_step > 0 else None
    # algorithmic work per step of the kernels with a roofline:
    #   attn_kernel: K and V rows of every gathered entry (2 x 256 B), its
    #     index entries (4 B), Q read, O write, the window partial (fp32 O and
    #     lse) read -- HBM-bound;
    #   band_attn_kernel: 4 x 128 FLOP per (window entry, query head) -- mma.sync;
    #   flat_cand_kernel / flat_sample_kernel: 2 x 64 FLOP per (row, scored
    #     centroid), every eligible / every 8th centroid -- tensor cores.
    G = hq // hkv
    rows_per_q = hq if cfg.agg else hkv
    NB = ((T + 3) // 4 + 127) // 128 * 64  # buckets per kv-head
    tt = np.arange(T, dtype=np.int64)
    lim = tt - c["window"]
    ncol = np.where(lim >= 0, np.minimum(NB, 64 * (np.maximum(lim, 0) // 512 + 1)), 0)
    work = {
        "attn_kernel": ("hbm", valid_g * (2 * 256 + 4) + T * hq * (2 * 256 + 4 * 129)),
        "band_attn_kernel": ("tensor", valid_w * G * 4 * 128),
        "flat_cand_kernel": ("tensor", 2 * 64 * rows_per_q * int(ncol.sum())),
        "flat_sample_kernel": ("tensor", 2 * 64 * rows_per_q * int(((ncol + 7) // 8).sum())),
    }

    def roof(name):
        bound, w = work[name]
        k = kernels.get(name)
        if not k:
            return None
        per_launch = w / k["launches_per_step"]
        sec = k["ms_per_launch"] / 1e3
        if bound == "hbm":
            ach, peak, unit = per_launch / sec / 1e9, pk["hbm_gbs"], "GB/s"
        else:
            ach, unit = per_launch / sec / 1e12, "TFLOP/s"
            peak = pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
        r = {"kernel": name, "bound": bound, "achieved": ach, "peak": peak, "unit": unit, "frac": ach / peak,
             "traffic": None, "peak_source": src + (" (sustained)" if bound == "tensor" else ""),
             "work_per_launch": per_launch, "ms_per_launch": k["ms_per_launch"],
             "share_of_step": k["share_of_step"]}
        if name == "attn_kernel":
            h = attn_kernel_hash()
            if (h and h == ATTN_TRAFFIC["kernel_sha256_prefix"] and args.workload == ATTN_TRAFFIC["workload"]
                    and ATTN_TRAFFIC["bytes_per_query_kvhead"]):
                r["traffic"] = ATTN_TRAFFIC["bytes_per_query_kvhead"] * T * hkv / k["launches_per_step"]
            r["note"] = ("gathered K/V rows are served mostly from L2 (one kv-head's K/V per wave), so the "
                         "algorithmic bytes can exceed the HBM copy peak; traffic = ncu DRAM bytes")
            # the same bytes against the L2-to-SM read path, whose peak ncu
            # gives as l1tex__m_xbar2l1tex_read_bytes' pct_of_peak (12.90
            # TB/s measured = 37.04% of peak in the 256K-prefix capture)
            l2_peak = L2_TO_SM_PEAK_GBS
            r["l2_view"] = {"achieved": ach, "peak": l2_peak, "unit": "GB/s", "frac": ach / l2_peak,
                            "peak_source": "ncu: l1tex__m_xbar2l1tex_read_bytes per second / its pct_of_peak"}
        return r

    ranked = sorted((n for n in work if n in kernels), key=lambda n: -kernels[n]["ms_per_step"])
    roofline = roof(ranked[0]) if ranked else None
    roofline_scoring = roof("flat_cand_kernel")
    if roofline_scoring:
        roofline_scoring["note"] = ("tcgen05 scores of every eligible centroid; the epilogue appends the candidates "
                                    "(score >= tau, about 2k keys' buckets per row), so the share of scores that are "
                                    "candidates -- high at short contexts -- bounds it with the tensor core's "
                                    "shared-memory operand reads")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        if not host_drawn:  # the oracle sample reads head 0's K/V and the query rows
            inp = {"Wk": Wk_np, "Wq": Wq_np, "K": bits_of(hK[:, :1]), "V": bits_of(hV[:, :1]),
                   "Q": bits_of(hQ)}
        per_layer, desc, spent = oracle_sample(inp, c, n_blocks=None if T <= 131072 else 64,
                                               n_queries=2048 if T <= 131072 else 64)
        cpu = {"value": T / per_layer, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
               "sample_seconds": spent}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_json(args, c, world, chunk), "clocks": clk, "e2e": e2e,
            "gpu_launches": int(launches), "roofline": roofline, "roofline_scoring": roofline_scoring,
            "kernels": kernels, "cpu_baseline": cpu,
            "stages_ms_per_step": {"build": build_ms / args.steps, "select": sel_ms / args.steps,
                                   "attention": attn_ms / args.steps},
            "select_fallback_rows_per_step": fallback_rows / args.steps,
        }
        emit_json(line)
    if world > 1:
        dist.destroy_process_group()


def run_decode(args):
    """Batched decode: `batch` requests whose prompts (built with
    lsa_decode_load, outside the timing) end so that the middle timed step
    appends the last key of a 512-key block in every request: the timed
    steps include one streaming Ward pass per request (with 512 timed steps
    that is exactly the steady-state rate of one block per 512 tokens)."""
    import torch
    import torch.distributed as dist

    import clustered_key_indexing_b200 as lsa
    from clustered_key_indexing_b200._lib import check, lib

    world, rank, local = dist_setup(args)
    c = workload_cfg(args)
    B, hkv, hq, T = c["batch"], c["hkv"], c["hq"], c["T"]
    cfg = lsa.Config(k=c["k"], sinks=c["sinks"], window=c["window"], beam=c["beam"],
                     mode=c["mode"], agg=c["agg"])
    dev = torch.device("cuda", torch.cuda.current_device())
    nsteps = args.warmup + args.steps
    n0 = decode_prompt_len(T, args.warmup, args.steps)
    cap = -(-(n0 + nsteps) // 512) * 512
    Wk_np, Wq_np = synth.projections(rank, c["d"], c["dl"])
    Wk, Wq = torch.from_numpy(Wk_np).to(dev), torch.from_numpy(Wq_np).to(dev)
    ccfg = cfg.c()
    if c.get("shared_prefix"):
        # one shared K/V for the prompt's whole blocks but the last, every
        # request's own tokens after it
        sl = 512 * ((n0 - 512) // 512)
        shared = synth.device_shared_prefix(c, rank, dev, sl)
        dec = lsa.Decode(B, hkv, hq, cap, cfg, device=dev, shared=shared)
        q, kk, vv = synth.device_decode_tails(c, rank, dev, sl, n0, nsteps, dec.K, dec.V)
    else:
        sl = 0
        dec = lsa.Decode(B, hkv, hq, cap, cfg, device=dev)
        q, kk, vv = synth.device_decode(c, rank, dev, n0, nsteps, dec.K, dec.V)
    for r in range(B):
        check(lib().lsa_decode_load(ctypes_ref(dec.d), r, n0, ctypes_ptr(Wk), ctypes_ref(ccfg),
                                    ctypes_ptr(dec.ws), dec.ws.numel(), None), "lsa_decode_load")
    o = torch.empty((B, hq, c["d"]), dtype=torch.bfloat16, device=dev)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    for s_ in range(args.warmup):
        dec.step(q[s_], kk[s_], vv[s_], Wk, Wq, o=o)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    lens0 = dec.len
    clocks = Clocks(torch.cuda.current_device())
    nl0 = lib().lsa_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    kt = lsa.KernelTimer()
    with kt:
        e0.record(stream)
        sev[0].record(stream)
        for i, s_ in enumerate(range(args.warmup, nsteps)):
            dec.step(q[s_], kk[s_], vv[s_], Wk, Wq, o=o)
            sev[i + 1].record(stream)
        e1.record(stream)
        torch.cuda.synchronize()
    step_ms = [sev[i].elapsed_time(sev[i + 1]) for i in range(args.steps)]
    # steps that append the last key of a block run the streaming Ward pass
    cl = [(n0 + args.warmup + i + 1) % 512 == 0 for i in range(args.steps)]
    plain = [m for m, f in zip(step_ms, cl) if not f]
    clus = [m for m, f in zip(step_ms, cl) if f]
    clk = clocks.stop()
    kernels = {}
    for name in ("decode_score_kernel", "decode_keep_kernel", "decode_resolve_kernel", "attn_kernel_split",
                 "decode_append_kernel", "latent_kernel", "ward_kernel", "tree_select_kernel"):
        kms, kn = kt.get(name)
        if kn:
            kernels[name] = {"ms_per_step": kms / args.steps, "launches_per_step": kn / args.steps}
    launches = lib().lsa_launch_count() - nl0
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    lsa.check_device_error()
    ms_step = ms / args.steps
    # algorithmic bytes per step: the centroids the search must read (128 B,
    # with a 4-byte record) -- flat: every eligible bucket; tree: the children
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
            byts += hkv * (nb * 132 + row * 512) + 2 * hq * c["d"] * 2
    byts /= args.steps
    pk, src = peaks()
    achieved = byts / (ms_step / 1e3) / 1e9
    if rank == 0:
        line = {
            "metric": "LSA decode steps/s", "value": job_rate(world, 1, ms_step), "unit": "steps/s",
            "tokens_per_s": job_rate(world, B, ms_step), "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "batch": B, "context": T, "shared_prefix": sl, "hkv": hkv, "hq": hq,
                       "k": c["k"], "sinks": c["sinks"], "window": c["window"],
                       "search": "flat" if c["mode"] == 0 else f"tree(beam={c['beam']})",
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
        emit_json(line)
    if world > 1:
        dist.destroy_process_group()


def decode_prompt_len(T, warmup, steps):
    """Prompt length after which step warmup + steps // 2 appends position
    T - 1 (T a multiple of 512: the last key of a cluster block)."""
    return T - 1 - warmup - steps // 2


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
