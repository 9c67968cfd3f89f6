#!/usr/bin/env python
"""Benchmark of the routed MoE FFN layer on B200 (one JSON line on stdout, rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one moe_forward of the whole layer (router -> top-k -> bucketing -> experts ->
combine with the shared expert) over one batch of synthetic tokens.  Workloads (seed 0,
synthetic inputs of the pages' model shapes; no datasets or trained weights):

  glm_decode   (default) GLM-5.2-like layer, T=1: d=6144, E=256, top-8 sigmoid router with
               selection bias, x2.5 scaling, f=2048 int4 experts (+1 shared), ~4.8 GB resident
  glm_union2   the same layer, T=2 (batch-union)
  glm_union32  the same layer, T=32 (batch-union)
  glm_prefill  the same layer, T=2048, bf16 output
  granite      Granite-1B-a400m-like decode layer: T=1, d=1024, E=32, top-8 softmax, f=512 bf16
  tiny         T=4, d=256, E=8, top-2 softmax, f=128 int4

The JSON line's top level is the headline workload (--workload, glm_decode by default); the
other five workloads are measured in the same run and reported under "workloads", each with its
own roofline, end-to-end figure and CPU baseline (--workloads none skips them).

Timing: CUDA events on the launching stream around every step; between steps, outside the
events, a read-only sweep of a 512 MiB buffer evicts L2 (it leaves no dirty lines behind, so no
write-back lands inside the next step).  Multi-GPU: one process per GPU, each a data-parallel
replica with its own token stream; value = all ranks' tokens / max over ranks of device time.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic as syn  # noqa: E402

METRIC = "MoE-layer tokens/s"
WORKLOADS = {
    "glm_decode": "GLM-5.2-like MoE layer decode, T=1, d=6144, E=256, top-8 sigmoid+bias x2.5, f=2048 int4 + 1 shared",
    "glm_union2": "GLM-5.2-like MoE layer batch-union decode, T=2",
    "glm_union32": "GLM-5.2-like MoE layer batch-union decode, T=32",
    "glm_prefill": "GLM-5.2-like MoE layer prefill, T=2048, bf16 out",
    "granite": "Granite-1B-a400m-like MoE layer decode, T=1, d=1024, E=32, top-8 softmax, f=512 bf16",
    "tiny": "tiny MoE layer, T=4, d=256, E=8, top-2 softmax, f=128 int4",
    "glm_decode_int8": "GLM-5.2-like MoE layer decode, T=1, experts in the int8 container (one code per byte)",
    "glm_decode_int2": "GLM-5.2-like MoE layer decode, T=1, experts in the packed int2 container (four codes per byte)",
    "glm_decode_variants": "GLM-5.2-like MoE layer decode, T=1, group-limited selection (8 groups, 4 kept) and "
                           "adaptive expert top-p 0.7",
    "glm_decode_tiered": "GLM-5.2-like MoE layer decode, T=1, routed experts in pinned host memory behind a tier of "
                         "64 expert slots in HBM (each step: route, stream the missing experts in, forward)",
}
TIER_SLOTS = 64
# layer options of workloads that use the router variants: (n_group, topk_group, top_p)
ROUTER_VARIANTS = {"glm_decode_variants": (8, 4, 0.7)}
WORKLOAD_ORDER = ["glm_decode", "glm_union2", "glm_union32", "glm_prefill", "glm_decode_variants", "glm_decode_tiered",
                  "granite", "tiny", "glm_decode_int8", "glm_decode_int2"]
DEFAULT_STEPS = {"glm_decode_int8": 500, "glm_decode_int2": 500, "glm_decode_variants": 500, "glm_decode_tiered": 100, "glm_decode": 2000, "glm_union2": 1000, "glm_union32": 200, "glm_prefill": 60, "granite": 2000,
                 "tiny": 200}
FLUSH_BYTES = 512 << 20
# The Granite layer's 32 experts (100 MB of bf16) fit in L2, so its token stream is also timed
# L2-warm, both as plain launches and as one CUDA graph (labelled: not HBM figures).
DEFAULT_WARM_PASSES = {"granite": "both"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="glm_decode", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the oracle CPU baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's tokens per step (smaller cases for profiling)")
    ap.add_argument("--t1-mode", type=int, default=None, choices=[0, 1, 2],
                    help="single-token path: 2 one launch, 1 three kernels, 0 general kernels (default: the library's)")
    ap.add_argument("--experts", type=int, default=None,
                    help="override E (smaller device footprint for profiler captures; same per-token work)")
    ap.add_argument("--workloads", default="all",
                    help="workloads measured besides the headline one: all, none, or a comma-separated list")
    ap.add_argument("--warm-passes", default=None, choices=["none", "stream", "graph", "both"],
                    help="extra L2-warm passes (no flush between steps; not HBM figures): the steps as plain "
                         "stream launches, replayed from one CUDA graph, or both (default: both for granite)")
    a = ap.parse_args()
    a.steps_given = a.steps
    if a.steps is None:
        a.steps = DEFAULT_STEPS[a.workload]
    a.warmup = max(a.warmup, 3)
    return a


# columns per byte of a weight row, per container (bf16 is 2 bytes per column, no scales)
CODES_PER_BYTE = {syn.W_INT4: 2, syn.W_INT8: 1, syn.W_INT2: 4}


def row_bytes(cfg, cols) -> int:
    """Bytes of one weight row of `cols` columns, with its fp32 scale when the container has one."""
    if cfg.wkind == syn.W_BF16:
        return cols * 2
    return cols // CODES_PER_BYTE[cfg.wkind] + 4


def expert_bytes(cfg, f=None) -> int:
    f = cfg.f if f is None else f
    return 2 * f * row_bytes(cfg, cfg.d) + cfg.d * row_bytes(cfg, f)


def workload_config(name):
    """The layer configuration of a workload: the five synthetic configurations, and the GLM decode
    layer in the int8 and packed int2 containers."""
    if name in syn.CONFIGS:
        return syn.CONFIGS[name]
    if name in ROUTER_VARIANTS or name == "glm_decode_tiered":
        return dataclasses.replace(syn.CONFIGS["glm_decode"], name=name)
    base, kind = name.rsplit("_", 1)
    return dataclasses.replace(syn.CONFIGS[base], name=name,
                               wkind={"int8": syn.W_INT8, "int2": syn.W_INT2}[kind])


# ------------------------------------------------------------------------------------------
# device-side layer and inputs
# ------------------------------------------------------------------------------------------

def build_device_layer(cfg, seed, max_tokens, device):
    import torch

    import quantized_expert_ffn_02_b200 as qe

    E, d, f = cfg.E, cfg.d, cfg.f
    int4 = cfg.wkind != syn.W_BF16       # a container of codes with per-row scales
    W = {}
    if int4:
        cpb = CODES_PER_BYTE[cfg.wkind]
        dt = torch.int8 if cfg.wkind == syn.W_INT8 else torch.uint8
        packer = {syn.W_INT4: qe.moe_pack_int4, syn.W_INT8: qe.moe_pack_int8, syn.W_INT2: qe.moe_pack_int2}[cfg.wkind]

    def mat(name, rows, cols):
        return syn.torch_normal_fp32(seed, name, rows * cols, syn.WEIGHT_STD, device).view(rows, cols)

    def alloc(prefix, n, f_):
        if int4:
            W[prefix + "gate_up"] = torch.empty((n, 2 * f_, d // cpb), dtype=dt, device=device)
            W[prefix + "gate_up_scale"] = torch.empty((n, 2 * f_), dtype=torch.float32, device=device)
            W[prefix + "down"] = torch.empty((n, d, f_ // cpb), dtype=dt, device=device)
            W[prefix + "down_scale"] = torch.empty((n, d), dtype=torch.float32, device=device)
        else:
            W[prefix + "gate_up"] = torch.empty((n, 2 * f_, d), dtype=torch.int16, device=device)
            W[prefix + "down"] = torch.empty((n, d, f_), dtype=torch.int16, device=device)

    def fill(prefix, i, e, f_):
        for which, rows, cols in (("gate_up", 2 * f_, d), ("down", d, f_)):
            w = mat(syn.expert_tensor_name(e, which), rows, cols)
            if int4:
                packer(w, W[prefix + which][i], W[prefix + which + "_scale"][i])
            else:
                W[prefix + which][i].copy_(w.to(torch.bfloat16).view(torch.int16))

    alloc("", E, f)
    for e in range(E):
        fill("", e, e, f)
    if cfg.n_shared:
        alloc("shared_", 1, cfg.f_shared)
        fill("shared_", 0, "shared", cfg.f_shared)
        for key in list(W):
            if key.startswith("shared_"):
                W[key] = W[key][0]
    W["router_w"] = torch.from_numpy(syn.gen_router_w(cfg, seed)).to(device)
    b = syn.gen_router_bias(cfg, seed)
    W["router_bias"] = None if b is None else torch.from_numpy(b).to(device)
    torch.cuda.synchronize()
    return layer_on(cfg, W, max_tokens), W


class TieredLayer:
    """The GLM layer with its routed experts in pinned host memory behind a tier of expert slots in
    HBM (moe_expert_cache_*): each forward first makes the batch's experts resident."""

    def __init__(self, cfg, W, max_tokens, n_slots):
        import quantized_expert_ffn_02_b200 as qe
        self.qe = qe
        device = {n: W.get(n) for n in ("router_w", "router_bias", "shared_gate_up", "shared_gate_up_scale",
                                        "shared_down", "shared_down_scale")}
        self.host = {n: W[n].cpu().pin_memory() for n in ("gate_up", "gate_up_scale", "down", "down_scale")}
        self.cache = qe.ExpertCache(cfg.d, cfg.f, cfg.E, cfg.k, max_tokens, cfg.router, cfg.wkind, device, self.host,
                                    n_slots, n_shared=cfg.n_shared, f_shared=cfg.f_shared,
                                    routed_scaling_factor=cfg.scaling, out_bf16=cfg.out_bf16)
        self.handle = self.cache.layer
        self._xd = None

    def route(self, x, idx, w, stream=None):
        self.qe.moe_route(self.handle, x, x.shape[0], idx, w, stream)

    def forward(self, x, out, stream=None):
        self.cache.prepare(x, stream)
        self.qe.moe_forward(self.handle, x, x.shape[0], out, stream)

    def forward_host_async(self, x_host, out_host, stream=None):
        import torch
        if self._xd is None or self._xd.shape != x_host.shape:
            self._xd = torch.empty(x_host.shape, dtype=x_host.dtype, device="cuda")
            self._od = torch.empty(out_host.shape, dtype=out_host.dtype, device="cuda")
        self._xd.copy_(x_host, non_blocking=True)
        self.forward(self._xd, self._od, stream)
        out_host.copy_(self._od, non_blocking=True)

    def forward_host(self, x_host, out_host, stream=None):
        import torch
        self.forward_host_async(x_host, out_host, stream)
        torch.cuda.current_stream().synchronize()

    def last_error(self):
        return self.qe.moe_last_error(self.handle)

    def last_launches(self):
        return self.qe.moe_layer_last_launches(self.handle)

    def set_single_token_mode(self, mode):
        self.qe.moe_layer_set_option(self.handle, self.qe.MOE_OPT_SINGLE_TOKEN_KERNELS, int(mode))

    def profile(self, on):
        self.qe.moe_profile_enable(self.handle, on)

    def profile_read(self):
        out = {}
        for kid, kname in enumerate(self.qe.KERNELS):
            ms, n = self.qe.moe_profile_read(self.handle, kid)
            if n:
                out[kname] = (ms, n)
        return out

    def stats(self):
        return self.cache.stats()

    def close(self):
        self.cache.close()


def layer_on(cfg, W, max_tokens):
    """A layer handle over already-resident weights (several handles may share one set)."""
    import quantized_expert_ffn_02_b200 as qe
    return qe.MoELayer(cfg.d, cfg.f, cfg.E, cfg.k, max_tokens, cfg.router, cfg.wkind, W, n_shared=cfg.n_shared,
                       f_shared=cfg.f_shared, routed_scaling_factor=cfg.scaling, out_bf16=cfg.out_bf16)


def make_batches(cfg, T, n, seed, token_offset, device):
    """n batches of T tokens: token stream "x" from `token_offset` on (bf16 bits as int16)."""
    import torch
    out = []
    for i in range(n):
        v = syn.torch_normal_fp32(seed, "x", T * cfg.d, 1.0, device, offset=(token_offset + i * T) * cfg.d)
        out.append(v.to(torch.bfloat16).view(torch.int16).view(T, cfg.d))
    return out


# ------------------------------------------------------------------------------------------
# replicas (one process per GPU, no data-path collective)
# ------------------------------------------------------------------------------------------

def replica_token_base(rank: int) -> int:
    """First token of a rank's own stream: every replica decodes different tokens."""
    return rank * 1_000_000


def slowest_rank_ms(ms: float, dist, device) -> float:
    """The largest of the ranks' timed-region durations (the job is as slow as its slowest rank)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def step_percentiles(step_ms) -> dict:
    """p10 / p50 / p90 of the per-step device times (ms), nearest-rank."""
    v = sorted(float(t) for t in step_ms)
    if not v:
        return {}
    pick = lambda q: v[min(len(v) - 1, max(0, int(round(q * (len(v) - 1)))))]  # noqa: E731
    return {"p10": pick(0.10), "p50": pick(0.50), "p90": pick(0.90)}


def job_tokens_per_s(world: int, steps: int, T: int, max_ms: float) -> float:
    """Whole-job throughput: the tokens every rank processed over the slowest rank's time."""
    return world * steps * T / (max_ms / 1e3)


# ------------------------------------------------------------------------------------------
# clocks during the timed region
# ------------------------------------------------------------------------------------------

class Clocks:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 8:
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for n, v in zip(names, r[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        load = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------------------------------------
# oracle CPU baseline (host cores): the plain fp64 oracle as it stands
# ------------------------------------------------------------------------------------------

def oracle_sample_layer(cfg, seed, x_bits):
    """Oracle layer holding the experts that the sample's tokens route to (host-drawn)."""
    import oracle
    G, TG, p = ROUTER_VARIANTS.get(cfg.name, (1, 1, 0.0))
    variants = {"n_group": G, "topk_group": TG, "top_p": p}
    router = oracle.Layer(cfg.d, cfg.f, cfg.E, cfg.k, cfg.router, cfg.scaling, cfg.wkind,
                          syn.gen_router_w(cfg, seed), syn.gen_router_bias(cfg, seed), f_shared=cfg.f_shared or cfg.f,
                          **variants)
    need = sorted(e for e in set(router.route(x_bits)["idx"].reshape(-1).tolist()) if e >= 0)

    def host_expert(e):
        out = {}
        for which in ("gate_up", "down"):
            w = syn.gen_expert_fp32(cfg, e, which, seed)
            if cfg.wkind == syn.W_BF16:
                out[which] = syn.fp32_to_bf16_bits(w)
            elif cfg.wkind == syn.W_INT8:
                out[which], out[which + "_scale"] = oracle.quantize_tier(w, 8)
            elif cfg.wkind == syn.W_INT2:
                out[which], out[which + "_scale"] = oracle.pack_int2(w)
            else:
                out[which], out[which + "_scale"] = oracle.pack_int4(w)
        return out

    experts = {e: host_expert(e) for e in need}
    shared = host_expert("shared") if cfg.n_shared else None
    return oracle.Layer(cfg.d, cfg.f, cfg.E, cfg.k, cfg.router, cfg.scaling, cfg.wkind, router.router_w,
                        router.router_bias, experts=experts, shared=shared, f_shared=cfg.f_shared or cfg.f, **variants)


def oracle_sample_tokens(cfg, name):
    """Tokens of one oracle sample call: a single token for decode, a slice for the larger batches."""
    return {"glm_union2": 2, "glm_union32": 2, "glm_prefill": 2}.get(name, cfg.T)


def time_oracle(cfg, name, seed, budget_s, min_calls=1, max_calls=None, threads=None, layer=None):
    """The oracle's tokens/s on a bounded sample of the workload: calls of oracle_sample_tokens
    tokens until budget_s has passed.  threads: OpenMP threads for this timing only (default:
    all host cores).  layer: a (layer, x) pair from an earlier call, to skip building it again."""
    import oracle
    n_tok = oracle_sample_tokens(cfg, name)
    if layer is None:
        x = syn.gen_x(cfg, seed, T=n_tok)
        layer = (oracle_sample_layer(cfg, seed, x), x)
    L, x = layer
    all_cores = oracle.num_threads()
    if threads:
        oracle.set_num_threads(threads)
    try:
        cores = oracle.num_threads()
        calls, t0 = 0, time.perf_counter()
        while True:
            L.forward(x)
            calls += 1
            el = time.perf_counter() - t0
            if calls >= min_calls and (el >= budget_s or (max_calls and calls >= max_calls)):
                break
    finally:
        if threads:
            oracle.set_num_threads(all_cores)
    where = "host cores" if cores > 1 else "one host core"
    return {"value": calls * n_tok / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{calls} oracle calls of {n_tok} token(s) of the {name} workload ({el:.1f} s on {where})",
            "layer": layer}


def cpu_baseline(cfg, name, seed, budget_s):
    """The oracle on all host cores, plus the same sample on one core (a quarter of the budget)."""
    res = time_oracle(cfg, name, seed, budget_s)
    one = time_oracle(cfg, name, seed, budget_s / 4, threads=1, layer=res.pop("layer"))
    one.pop("layer")
    res["single_core"] = {k: one[k] for k in ("value", "unit", "cores", "sample")}
    return res


# ------------------------------------------------------------------------------------------
# roofline helpers
# ------------------------------------------------------------------------------------------

def kernel_work(cfg, T, n_unique):
    """Algorithmic work per launch of the expert kernels for a batch with n_unique routed experts:
    {kernel: ("hbm", bytes) | ("tensor", flops)}.  Bytes count the weight rows and scales read
    once, the activations read and the intermediate written; flops count 2 per multiply-add of
    the expert FFN (padding columns of a GEMM tile are not counted)."""
    S = 1 if cfg.n_shared else 0
    slots = T * cfg.k + T * S
    fmax = max(cfg.f, cfg.f_shared if S else 0)
    gu_rows = n_unique * 2 * cfg.f + S * 2 * cfg.f_shared
    gu = gu_rows * row_bytes(cfg, cfg.d) + T * cfg.d * 2 + slots * fmax * 2
    f_of = lambda ff: row_bytes(cfg, ff)  # noqa: E731
    dn_w = n_unique * cfg.d * f_of(cfg.f) + S * cfg.d * f_of(cfg.f_shared) + slots * fmax * 2
    # the single-token kernel adds the slots itself and writes the output; the others write y per slot
    dn = dn_w + (T * cfg.d * 4 if T == 1 else slots * cfg.d * 4)
    mac = T * cfg.k * cfg.d * cfg.f + T * S * cfg.d * cfg.f_shared
    # the single launch (T = 1 or 2): router matrix and bias, then gu (x, gate/up rows, h written)
    # and dn_w (down rows, h read back), and the output
    fused = cfg.E * cfg.d * 4 + cfg.E * 4 + gu + dn_w + T * cfg.d * 4
    # router kernels: the fp32 router matrix and x read, fp64 logits written
    router = cfg.E * cfg.d * 4 + T * cfg.d * 2 + T * cfg.E * 8
    return {"gateup": ("hbm", gu), "down": ("hbm", dn), "gemm_gateup": ("tensor", 4 * mac),
            "gemm_down": ("tensor", 2 * mac), "fused": ("hbm", fused), "router_logits": ("hbm", router)}


def source_sha(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel, workload):
    """dram bytes per launch of `kernel` in `workload` from a committed ncu capture, if the
    kernel's sources are unchanged since (entries are keyed "workload:kernel")."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(f"{workload}:{kernel}")
    if not rec:
        return None
    try:
        if source_sha(rec["sources"]) != rec["source_sha"]:
            return None
    except OSError:
        return None
    return rec.get("bytes_per_launch")


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return p.get("hbm_gbs", 6650.0), p.get("bf16_tflops", 1590.0), "measured"
    return 6650.0, 1590.0, "fallback"


# ------------------------------------------------------------------------------------------
# arms
# ------------------------------------------------------------------------------------------

def run_reference(a, rank, world):
    """The oracle on host cores: each step one bounded oracle call of the workload."""
    if rank != 0:
        return
    cfg = workload_config(a.workload)
    import oracle
    n_tok = oracle_sample_tokens(cfg, a.workload)
    x = syn.gen_x(cfg, a.seed, T=n_tok)
    L = oracle_sample_layer(cfg, a.seed, x)
    for _ in range(a.warmup):
        L.forward(x)
    t0 = time.perf_counter()
    for _ in range(a.steps):
        L.forward(x)
    el = time.perf_counter() - t0
    value = a.steps * n_tok / el
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference", "n_gpus": a.gpus,
            "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * el / a.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": a.workload, "desc": WORKLOADS[a.workload], "tokens_per_step": n_tok,
                       "parallelism": "host cores"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"{a.steps} timed oracle calls of {n_tok} token(s) of {a.workload}"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def measure_workload(a, name, cfg, layer, dev, dist, world, rank, local_rank, flush, cpu_budget):
    """Times one workload on an existing layer; returns its part of the JSON line."""
    import torch

    import quantized_expert_ffn_02_b200 as qe

    T = cfg.T
    if a.t1_mode is not None:
        layer.set_single_token_mode(a.t1_mode)
    if name in ROUTER_VARIANTS:
        G, TG, p = ROUTER_VARIANTS[name]
        layer.set_router_groups(G, TG)
        layer.set_router_top_p(p)
    # every rank is an independent replica with its own tokens
    n_batches = a.warmup + a.steps if T <= 32 else 4
    token_base = replica_token_base(rank)
    xs = make_batches(cfg, T, n_batches, a.seed, token_base, dev)
    out = torch.empty((T, cfg.d), dtype=torch.int16 if cfg.out_bf16 else torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    # census of unique experts per batch (outside timing) for the algorithmic byte counts
    uniq = []
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
    wts = torch.empty((T, cfg.k), dtype=torch.float32, device=dev)
    for x in xs:
        layer.route(x, idx, wts)
        uniq.append(len([e for e in torch.unique(idx).tolist() if e >= 0]))     # -1: dropped by top-p
    torch.cuda.synchronize()

    def bx(i):
        return xs[i % len(xs)]

    for i in range(a.warmup):
        layer.forward(bx(i), out)
    torch.cuda.synchronize()
    if layer.last_error() != qe.MOE_OK:
        raise RuntimeError(f"{name}: device status after warm-up: " + qe.status_str(layer.last_error()))
    launches_per_step = layer.last_launches()

    def timed_pass(profile: bool):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(a.steps)]
        layer.profile(profile)
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(a.steps):
            flush()
            evs[i][0].record(stream)
            layer.forward(bx(a.warmup + i), out)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        layer.profile(False)
        return [s.elapsed_time(e) for s, e in evs]

    clocks = Clocks(local_rank)
    clocks.start()
    step_ms = timed_pass(False)
    clk = clocks.stop()
    total_ms = sum(step_ms)
    prof_ms = sum(timed_pass(True))
    prof = layer.profile_read()
    if layer.last_error() != qe.MOE_OK:
        raise RuntimeError(f"{name}: device status after timing: " + qe.status_str(layer.last_error()))
    total_ms = slowest_rank_ms(total_ms, dist, dev)
    value = job_tokens_per_s(world, a.steps, T, total_ms)

    # end to end: host buffers through the C ABI, copies inside the timed region.  Every step
    # copies its x in from pinned host memory and its output back out.  The calls are enqueued
    # back to back (moe_forward_host_async) and the host waits once at the end, as a serving loop
    # would; L2 is not flushed between these steps.  The form that waits after every step
    # (moe_forward_host) is timed beside it.
    xh = [bx(a.warmup + i).cpu().pin_memory() for i in range(min(a.steps, len(xs)))]
    oh = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    e2e_steps = a.steps

    def e2e_pass(pipelined: bool):
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(e2e_steps):
            if pipelined:
                layer.forward_host_async(xh[i % len(xh)], oh[i % 2])
            else:
                layer.forward_host(xh[i % len(xh)], oh[i % 2])
        t1.record(stream)
        torch.cuda.synchronize()
        if layer.last_error() != qe.MOE_OK:
            raise RuntimeError(f"{name}: device status after the end-to-end pass: " +
                               qe.status_str(layer.last_error()))
        return slowest_rank_ms(t0.elapsed_time(t1), dist, dev)

    sync_ms = e2e_pass(False)
    try:
        e2e_ms, e2e_api = e2e_pass(True), "moe_forward_host_async, one wait at the end"
    except AttributeError as exc:      # an older library without the call
        e2e_ms, e2e_api = sync_ms, "moe_forward_host (no pipelined call: %s)" % str(exc).splitlines()[0][:120]
    e2e = {"value": job_tokens_per_s(world, e2e_steps, T, e2e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": T * cfg.d * 2, "d2h_bytes_per_step": T * cfg.d * out.element_size(),
           "api": e2e_api, "l2": "not flushed between steps (back-to-back serving loop)",
           "wait_every_step": {"value": job_tokens_per_s(world, e2e_steps, T, sync_ms), "unit": "tokens/s",
                               "api": "moe_forward_host"}}

    # L2-warm passes: the same steps back to back with no flush in between
    def warm_pass(graph: bool):
        g = None
        if graph:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):          # the binding launches on the capturing stream
                for i in range(a.steps):
                    layer.forward(bx(a.warmup + i), out)
            torch.cuda.synchronize()
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        if g is not None:
            g.replay()
        else:
            for i in range(a.steps):
                layer.forward(bx(a.warmup + i), out)
        t1.record(stream)
        torch.cuda.synchronize()
        ms = slowest_rank_ms(t0.elapsed_time(t1), dist, dev)
        if g is not None:
            g.reset()
        if layer.last_error() != qe.MOE_OK:
            raise RuntimeError(f"{name}: device status after an L2-warm pass: " + qe.status_str(layer.last_error()))
        return {"value": job_tokens_per_s(world, a.steps, T, ms), "unit": "tokens/s", "ms_per_step": ms / a.steps,
                "steps": a.steps, "launch": "one CUDA graph" if graph else "stream launches",
                "l2": "warm: no flush between steps, not an HBM figure"}

    warm_mode = a.warm_passes if a.warm_passes is not None else DEFAULT_WARM_PASSES.get(name, "none")
    warm = {}
    if warm_mode in ("stream", "both"):
        warm["stream"] = warm_pass(False)
    if warm_mode in ("graph", "both"):
        try:
            warm["graph"] = warm_pass(True)
        except RuntimeError as exc:                # a capture the runtime refused: report it
            torch.cuda.synchronize()
            warm["graph"] = {"error": str(exc).splitlines()[0][:200]}

    # roofline of the dominant kernel (device time measured by the library's event pairs)
    hbm, tf, peak_kind = measured_peaks()
    dom = max(prof, key=lambda k: prof[k][0]) if prof else None
    roof = None
    if dom:
        ms, n = prof[dom]
        per_launch_ms = ms / n
        timed_uniq = [uniq[(a.warmup + i) % len(xs)] for i in range(a.steps)]
        works = [kernel_work(cfg, T, u).get(dom) for u in timed_uniq]
        if works[0] is not None:
            kind = works[0][0]
            amount = statistics.mean(w[1] for w in works)
            if kind == "hbm":
                achieved = amount / (per_launch_ms / 1e3) / 1e9
                roof = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                        "frac": achieved / hbm, "traffic": traffic_for(dom, name),
                        "peak_kind": f"{peak_kind} copy bandwidth",
                        "algorithmic_bytes_per_launch": amount, "ms_per_launch": per_launch_ms}
            else:
                achieved = amount / (per_launch_ms / 1e3) / 1e12
                roof = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": tf, "unit": "TFLOP/s",
                        "frac": achieved / tf, "traffic": traffic_for(dom, name),
                        "peak_kind": f"{peak_kind} bf16 dense (burst)",
                        "algorithmic_flops_per_launch": amount, "ms_per_launch": per_launch_ms}
    step_bytes = statistics.mean(uniq[(a.warmup + i) % len(xs)] for i in range(a.steps)) * expert_bytes(cfg) + \
        (expert_bytes(cfg, cfg.f_shared) if cfg.n_shared else 0) + cfg.E * cfg.d * 4
    ms_per_step = total_ms / a.steps
    res = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": a.steps, "warmup": a.warmup,
        "ms_per_step": ms_per_step, "step_ms_percentiles": step_percentiles(step_ms), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": {syn.W_INT4: "int4xbf16->f32", syn.W_INT8: "int8xbf16->f32", syn.W_INT2: "int2xbf16->f32"}.get(
            cfg.wkind, "bf16->f32"), "data": "synthetic",
        "config": {"workload": name, "desc": WORKLOADS[name], "tokens_per_step": T,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "evicted between steps by a read-only sweep of a 512 MiB buffer, outside the step events",
                   "weights": "seed 0, drawn on the device by the counter-based generator"},
        "roofline": roof,
        "step_hbm": {"gbs": step_bytes / (ms_per_step / 1e3) / 1e9, "frac": step_bytes / (ms_per_step / 1e3) / 1e9 / hbm,
                     "bytes_per_step": step_bytes, "unique_experts_mean": statistics.mean(uniq)},
        "kernels": {k: {"ms_per_launch": v[0] / v[1], "launches": v[1]} for k, v in prof.items()},
        "profiled_ms_per_step": prof_ms / a.steps,
        "e2e": e2e,
        "gpu_launches": launches_per_step * a.steps,
        "clocks": clk,
    }
    if cfg.wkind == syn.W_INT4 and T >= 128 and "gemm_gateup" in prof:
        flops = 2 * T * (cfg.k * 3 * cfg.d * cfg.f + (3 * cfg.d * cfg.f_shared if cfg.n_shared else 0))
        res["step_tensor"] = {"tflops": flops / (ms_per_step / 1e3) / 1e12,
                              "frac": flops / (ms_per_step / 1e3) / 1e12 / tf, "flops_per_step": flops,
                              "peak": tf, "peak_kind": f"{peak_kind} bf16 dense (burst)"}
    if warm:
        res["l2_warm"] = warm
    if hasattr(layer, "stats"):
        st = layer.stats()
        calls = st["hits"] + st["misses"]
        res["expert_tier"] = {"slots": TIER_SLOTS, "hit_rate": st["hits"] / calls if calls else None,
                              "h2d_gb_streamed": st["bytes_in"] / 1e9, "note": "counts cover every pass of this row "
                              "(census, warm-up, timed, profiled, end-to-end)"}
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(cfg, name, a.seed, cpu_budget)
    return res


def selected_workloads(a):
    if a.workloads == "none":
        extra = []
    elif a.workloads == "all":
        extra = [n for n in WORKLOAD_ORDER if n != a.workload]
    else:
        extra = [n.strip() for n in a.workloads.split(",") if n.strip() and n.strip() != a.workload]
        for n in extra:
            if n not in WORKLOADS:
                raise SystemExit(f"unknown workload {n}")
    return [a.workload] + extra


def run_ours(a, rank, world, local_rank):
    import torch

    import dataclasses

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    flush_buf = torch.zeros(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush():
        flush_buf.sum()          # reads 512 MiB: every line of L2 is replaced by a clean one

    names = selected_workloads(a)
    # workloads over the same weights (the four int4 GLM workloads) share one resident copy of the
    # experts (4.8 GB); each gets a layer handle with its own token limit and output type
    def weight_key(n):
        c = workload_config(n)
        return (c.d, c.E, c.f, c.wkind, c.router)
    results = {}
    first_sharer = {n: next(m for m in WORKLOAD_ORDER if weight_key(m) == weight_key(n)) for n in names}
    order = sorted(names, key=lambda n: (WORKLOAD_ORDER.index(first_sharer[n]), WORKLOAD_ORDER.index(n)))
    held = (None, None)
    for i, name in enumerate(order):
        layer = None
        cfg = workload_config(name)
        if a.experts:
            cfg = dataclasses.replace(cfg, E=a.experts)
        if a.tokens and name == a.workload:
            cfg = dataclasses.replace(cfg, T=a.tokens)
        if held[0] != weight_key(name):
            held = (None, None)
            torch.cuda.empty_cache()
            layer, W = build_device_layer(cfg, a.seed, cfg.T, dev)
            held = (weight_key(name), W)
            if name == "glm_decode_tiered":
                layer.close()
        if name == "glm_decode_tiered":
            layer = TieredLayer(cfg, held[1], cfg.T, TIER_SLOTS)
        elif layer is None or getattr(layer, "handle", None) is None:
            layer = layer_on(cfg, held[1], cfg.T)
        budget = a.cpu_seconds if name == a.workload else a.cpu_seconds / 3
        aw = a if a.steps_given is not None else argparse.Namespace(**{**vars(a), "steps": DEFAULT_STEPS[name]})
        results[name] = measure_workload(aw, name, cfg, layer, dev, dist, world, rank, local_rank, flush, budget)
        layer.close()
    held = (None, None)
    line = results.pop(a.workload)
    if results:
        line["workloads"] = results
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


def main():
    a = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if a.impl == "reference":
        run_reference(a, rank, world)
    else:
        run_ours(a, rank, world, local_rank)


if __name__ == "__main__":
    main()
