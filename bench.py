#!/usr/bin/env python
"""Decode-step benchmark of the latent-KV path on B200.

One step = the whole hot path for one batch: append each sequence's new token
to the latent cache (palu_compress_append: z = x·A, scattered into its page)
and run one decode step of attention over every cached token
(palu_decode_attn: split kernel + log-sum-exp combine).  The context grows by
one token per step.

Metric: decode-attention tokens·heads per second = Σ_b T_b · H / t_step,
whole job over all ranks (weak scaling: every rank runs its own batch of
sequences; the step has no cross-GPU data exchange).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Rank 0 prints one JSON line.
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
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "7b_bf16_r256v128_b16_t16k"
METRIC = "decode attn tokens·heads/s"
UNIT = "tokens·heads/s"


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--num-splits", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU oracle sample budget")
    ap.add_argument("--queries", type=int, default=1,
                    help="query tokens per sequence per step (multi-token decode: appended together, "
                         "each attends causally; palu_decode_attn_multi)")
    ap.add_argument("--prefill", type=int, default=None,
                    help="also time palu_compress_append of this many prompt tokens (default: 8192 for "
                         "the batch-32 prefill + decode workload, else off)")
    return ap.parse_args()


# ----------------------------------------------------------------- peaks and counters
def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# The sources the decode kernels are built from (their own files and the headers of
# the package they include; from include/palu.h they take only the ABI-fixed dtype
# and status codes); a committed traffic figure is used only while these are unchanged.
DECODE_SOURCES = ["decode_tc.cu", "decode_fused.cu", "decode_simt.cu", "palu_common.cuh", "palu_internal.h",
                  "palu_tc.h", "tc_ptx.cuh"]


def csrc_hash() -> str:
    h = hashlib.sha256()
    paths = [os.path.join(ROOT, "rank_kv_cache_palu_b200", "csrc", n) for n in DECODE_SOURCES]
    for p in paths:
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if its source hash is current."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("csrc_hash") != csrc_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------- clocks (NVML, read-only)
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


class ClockSampler:
    """Samples SM clock and clock-event reasons of one GPU from a background thread."""

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            handle = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                hd = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hd)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    handle = hd
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nvml, self.h = pynvml, handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: no clock record
            self.err = repr(e)

    def _run(self):
        nv = self.nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self) -> dict:
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": getattr(self, "max_mhz", None), "reasons": [],
                    "samples": 0}
        busy = [s for s in self.samples if not (s[1] & 0x1)] or self.samples
        reasons = set()
        for _, rs in busy:
            for bit, name in REASONS.items():
                if rs & bit and bit != 0x1:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in busy), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(busy)}


# ----------------------------------------------------------------- work accounting
def step_work(w, seq_lens):
    """Algorithmic bytes and flops of one decode call (latents + B + q/out), per the layout.

    Sums over the head groups, each with its own (r_k, r_v) (all equal unless the
    workload carries a rank-search output)."""
    elt = {"f32": 4, "f16": 2, "bf16": 2}[w.act_dtype]
    W, gs, d_h = w.width, w.group_size, w.head_dim
    tok = sum(seq_lens)
    nb = len(seq_lens)
    bytes_ = nb * w.num_heads * d_h * elt * 2
    flops = 0
    for rk, rv in zip(*w.group_ranks):
        if w.latent_dtype == "int4":
            row = rk // 2 + rv // 2 + 2 * (rk // 32 + rv // 32)
        else:
            row = (rk + rv) * {"f32": 4, "f16": 2, "bf16": 2}[w.latent_dtype]
        bytes_ += tok * row + (rk + rv) * W * elt
        if w.rope_base == 0:
            # fused path: scores in latent space (q̃ = B_k q per head, r_k long)
            flops += tok * (2 * gs * rk + 2 * gs * rv) + nb * gs * 2 * (rk + rv) * d_h
        else:
            flops += tok * (2 * rk * W + 2 * gs * rv) + nb * gs * 2 * rv * d_h
    return bytes_, flops


# ----------------------------------------------------------------- CPU oracle timing
def oracle_sample(w, seconds: float, seed: int = 99):
    """Time the oracle's decode on (sequence, head) units at the workload's context.

    Returns (tokens·heads per second, description, threads used).
    """
    import numpy as np

    from oracle import palu_oracle as O
    from rank_kv_cache_palu_b200.synth import normal
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = os.cpu_count() or 1
    T, G, W = w.context, w.groups, w.width
    q = normal(seed, "cpu_q", (w.num_heads, w.head_dim)).astype(np.float64)
    pos = np.arange(T)
    heads = 0
    t0 = time.perf_counter()
    if not w.ranked:
        rk, rv = w.rank_k, w.rank_v
        zk = normal(seed, "cpu_zk", (G, T, rk)).astype(np.float64)
        zv = normal(seed, "cpu_zv", (G, T, rv)).astype(np.float64)
        Bk = normal(seed, "cpu_Bk", (G, rk, W), 1 / math.sqrt(rk)).astype(np.float64)
        Bv = normal(seed, "cpu_Bv", (G, rv, W), 1 / math.sqrt(rv)).astype(np.float64)
        t0 = time.perf_counter()
        while True:
            h = heads % w.num_heads
            O.decode_attention_head(h, q, T - 1, zk, zv, pos, Bk, Bv, w.group_size, w.rope_base)
            heads += 1
            el = time.perf_counter() - t0
            if el >= seconds:
                break
        what = "decode_attention_head on %d (sequence, head) units" % heads
    else:
        # one group (its group_size heads) per call, each with its own ranks
        rks, rvs = w.group_ranks
        gs = w.group_size
        zk = [normal(seed, f"cpu_zk{g}", (T, r)).astype(np.float64) for g, r in enumerate(rks)]
        zv = [normal(seed, f"cpu_zv{g}", (T, r)).astype(np.float64) for g, r in enumerate(rvs)]
        Bk = [normal(seed, f"cpu_Bk{g}", (r, W), 1 / math.sqrt(r)).astype(np.float64) for g, r in enumerate(rks)]
        Bv = [normal(seed, f"cpu_Bv{g}", (r, W), 1 / math.sqrt(r)).astype(np.float64) for g, r in enumerate(rvs)]
        t0 = time.perf_counter()
        while True:
            g = (heads // gs) % G
            O.decode_attention_ranked(q[g * gs:(g + 1) * gs][None], [T - 1], [zk[g]], [zv[g]], pos, [Bk[g]],
                                      [Bv[g]], gs, w.rope_base)
            heads += gs
            el = time.perf_counter() - t0
            if el >= seconds:
                break
        what = "decode_attention_ranked, one group per call, on %d (sequence, head) units" % heads
    desc = f"oracle {what} of one sequence at context {T} ({el:.1f} s of CPU work)"
    return heads * T / el, desc, threads, heads * T


# ----------------------------------------------------------------- reference arm
def run_reference(args):
    from rank_kv_cache_palu_b200.dist import env_world
    from rank_kv_cache_palu_b200.synth import WORKLOADS
    rank, world, _ = env_world()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    per = max(1.0, min(args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, per / 4)
    vals, units, descs = [], 0, ""
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, descs, threads, u = oracle_sample(w, per)
        vals.append(v)
        units += u
    el = time.perf_counter() - t0
    value = units / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "context": w.context,
                   "parallelism": "oracle on rank 0 only"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": "each step: " + descs},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- our arm
def run_ours(args):
    import numpy as np
    import torch

    from rank_kv_cache_palu_b200 import api as P
    from rank_kv_cache_palu_b200 import dist as D
    from rank_kv_cache_palu_b200.synth import TORCH_DTYPE, WORKLOADS, page_permutation

    rank, world, local = D.init("nccl")
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs CUDA devices")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    cfg = P.make_config(w.num_heads, w.head_dim, w.group_size, w.rank_k, w.rank_v, w.page_size,
                        w.rope_base, w.act_dtype, w.latent_dtype)
    b, T0, G, W = w.batch, w.context, w.groups, w.width
    Pz = w.page_size
    Q = args.queries
    steps_total = 2 * (args.warmup + args.steps) + 2
    max_tokens = T0 + steps_total * Q
    max_pages = (max_tokens + Pz - 1) // Pz
    num_pages = b * max_pages
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + rank)
    act = TORCH_DTYPE[w.act_dtype]

    # ---- the latent cache, filled with N(0,1) latents (the distribution of x·A)
    rks, rvs = w.group_ranks
    rk_arg, rv_arg = (rks, rvs) if w.ranked else (None, None)
    cache = P.LatentCache.allocate(cfg, num_pages, device=dev, ranks_k=rk_arg, ranks_v=rv_arg)
    for pool in (cache.zk, cache.zv):
        if w.latent_dtype == "int4":
            pool.copy_(torch.randint(0, 256, pool.shape, dtype=torch.uint8, device=dev, generator=gen))
        else:
            view = pool.view(TORCH_DTYPE[w.latent_dtype])
            chunk = 1 << 28
            for i in range(0, view.numel(), chunk):
                seg = view[i:i + chunk]
                seg.copy_(torch.randn(seg.shape, device=dev, generator=gen, dtype=torch.float32))
    for sp in (cache.zks, cache.zvs):
        if sp is not None:
            sp.view(torch.float16).fill_(0.3)
    perm = torch.from_numpy(page_permutation(7 + rank, num_pages)).to(dev)
    page_table = perm.view(b, max_pages).contiguous()
    pt_host = page_table.cpu().numpy()

    d_model = w.d_model
    # A_k [d_model][Σ r_k], B_k [Σ r_k][W]: group g's columns / rows follow the groups before it
    A_k = (torch.randn((d_model, sum(rks)), device=dev, generator=gen) / math.sqrt(d_model)).to(act)
    A_v = (torch.randn((d_model, sum(rvs)), device=dev, generator=gen) / math.sqrt(d_model)).to(act)
    B_k = torch.cat([torch.randn((r, W), device=dev, generator=gen) / math.sqrt(r) for r in rks]).to(act)
    B_v = torch.cat([torch.randn((r, W), device=dev, generator=gen) / math.sqrt(r) for r in rvs]).to(act)
    ring = 4
    xs = [torch.randn((b * Q, d_model), device=dev, generator=gen).to(act) for _ in range(ring)]
    qshape = (b, w.num_heads, w.head_dim) if Q == 1 and not w.ranked else (b, Q, w.num_heads, w.head_dim)
    qs = [torch.randn(qshape, device=dev, generator=gen).to(act) for _ in range(ring)]

    # per-step metadata, all on the device before timing: the step appends Q
    # tokens per sequence at positions base .. base + Q - 1, then queries them
    def meta(step):
        base = T0 + step * Q
        slots = np.array([pt_host[i, (base + j) // Pz] * Pz + (base + j) % Pz for i in range(b) for j in range(Q)],
                         np.int32)
        qpos = np.array([[base + j for j in range(Q)] for _ in range(b)], np.int32)
        return (torch.from_numpy(slots).to(dev), torch.from_numpy(qpos.reshape(b) if Q == 1 else qpos).to(dev),
                torch.full((b,), base + Q, dtype=torch.int32, device=dev))
    metas = [meta(s) for s in range(steps_total)]

    def step_units(s):
        base = T0 + s * Q
        return b * w.num_heads * sum(base + j + 1 for j in range(Q))

    if w.ranked:
        # one split count per rank class, chosen by the library (0 = automatic)
        S = args.num_splits
        ws_d = torch.zeros(P.palu_decode_ranked_workspace_size(cfg, rks, rvs, b, Q, max_pages, S),
                           dtype=torch.uint8, device=dev)
        ws_c = torch.zeros(P.palu_compress_ranked_workspace_size(cfg, rks, rvs, b * Q, d_model),
                           dtype=torch.uint8, device=dev)
    else:
        S = args.num_splits or P.palu_decode_num_splits(cfg, b, max_pages)
        ws_d = torch.zeros(P.palu_decode_multi_workspace_size(cfg, b, Q, max_pages, S), dtype=torch.uint8,
                           device=dev)
        ws_c = torch.zeros(P.palu_compress_workspace_size(cfg, b * Q, d_model), dtype=torch.uint8, device=dev)
    out = torch.empty(qshape, dtype=act, device=dev)
    stream = torch.cuda.current_stream(dev)

    def decode(q, qpos, lens):
        if w.ranked:
            P.palu_decode_attn_ranked(cfg, rks, rvs, q, qpos, cache.zk, cache.zv, cache.zks, cache.zvs, None,
                                      page_table, lens, num_pages, B_k, B_v, out, None, ws_d, S, stream)
            return
        fn = P.palu_decode_attn if Q == 1 else P.palu_decode_attn_multi
        fn(cfg, q, qpos, cache.zk, cache.zv, cache.zks, cache.zvs, None, page_table, lens, num_pages, B_k, B_v,
           out, None, ws_d, S, stream)

    def compress(x, slots):
        if w.ranked:
            P.palu_compress_append_ranked(cfg, rks, rvs, x, A_k, A_v, slots, None, cache.zk, cache.zv, cache.zks,
                                          cache.zvs, None, num_pages, ws_c, stream)
        else:
            P.palu_compress_append(cfg, x, A_k, A_v, slots, None, cache.zk, cache.zv, cache.zks, cache.zvs, None,
                                   num_pages, ws_c, stream)

    def step(s, x=None, q=None):
        slots, qpos, lens = metas[s]
        compress(xs[s % ring] if x is None else x, slots)
        decode(qs[s % ring] if q is None else q, qpos, lens)

    # ---- device-resident timing
    s_idx = 0
    for _ in range(args.warmup):
        step(s_idx)
        s_idx += 1
    torch.cuda.synchronize(dev)
    D.barrier(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = P.palu_kernel_launches()
    first_step = s_idx
    with ClockSampler(dev.index) as clk:
        torch.cuda.synchronize(dev)
        start.record(stream)
        for k in range(args.steps):
            slots, qpos, lens = metas[s_idx]
            ev[k][0].record(stream)
            compress(xs[s_idx % ring], slots)
            ev[k][1].record(stream)
            decode(qs[s_idx % ring], qpos, lens)
            ev[k][2].record(stream)
            s_idx += 1
        end.record(stream)
        torch.cuda.synchronize(dev)
    launches = P.palu_kernel_launches() - launches0
    D.barrier(dev)
    st_d, det_d = P.palu_get_device_status(ws_d)
    st_c, det_c = P.palu_get_device_status(ws_c)
    if st_d or st_c:
        raise RuntimeError(f"device status decode={st_d}({det_d}) compress={st_c}({det_c})")
    el_ms = D.max_over_ranks(start.elapsed_time(end), dev)
    dec_ms = [e[1].elapsed_time(e[2]) for e in ev]
    cmp_ms = [e[0].elapsed_time(e[1]) for e in ev]
    units = sum(step_units(s) for s in range(first_step, first_step + args.steps))
    value = D.sum_over_ranks(units, dev) / (el_ms / 1e3)

    # ---- end to end through the public API: pinned host inputs -> H2D -> step -> D2H
    xh = [t.cpu().pin_memory() for t in xs]
    qh = [t.cpu().pin_memory() for t in qs]
    meta_h = [tuple(m.cpu().pin_memory() for m in metas[s]) for s in range(steps_total)]
    outh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    x_d, q_d = torch.empty_like(xs[0]), torch.empty_like(qs[0])
    m_d = tuple(torch.empty_like(m) for m in metas[0])
    h2d = xs[0].numel() * xs[0].element_size() + qs[0].numel() * qs[0].element_size() + \
        sum(m.numel() * m.element_size() for m in metas[0])
    d2h = out.numel() * out.element_size()

    def e2e_step(s):
        x_d.copy_(xh[s % ring], non_blocking=True)
        q_d.copy_(qh[s % ring], non_blocking=True)
        for dst, src in zip(m_d, meta_h[s]):
            dst.copy_(src, non_blocking=True)
        compress(x_d, m_d[0])
        decode(q_d, m_d[1], m_d[2])
        outh.copy_(out, non_blocking=True)

    for _ in range(min(args.warmup, 3)):
        e2e_step(s_idx)
        s_idx += 1
    torch.cuda.synchronize(dev)
    D.barrier(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_units = 0
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step(s_idx)
        e2e_units += step_units(s_idx)
        s_idx += 1
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = D.max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_value = D.sum_over_ranks(e2e_units, dev) / (e2e_ms / 1e3)

    # ---- prefill: palu_compress_append of a prompt (x·A for n tokens into fresh pages)
    prefill = None
    n_pre = args.prefill if args.prefill is not None else (8192 if w.name == "7b_bf16_r256_b32_t16k" else 0)
    if n_pre > 0 and world >= 1 and not w.ranked:
        pre_pages = (n_pre + Pz - 1) // Pz
        pcache = P.LatentCache.allocate(cfg, pre_pages, device=dev)
        xp = torch.randn((n_pre, d_model), device=dev, generator=gen).to(act)
        pslots = torch.arange(n_pre, dtype=torch.int32, device=dev)
        ws_p = torch.zeros(P.palu_compress_workspace_size(cfg, n_pre, d_model), dtype=torch.uint8, device=dev)
        def pre():
            P.palu_compress_append(cfg, xp, A_k, A_v, pslots, None, pcache.zk, pcache.zv, pcache.zks,
                                   pcache.zvs, None, pre_pages, ws_p, stream)
        for _ in range(3):
            pre()
        torch.cuda.synchronize(dev)
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = 10
        p0.record(stream)
        for _ in range(reps):
            pre()
        p1.record(stream)
        torch.cuda.synchronize(dev)
        pre_ms = p0.elapsed_time(p1) / reps
        st_p, det_p = P.palu_get_device_status(ws_p)
        if st_p:
            raise RuntimeError(f"device status prefill={st_p}({det_p})")
        pre_flops = 2.0 * n_pre * d_model * G * (w.rank_k + w.rank_v)
        pk = measured_peaks()
        prefill = {"tokens": n_pre, "ms": pre_ms, "tflops": pre_flops / pre_ms / 1e9,
                   "frac_of_sustained_bf16": pre_flops / pre_ms / 1e9 / pk["bf16_tflops_sustained"],
                   "kernel": "compress_tc_kernel (x·[A_k | A_v], tcgen05) + page scatter",
                   "flops": pre_flops}
        del pcache, xp, ws_p

    # ---- roofline of the dominant kernel (the decode step: split + combine)
    peaks = measured_peaks()
    # the step's algorithmic work: the cache read once, every query's flops
    mean_T = T0 + (first_step + args.steps / 2) * Q + Q
    dbytes, dflops = step_work(w, [mean_T] * b)
    dflops *= Q
    dec_avg_s = statistics.mean(dec_ms) / 1e3
    gbs = dbytes / dec_avg_s / 1e9
    tfs = dflops / dec_avg_s / 1e12
    t_hbm = dbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = dflops / (peaks["bf16_tflops_sustained"] * 1e12)
    kinds = sorted({P.palu_decode_kernel_kind(P.make_config(w.num_heads, w.head_dim, w.group_size, rk, rv, Pz,
                                                             w.rope_base, w.act_dtype, w.latent_dtype))
                    for rk, rv in zip(rks, rvs)})
    kind = kinds[0] if len(kinds) == 1 else kinds
    if t_tc > t_hbm:
        roof = {"bound": "tensor", "achieved": tfs, "peak": peaks["bf16_tflops_sustained"],
                "unit": "TFLOP/s", "frac": tfs / peaks["bf16_tflops_sustained"]}
    else:
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"]}
    roof["traffic"] = profiled_traffic(w.name, "decode")
    roof["peak_source"] = peaks["source"] + (" sustained" if roof["bound"] == "tensor" else " copy")
    roof["hbm_achieved_gbs"] = gbs
    roof["hbm_frac"] = gbs / peaks["hbm_gbs"]
    roof["tensor_achieved_tflops"] = tfs
    roof["algorithmic_bytes_per_launch"] = dbytes
    roof["algorithmic_flops_per_launch"] = dflops
    roof["kernel"] = "palu_decode_attn (%s), kernel kind %s%s" % (
        "fold-query + fused split + combine" if kind == 3 else "split + combine", kind,
        ", one launch set per rank class (%d classes)" % len(set(zip(rks, rvs))) if w.ranked else "")
    roof["avg_launch_ms"] = dec_avg_s * 1e3

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": el_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.act_dtype if w.latent_dtype != "int4" else "f16/int4",
        "data": "synthetic",
        "config": {"workload": w.name, "batch_per_gpu": b, "global_batch": b * world,
                   "context_at_first_timed_step": T0 + first_step + 1, "heads": w.num_heads,
                   "head_dim": w.head_dim, "group_size": w.group_size, "rank_k": w.rank_k,
                   "rank_v": w.rank_v, "latent_dtype": w.latent_dtype, "page_size": Pz,
                   "num_splits": S if S else "automatic per rank class", "decode_kernel_kind": kind,
                   "queries_per_step": Q,
                   **({"ranks_k": list(rks), "ranks_v": list(rvs)} if w.ranked else {}),
                   "l2": "inputs larger than L2 (latent cache %.2f GB vs 126 MB L2)" %
                         ((cache.zk.numel() + cache.zv.numel()) / 1e9),
                   "parallelism": f"dp{world} replicas (independent sequences per GPU)"},
        "roofline": roof,
        "decode_ms_mean": statistics.mean(dec_ms), "compress_append_ms_mean": statistics.mean(cmp_ms),
        "clocks": clk.summary(),
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        **({"prefill": prefill} if prefill else {}),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, threads, _ = oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    D.finalize()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
