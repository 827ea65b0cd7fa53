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

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--no-sweep]
  python bench.py --impl reference ...   # the CPU oracle on a bounded sample

Besides the headline workload, the line carries a "sweep": every workload the
metric is quoted on (the fp16 4k point, the bf16 context sweep 4k/16k/64k x
batch 1/8/16, int4 latents at 32k x 8, and an 8192-token prefill followed by 32
decode steps at batch 32), each timed in the same run with CUDA events and
given its own roofline.

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
    ap.add_argument("--cpu-workers", type=int, default=16, help="oracle worker processes (at most the host's cores)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the timing of every other workload of the metric (the 'sweep' key)")
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
DECODE_SOURCES = ["decode_tc.cu", "decode_tc_int4.cu", "decode_tc_kernel.cuh", "decode_fused.cu", "decode_simt.cu", "palu_common.cuh", "palu_internal.h",
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
# The oracle as it stands, timed over (sequence, group) units in worker processes.
# The workers are spawned (none inherits a CUDA context) with one BLAS thread each,
# and hold the unit's synthetic inputs from their start, so the timed tasks run
# nothing but the oracle.
_BLAS_VARS = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
_UNIT = {}


def _oracle_worker_init(wname: str, T: int, seed: int, root: str) -> None:
    sys.path.insert(0, root)
    import numpy as np

    from rank_kv_cache_palu_b200.synth import WORKLOADS, normal
    w = WORKLOADS[wname]
    gs, W, d_h = w.group_size, w.width, w.head_dim
    rks, rvs = w.group_ranks
    groups = []
    # uniform ranks: one (sequence, group) template serves every unit; per-group ranks:
    # one template per group
    for g in (range(w.groups) if w.ranked else [0]):
        rk, rv = rks[g], rvs[g]
        q = normal(seed, f"cpu_q{g}", (gs, d_h)).astype(np.float64)
        Bk = normal(seed, f"cpu_Bk{g}", (rk, W), 1 / math.sqrt(rk)).astype(np.float64)
        Bv = normal(seed, f"cpu_Bv{g}", (rv, W), 1 / math.sqrt(rv)).astype(np.float64)
        if w.latent_dtype == "int4":
            rng = np.random.default_rng([seed, g])
            zk = (rng.integers(0, 256, (T, rk // 2), dtype=np.uint8),
                  rng.uniform(0.05, 0.5, (T, rk // 32)).astype(np.float16))
            zv = (rng.integers(0, 256, (T, rv // 2), dtype=np.uint8),
                  rng.uniform(0.05, 0.5, (T, rv // 32)).astype(np.float16))
        else:
            zk = normal(seed, f"cpu_zk{g}", (T, rk)).astype(np.float64)
            zv = normal(seed, f"cpu_zv{g}", (T, rv)).astype(np.float64)
        groups.append((q, zk, zv, Bk, Bv))
    _UNIT.update(w=w, T=T, groups=groups, pos=np.arange(T))


def _oracle_task(i: int) -> int:
    """One (sequence, group) unit: the group's heads over T tokens; returns tokens·heads."""
    from oracle import palu_oracle as O
    w, T, pos = _UNIT["w"], _UNIT["T"], _UNIT["pos"]
    q, zk, zv, Bk, Bv = _UNIT["groups"][i % len(_UNIT["groups"])]
    if w.latent_dtype == "int4":   # dequantisation is part of the oracle's decode step
        zk = O.dequantize_int4(zk[0], zk[1], w.act_dtype)
        zv = O.dequantize_int4(zv[0], zv[1], w.act_dtype)
    O.decode_attention_ranked(q[None], [T - 1], [zk], [zv], pos, [Bk], [Bv], w.group_size, w.rope_base)
    return w.group_size * T


class OraclePool:
    """Worker processes running the oracle on (sequence, group) units of one workload."""

    def __init__(self, w, workers: int, seed: int = 99):
        import multiprocessing as mp
        try:
            avail = len(os.sched_getaffinity(0))
        except AttributeError:
            avail = os.cpu_count() or 1
        self.n = max(1, min(workers, avail))
        self.w = w
        old = {k: os.environ.get(k) for k in _BLAS_VARS}
        for k in _BLAS_VARS:
            os.environ[k] = "1"
        try:
            self.pool = mp.get_context("spawn").Pool(self.n, initializer=_oracle_worker_init,
                                                     initargs=(w.name, w.context, seed, ROOT))
        finally:
            for k, v in old.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        # one unit per worker warms every worker (imports, first touch of the inputs);
        # a second round gives the cost of a round
        self.pool.map(_oracle_task, range(self.n), chunksize=1)
        t0 = time.perf_counter()
        self.pool.map(_oracle_task, range(self.n), chunksize=1)
        self.t_round = time.perf_counter() - t0

    def run(self, seconds: float) -> tuple[int, float, int]:
        """Rounds of one unit per worker filling about `seconds`: (tokens·heads, wall s, units)."""
        rounds = max(1, int(seconds / max(self.t_round, 1e-3)))
        t0 = time.perf_counter()
        done = sum(self.pool.map(_oracle_task, range(rounds * self.n), chunksize=1))
        return done, time.perf_counter() - t0, rounds * self.n

    def close(self):
        self.pool.terminate()
        self.pool.join()


def oracle_sample(w, seconds: float, workers: int):
    """(tokens·heads/s, description, worker processes) of the oracle on a bounded sample."""
    pool = OraclePool(w, workers)
    try:
        done, el, units = pool.run(seconds)
    finally:
        pool.close()
    desc = (f"oracle decode step (float64 numpy) on {units} (sequence, group) units of {w.group_size} heads "
            f"at context {w.context}, {pool.n} worker processes with one BLAS thread each, {el:.1f} s wall")
    return done / el, desc, pool.n


# ----------------------------------------------------------------- reference arm
def run_reference(args):
    from rank_kv_cache_palu_b200.dist import env_world
    from rank_kv_cache_palu_b200.synth import WORKLOADS
    rank, world, _ = env_world()
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    per = max(1.0, min(args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup)))
    pool = OraclePool(w, args.cpu_workers)
    try:
        for _ in range(args.warmup):
            pool.run(per / 4)
        done, el, units = 0, 0.0, 0
        for _ in range(args.steps):
            d, e, u = pool.run(per)
            done, el, units = done + d, el + e, units + u
    finally:
        pool.close()
    value = done / el
    desc = (f"each step: oracle decode step (float64 numpy) on rounds of one (sequence, group) unit per worker "
            f"at context {w.context}, {pool.n} worker processes with one BLAS thread each; {units} units in all")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "context": w.context,
                   "parallelism": "oracle on rank 0 only"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": pool.n, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- our arm
class Setup:
    """Device buffers and calls of one workload: the latent cache (N(0,1) latents), A and B,
    step inputs and per-step metadata, workspaces.  A step appends Q tokens per sequence
    (palu_compress_append) and runs the decode step over every cached token."""

    def __init__(self, w, dev, seed: int, Q: int, steps_total: int, num_splits: int):
        import numpy as np
        import torch

        from rank_kv_cache_palu_b200 import api as P
        from rank_kv_cache_palu_b200.synth import TORCH_DTYPE, page_permutation
        self.w, self.dev, self.Q, self.P = w, dev, Q, P
        self.cfg = cfg = P.make_config(w.num_heads, w.head_dim, w.group_size, w.rank_k, w.rank_v, w.page_size,
                                       w.rope_base, w.act_dtype, w.latent_dtype)
        b, T0, W, Pz = w.batch, w.context, w.width, w.page_size
        self.b, self.T0 = b, T0
        max_pages = (T0 + steps_total * Q + Pz - 1) // Pz
        self.num_pages = num_pages = b * max_pages
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed)
        self.gen = gen
        act = self.act = TORCH_DTYPE[w.act_dtype]
        self.rks, self.rvs = rks, rvs = w.group_ranks
        rk_arg, rv_arg = (rks, rvs) if w.ranked else (None, None)
        self.cache = cache = P.LatentCache.allocate(cfg, num_pages, device=dev, ranks_k=rk_arg, ranks_v=rv_arg)
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
        perm = torch.from_numpy(page_permutation(seed + 7, num_pages)).to(dev)
        self.page_table = perm.view(b, max_pages).contiguous()
        pt_host = self.page_table.cpu().numpy()
        d_model = self.d_model = w.d_model
        # A_k [d_model][Σ r_k], B_k [Σ r_k][W]: group g's columns / rows follow the groups before it
        self.A_k = (torch.randn((d_model, sum(rks)), device=dev, generator=gen) / math.sqrt(d_model)).to(act)
        self.A_v = (torch.randn((d_model, sum(rvs)), device=dev, generator=gen) / math.sqrt(d_model)).to(act)
        self.B_k = torch.cat([torch.randn((r, W), device=dev, generator=gen) / math.sqrt(r) for r in rks]).to(act)
        self.B_v = torch.cat([torch.randn((r, W), device=dev, generator=gen) / math.sqrt(r) for r in rvs]).to(act)
        self.ring = ring = 4
        self.xs = [torch.randn((b * Q, d_model), device=dev, generator=gen).to(act) for _ in range(ring)]
        self.qshape = (b, w.num_heads, w.head_dim) if Q == 1 and not w.ranked else (b, Q, w.num_heads, w.head_dim)
        self.qs = [torch.randn(self.qshape, device=dev, generator=gen).to(act) for _ in range(ring)]

        # per-step metadata, all on the device before timing: step s appends Q tokens per
        # sequence at positions base .. base + Q - 1, then queries them
        def meta(step):
            base = T0 + step * Q
            slots = np.array([pt_host[i, (base + j) // Pz] * Pz + (base + j) % Pz for i in range(b) for j in range(Q)],
                             np.int32)
            qpos = np.array([[base + j for j in range(Q)] for _ in range(b)], np.int32)
            return (torch.from_numpy(slots).to(dev), torch.from_numpy(qpos.reshape(b) if Q == 1 else qpos).to(dev),
                    torch.full((b,), base + Q, dtype=torch.int32, device=dev))
        self.metas = [meta(s) for s in range(steps_total)]
        if w.ranked:
            S = self.S = num_splits     # one split count per decode set, chosen by the library (0 = automatic)
            self.ws_d = torch.zeros(P.palu_decode_ranked_workspace_size(cfg, rks, rvs, b, Q, max_pages, S),
                                    dtype=torch.uint8, device=dev)
            self.ws_c = torch.zeros(P.palu_compress_ranked_workspace_size(cfg, rks, rvs, b * Q, d_model),
                                    dtype=torch.uint8, device=dev)
        else:
            S = self.S = num_splits or P.palu_decode_num_splits(cfg, b, max_pages)
            self.ws_d = torch.zeros(P.palu_decode_multi_workspace_size(cfg, b, Q, max_pages, S),
                                    dtype=torch.uint8, device=dev)
            self.ws_c = torch.zeros(P.palu_compress_workspace_size(cfg, b * Q, d_model), dtype=torch.uint8,
                                    device=dev)
        self.out = torch.empty(self.qshape, dtype=act, device=dev)
        self.stream = torch.cuda.current_stream(dev)

    def decode(self, q, qpos, lens, out=None):
        w, P, c = self.w, self.P, self.cache
        out = self.out if out is None else out
        if w.ranked:
            P.palu_decode_attn_ranked(self.cfg, self.rks, self.rvs, q, qpos, c.zk, c.zv, c.zks, c.zvs, None,
                                      self.page_table, lens, self.num_pages, self.B_k, self.B_v, out, None,
                                      self.ws_d, self.S, self.stream)
            return
        fn = P.palu_decode_attn if self.Q == 1 else P.palu_decode_attn_multi
        fn(self.cfg, q, qpos, c.zk, c.zv, c.zks, c.zvs, None, self.page_table, lens, self.num_pages, self.B_k,
           self.B_v, out, None, self.ws_d, self.S, self.stream)

    def compress(self, x, slots):
        w, P, c = self.w, self.P, self.cache
        if w.ranked:
            P.palu_compress_append_ranked(self.cfg, self.rks, self.rvs, x, self.A_k, self.A_v, slots, None, c.zk,
                                          c.zv, c.zks, c.zvs, None, self.num_pages, self.ws_c, self.stream)
        else:
            P.palu_compress_append(self.cfg, x, self.A_k, self.A_v, slots, None, c.zk, c.zv, c.zks, c.zvs, None,
                                   self.num_pages, self.ws_c, self.stream)

    def step(self, s):
        slots, qpos, lens = self.metas[s]
        self.compress(self.xs[s % self.ring], slots)
        self.decode(self.qs[s % self.ring], qpos, lens)

    def step_units(self, s):
        """tokens·heads of step s: every query's attended tokens times the heads."""
        base = self.T0 + s * self.Q
        return self.b * self.w.num_heads * sum(base + j + 1 for j in range(self.Q))

    def check_status(self, what=""):
        for name, ws in (("decode", self.ws_d), ("compress", self.ws_c)):
            st, det = self.P.palu_get_device_status(ws)
            if st:
                raise RuntimeError(f"{what}: device status {name}={st}({det})")

    def prefill_ms(self, n_pre: int, reps: int = 10):
        """palu_compress_append of an n_pre-token prompt into fresh pages: (ms per call, flops)."""
        import torch
        P, w = self.P, self.w
        Pz = w.page_size
        pre_pages = (n_pre + Pz - 1) // Pz
        pcache = P.LatentCache.allocate(self.cfg, pre_pages, device=self.dev)
        xp = torch.randn((n_pre, self.d_model), device=self.dev, generator=self.gen).to(self.act)
        pslots = torch.arange(n_pre, dtype=torch.int32, device=self.dev)
        ws_p = torch.zeros(P.palu_compress_workspace_size(self.cfg, n_pre, self.d_model), dtype=torch.uint8,
                           device=self.dev)

        def pre():
            P.palu_compress_append(self.cfg, xp, self.A_k, self.A_v, pslots, None, pcache.zk, pcache.zv,
                                   pcache.zks, pcache.zvs, None, pre_pages, ws_p, self.stream)
        for _ in range(3):
            pre()
        torch.cuda.synchronize(self.dev)
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record(self.stream)
        for _ in range(reps):
            pre()
        p1.record(self.stream)
        torch.cuda.synchronize(self.dev)
        st, det = P.palu_get_device_status(ws_p)
        if st:
            raise RuntimeError(f"device status prefill={st}({det})")
        flops = 2.0 * n_pre * self.d_model * (sum(self.rks) + sum(self.rvs))
        return p0.elapsed_time(p1) / reps, flops


def roofline_of(w, seq_lens, Q, seconds, peaks, tc_peak_key):
    """Roofline of one decode call: algorithmic bytes and flops (step_work) over its duration."""
    dbytes, dflops = step_work(w, seq_lens)
    dflops *= Q
    gbs, tfs = dbytes / seconds / 1e9, dflops / seconds / 1e12
    t_hbm = dbytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = dflops / (peaks[tc_peak_key] * 1e12)
    if t_tc > t_hbm:
        roof = {"bound": "tensor", "achieved": tfs, "peak": peaks[tc_peak_key], "unit": "TFLOP/s",
                "frac": tfs / peaks[tc_peak_key]}
    else:
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"]}
    roof.update(hbm_achieved_gbs=gbs, hbm_frac=gbs / peaks["hbm_gbs"], tensor_achieved_tflops=tfs,
                tensor_frac=tfs / peaks[tc_peak_key], algorithmic_bytes_per_launch=dbytes,
                algorithmic_flops_per_launch=dflops, roofline_ms=max(t_hbm, t_tc) * 1e3)
    return roof


# Every workload the metric is quoted on, timed in one run (1 GPU): the fp16 4k point,
# the bf16 context sweep, int4 latents, and a prefill followed by 32 decode steps.
SWEEP = ([("fp16 4k x b1, rank 256/256", "7b_f16_r256_b1_t4k", {})] +
         [(f"bf16 {t}k x b{b}, rank 256/128", f"7b_bf16_r256v128_b{b}_t{t}k", {})
          for t in (4, 16, 64) for b in (1, 8, 16)] +
         [("int4 latents 32k x b8, rank 256/256, fp16 compute", "7b_int4_r256_b8_t32k", {}),
          ("prefill of 8192 tokens, then 32 decode steps at b32 x 16k, bf16 rank 256/256",
           "7b_bf16_r256_b32_t16k", {"prefill": 8192, "steps": 32})])


def measure_sweep_entry(label, wname, opts, dev, peaks, steps=10, warmup=3):
    import torch

    from rank_kv_cache_palu_b200 import api as P
    from rank_kv_cache_palu_b200.synth import WORKLOADS
    w = WORKLOADS[wname]
    K = opts.get("steps", steps)
    su = Setup(w, dev, seed=4321, Q=1, steps_total=warmup + K + 1, num_splits=0)
    entry = {"label": label, "workload": w.name, "batch": w.batch, "context": w.context,
             "act_dtype": w.act_dtype, "latent_dtype": w.latent_dtype, "rank_k": w.rank_k, "rank_v": w.rank_v,
             "num_splits": su.S, "decode_kernel_kind": P.palu_decode_kernel_kind(su.cfg)}
    if "prefill" in opts:
        pre_ms, pre_flops = su.prefill_ms(opts["prefill"])
        entry["prefill"] = {"tokens": opts["prefill"], "ms": pre_ms, "tflops": pre_flops / pre_ms / 1e9,
                            "frac_of_burst_bf16": pre_flops / pre_ms / 1e9 / peaks["bf16_tflops"],
                            "bound": "tensor", "flops": pre_flops}
    for s in range(warmup):
        su.step(s)
    torch.cuda.synchronize(dev)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(su.stream)
    units = 0
    for k in range(K):
        s = warmup + k
        slots, qpos, lens = su.metas[s]
        ev[k][0].record(su.stream)
        su.compress(su.xs[s % su.ring], slots)
        ev[k][1].record(su.stream)
        su.decode(su.qs[s % su.ring], qpos, lens)
        ev[k][2].record(su.stream)
        units += su.step_units(s)
    end.record(su.stream)
    torch.cuda.synchronize(dev)
    su.check_status(label)
    el_ms = start.elapsed_time(end)
    dec_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    cmp_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    mean_T = w.context + warmup + K / 2 + 1
    entry.update(steps=K, ms_per_step=el_ms / K, decode_ms=dec_ms, compress_append_ms=cmp_ms,
                 value=units / (el_ms / 1e3), unit=UNIT,
                 roofline=roofline_of(w, [mean_T] * w.batch, 1, dec_ms / 1e3, peaks, "bf16_tflops"))
    entry["roofline"]["peak_source"] = "measured burst (each timed region is milliseconds long)"
    if "prefill" in opts:
        entry["prefill_plus_steps_ms"] = entry["prefill"]["ms"] + el_ms
    del su
    torch.cuda.empty_cache()
    return entry


def run_ours(args):
    import torch

    from rank_kv_cache_palu_b200 import api as P
    from rank_kv_cache_palu_b200 import dist as D
    from rank_kv_cache_palu_b200.synth import WORKLOADS

    rank, world, local = D.init("nccl")
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs CUDA devices")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = WORKLOADS[args.workload]
    Q = args.queries
    steps_total = 2 * (args.warmup + args.steps) + 2
    su = Setup(w, dev, seed=1234 + rank, Q=Q, steps_total=steps_total, num_splits=args.num_splits)
    b, T0 = w.batch, w.context
    stream = su.stream

    # ---- device-resident timing
    s_idx = 0
    for _ in range(args.warmup):
        su.step(s_idx)
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
            slots, qpos, lens = su.metas[s_idx]
            ev[k][0].record(stream)
            su.compress(su.xs[s_idx % su.ring], slots)
            ev[k][1].record(stream)
            su.decode(su.qs[s_idx % su.ring], qpos, lens)
            ev[k][2].record(stream)
            s_idx += 1
        end.record(stream)
        torch.cuda.synchronize(dev)
    launches = P.palu_kernel_launches() - launches0
    D.barrier(dev)
    su.check_status("timed steps")
    el_ms = D.max_over_ranks(start.elapsed_time(end), dev)
    dec_ms = [e[1].elapsed_time(e[2]) for e in ev]
    cmp_ms = [e[0].elapsed_time(e[1]) for e in ev]
    units = sum(su.step_units(s) for s in range(first_step, first_step + args.steps))
    value = D.sum_over_ranks(units, dev) / (el_ms / 1e3)

    # ---- end to end through the public API: pinned host inputs -> H2D -> step -> D2H.
    # A step's inputs (x, q, slots, query positions, lengths) travel as one copy from one
    # pinned buffer, and its output comes back as one copy.  Two device input and output
    # buffers alternate, so that on copy streams the upload of step s + 1 and the read-back
    # of step s run while step s computes; events order every copy against the steps that
    # produce or consume its buffer, and all copies lie inside the timed region.
    def packed(ts):
        offs, n = [], 0
        for t in ts:
            n = (n + 255) // 256 * 256
            offs.append(n)
            n += t.numel() * t.element_size()
        return offs, n
    in_parts = [su.xs[0], su.qs[0], *su.metas[0]]
    in_offs, in_bytes = packed(in_parts)

    def host_inputs(s):
        buf = torch.zeros(in_bytes, dtype=torch.uint8).pin_memory()
        for t, o in zip([su.xs[s % su.ring], su.qs[s % su.ring], *su.metas[s]], in_offs):
            flat = t.detach().cpu().contiguous().view(torch.uint8).reshape(-1)
            buf[o:o + flat.numel()].copy_(flat)
        return buf
    host_in = [host_inputs(s) for s in range(steps_total)]
    dev_in = [torch.empty(in_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]

    def views(buf):
        return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for t, o in zip(in_parts, in_offs)]
    dev_views = [views(d) for d in dev_in]
    out_d = [torch.empty_like(su.out) for _ in range(2)]
    out_h = [torch.empty(su.out.shape, dtype=su.out.dtype).pin_memory() for _ in range(2)]
    h2d = in_bytes
    d2h = su.out.numel() * su.out.element_size()
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in_ready = [torch.cuda.Event() for _ in range(2)]
    ev_in_free = [torch.cuda.Event() for _ in range(2)]
    ev_out_ready = [torch.cuda.Event() for _ in range(2)]
    ev_out_free = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def upload(s, j):
        with torch.cuda.stream(up):
            if used[j]:
                up.wait_event(ev_in_free[j])      # the step that read this buffer is done
            dev_in[j].copy_(host_in[s], non_blocking=True)
            ev_in_ready[j].record(up)

    def compute(s, j):
        stream.wait_event(ev_in_ready[j])
        if used[j]:
            stream.wait_event(ev_out_free[j])     # the previous result in this buffer is back
        x_d, q_d, slots_d, qpos_d, lens_d = dev_views[j]
        su.compress(x_d, slots_d)
        su.decode(q_d, qpos_d, lens_d, out=out_d[j])
        ev_in_free[j].record(stream)
        ev_out_ready[j].record(stream)
        used[j] = True

    def download(j):
        with torch.cuda.stream(down):
            down.wait_event(ev_out_ready[j])
            out_h[j].copy_(out_d[j], non_blocking=True)
            ev_out_free[j].record(down)

    def run_steps(first, count, start_ev=None):
        if start_ev is not None:
            up.wait_event(start_ev)
            down.wait_event(start_ev)
        upload(first, 0)
        for i in range(count):
            j = i % 2
            if i + 1 < count:
                upload(first + i + 1, (i + 1) % 2)
            compute(first + i, j)
            download(j)
        for j in range(min(count, 2)):
            stream.wait_event(ev_out_free[j])     # every read-back is in before the end event

    run_steps(s_idx, min(args.warmup, 3))
    s_idx += min(args.warmup, 3)
    torch.cuda.synchronize(dev)
    D.barrier(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run_steps(s_idx, args.steps, start_ev=e0)
    e2e_units = sum(su.step_units(s) for s in range(s_idx, s_idx + args.steps))
    s_idx += args.steps
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = D.max_over_ranks(e0.elapsed_time(e1), dev)
    e2e_value = D.sum_over_ranks(e2e_units, dev) / (e2e_ms / 1e3)
    su.check_status("end-to-end steps")

    # ---- prefill: palu_compress_append of a prompt (x·A for n tokens into fresh pages)
    peaks = measured_peaks()
    prefill = None
    n_pre = args.prefill if args.prefill is not None else (8192 if w.name == "7b_bf16_r256_b32_t16k" else 0)
    if n_pre > 0 and not w.ranked:
        pre_ms, pre_flops = su.prefill_ms(n_pre)
        prefill = {"tokens": n_pre, "ms": pre_ms, "tflops": pre_flops / pre_ms / 1e9,
                   "frac_of_burst_bf16": pre_flops / pre_ms / 1e9 / peaks["bf16_tflops"],
                   "kernel": "compress_tc_persistent_kernel (x·[A_k | A_v], tcgen05) + page scatter",
                   "flops": pre_flops}

    # ---- roofline of the dominant kernel (the decode step: split + combine).  The
    # timed region is K decode calls of ~1 ms, far shorter than the seconds-long loop
    # behind the sustained peak, so the burst peak applies unless the region runs for
    # seconds.
    region_s = sum(dec_ms) / 1e3
    tc_key = "bf16_tflops" if region_s < 1.0 else "bf16_tflops_sustained"
    mean_T = T0 + (first_step + args.steps / 2) * Q + Q
    dec_avg_s = statistics.mean(dec_ms) / 1e3
    roof = roofline_of(w, [mean_T] * b, Q, dec_avg_s, peaks, tc_key)
    kinds = sorted({P.palu_decode_kernel_kind(P.make_config(w.num_heads, w.head_dim, w.group_size, rk, rv,
                                                             w.page_size, w.rope_base, w.act_dtype,
                                                             w.latent_dtype))
                    for rk, rv in zip(su.rks, su.rvs)})
    kind = kinds[0] if len(kinds) == 1 else kinds
    roof["traffic"] = profiled_traffic(w.name, "decode")
    roof["peak_source"] = (peaks["source"] + (" burst" if tc_key == "bf16_tflops" else " sustained") +
                           (" bf16 matmul" if roof["bound"] == "tensor" else " copy bandwidth") +
                           f" (timed decode region {region_s * 1e3:.1f} ms)")
    roof["kernel"] = "palu_decode_attn (%s), kernel kind %s%s" % (
        "fold-query + fused split + combine" if kind == 3 else "split + combine", kind,
        ", one launch set per decode set" if w.ranked else "")
    roof["avg_launch_ms"] = dec_avg_s * 1e3

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": el_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.act_dtype if w.latent_dtype != "int4" else "f16/int4",
        "data": "synthetic",
        "config": {"workload": w.name, "batch_per_gpu": b, "global_batch": b * world,
                   "context_at_first_timed_step": T0 + first_step + 1, "heads": w.num_heads,
                   "head_dim": w.head_dim, "group_size": w.group_size, "rank_k": w.rank_k,
                   "rank_v": w.rank_v, "latent_dtype": w.latent_dtype, "page_size": w.page_size,
                   "num_splits": su.S if su.S else "automatic per decode set", "decode_kernel_kind": kind,
                   "queries_per_step": Q,
                   **({"ranks_k": list(su.rks), "ranks_v": list(su.rvs)} if w.ranked else {}),
                   "l2": "inputs larger than L2 (latent cache %.2f GB vs 126 MB L2)" %
                         ((su.cache.zk.numel() + su.cache.zv.numel()) / 1e9),
                   "parallelism": f"dp{world} replicas (independent sequences per GPU)"},
        "roofline": roof,
        "decode_ms_mean": statistics.mean(dec_ms), "compress_append_ms_mean": statistics.mean(cmp_ms),
        "clocks": clk.summary(),
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches,
        **({"prefill": prefill} if prefill else {}),
    }
    del su
    torch.cuda.empty_cache()
    # ---- every other workload of the metric, one GPU (rank 0 alone would hold the others at a barrier)
    if world == 1 and not args.no_sweep:
        line["sweep"] = [measure_sweep_entry(lbl, wn, opts, dev, peaks) for lbl, wn, opts in SWEEP]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, n = oracle_sample(w, args.cpu_seconds, args.cpu_workers)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": n, "kind": "oracle", "sample": desc}
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
