"""Host-side logic of bench.py: the algorithmic work a decode call is credited
with, the roofline's choice of bound, and the oracle worker pool behind the CPU
baseline (no GPU needed)."""
import importlib
import os

import pytest

from rank_kv_cache_palu_b200.synth import WORKLOADS


def _bench():
    # imported by its module name (the repository root is on sys.path), so that the
    # spawned oracle workers can import the same module
    return importlib.import_module("bench")


def test_step_work_hand_count():
    B = _bench()
    w = WORKLOADS["7b_bf16_r256v128_b16_t16k"]
    T = 16400
    by, fl = B.step_work(w, [T] * 16)
    # latents: (256 + 128) bf16 entries per token and group; B_k and B_v once; q and out
    lat = 16 * T * 8 * (256 + 128) * 2
    bmat = 8 * (256 + 128) * 512 * 2
    qo = 16 * 32 * 128 * 2 * 2
    assert by == lat + bmat + qo
    # per (token, group): the key rebuild 2·r_k·W and the latent value sum 2·g·r_v; per
    # (sequence, head): the up-projection 2·r_v·d_h
    assert fl == 16 * T * 8 * (2 * 256 * 512 + 2 * 4 * 128) + 16 * 4 * 8 * 2 * 128 * 128


def test_step_work_int4_counts_scales():
    B = _bench()
    w = WORKLOADS["7b_int4_r256_b8_t32k"]
    by, _ = B.step_work(w, [1000])
    # 288 bytes per (token, group): 256 of codes, 32 of fp16 scales
    assert by == 1000 * 8 * 288 + 8 * 512 * 512 * 2 + 32 * 128 * 2 * 2


def test_roofline_picks_the_slower_bound():
    B = _bench()
    peaks = {"hbm_gbs": 6550.0, "bf16_tflops": 1640.0, "bf16_tflops_sustained": 1366.0}
    w = WORKLOADS["7b_bf16_r256v128_b16_t16k"]
    r = B.roofline_of(w, [16400] * 16, 1, 1e-3, peaks, "bf16_tflops")
    assert r["bound"] == "tensor"           # rank 256/128 with RoPE: the key rebuild dominates
    assert r["frac"] == pytest.approx(r["achieved"] / 1640.0)
    wn = WORKLOADS["7b_bf16_r256v128_b16_t16k_norope"]
    r = B.roofline_of(wn, [16400] * 16, 1, 1e-3, peaks, "bf16_tflops")
    assert r["bound"] == "hbm"              # without RoPE the scores come straight from the latents
    assert r["frac"] == pytest.approx(r["hbm_achieved_gbs"] / 6550.0)


def test_sweep_covers_every_workload_of_the_metric():
    B = _bench()
    names = [wn for _, wn, _ in B.SWEEP]
    assert "7b_f16_r256_b1_t4k" in names and "7b_int4_r256_b8_t32k" in names
    for t in (4, 16, 64):
        for b in (1, 8, 16):
            assert f"7b_bf16_r256v128_b{b}_t{t}k" in names
    pre = [o for _, wn, o in B.SWEEP if wn == "7b_bf16_r256_b32_t16k"]
    assert pre == [{"prefill": 8192, "steps": 32}]
    assert all(wn in WORKLOADS for wn in names)


def test_oracle_pool_runs_units_in_spawned_workers():
    B = _bench()
    pool = B.OraclePool(WORKLOADS["tiny_f32"], workers=2)
    try:
        done, el, units = pool.run(0.01)
    finally:
        pool.close()
    assert pool.n == min(2, len(os.sched_getaffinity(0)))
    assert units >= pool.n and done == units * 4 * 256      # group of 4 heads x 256 tokens per unit
    assert el > 0
