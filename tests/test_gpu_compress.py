"""GPU parity of palu_compress_append (z = x·A into the paged cache) against the oracle."""
import dataclasses
import math

import numpy as np
import pytest
import torch

from oracle import palu_oracle as O
from palu_testlib import unswizzle_block
from rank_kv_cache_palu_b200 import api as P
from rank_kv_cache_palu_b200.synth import TORCH_DTYPE, WORKLOADS, normal_tensor

pytestmark = pytest.mark.gpu

SENTINEL = 0xAB


def run_compress(w, x, A_k, A_v, slots, positions, num_pages):
    cfg = P.make_config(w.num_heads, w.head_dim, w.group_size, w.rank_k, w.rank_v, w.page_size,
                        w.rope_base, w.act_dtype, w.latent_dtype)
    cache = P.LatentCache.allocate(cfg, num_pages, with_positions=True, fill=SENTINEL)
    n, d_model = x.shape
    ws = torch.zeros(P.palu_compress_workspace_size(cfg, n, d_model), dtype=torch.uint8, device="cuda")
    P.palu_compress_append(cfg, x.cuda(), A_k.cuda(), A_v.cuda(), torch.from_numpy(slots).cuda(),
                           None if positions is None else torch.from_numpy(positions).cuda(),
                           cache.zk, cache.zv, cache.zks, cache.zvs, cache.pos, num_pages, ws)
    torch.cuda.synchronize()
    st, detail = P.palu_get_device_status(ws)
    return cache, st, detail


def gather_rows(pool: torch.Tensor, w, slots, r, row_bytes, swizzled=True):
    """Bytes of each token's row per group: [n, G, row_bytes] (slot < 0 rows are zero)."""
    host = pool.cpu().numpy().reshape(-1, w.groups, w.page_size * row_bytes)
    out = np.zeros((len(slots), w.groups, row_bytes), np.uint8)
    cache = {}
    for i, s in enumerate(slots):
        if s >= 0:
            for g in range(w.groups):
                key = (s // w.page_size, g)
                if key not in cache:
                    img = host[key[0], g]
                    cache[key] = unswizzle_block(img, w.page_size) if swizzled else \
                        img.reshape(w.page_size, row_bytes)
                out[i, g] = cache[key][s % w.page_size]
    return out


def as_values(rows: np.ndarray, dtype: str) -> np.ndarray:
    t = torch.from_numpy(rows.copy()).view(TORCH_DTYPE[dtype])
    return t.to(torch.float64).numpy()


def make_slots(n, num_pages, page_size, seed, holes=True):
    rng = np.random.default_rng(seed)
    slots = rng.choice(num_pages * page_size, size=n, replace=False).astype(np.int32)
    if holes and n > 4:
        slots[rng.choice(n, size=max(1, n // 16), replace=False)] = -1
    return slots


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("n", [1, 37, 200])
def test_compress_small(dt, n):
    w = dataclasses.replace(WORKLOADS["tiny_f32"], act_dtype=dt, latent_dtype=dt, rank_k=64,
                            rank_v=128, d_model=192)
    x = normal_tensor(7, "x", (n, w.d_model), dt)
    A_k = normal_tensor(7, "A_k", (w.d_model, w.groups * w.rank_k), dt, 1 / math.sqrt(w.d_model))
    A_v = normal_tensor(7, "A_v", (w.d_model, w.groups * w.rank_v), dt, 1 / math.sqrt(w.d_model))
    num_pages = (n + w.page_size - 1) // w.page_size + 2
    slots = make_slots(n, num_pages, w.page_size, seed=n)
    positions = (np.arange(n) * 3 + 5).astype(np.int32)
    cache, st, _ = run_compress(w, x, A_k, A_v, slots, positions, num_pages)
    assert st == 0
    esz = 4 if dt == "f32" else 2
    tol = {"f32": 1e-5, "f16": 2 ** -10, "bf16": 2 ** -7}[dt]
    for pool, A, r in ((cache.zk, A_k, w.rank_k), (cache.zv, A_v, w.rank_v)):
        got = as_values(gather_rows(pool, w, slots, r, r * esz), dt)       # [n, G, r]
        ref = O.compress(x.to(torch.float64).numpy(), A.to(torch.float64).numpy(), dt)
        ref = ref.reshape(n, w.groups, r)
        keep = slots >= 0
        err = np.abs(got[keep] - ref[keep])
        # within one rounding step of the dtype (float32 accumulation may cross a tie)
        assert np.all(err <= tol * np.abs(ref[keep]) + 1e-6 * np.max(np.abs(ref))), float(err.max())
    # skipped rows untouched, positions written
    pos = cache.pos.cpu().numpy()
    for i, s in enumerate(slots):
        if s >= 0:
            assert pos[s] == positions[i]


def exact_inputs(w, n, seed):
    """x on a dyadic grid and A a 0/1 column-selection matrix: x·A is exact in float32."""
    rng = np.random.default_rng(seed)
    x = (rng.integers(-24, 25, size=(n, w.d_model)) / 8.0).astype(np.float32)
    def sel(ncol):
        A = np.zeros((w.d_model, ncol), np.float32)
        A[rng.integers(0, w.d_model, size=ncol), np.arange(ncol)] = 1.0
        return A
    t = TORCH_DTYPE[w.act_dtype]
    return (torch.from_numpy(x).to(t), torch.from_numpy(sel(w.groups * w.rank_k)).to(t),
            torch.from_numpy(sel(w.groups * w.rank_v)).to(t))


@pytest.mark.parametrize("act", ["f16", "bf16"])
def test_compress_int4_bit_exact(act):
    # exactly representable latents: quantisation codes, bytes and scales match bit for bit
    w = dataclasses.replace(WORKLOADS["tiny_f32"], act_dtype=act, latent_dtype="int4", rank_k=256,
                            rank_v=512, d_model=256)
    n = 150
    x, A_k, A_v = exact_inputs(w, n, 3)
    num_pages = 4
    slots = make_slots(n, num_pages, w.page_size, seed=5)
    cache, st, _ = run_compress(w, x, A_k, A_v, slots, None, num_pages)
    assert st == 0
    kb, vb, ksb, vsb = P.palu_cache_strides(P.make_config(
        w.num_heads, w.head_dim, w.group_size, w.rank_k, w.rank_v, w.page_size, 10000.0, act, "int4"))
    for pool, spool, A, r in ((cache.zk, cache.zks, A_k, w.rank_k), (cache.zv, cache.zvs, A_v, w.rank_v)):
        z = O.compress(x.to(torch.float64).numpy(), A.to(torch.float64).numpy(), "f32")
        packed, sc = O.quantize_int4(z.reshape(n, w.groups, r).astype(np.float32))
        srow = (2 * (r // 32) + 15) // 16 * 16
        got = gather_rows(pool, w, slots, r, r // 2)
        got_s = gather_rows(spool, w, slots, r, srow, swizzled=False)[..., : 2 * (r // 32)].copy().view(np.float16)
        keep = slots >= 0
        np.testing.assert_array_equal(got[keep], packed[keep])
        np.testing.assert_array_equal(got_s[keep], sc[keep])


def test_compress_int4_general():
    # N(0,1) inputs: codes may differ from the oracle's only where float32
    # accumulation order moves a value across a rounding boundary
    w = dataclasses.replace(WORKLOADS["tiny_f32"], act_dtype="f16", latent_dtype="int4", rank_k=256,
                            rank_v=256, d_model=256)
    n = 100
    x = normal_tensor(11, "x", (n, w.d_model), "f16")
    A_k = normal_tensor(11, "A_k", (w.d_model, w.groups * w.rank_k), "f16", 1 / 16)
    A_v = normal_tensor(11, "A_v", (w.d_model, w.groups * w.rank_v), "f16", 1 / 16)
    slots = make_slots(n, 2, w.page_size, seed=9, holes=False)
    cache, st, _ = run_compress(w, x, A_k, A_v, slots, None, 2)
    assert st == 0
    for pool, spool, A, r in ((cache.zk, cache.zks, A_k, w.rank_k), (cache.zv, cache.zvs, A_v, w.rank_v)):
        z = O.compress(x.to(torch.float64).numpy(), A.to(torch.float64).numpy(), None).reshape(n, w.groups, r)
        srow = (2 * (r // 32) + 15) // 16 * 16
        got = gather_rows(pool, w, slots, r, r // 2)
        got_s = gather_rows(spool, w, slots, r, srow, swizzled=False)[..., : 2 * (r // 32)].copy().view(np.float16)
        deq = O.dequantize_int4(got, got_s, "f16")
        s_full = np.repeat(got_s.astype(np.float64), 32, axis=-1)
        # quantisation step (s/2, s itself rounded to fp16), plus the fp16 rounding of
        # the dequantised product code*s (half an ulp at |code*s| <= 7s), plus the
        # float32 accumulation of x.A
        bound = 0.5 * s_full * (1 + 2 ** -10) + 7 * s_full * 2 ** -11 + 1e-5 * (np.abs(z) + 1)
        assert np.all(np.abs(deq - z) <= bound), float(np.max(np.abs(deq - z) / s_full))
        _, sc_ref = O.quantize_int4(z.astype(np.float32))
        assert np.all(np.abs(got_s.astype(np.float64) - sc_ref.astype(np.float64))
                      <= 2 ** -10 * np.abs(sc_ref.astype(np.float64)) + 1e-7)


def test_compress_bad_slot_reports_bounds():
    w = dataclasses.replace(WORKLOADS["tiny_f32"], d_model=128)
    n = 10
    x = normal_tensor(1, "x", (n, w.d_model), "f32")
    A_k = normal_tensor(1, "A_k", (w.d_model, w.groups * w.rank_k), "f32", 0.1)
    A_v = normal_tensor(1, "A_v", (w.d_model, w.groups * w.rank_v), "f32", 0.1)
    slots = np.arange(n, dtype=np.int32)
    slots[3] = 10 ** 6
    _, st, _ = run_compress(w, x, A_k, A_v, slots, None, 1)
    assert st == 7


def _check_rows(w, x, A, pool, slots, rows, r, dt):
    """Oracle z for the sampled token rows vs the cache contents of those tokens."""
    esz = 2
    got = as_values(gather_rows(pool, w, slots[rows], r, r * esz), dt)
    ref = O.compress(x[rows].to(torch.float64).numpy(), A.to(torch.float64).numpy(), dt)
    ref = ref.reshape(len(rows), w.groups, r)
    tol = {"f16": 2 ** -10, "bf16": 2 ** -7}[dt]
    err = np.abs(got - ref)
    assert np.all(err <= tol * np.abs(ref) + 1e-6 * np.max(np.abs(ref))), float(err.max())


@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_compress_prefill_multi_tile(dt):
    # several 256-token tiles and a ragged last one (no K split)
    w = dataclasses.replace(WORKLOADS["7b_bf16_r256v128_b1_t4k"], act_dtype=dt, latent_dtype=dt,
                            num_heads=8, d_model=512)
    n = 600
    x = normal_tensor(21, "x", (n, w.d_model), dt)
    A_k = normal_tensor(21, "A_k", (w.d_model, w.groups * w.rank_k), dt, 1 / math.sqrt(w.d_model))
    A_v = normal_tensor(21, "A_v", (w.d_model, w.groups * w.rank_v), dt, 1 / math.sqrt(w.d_model))
    num_pages = 8
    slots = make_slots(n, num_pages, w.page_size, seed=21)
    cache, st, _ = run_compress(w, x, A_k, A_v, slots, None, num_pages)
    assert st == 0
    rows = np.flatnonzero(slots >= 0)
    _check_rows(w, x, A_k, cache.zk, slots, rows, w.rank_k, dt)
    _check_rows(w, x, A_v, cache.zv, slots, rows, w.rank_v, dt)


@pytest.mark.slow
def test_compress_prefill_full_size_sampled():
    # 8192 tokens of a 7B layer, x [8192 x 4096] bf16 into rank 256/256 latents; sampled tokens
    w = WORKLOADS["7b_bf16_r256_b32_t16k"]
    n = 8192
    x = normal_tensor(5, "x", (n, w.d_model), "bf16")
    A_k = normal_tensor(5, "A_k", (w.d_model, w.groups * w.rank_k), "bf16", 1 / math.sqrt(w.d_model))
    A_v = normal_tensor(5, "A_v", (w.d_model, w.groups * w.rank_v), "bf16", 1 / math.sqrt(w.d_model))
    num_pages = n // w.page_size + 1
    slots = np.random.default_rng(5).permutation(num_pages * w.page_size)[:n].astype(np.int32)
    cache, st, _ = run_compress(w, x, A_k, A_v, slots, None, num_pages)
    assert st == 0
    rows = np.random.default_rng(6).choice(n, size=48, replace=False)
    rows = np.concatenate([rows, [0, 255, 256, n - 1]])
    _check_rows(w, x, A_k, cache.zk, slots, rows, w.rank_k, "bf16")
    _check_rows(w, x, A_v, cache.zv, slots, rows, w.rank_v, "bf16")


def test_compress_append_step_full_size():
    # the per-step append of a decode batch: 32 tokens of a 7B layer (K split across CTAs)
    w = WORKLOADS["7b_bf16_r256v128_b16_t16k"]
    n = 32
    x = normal_tensor(9, "x", (n, w.d_model), "bf16")
    A_k = normal_tensor(9, "A_k", (w.d_model, w.groups * w.rank_k), "bf16", 1 / math.sqrt(w.d_model))
    A_v = normal_tensor(9, "A_v", (w.d_model, w.groups * w.rank_v), "bf16", 1 / math.sqrt(w.d_model))
    num_pages = 40
    slots = make_slots(n, num_pages, w.page_size, seed=9)
    for _ in range(2):                       # twice: the split counters must come back to zero
        cache, st, _ = run_compress(w, x, A_k, A_v, slots, None, num_pages)
        assert st == 0
    rows = np.flatnonzero(slots >= 0)
    _check_rows(w, x, A_k, cache.zk, slots, rows, w.rank_k, "bf16")
    _check_rows(w, x, A_v, cache.zv, slots, rows, w.rank_v, "bf16")


@pytest.mark.parametrize("act", ["f16", "bf16"])
def test_compress_int4_prefill_bit_exact(act):
    # several 256-token tiles (the persistent prefill kernel) with int4 latents: exactly
    # representable latents give bit-exact codes, bytes and scales; positions are written once
    w = dataclasses.replace(WORKLOADS["tiny_f32"], act_dtype=act, latent_dtype="int4", rank_k=256,
                            rank_v=512, d_model=256)
    n = 700
    x, A_k, A_v = exact_inputs(w, n, 13)
    num_pages = 8
    slots = make_slots(n, num_pages, w.page_size, seed=17)
    positions = (np.arange(n) * 7 + 3).astype(np.int32)
    cache, st, _ = run_compress(w, x, A_k, A_v, slots, positions, num_pages)
    assert st == 0
    keep = slots >= 0
    for pool, spool, A, r in ((cache.zk, cache.zks, A_k, w.rank_k), (cache.zv, cache.zvs, A_v, w.rank_v)):
        z = O.compress(x.to(torch.float64).numpy(), A.to(torch.float64).numpy(), "f32")
        packed, sc = O.quantize_int4(z.reshape(n, w.groups, r).astype(np.float32))
        srow = (2 * (r // 32) + 15) // 16 * 16
        got = gather_rows(pool, w, slots, r, r // 2)
        got_s = gather_rows(spool, w, slots, r, srow, swizzled=False)[..., : 2 * (r // 32)].copy().view(np.float16)
        np.testing.assert_array_equal(got[keep], packed[keep])
        np.testing.assert_array_equal(got_s[keep], sc[keep])
    pos = cache.pos.cpu().numpy()
    np.testing.assert_array_equal(pos[slots[keep]], positions[keep])


@pytest.mark.parametrize("n", [16, 600])
def test_compress_tc_bad_slot_and_holes(n):
    # Tensor-core compress, both forms: 16 tokens (one token tile, K split across CTAs) and
    # 600 (the persistent prefill, several tiles and a ragged one).  Each tile looks its
    # tokens' slots up once; an out-of-pool slot is reported (PALU_ERR_DEVICE_BOUNDS) and,
    # like a skipped one (-1), writes nothing, while every other token lands in its slot
    # with its position.
    dt = "bf16"
    w = dataclasses.replace(WORKLOADS["7b_bf16_r256v128_b1_t4k"], num_heads=8, d_model=512)
    x = normal_tensor(31, "x", (n, w.d_model), dt)
    A_k = normal_tensor(31, "A_k", (w.d_model, w.groups * w.rank_k), dt, 1 / math.sqrt(w.d_model))
    A_v = normal_tensor(31, "A_v", (w.d_model, w.groups * w.rank_v), dt, 1 / math.sqrt(w.d_model))
    num_pages = 8
    cap = num_pages * w.page_size
    slots = make_slots(n, num_pages, w.page_size, seed=31)
    valid = np.flatnonzero(slots >= 0)
    slots[valid[len(valid) // 2]] = cap + 5
    positions = (np.arange(n) * 5 + 1).astype(np.int32)
    cache, st, _ = run_compress(w, x, A_k, A_v, slots, positions, num_pages)
    assert st == 7
    keep = (slots >= 0) & (slots < cap)
    rows = np.flatnonzero(keep)
    _check_rows(w, x, A_k, cache.zk, slots, rows, w.rank_k, dt)
    _check_rows(w, x, A_v, cache.zv, slots, rows, w.rank_v, dt)
    others = np.setdiff1d(np.arange(cap, dtype=np.int32), slots[keep])
    for pool, r in ((cache.zk, w.rank_k), (cache.zv, w.rank_v)):
        assert np.all(gather_rows(pool, w, others, r, r * 2) == SENTINEL)
    pos = cache.pos.cpu().numpy()
    np.testing.assert_array_equal(pos[slots[keep]], positions[keep])
    assert np.all(pos[others] == 0)
