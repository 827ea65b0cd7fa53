"""GPU parity of the tensor-core decode path (head_dim 128, 7B head layout)
against the CPU oracle, through the C ABI."""
import dataclasses
import math

import numpy as np
import pytest
import torch

from oracle import palu_oracle as O
from palu_testlib import (TOL, build_pools, make_decode_case, oracle_decode, rel_err, run_gpu_decode,
                          swizzle_block, unswizzle_block)
from rank_kv_cache_palu_b200 import api as P
from rank_kv_cache_palu_b200.synth import TORCH_DTYPE, WORKLOADS, normal, normal_tensor, page_permutation

pytestmark = pytest.mark.gpu


def small_7b(dt="bf16", r_k=256, r_v=128, gs=4, H=32, **kw):
    return dataclasses.replace(WORKLOADS["7b_bf16_r256v128_b1_t4k"], act_dtype=dt, latent_dtype=dt,
                               rank_k=r_k, rank_v=r_v, group_size=gs, num_heads=H, **kw)


def check(case, num_splits=0, tol=None):
    out, lse = run_gpu_decode(case, num_splits)
    tol = TOL[case.w.act_dtype] if tol is None else tol
    worst = 0.0
    for b, T in enumerate(case.seq_lens):
        ref, ref_lse = oracle_decode(case, b)
        if T == 0:
            assert np.all(out[b] == 0) and np.all(np.isneginf(lse[b]))
            continue
        err = rel_err(out[b], ref)
        worst = max(worst, err)
        assert err <= tol, f"seq {b} (T={T}): rel err {err:.3e}"
        np.testing.assert_allclose(lse[b], ref_lse, rtol=0, atol=2e-2)
    return worst


def test_tc_path_is_selected():
    w = small_7b()
    case = make_decode_case(w, [10])
    assert P.palu_decode_kernel_kind(case.cfg) == 2


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("r_v", [128, 256])
def test_tc_ragged_batch_and_splits(dt, r_v):
    w = small_7b(dt, r_v=r_v, H=8)
    case = make_decode_case(w, [1, 127, 128, 129, 300, 0, 1000, 640])
    for s in (1, 3, 0):
        err = check(case, num_splits=s)
    print(f"{dt} r_v={r_v}: worst rel err {err:.2e}")


@pytest.mark.parametrize("r_k", [64, 128, 192])
def test_tc_smaller_key_ranks(r_k):
    w = small_7b("bf16", r_k=r_k, r_v=128, H=8)
    check(make_decode_case(w, [257, 1024]), num_splits=2)


def test_tc_group_size_two():
    w = small_7b("bf16", gs=2, H=8, r_k=128, r_v=128)
    check(make_decode_case(w, [300, 777]))


def test_tc_explicit_positions_and_peaky_query():
    w = small_7b("bf16", H=8)
    check(make_decode_case(w, [200, 513, 1280], explicit_positions=True, q_scale=8.0), num_splits=2)


def test_tc_large_positions():
    w = small_7b("f16", H=8)
    case = make_decode_case(w, [384])
    case.pos = [np.arange(65000, 65384, dtype=np.int32)]
    case.q_pos = np.array([65500], np.int32)
    check(case)


def test_tc_no_rope():
    w = small_7b("bf16", H=8, rope_base=0.0)
    check(make_decode_case(w, [300, 129]))


def test_tc_split_count_independence():
    w = small_7b("bf16", H=8)
    case = make_decode_case(w, [2048, 1500])
    pools = build_pools(case)
    outs = [run_gpu_decode(case, s, pools=pools)[0] for s in (1, 2, 5, 16)]
    for o in outs[1:]:
        # the split only changes rounding (bf16 P, the order of partial sums)
        assert rel_err(o, outs[0]) <= 1e-2


def test_tc_nan_in_unused_page_rows_is_ignored():
    # the tail of a sequence's last page may hold anything (here NaN); only the
    # valid rows may influence the result
    w = small_7b("bf16", H=8)
    case = make_decode_case(w, [200])
    pools = build_pools(case)
    G, Pz = w.groups, w.page_size
    last_page = int(case.page_table[0, 1])
    nan = np.frombuffer(np.array([np.nan], np.float32).astype(np.float32).tobytes()[2:], np.uint8)  # bf16 NaN
    for name, r in (("zk", w.rank_k), ("zv", w.rank_v)):
        blocks = pools[name].view(case.num_pages, G, Pz * r * 2)
        for g in range(G):
            img = blocks[last_page, g].cpu().numpy()
            rows = unswizzle_block(img, Pz).copy()
            rows[200 - Pz:, 0::2] = nan[0]
            rows[200 - Pz:, 1::2] = nan[1]
            blocks[last_page, g] = torch.from_numpy(swizzle_block(rows)).cuda()
    out, _ = run_gpu_decode(case, 1, pools=pools)
    ref, _ = oracle_decode(case, 0)
    assert np.all(np.isfinite(out))
    assert rel_err(out[0], ref) <= 1e-2


def test_tc_bad_page_reports_bounds():
    w = small_7b("bf16", H=8)
    case = make_decode_case(w, [300])
    pools = build_pools(case)
    bad = case.page_table.copy()
    bad[0, 1] = case.num_pages + 3
    cfg = case.cfg
    ws = torch.zeros(P.palu_decode_workspace_size(cfg, 1, bad.shape[1], 1), dtype=torch.uint8, device="cuda")
    out = torch.empty((1, w.num_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    P.palu_decode_attn(cfg, case.q.cuda(), torch.from_numpy(case.q_pos).cuda(), pools["zk"], pools["zv"],
                       None, None, None, torch.from_numpy(bad).cuda(),
                       torch.tensor(case.seq_lens, dtype=torch.int32).cuda(), case.num_pages,
                       case.B_k.cuda(), case.B_v.cuda(), out, None, ws, 1)
    st, _ = P.palu_get_device_status(ws)
    assert st == 7


# ------------------------------------------------------------ int4 latents on the tensor cores
def int4_7b(act="f16", H=8):
    return dataclasses.replace(WORKLOADS["7b_int4_r256_b8_t32k"], act_dtype=act, num_heads=H)


def test_tc_int4_path_is_selected():
    for act in ("f16", "bf16"):
        case = make_decode_case(int4_7b(act), [10])
        assert P.palu_decode_kernel_kind(case.cfg) == 2


@pytest.mark.parametrize("act", ["f16", "bf16"])
def test_tc_int4_ragged_batch_and_splits(act):
    # full pages, a ragged last page, single tokens, an empty sequence; two split counts
    case = make_decode_case(int4_7b(act), [300, 1, 1000, 129, 0, 128, 640])
    check(case)
    check(case, num_splits=3)


def test_tc_int4_explicit_positions_and_peaky_query():
    case = make_decode_case(int4_7b("f16"), [700, 257], explicit_positions=True, q_scale=4.0)
    check(case)


# ------------------------------------------------------------ full-size, sampled units
def sampled_full_size(w, context, units, seed=123, num_splits=0):
    """Run the full workload on the GPU; check the sampled (sequence, group) units.

    Unsampled units are filled on the device with N(0,1) latents (they do not
    influence the sampled outputs); sampled units come from the host generator,
    as do q and B.
    """
    b, G, W, Pz = w.batch, w.groups, w.width, w.page_size
    cfg = P.make_config(w.num_heads, w.head_dim, w.group_size, w.rank_k, w.rank_v, Pz, w.rope_base,
                        w.act_dtype, w.latent_dtype)
    max_pages = (context + Pz - 1) // Pz
    num_pages = b * max_pages
    pt = page_permutation(seed, num_pages).reshape(b, max_pages)
    dev = torch.device("cuda")
    int4 = w.latent_dtype == "int4"
    cache = P.LatentCache.allocate(cfg, num_pages, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    for pool in (cache.zk, cache.zv):
        if int4:                                   # random codes, every nibble value included
            pool.copy_(torch.randint(0, 256, pool.shape, dtype=torch.uint8, device=dev, generator=gen))
            continue
        view = pool.view(TORCH_DTYPE[w.latent_dtype])
        for i in range(0, view.numel(), 1 << 28):
            seg = view[i:i + (1 << 28)]
            seg.copy_(torch.randn(seg.shape, device=dev, generator=gen))
    for sp in (cache.zks, cache.zvs):
        if sp is not None:
            sp.view(torch.float16).copy_(torch.rand(sp.numel() // 2, device=dev, generator=gen) * 0.5)
    host = {}
    for (bi, g) in units:
        for name, r, pool, spool in (("zk", w.rank_k, cache.zk, cache.zks), ("zv", w.rank_v, cache.zv, cache.zvs)):
            z32 = normal(seed, name, (context, r), unit=(bi, g))
            if int4:
                packed, sc = O.quantize_int4(z32)
                host[(name, bi, g)] = torch.from_numpy(O.dequantize_int4(packed, sc, w.act_dtype))
                zb, row_bytes = packed, r // 2
                srows = spool.view(num_pages, G, Pz, -1)
                sb = np.zeros((context, srows.shape[3]), np.uint8)
                sb[:, : sc.shape[1] * 2] = sc.view(np.uint8)
            else:
                z = torch.from_numpy(z32).to(TORCH_DTYPE[w.latent_dtype])
                host[(name, bi, g)] = z
                zb, row_bytes = z.view(torch.uint8).numpy(), r * 2
            blocks = pool.view(num_pages, G, Pz * row_bytes)
            for p in range(max_pages):
                t0, t1 = p * Pz, min(context, (p + 1) * Pz)
                rows = np.zeros((Pz, row_bytes), np.uint8)
                rows[: t1 - t0] = zb[t0:t1]
                blocks[pt[bi, p], g].copy_(torch.from_numpy(swizzle_block(rows)).to(dev))
                if int4:
                    srow = np.zeros((Pz, srows.shape[3]), np.uint8)
                    srow[: t1 - t0] = sb[t0:t1]
                    srows[pt[bi, p], g].copy_(torch.from_numpy(srow).to(dev))
    q = normal_tensor(seed, "q", (b, w.num_heads, w.head_dim), w.act_dtype)
    B_k = normal_tensor(seed, "B_k", (G, w.rank_k, W), w.act_dtype, 1 / math.sqrt(w.rank_k))
    B_v = normal_tensor(seed, "B_v", (G, w.rank_v, W), w.act_dtype, 1 / math.sqrt(w.rank_v))
    S = num_splits or P.palu_decode_num_splits(cfg, b, max_pages)
    ws = torch.zeros(P.palu_decode_workspace_size(cfg, b, max_pages, S), dtype=torch.uint8, device=dev)
    out = torch.empty((b, w.num_heads, w.head_dim), dtype=TORCH_DTYPE[w.act_dtype], device=dev)
    lse = torch.empty((b, w.num_heads), dtype=torch.float32, device=dev)
    q_pos = torch.full((b,), context - 1, dtype=torch.int32, device=dev)
    lens = torch.full((b,), context, dtype=torch.int32, device=dev)
    P.palu_decode_attn(cfg, q.to(dev), q_pos, cache.zk, cache.zv, cache.zks, cache.zvs, None,
                       torch.from_numpy(pt).to(dev), lens, num_pages, B_k.to(dev), B_v.to(dev), out, lse,
                       ws, S)
    torch.cuda.synchronize()
    assert P.palu_get_device_status(ws)[0] == 0
    got = out.to(torch.float64).cpu().numpy()
    Bk, Bv = B_k.to(torch.float64).numpy(), B_v.to(torch.float64).numpy()
    qn = q.to(torch.float64).numpy()
    worst = 0.0
    for (bi, g) in units:
        zk = np.zeros((G, context, w.rank_k))
        zv = np.zeros((G, context, w.rank_v))
        zk[g] = host[("zk", bi, g)].to(torch.float64).numpy()
        zv[g] = host[("zv", bi, g)].to(torch.float64).numpy()
        for j in range(w.group_size):
            h = g * w.group_size + j
            ref, _ = O.decode_attention_head(h, qn[bi], context - 1, zk, zv, np.arange(context), Bk, Bv,
                                             w.group_size, w.rope_base)
            err = rel_err(got[bi, h], ref)
            worst = max(worst, err)
            assert err <= TOL[w.act_dtype], f"unit ({bi},{g}) head {h}: {err:.3e}"
    return worst, S


@pytest.mark.slow
def test_full_size_7b_bf16_b16_t16k_sampled():
    # the bench workload: 7B-shaped bf16, rank 256/128, batch 16, context 16k (+5, a ragged page)
    w = WORKLOADS["7b_bf16_r256v128_b16_t16k"]
    worst, S = sampled_full_size(w, w.context + 5, [(0, 0), (7, 3), (15, 7)])
    print(f"16k x 16 (S={S}): worst rel err {worst:.2e}")


@pytest.mark.slow
def test_full_size_7b_bf16_b16_t64k_sampled():
    w = WORKLOADS["7b_bf16_r256v128_b16_t64k"]
    worst, S = sampled_full_size(w, w.context, [(3, 5), (12, 1)])
    print(f"64k x 16 (S={S}): worst rel err {worst:.2e}")


@pytest.mark.slow
def test_full_size_7b_bf16_r256_b32_t16k_sampled():
    w = WORKLOADS["7b_bf16_r256_b32_t16k"]
    worst, S = sampled_full_size(w, w.context + 31, [(0, 2), (31, 6)])
    print(f"r256/256 16k x 32 (S={S}): worst rel err {worst:.2e}")


@pytest.mark.slow
def test_full_size_7b_int4_b8_t32k_sampled():
    # int4 latents (rank 256/256, fp16 compute), batch 8, context 32k (+77, a ragged page)
    w = WORKLOADS["7b_int4_r256_b8_t32k"]
    worst, S = sampled_full_size(w, w.context + 77, [(0, 1), (5, 6)])
    print(f"int4 32k x 8 (S={S}): worst rel err {worst:.2e}")
