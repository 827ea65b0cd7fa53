"""GPU parity of layers whose head groups carry their own ranks (the output of
Palu's rank search) against the CPU oracle, through the C ABI: the decode step
on every kernel family (a layer's rank classes may land on different kernels),
multi-token steps, int4 latents, and the compress/append into the ranked
cache layout."""
import dataclasses
import math

import numpy as np
import pytest
import torch

from oracle import palu_oracle as O
from palu_testlib import TOL, build_ranked_pools, make_ranked_case, ranked_offsets, rel_err, unswizzle_block
from rank_kv_cache_palu_b200 import api as P
from rank_kv_cache_palu_b200.synth import TORCH_DTYPE, WORKLOADS, normal_tensor

pytestmark = pytest.mark.gpu


def run_ranked(case, num_splits=0, pools=None):
    w = case.w
    cfg = case.cfg
    pools = build_ranked_pools(case) if pools is None else pools
    b, nq = case.q.shape[0], case.q.shape[1]
    dev = "cuda"
    ws = torch.zeros(P.palu_decode_ranked_workspace_size(cfg, case.ranks_k, case.ranks_v, b, nq,
                                                         case.page_table.shape[1], num_splits),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((b, nq, w.num_heads, w.head_dim), dtype=TORCH_DTYPE[w.act_dtype], device=dev)
    lse = torch.empty((b, nq, w.num_heads), dtype=torch.float32, device=dev)
    P.palu_decode_attn_ranked(cfg, case.ranks_k, case.ranks_v, case.q.to(dev),
                              torch.from_numpy(case.q_pos).to(dev), pools["zk"], pools["zv"], pools["zks"],
                              pools["zvs"], pools["pos"], torch.from_numpy(case.page_table).to(dev),
                              torch.tensor(case.seq_lens, dtype=torch.int32, device=dev), case.num_pages,
                              case.B_k.to(dev), case.B_v.to(dev), out, lse, ws, num_splits)
    torch.cuda.synchronize()
    st, detail = P.palu_get_device_status(ws)
    assert st == 0, f"device status {st} ({detail})"
    return out.to(torch.float64).cpu().numpy(), lse.cpu().numpy()


def check_ranked(case, num_splits=0):
    w = case.w
    out, lse = run_ranked(case, num_splits)
    qn = case.q.to(torch.float64).numpy()
    for i in range(len(case.seq_lens)):
        zk, zv, Bk, Bv = case.oracle_inputs(i)
        ref, ref_lse = O.decode_attention_ranked(qn[i], case.q_pos[i], zk, zv, case.positions(i), Bk, Bv,
                                                 w.group_size, w.rope_base)
        for j in range(qn.shape[1]):
            if np.isneginf(ref_lse[j]).all():
                assert np.all(out[i, j] == 0) and np.all(np.isneginf(lse[i, j]))
                continue
            err = rel_err(out[i, j], ref[j])
            assert err <= TOL[w.act_dtype], f"seq {i} query {j}: rel err {err:.3e}"
            np.testing.assert_allclose(lse[i, j], ref_lse[j], rtol=0, atol=2e-2)


def layer(**kw):
    # 7B head shape with four groups of four heads
    return dataclasses.replace(WORKLOADS["7b_bf16_r256v128_b1_t4k"], num_heads=16, **kw)


def class_kinds(case):
    out = set()
    for rk, rv in set(zip(case.ranks_k, case.ranks_v)):
        w = case.w
        c = P.make_config(w.num_heads, w.head_dim, w.group_size, rk, rv, w.page_size, w.rope_base,
                          w.act_dtype, w.latent_dtype)
        out.add(P.palu_decode_kernel_kind(c))
    return out


def test_ranked_rope_classes_on_tensor_core_and_cuda_core_kernels():
    # rank 384 keys exceed the tensor-core kernel's shared memory: that class runs
    # on the CUDA-core kernel, the others on tcgen05
    case = make_ranked_case(layer(), [256, 128, 384, 128], [128, 256, 128, 128], [300, 130, 1000, 5])
    assert class_kinds(case) == {1, 2}
    check_ranked(case)
    check_ranked(case, num_splits=3)


@pytest.mark.parametrize("act", ["bf16", "f16"])
def test_ranked_no_rope_fused(act):
    case = make_ranked_case(layer(rope_base=0.0, act_dtype=act, latent_dtype=act), [64, 192, 128, 512],
                            [128, 128, 256, 256], [300, 129, 1000, 5])
    assert class_kinds(case) == {3}
    check_ranked(case)
    check_ranked(case, num_splits=2)


@pytest.mark.parametrize("nq", [3, 5])
def test_ranked_multi_query(nq):
    case = make_ranked_case(layer(rope_base=0.0), [128, 64, 128, 256], [256, 128, 256, 128], [400, 77],
                            nq=nq, explicit_positions=True)
    check_ranked(case)
    case = make_ranked_case(layer(), [128, 64, 128, 256], [256, 128, 256, 128], [400, 77], nq=nq)
    check_ranked(case)


def test_ranked_int4():
    w = dataclasses.replace(WORKLOADS["7b_int4_r256_b8_t32k"], num_heads=16)
    case = make_ranked_case(w, [256, 512, 256, 256], [256, 256, 512, 256], [520, 129])
    assert class_kinds(case) == {1, 2}
    check_ranked(case)
    # groups 0 and 1 share a value rank on the CUDA-core kernel with key ranks 256 and 512
    # (one launch; per-group scale rows)
    check_ranked(make_ranked_case(w, [256, 512, 512, 256], [512, 512, 256, 256], [300, 77]))


def test_ranked_equal_ranks_is_the_uniform_call():
    # one rank for every group: the ranked call and the uniform call read the
    # same bytes and launch the same kernels, so their outputs agree bit for bit
    case = make_ranked_case(layer(), [256] * 4, [128] * 4, [300, 130])
    out_r, lse_r = run_ranked(case, num_splits=2)
    pools = build_ranked_pools(case)
    cfg = P.make_config(16, 128, 4, 256, 128, 128, case.w.rope_base, "bf16", "bf16")
    b = len(case.seq_lens)
    ws = torch.zeros(P.palu_decode_workspace_size(cfg, b, case.page_table.shape[1], 2), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((b, 16, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((b, 16), dtype=torch.float32, device="cuda")
    P.palu_decode_attn(cfg, case.q[:, 0].cuda(), torch.from_numpy(case.q_pos[:, 0].copy()).cuda(), pools["zk"],
                       pools["zv"], None, None, None, torch.from_numpy(case.page_table).cuda(),
                       torch.tensor(case.seq_lens, dtype=torch.int32, device="cuda"), case.num_pages,
                       case.B_k.cuda(), case.B_v.cuda(), out, lse, ws, 2)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(out.to(torch.float64).cpu().numpy(), out_r[:, 0])
    np.testing.assert_array_equal(lse.cpu().numpy(), lse_r[:, 0])


def exact_inputs(n, d_model, ncols_k, ncols_v, seed):
    """x on a dyadic grid and A a 0/1 column-selection matrix: x·A is exact in float32."""
    rng = np.random.default_rng(seed)
    x = (rng.integers(-24, 25, size=(n, d_model)) / 8.0).astype(np.float32)
    def sel(ncol):
        A = np.zeros((d_model, ncol), np.float32)
        A[rng.integers(0, d_model, size=ncol), np.arange(ncol)] = 1.0
        return torch.from_numpy(A).to(torch.bfloat16)
    return torch.from_numpy(x).to(torch.bfloat16), sel(ncols_k), sel(ncols_v)


@pytest.mark.parametrize("lat", ["bf16", "int4"])
def test_ranked_compress_append(lat):
    w = layer(latent_dtype=lat, d_model=512)
    ranks_k = [256, 512, 256, 256] if lat == "int4" else [64, 192, 128, 256]
    ranks_v = [256, 256, 512, 256] if lat == "int4" else [128, 64, 256, 128]
    cfg = P.make_config(16, 128, 4, ranks_k[0], ranks_v[0], 128, w.rope_base, "bf16", lat)
    n, d_model, num_pages = 300, w.d_model, 5
    if lat == "int4":
        # exactly representable latents: codes, bytes and scales match bit for bit
        x, A_k, A_v = exact_inputs(n, d_model, sum(ranks_k), sum(ranks_v), 3)
    else:
        x = normal_tensor(9, "x", (n, d_model), "bf16")
        A_k = normal_tensor(9, "A_k", (d_model, sum(ranks_k)), "bf16", 1 / math.sqrt(d_model))
        A_v = normal_tensor(9, "A_v", (d_model, sum(ranks_v)), "bf16", 1 / math.sqrt(d_model))
    slots = np.random.default_rng(5).choice(num_pages * 128, size=n, replace=False).astype(np.int32)
    slots[::17] = -1
    kb, vb, ksb, vsb, koff, voff = P.palu_cache_strides_ranked(cfg, ranks_k, ranks_v)
    layout = ranked_offsets(w, ranks_k, ranks_v)
    assert (kb, koff) == (layout["zk"][2], layout["zk"][1]) and (vb, voff) == (layout["zv"][2], layout["zv"][1])
    assert ksb == (layout["zks"][2] if lat == "int4" else 0)
    pools = {k: (torch.full((num_pages * sz,), 0xAB, dtype=torch.uint8, device="cuda") if sz else None)
             for k, sz in (("zk", kb), ("zv", vb), ("zks", ksb), ("zvs", vsb))}
    ws = torch.zeros(P.palu_compress_ranked_workspace_size(cfg, ranks_k, ranks_v, n, d_model), dtype=torch.uint8,
                     device="cuda")
    P.palu_compress_append_ranked(cfg, ranks_k, ranks_v, x.cuda(), A_k.cuda(), A_v.cuda(),
                                  torch.from_numpy(slots).cuda(), None, pools["zk"], pools["zv"], pools["zks"],
                                  pools["zvs"], None, num_pages, ws)
    torch.cuda.synchronize()
    assert P.palu_get_device_status(ws)[0] == 0
    xf = x.to(torch.float64).numpy()
    keep = slots >= 0
    for side, A, ranks in (("zk", A_k, ranks_k), ("zv", A_v, ranks_v)):
        rows, offs, page_bytes = layout[side]
        host = pools[side].cpu().numpy().reshape(num_pages, page_bytes)
        col0 = np.concatenate([[0], np.cumsum(ranks)])
        Af = A.to(torch.float64).numpy()
        if lat == "int4":
            srows, soffs, spage = layout[side + "s"]
            shost = pools[side + "s"].cpu().numpy().reshape(num_pages, spage)
        for g, r in enumerate(ranks):
            Ag = Af[:, col0[g]: col0[g + 1]]             # group g's columns of A
            blocks = [unswizzle_block(host[p, offs[g]: offs[g] + 128 * rows[g]], 128) for p in range(num_pages)]
            got = np.stack([blocks[s // 128][s % 128] for s in slots[keep]])
            if lat == "int4":
                packed, sc = O.quantize_int4(O.compress(xf, Ag, "f32")[keep].astype(np.float32))
                sgot = np.stack([shost[s // 128, soffs[g] + (s % 128) * srows[g]:][: r // 32 * 2]
                                 for s in slots[keep]])
                np.testing.assert_array_equal(got, packed)
                np.testing.assert_array_equal(sgot.copy().view(np.float16), sc)
            else:
                ref = O.compress(xf, Ag, "bf16")[keep]
                val = torch.from_numpy(got.copy()).view(torch.bfloat16).to(torch.float64).numpy()
                err = np.abs(val - ref)
                # within one rounding step of bf16 (float32 accumulation may cross a tie)
                assert np.all(err <= 2 ** -7 * np.abs(ref) + 1e-6 * np.abs(ref).max()), (side, g, float(err.max()))


def ranked_full_size(w, context, units, seed=321):
    """The ranked bench workload at full size on the GPU, in the bench's launch configuration
    (automatic split counts per decode set); the sampled (sequence, group) units come from the
    host generator and are checked against the oracle, the rest of the cache is N(0,1) noise."""
    from palu_testlib import swizzle_block
    from rank_kv_cache_palu_b200.synth import normal, page_permutation
    b, G, W, Pz = w.batch, w.groups, w.width, w.page_size
    rks, rvs = w.group_ranks
    cfg = P.make_config(w.num_heads, w.head_dim, w.group_size, w.rank_k, w.rank_v, Pz, w.rope_base,
                        w.act_dtype, w.latent_dtype)
    max_pages = (context + Pz - 1) // Pz
    num_pages = b * max_pages
    pt = page_permutation(seed, num_pages).reshape(b, max_pages)
    dev = torch.device("cuda")
    cache = P.LatentCache.allocate(cfg, num_pages, device=dev, ranks_k=rks, ranks_v=rvs)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    for pool in (cache.zk, cache.zv):
        view = pool.view(TORCH_DTYPE[w.latent_dtype])
        for i in range(0, view.numel(), 1 << 28):
            seg = view[i:i + (1 << 28)]
            seg.copy_(torch.randn(seg.shape, device=dev, generator=gen))
    layout = ranked_offsets(w, rks, rvs)
    host = {}
    for (bi, g) in units:
        for name, ranks, pool in (("zk", rks, cache.zk), ("zv", rvs, cache.zv)):
            r = ranks[g]
            rows_g, offs, page_bytes = layout[name]
            z = torch.from_numpy(normal(seed, name, (context, r), unit=(bi, g))).to(TORCH_DTYPE[w.latent_dtype])
            host[(name, bi, g)] = z.to(torch.float64).numpy()
            zb = z.view(torch.uint8).numpy()
            pages = pool.view(num_pages, page_bytes)
            for p in range(max_pages):
                t0, t1 = p * Pz, min(context, (p + 1) * Pz)
                rows = np.zeros((Pz, rows_g[g]), np.uint8)
                rows[: t1 - t0] = zb[t0:t1]
                pages[pt[bi, p], offs[g]: offs[g] + Pz * rows_g[g]].copy_(torch.from_numpy(swizzle_block(rows)).to(dev))
    q = normal_tensor(seed, "q", (b, 1, w.num_heads, w.head_dim), w.act_dtype)
    B_k = torch.cat([normal_tensor(seed, f"B_k{g}", (r, W), w.act_dtype, 1 / math.sqrt(r)) for g, r in enumerate(rks)])
    B_v = torch.cat([normal_tensor(seed, f"B_v{g}", (r, W), w.act_dtype, 1 / math.sqrt(r)) for g, r in enumerate(rvs)])
    ws = torch.zeros(P.palu_decode_ranked_workspace_size(cfg, rks, rvs, b, 1, max_pages, 0), dtype=torch.uint8,
                     device=dev)
    out = torch.empty((b, 1, w.num_heads, w.head_dim), dtype=TORCH_DTYPE[w.act_dtype], device=dev)
    lse = torch.empty((b, 1, w.num_heads), dtype=torch.float32, device=dev)
    q_pos = torch.full((b, 1), context - 1, dtype=torch.int32, device=dev)
    lens = torch.full((b,), context, dtype=torch.int32, device=dev)
    P.palu_decode_attn_ranked(cfg, rks, rvs, q.to(dev), q_pos, cache.zk, cache.zv, None, None, None,
                              torch.from_numpy(pt).to(dev), lens, num_pages, B_k.to(dev), B_v.to(dev), out, lse, ws, 0)
    torch.cuda.synchronize()
    assert P.palu_get_device_status(ws)[0] == 0
    got = out.to(torch.float64).cpu().numpy()
    qn = q.to(torch.float64).numpy()
    Bk_l = [t.to(torch.float64).numpy() for t in torch.split(B_k, list(rks))]
    Bv_l = [t.to(torch.float64).numpy() for t in torch.split(B_v, list(rvs))]
    worst = 0.0
    gs = w.group_size
    for (bi, g) in units:
        heads = slice(g * gs, (g + 1) * gs)
        ref, _ = O.decode_attention_ranked(qn[bi][:, heads], np.array([context - 1]), [host[("zk", bi, g)]],
                                           [host[("zv", bi, g)]], np.arange(context), [Bk_l[g]], [Bv_l[g]], gs,
                                           w.rope_base)
        err = rel_err(got[bi, 0, heads], ref[0])
        worst = max(worst, err)
        assert err <= TOL[w.act_dtype], f"unit ({bi},{g}): {err:.3e}"
    return worst


@pytest.mark.slow
@pytest.mark.parametrize("name", ["7b_bf16_ranked_b16_t16k", "7b_bf16_ranked_b16_t16k_norope"])
def test_ranked_full_size_sampled(name):
    # the ranked bench workloads (16 x 16k + a ragged page), one sampled unit per key / value rank
    w = WORKLOADS[name]
    worst = ranked_full_size(w, w.context + 9, [(0, 0), (5, 1), (9, 3), (15, 6)])
    print(f"{name}: worst rel err {worst:.2e}")
