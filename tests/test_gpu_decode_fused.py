"""GPU parity of the fused decode path (attention without RoPE: B_k folded into
the query, scores taken on the cached latents) against the CPU oracle, through
the C ABI.  The oracle materialises K and V in full, so agreement also checks
the fold q·(z_k B_k)ᵀ = (q B_kᵀ)·z_kᵀ on real data."""
import dataclasses

import numpy as np
import pytest
import torch

from palu_testlib import TOL, build_pools, make_decode_case, oracle_decode, rel_err, run_gpu_decode
from rank_kv_cache_palu_b200 import api as P
from rank_kv_cache_palu_b200.synth import WORKLOADS

pytestmark = pytest.mark.gpu

import test_gpu_decode_tc as tc   # noqa: E402  (shared checks and the full-size sampler)


def norope(dt="bf16", r_k=256, r_v=128, gs=4, H=8):
    return dataclasses.replace(WORKLOADS["7b_bf16_r256v128_b1_t4k"], act_dtype=dt, latent_dtype=dt,
                               rank_k=r_k, rank_v=r_v, group_size=gs, num_heads=H, rope_base=0.0)


def test_fused_path_is_selected():
    assert P.palu_decode_kernel_kind(make_decode_case(norope(), [10]).cfg) == 3
    assert P.palu_decode_kernel_kind(make_decode_case(tc.small_7b(), [10]).cfg) == 2


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("r_v", [128, 256])
def test_fused_ragged_batch_and_splits(dt, r_v):
    case = make_decode_case(norope(dt, r_v=r_v), [300, 1, 1000, 129, 0, 128, 640])
    tc.check(case)
    tc.check(case, num_splits=3)


@pytest.mark.parametrize("r_k", [64, 128, 512])
def test_fused_key_ranks(r_k):
    tc.check(make_decode_case(norope(r_k=r_k), [700, 65]))


def test_fused_group_size_two_and_peaky_query():
    tc.check(make_decode_case(norope(gs=2), [513, 40], q_scale=4.0))


def test_fused_nan_in_unused_page_rows_is_ignored():
    # the tail of a sequence's last page may hold anything (here NaN); only the
    # valid rows may influence the result
    w = norope()
    case = make_decode_case(w, [200])
    pools = build_pools(case)
    G, Pz = w.groups, w.page_size
    last_page = int(case.page_table[0, 1])
    nan = np.frombuffer(np.array([np.nan], np.float32).tobytes()[2:], np.uint8)  # bf16 NaN
    for name, r in (("zk", w.rank_k), ("zv", w.rank_v)):
        blocks = pools[name].view(case.num_pages, G, Pz * r * 2)
        for g in range(G):
            rows = tc.unswizzle_block(blocks[last_page, g].cpu().numpy(), Pz).copy()
            rows[200 - Pz:, 0::2] = nan[0]
            rows[200 - Pz:, 1::2] = nan[1]
            blocks[last_page, g] = torch.from_numpy(tc.swizzle_block(rows)).cuda()
    out, _ = run_gpu_decode(case, 1, pools=pools)
    ref, _ = oracle_decode(case, 0)
    assert np.all(np.isfinite(out))
    assert rel_err(out[0], ref) <= TOL["bf16"]


def test_fused_bad_page_reports_bounds():
    case = make_decode_case(norope(), [300])
    pools = build_pools(case)
    cfg = case.cfg
    bad = case.page_table.copy()
    bad[0, 1] = case.num_pages + 5
    ws = torch.zeros(P.palu_decode_workspace_size(cfg, 1, bad.shape[1], 1), dtype=torch.uint8, device="cuda")
    out = torch.empty((1, case.w.num_heads, 128), dtype=torch.bfloat16, device="cuda")
    P.palu_decode_attn(cfg, case.q.cuda(), torch.from_numpy(case.q_pos).cuda(), pools["zk"], pools["zv"],
                       None, None, None, torch.from_numpy(bad).cuda(),
                       torch.tensor(case.seq_lens, dtype=torch.int32).cuda(), case.num_pages,
                       case.B_k.cuda(), case.B_v.cuda(), out, None, ws, 1)
    st, _ = P.palu_get_device_status(ws)
    assert st == 7


@pytest.mark.slow
def test_full_size_7b_bf16_b16_t16k_norope_sampled():
    w = WORKLOADS["7b_bf16_r256v128_b16_t16k_norope"]
    worst, S = tc.sampled_full_size(w, w.context + 5, [(0, 0), (9, 5), (15, 7)])
    print(f"no-RoPE 16k x 16 (S={S}): worst rel err {worst:.2e}")
