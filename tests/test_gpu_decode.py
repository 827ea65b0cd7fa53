"""GPU parity of palu_decode_attn against the CPU oracle, through the C ABI."""
import dataclasses

import numpy as np
import pytest
import torch

from palu_testlib import TOL, build_pools, make_decode_case, oracle_decode, rel_err, run_gpu_decode
from rank_kv_cache_palu_b200 import api as P
from rank_kv_cache_palu_b200.synth import WORKLOADS

pytestmark = pytest.mark.gpu


def check_case(case, num_splits=0, heads=None, seqs=None, tol=None):
    out, lse = run_gpu_decode(case, num_splits)
    seqs = range(len(case.seq_lens)) if seqs is None else seqs
    tol = TOL[case.w.act_dtype] if tol is None else tol
    worst = 0.0
    for b in seqs:
        hs = list(range(case.w.num_heads)) if heads is None else heads
        ref, ref_lse = oracle_decode(case, b, hs)
        if case.seq_lens[b] == 0:
            assert np.all(out[b][hs] == 0) and np.all(np.isneginf(lse[b][hs]))
            continue
        err = rel_err(out[b][hs], ref)
        worst = max(worst, err)
        assert err <= tol, f"seq {b}: rel err {err:.3e} > {tol}"
        np.testing.assert_allclose(lse[b][hs], ref_lse, rtol=0, atol=5e-3 if tol > 1e-3 else 1e-4)
    return worst


def test_tiny_f32_config():
    # the fp32 oracle case: batch 1, 8 heads of 64, groups of 4, rank 64/64, context 256
    w = WORKLOADS["tiny_f32"]
    case = make_decode_case(w, [w.context])
    err = check_case(case, num_splits=1)
    assert err <= 1e-4
    check_case(case)                                   # automatic split count


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_ragged_batch_shuffled_pages(dt):
    w = dataclasses.replace(WORKLOADS["tiny_f32"], act_dtype=dt, latent_dtype=dt, rank_k=64, rank_v=64)
    case = make_decode_case(w, [1, 127, 128, 129, 300, 0, 1000])
    for s in (1, 3, 0):
        check_case(case, num_splits=s)


@pytest.mark.parametrize("dt", ["f32", "bf16"])
def test_explicit_positions_and_peaky_query(dt):
    w = dataclasses.replace(WORKLOADS["tiny_f32"], act_dtype=dt, latent_dtype=dt)
    case = make_decode_case(w, [200, 513], explicit_positions=True, q_scale=8.0)
    check_case(case, num_splits=2)


def test_large_positions_rope():
    # positions near 60k exercise the angle reduction at large arguments
    w = dataclasses.replace(WORKLOADS["tiny_f32"])
    case = make_decode_case(w, [256])
    case.pos = [np.arange(60000, 60256, dtype=np.int32)]
    case.q_pos = np.array([60300], np.int32)
    check_case(case)


def test_no_rope():
    w = dataclasses.replace(WORKLOADS["tiny_f32"], rope_base=0.0)
    check_case(make_decode_case(w, [77, 300]))


def test_split_count_independence_f32():
    w = WORKLOADS["tiny_f32"]
    case = make_decode_case(w, [1000, 555])
    pools = build_pools(case)
    outs = []
    for s in (1, 2, 4, 8):
        o, _ = run_gpu_decode(case, s, pools=pools)
        outs.append(o)
    for o in outs[1:]:
        assert np.max(np.abs(o - outs[0])) <= 1e-5 * np.max(np.abs(outs[0]))


def test_7b_f16_full_size():
    # Llama-2-7B-shaped layer, fp16, rank 256/256, batch 1, context 4096: every head
    w = WORKLOADS["7b_f16_r256_b1_t4k"]
    check_case(make_decode_case(w, [w.context]))


def test_bad_page_index_reports_bounds():
    # a page index past the pool: the kernel skips the access and records the fault
    w = WORKLOADS["tiny_f32"]
    case = make_decode_case(w, [300])
    pools = build_pools(case)
    bad = case.page_table.copy()
    bad[0, 1] = case.num_pages + 5
    cfg = case.cfg
    ws = torch.zeros(P.palu_decode_workspace_size(cfg, 1, bad.shape[1], 1), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty((1, w.num_heads, w.head_dim), dtype=torch.float32, device="cuda")
    P.palu_decode_attn(cfg, case.q.cuda(), torch.from_numpy(case.q_pos).cuda(), pools["zk"],
                       pools["zv"], None, None, None, torch.from_numpy(bad).cuda(),
                       torch.tensor(case.seq_lens, dtype=torch.int32).cuda(), case.num_pages,
                       case.B_k.cuda(), case.B_v.cuda(), out, None, ws, 1)
    st, _ = P.palu_get_device_status(ws)
    assert st == 7                                      # PALU_ERR_DEVICE_BOUNDS
    st2, _ = P.palu_get_device_status(ws)               # reading cleared it
    assert st2 == 0


@pytest.mark.parametrize("act", ["f16", "bf16"])
def test_int4_cuda_core_path(act):
    # head_dim 64 is not a tensor-core shape: int4 latents through the CUDA-core split kernel
    w = dataclasses.replace(WORKLOADS["tiny_f32"], act_dtype=act, latent_dtype="int4", rank_k=256,
                            rank_v=256)
    case = make_decode_case(w, [256, 77, 300, 0])
    assert P.palu_decode_kernel_kind(case.cfg) == 1
    out, lse = run_gpu_decode(case)
    for b, T in enumerate(case.seq_lens):
        if T == 0:
            assert np.all(out[b] == 0) and np.all(np.isneginf(lse[b]))
            continue
        ref, ref_lse = oracle_decode(case, b)
        assert rel_err(out[b], ref) <= TOL[act]
        np.testing.assert_allclose(lse[b], ref_lse, rtol=0, atol=2e-2)
