"""GPU parity of the multi-token decode step (several queries per sequence,
causal by position) against the CPU oracle, through the C ABI, on every
decode path: tensor-core RoPE kernel, fused no-RoPE kernel, int4 latents and
the CUDA-core kernel."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import palu_oracle as O
from palu_testlib import TOL, build_pools, make_decode_case, rel_err
from rank_kv_cache_palu_b200 import api as P
from rank_kv_cache_palu_b200.synth import TORCH_DTYPE, WORKLOADS, normal_tensor

pytestmark = pytest.mark.gpu


def run_multi(case, q, q_pos, num_splits=0):
    w = case.w
    cfg = case.cfg
    pools = build_pools(case)
    b, nq = q.shape[0], q.shape[1]
    dev = "cuda"
    ws = torch.zeros(P.palu_decode_multi_workspace_size(cfg, b, nq, case.page_table.shape[1], num_splits),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((b, nq, w.num_heads, w.head_dim), dtype=TORCH_DTYPE[w.act_dtype], device=dev)
    lse = torch.empty((b, nq, w.num_heads), dtype=torch.float32, device=dev)
    P.palu_decode_attn_multi(cfg, q.to(dev), torch.from_numpy(q_pos).to(dev), pools["zk"], pools["zv"],
                             pools["zks"], pools["zvs"], pools["pos"], torch.from_numpy(case.page_table).to(dev),
                             torch.tensor(case.seq_lens, dtype=torch.int32, device=dev), case.num_pages,
                             case.B_k.to(dev), case.B_v.to(dev), out, lse, ws, num_splits)
    torch.cuda.synchronize()
    st, detail = P.palu_get_device_status(ws)
    assert st == 0, f"device status {st} ({detail})"
    return out.to(torch.float64).cpu().numpy(), lse.cpu().numpy()


def check_multi(case, nq, num_splits=0, q_pos=None):
    w = case.w
    b = len(case.seq_lens)
    q = normal_tensor(w.seed, "q_multi", (b, nq, w.num_heads, w.head_dim), w.act_dtype)
    if q_pos is None:
        # the last nq cached tokens are the new ones
        q_pos = np.array([[int(case.positions(i)[max(T - nq + j, 0)]) if T else j for j in range(nq)]
                          for i, T in enumerate(case.seq_lens)], np.int32)
    out, lse = run_multi(case, q, q_pos, num_splits)
    qn = q.to(torch.float64).numpy()
    Bk, Bv = case.B_k.to(torch.float64).numpy(), case.B_v.to(torch.float64).numpy()
    for i, T in enumerate(case.seq_lens):
        zk, zv = case.oracle_latents(i)
        ref, ref_lse = O.decode_attention_multi(qn[i], q_pos[i], zk, zv, case.positions(i), Bk, Bv,
                                                w.group_size, w.rope_base)
        for j in range(nq):
            if np.isneginf(ref_lse[j]).all():
                assert np.all(out[i, j] == 0) and np.all(np.isneginf(lse[i, j]))
                continue
            err = rel_err(out[i, j], ref[j])
            assert err <= TOL[w.act_dtype], f"seq {i} query {j}: rel err {err:.3e}"
            np.testing.assert_allclose(lse[i, j], ref_lse[j], rtol=0, atol=2e-2)


def bf16_7b(**kw):
    return dataclasses.replace(WORKLOADS["7b_bf16_r256v128_b1_t4k"], num_heads=8, **kw)


@pytest.mark.parametrize("nq", [1, 4])
def test_multi_tensor_core_rope(nq):
    case = make_decode_case(bf16_7b(), [300, 130, 1000, 5])
    assert P.palu_decode_kernel_kind(case.cfg) == 2
    check_multi(case, nq)
    check_multi(case, nq, num_splits=3)


@pytest.mark.parametrize("nq", [2, 3, 5, 8])
def test_multi_fused_no_rope(nq):
    # the fused kernel serves 4, 2 or 1 queries per pass over the cache
    case = make_decode_case(bf16_7b(rope_base=0.0), [300, 130, 1000, 5])
    assert P.palu_decode_kernel_kind(case.cfg) == 3
    check_multi(case, nq)
    check_multi(case, nq, num_splits=3)


def test_multi_fused_rank_v_256_explicit_positions():
    w = dataclasses.replace(bf16_7b(rope_base=0.0), rank_v=256, act_dtype="f16", latent_dtype="f16")
    check_multi(make_decode_case(w, [700, 129], explicit_positions=True), 4)


def test_multi_int4():
    w = dataclasses.replace(WORKLOADS["7b_int4_r256_b8_t32k"], num_heads=8)
    check_multi(make_decode_case(w, [520, 129]), 3)


def test_multi_cuda_core_f32_explicit_positions():
    case = make_decode_case(WORKLOADS["tiny_f32"], [256, 77], explicit_positions=True)
    assert P.palu_decode_kernel_kind(case.cfg) == 1
    check_multi(case, 5)


def test_multi_query_before_every_token_sees_nothing():
    case = make_decode_case(bf16_7b(), [200])
    check_multi(case, 2, q_pos=np.array([[-5, 150]], np.int32))
