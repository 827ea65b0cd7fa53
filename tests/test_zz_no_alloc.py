"""The allocation-free decode entry point against the regular one.

palu_decode_attn_noalloc serves callers that cannot call cudaMalloc (a host
framework that owns all device memory, a fixed device-memory budget, a path
that must not pay for an allocation): it keeps the decode workspace in a fixed
array of device memory inside the library.  These tests call it through the
C ABI twice in a row and check both results against palu_decode_attn with a
caller workspace, within the parity tolerance the decode tests use.
"""
import dataclasses

import numpy as np
import pytest
import torch

from palu_testlib import TOL, build_pools, make_decode_case, rel_err
from rank_kv_cache_palu_b200 import api as P
from rank_kv_cache_palu_b200.synth import TORCH_DTYPE, WORKLOADS

pytestmark = pytest.mark.gpu


def _inputs(case):
    dev = "cuda"
    pools = build_pools(case)
    return dict(q=case.q.to(dev), q_pos=torch.from_numpy(case.q_pos).to(dev), pools=pools,
                page_table=torch.from_numpy(case.page_table).to(dev),
                seq_lens=torch.tensor(case.seq_lens, dtype=torch.int32, device=dev),
                B_k=case.B_k.to(dev), B_v=case.B_v.to(dev))


def _outputs(case):
    w = case.w
    b = len(case.seq_lens)
    return (torch.empty((b, w.num_heads, w.head_dim), dtype=TORCH_DTYPE[w.act_dtype], device="cuda"),
            torch.empty((b, w.num_heads), dtype=torch.float32, device="cuda"))


def _with_workspace(case, x):
    cfg = case.cfg
    out, lse = _outputs(case)
    ws = torch.zeros(P.palu_decode_workspace_size(cfg, len(case.seq_lens), case.page_table.shape[1]),
                     dtype=torch.uint8, device="cuda")
    p = x["pools"]
    P.palu_decode_attn(cfg, x["q"], x["q_pos"], p["zk"], p["zv"], p["zks"], p["zvs"], p["pos"],
                       x["page_table"], x["seq_lens"], case.num_pages, x["B_k"], x["B_v"], out, lse, ws)
    torch.cuda.synchronize()
    return out.to(torch.float64).cpu().numpy(), lse.cpu().numpy()


def _no_alloc(case, x, report_status):
    cfg = case.cfg
    out, lse = _outputs(case)
    p = x["pools"]
    P.palu_decode_attn_noalloc(cfg, x["q"], x["q_pos"], p["zk"], p["zv"], p["zks"], p["zvs"], p["pos"],
                               x["page_table"], x["seq_lens"], case.num_pages, x["B_k"], x["B_v"], out,
                               lse, report_status=report_status)
    torch.cuda.synchronize()
    return out.to(torch.float64).cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("kind", ["tensor_core_bf16", "cuda_core_f32"])
def test_no_alloc_matches_workspace_entry_point_twice(kind):
    if kind == "tensor_core_bf16":
        w = dataclasses.replace(WORKLOADS["7b_bf16_r256v128_b1_t4k"], num_heads=8)
        case = make_decode_case(w, [300, 1, 1000, 129])
    else:
        w = WORKLOADS["tiny_f32"]
        case = make_decode_case(w, [256, 77])
    x = _inputs(case)
    ref, ref_lse = _with_workspace(case, x)
    tol = TOL[w.act_dtype]
    for call, report in enumerate((False, True)):
        got, got_lse = _no_alloc(case, x, report)
        assert rel_err(got, ref) <= tol, f"call {call}: {rel_err(got, ref):.3e}"
        np.testing.assert_allclose(got_lse, ref_lse, rtol=0, atol=1e-4)


def test_no_alloc_rejects_workspace_beyond_the_array():
    w = dataclasses.replace(WORKLOADS["7b_bf16_r256_b32_t16k"], batch=64)
    cfg = P.make_config(w.num_heads, w.head_dim, w.group_size, w.rank_k, w.rank_v, 128, 10000.0,
                        "bf16", "bf16")
    max_pages, splits = 256, 64
    assert P.palu_decode_workspace_size(cfg, 64, max_pages, splits) > P.NOALLOC_SCRATCH_BYTES
    d = torch.zeros(16, dtype=torch.uint8, device="cuda")
    t = torch.zeros((64, max_pages), dtype=torch.int32, device="cuda")
    v = torch.zeros(64, dtype=torch.int32, device="cuda")
    q = torch.zeros((64, 32, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(P.PaluError) as e:
        P.palu_decode_attn_noalloc(cfg, q, v, d, d, None, None, None, t, v, 1, d, d, q, None,
                                   num_splits=splits)
    assert e.value.status == 4   # PALU_ERR_WORKSPACE, before anything is launched
