"""The allocation-free decode entry point against the regular one.

palu_decode_attn_noalloc serves callers that cannot call cudaMalloc (a host
framework that owns all device memory, a fixed device-memory budget, a path
that must not pay for an allocation): it keeps the decode workspace in a fixed
array of device memory inside the library.  It runs the same kernels with the
same split count on the same bytes as palu_decode_attn with a caller
workspace, so its results must be identical bit for bit, call after call,
whatever an earlier call left in the shared array.
"""
import dataclasses

import numpy as np
import pytest
import torch

from palu_testlib import build_pools, make_decode_case
from rank_kv_cache_palu_b200 import api as P
from rank_kv_cache_palu_b200.synth import TORCH_DTYPE, WORKLOADS

pytestmark = pytest.mark.gpu


def _inputs(case, page_table=None):
    dev = "cuda"
    pools = build_pools(case)
    pt = case.page_table if page_table is None else page_table
    return dict(q=case.q.to(dev), q_pos=torch.from_numpy(case.q_pos).to(dev), pools=pools,
                page_table=torch.from_numpy(pt).to(dev),
                seq_lens=torch.tensor(case.seq_lens, dtype=torch.int32, device=dev),
                B_k=case.B_k.to(dev), B_v=case.B_v.to(dev))


def _outputs(case):
    w = case.w
    b = len(case.seq_lens)
    return (torch.full((b, w.num_heads, w.head_dim), float("nan"), dtype=TORCH_DTYPE[w.act_dtype], device="cuda"),
            torch.full((b, w.num_heads), float("nan"), dtype=torch.float32, device="cuda"))


def _with_workspace(case, x):
    cfg = case.cfg
    out, lse = _outputs(case)
    ws = torch.zeros(P.palu_decode_workspace_size(cfg, len(case.seq_lens), case.page_table.shape[1]),
                     dtype=torch.uint8, device="cuda")
    p = x["pools"]
    P.palu_decode_attn(cfg, x["q"], x["q_pos"], p["zk"], p["zv"], p["zks"], p["zvs"], p["pos"],
                       x["page_table"], x["seq_lens"], case.num_pages, x["B_k"], x["B_v"], out, lse, ws)
    torch.cuda.synchronize()
    assert P.palu_get_device_status(ws)[0] == 0
    return out.cpu(), lse.cpu()


def _no_alloc(case, x, report_status):
    cfg = case.cfg
    out, lse = _outputs(case)
    p = x["pools"]
    P.palu_decode_attn_noalloc(cfg, x["q"], x["q_pos"], p["zk"], p["zv"], p["zks"], p["zvs"], p["pos"],
                               x["page_table"], x["seq_lens"], case.num_pages, x["B_k"], x["B_v"], out,
                               lse, report_status=report_status)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu()


def _same(got, ref, what):
    for g, r, name in zip(got, ref, ("out", "lse")):
        assert torch.equal(g.view(torch.uint8) if g.dtype != torch.float32 else g.view(torch.int32),
                           r.view(torch.uint8) if r.dtype != torch.float32 else r.view(torch.int32)), \
            f"{what}: {name} differs from palu_decode_attn"


def _cases(kind):
    if kind == "tensor_core_bf16":
        w = dataclasses.replace(WORKLOADS["7b_bf16_r256v128_b1_t4k"], num_heads=8)
        return make_decode_case(w, [300, 1, 1000, 129]), make_decode_case(w, [640, 77], seed=9)
    w = WORKLOADS["tiny_f32"]
    return make_decode_case(w, [256, 77]), make_decode_case(w, [500, 3, 128], seed=9)


@pytest.mark.parametrize("kind", ["tensor_core_bf16", "cuda_core_f32"])
def test_no_alloc_matches_workspace_entry_point_bit_for_bit(kind):
    case, other = _cases(kind)
    x, xo = _inputs(case), _inputs(other)
    ref, ref_other = _with_workspace(case, x), _with_workspace(other, xo)
    _same(_no_alloc(case, x, False), ref, "first call")
    # a call with another batch in between leaves other partials in the shared array
    _same(_no_alloc(other, xo, True), ref_other, "call with another batch")
    _same(_no_alloc(case, x, True), ref, "call after it")


def test_no_alloc_clears_an_earlier_calls_device_status():
    # A call with a page entry past the pool (the kernels skip it and record
    # PALU_ERR_DEVICE_BOUNDS in the shared status word) that does not read the
    # status back, then a valid call that does: it must see only its own status.
    case, _ = _cases("tensor_core_bf16")
    bad = case.page_table.copy()
    bad[0, 1] = case.num_pages + 3
    xb, x = _inputs(case, bad), _inputs(case)
    ref = _with_workspace(case, x)
    _no_alloc(case, xb, False)
    _same(_no_alloc(case, x, True), ref, "valid call after a faulty one")
    with pytest.raises(P.PaluError) as e:
        _no_alloc(case, xb, True)
    assert e.value.status == 7                       # PALU_ERR_DEVICE_BOUNDS, reported when asked


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
