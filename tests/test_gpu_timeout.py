"""The kernels' timeout path, exercised without a GPU fault.

Every wait inside the tensor-core kernels is bounded.  When a bound runs out the
kernel records PALU_ERR_DEVICE_TIMEOUT in the workspace status word, waits
(with a bound of its own) for the copies and MMAs it has already issued, frees
its tensor memory and returns, so the context stays usable.  These tests make a
wait run out on purpose through the library's test hook (a short bound, and
an MMA thread that first waits on a barrier phase nothing completes before its
own teardown), read the status back, restore normal operation and run the same
case again in the same process to parity.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

from palu_testlib import TOL, build_pools, make_decode_case, oracle_decode, rel_err, run_gpu_decode
from rank_kv_cache_palu_b200 import api as P
from rank_kv_cache_palu_b200.synth import TORCH_DTYPE, WORKLOADS, normal_tensor

pytestmark = pytest.mark.gpu

SHORT_WAIT = 1 << 20          # SM cycles, about half a millisecond


def _decode_case(kind):
    if kind == "rope_bf16":
        w = dataclasses.replace(WORKLOADS["7b_bf16_r256v128_b1_t4k"], num_heads=8)
    elif kind == "rope_int4":
        w = dataclasses.replace(WORKLOADS["7b_int4_r256_b8_t32k"], num_heads=8)
    else:
        w = dataclasses.replace(WORKLOADS["7b_bf16_r256v128_b16_t16k_norope"], num_heads=8)
    case = make_decode_case(w, [300, 1000, 129])
    assert P.palu_decode_kernel_kind(case.cfg) == (3 if kind == "norope" else 2)
    return case


@pytest.mark.parametrize("kind", ["rope_bf16", "rope_int4", "norope"])
def test_decode_timeout_reports_and_recovers(kind):
    case = _decode_case(kind)
    pools = build_pools(case)
    w = case.w
    b = len(case.seq_lens)
    ws = torch.zeros(P.palu_decode_workspace_size(case.cfg, b, case.page_table.shape[1], 2),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty((b, w.num_heads, w.head_dim), dtype=TORCH_DTYPE[w.act_dtype], device="cuda")
    P.palu_debug_timeout_test(SHORT_WAIT, stall=True)
    try:
        P.palu_decode_attn(case.cfg, case.q.cuda(), torch.from_numpy(case.q_pos).cuda(), pools["zk"], pools["zv"],
                           pools["zks"], pools["zvs"], pools["pos"], torch.from_numpy(case.page_table).cuda(),
                           torch.tensor(case.seq_lens, dtype=torch.int32, device="cuda"), case.num_pages,
                           case.B_k.cuda(), case.B_v.cuda(), out, None, ws, 2)
    finally:
        P.palu_debug_timeout_test()
    st, detail = P.palu_get_device_status(ws)
    assert st == 6, f"expected PALU_ERR_DEVICE_TIMEOUT, got {st} (detail {detail})"
    assert detail < 90000, f"a teardown drain ran out too (detail {detail})"
    # the same case, same process, normal bounds: parity with the oracle
    got, lse = run_gpu_decode(case, pools=pools)
    for i in range(b):
        ref, _ = oracle_decode(case, i)
        assert rel_err(got[i], ref) <= TOL[w.act_dtype]


def _compress_inputs(n):
    w = WORKLOADS["7b_bf16_r256_b32_t16k"]
    cfg = P.make_config(w.num_heads, w.head_dim, w.group_size, w.rank_k, w.rank_v, w.page_size, w.rope_base,
                        w.act_dtype, w.latent_dtype)
    x = normal_tensor(3, "x", (n, w.d_model), "bf16").cuda()
    A_k = normal_tensor(3, "A_k", (w.d_model, w.groups * w.rank_k), "bf16", 1 / math.sqrt(w.d_model)).cuda()
    A_v = normal_tensor(3, "A_v", (w.d_model, w.groups * w.rank_v), "bf16", 1 / math.sqrt(w.d_model)).cuda()
    num_pages = (n + w.page_size - 1) // w.page_size + 1
    slots = torch.from_numpy(np.random.default_rng(n).permutation(num_pages * w.page_size)[:n].astype(np.int32)).cuda()
    return cfg, x, A_k, A_v, slots, num_pages


def _compress(cfg, x, A_k, A_v, slots, num_pages, ws):
    cache = P.LatentCache.allocate(cfg, num_pages, fill=0)
    P.palu_compress_append(cfg, x, A_k, A_v, slots, None, cache.zk, cache.zv, cache.zks, cache.zvs, None,
                           num_pages, ws)
    torch.cuda.synchronize()
    return cache


@pytest.mark.parametrize("n", [16, 1024])      # K-split append kernel; persistent prefill kernel
def test_compress_timeout_reports_and_recovers(n):
    cfg, x, A_k, A_v, slots, num_pages = _compress_inputs(n)
    ws_bytes = P.palu_compress_workspace_size(cfg, n, x.shape[1])
    clean = _compress(cfg, x, A_k, A_v, slots, num_pages, torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda"))
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    P.palu_debug_timeout_test(SHORT_WAIT, stall=True)
    try:
        _compress(cfg, x, A_k, A_v, slots, num_pages, ws)
    finally:
        P.palu_debug_timeout_test()
    st, detail = P.palu_get_device_status(ws)
    assert st == 6, f"expected PALU_ERR_DEVICE_TIMEOUT, got {st} (detail {detail})"
    assert detail < 90000, f"a teardown drain ran out too (detail {detail})"
    ws.zero_()                                   # a workspace is zero-filled again after a timeout
    again = _compress(cfg, x, A_k, A_v, slots, num_pages, ws)
    assert P.palu_get_device_status(ws)[0] == 0
    assert torch.equal(again.zk, clean.zk) and torch.equal(again.zv, clean.zv)
