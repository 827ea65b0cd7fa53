"""The C-ABI library loads, exports every symbol the header declares, and its
host-side argument checks return the documented statuses.  CPU only: none of
these calls reaches a kernel launch."""
import ctypes
import os
import re

import pytest

from rank_kv_cache_palu_b200 import api as P
from rank_kv_cache_palu_b200._lib import LIB_PATH, SIGNATURES, PaluConfig, load

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "palu.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(palu_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(LIB_PATH)
    names = declared_symbols()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), f"{n} declared in palu.h but not exported"
        assert n in SIGNATURES, f"{n} has no binding signature"


def cfg(**kw):
    base = dict(num_heads=32, head_dim=128, group_size=4, rank_k=256, rank_v=128, page_size=128,
                rope_base=10000.0, act_dtype="bf16", latent_dtype=None)
    base.update(kw)
    return P.make_config(**base)


def status_of(fn, *args):
    return int(fn(*args))


def test_cache_strides():
    assert P.palu_cache_strides(cfg()) == (8 * 128 * 512, 8 * 128 * 256, 0, 0)
    k, v, ks, vs = P.palu_cache_strides(cfg(act_dtype="f16", latent_dtype="int4", rank_v=256))
    assert (k, v) == (8 * 128 * 128, 8 * 128 * 128)
    assert ks == vs == 8 * 128 * 16            # 8 fp16 scales per 256-entry row, 16-byte padded


@pytest.mark.parametrize("bad,code", [
    (dict(num_heads=30), 1),                  # not a multiple of the group size
    (dict(head_dim=0), 1),
    (dict(head_dim=127), 1),                  # odd head_dim
    (dict(rope_base=-1.0), 1),
    (dict(act_dtype="f32", latent_dtype="bf16"), 2),
    (dict(act_dtype="f32", latent_dtype="int4"), 2),
    (dict(head_dim=256), 2),
    (dict(rank_k=100), 3),                    # 16-byte rows need r % 8 == 0
    (dict(act_dtype="f16", latent_dtype="int4", rank_k=48), 3),
])
def test_config_validation(bad, code):
    lib = load()
    k = ctypes.c_size_t()
    c = cfg(**bad)
    assert lib.palu_cache_strides(ctypes.byref(c), ctypes.byref(k), None, None, None) == code


def test_workspace_size_and_splits():
    c = cfg()
    S = P.palu_decode_num_splits(c, 16, 128)
    assert 1 <= S <= 128
    ws = P.palu_decode_workspace_size(c, 16, 128, S)
    assert ws >= 256 + 16 * 32 * S * (128 + 2) * 4
    assert ws % 256 == 0
    assert P.palu_decode_num_splits(c, 1, 1) == 1
    assert P.palu_compress_workspace_size(c, 32, 4096) >= 256


def test_decode_rejects_missing_workspace_before_launch():
    lib = load()
    c = cfg()
    st = lib.palu_decode_attn(ctypes.byref(c), 1, None, None, None, None, None, None, None, None, 4,
                              None, 8, None, None, None, None, None, 0, 0, None)
    assert st == 4  # PALU_ERR_WORKSPACE


def test_decode_rejects_too_many_splits():
    lib = load()
    c = cfg()
    st = lib.palu_decode_attn(ctypes.byref(c), 1, None, None, None, None, None, None, None, None, 4,
                              None, 8, None, None, None, None, None, 1 << 20, 5, None)
    assert st == 1  # more splits than pages


def test_decode_rejects_null_and_misaligned_pointers():
    lib = load()
    c = cfg()
    ws = ctypes.create_string_buffer((1 << 20) + 512)
    base = (ctypes.addressof(ws) + 255) // 256 * 256
    st = lib.palu_decode_attn(ctypes.byref(c), 1, None, None, None, None, None, None, None, None, 4,
                              None, 8, None, None, None, None, base, 1 << 20, 1, None)
    assert st == 1  # NULL q etc.
    p = base + 8   # not 16-byte aligned
    st = lib.palu_decode_attn(ctypes.byref(c), 1, p, p, p, p, None, None, None, p, 4, p, 8, p, p,
                              p, None, base, 1 << 20, 1, None)
    assert st == 3  # PALU_ERR_ALIGNMENT


def test_compress_rejects_bad_arguments():
    lib = load()
    c = cfg()
    ws = ctypes.create_string_buffer(4096)
    base = (ctypes.addressof(ws) + 255) // 256 * 256
    assert lib.palu_compress_append(ctypes.byref(c), 4, 100, None, None, None, None, None, None, None,
                                    None, None, None, 1, base, 1024, None) == 2   # d_model % 64
    assert lib.palu_compress_append(ctypes.byref(c), 4, 128, None, None, None, None, None, None, None,
                                    None, None, None, 1, None, 0, None) == 4      # no workspace
    assert lib.palu_compress_append(ctypes.byref(c), 0, 128, None, None, None, None, None, None, None,
                                    None, None, None, 1, base, 1024, None) == 0   # nothing to do
    assert lib.palu_compress_append(ctypes.byref(c), 4, 128, None, None, None, None, None, None, None,
                                    None, None, None, 1, base, 1024, None) == 1   # NULL inputs


def test_status_strings():
    lib = load()
    for s in range(8):
        assert lib.palu_status_string(s)
    assert P.palu_kernel_launches() >= 0


def test_product_path_does_not_import_oracle():
    import rank_kv_cache_palu_b200
    pkg = os.path.dirname(rank_kv_cache_palu_b200.__file__)
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(root, f), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_tensor_core_kernel_fits_every_7b_workload():
    # host-side check (no GPU): the tensor-core split kernel's shared-memory
    # layout fits for every 7B-shaped workload, int4 latents included (the
    # fused kernel for the workloads without RoPE)
    from rank_kv_cache_palu_b200.synth import WORKLOADS
    for w in WORKLOADS.values():
        if w.head_dim != 128:
            continue
        c = P.make_config(w.num_heads, w.head_dim, w.group_size, w.rank_k, w.rank_v, w.page_size,
                          w.rope_base, w.act_dtype, w.latent_dtype)
        assert P.palu_decode_kernel_kind(c) == (3 if w.rope_base == 0 else 2), w.name


def test_fused_path_selected_without_rope():
    # host-side: attention without RoPE takes the fused (latent-space) kernel,
    # whose workspace also holds the folded queries
    c = cfg(rope_base=0.0)
    assert P.palu_decode_kernel_kind(c) == 3
    assert P.palu_decode_kernel_kind(cfg()) == 2
    S = P.palu_decode_num_splits(c, 16, 128)
    assert P.palu_decode_workspace_size(c, 16, 128, S) >= 256 + 16 * 32 * S * 130 * 4 + 16 * 8 * 8 * 256 * 2


def test_multi_query_workspace():
    # fused path: up to four queries share a pass, so their partials and folded
    # queries sit side by side; other paths run one query per launch
    c = cfg(rope_base=0.0)
    one = P.palu_decode_workspace_size(c, 16, 128, 4)
    assert P.palu_decode_multi_workspace_size(c, 16, 1, 128, 4) == one
    assert P.palu_decode_multi_workspace_size(c, 16, 8, 128, 4) > 3 * one
    r = cfg()
    assert P.palu_decode_multi_workspace_size(r, 16, 8, 128, 4) == P.palu_decode_workspace_size(r, 16, 128, 4)
    with pytest.raises(P.PaluError):
        P.palu_decode_multi_workspace_size(c, 16, P.MAX_QUERIES + 1, 128, 4)


def test_ranked_layout_equal_ranks_is_uniform():
    # one rank pair for every group: the ranked layout is the uniform one, byte for byte
    c = cfg()
    kb, vb, ksb, vsb, ko, vo = P.palu_cache_strides_ranked(c, [256] * 8, [128] * 8)
    assert (kb, vb, ksb, vsb) == P.palu_cache_strides(c)
    assert ko == [g * 128 * 512 for g in range(8)] and vo == [g * 128 * 256 for g in range(8)]
    assert P.palu_cache_strides_ranked(c, None, None)[:4] == P.palu_cache_strides(c)
    for Q in (1, 3):
        assert P.palu_decode_ranked_workspace_size(c, [256] * 8, [128] * 8, 16, Q, 128, 0) == \
            P.palu_decode_multi_workspace_size(c, 16, Q, 128, 0)
    assert P.palu_compress_ranked_workspace_size(c, [256] * 8, [128] * 8, 64, 4096) == \
        P.palu_compress_workspace_size(c, 64, 4096)


def test_ranked_layout_offsets_are_prefix_sums():
    c = cfg(num_heads=16)
    rk, rv = [64, 384, 128, 256], [128, 64, 256, 128]
    kb, vb, ksb, vsb, ko, vo = P.palu_cache_strides_ranked(c, rk, rv)
    assert kb == 128 * 2 * sum(rk) and vb == 128 * 2 * sum(rv) and ksb == vsb == 0
    assert ko == [128 * 2 * sum(rk[:g]) for g in range(4)]
    assert vo == [128 * 2 * sum(rv[:g]) for g in range(4)]
    ci = cfg(num_heads=16, act_dtype="f16", latent_dtype="int4")
    kb, vb, ksb, vsb, ko, vo = P.palu_cache_strides_ranked(ci, [256, 512, 256, 512], [256] * 4)
    assert ko == [0, 128 * 128, 128 * 384, 128 * 512] and kb == 128 * 768
    srow = lambda r: (2 * (r // 32) + 15) // 16 * 16
    assert ksb == 128 * sum(srow(r) for r in [256, 512, 256, 512])


def test_ranked_argument_checks():
    lib = load()
    c = cfg(num_heads=16)
    arr = lambda v: (ctypes.c_int32 * 4)(*v)
    k = ctypes.c_size_t()
    # a rank that breaks the row rule, one rank array without the other
    assert lib.palu_cache_strides_ranked(ctypes.byref(c), arr([256, 100, 256, 256]), arr([128] * 4),
                                         ctypes.byref(k), None, None, None, None, None) == 3
    assert lib.palu_cache_strides_ranked(ctypes.byref(c), arr([256] * 4), None, ctypes.byref(k), None, None,
                                         None, None, None) == 1
    assert lib.palu_cache_strides_ranked(ctypes.byref(c), arr([256, 1024, 256, 256]), arr([128] * 4),
                                         ctypes.byref(k), None, None, None, None, None) == 2
    # decode: too small a workspace, unaligned workspace
    ws = P.palu_decode_ranked_workspace_size(c, [256, 128, 384, 128], [128, 256, 128, 128], 2, 1, 8, 0)
    p = ctypes.c_void_p(4096)
    call = lambda wsp, nbytes: lib.palu_decode_attn_ranked(
        ctypes.byref(c), arr([256, 128, 384, 128]), arr([128, 256, 128, 128]), 2, 1, p, p, p, p, None, None,
        None, p, 8, p, 8, p, p, p, None, wsp, nbytes, 0, None)
    assert call(p, ws - 1) == 4                                  # PALU_ERR_WORKSPACE
    assert call(ctypes.c_void_p(4096 + 16), ws) == 3             # PALU_ERR_ALIGNMENT
    # compress: d_model not a multiple of 64
    assert lib.palu_compress_append_ranked(ctypes.byref(c), arr([256] * 4), arr([128] * 4), 4, 100, None,
                                           None, None, None, None, None, None, None, None, None, 8, p, 1 << 20,
                                           None) == 2


def test_ranked_workspace_covers_every_decode_set():
    # decode launches group the heads by value rank and kernel family (key ranks
    # may differ within one); the sets run one after another and share the
    # workspace, which is as large as the largest set's
    c = cfg(num_heads=16)
    rk, rv = [256, 128, 384, 128], [128, 256, 128, 128]
    ws = P.palu_decode_ranked_workspace_size(c, rk, rv, 16, 1, 128, 4)
    for r_k, r_v in zip(rk, rv):
        one = cfg(num_heads=4, rank_k=r_k, rank_v=r_v)        # one group
        assert ws >= P.palu_decode_workspace_size(one, 16, 128, 4)
    # set (r_v 128, tensor cores) = groups 0 and 3 (key ranks 256 and 128): 8 heads;
    # group 2 (key rank 384) runs on the CUDA-core kernel, group 1 (r_v 256) alone
    assert ws == 256 + 16 * 8 * 4 * 130 * 4


def test_split_count_model():
    # tensor-core launches: the split count minimises ceil(units·S / 148) · (pages/S + 2) from one
    # full round of CTAs up, or from the largest count fitting one round when that keeps >= 90 % of
    # the SMs busy (smallest on ties); a pass of several fused queries adds S·Q
    def model(units, pages, qn=1):
        s0 = -(-148 // units)
        if units * (148 // units) * 10 >= 9 * 148:
            s0 = 148 // units
        s0 = max(1, min(pages, s0))
        best = None
        for S in range(s0, min(pages, 64) + 1):
            t = -(-units * S // 148) * (-(-pages // S) + 2) + (S * qn if qn > 1 else 0)
            if best is None or t < best[0]:
                best = (t, S)
        return best[1]
    rope = cfg()                                   # 32 heads / 4: 8 groups x 2 head pairs per sequence
    norope = cfg(rope_base=0.0)                    # fused kernel: one CTA per (sequence, group)
    for batch, pages in ((16, 130), (8, 130), (32, 130), (1, 34), (16, 514)):
        assert P.palu_decode_num_splits(rope, batch, pages) == model(batch * 16, pages)
        assert P.palu_decode_num_splits(norope, batch, pages) == model(batch * 8, pages)
    assert P.palu_decode_num_splits(rope, 16, 130) == 4 and P.palu_decode_num_splits(norope, 16, 130) == 8
    # the multi-query workspace is sized for the split count of its passes (4 queries: fewer splits)
    one = P.palu_decode_multi_workspace_size(norope, 16, 4, 130, model(128, 130, 4))
    assert P.palu_decode_multi_workspace_size(norope, 16, 4, 130, 0) == one
