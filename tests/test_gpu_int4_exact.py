"""Int4 latents: the decode kernels' unpacking checked exactly, through the C ABI.

The int4 scheme (per token and per 32 latent entries one fp16 scale, codes in
4-bit two's complement, even entry in the low nibble, value = code × scale
rounded to the compute dtype) is this library's reading of the quantisation
compatibility that "Palu: Compressing KV-Cache with Low-Rank Projection" (v2
abstract) claims.  The ordinary parity tests see the dequantised latents only
through attention outputs at the 1e-2 bar, where one wrong nibble in a lane
with little softmax weight would pass.  These cases are built so that the
outputs expose every dequantised entry on its own:

* values: every key code is 0 except those of one token t*, whose score is then
  ~1e3 above every other token's, so its softmax weight is exactly 1 and every
  other weight exactly 0; with a 0/1 column-selection B_v, every output element
  is one dequantised value latent of t*, compared bit for bit with the
  oracle's dequantisation.  t* runs over every row of a page, so every
  converting lane and every latent entry is covered.
* keys: the value latents are a token-identity (entry t of token t is 1), so
  each head's output is the softmax distribution over the page's tokens; a
  one-hot query and a 0/1 B_k make each token's score a known multiple of one
  dequantised key latent.  Log-ratios of the outputs recover every token's
  score to ~1e-3, against a step of >= 0.13 for a one-code error: every
  decoded key code and scale is identified exactly.  (The rounding of code ×
  scale is pinned bit for bit on the value side, which runs the same
  conversion.)

Both kernel families are covered: the tensor-core kernel (its dequantising
producers, and the CUDA-core value sum of a partial last page) and the
CUDA-core split kernel (head_dim 64, not a tensor-core shape).
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

from oracle import palu_oracle as O
from palu_testlib import DecodeCase, build_pools
from rank_kv_cache_palu_b200 import api as P
from rank_kv_cache_palu_b200.synth import TORCH_DTYPE, WORKLOADS, page_permutation

pytestmark = pytest.mark.gpu


def _workload(kind, act):
    if kind == "tensor_core":
        return dataclasses.replace(WORKLOADS["7b_int4_r256_b8_t32k"], act_dtype=act)
    # head_dim 64 takes the CUDA-core split kernel
    return dataclasses.replace(WORKLOADS["tiny_f32"], act_dtype=act, latent_dtype="int4", rank_k=256,
                               rank_v=256)


def _pack(codes: np.ndarray) -> np.ndarray:
    """Codes in [-8, 7] [..., r] -> bytes [..., r/2] in the documented layout (even entry low)."""
    nib = (codes.astype(np.int16) & 0xF).astype(np.uint8)
    return (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)


def _page_table(seed, seq_lens, Pz):
    b = len(seq_lens)
    max_pages = max((t + Pz - 1) // Pz for t in seq_lens)
    total = sum((t + Pz - 1) // Pz for t in seq_lens) + 2
    perm = page_permutation(seed, total)
    pt = np.full((b, max_pages), perm[-1], np.int32)
    k = 0
    for i, t in enumerate(seq_lens):
        for p in range((t + Pz - 1) // Pz):
            pt[i, p] = perm[k]
            k += 1
    return pt, total


def _selection_B_v(w):
    """0/1 B_v [G, r_v, W]: column c of head j of a group reads latent entry
    (j·d_h + c) mod r_v, so the heads of a group read every entry between them."""
    G, W, d_h, r = w.groups, w.width, w.head_dim, w.rank_v
    B = np.zeros((G, r, W), np.float32)
    for j in range(w.group_size):
        for c in range(d_h):
            B[:, (j * d_h + c) % r, j * d_h + c] = 1.0
    return B


def _sel(w, h, c):
    return ((h % w.group_size) * w.head_dim + c) % w.rank_v


def _run(case, pools, num_splits):
    w = case.w
    b = len(case.seq_lens)
    dev = "cuda"
    ws = torch.zeros(P.palu_decode_workspace_size(case.cfg, b, case.page_table.shape[1], num_splits),
                     dtype=torch.uint8, device=dev)
    out = torch.empty((b, w.num_heads, w.head_dim), dtype=TORCH_DTYPE[w.act_dtype], device=dev)
    lse = torch.empty((b, w.num_heads), dtype=torch.float32, device=dev)
    P.palu_decode_attn(case.cfg, case.q.to(dev), torch.from_numpy(case.q_pos).to(dev), pools["zk"], pools["zv"],
                       pools["zks"], pools["zvs"], pools["pos"], torch.from_numpy(case.page_table).to(dev),
                       torch.tensor(case.seq_lens, dtype=torch.int32, device=dev), case.num_pages,
                       case.B_k.to(dev), case.B_v.to(dev), out, lse, ws, num_splits)
    torch.cuda.synchronize()
    st, detail = P.palu_get_device_status(ws)
    assert st == 0, f"device status {st} detail {detail}"
    return out.to(torch.float64).cpu().numpy(), lse.cpu().numpy()


# ------------------------------------------------------------------------- values
@pytest.mark.parametrize("kind,act", [("tensor_core", "f16"), ("tensor_core", "bf16"),
                                      ("cuda_core", "f16"), ("cuda_core", "bf16")])
@pytest.mark.parametrize("ragged", [False, True])
def test_int4_value_unpack_bit_exact(kind, act, ragged):
    w = _workload(kind, act)
    G, Pz, rk, rv = w.groups, w.page_size, w.rank_k, w.rank_v
    rng = np.random.default_rng([11, int(ragged), len(act)])
    # full pages: t* walks every row of a page and all three pages of a sequence;
    # ragged: three pages of which the last holds 44 tokens, t* on that partial page
    if ragged:
        T, rows = 2 * Pz + 44, list(range(44))
        t_star = [2 * Pz + r for r in rows]
    else:
        T, rows = 3 * Pz, list(range(Pz))
        t_star = [Pz * (r % 3) + r for r in rows]
    seq_lens = [T] * len(t_star)
    pt, npg = _page_table(5, seq_lens, Pz)
    zk, zks, zv, zvs = [], [], [], []
    for ts in t_star:
        kc = np.zeros((G, T, rk), np.int16)
        kc[:, ts, :] = 7                                    # only t* has a non-zero key
        zk.append(torch.from_numpy(_pack(kc)))
        zks.append(torch.from_numpy(np.ones((G, T, rk // 32), np.float16)))
        zv.append(torch.from_numpy(rng.integers(0, 256, (G, T, rv // 2), dtype=np.uint8)))   # every nibble
        zvs.append(torch.from_numpy(rng.uniform(1 / 16, 2, (G, T, rv // 32)).astype(np.float16)))
    dt = TORCH_DTYPE[act]
    q = torch.ones((len(t_star), w.num_heads, w.head_dim), dtype=dt)
    B_k = torch.full((G, rk, w.width), 1 / 16, dtype=dt)
    B_v = torch.from_numpy(_selection_B_v(w)).to(dt)
    case = DecodeCase(w, seq_lens, q, np.array(t_star, np.int32), B_k, B_v, zk, zv, zks, zvs,
                      [None] * len(t_star), pt, npg)
    pools = build_pools(case)
    # the expected output: one dequantised value latent of t* per element
    expect = np.zeros((len(t_star), w.num_heads, w.head_dim))
    for b, ts in enumerate(t_star):
        deq = O.dequantize_int4(zv[b].numpy(), zvs[b].numpy(), act)          # [G, T, r_v]
        for h in range(w.num_heads):
            g = h // w.group_size
            expect[b, h] = deq[g, ts, [_sel(w, h, c) for c in range(w.head_dim)]]
    for S in (1, 2, 0):
        out, lse = _run(case, pools, S)
        np.testing.assert_array_equal(out, expect, err_msg=f"{kind} {act} splits={S}")
        assert np.all(lse > 100), "t* must hold the whole softmax weight"


# ------------------------------------------------------------------------- keys
@pytest.mark.parametrize("kind,act", [("tensor_core", "f16"), ("tensor_core", "bf16"),
                                      ("cuda_core", "f16"), ("cuda_core", "bf16")])
def test_int4_key_unpack_identified_exactly(kind, act):
    w = _workload(kind, act)
    G, Pz, rk, rv, d_h, gs = w.groups, w.page_size, w.rank_k, w.rank_v, w.head_dim, w.group_size
    rng = np.random.default_rng([12, len(act), len(kind)])
    nseq = 3
    seq_lens = [Pz] * nseq                                   # one full page each: every row
    pt, npg = _page_table(6, seq_lens, Pz)
    zk, zks, zv, zvs = [], [], [], []
    vc = np.zeros((G, Pz, rv), np.int16)
    for t in range(Pz):                                      # token t: entries t and t + 128 are 1
        vc[:, t, t % rv] = 1
        vc[:, t, (t + 128) % rv] = 1
    for _ in range(nseq):
        zk.append(torch.from_numpy(rng.integers(0, 256, (G, Pz, rk // 2), dtype=np.uint8)))
        zks.append(torch.from_numpy(rng.uniform(0.5, 1.0, (G, Pz, rk // 32)).astype(np.float16)))
        zv.append(torch.from_numpy(_pack(vc)))
        zvs.append(torch.from_numpy(np.ones((G, Pz, rv // 32), np.float16)))
    dt = TORCH_DTYPE[act]
    i0 = d_h // 2 - 1                                        # the lowest RoPE frequency
    Q0 = 3.0
    q = torch.zeros((nseq, w.num_heads, d_h), dtype=dt)
    q[:, :, i0] = Q0
    B_v = torch.from_numpy(_selection_B_v(w)).to(dt)
    q_pos = np.full(nseq, Pz - 1, np.int32)
    deq_k = [O.dequantize_int4(zk[b].numpy(), zks[b].numpy(), act) for b in range(nseq)]
    deq_v = [O.dequantize_int4(zv[b].numpy(), zvs[b].numpy(), act) for b in range(nseq)]
    smallest_step = Q0 * 0.5 / math.sqrt(d_h) * math.cos((Pz - 1) * 10000.0 ** (-2 * i0 / d_h))
    tol = 5e-3 if act == "f16" else 2e-2
    assert tol < smallest_step / 4
    covered = np.zeros((Pz, rk), bool)                       # (row, latent entry) pairs checked
    ncalls = 0
    while not covered.all():
        # head j of group g reads key entry e(g, j) through column i0 of its B_k block
        Bk = np.zeros((G, rk, w.width), np.float32)
        ent = {}
        # after every entry has had a head, the entries move on by one head, so that each
        # is also read by a head that sees the other tokens (a head with 64 output columns
        # shows 64 of the page's 128 tokens)
        cycle = ncalls // (rk // (G * gs))
        for g in range(G):
            for j in range(gs):
                e = (ncalls * G * gs + g * gs + (j + cycle) % gs) % rk
                Bk[g, e, j * d_h + i0] = 1.0
                ent[(g, j)] = e
        case = DecodeCase(w, seq_lens, q, q_pos, torch.from_numpy(Bk).to(dt), B_v, zk, zv, zks, zvs,
                          [None] * nseq, pt, npg)
        if ncalls == 0:
            pools = build_pools(case)
        out, _ = _run(case, pools, 0)
        for b in range(nseq):
            for h in range(w.num_heads):
                g, j = h // gs, h % gs
                # output column c shows token t(c): the token whose identity entry the column reads
                cols = np.arange(d_h)
                toks = np.array([_sel(w, h, c) % 128 for c in cols])
                got = np.log(out[b, h])
                _, _, s = O.decode_attention_head(h, q[b].to(torch.float64).numpy(), int(q_pos[b]), deq_k[b],
                                                  deq_v[b], np.arange(Pz), Bk, B_v.to(torch.float64).numpy(),
                                                  gs, w.rope_base, return_scores=True)
                ref = s[toks]
                err = np.max(np.abs((got - got.mean()) - (ref - ref.mean())))
                assert err <= tol, f"{kind} {act} seq {b} head {h} entry {ent[(g, j)]}: score error {err:.2e}"
                covered[toks, ent[(g, j)]] = True
        ncalls += 1
        assert ncalls <= 64
