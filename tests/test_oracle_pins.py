"""Pins for the CPU oracle: each check ties an oracle function to something other
than itself — a library routine, a closed form, brute force, an invariant or a
value the pages print.  CPU only."""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import palu_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rng(seed=0):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------- rounding
def test_round_f16_matches_numpy_half():
    x = rng(1).standard_normal(20000) * np.logspace(-9, 5, 20000)
    ref = x.astype(np.float16).astype(np.float64)          # numpy rounds double->half once, RNE
    np.testing.assert_array_equal(O.round_to_dtype(x, "f16"), ref)


def test_round_f32_matches_numpy_single():
    x = rng(2).standard_normal(20000) * np.logspace(-40, 30, 20000)
    np.testing.assert_array_equal(O.round_to_dtype(x, "f32"), x.astype(np.float32).astype(np.float64))


def test_round_bf16_matches_torch_on_float32_inputs():
    # float32 inputs: torch's float->bfloat16 conversion is a single RNE rounding
    x = (rng(3).standard_normal(20000) * np.logspace(-30, 30, 20000)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_to_dtype(x.astype(np.float64), "bf16"), ref)


def test_round_bf16_ties_and_overflow():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1
    assert O.round_to_dtype(1 + 2 ** -8, "bf16") == 1.0
    # 1 + 3*2^-8 is halfway between 1+2^-7 (odd) and 1+2^-6 (even) -> 1+2^-6
    assert O.round_to_dtype(1 + 3 * 2 ** -8, "bf16") == 1 + 2 ** -6
    # just above the tie rounds up
    assert O.round_to_dtype(1 + 2 ** -8 + 2 ** -30, "bf16") == 1 + 2 ** -7
    assert O.round_to_dtype(-(1 + 2 ** -8), "bf16") == -1.0
    assert np.isinf(O.round_to_dtype(3.5e38, "bf16"))
    assert O.round_to_dtype(65519.0, "f16") == 65504.0 and np.isinf(O.round_to_dtype(65520.0, "f16"))


# ----------------------------------------------------------------- compress
def test_compress_brute_force():
    r = rng(4)
    x = r.standard_normal((3, 7))
    A = r.standard_normal((7, 5))
    z = O.compress(x, A, None)
    for i in range(3):
        for j in range(5):
            acc = 0.0
            for k in range(7):
                acc += x[i, k] * A[k, j]
            assert abs(z[i, j] - acc) < 1e-12
    zb = O.compress(x, A, "bf16")
    np.testing.assert_array_equal(zb, O.round_to_dtype(z, "bf16"))


# ----------------------------------------------------------------- RoPE
def test_inv_freq_spot_values():
    f = O.rope_inv_freq(128, 10000.0)
    assert f[0] == 1.0
    assert abs(f[32] - 0.01) < 1e-15          # 10000^(-64/128) = 1/100
    assert abs(f[16] - 0.1) < 1e-15           # 10000^(-32/128) = 1/10
    assert len(f) == 64


def test_rope_matches_complex_rotation():
    # rotate-half RoPE == multiplying (x_i + i x_{i+d/2}) by exp(i * pos * theta_i)
    r = rng(5)
    d = 16
    v = r.standard_normal((6, d))
    pos = np.array([0, 1, 5, 100, 4095, 65535])
    theta = 10000.0 ** (-np.arange(d // 2) * 2.0 / d)
    zc = (v[:, : d // 2] + 1j * v[:, d // 2:]) * np.exp(1j * np.outer(pos, theta))
    ref = np.concatenate([zc.real, zc.imag], axis=1)
    np.testing.assert_allclose(O.apply_rope(v, pos, 10000.0), ref, rtol=0, atol=1e-12)


def test_rope_identity_cases():
    v = rng(6).standard_normal((4, 8))
    np.testing.assert_array_equal(O.apply_rope(v, [0, 0, 0, 0], 10000.0), v)
    np.testing.assert_array_equal(O.apply_rope(v, [3, 9, 1, 2], 0.0), v)       # base 0: off
    rot = O.apply_rope(v, [3, 9, 1, 2], 10000.0)
    np.testing.assert_allclose(np.linalg.norm(rot, axis=1), np.linalg.norm(v, axis=1), rtol=1e-13)


# ----------------------------------------------------------------- decode
def make_seq(seed, H=8, d_h=16, g=4, r_k=12, r_v=10, T=37, base=10000.0, q_scale=1.0):
    r = rng(seed)
    G = H // g
    W = g * d_h
    return dict(
        q=r.standard_normal((H, d_h)) * q_scale,
        q_pos=T - 1,
        z_k=r.standard_normal((G, T, r_k)),
        z_v=r.standard_normal((G, T, r_v)),
        pos=np.arange(T),
        B_k=r.standard_normal((G, r_k, W)) / math.sqrt(r_k),
        B_v=r.standard_normal((G, r_v, W)) / math.sqrt(r_v),
        group_size=g,
        rope_base=base,
    )


def complex_rope(v, pos, base):
    d = v.shape[-1]
    theta = base ** (-np.arange(d // 2) * 2.0 / d)
    zc = (v[..., : d // 2] + 1j * v[..., d // 2:]) * np.exp(1j * np.outer(pos, theta))
    return np.concatenate([zc.real, zc.imag], axis=-1)


def test_full_rank_reduces_to_textbook_attention():
    # r = W and B = I: the latents ARE the keys/values.  Compare with torch's SDPA in float64.
    H, d_h, g, T = 8, 16, 4, 29
    G, W = H // g, g * d_h
    r = rng(7)
    q = r.standard_normal((H, d_h))
    K = r.standard_normal((G, T, W))
    V = r.standard_normal((G, T, W))
    eye = np.stack([np.eye(W)] * G)
    pos = np.arange(T) * 3 + 1
    out, lse = O.decode_attention(q, 500, K, V, pos, eye, eye, g, 10000.0)
    for h in range(H):
        gi, j = h // g, h % g
        kh = complex_rope(K[gi][:, j * d_h:(j + 1) * d_h], pos, 10000.0)
        qh = complex_rope(q[h][None, :], [500], 10000.0)
        vh = V[gi][:, j * d_h:(j + 1) * d_h]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qh)[None, None], torch.from_numpy(kh)[None, None],
            torch.from_numpy(vh)[None, None])[0, 0, 0].numpy()
        np.testing.assert_allclose(out[h], ref, rtol=0, atol=1e-12)
        s = kh @ qh[0] / math.sqrt(d_h)
        assert abs(lse[h] - scipy.special.logsumexp(s)) < 1e-12


def test_softmax_against_scipy():
    c = make_seq(8)
    for h in range(8):
        out, lse, s = O.decode_attention_head(h, **c, return_scores=True)
        gi, j = h // 4, h % 4
        V = c["z_v"][gi] @ c["B_v"][gi][:, j * 16:(j + 1) * 16]
        np.testing.assert_allclose(out, scipy.special.softmax(s) @ V, rtol=0, atol=1e-12)
        assert abs(lse - scipy.special.logsumexp(s)) < 1e-12


def test_q_zero_closed_form():
    c = make_seq(9)
    c["q"] = np.zeros_like(c["q"])
    out, lse = O.decode_attention(**c)
    T = c["z_k"].shape[1]
    for h in range(8):
        gi, j = h // 4, h % 4
        ref = c["z_v"][gi].mean(axis=0) @ c["B_v"][gi][:, j * 16:(j + 1) * 16]
        np.testing.assert_allclose(out[h], ref, rtol=0, atol=1e-12)
        assert abs(lse[h] - math.log(T)) < 1e-12


def test_single_token_returns_its_value():
    c = make_seq(10, T=1)
    out, lse = O.decode_attention(**c)
    for h in range(8):
        gi, j = h // 4, h % 4
        np.testing.assert_allclose(out[h], c["z_v"][gi][0] @ c["B_v"][gi][:, j * 16:(j + 1) * 16],
                                   rtol=0, atol=1e-12)


def test_empty_sequence():
    c = make_seq(11, T=1)
    c["z_k"] = c["z_k"][:, :0]
    c["z_v"] = c["z_v"][:, :0]
    c["pos"] = c["pos"][:0]
    out, lse = O.decode_attention(**c)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_no_rope_identity_scores():
    # without RoPE: q·(z_k B_k)^T == (q B_k^T)·z_k^T
    c = make_seq(12, base=0.0)
    for h in range(8):
        _, _, s = O.decode_attention_head(h, **c, return_scores=True)
        gi, j = h // 4, h % 4
        qt = c["q"][h] @ c["B_k"][gi][:, j * 16:(j + 1) * 16].T      # [r_k]
        np.testing.assert_allclose(s, (c["z_k"][gi] @ qt) / 4.0, rtol=0, atol=1e-12)


def brute_force_decode(c):
    """Plain loops, math module only."""
    q, zk, zv, Bk, Bv = c["q"], c["z_k"], c["z_v"], c["B_k"], c["B_v"]
    H, d = q.shape
    g = c["group_size"]
    T = zk.shape[1]
    base = c["rope_base"]
    half = d // 2
    outs = []
    for h in range(H):
        gi, j = h // g, h % g
        qr = [0.0] * d
        for i in range(half):
            a = c["q_pos"] * base ** (-2.0 * i / d)
            qr[i] = q[h][i] * math.cos(a) - q[h][i + half] * math.sin(a)
            qr[i + half] = q[h][i + half] * math.cos(a) + q[h][i] * math.sin(a)
        scores = []
        vals = []
        for t in range(T):
            k = [sum(zk[gi][t][rr] * Bk[gi][rr][j * d + dd] for rr in range(zk.shape[2])) for dd in range(d)]
            v = [sum(zv[gi][t][rr] * Bv[gi][rr][j * d + dd] for rr in range(zv.shape[2])) for dd in range(d)]
            kr = [0.0] * d
            for i in range(half):
                a = c["pos"][t] * base ** (-2.0 * i / d)
                kr[i] = k[i] * math.cos(a) - k[i + half] * math.sin(a)
                kr[i + half] = k[i + half] * math.cos(a) + k[i] * math.sin(a)
            scores.append(sum(qr[i] * kr[i] for i in range(d)) / math.sqrt(d))
            vals.append(v)
        m = max(scores)
        w = [math.exp(s - m) for s in scores]
        tot = sum(w)
        outs.append([sum(w[t] * vals[t][dd] for t in range(T)) / tot for dd in range(d)])
    return np.array(outs)


def test_brute_force_loops():
    c = make_seq(13, H=4, d_h=4, g=2, r_k=3, r_v=2, T=6)
    c["pos"] = np.array([0, 3, 1, 7, 2, 9])
    c["q_pos"] = 11
    out, _ = O.decode_attention(**c)
    np.testing.assert_allclose(out, brute_force_decode(c), rtol=0, atol=1e-12)


def brute_force_multi(c, q, q_pos):
    """Causal multi-query step by plain loops: each query over the tokens at or before it."""
    outs = []
    for j in range(len(q_pos)):
        keep = [t for t in range(len(c["pos"])) if c["pos"][t] <= q_pos[j]]
        cj = dict(c, q=q[j], q_pos=q_pos[j], z_k=c["z_k"][:, keep], z_v=c["z_v"][:, keep],
                  pos=[c["pos"][t] for t in keep])
        outs.append(brute_force_decode(cj) if keep else np.zeros(q[j].shape))
    return np.array(outs)


def test_multi_query_brute_force_and_causal_mask():
    c = make_seq(31, H=4, d_h=4, g=2, r_k=3, r_v=2, T=7)
    c["pos"] = np.array([0, 3, 1, 7, 2, 9, 5])
    q = rng(32).standard_normal((3, 4, 4))
    q_pos = np.array([4, 9, 1])
    out, lse = O.decode_attention_multi(q, q_pos, c["z_k"], c["z_v"], c["pos"], c["B_k"], c["B_v"],
                                        c["group_size"], c["rope_base"])
    np.testing.assert_allclose(out, brute_force_multi(c, q, q_pos), rtol=0, atol=1e-12)
    # a token after a query's position has no influence on it
    zk2 = c["z_k"].copy()
    zk2[:, 5] += 100.0                              # the token at position 9
    out2, _ = O.decode_attention_multi(q, q_pos, zk2, c["z_v"], c["pos"], c["B_k"], c["B_v"],
                                       c["group_size"], c["rope_base"])
    np.testing.assert_array_equal(out2[0], out[0])
    np.testing.assert_array_equal(out2[2], out[2])
    assert np.abs(out2[1] - out[1]).max() > 1e-6
    # a query before every token sees nothing
    o3, l3 = O.decode_attention_multi(q[:1], np.array([-1]), c["z_k"], c["z_v"], c["pos"], c["B_k"],
                                      c["B_v"], c["group_size"], c["rope_base"])
    assert np.all(o3 == 0) and np.all(np.isneginf(l3))


def test_multi_query_single_query_is_the_decode_step():
    c = make_seq(33, T=29)
    out, lse = O.decode_attention_multi(c["q"][None], np.array([c["q_pos"]]), c["z_k"], c["z_v"],
                                        np.arange(29), c["B_k"], c["B_v"], c["group_size"], c["rope_base"])
    ref, ref_lse = O.decode_attention(**dict(c, pos=np.arange(29)))
    np.testing.assert_allclose(out[0], ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], ref_lse, rtol=0, atol=1e-12)


def make_ranked(seed, ranks_k, ranks_v, H=8, d_h=8, g=2, T=23, base=10000.0):
    r = rng(seed)
    W = g * d_h
    return dict(
        z_k=[r.standard_normal((T, rk)) for rk in ranks_k],
        z_v=[r.standard_normal((T, rv)) for rv in ranks_v],
        B_k=[r.standard_normal((rk, W)) / math.sqrt(rk) for rk in ranks_k],
        B_v=[r.standard_normal((rv, W)) / math.sqrt(rv) for rv in ranks_v],
        pos=np.arange(T) * 2 + 1, group_size=g, rope_base=base,
    ), r.standard_normal((3, H, d_h)), np.array([2 * T - 1, 17, 6])


def test_ranked_equals_zero_padded_uniform():
    # z·B is unchanged when z gains zero columns and B gains rows (any rows):
    # padding every group to the largest rank gives the uniform step
    ranks_k, ranks_v = [3, 7, 1, 5], [2, 6, 4, 4]
    c, q, q_pos = make_ranked(41, ranks_k, ranks_v)
    out, lse = O.decode_attention_ranked(q, q_pos, **c)
    T = len(c["pos"])
    rk, rv = max(ranks_k), max(ranks_v)
    fill = rng(42)
    zk = np.zeros((4, T, rk))
    zv = np.zeros((4, T, rv))
    Bk = fill.standard_normal((4, rk, 16))          # the padded rows are junk on purpose
    Bv = fill.standard_normal((4, rv, 16))
    for gi in range(4):
        zk[gi, :, : ranks_k[gi]] = c["z_k"][gi]
        zv[gi, :, : ranks_v[gi]] = c["z_v"][gi]
        Bk[gi, : ranks_k[gi]] = c["B_k"][gi]
        Bv[gi, : ranks_v[gi]] = c["B_v"][gi]
    ref, ref_lse = O.decode_attention_multi(q, q_pos, zk, zv, c["pos"], Bk, Bv, 2, 10000.0)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)


def test_ranked_brute_force_and_group_independence():
    ranks_k, ranks_v = [3, 1], [2, 4]
    c, q, q_pos = make_ranked(43, ranks_k, ranks_v, H=4, d_h=4, g=2, T=6)
    out, _ = O.decode_attention_ranked(q, q_pos, **c)
    # brute force, one group at a time, each with its own rank
    for gi in range(2):
        cg = dict(q=None, q_pos=None, z_k=np.asarray(c["z_k"][gi])[None], z_v=np.asarray(c["z_v"][gi])[None],
                  pos=c["pos"], B_k=np.asarray(c["B_k"][gi])[None], B_v=np.asarray(c["B_v"][gi])[None],
                  group_size=2, rope_base=10000.0)
        bf = brute_force_multi(cg, q[:, 2 * gi: 2 * gi + 2], q_pos)
        np.testing.assert_allclose(out[:, 2 * gi: 2 * gi + 2], bf, rtol=0, atol=1e-12)
    # changing one group's latents leaves the other group's heads untouched
    c2 = dict(c, z_k=[c["z_k"][0] + 5.0, c["z_k"][1]])
    out2, _ = O.decode_attention_ranked(q, q_pos, **c2)
    np.testing.assert_array_equal(out2[:, 2:], out[:, 2:])
    assert np.abs(out2[:, :2] - out[:, :2]).max() > 1e-6


def test_latent_formulation_matches_materialised():
    c = make_seq(14, T=53)
    a, la = O.decode_attention(**c)
    b, lb = O.decode_attention_latent(**c)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    np.testing.assert_allclose(la, lb, rtol=0, atol=1e-12)


def test_token_permutation_invariance():
    c = make_seq(15, T=41)
    c["pos"] = np.arange(41) * 7 % 50
    a, _ = O.decode_attention(**c)
    perm = rng(16).permutation(41)
    c2 = dict(c, z_k=c["z_k"][:, perm], z_v=c["z_v"][:, perm], pos=c["pos"][perm])
    b, _ = O.decode_attention(**c2)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)


def test_rope_relative_shift_invariance():
    c = make_seq(17, T=33)
    a, _ = O.decode_attention(**c)
    c2 = dict(c, pos=c["pos"] + 1000, q_pos=c["q_pos"] + 1000)
    b, _ = O.decode_attention(**c2)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-9)
    # ... and a shift of the query alone does change it
    c3 = dict(c, q_pos=c["q_pos"] + 5)
    d, _ = O.decode_attention(**c3)
    assert np.max(np.abs(a - d)) > 1e-3


def test_zero_keys_give_uniform_weights():
    c = make_seq(18, T=19)
    c["B_k"] = np.zeros_like(c["B_k"])
    out, lse = O.decode_attention(**c)
    for h in range(8):
        gi, j = h // 4, h % 4
        ref = c["z_v"][gi].mean(0) @ c["B_v"][gi][:, j * 16:(j + 1) * 16]
        np.testing.assert_allclose(out[h], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("bounds", [
    [(0, 61)],
    [(0, 30), (30, 61)],
    [(0, 7), (7, 7), (7, 50), (50, 61)],          # includes an empty split
    [(0, 1), (1, 2), (2, 61)],
])
def test_split_combine_matches_unsplit(bounds):
    c = make_seq(19, T=61, q_scale=3.0)
    for h in (0, 5):
        ref, ref_lse = O.decode_attention_head(h, **c)
        parts = O.split_partials(h, c["q"], c["q_pos"], c["z_k"], c["z_v"], c["pos"], c["B_k"],
                                 c["group_size"], c["rope_base"], bounds)
        gi, j = h // 4, h % 4
        out, lse = O.lse_combine(parts, c["B_v"][gi][:, j * 16:(j + 1) * 16])
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
        assert abs(lse - ref_lse) < 1e-12


def test_combine_all_empty():
    parts = [(-math.inf, 0.0, np.zeros(4))] * 3
    out, lse = O.lse_combine(parts, np.ones((4, 2)))
    assert np.all(out == 0) and lse == -math.inf


# ----------------------------------------------------------------- int4
def test_int4_worked_block():
    z = np.zeros(32, np.float32)
    z[:8] = [7.0, -7.0, 3.5, 2.5, -2.5, 0.49, -0.51, 1.0]
    packed, s = O.quantize_int4(z)
    assert s.dtype == np.float16 and s[0] == 1.0                 # 7/7
    codes = O.unpack_int4(packed)
    assert list(codes[:8]) == [7, -7, 4, 2, -2, 0, -1, 1]       # ties to even: 3.5->4, 2.5->2
    assert packed[0] == 0x97                                    # 7 low, -7 (0x9) high
    assert packed[1] == 0x24                                    # 4 low, 2 high
    assert packed[2] == 0x0E                                    # -2 (0xE) low, 0 high
    assert packed[3] == 0x1F                                    # -1 (0xF) low, 1 high
    np.testing.assert_array_equal(O.dequantize_int4(packed, s, "f16")[:8],
                                  [7, -7, 4, 2, -2, 0, -1, 1])


def test_int4_zero_block_and_scale_rounding():
    z = np.zeros(64, np.float32)
    z[32:] = np.linspace(-1, 1, 32, dtype=np.float32)
    packed, s = O.quantize_int4(z)
    assert s[0] == 0 and np.all(packed[:16] == 0)
    assert s[1] == np.float16(np.float32(1.0) / np.float32(7.0))
    codes = O.unpack_int4(packed)[32:]
    assert codes.min() == -7 and codes.max() == 7


def test_int4_error_bound_and_roundtrip():
    z = (rng(20).standard_normal((5, 9, 256)) * 2).astype(np.float32)
    packed, s = O.quantize_int4(z)
    deq = O.dequantize_int4(packed, s, "f16")
    sb = np.repeat(s.astype(np.float64), 32, axis=-1)
    # |z - code*s| <= s/2 (+ the tiny overshoot of fp16 scale rounding, + fp16 rounding of the product)
    assert np.all(np.abs(z - deq) <= 0.5 * sb * (1 + 2 ** -9) + np.abs(deq) * 2 ** -11 + 1e-12)
    codes = O.unpack_int4(packed)
    assert codes.min() >= -7 and codes.max() <= 7
    # Re-quantising code*s (exact in float32: an 11-bit scale times a 3-bit code) gives the same
    # bytes and scales back.  With a normal fp16 scale, max|z|/s rounds to 7, so the largest code
    # of every block is +-7 and the block's new maximum 7*s divides back to s exactly.
    assert np.all(np.abs(s.astype(np.float32)) >= np.float32(2.0 ** -14))
    z2 = (codes.reshape(5, 9, 8, 32).astype(np.float32) * s.astype(np.float32)[..., None]).reshape(5, 9, 256)
    packed2, s2 = O.quantize_int4(z2)
    np.testing.assert_array_equal(packed2, packed)
    np.testing.assert_array_equal(s2.view(np.uint16), s.view(np.uint16))
    assert np.all(np.max(np.abs(codes.reshape(5, 9, 8, 32)), axis=-1) == 7)


def test_int4_cache_bytes_hand_count():
    # r_k = r_v = 256 per group, int4: 128 bytes of codes per side (two entries a byte) and
    # 256/32 = 8 fp16 scales per side -> 2*128 + 2*8*2 = 288 bytes per (token, group); 8 groups.
    latent, full = O.cache_bytes_per_token(32, 128, 4, 256, 256, "int4")
    assert latent == 8 * 288
    assert full == 2 * 32 * 128 * 2                       # fp16 K and V of 32 heads x 128
    # the same count from what the quantiser actually emits for one token of one group
    z = rng(21).standard_normal((2, 1, 256)).astype(np.float32)
    packed, s = O.quantize_int4(z)
    assert packed.nbytes + s.nbytes == 288
    # unequal ranks and another group count: 8 groups x ((128 + 384)/2 + (4 + 12)*2) bytes
    latent, _ = O.cache_bytes_per_token(32, 128, 4, 128, 384, "int4")
    assert latent == 8 * (256 + 32)


# ----------------------------------------------------------------- compression ratio (printed value)
def test_compression_ratio_golden():
    with open(os.path.join(GOLDEN, "compression_ratio.json")) as f:
        gold = json.load(f)
    sh = gold["shape"]
    latent, full = O.cache_bytes_per_token(sh["num_heads"], sh["head_dim"], sh["group_size"],
                                           sh["rank_k"], sh["rank_v"], sh["dtype"])
    assert latent / full == gold["latent_over_full_bytes"]
