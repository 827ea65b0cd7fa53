"""CPU oracle for Palu's latent-KV decode path.  TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the bench's ``cpu_baseline`` /
reference leg may import this module.  The product path (the C-ABI library and
its Python binding) never calls it, and it shares no code with the CUDA path:
it is plain numpy in float64, written from the method's definition.

Sources (cited by page title and section):

* [EXPL] "PALU 论文低秩投影分解：从数学结构到工程落地，一次讲透"
  (palu-low-rank pages.dev explainer).
  - §低秩投影分解 (the decomposition): K = x W_k, V = x W_v with
    W_k ≈ A_k B_k, W_v ≈ A_v B_v, A ∈ R^{d_model×r}, B ∈ R^{r×d};
    z_k = x A_k, K ≈ z_k B_k; z_v = x A_v, V ≈ z_v B_v; the cache holds z.
  - §把它放进一次真实推理流程里看, Prefill 阶段: compute z = x A and cache it.
  - §把它放进一次真实推理流程里看, Decode 阶段: read z, rebuild K/V through B
    (or fuse into the attention kernel, without materialising K/V).
  - §先说结论: about 50 % KV-cache compression.
* [ABS2] "Palu: Compressing KV-Cache with Low-Rank Projection" (arXiv 2407.21118
  v2 abstract): medium-grained (group-head) decomposition, RoPE-based
  attention, quantisation compatibility.

Readings where the pages are silent (the oracle and the kernels take the same ones):

* heads are grouped consecutively, group_size heads per group; head h uses
  columns [(h mod g)·d_h, +d_h) of its group's B;
* RoPE is the rotate-half convention, inverse frequency base^(-2i/d_h), angle
  = position × inverse frequency taken as an exact real number (float64 here);
  keys rotate at their own position, the query at q_pos; rope_base = 0 turns
  RoPE off;
* scores are q'·k'/sqrt(d_h); softmax over every cached token (no mask);
* the int4 latent scheme: per token and per 32 consecutive latent entries, a
  symmetric scale s = fp16(fp32(max|z|) / 7), codes clamp(rint(z/s), -7, 7) in
  4-bit two's complement (even entry in the low nibble), dequantised as
  round(code × s) to the compute dtype.  The quantised decision is taken in
  float32, the precision the compress kernel accumulates in.

Parity pins: the tests under tests/test_oracle_pins.py tie every function here
to something other than itself (library routines, closed forms, brute force,
invariants).  Nothing in this module is "parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "round_to_dtype",
    "compress",
    "rope_inv_freq",
    "rope_angles",
    "apply_rope",
    "decode_attention_head",
    "decode_attention",
    "decode_attention_latent",
    "split_partials",
    "lse_combine",
    "decode_attention_multi",
    "decode_attention_ranked",
    "quantize_int4",
    "dequantize_int4",
    "cache_bytes_per_token",
]


# --------------------------------------------------------------------------
# Rounding to storage dtypes (round to nearest, ties to even), directly from
# float64 so that there is a single rounding.
# --------------------------------------------------------------------------
_FORMATS = {
    # name: (fraction bits, minimum normal exponent, largest finite value)
    "f32": (23, -126, float(np.finfo(np.float32).max)),
    "f16": (10, -14, 65504.0),
    "bf16": (7, -126, (2.0 - 2.0 ** -7) * 2.0 ** 127),
}


def round_to_dtype(x, dtype: str) -> np.ndarray:
    """Round float64 values to the nearest value of ``dtype`` (ties to even).

    Returns float64.  Subnormals of the target format keep their fixed
    quantum; values past the largest finite one become +-inf.
    """
    x = np.asarray(x, dtype=np.float64)
    frac_bits, emin, fmax = _FORMATS[dtype]
    ax = np.abs(x)
    _, e = np.frexp(ax)                      # ax = m * 2**e with m in [0.5, 1)
    lead = np.maximum(e - 1, emin)           # exponent of the leading bit
    quantum = np.ldexp(1.0, lead - frac_bits)
    r = np.rint(ax / quantum) * quantum      # scaling by a power of two is exact
    r = np.where(r > fmax, np.inf, r)
    r = np.where(np.isnan(x), np.nan, r)
    return np.copysign(r, x)


# --------------------------------------------------------------------------
# Compress / append: z = x · A, rounded to the cache dtype.
# [EXPL] §低秩投影分解 (z_k = x A_k, z_v = x A_v) and §推理流程 Prefill 阶段.
# --------------------------------------------------------------------------
def compress(x: np.ndarray, A: np.ndarray, dtype: str | None) -> np.ndarray:
    """z = x @ A in float64, then rounded to ``dtype`` (None: no rounding).

    x: [n, d_model]; A: [d_model, N] (the group blocks of A_k or A_v side by
    side).  The rounding is part of the definition: the cache stores that dtype.
    """
    z = np.asarray(x, np.float64) @ np.asarray(A, np.float64)
    return z if dtype is None else round_to_dtype(z, dtype)


# --------------------------------------------------------------------------
# RoPE (rotate-half).  [EXPL] §先说结论 and [ABS2] name RoPE-based attention;
# the convention itself is a reading (see the module docstring).
# --------------------------------------------------------------------------
def rope_inv_freq(head_dim: int, base: float) -> np.ndarray:
    """Inverse frequencies base^(-2i/head_dim) for i in [0, head_dim/2)."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / head_dim)


def rope_angles(pos, head_dim: int, base: float) -> np.ndarray:
    """Angles pos × inv_freq, shape [len(pos), head_dim/2], in float64."""
    pos = np.asarray(pos, dtype=np.float64).reshape(-1)
    return np.outer(pos, rope_inv_freq(head_dim, base))


def apply_rope(v: np.ndarray, pos, base: float) -> np.ndarray:
    """Rotate each row of v ([n, d]) at its position (rotate-half pairs (i, i+d/2)).

    base == 0 means no rotation.
    """
    v = np.asarray(v, dtype=np.float64)
    if base == 0:
        return v.copy()
    n, d = v.shape
    half = d // 2
    ang = rope_angles(pos, d, base)
    assert ang.shape == (n, half)
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = v[:, :half], v[:, half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=1)


# --------------------------------------------------------------------------
# Decode attention, the plain definition: rebuild full K and V from the latents
# ([EXPL] §低秩投影分解: K ≈ z_k B_k, V ≈ z_v B_v), rotate, softmax, weighted sum.
# --------------------------------------------------------------------------
def _head_cols(h: int, group_size: int, head_dim: int) -> tuple[int, slice]:
    g = h // group_size
    j = h % group_size
    return g, slice(j * head_dim, (j + 1) * head_dim)


def decode_attention_head(h: int, q: np.ndarray, q_pos: int, z_k: np.ndarray, z_v: np.ndarray,
                          pos: np.ndarray, B_k: np.ndarray, B_v: np.ndarray, group_size: int,
                          rope_base: float, return_scores: bool = False):
    """One query head over one sequence.

    q: [H, d_h]; z_k: [G, T, r_k]; z_v: [G, T, r_v]; pos: [T];
    B_k: [G, r_k, G_w]; B_v: [G, r_v, G_w] with G_w = group_size·d_h.
    Returns (out [d_h], lse) — and the scaled scores if asked.
    T == 0 gives out = 0 and lse = -inf.
    """
    d_h = q.shape[-1]
    g, cols = _head_cols(h, group_size, d_h)
    T = z_k.shape[1]
    if T == 0:
        out = np.zeros(d_h)
        return (out, -math.inf, np.zeros(0)) if return_scores else (out, -math.inf)
    K = np.asarray(z_k[g], np.float64) @ np.asarray(B_k[g][:, cols], np.float64)   # [T, d_h]
    V = np.asarray(z_v[g], np.float64) @ np.asarray(B_v[g][:, cols], np.float64)   # [T, d_h]
    k_rot = apply_rope(K, pos, rope_base)
    q_rot = apply_rope(np.asarray(q[h], np.float64)[None, :], [q_pos], rope_base)[0]
    s = (k_rot @ q_rot) / math.sqrt(d_h)
    m = s.max()
    e = np.exp(s - m)
    l_sum = e.sum()
    out = (e @ V) / l_sum
    lse = m + math.log(l_sum)
    return (out, lse, s) if return_scores else (out, lse)


def decode_attention(q, q_pos, z_k, z_v, pos, B_k, B_v, group_size, rope_base):
    """All heads of one sequence: returns (out [H, d_h], lse [H])."""
    H, d_h = q.shape
    out = np.zeros((H, d_h))
    lse = np.zeros(H)
    for h in range(H):
        out[h], lse[h] = decode_attention_head(h, q, q_pos, z_k, z_v, pos, B_k, B_v,
                                               group_size, rope_base)
    return out, lse


def decode_attention_multi(q, q_pos, z_k, z_v, pos, B_k, B_v, group_size, rope_base):
    """Several query tokens of one sequence in one step (multi-token decode).

    q: [Q, H, d_h]; q_pos: [Q].  Query j attends to the cached tokens whose
    position is at most its own, q_pos[j] (causal among the appended tokens;
    [EXPL] §推理流程 Prefill / Decode 阶段 consume the same latent cache, and a
    step that scores several new tokens at once is the same attention with a
    per-query causal bound).  With one query at q_pos = T-1 this is
    ``decode_attention``.  Returns (out [Q, H, d_h], lse [Q, H]); a query that
    sees no token gives zeros and -inf.
    """
    q = np.asarray(q)
    Q, H, d_h = q.shape
    pos = np.asarray(pos)
    out = np.zeros((Q, H, d_h))
    lse = np.full((Q, H), -math.inf)
    for j in range(Q):
        keep = pos <= int(q_pos[j])
        if not keep.any():
            continue
        zk_j, zv_j = z_k[:, keep], z_v[:, keep]
        out[j], lse[j] = decode_attention(q[j], int(q_pos[j]), zk_j, zv_j, pos[keep], B_k, B_v,
                                          group_size, rope_base)
    return out, lse


def decode_attention_ranked(q, q_pos, z_k, z_v, pos, B_k, B_v, group_size, rope_base):
    """The multi-query step of a layer whose head groups have their own ranks.

    The rank is chosen by a search, per layer and per group of heads, rather
    than cut to one value everywhere ([EXPL] §为什么还能保精度; §怎么落地, 路线 B;
    §风险、边界和别踩的坑, 风险 1).  z_k, z_v, B_k, B_v are length-G sequences:
    z_k[g] [T, r_k,g], z_v[g] [T, r_v,g], B_k[g] [r_k,g, G_w], B_v[g] [r_v,g, G_w].
    In the group-head decomposition ([ABS2]) the heads of group g read only
    group g's latents and B, so each group is the step above on its own.
    q: [Q, H, d_h]; q_pos: [Q].  Returns (out [Q, H, d_h], lse [Q, H]).
    """
    q = np.asarray(q)
    Q, H, d_h = q.shape
    G = H // group_size
    out = np.zeros((Q, H, d_h))
    lse = np.full((Q, H), -math.inf)
    for g in range(G):
        heads = slice(g * group_size, (g + 1) * group_size)
        out[:, heads], lse[:, heads] = decode_attention_multi(
            q[:, heads], q_pos, np.asarray(z_k[g])[None], np.asarray(z_v[g])[None], pos,
            np.asarray(B_k[g])[None], np.asarray(B_v[g])[None], group_size, rope_base)
    return out, lse


def decode_attention_latent(q, q_pos, z_k, z_v, pos, B_k, B_v, group_size, rope_base):
    """The same step with the value side kept in latent space: o = (p · z_v) · B_v.

    [EXPL] §推理流程 Decode 阶段 allows consuming the latents without
    materialising V; by associativity (P z_v) B_v = P (z_v B_v).  Independent
    second formulation used to cross-check ``decode_attention``.
    """
    H, d_h = q.shape
    out = np.zeros((H, d_h))
    lse = np.zeros(H)
    for h in range(H):
        g, cols = _head_cols(h, group_size, d_h)
        if z_k.shape[1] == 0:
            lse[h] = -math.inf
            continue
        K = np.asarray(z_k[g], np.float64) @ np.asarray(B_k[g][:, cols], np.float64)
        k_rot = apply_rope(K, pos, rope_base)
        q_rot = apply_rope(np.asarray(q[h], np.float64)[None, :], [q_pos], rope_base)[0]
        s = (k_rot @ q_rot) / math.sqrt(d_h)
        m = s.max()
        p = np.exp(s - m)
        a = p @ np.asarray(z_v[g], np.float64)                      # [r_v] latent sum
        out[h] = (a @ np.asarray(B_v[g][:, cols], np.float64)) / p.sum()
        lse[h] = m + math.log(p.sum())
    return out, lse


# --------------------------------------------------------------------------
# Split-sequence decode: partial (m, l, a) per token range, then a log-sum-exp
# merge.  The split itself is how the decode step is parallelised over a long
# context; the merge is exact up to rounding.
# --------------------------------------------------------------------------
def split_partials(h, q, q_pos, z_k, z_v, pos, B_k, group_size, rope_base, bounds):
    """Per token range [t0, t1): running max m, sum l = Σ exp(s - m), latent a = Σ exp(s - m) z_v.

    Empty ranges give (m=-inf, l=0, a=0).
    """
    d_h = q.shape[-1]
    g, cols = _head_cols(h, group_size, d_h)
    r_v = z_v.shape[2]
    parts = []
    for t0, t1 in bounds:
        if t1 <= t0:
            parts.append((-math.inf, 0.0, np.zeros(r_v)))
            continue
        K = np.asarray(z_k[g, t0:t1], np.float64) @ np.asarray(B_k[g][:, cols], np.float64)
        k_rot = apply_rope(K, pos[t0:t1], rope_base)
        q_rot = apply_rope(np.asarray(q[h], np.float64)[None, :], [q_pos], rope_base)[0]
        s = (k_rot @ q_rot) / math.sqrt(d_h)
        m = s.max()
        p = np.exp(s - m)
        parts.append((m, p.sum(), p @ np.asarray(z_v[g, t0:t1], np.float64)))
    return parts


def lse_combine(parts, B_v_cols: np.ndarray):
    """Merge split partials and up-project: returns (out [d_h], lse)."""
    ms = np.array([p[0] for p in parts])
    m = ms.max()
    if m == -math.inf:
        return np.zeros(B_v_cols.shape[1]), -math.inf
    w = np.exp(ms - m)
    l_sum = sum(wi * p[1] for wi, p in zip(w, parts))
    a = sum(wi * p[2] for wi, p in zip(w, parts)) / l_sum
    return a @ np.asarray(B_v_cols, np.float64), m + math.log(l_sum)


# --------------------------------------------------------------------------
# Int4 latents ([ABS2]: low-rank-aware quantisation compatibility; [EXPL]
# §先说结论: stacks with quantisation).  The scheme is a reading.
# --------------------------------------------------------------------------
QBLOCK = 32


def quantize_int4(z32: np.ndarray):
    """Quantise float32 latents [..., r] (r a multiple of 32).

    Returns (packed uint8 [..., r/2], scales float16 [..., r/32]).
    """
    z32 = np.asarray(z32, dtype=np.float32)
    *lead, r = z32.shape
    assert r % QBLOCK == 0
    blocks = z32.reshape(*lead, r // QBLOCK, QBLOCK)
    amax = np.max(np.abs(blocks), axis=-1)                          # float32, exact
    s16 = (amax / np.float32(7.0)).astype(np.float32).astype(np.float16)
    s32 = s16.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (blocks / s32).astype(np.float32)                   # IEEE float32 division
    codes = np.clip(np.rint(ratio), -7, 7)
    codes = np.where(s32 == 0, 0, codes).astype(np.int8).reshape(*lead, r)
    nib = (codes.astype(np.int16) & 0xF).astype(np.uint8)
    packed = (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)
    return packed, s16


def unpack_int4(packed: np.ndarray) -> np.ndarray:
    """4-bit two's-complement codes from packed bytes (even entry in the low nibble)."""
    packed = np.asarray(packed, dtype=np.uint8)
    lo = (packed & 0xF).astype(np.int16)
    hi = (packed >> 4).astype(np.int16)
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.int16)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def dequantize_int4(packed: np.ndarray, scales: np.ndarray, dtype: str) -> np.ndarray:
    """round_to_dtype(code × scale): the value the decode step computes with."""
    codes = unpack_int4(packed).astype(np.float64)
    *lead, r = codes.shape
    s = np.asarray(scales, np.float16).astype(np.float64)
    prod = codes.reshape(*lead, r // QBLOCK, QBLOCK) * s[..., None]
    return round_to_dtype(prod.reshape(*lead, r), dtype)


# --------------------------------------------------------------------------
# Cache footprint ([EXPL] §先说结论: ~50 % compression; §对线上观测要补哪些指标:
# average cache bytes per token).
# --------------------------------------------------------------------------
_ELT_BYTES = {"f32": 4.0, "f16": 2.0, "bf16": 2.0, "int4": 0.5}


def cache_bytes_per_token(num_heads, head_dim, group_size, rank_k, rank_v, dtype: str,
                          scale_bytes: float = 2.0) -> tuple[float, float]:
    """(latent bytes per token per layer, full fp K/V bytes per token per layer).

    Int4 adds one fp16 scale per 32 latent entries.
    """
    G = num_heads // group_size
    elt = _ELT_BYTES[dtype]
    latent = G * (rank_k + rank_v) * elt
    if dtype == "int4":
        latent += G * (rank_k + rank_v) / QBLOCK * scale_bytes
    full_elt = 2.0 if dtype in ("int4", "f16", "bf16") else elt
    full = 2 * num_heads * head_dim * full_elt
    return latent, full
