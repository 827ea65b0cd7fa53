"""Test infrastructure shared by the parity tests: build seeded decode cases,
lay logical latents out in the paged pool, run the oracle, compare.

Nothing here computes the method: the oracle does that, from the same host
tensors the GPU receives.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from oracle import palu_oracle as O
from rank_kv_cache_palu_b200 import api as P
from rank_kv_cache_palu_b200.synth import TORCH_DTYPE, Workload, normal, normal_tensor, page_permutation

TOL = {"f32": 1e-4, "f16": 1e-2, "bf16": 1e-2}


def rel_err(gpu: np.ndarray, ref: np.ndarray) -> float:
    """max |gpu - ref| / max |ref| over the whole tensor (the stated parity metric)."""
    den = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(gpu - ref))) / (den if den > 0 else 1.0)


@dataclass
class DecodeCase:
    w: Workload
    seq_lens: list[int]
    q: torch.Tensor              # [b, H, d_h] act dtype (CPU)
    q_pos: np.ndarray            # [b]
    B_k: torch.Tensor            # [G, r_k, W]
    B_v: torch.Tensor            # [G, r_v, W]
    zk: list                     # per b: storage tensor [G, T, r_k] (int4: packed uint8 [G, T, r/2])
    zv: list
    zks: list | None             # int4: per b fp16 scales [G, T, r/32]
    zvs: list | None
    pos: list                    # per b: int32 positions [T] or None (index)
    page_table: np.ndarray       # [b, max_pages]
    num_pages: int

    @property
    def cfg(self):
        w = self.w
        return P.make_config(w.num_heads, w.head_dim, w.group_size, w.rank_k, w.rank_v,
                             w.page_size, w.rope_base, w.act_dtype, w.latent_dtype)

    def oracle_latents(self, b: int):
        """Float64 latents [G, T, r] as the decode step sees them (int4: dequantised)."""
        w = self.w
        if w.latent_dtype == "int4":
            zk = O.dequantize_int4(self.zk[b].numpy(), self.zks[b].numpy(), w.act_dtype)
            zv = O.dequantize_int4(self.zv[b].numpy(), self.zvs[b].numpy(), w.act_dtype)
            return zk, zv
        return self.zk[b].to(torch.float64).numpy(), self.zv[b].to(torch.float64).numpy()

    def positions(self, b: int) -> np.ndarray:
        return np.arange(self.seq_lens[b]) if self.pos[b] is None else self.pos[b].astype(np.int64)


def make_decode_case(w: Workload, seq_lens, seed=None, explicit_positions=False, q_scale=1.0,
                     extra_pages=3, q_pos=None) -> DecodeCase:
    seed = w.seed if seed is None else seed
    G, W, d_h = w.groups, w.width, w.head_dim
    b = len(seq_lens)
    Pz = w.page_size
    max_pages = max(1, max((t + Pz - 1) // Pz for t in seq_lens))
    total_pages = sum((t + Pz - 1) // Pz for t in seq_lens) + extra_pages
    perm = page_permutation(seed, total_pages)
    page_table = np.full((b, max_pages), -1, np.int32)
    k = 0
    for i, t in enumerate(seq_lens):
        for p in range((t + Pz - 1) // Pz):
            page_table[i, p] = perm[k]
            k += 1
    page_table[page_table < 0] = perm[-1]           # unused entries: a valid but unread page
    q = normal_tensor(seed, "q", (b, w.num_heads, d_h), w.act_dtype, q_scale)
    B_k = normal_tensor(seed, "B_k", (G, w.rank_k, W), w.act_dtype, 1 / math.sqrt(w.rank_k))
    B_v = normal_tensor(seed, "B_v", (G, w.rank_v, W), w.act_dtype, 1 / math.sqrt(w.rank_v))
    zk, zv, zks, zvs, pos = [], [], [], [], []
    for i, t in enumerate(seq_lens):
        if w.latent_dtype == "int4":
            for side, r, out_c, out_s in (("zk", w.rank_k, zk, zks), ("zv", w.rank_v, zv, zvs)):
                lat = normal(seed, side, (G, t, r), unit=(i,))
                packed, sc = O.quantize_int4(lat)
                out_c.append(torch.from_numpy(packed))
                out_s.append(torch.from_numpy(sc))
        else:
            zk.append(normal_tensor(seed, "zk", (G, t, w.rank_k), w.latent_dtype, unit=(i,)))
            zv.append(normal_tensor(seed, "zv", (G, t, w.rank_v), w.latent_dtype, unit=(i,)))
        if explicit_positions:
            rng = np.random.default_rng([seed, i, 77])
            pos.append(np.sort(rng.choice(max(4 * t, 1), size=t, replace=False)).astype(np.int32)
                       if t > 0 else np.zeros(0, np.int32))
        else:
            pos.append(None)
    if q_pos is None:
        q_pos = np.array([(int(pp[-1]) + 1 if pp is not None and len(pp) else max(t - 1, 0))
                          for pp, t in zip(pos, seq_lens)], np.int32)
    return DecodeCase(w, list(seq_lens), q, np.asarray(q_pos, np.int32), B_k, B_v, zk, zv,
                      zks if w.latent_dtype == "int4" else None,
                      zvs if w.latent_dtype == "int4" else None, pos, page_table, total_pages)


# ------------------------------------------------------------------ cache page layout
# One (page, group) block holds P tokens x R bytes (R a multiple of 128) as
# 128-byte column blocks of all P tokens, the 16-byte units of token t's 128
# bytes permuted by XOR (t mod 8) -- the layout include/palu.h documents.
def _unit_perm(P: int) -> np.ndarray:
    return np.arange(8)[None, :] ^ (np.arange(P)[:, None] & 7)          # [P, 8]


def swizzle_block(rows: np.ndarray) -> np.ndarray:
    """[P, R] token-major bytes -> the swizzled block image (flat uint8, P*R)."""
    P, R = rows.shape
    assert R % 128 == 0
    src = rows.reshape(P, R // 128, 8, 16).transpose(1, 0, 2, 3)       # [nb, P, unit, 16]
    out = np.empty_like(src)
    out[:, np.arange(P)[:, None], _unit_perm(P), :] = src
    return out.reshape(-1)


def unswizzle_block(img: np.ndarray, P: int) -> np.ndarray:
    """Inverse of swizzle_block: flat block image -> [P, R] token-major bytes."""
    R = img.size // P
    blk = img.reshape(R // 128, P, 8, 16)
    src = blk[:, np.arange(P)[:, None], _unit_perm(P), :]               # [nb, P, unit, 16]
    return src.transpose(1, 0, 2, 3).reshape(P, R)


def _as_bytes(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.uint8).numpy() if t.dtype != torch.uint8 else t.numpy()


def build_pools(case: DecodeCase, device="cuda"):
    """Scatter each sequence's logical latents into the paged pools (host side), upload."""
    w = case.w
    cfg = case.cfg
    kb, vb, ksb, vsb = P.palu_cache_strides(cfg)
    G, Pz = w.groups, w.page_size
    npg = case.num_pages
    pools = {}
    for name, lst, page_bytes in (("zk", case.zk, kb), ("zv", case.zv, vb),
                                  ("zks", case.zks, ksb), ("zvs", case.zvs, vsb)):
        if not page_bytes:
            pools[name] = None
            continue
        row = page_bytes // (G * Pz)
        swz = name in ("zk", "zv")            # latent pools are swizzled; scale pools are token-major
        host = np.zeros((npg, G, Pz * row), np.uint8)
        for i, t in enumerate(case.seq_lens):
            if t == 0:
                continue
            data = _as_bytes(lst[i]).reshape(G, t, -1)
            for p in range((t + Pz - 1) // Pz):
                t0, t1 = p * Pz, min(t, (p + 1) * Pz)
                for g in range(G):
                    blk = np.zeros((Pz, row), np.uint8)
                    blk[: t1 - t0, : data.shape[2]] = data[g, t0:t1]
                    host[case.page_table[i, p], g] = swizzle_block(blk) if swz else blk.reshape(-1)
        pools[name] = torch.from_numpy(host.reshape(-1)).to(device)
    pos_pool = None
    if any(pp is not None for pp in case.pos):
        host = np.zeros((npg, Pz), np.int32)
        for i, t in enumerate(case.seq_lens):
            for p in range((t + Pz - 1) // Pz):
                t0, t1 = p * Pz, min(t, (p + 1) * Pz)
                src = case.pos[i] if case.pos[i] is not None else np.arange(t, dtype=np.int32)
                host[case.page_table[i, p], : t1 - t0] = src[t0:t1]
        pos_pool = torch.from_numpy(host.reshape(-1)).to(device)
    pools["pos"] = pos_pool
    return pools


def run_gpu_decode(case: DecodeCase, num_splits=0, device="cuda", pools=None, check_status=True):
    cfg = case.cfg
    if pools is None:
        pools = build_pools(case, device)
    b = len(case.seq_lens)
    w = case.w
    dev = lambda t: t.to(device)
    ws_bytes = P.palu_decode_workspace_size(cfg, b, case.page_table.shape[1], num_splits)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=device)
    out = torch.empty((b, w.num_heads, w.head_dim), dtype=TORCH_DTYPE[w.act_dtype], device=device)
    lse = torch.empty((b, w.num_heads), dtype=torch.float32, device=device)
    P.palu_decode_attn(cfg, dev(case.q), dev(torch.from_numpy(case.q_pos)), pools["zk"], pools["zv"],
                       pools["zks"], pools["zvs"], pools["pos"],
                       dev(torch.from_numpy(case.page_table)),
                       dev(torch.tensor(case.seq_lens, dtype=torch.int32)), case.num_pages,
                       dev(case.B_k), dev(case.B_v), out, lse, ws, num_splits)
    torch.cuda.synchronize()
    if check_status:
        st, detail = P.palu_get_device_status(ws)
        assert st == 0, f"device status {st} detail {detail}"
    return out.to(torch.float64).cpu().numpy(), lse.to(torch.float64).cpu().numpy()


def oracle_decode(case: DecodeCase, b: int, heads=None):
    """Oracle out [len(heads), d_h], lse for sequence b."""
    w = case.w
    zk, zv = case.oracle_latents(b)
    heads = range(w.num_heads) if heads is None else heads
    q = case.q[b].to(torch.float64).numpy()
    Bk = case.B_k.to(torch.float64).numpy()
    Bv = case.B_v.to(torch.float64).numpy()
    pos = case.positions(b)
    outs, lses = [], []
    for h in heads:
        o, l = O.decode_attention_head(h, q, int(case.q_pos[b]), zk, zv, pos, Bk, Bv,
                                       w.group_size, w.rope_base)
        outs.append(o)
        lses.append(l)
    return np.array(outs), np.array(lses)


# ------------------------------------------------------------------ per-group ranks
@dataclass
class RankedCase:
    """A layer whose head groups have their own ranks; every tensor on the host."""
    w: Workload                  # model shape, dtypes, RoPE (its rank fields are not used)
    ranks_k: list[int]
    ranks_v: list[int]
    seq_lens: list[int]
    q: torch.Tensor              # [b, Q, H, d_h] act dtype
    q_pos: np.ndarray            # [b, Q]
    B_k: torch.Tensor            # [Σ r_k, W]: group g's rows from Σ_{g'<g} r_k,g'
    B_v: torch.Tensor            # [Σ r_v, W]
    zk: list                     # zk[b][g]: storage [T, r_k,g] (int4: packed uint8 [T, r/2])
    zv: list
    zks: list | None             # int4: zks[b][g] fp16 [T, r/32]
    zvs: list | None
    pos: list
    page_table: np.ndarray
    num_pages: int

    @property
    def cfg(self):
        w = self.w
        return P.make_config(w.num_heads, w.head_dim, w.group_size, self.ranks_k[0], self.ranks_v[0],
                             w.page_size, w.rope_base, w.act_dtype, w.latent_dtype)

    def positions(self, b: int) -> np.ndarray:
        return np.arange(self.seq_lens[b]) if self.pos[b] is None else self.pos[b].astype(np.int64)

    def oracle_inputs(self, b: int):
        """(z_k list, z_v list, B_k list, B_v list) in float64, as the decode step sees them."""
        w = self.w
        if w.latent_dtype == "int4":
            zk = [O.dequantize_int4(c.numpy(), s.numpy(), w.act_dtype) for c, s in zip(self.zk[b], self.zks[b])]
            zv = [O.dequantize_int4(c.numpy(), s.numpy(), w.act_dtype) for c, s in zip(self.zv[b], self.zvs[b])]
        else:
            zk = [t.to(torch.float64).numpy() for t in self.zk[b]]
            zv = [t.to(torch.float64).numpy() for t in self.zv[b]]
        return zk, zv, split_rows(self.B_k, self.ranks_k), split_rows(self.B_v, self.ranks_v)


def split_rows(B: torch.Tensor, ranks) -> list:
    offs = np.concatenate([[0], np.cumsum(ranks)])
    Bn = B.to(torch.float64).numpy()
    return [Bn[offs[g]: offs[g + 1]] for g in range(len(ranks))]


def make_ranked_case(w: Workload, ranks_k, ranks_v, seq_lens, nq=1, seed=None, explicit_positions=False,
                     extra_pages=3) -> RankedCase:
    seed = w.seed if seed is None else seed
    G, W, d_h, Pz = w.groups, w.width, w.head_dim, w.page_size
    assert len(ranks_k) == G and len(ranks_v) == G
    b = len(seq_lens)
    max_pages = max(1, max((t + Pz - 1) // Pz for t in seq_lens))
    total_pages = sum((t + Pz - 1) // Pz for t in seq_lens) + extra_pages
    perm = page_permutation(seed, total_pages)
    page_table = np.full((b, max_pages), -1, np.int32)
    k = 0
    for i, t in enumerate(seq_lens):
        for p in range((t + Pz - 1) // Pz):
            page_table[i, p] = perm[k]
            k += 1
    page_table[page_table < 0] = perm[-1]
    q = normal_tensor(seed, "q_ranked", (b, nq, w.num_heads, d_h), w.act_dtype)
    B_k = torch.cat([normal_tensor(seed, f"B_k{g}", (r, W), w.act_dtype, 1 / math.sqrt(r))
                     for g, r in enumerate(ranks_k)])
    B_v = torch.cat([normal_tensor(seed, f"B_v{g}", (r, W), w.act_dtype, 1 / math.sqrt(r))
                     for g, r in enumerate(ranks_v)])
    zk, zv, zks, zvs, pos = [], [], [], [], []
    for i, t in enumerate(seq_lens):
        ck, cv, sk, sv = [], [], [], []
        for g in range(G):
            for side, r, out_c, out_s in ((f"zk{g}", ranks_k[g], ck, sk), (f"zv{g}", ranks_v[g], cv, sv)):
                if w.latent_dtype == "int4":
                    packed, sc = O.quantize_int4(normal(seed, side, (t, r), unit=(i,)))
                    out_c.append(torch.from_numpy(packed))
                    out_s.append(torch.from_numpy(sc))
                else:
                    out_c.append(normal_tensor(seed, side, (t, r), w.latent_dtype, unit=(i,)))
        zk.append(ck)
        zv.append(cv)
        zks.append(sk)
        zvs.append(sv)
        if explicit_positions:
            rng = np.random.default_rng([seed, i, 78])
            pos.append(np.sort(rng.choice(max(4 * t, 1), size=t, replace=False)).astype(np.int32)
                       if t > 0 else np.zeros(0, np.int32))
        else:
            pos.append(None)
    # the last nq cached tokens are the step's queries
    q_pos = np.array([[int((pp if pp is not None else np.arange(t))[max(t - nq + j, 0)]) if t else j
                       for j in range(nq)] for pp, t in zip(pos, seq_lens)], np.int32)
    int4 = w.latent_dtype == "int4"
    return RankedCase(w, list(ranks_k), list(ranks_v), list(seq_lens), q, q_pos, B_k, B_v, zk, zv,
                      zks if int4 else None, zvs if int4 else None, pos, page_table, total_pages)


def _row_bytes(dtype: str, r: int) -> int:
    return r // 2 if dtype == "int4" else r * {"f32": 4, "f16": 2, "bf16": 2}[dtype]


def _scale_row_bytes(r: int) -> int:
    return (2 * (r // 32) + 15) // 16 * 16


def ranked_offsets(w: Workload, ranks_k, ranks_v):
    """name -> (row bytes per group, byte offset of each group's block in a page, page bytes),
    the offsets Σ_{g'<g} page_size·row_g', for K, V and the int4 scale pools."""
    Pz = w.page_size
    lat = w.latent_dtype
    out = {}
    for name, ranks, fn in (("zk", ranks_k, lambda r: _row_bytes(lat, r)),
                            ("zv", ranks_v, lambda r: _row_bytes(lat, r)),
                            ("zks", ranks_k, _scale_row_bytes), ("zvs", ranks_v, _scale_row_bytes)):
        rows = [fn(r) for r in ranks]
        out[name] = (rows, [int(Pz * sum(rows[:g])) for g in range(len(ranks))], Pz * sum(rows))
    return out


def build_ranked_pools(case: RankedCase, device="cuda"):
    """Scatter each sequence's per-group latents into the ranked paged pools, upload."""
    w, Pz, npg = case.w, case.w.page_size, case.num_pages
    G = w.groups
    layout = ranked_offsets(w, case.ranks_k, case.ranks_v)
    pools = {}
    for name, lst in (("zk", case.zk), ("zv", case.zv), ("zks", case.zks), ("zvs", case.zvs)):
        if lst is None:
            pools[name] = None
            continue
        rows, offs, page_bytes = layout[name]
        swz = name in ("zk", "zv")
        host = np.zeros((npg, page_bytes), np.uint8)
        for i, t in enumerate(case.seq_lens):
            for g in range(G):
                data = _as_bytes(lst[i][g]).reshape(t, -1) if t else None
                for p in range((t + Pz - 1) // Pz):
                    t0, t1 = p * Pz, min(t, (p + 1) * Pz)
                    blk = np.zeros((Pz, rows[g]), np.uint8)
                    blk[: t1 - t0, : data.shape[1]] = data[t0:t1]
                    host[case.page_table[i, p], offs[g]: offs[g] + Pz * rows[g]] = \
                        swizzle_block(blk) if swz else blk.reshape(-1)
        pools[name] = torch.from_numpy(host.reshape(-1)).to(device)
    pos_pool = None
    if any(pp is not None for pp in case.pos):
        host = np.zeros((npg, Pz), np.int32)
        for i, t in enumerate(case.seq_lens):
            for p in range((t + Pz - 1) // Pz):
                t0, t1 = p * Pz, min(t, (p + 1) * Pz)
                src = case.pos[i] if case.pos[i] is not None else np.arange(t, dtype=np.int32)
                host[case.page_table[i, p], : t1 - t0] = src[t0:t1]
        pos_pool = torch.from_numpy(host.reshape(-1)).to(device)
    pools["pos"] = pos_pool
    return pools
