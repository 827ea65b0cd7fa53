"""Python binding of libpalu.so: the C-ABI entry points under the same names.

Argument marshalling only — every step of the path runs in the CUDA kernels.
Tensors are torch tensors used as device buffers; streams are torch streams.
Each call raises ``PaluError`` when the library returns a non-OK status.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from ._lib import PaluConfig, load

DTYPE_CODE = {"f32": 0, "f16": 1, "bf16": 2, "int4": 3}
TORCH_OF = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}

STATUS_NAMES = {
    0: "PALU_OK", 1: "PALU_ERR_INVALID_ARG", 2: "PALU_ERR_UNSUPPORTED", 3: "PALU_ERR_ALIGNMENT",
    4: "PALU_ERR_WORKSPACE", 5: "PALU_ERR_CUDA", 6: "PALU_ERR_DEVICE_TIMEOUT",
    7: "PALU_ERR_DEVICE_BOUNDS",
}


class PaluError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        msg = lib.palu_status_string(status).decode()
        if status == 5:
            msg += f" ({lib.palu_last_cuda_error().decode()})"
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != 0:
        raise PaluError(status, where)


def make_config(num_heads: int, head_dim: int, group_size: int, rank_k: int, rank_v: int,
                page_size: int = 128, rope_base: float = 10000.0, act_dtype: str = "bf16",
                latent_dtype: str | None = None) -> PaluConfig:
    return PaluConfig(num_heads, head_dim, group_size, rank_k, rank_v, page_size, float(rope_base),
                      DTYPE_CODE[act_dtype], DTYPE_CODE[latent_dtype or act_dtype])


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor or None")
    if t.numel() > 0 and not t.is_cuda:
        raise ValueError("palu tensors must live in CUDA device memory")
    if not t.is_contiguous():
        raise ValueError("palu tensors must be contiguous")
    return t.data_ptr() if t.numel() > 0 else None


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def palu_cache_strides(cfg: PaluConfig) -> tuple[int, int, int, int]:
    out = [ctypes.c_size_t() for _ in range(4)]
    _check(load().palu_cache_strides(ctypes.byref(cfg), *[ctypes.byref(o) for o in out]),
           "palu_cache_strides")
    return tuple(o.value for o in out)


def palu_compress_workspace_size(cfg: PaluConfig, n_tokens: int, d_model: int) -> int:
    out = ctypes.c_size_t()
    _check(load().palu_compress_workspace_size(ctypes.byref(cfg), n_tokens, d_model,
                                               ctypes.byref(out)), "palu_compress_workspace_size")
    return out.value


def palu_decode_num_splits(cfg: PaluConfig, batch: int, max_pages: int) -> int:
    out = ctypes.c_int()
    _check(load().palu_decode_num_splits(ctypes.byref(cfg), batch, max_pages, ctypes.byref(out)),
           "palu_decode_num_splits")
    return out.value


def palu_decode_workspace_size(cfg: PaluConfig, batch: int, max_pages: int, num_splits: int = 0) -> int:
    out = ctypes.c_size_t()
    _check(load().palu_decode_workspace_size(ctypes.byref(cfg), batch, max_pages, num_splits,
                                             ctypes.byref(out)), "palu_decode_workspace_size")
    return out.value


def palu_decode_kernel_kind(cfg: PaluConfig) -> int:
    return int(load().palu_decode_kernel_kind(ctypes.byref(cfg)))


def palu_kernel_launches() -> int:
    """Kernels launched by libpalu in this process so far."""
    return int(load().palu_kernel_launches())


def palu_debug_trace(buffer, tiles_per_cta: int = 0) -> None:
    """Record tensor-core decode phase timestamps into `buffer` (int64 CUDA tensor); None stops."""
    if buffer is None:
        _check(load().palu_debug_trace(None, 0, 0), "palu_debug_trace")
    else:
        _check(load().palu_debug_trace(_ptr(buffer), buffer.numel() * buffer.element_size(),
                                       tiles_per_cta), "palu_debug_trace")


def palu_debug_timeout_test(wait_cycles: int = 0, stall: bool = False) -> None:
    """Test hook of the kernels' timeout path: bound every wait of later tensor-core
    launches to wait_cycles SM cycles (0 = the default) and, with stall, make each
    such launch run that bound out.  palu_debug_timeout_test() restores normal operation."""
    _check(load().palu_debug_timeout_test(int(wait_cycles), 1 if stall else 0), "palu_debug_timeout_test")


def palu_compress_append(cfg: PaluConfig, x, A_k, A_v, slot_mapping, positions, zk_pool, zv_pool,
                         zk_scales, zv_scales, pos_pool, num_pages: int, workspace, stream=None):
    n, d_model = x.shape
    st = load().palu_compress_append(
        ctypes.byref(cfg), n, d_model, _ptr(x), _ptr(A_k), _ptr(A_v), _ptr(slot_mapping),
        _ptr(positions), _ptr(zk_pool), _ptr(zv_pool), _ptr(zk_scales), _ptr(zv_scales),
        _ptr(pos_pool), num_pages, _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(st, "palu_compress_append")


def palu_decode_attn(cfg: PaluConfig, q, q_pos, zk_pool, zv_pool, zk_scales, zv_scales, pos_pool,
                     page_table, seq_lens, num_pages: int, B_k, B_v, out, lse, workspace,
                     num_splits: int = 0, stream=None):
    batch = q.shape[0]
    max_pages = page_table.shape[1]
    st = load().palu_decode_attn(
        ctypes.byref(cfg), batch, _ptr(q), _ptr(q_pos), _ptr(zk_pool), _ptr(zv_pool),
        _ptr(zk_scales), _ptr(zv_scales), _ptr(pos_pool), _ptr(page_table), max_pages,
        _ptr(seq_lens), num_pages, _ptr(B_k), _ptr(B_v), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), num_splits, _stream(stream))
    _check(st, "palu_decode_attn")


MAX_QUERIES = 16


def palu_decode_multi_workspace_size(cfg: PaluConfig, batch: int, num_queries: int, max_pages: int,
                                     num_splits: int = 0) -> int:
    out = ctypes.c_size_t()
    _check(load().palu_decode_multi_workspace_size(ctypes.byref(cfg), batch, num_queries, max_pages,
                                                   num_splits, ctypes.byref(out)),
           "palu_decode_multi_workspace_size")
    return int(out.value)


def palu_decode_attn_multi(cfg: PaluConfig, q, q_pos, zk_pool, zv_pool, zk_scales, zv_scales, pos_pool,
                           page_table, seq_lens, num_pages: int, B_k, B_v, out, lse, workspace,
                           num_splits: int = 0, stream=None):
    """Several query tokens per sequence: q [batch][Q][H][d_h], q_pos [batch][Q]; causal by position."""
    batch, nq = q.shape[0], q.shape[1]
    max_pages = page_table.shape[1]
    st = load().palu_decode_attn_multi(
        ctypes.byref(cfg), batch, nq, _ptr(q), _ptr(q_pos), _ptr(zk_pool), _ptr(zv_pool),
        _ptr(zk_scales), _ptr(zv_scales), _ptr(pos_pool), _ptr(page_table), max_pages,
        _ptr(seq_lens), num_pages, _ptr(B_k), _ptr(B_v), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), num_splits, _stream(stream))
    _check(st, "palu_decode_attn_multi")


def _ranks(r):
    """Host int32 array of per-group ranks (None: the config's uniform ranks)."""
    return None if r is None else (ctypes.c_int32 * len(r))(*[int(v) for v in r])


def palu_cache_strides_ranked(cfg: PaluConfig, ranks_k, ranks_v):
    """(k_page, v_page, k_scale_page, v_scale_page, k_group_offsets, v_group_offsets) in bytes."""
    G = cfg.num_heads // cfg.group_size
    out = [ctypes.c_size_t() for _ in range(4)]
    ko, vo = (ctypes.c_size_t * G)(), (ctypes.c_size_t * G)()
    _check(load().palu_cache_strides_ranked(ctypes.byref(cfg), _ranks(ranks_k), _ranks(ranks_v),
                                            *[ctypes.byref(o) for o in out], ko, vo),
           "palu_cache_strides_ranked")
    return (*[o.value for o in out], list(ko), list(vo))


def palu_compress_ranked_workspace_size(cfg: PaluConfig, ranks_k, ranks_v, n_tokens: int, d_model: int) -> int:
    out = ctypes.c_size_t()
    _check(load().palu_compress_ranked_workspace_size(ctypes.byref(cfg), _ranks(ranks_k), _ranks(ranks_v),
                                                      n_tokens, d_model, ctypes.byref(out)),
           "palu_compress_ranked_workspace_size")
    return int(out.value)


def palu_compress_append_ranked(cfg: PaluConfig, ranks_k, ranks_v, x, A_k, A_v, slot_mapping, positions,
                                zk_pool, zv_pool, zk_scales, zv_scales, pos_pool, num_pages: int, workspace,
                                stream=None):
    """palu_compress_append for a layer with a rank pair per group (A columns stacked by group)."""
    n, d_model = x.shape
    st = load().palu_compress_append_ranked(
        ctypes.byref(cfg), _ranks(ranks_k), _ranks(ranks_v), n, d_model, _ptr(x), _ptr(A_k), _ptr(A_v),
        _ptr(slot_mapping), _ptr(positions), _ptr(zk_pool), _ptr(zv_pool), _ptr(zk_scales), _ptr(zv_scales),
        _ptr(pos_pool), num_pages, _ptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream))
    _check(st, "palu_compress_append_ranked")


def palu_decode_ranked_workspace_size(cfg: PaluConfig, ranks_k, ranks_v, batch: int, num_queries: int,
                                      max_pages: int, num_splits: int = 0) -> int:
    out = ctypes.c_size_t()
    _check(load().palu_decode_ranked_workspace_size(ctypes.byref(cfg), _ranks(ranks_k), _ranks(ranks_v), batch,
                                                    num_queries, max_pages, num_splits, ctypes.byref(out)),
           "palu_decode_ranked_workspace_size")
    return int(out.value)


def palu_decode_attn_ranked(cfg: PaluConfig, ranks_k, ranks_v, q, q_pos, zk_pool, zv_pool, zk_scales, zv_scales,
                            pos_pool, page_table, seq_lens, num_pages: int, B_k, B_v, out, lse, workspace,
                            num_splits: int = 0, stream=None):
    """Decode step of a layer with a rank pair per group: q [batch][Q][H][d_h], q_pos [batch][Q]
    (Q = 1 is the single-query step); B_k / B_v rows stacked by group."""
    batch, nq = q.shape[0], q.shape[1]
    max_pages = page_table.shape[1]
    st = load().palu_decode_attn_ranked(
        ctypes.byref(cfg), _ranks(ranks_k), _ranks(ranks_v), batch, nq, _ptr(q), _ptr(q_pos), _ptr(zk_pool),
        _ptr(zv_pool), _ptr(zk_scales), _ptr(zv_scales), _ptr(pos_pool), _ptr(page_table), max_pages,
        _ptr(seq_lens), num_pages, _ptr(B_k), _ptr(B_v), _ptr(out), _ptr(lse), _ptr(workspace),
        workspace.numel() * workspace.element_size(), num_splits, _stream(stream))
    _check(st, "palu_decode_attn_ranked")


NOALLOC_SCRATCH_BYTES = 8 << 20


def palu_decode_attn_noalloc(cfg: PaluConfig, q, q_pos, zk_pool, zv_pool, zk_scales, zv_scales,
                             pos_pool, page_table, seq_lens, num_pages: int, B_k, B_v, out, lse,
                             num_splits: int = 0, stream=None, report_status: bool = False):
    """palu_decode_attn without a caller workspace (the library's fixed device array).

    report_status=True waits for the stream and raises on a device-detected fault.
    """
    batch = q.shape[0]
    max_pages = page_table.shape[1]
    detail = ctypes.c_int32()
    st = load().palu_decode_attn_noalloc(
        ctypes.byref(cfg), batch, _ptr(q), _ptr(q_pos), _ptr(zk_pool), _ptr(zv_pool),
        _ptr(zk_scales), _ptr(zv_scales), _ptr(pos_pool), _ptr(page_table), max_pages,
        _ptr(seq_lens), num_pages, _ptr(B_k), _ptr(B_v), _ptr(out), _ptr(lse), num_splits,
        _stream(stream), ctypes.byref(detail) if report_status else None)
    _check(st, "palu_decode_attn_noalloc")


def palu_get_device_status(workspace, stream=None) -> tuple[int, int]:
    """(status, detail) of the device status word; clears it."""
    detail = ctypes.c_int32()
    st = load().palu_get_device_status(_ptr(workspace), _stream(stream), ctypes.byref(detail))
    return int(st), int(detail.value)


@dataclass
class LatentCache:
    """Device buffers of a paged latent cache for one layer (caller-owned memory).

    Pools are uint8 tensors of num_pages pages each, laid out as include/palu.h
    states; ``view_*`` give typed views for inspection.
    """

    cfg: PaluConfig
    num_pages: int
    zk: torch.Tensor
    zv: torch.Tensor
    zks: torch.Tensor | None
    zvs: torch.Tensor | None
    pos: torch.Tensor | None
    ranks_k: tuple | None = None     # per-group ranks (None: the config's for every group)
    ranks_v: tuple | None = None

    @classmethod
    def allocate(cls, cfg: PaluConfig, num_pages: int, device="cuda", with_positions=False,
                 fill=None, ranks_k=None, ranks_v=None) -> "LatentCache":
        """Pools for num_pages pages; with ranks_k / ranks_v, the layout of a layer whose
        groups carry their own ranks (each page holds every group's block back to back)."""
        if ranks_k is None:
            kb, vb, ksb, vsb = palu_cache_strides(cfg)
        else:
            kb, vb, ksb, vsb, _, _ = palu_cache_strides_ranked(cfg, ranks_k, ranks_v)
        mk = (lambda n: torch.empty(n, dtype=torch.uint8, device=device)) if fill is None else \
            (lambda n: torch.full((n,), fill, dtype=torch.uint8, device=device))
        zks = mk(num_pages * ksb) if ksb else None
        zvs = mk(num_pages * vsb) if vsb else None
        pos = torch.zeros(num_pages * cfg.page_size, dtype=torch.int32, device=device) \
            if with_positions else None
        return cls(cfg, num_pages, mk(num_pages * kb), mk(num_pages * vb), zks, zvs, pos,
                   None if ranks_k is None else tuple(ranks_k), None if ranks_v is None else tuple(ranks_v))
