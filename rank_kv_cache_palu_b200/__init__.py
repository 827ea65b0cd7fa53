"""Palu latent-KV decode on B200: a C-ABI CUDA library (libpalu.so) and its thin binding.

Keys and values are cached per head group as rank-r latents z = x·A in a paged,
token-major cache; each decode step rebuilds keys from the latents on the fly
(z_k·B_k, RoPE), runs an online softmax, reduces values in latent space and
up-projects them once ((p·z_v)·B_v).
"""
from .api import (  # noqa: F401
    LatentCache, PaluError, make_config, palu_cache_strides, palu_compress_append,
    palu_compress_workspace_size, palu_decode_attn, palu_decode_kernel_kind,
    palu_decode_num_splits, palu_decode_workspace_size, palu_get_device_status,
)
