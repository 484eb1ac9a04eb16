"""Tiled MonarchRT attention forward pass for NVIDIA B200 (sm_100a).

    from structured_attention_video_b200 import monarch_attention
    y = monarch_attention(q, k, v, f=21, h=45, w=80, b1=945, b2=80, tiles=4, iters=1)

q, k, v are contiguous CUDA tensors [B, H, N, d] (float32 or bfloat16) with
N = f*h*w tokens in (frame, row, column) order.  The computation runs in the
CUDA kernels of libmonarch.so (C ABI: include/monarch_attn.h); importing the
attention entry points fails loudly when that library is missing.
"""

__all__ = ["monarch_attention", "workspace_bytes", "kernel_path"]


def __getattr__(name):
    if name in __all__:
        from . import attention
        return getattr(attention, name)
    raise AttributeError(name)
