"""svga -- block-sparse spatio-temporal attention for video diffusion on B200 (sm_100a).

The compute path is the CUDA library ``libsvga.so`` (C ABI in ``include/svga.h``);
``block_sparse_spatio_attn_b200.svga`` is its thin Python binding.  The binding is
loaded on first use, so ``configs`` and ``inputs`` import without the library.
"""
__all__ = ["configs", "inputs", "svga"]


def __getattr__(name):
    if name == "svga":
        from . import svga as _svga
        return _svga
    raise AttributeError(name)
