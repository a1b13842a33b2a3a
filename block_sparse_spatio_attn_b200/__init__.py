"""svga -- block-sparse spatio-temporal attention for video diffusion on B200 (sm_100a).

The compute path is the CUDA library ``libsvga.so`` (C ABI in ``include/svga.h``);
``block_sparse_spatio_attn_b200.svga`` is its thin Python binding, which loads the
library on first use, so ``configs`` and ``inputs`` import without it.
"""
