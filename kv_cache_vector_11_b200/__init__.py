"""TurboQuant KV-cache quantization and decode attention on NVIDIA B200.

Thin Python binding over the C ABI in ``include/tq.h`` (``libtq.so``, built
in-tree by ``python kv_cache_vector_11_b200/build.py``).  Every function
below only marshals arguments: all computation runs in the library's CUDA
kernels, or in its host generators for rotations and codebooks.  PyTorch is
used for device buffers and streams.  There is no fallback: if the library is
missing, importing this package raises.
"""

from ._lib import (  # noqa: F401
    FMT_GROUPED,
    FMT_NORM_CORRECTED,
    FMT_NORM_F32,
    FORMAT_VERSION,
    STATUS_NONFINITE,
    STATUS_NORM_SATURATED,
    TQError,
    Rotation,
    attn_logits,
    build_codebook,
    code_words_per_row,
    decode_append_paged,
    decode_attention,
    decode_attention_static,
    DECODE_STATIC_SCRATCH_BYTES,
    decode_workspace_size,
    exported_symbols,
    lib_path,
    quantize_kv,
    rotation_generate,
    search_topk,
    search_workspace_size,
)
