"""B200 (sm_100a) decode attention over a transformed, percentile-clipped, affine-quantized
2/4-bit KV cache, and the quantize-append step that fills it.

The computation lives in ``libkvq.so`` (hand-written CUDA, C ABI declared in
``include/kvq.h``). This package is the Python binding: the same entry points, taking
PyTorch CUDA tensors and forwarding raw device pointers, sizes and the current stream.
PyTorch supplies device memory and streams only; no step of the path runs here.
"""
from .kvq import (  # noqa: F401
    KVQ_DEVERR_NONFINITE,
    KVQ_DEVERR_PAGE_RANGE,
    KVQ_DEVERR_POS_RANGE,
    KVQ_DEVERR_SEQLEN_CLAMPED,
    KVQ_DEVERR_WAIT_TIMEOUT,
    KVQ_QUANT_PERCENTILE,
    KVQ_QUANT_QUEST,
    KvqError,
    KVCache,
    QParams,
    VQCache,
    bf16_decode,
    bf16_decode_workspace_bytes,
    cache_plane_bytes,
    decode_attention,
    decode_attention_noalloc,
    decode_attention_window,
    decode_workspace_bytes,
    library_path,
    load,
    quantize_append,
    vq_append,
    vq_decode_attention,
    vq_decode_workspace_bytes,
    window_append,
)
