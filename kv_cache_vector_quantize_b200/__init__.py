"""B200-native TurboQuant KV-cache quantization: Python binding of libtq.so.

The package is a thin layer over the C ABI declared in ``include/tq.h``:
``tq_quantize_append`` (online quantization of K/V head-vectors into a packed
cache), ``tq_logits`` (attention logits on the packed keys) and
``tq_attend_v`` (softmax-weighted packed values), ``tq_decode_attend`` (the
three decode steps in one call, one pass over the tokens where the shapes allow),
``tq_nn_search`` (top-k inner-product search over a packed key stream),
mixed-rate caches for fractional bits per channel (``PackedCache.empty(...,
n_hi=...)``, ``tq_record_words_mixed``), plus the setup helpers
``tq_codebook_fit`` and ``tq_sketch_rotation``. All compute runs in the CUDA
kernels of ``csrc/`` built for sm_100a.
"""

from ._binding import (  # noqa: F401
    LIB_PATH,
    STATUS_NAMES,
    TQ_ERR_CAPACITY,
    TQ_ERR_CUDA,
    TQ_ERR_DEVICE,
    TQ_ERR_INVALID,
    TQ_ERR_UNSUPPORTED,
    TQ_ERR_WORKSPACE,
    TQ_OK,
    PackedCache,
    TqCacheDesc,
    TQError,
    declared_symbols,
    raw_lib,
    tq_attend_merge,
    tq_attend_v,
    tq_attend_v_partial,
    tq_attend_workspace_size,
    tq_codebook_fit,
    tq_debug_inject,
    tq_debug_stall_consumers,
    tq_decode_attend,
    tq_decode_workspace_size,
    tq_last_error,
    tq_logits,
    tq_logits_workspace_size,
    tq_nn_merge,
    tq_nn_search,
    tq_nn_workspace_size,
    tq_quantize_append,
    tq_quantize_append_hadamard,
    tq_record_words,
    tq_record_words_mixed,
    tq_sketch_rotation,
    tq_workspace_status,
)
