"""ctypes binding of libtq.so (include/tq.h), with the C entry points' names.

Argument marshalling only: torch tensors are checked for device, dtype and
layout, outputs and workspaces are allocated through torch when the caller
does not pass them, and data pointers plus the current CUDA stream go to the
C functions. Every step of the method runs in the library's kernels; there is
no Python or CPU implementation to fall back on, and importing this module
fails loudly when the library has not been built.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os
import re

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtq.so")
HEADER_PATH = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "tq.h")

TQ_OK, TQ_ERR_INVALID, TQ_ERR_UNSUPPORTED, TQ_ERR_CAPACITY, TQ_ERR_WORKSPACE, TQ_ERR_CUDA, TQ_ERR_DEVICE = range(7)
STATUS_NAMES = {0: "TQ_OK", 1: "TQ_ERR_INVALID", 2: "TQ_ERR_UNSUPPORTED", 3: "TQ_ERR_CAPACITY",
                4: "TQ_ERR_WORKSPACE", 5: "TQ_ERR_CUDA", 6: "TQ_ERR_DEVICE"}
TQ_BF16, TQ_FP16, TQ_FP32 = 0, 1, 2
_DTYPE = {torch.bfloat16: TQ_BF16, torch.float16: TQ_FP16, torch.float32: TQ_FP32}


class TQError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class TqCacheDesc(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("idx_bits", ctypes.c_int32), ("qjl", ctypes.c_int32),
                ("n_seq", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32), ("n_hi", ctypes.c_int32),
                ("capacity", ctypes.c_int64), ("records", ctypes.c_void_p), ("norm", ctypes.c_void_p),
                ("rnorm", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python kv_cache_vector_quantize_b200/build.py` "
                          "(the CUDA library is the only implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    D = ctypes.POINTER(TqCacheDesc)
    sig = {
        "tq_record_words": (I32, [I32, I32, I32]),
        "tq_record_words_mixed": (I32, [I32, I32, I32, I32]),
        "tq_codebook_fit": (I32, [I32, I32, P]),
        "tq_sketch_rotation": (I32, [I32, P, P, P, P]),
        "tq_quantize_append": (I32, [D, P, I32, I64, I64, P, P, P, P]),
        "tq_quantize_append_hadamard": (I32, [D, P, I32, I64, I64, P, P, P, P]),
        "tq_logits_workspace_size": (SZ, [D, I32]),
        "tq_logits": (I32, [D, P, I32, I64, P, P, P, P, P, SZ, P]),
        "tq_attend_workspace_size": (SZ, [D, I32, I64]),
        "tq_attend_v": (I32, [D, P, F, I32, I64, P, P, P, P, SZ, P]),
        "tq_attend_v_noalloc": (I32, [D, P, F, I32, I64, P, P, P, P]),
        "tq_attend_v_noalloc_status": (I32, [P]),
        "tq_attend_v_partial": (I32, [D, P, F, I32, I64, P, P, P, SZ, P]),
        "tq_attend_merge": (I32, [P, I32, I32, I32, P, P, P]),
        "tq_nn_merge": (I32, [P, P, I32, I32, I32, P, P, P]),
        "tq_decode_workspace_size": (SZ, [D, D, I32, I64]),
        "tq_decode_attend": (I32, [D, D, P, I32, I64, F, P, P, P, P, P, P, SZ, P]),
        "tq_nn_workspace_size": (SZ, [D, I32, I64]),
        "tq_nn_search": (I32, [D, P, I32, I64, P, P, P, I32, P, P, P, SZ, P]),
        "tq_workspace_status": (I32, [P, P]),
        "tq_last_error": (ctypes.c_char_p, []),
        "tq_debug_inject": (None, [I32, I32]),
        "tq_debug_stall_consumers": (None, [ctypes.c_uint32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def declared_symbols() -> list[str]:
    """Function names declared in include/tq.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b(tq_\w+)\s*\(", text, flags=re.M)))


def _check(status: int) -> None:
    if status != TQ_OK:
        raise TQError(status, _lib.tq_last_error().decode())


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, shape=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must have dtype {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


# ----------------------------------------------------------------------------
# cache container (caller-owned memory, allocated through torch)
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class PackedCache:
    d: int
    idx_bits: int
    qjl: bool
    n_seq: int
    n_kv_heads: int
    capacity: int
    records: torch.Tensor            # int32 view of the uint32 words [n_seq, n_kv_heads, capacity, R]
    norm: torch.Tensor               # float32 [n_seq, n_kv_heads, capacity]
    rnorm: torch.Tensor | None
    n_hi: int = 0                    # mixed rate: leading coordinates at idx_bits + 1 code bits

    @classmethod
    def empty(cls, d, idx_bits, qjl, n_seq, n_kv_heads, capacity, device="cuda", n_hi=0):
        rw = tq_record_words_mixed(d, idx_bits, n_hi, qjl)
        rec = torch.zeros((n_seq, n_kv_heads, capacity, rw), dtype=torch.int32, device=device)
        norm = torch.zeros((n_seq, n_kv_heads, capacity), dtype=torch.float32, device=device)
        rnorm = torch.zeros_like(norm) if qjl else None
        return cls(d, idx_bits, bool(qjl), n_seq, n_kv_heads, capacity, rec, norm, rnorm, int(n_hi))

    @property
    def codebook_len(self) -> int:
        """Floats of the codebook argument: 2^idx_bits, plus 2^(idx_bits+1) for a mixed-rate cache."""
        return (1 << self.idx_bits) + ((2 << self.idx_bits) if self.n_hi else 0)

    def desc(self) -> TqCacheDesc:
        return TqCacheDesc(self.d, self.idx_bits, int(self.qjl), self.n_seq, self.n_kv_heads, self.n_hi, self.capacity,
                           self.records.data_ptr(), self.norm.data_ptr(),
                           self.rnorm.data_ptr() if self.rnorm is not None else None)

    @property
    def device(self):
        return self.records.device

    def nbytes(self, n_tokens: int | None = None) -> int:
        """Bytes of the packed cache holding `n_tokens` tokens per (sequence, head)."""
        t = self.capacity if n_tokens is None else n_tokens
        per = 4 * self.records.shape[-1] + 4 * (2 if self.qjl else 1)
        return self.n_seq * self.n_kv_heads * t * per


# ----------------------------------------------------------------------------
# entry points
# ----------------------------------------------------------------------------

def tq_record_words(d: int, idx_bits: int, qjl) -> int:
    w = _lib.tq_record_words(d, idx_bits, int(qjl))
    if w < 0:
        raise TQError(TQ_ERR_UNSUPPORTED, f"unsupported d={d} idx_bits={idx_bits}")
    return w


def tq_record_words_mixed(d: int, idx_bits: int, n_hi: int, qjl) -> int:
    w = _lib.tq_record_words_mixed(d, idx_bits, int(n_hi), int(qjl))
    if w < 0:
        raise TQError(TQ_ERR_UNSUPPORTED, f"unsupported d={d} idx_bits={idx_bits} n_hi={n_hi}")
    return w


def tq_codebook_fit(d: int, idx_bits: int) -> torch.Tensor:
    """Lloyd-Max centroids for the coordinate law (host computation), float32 CPU tensor."""
    out = torch.empty(1 << idx_bits, dtype=torch.float32)
    _check(_lib.tq_codebook_fit(d, idx_bits, ctypes.c_void_p(out.data_ptr())))
    return out


def tq_sketch_rotation(Pi: torch.Tensor, S: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    d = Pi.shape[0]
    _need(Pi, "Pi", torch.float32, (d, d))
    _need(S, "S", torch.float32, (d, d), Pi.device)
    if out is None:
        out = torch.empty_like(Pi)
    _need(out, "out", torch.float32, (d, d), Pi.device)
    _check(_lib.tq_sketch_rotation(d, _ptr(Pi), _ptr(S), _ptr(out), _stream(stream)))
    return out


def tq_quantize_append(cache: PackedCache, x: torch.Tensor, pos: int, Pi: torch.Tensor, SPiT: torch.Tensor | None,
                       codebook: torch.Tensor, stream=None) -> None:
    """x: [n_seq, n_kv_heads, n_tokens, d] (bf16/fp16/fp32) written to slots [pos, pos + n_tokens)."""
    if x.dim() != 4 or x.shape[0] != cache.n_seq or x.shape[1] != cache.n_kv_heads or x.shape[3] != cache.d:
        raise ValueError(f"x must be [{cache.n_seq}, {cache.n_kv_heads}, T, {cache.d}], got {tuple(x.shape)}")
    _need(x, "x", device=cache.device)
    if x.dtype not in _DTYPE:
        raise ValueError(f"x dtype {x.dtype} unsupported")
    _need(Pi, "Pi", torch.float32, (cache.d, cache.d), cache.device)
    _need(codebook, "codebook", torch.float32, (cache.codebook_len,), cache.device)
    if cache.qjl:
        _need(SPiT, "SPiT", torch.float32, (cache.d, cache.d), cache.device)
    desc = cache.desc()
    _check(_lib.tq_quantize_append(ctypes.byref(desc), _ptr(x), _DTYPE[x.dtype], int(pos), int(x.shape[2]),
                                   _ptr(Pi), _ptr(SPiT), _ptr(codebook), _stream(stream)))


def tq_quantize_append_hadamard(cache: PackedCache, x: torch.Tensor, pos: int, signs: torch.Tensor,
                                SPiT: torch.Tensor | None, codebook: torch.Tensor, stream=None) -> None:
    """tq_quantize_append with Pi = H diag(signs) / sqrt(d) applied by a fast Walsh-Hadamard transform;
    signs: [d] float32 of +-1, d a power of two in [32, 256]."""
    if x.dim() != 4 or x.shape[0] != cache.n_seq or x.shape[1] != cache.n_kv_heads or x.shape[3] != cache.d:
        raise ValueError(f"x must be [{cache.n_seq}, {cache.n_kv_heads}, T, {cache.d}], got {tuple(x.shape)}")
    _need(x, "x", device=cache.device)
    if x.dtype not in _DTYPE:
        raise ValueError(f"x dtype {x.dtype} unsupported")
    _need(signs, "signs", torch.float32, (cache.d,), cache.device)
    _need(codebook, "codebook", torch.float32, (cache.codebook_len,), cache.device)
    if cache.qjl:
        _need(SPiT, "SPiT", torch.float32, (cache.d, cache.d), cache.device)
    desc = cache.desc()
    _check(_lib.tq_quantize_append_hadamard(ctypes.byref(desc), _ptr(x), _DTYPE[x.dtype], int(pos), int(x.shape[2]),
                                            _ptr(signs), _ptr(SPiT), _ptr(codebook), _stream(stream)))


def tq_logits_workspace_size(cache: PackedCache, n_q_heads: int) -> int:
    desc = cache.desc()
    return int(_lib.tq_logits_workspace_size(ctypes.byref(desc), n_q_heads))


def tq_logits(cache: PackedCache, q: torch.Tensor, n_tokens: int, Pi: torch.Tensor, S: torch.Tensor,
              codebook: torch.Tensor, logits: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    """q: [n_seq, n_q_heads, d] float32 -> logits [n_seq, n_q_heads, n_tokens] float32."""
    if q.dim() != 3 or q.shape[0] != cache.n_seq or q.shape[2] != cache.d:
        raise ValueError(f"q must be [{cache.n_seq}, H_q, {cache.d}], got {tuple(q.shape)}")
    hq = q.shape[1]
    _need(q, "q", torch.float32, device=cache.device)
    _need(Pi, "Pi", torch.float32, (cache.d, cache.d), cache.device)
    _need(S, "S", torch.float32, (cache.d, cache.d), cache.device)
    _need(codebook, "codebook", torch.float32, (cache.codebook_len,), cache.device)
    if logits is None:
        logits = torch.empty((cache.n_seq, hq, n_tokens), dtype=torch.float32, device=cache.device)
    _need(logits, "logits", torch.float32, (cache.n_seq, hq, n_tokens), cache.device)
    need = tq_logits_workspace_size(cache, hq)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=cache.device)
    desc = cache.desc()
    _check(_lib.tq_logits(ctypes.byref(desc), _ptr(q), hq, int(n_tokens), _ptr(Pi), _ptr(S), _ptr(codebook),
                          _ptr(logits), _ptr(workspace), workspace.numel() * workspace.element_size(),
                          _stream(stream)))
    return logits


def tq_attend_workspace_size(cache: PackedCache, n_q_heads: int, n_tokens: int) -> int:
    desc = cache.desc()
    return int(_lib.tq_attend_workspace_size(ctypes.byref(desc), n_q_heads, int(n_tokens)))


def tq_attend_v(cache: PackedCache, logits: torch.Tensor, scale: float, n_tokens: int, Pi: torch.Tensor,
                codebook: torch.Tensor, out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """logits [n_seq, H_q, n_tokens] float32 -> out [n_seq, H_q, d] float32."""
    if logits.dim() != 3 or logits.shape[0] != cache.n_seq or logits.shape[2] != n_tokens:
        raise ValueError(f"logits must be [{cache.n_seq}, H_q, {n_tokens}], got {tuple(logits.shape)}")
    hq = logits.shape[1]
    _need(logits, "logits", torch.float32, device=cache.device)
    _need(Pi, "Pi", torch.float32, (cache.d, cache.d), cache.device)
    _need(codebook, "codebook", torch.float32, (cache.codebook_len,), cache.device)
    if out is None:
        out = torch.empty((cache.n_seq, hq, cache.d), dtype=torch.float32, device=cache.device)
    _need(out, "out", torch.float32, (cache.n_seq, hq, cache.d), cache.device)
    need = tq_attend_workspace_size(cache, hq, n_tokens)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=cache.device)
    desc = cache.desc()
    _check(_lib.tq_attend_v(ctypes.byref(desc), _ptr(logits), float(scale), hq, int(n_tokens), _ptr(Pi),
                            _ptr(codebook), _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                            _stream(stream)))
    return out


def tq_attend_v_partial(cache: PackedCache, logits: torch.Tensor, scale: float, n_tokens: int, codebook: torch.Tensor,
                        partial: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """logits [n_seq, H_q, n_tokens] -> the mergeable partial [n_seq * H_q, d + 2] (M, L, A) of these tokens."""
    if logits.dim() != 3 or logits.shape[0] != cache.n_seq or logits.shape[2] != n_tokens:
        raise ValueError(f"logits must be [{cache.n_seq}, H_q, {n_tokens}], got {tuple(logits.shape)}")
    hq = logits.shape[1]
    _need(logits, "logits", torch.float32, device=cache.device)
    _need(codebook, "codebook", torch.float32, (cache.codebook_len,), cache.device)
    if partial is None:
        partial = torch.empty((cache.n_seq * hq, cache.d + 2), dtype=torch.float32, device=cache.device)
    _need(partial, "partial", torch.float32, (cache.n_seq * hq, cache.d + 2), cache.device)
    if workspace is None:
        workspace = torch.empty(max(tq_attend_workspace_size(cache, hq, n_tokens), 256), dtype=torch.uint8,
                                device=cache.device)
    desc = cache.desc()
    _check(_lib.tq_attend_v_partial(ctypes.byref(desc), _ptr(logits), float(scale), hq, int(n_tokens), _ptr(codebook),
                                    _ptr(partial), _ptr(workspace), workspace.numel() * workspace.element_size(),
                                    _stream(stream)))
    return partial


def tq_attend_merge(partials: torch.Tensor, Pi: torch.Tensor, out: torch.Tensor | None = None,
                    stream=None) -> torch.Tensor:
    """partials [rows, n_parts, d + 2] (M, L, A of token ranges) -> out [rows, d]."""
    if partials.dim() != 3:
        raise ValueError(f"partials must be [rows, n_parts, d + 2], got {tuple(partials.shape)}")
    rows, n_parts, d2 = partials.shape
    d = d2 - 2
    _need(partials, "partials", torch.float32)
    _need(Pi, "Pi", torch.float32, (d, d), partials.device)
    if out is None:
        out = torch.empty((rows, d), dtype=torch.float32, device=partials.device)
    _need(out, "out", torch.float32, (rows, d), partials.device)
    _check(_lib.tq_attend_merge(_ptr(partials), n_parts, rows, d, _ptr(Pi), _ptr(out), _stream(stream)))
    return out


def tq_nn_merge(part_scores: torch.Tensor, part_ids: torch.Tensor, scores: torch.Tensor | None = None,
                ids: torch.Tensor | None = None, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """part_scores / part_ids [n_parts, n_q, k] (sorted per-shard top-k lists, global ids) ->
    the merged top-k (scores [n_q, k], ids [n_q, k])."""
    if part_scores.dim() != 3 or part_ids.shape != part_scores.shape:
        raise ValueError("part_scores and part_ids must both be [n_parts, n_q, k]")
    n_parts, nq, k = part_scores.shape
    _need(part_scores, "part_scores", torch.float32)
    _need(part_ids, "part_ids", torch.int64, device=part_scores.device)
    if scores is None:
        scores = torch.empty((nq, k), dtype=torch.float32, device=part_scores.device)
    if ids is None:
        ids = torch.empty((nq, k), dtype=torch.int64, device=part_scores.device)
    _need(scores, "scores", torch.float32, (nq, k), part_scores.device)
    _need(ids, "ids", torch.int64, (nq, k), part_scores.device)
    _check(_lib.tq_nn_merge(_ptr(part_scores), _ptr(part_ids), n_parts, nq, k, _ptr(scores), _ptr(ids),
                            _stream(stream)))
    return scores, ids


def tq_decode_workspace_size(kcache: PackedCache, vcache: PackedCache, n_q_heads: int, n_tokens: int) -> int:
    kd, vd = kcache.desc(), vcache.desc()
    return int(_lib.tq_decode_workspace_size(ctypes.byref(kd), ctypes.byref(vd), n_q_heads, int(n_tokens)))


def tq_decode_attend(kcache: PackedCache, vcache: PackedCache, q: torch.Tensor, n_tokens: int, scale: float,
                     Pi: torch.Tensor, S: torch.Tensor, codebook_k: torch.Tensor, codebook_v: torch.Tensor,
                     out: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """q [n_seq, H_q, d] float32 -> out [n_seq, H_q, d] float32 (logits, softmax and values in one call)."""
    if q.dim() != 3 or q.shape[0] != kcache.n_seq or q.shape[2] != kcache.d:
        raise ValueError(f"q must be [{kcache.n_seq}, H_q, {kcache.d}], got {tuple(q.shape)}")
    hq = q.shape[1]
    _need(q, "q", torch.float32, device=kcache.device)
    _need(Pi, "Pi", torch.float32, (kcache.d, kcache.d), kcache.device)
    _need(S, "S", torch.float32, (kcache.d, kcache.d), kcache.device)
    _need(codebook_k, "codebook_k", torch.float32, (kcache.codebook_len,), kcache.device)
    _need(codebook_v, "codebook_v", torch.float32, (vcache.codebook_len,), kcache.device)
    if out is None:
        out = torch.empty((kcache.n_seq, hq, kcache.d), dtype=torch.float32, device=kcache.device)
    _need(out, "out", torch.float32, (kcache.n_seq, hq, kcache.d), kcache.device)
    if workspace is None:
        workspace = torch.empty(max(tq_decode_workspace_size(kcache, vcache, hq, n_tokens), 256), dtype=torch.uint8,
                                device=kcache.device)
    kd, vd = kcache.desc(), vcache.desc()
    _check(_lib.tq_decode_attend(ctypes.byref(kd), ctypes.byref(vd), _ptr(q), hq, int(n_tokens), float(scale),
                                 _ptr(Pi), _ptr(S), _ptr(codebook_k), _ptr(codebook_v), _ptr(out), _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def tq_nn_workspace_size(db: PackedCache, n_queries: int, n_db: int) -> int:
    d = db.desc()
    return int(_lib.tq_nn_workspace_size(ctypes.byref(d), int(n_queries), int(n_db)))


def tq_nn_search(db: PackedCache, queries: torch.Tensor, n_db: int, Pi: torch.Tensor, S: torch.Tensor,
                 codebook: torch.Tensor, k: int, scores: torch.Tensor | None = None, ids: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """queries [n_q, d] float32 -> (scores [n_q, k] float32, ids [n_q, k] int64): the k database
    vectors of db[0, 0, :n_db] with the largest estimated inner product per query."""
    if queries.dim() != 2 or queries.shape[1] != db.d:
        raise ValueError(f"queries must be [n_q, {db.d}], got {tuple(queries.shape)}")
    nq = queries.shape[0]
    _need(queries, "queries", torch.float32, device=db.device)
    _need(Pi, "Pi", torch.float32, (db.d, db.d), db.device)
    _need(S, "S", torch.float32, (db.d, db.d), db.device)
    _need(codebook, "codebook", torch.float32, (db.codebook_len,), db.device)
    if scores is None:
        scores = torch.empty((nq, k), dtype=torch.float32, device=db.device)
    if ids is None:
        ids = torch.empty((nq, k), dtype=torch.int64, device=db.device)
    _need(scores, "scores", torch.float32, (nq, k), db.device)
    _need(ids, "ids", torch.int64, (nq, k), db.device)
    if workspace is None:
        workspace = torch.empty(max(tq_nn_workspace_size(db, nq, n_db), 256), dtype=torch.uint8, device=db.device)
    d = db.desc()
    _check(_lib.tq_nn_search(ctypes.byref(d), _ptr(queries), nq, int(n_db), _ptr(Pi), _ptr(S), _ptr(codebook),
                             int(k), _ptr(scores), _ptr(ids), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)))
    return scores, ids


def tq_workspace_status(workspace: torch.Tensor, stream=None) -> None:
    _check(_lib.tq_workspace_status(_ptr(workspace), _stream(stream)))


def tq_last_error() -> str:
    return _lib.tq_last_error().decode()


def tq_debug_inject(status: int, count: int) -> None:
    _lib.tq_debug_inject(int(status), int(count))


def tq_debug_stall_consumers(tries: int) -> None:
    """Test hook: softmax.V consumers wait `tries` times on a barrier nothing completes (0 disarms)."""
    _lib.tq_debug_stall_consumers(int(tries))


def raw_lib() -> ctypes.CDLL:
    """The loaded library (tests call the C entry points directly through it)."""
    return _lib
