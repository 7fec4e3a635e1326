"""C-ABI library on the host (no GPU needed): it loads, exports every symbol
that include/tq.h declares, computes its record sizes and codebooks, and
rejects bad arguments with the right status before launching anything.

The argument-check tests pass placeholder device addresses; each such call
must fail in the host checks. As a guard, a fault is armed with
tq_debug_inject first, so a call that wrongly got past the checks returns the
injected status instead of launching a kernel.
"""

import ctypes

import numpy as np
import pytest

import kv_cache_vector_quantize_b200 as tqb
from oracle import codebook as ocb
from oracle import turboquant as otq

lib = tqb.raw_lib()
FAKE = 0x7F0000000000     # 256-byte aligned placeholder address (never dereferenced)


def _desc(d=128, bits=2, qjl=1, n_seq=1, heads=2, cap=64, records=FAKE, norm=FAKE + 4096, rnorm=FAKE + 8192):
    return tqb.TqCacheDesc(d, bits, qjl, n_seq, heads, 0, cap, records, norm, rnorm if qjl else None)


@pytest.fixture(autouse=True)
def _guard():
    tqb.tq_debug_inject(tqb.TQ_ERR_CUDA, 1000)   # any call that passes the checks returns TQ_ERR_CUDA
    yield
    tqb.tq_debug_inject(tqb.TQ_OK, 0)


def test_every_declared_symbol_is_exported():
    names = tqb.declared_symbols()
    assert len(names) >= 11
    for n in names:
        assert hasattr(lib, n), n


@pytest.mark.parametrize("d,bits,qjl", [(8, 1, 1), (128, 2, 1), (128, 3, 0), (200, 3, 1), (200, 4, 0), (256, 4, 1)])
def test_record_words_match_layout(d, bits, qjl):
    assert tqb.tq_record_words(d, bits, qjl) == otq.record_words(d, bits, bool(qjl))


def test_record_words_rejects_unsupported():
    for d, bits in ((7, 2), (12, 2), (264, 2), (128, 0), (128, 5)):
        assert lib.tq_record_words(d, bits, 1) == -1


@pytest.mark.parametrize("d", [8, 64, 128, 200, 256])
def test_codebook_fit_matches_oracle_bit_exactly(d):
    # The library integrates the law with the Wallis recurrence; the oracle with
    # the regularized incomplete beta function. After rounding to float32 the two
    # Lloyd-Max fixed points must be the same numbers.
    for bits in (1, 2, 3, 4):
        got = tqb.tq_codebook_fit(d, bits).numpy()
        want = ocb.fit_codebook(d, bits)[0]
        assert np.array_equal(got, want), (d, bits, got - want)


def test_codebook_fit_more_levels_and_small_d():
    for d, bits in ((128, 5), (128, 6), (3, 3), (5, 2)):
        got = tqb.tq_codebook_fit(d, bits).numpy()
        want = ocb.fit_codebook(d, bits)[0]
        assert np.allclose(got, want, rtol=0, atol=2e-7 * np.abs(want).max()), (d, bits)
    with pytest.raises(tqb.TQError) as e:
        tqb.tq_codebook_fit(2, 2)
    assert e.value.status == tqb.TQ_ERR_UNSUPPORTED


def _q(desc, x=FAKE, pos=0, n=8, Pi=FAKE, SPiT=FAKE, cb=FAKE, dtype=0):
    return lib.tq_quantize_append(ctypes.byref(desc) if desc is not None else None, x, dtype, pos, n, Pi, SPiT, cb, None)


def test_quantize_hadamard_argument_checks():
    def qh(desc, x=FAKE, pos=0, n=8, signs=FAKE, SPiT=FAKE, cb=FAKE, dtype=0):
        return lib.tq_quantize_append_hadamard(ctypes.byref(desc) if desc is not None else None, x, dtype, pos, n,
                                               signs, SPiT, cb, None)
    assert qh(None) == tqb.TQ_ERR_INVALID
    for d in (8, 16, 96, 200, 512):          # not a power of two in [32, 256] (or an invalid cache)
        assert qh(_desc(d=d)) in (tqb.TQ_ERR_UNSUPPORTED, tqb.TQ_ERR_INVALID), d
    assert qh(_desc(d=200)) == tqb.TQ_ERR_UNSUPPORTED
    assert qh(_desc(), dtype=7) == tqb.TQ_ERR_INVALID
    assert qh(_desc(), pos=-1) == tqb.TQ_ERR_INVALID
    assert qh(_desc(cap=16), pos=10, n=8) == tqb.TQ_ERR_CAPACITY
    assert qh(_desc(), n=0) == tqb.TQ_OK                     # no-op, nothing launched
    assert qh(_desc(), signs=None) == tqb.TQ_ERR_INVALID
    assert qh(_desc(), cb=None) == tqb.TQ_ERR_INVALID
    assert qh(_desc(qjl=1), SPiT=None) == tqb.TQ_ERR_INVALID
    assert qh(_desc(qjl=0), SPiT=None) == tqb.TQ_ERR_CUDA    # values need no SPiT: checks pass, injected error
    for d in (32, 64, 128, 256):
        assert qh(_desc(d=d)) == tqb.TQ_ERR_CUDA            # every check passes: the injected launch error


def test_quantize_argument_checks():
    assert _q(None) == tqb.TQ_ERR_INVALID
    assert _q(_desc(d=12)) == tqb.TQ_ERR_UNSUPPORTED
    assert _q(_desc(bits=5)) == tqb.TQ_ERR_UNSUPPORTED
    assert _q(_desc(cap=64), pos=60, n=5) == tqb.TQ_ERR_CAPACITY
    assert "capacity" in tqb.tq_last_error()
    assert _q(_desc(records=FAKE + 4)) == tqb.TQ_ERR_INVALID
    assert _q(_desc(), dtype=7) == tqb.TQ_ERR_INVALID
    assert _q(_desc(), SPiT=None) == tqb.TQ_ERR_INVALID
    assert _q(_desc(qjl=0), SPiT=None) == tqb.TQ_ERR_CUDA          # passes the checks -> injected
    assert _q(_desc(), n=0) == tqb.TQ_OK                           # nothing to do, nothing launched
    d = _desc()
    d.rnorm = None
    assert _q(d) == tqb.TQ_ERR_INVALID


def _lg(desc, hq=4, n=8, ws=FAKE, ws_bytes=1 << 20):
    return lib.tq_logits(ctypes.byref(desc), FAKE, hq, n, FAKE, FAKE, FAKE, FAKE, ws, ws_bytes, None)


def test_logits_argument_checks():
    assert _lg(_desc(qjl=0)) == tqb.TQ_ERR_INVALID
    assert _lg(_desc(heads=2), hq=3) == tqb.TQ_ERR_INVALID
    assert _lg(_desc(cap=64), n=65) == tqb.TQ_ERR_CAPACITY
    assert _lg(_desc(), ws=FAKE + 16) == tqb.TQ_ERR_WORKSPACE
    assert _lg(_desc(), ws_bytes=16) == tqb.TQ_ERR_WORKSPACE
    assert _lg(_desc(), n=0) == tqb.TQ_OK                           # nothing to scan
    assert _lg(_desc()) == tqb.TQ_ERR_CUDA                         # passes the checks -> injected
    # status header + Pi q and S q (4 query heads) ...
    proj = 256 + 2 * 4 * 4 * 128
    assert lib.tq_logits_workspace_size(ctypes.byref(_desc(bits=3)), 4) == proj
    # ... and, for grouped queries on 1- or 2-bit codes, a 128 KB table block per
    # (KV head, block of up to 4 query heads) plus one float scale per query head (256-byte aligned)
    assert lib.tq_logits_workspace_size(ctypes.byref(_desc()), 4) == proj + 2 * 131072 + 256
    assert lib.tq_logits_workspace_size(ctypes.byref(_desc(heads=1)), 4) == 256 + 2 * 4 * 4 * 128 + 131072 + 256
    assert lib.tq_logits_workspace_size(ctypes.byref(_desc(heads=4)), 4) == proj   # one query head per KV head


def test_attend_argument_checks():
    def call(desc, hq=4, n=8, scale=0.1, ws_bytes=1 << 20):
        return lib.tq_attend_v(ctypes.byref(desc), FAKE, ctypes.c_float(scale), hq, n, FAKE, FAKE, FAKE, FAKE,
                               ws_bytes, None)
    assert call(_desc(qjl=1)) == tqb.TQ_ERR_INVALID
    assert call(_desc(qjl=0), hq=3) == tqb.TQ_ERR_INVALID
    assert call(_desc(qjl=0), scale=float("nan")) == tqb.TQ_ERR_INVALID
    assert call(_desc(qjl=0), ws_bytes=8) == tqb.TQ_ERR_WORKSPACE
    assert call(_desc(qjl=0)) == tqb.TQ_ERR_CUDA                   # passes the checks -> injected


def test_decode_attend_argument_checks():
    def call(kd, vd, hq=2, n=8, scale=0.1, ws_bytes=1 << 24, q=FAKE):
        return lib.tq_decode_attend(ctypes.byref(kd), ctypes.byref(vd), q, hq, n, ctypes.c_float(scale), FAKE, FAKE,
                                    FAKE, FAKE, FAKE, FAKE, ws_bytes, None)
    k, v = _desc(qjl=1), _desc(qjl=0, records=FAKE + (1 << 20), norm=FAKE + (2 << 20))
    assert call(v, v) == tqb.TQ_ERR_INVALID                        # keys must carry the sign field
    assert call(k, k) == tqb.TQ_ERR_INVALID                        # values must not
    assert call(k, _desc(qjl=0, heads=4)) == tqb.TQ_ERR_INVALID    # different KV head counts
    assert call(k, _desc(qjl=0, d=64)) == tqb.TQ_ERR_INVALID       # different head dimensions
    assert call(k, v, hq=3) == tqb.TQ_ERR_INVALID
    assert call(k, _desc(qjl=0, cap=16), n=17) == tqb.TQ_ERR_CAPACITY
    assert call(k, v, scale=float("inf")) == tqb.TQ_ERR_INVALID
    assert call(k, v, q=None) == tqb.TQ_ERR_INVALID
    assert call(k, v, ws_bytes=64) == tqb.TQ_ERR_WORKSPACE
    assert call(k, v) == tqb.TQ_ERR_CUDA                           # passes the checks -> injected
    # one query head per KV head, d = 128, 2-bit key codes: status | Pi q | S q | partials of 512-token chunks
    rows, nt = 2, 1000
    fused = 256 + 2 * rows * 128 * 4 + rows * 2 * 130 * 4
    assert lib.tq_decode_workspace_size(ctypes.byref(k), ctypes.byref(v), 2, nt) == fused
    # grouped queries: status | logits | the tq_logits and tq_attend_v workspaces
    lg = (4 * nt * 4 + 255) // 256 * 256
    ws_l = (lib.tq_logits_workspace_size(ctypes.byref(k), 4) + 255) // 256 * 256
    ws_a = lib.tq_attend_workspace_size(ctypes.byref(v), 4, nt)
    assert lib.tq_decode_workspace_size(ctypes.byref(k), ctypes.byref(v), 4, nt) == 256 + lg + ws_l + ws_a
    assert lib.tq_decode_workspace_size(ctypes.byref(k), ctypes.byref(_desc(qjl=0, heads=4)), 2, nt) == 0


def test_nn_search_argument_checks():
    def call(db, nq=300, ndb=40, k=10, ws_bytes=1 << 26, q=FAKE, Pi=FAKE):
        return lib.tq_nn_search(ctypes.byref(db), q, nq, ndb, Pi, FAKE, FAKE, k, FAKE, FAKE, FAKE, ws_bytes, None)
    db = _desc(d=200, bits=1, heads=1)
    assert call(_desc(d=200, bits=1, qjl=0, heads=1, rnorm=None)) == tqb.TQ_ERR_INVALID   # needs the sign field
    assert call(_desc(d=200, bits=1, heads=2)) == tqb.TQ_ERR_INVALID                      # one stream
    assert call(_desc(d=64, bits=1, heads=1)) == tqb.TQ_ERR_UNSUPPORTED
    assert call(_desc(d=200, bits=4, heads=1)) == tqb.TQ_ERR_UNSUPPORTED
    assert call(db, k=0) == tqb.TQ_ERR_INVALID
    assert call(db, k=17) == tqb.TQ_ERR_INVALID
    assert call(db, nq=-1) == tqb.TQ_ERR_INVALID
    assert call(db, ndb=65) == tqb.TQ_ERR_CAPACITY
    assert call(db, nq=0) == tqb.TQ_OK                                                    # nothing to do
    assert call(db, q=None) == tqb.TQ_ERR_INVALID
    assert call(db, Pi=FAKE + 4) == tqb.TQ_ERR_INVALID                                    # float4 rows
    assert call(_desc(d=200, bits=1, heads=1, norm=FAKE + 4100)) == tqb.TQ_ERR_INVALID     # bulk-copied norms
    assert call(_desc(d=200, bits=1, heads=1, rnorm=FAKE + 8196)) == tqb.TQ_ERR_INVALID
    assert call(db, ws_bytes=1024) == tqb.TQ_ERR_WORKSPACE
    assert call(db) == tqb.TQ_ERR_CUDA                                                    # passes -> injected
    # status | fp16 query rows (padded K 448) | scales | 2 lists of 16 scores and ids per row of (CTAs + blocks - 1)
    up = lambda v: (v + 255) // 256 * 256
    nqb, tiles = 3, 1
    slots = min(nqb * tiles, 256) + nqb - 1
    want = 256 + up(nqb * 128 * 448 * 2) + up(nqb * 128 * 4) + 2 * up(slots * 128 * 2 * 16 * 4)
    assert lib.tq_nn_workspace_size(ctypes.byref(db), 300, 40) == want
    assert lib.tq_nn_workspace_size(ctypes.byref(db), 300, 0) == 256 + up(nqb * 128 * 448 * 2) + up(nqb * 128 * 4)


def test_fault_injection_counts_down():
    tqb.tq_debug_inject(tqb.TQ_ERR_DEVICE, 2)
    assert _q(_desc(qjl=0)) == tqb.TQ_ERR_DEVICE
    assert _q(_desc(qjl=0)) == tqb.TQ_ERR_DEVICE
    assert "injected" in tqb.tq_last_error()
    tqb.tq_debug_inject(tqb.TQ_ERR_CUDA, 1000)


def test_noalloc_checks_arguments_before_its_scratch_size():
    # n_q_heads = 63 is not a multiple of 8 KV heads; the shape is also far beyond the
    # built-in array. The argument error must win, with the same status as tq_attend_v.
    desc = _desc(d=128, bits=3, qjl=0, n_seq=8, heads=8, cap=131072)
    st = lib.tq_attend_v_noalloc(ctypes.byref(desc), FAKE, ctypes.c_float(0.1), 63, 131072, FAKE, FAKE, FAKE, None)
    assert st == tqb.TQ_ERR_INVALID
    assert "multiple" in tqb.tq_last_error()
    st2 = lib.tq_attend_v(ctypes.byref(desc), FAKE, ctypes.c_float(0.1), 63, 131072, FAKE, FAKE, FAKE, FAKE, 1 << 30,
                          None)
    assert st2 == st


def test_attend_workspace_size_does_not_wrap():
    # a descriptor whose partials would overflow a size_t: the size query saturates and
    # the call refuses the shape instead of writing past a small workspace
    desc = _desc(d=256, bits=3, qjl=0, n_seq=2 ** 31 - 1, heads=1, cap=2 ** 62)
    need = lib.tq_attend_workspace_size(ctypes.byref(desc), 2 ** 31 - 1, 2 ** 62)
    assert need == 2 ** 64 - 1
    st = lib.tq_attend_v(ctypes.byref(desc), FAKE, ctypes.c_float(0.1), 2 ** 31 - 1, 2 ** 62, FAKE, FAKE, FAKE, FAKE,
                         1 << 30, None)
    assert st == tqb.TQ_ERR_UNSUPPORTED


@pytest.mark.parametrize("d,bits,n_hi,qjl", [(128, 2, 64, 1), (128, 3, 64, 0), (128, 1, 32, 1), (200, 2, 96, 1),
                                             (64, 3, 32, 0), (256, 2, 224, 1)])
def test_mixed_record_words_match_layout(d, bits, n_hi, qjl):
    from oracle import mixed_rate as omr
    assert tqb.tq_record_words_mixed(d, bits, n_hi, qjl) == omr.record_words(d, bits, n_hi, bool(qjl))
    assert lib.tq_record_words_mixed(d, bits, 0, qjl) == lib.tq_record_words(d, bits, qjl)


def test_mixed_rate_descriptors_checked():
    for d, bits, n_hi in ((128, 2, 48), (128, 2, 128), (128, 2, -32), (128, 4, 32), (64, 2, 96)):
        assert lib.tq_record_words_mixed(d, bits, n_hi, 1) == -1
        desc = tqb.TqCacheDesc(d, bits, 1, 1, 2, n_hi, 64, FAKE, FAKE + 4096, FAKE + 8192)
        st = lib.tq_quantize_append(ctypes.byref(desc), FAKE, 0, 0, 8, FAKE, FAKE, FAKE, None)   # dtype 0: bf16
        assert st == tqb.TQ_ERR_UNSUPPORTED, (d, bits, n_hi)
        assert "n_hi" in tqb.tq_last_error()
    # the nearest-neighbour search takes integer-rate databases only
    desc = tqb.TqCacheDesc(128, 2, 1, 1, 1, 64, 1000, FAKE, FAKE + 4096, FAKE + 8192)
    st = lib.tq_nn_search(ctypes.byref(desc), FAKE, 10, 1000, FAKE, FAKE, FAKE, 10, FAKE, FAKE, FAKE, 1 << 30, None)
    assert st == tqb.TQ_ERR_UNSUPPORTED


def test_merge_and_partial_entry_points_check_arguments():
    # top-k merge: k outside 1..16, no parts, NULL outputs
    assert lib.tq_nn_merge(FAKE, FAKE, 2, 10, 17, FAKE, FAKE, None) == tqb.TQ_ERR_INVALID
    assert lib.tq_nn_merge(FAKE, FAKE, 0, 10, 5, FAKE, FAKE, None) == tqb.TQ_ERR_INVALID
    assert lib.tq_nn_merge(FAKE, FAKE, 2, 10, 5, None, FAKE, None) == tqb.TQ_ERR_INVALID
    assert lib.tq_nn_merge(FAKE, FAKE, 2, 0, 5, None, None, None) == tqb.TQ_OK      # nothing to merge
    # softmax.V merge: unsupported d, no parts, NULL matrix
    assert lib.tq_attend_merge(FAKE, 2, 4, 12, FAKE, FAKE, None) == tqb.TQ_ERR_UNSUPPORTED
    assert lib.tq_attend_merge(FAKE, 0, 4, 128, FAKE, FAKE, None) == tqb.TQ_ERR_INVALID
    assert lib.tq_attend_merge(FAKE, 2, 4, 128, None, FAKE, None) == tqb.TQ_ERR_INVALID
    # partial: the checks of tq_attend_v (a key cache is refused; NULL output), without Pi
    kdesc = _desc(qjl=1)
    assert lib.tq_attend_v_partial(ctypes.byref(kdesc), FAKE, ctypes.c_float(0.1), 2, 8, FAKE, FAKE, FAKE, 1 << 20,
                                   None) == tqb.TQ_ERR_INVALID
    vdesc = _desc(qjl=0, bits=3)
    assert lib.tq_attend_v_partial(ctypes.byref(vdesc), FAKE, ctypes.c_float(0.1), 2, 8, FAKE, None, FAKE, 1 << 20,
                                   None) == tqb.TQ_ERR_INVALID
    # valid arguments reach the (injected) launch failure
    assert lib.tq_attend_v_partial(ctypes.byref(vdesc), FAKE, ctypes.c_float(0.1), 2, 8, FAKE, FAKE, FAKE, 1 << 20,
                                   None) == tqb.TQ_ERR_CUDA
