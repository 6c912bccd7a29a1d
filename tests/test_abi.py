"""The C-ABI library loads and exports every entry point the header declares;
host-side argument validation rejects bad calls before touching the GPU."""
import ctypes
import glob
import os
import re


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "sparse_decode_attention_spkv_b200", "libspkv.so")


def _declared():
    names = []
    for hdr in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(hdr).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^[A-Za-z_][\w \*]*?\b(spkv_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_hot_path():
    names = _declared()
    for required in ["spkv_score", "spkv_write_compact", "spkv_decode_attn", "spkv_prefill_attn",
                     "spkv_decode_append", "spkv_ring_write"]:
        assert required in names


def test_library_exports_every_declared_symbol():
    assert os.path.exists(LIB), "build the library first"
    lib = ctypes.CDLL(LIB)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_argument_validation_without_gpu():
    from sparse_decode_attention_spkv_b200 import spkv as S
    assert S.lib.spkv_version() >= 100
    assert S.status_str(S.ERR_CAPACITY) == "cache capacity exhausted"
    # NULL params, bad head_dim, bad group size, NaN threshold: rejected on the host
    assert S.lib.spkv_score(None, None, 4, None, None, None, None, None, None, None) == S.ERR_ARG
    bad = [S.make_params(1, 4, 2, 96, 256, 64, 128, 0.5, S.F32),
           S.make_params(1, 6, 2, 64, 256, 64, 128, 0.5, S.F32),
           S.make_params(1, 4, 2, 64, 256, 64, 128, float("nan"), S.F32),
           S.make_params(1, 4, 2, 64, 256, 64, 0, 0.5, S.F32),
           S.make_params(0, 4, 2, 64, 256, 64, 128, 0.5, S.BF16)]
    for p in bad:
        assert S.lib.spkv_score(ctypes.byref(p), None, 4, None, None, None, None, None, None,
                                None) == S.ERR_ARG
    good = S.make_params(1, 4, 2, 64, 256, 64, 128, 0.5, S.F32)
    # h and W1 must be 16-byte aligned (vector and tensor-map loads)
    assert S.lib.spkv_score(ctypes.byref(good), 8, 4, 16, 16, 16, 16, None, 16, None) == S.ERR_ARG
    assert S.lib.spkv_score(ctypes.byref(good), 16, 4, 24, 16, 16, 16, None, 16, None) == S.ERR_ARG
    # zero tokens is a no-op that needs no pointers
    assert S.lib.spkv_score(ctypes.byref(good), None, 0, None, None, None, None, None, None,
                            None) == S.OK
    # missing cache buffers
    cache = S.spkv_cache()
    ring = S.spkv_ring()
    assert S.lib.spkv_decode_attn(ctypes.byref(good), ctypes.byref(cache), ctypes.byref(ring),
                                  None, None, None, None, None, 0, None) == S.ERR_ARG
    assert S.lib.spkv_prefill_attn(ctypes.byref(good), ctypes.byref(cache), ctypes.byref(ring),
                                   None, None, None, 0, 16, None, None, None, 0, None) == S.ERR_ARG
    # misaligned pool pointer
    cache = S.spkv_cache(8, 16, 16, 16, 16, 16, 16, 16, None, 4, 64, 4)
    assert S.lib.spkv_cache_reset(ctypes.byref(good), ctypes.byref(cache), None, None) == S.ERR_ARG
    # page_rows other than 64
    cache = S.spkv_cache(16, 16, 16, 16, 16, 16, 16, 16, None, 4, 32, 4)
    assert S.lib.spkv_cache_reset(ctypes.byref(good), ctypes.byref(cache), None, None) == S.ERR_ARG
    # ring compaction longer than the window, negative gated_from
    cache = S.spkv_cache(16, 16, 16, 16, 16, 16, 16, 16, None, 4, 64, 4)
    ring = S.spkv_ring(16, 16, 16, None)
    assert S.lib.spkv_write_compact(ctypes.byref(good), ctypes.byref(cache), ctypes.byref(ring),
                                    S.SRC_RING, None, None, 16, None, 16, 129, 129, None) == S.ERR_ARG
    assert S.lib.spkv_ring_write(ctypes.byref(good), ctypes.byref(ring), 16, 16, 16, None, -1, 16, 4,
                                 4, None) == S.ERR_ARG
    assert S.lib.spkv_ring_write(ctypes.byref(good), ctypes.byref(ring), 16, 16, None, None, 0, 16, 4,
                                 4, None) == S.ERR_ARG
    # utilities kept in the cache: the compaction needs them; the ring's pending
    # utilities need u_src / u_new; re-threshold needs the cache's utilities
    cache_u = S.spkv_cache(16, 16, 16, 16, 16, 16, 16, 16, 16, 4, 64, 4)
    assert S.lib.spkv_write_compact(ctypes.byref(good), ctypes.byref(cache_u), None, S.SRC_CHUNK,
                                    16, 16, 16, None, 16, 4, 4, None) == S.ERR_ARG
    ring_u = S.spkv_ring(16, 16, 16, 16)
    assert S.lib.spkv_ring_write(ctypes.byref(good), ctypes.byref(ring_u), 16, 16, 16, None, 0, 16,
                                 4, 4, None) == S.ERR_ARG
    assert S.lib.spkv_decode_append(ctypes.byref(good), ctypes.byref(cache), ctypes.byref(ring_u),
                                    16, 16, 16, 16, None, 1, None) == S.ERR_ARG
    assert S.lib.spkv_cache_rethreshold(ctypes.byref(good), ctypes.byref(cache), None,
                                        ctypes.c_float(0.6), 16, 1 << 20, None) == S.ERR_ARG
    assert S.lib.spkv_cache_rethreshold(ctypes.byref(good), ctypes.byref(cache_u), None,
                                        ctypes.c_float(float("nan")), 16, 1 << 20, None) == S.ERR_ARG
    assert S.lib.spkv_rethreshold_workspace_bytes(ctypes.byref(good), ctypes.byref(cache_u)) > 0
    # attention before the step's update: needs the new rows; fp32 is not supported
    assert S.lib.spkv_decode_attn_before_append(ctypes.byref(good), ctypes.byref(cache),
                                                ctypes.byref(ring), 16, 16, None, 16, 16, None,
                                                16, 1 << 20, 0, None) == S.ERR_ARG
    assert S.lib.spkv_decode_attn_before_append(ctypes.byref(good), ctypes.byref(cache),
                                                ctypes.byref(ring), 16, 16, 16, 8, 16, None,
                                                16, 1 << 20, 0, None) == S.ERR_ARG
    assert S.lib.spkv_decode_attn_before_append(ctypes.byref(good), ctypes.byref(cache),
                                                ctypes.byref(ring), 16, 16, 16, 16, 16, None,
                                                16, 1 << 20, 2, None) == S.ERR_ARG
    assert S.lib.spkv_decode_attn_before_append_supported(ctypes.byref(good)) == 0
    assert S.lib.spkv_decode_attn_before_append_supported(None) == 0
    assert S.lib.spkv_decode_attn_before_append(ctypes.byref(good), ctypes.byref(cache),
                                                ctypes.byref(ring), 16, 16, 16, 16, 16, None,
                                                16, 1 << 20, S.DECODE_STATE_SETTLED,
                                                None) == S.ERR_UNSUPPORTED


def test_noalloc_argument_checks_match_decode_attn():
    """The no-allocation decode applies spkv_decode_attn's argument rules (host side,
    before anything is enqueued): the same bad calls give the same status."""
    from sparse_decode_attention_spkv_b200 import spkv as S
    good = S.make_params(2, 8, 2, 128, 256, 64, 128, 0.5, S.BF16)
    nan_tau = S.make_params(2, 8, 2, 128, 256, 64, 128, float("nan"), S.BF16)
    ring = S.spkv_ring(16, 16, 16, None)
    ok_cache = S.spkv_cache(16, 16, 16, 16, 16, 16, 16, 16, None, 4, 64, 4)
    bad_caches = [S.spkv_cache(16, 16, 16, 16, 16, 16, 16, 16, None, 0, 64, 4),   # no pages
                  S.spkv_cache(16, 16, 16, 16, 16, 16, 16, 16, None, 4, 64, 0),   # no table
                  S.spkv_cache(16, 16, 16, 16, 16, None, 16, 16, None, 4, 64, 4),  # count_prev
                  S.spkv_cache(16, 16, 16, 16, 16, 16, None, 16, None, 4, 64, 4)]  # pool_top
    calls = [(good, c, ring, 16, 16, 16) for c in bad_caches]
    calls += [(nan_tau, ok_cache, ring, 16, 16, 16),     # NaN threshold
              (good, ok_cache, ring, 8, 16, 16),         # misaligned query
              (good, ok_cache, ring, 16, None, 16),      # no positions
              (good, ok_cache, S.spkv_ring(16, 16, None, None), 16, 16, 16)]  # no gates
    for p, c, r, q, t, o in calls:
        a = S.lib.spkv_decode_attn(ctypes.byref(p), ctypes.byref(c), ctypes.byref(r), q, t, o, None,
                                   16, 1 << 30, None)
        b = S.lib.spkv_decode_attn_noalloc(ctypes.byref(p), ctypes.byref(c), ctypes.byref(r), q, t,
                                           o, None, None)
        assert a == b == S.ERR_ARG, (a, b)


def test_sequence_split_argument_checks():
    """Partial decode and merge of a split sequence: argument errors on the host."""
    from sparse_decode_attention_spkv_b200 import spkv as S
    bf = S.make_params(2, 8, 2, 128, 256, 64, 128, 0.5, S.BF16)
    f32 = S.make_params(2, 8, 2, 128, 256, 64, 128, 0.5, S.F32)
    cache = S.spkv_cache(16, 16, 16, 16, 16, 16, 16, 16, None, 4, 64, 4)
    ring = S.spkv_ring(16, 16, 16, None)
    part = S.lib.spkv_decode_attn_partial
    r = ctypes.byref
    assert part(r(bf), r(cache), r(ring), 16, 16, 2, 16, 16, 16, 1 << 30, None) == S.ERR_ARG  # flag
    assert part(r(bf), None, None, 16, 16, 0, 16, 16, 16, 1 << 30, None) == S.ERR_ARG  # no keys
    assert part(r(bf), None, None, 16, 16, S.SLICE_WINDOW, 16, 16, 16, 1 << 30,
                None) == S.ERR_ARG  # window without a ring
    assert part(r(bf), r(cache), None, 16, 16, 0, 16, None, 16, 1 << 30, None) == S.ERR_ARG  # lse
    assert part(r(bf), r(cache), None, 16, 16, 0, 8, 16, 16, 1 << 30, None) == S.ERR_ARG  # align
    assert part(r(f32), r(cache), None, 16, 16, 0, 16, 16, 16, 1 << 30,
                None) == S.ERR_UNSUPPORTED
    assert S.lib.spkv_decode_attn_partial_supported(r(f32)) == 0
    merge = S.lib.spkv_decode_merge
    assert merge(r(bf), 0, 16, 16, 16, None, None) == S.ERR_ARG      # no part
    assert merge(r(bf), 2, None, 16, 16, None, None) == S.ERR_ARG
    assert merge(r(bf), 2, 16, 16, 8, None, None) == S.ERR_ARG       # misaligned output


def test_prefill_workspace_checks():
    """The optional tile-counter workspace of the prefill attention: too small or
    misaligned is an argument error, found before anything is launched."""
    from sparse_decode_attention_spkv_b200 import spkv as S
    bf = S.make_params(2, 8, 2, 128, 256, 64, 128, 0.5, S.BF16)
    cache = S.spkv_cache(16, 16, 16, 16, 16, 16, 16, 16, None, 4, 64, 4)
    ring = S.spkv_ring(16, 16, 16, None)
    pre = S.lib.spkv_prefill_attn
    r = ctypes.byref
    n = S.PREFILL_WORKSPACE_BYTES
    assert pre(r(bf), r(cache), r(ring), 16, 16, 16, 0, 128, 16, None, 16, n - 1, None) == S.ERR_ARG
    assert pre(r(bf), r(cache), r(ring), 16, 16, 16, 0, 128, 16, None, 8, n, None) == S.ERR_ARG
    # an empty chunk is a no-op whatever the workspace
    assert pre(r(bf), r(cache), r(ring), 16, 16, 16, 0, 0, 16, None, 8, 0, None) == S.OK
