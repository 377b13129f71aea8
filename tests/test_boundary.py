"""The C ABI without a GPU: the library loads, exports every declared entry point, and rejects bad
arguments on the host before anything is launched."""
import ctypes
import os
import re

import pytest

import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def h():
    import long_context_compressed_05_b200 as h
    from long_context_compressed_05_b200 import build
    build.build()
    return h


def declared_functions():
    src = open(os.path.join(ROOT, "include", "hca_csa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return set(re.findall(r"\b([a-z_0-9]+)\s*\(", src)) - {"if", "sizeof"}


def test_header_and_binding_agree(h):
    decl = declared_functions()
    assert decl == set(h.EXPORTS), decl ^ set(h.EXPORTS)


def test_library_exports_every_declared_symbol(h):
    lib = h.load()
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings_and_version(h):
    assert h.hcsa_version() >= 100
    for code in range(10):
        assert h.hcsa_status_string(code)
    assert h.hcsa_status_string(99) == "unknown status"


def _params(h, **kw):
    spec = synth.PREFILL["csa_bf16_t131072"]
    p = h.params_for(spec)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


FAKE = 0x10000  # an aligned address that is never dereferenced (errors are found before any launch)


def test_argument_errors_return_before_launch(h):
    lib = h.load()
    p = _params(h)
    P = ctypes.byref(p)
    V = ctypes.c_void_p
    # null tensor
    assert lib.csa_compress(P, None, 1024, V(FAKE), 1024, V(FAKE), 64, V(FAKE), V(FAKE), V(FAKE), None) == 1
    # misaligned pointer / leading dimension
    assert lib.csa_compress(P, V(FAKE + 2), 36960, V(FAKE), 36960, V(FAKE), 36960, V(FAKE), V(FAKE), V(FAKE),
                            None) == 4
    assert lib.csa_compress(P, V(FAKE), 1025, V(FAKE), 36960, V(FAKE), 36960, V(FAKE), V(FAKE), V(FAKE), None) == 4
    # bad dtype / shape
    pd = _params(h, dtype=7)
    assert lib.csa_compress(ctypes.byref(pd), V(FAKE), 36960, V(FAKE), 36960, V(FAKE), 36960, V(FAKE), V(FAKE),
                            V(FAKE), None) == 3
    ps = _params(h, dh=100)
    assert lib.hca_attend(ctypes.byref(ps), V(FAKE), 36960, V(FAKE), 36960, V(FAKE), V(FAKE), None, 0, None) == 2
    pw = _params(h, width=2)   # width < m
    assert lib.hca_compress(ctypes.byref(pw), V(FAKE), 36960, V(FAKE), 36960, V(FAKE), V(FAKE), None) == 2
    # workspace too small
    assert lib.csa_index_topk(P, V(FAKE), 36960, V(FAKE), 36960, V(FAKE), V(FAKE), V(FAKE), 1024, None) == 5
    # decode: window smaller than the pool width, and missing cache pointers
    pdc = _params(h, B=2, n_cap=16, window=4)
    cache = h.make_cache(None, None, None)
    cache.entries = cache.win_kv = cache.ring_g = cache.idx_keys = cache.ring_ki = FAKE
    assert lib.hcsa_cache_append(ctypes.byref(pdc), ctypes.byref(cache), V(FAKE), V(FAKE), 1024, V(FAKE), 1024,
                                 V(FAKE), 64, V(FAKE), None) == 2
    pdc.window = 128
    cache.ring_ki = None
    assert lib.csa_decode_index_topk(ctypes.byref(pdc), ctypes.byref(cache), V(FAKE), V(FAKE), 2048, V(FAKE), 32,
                                     V(FAKE), V(FAKE), 1 << 30, None) == 1


def test_workspace_sizes(h):
    p = _params(h)
    assert h.hcsa_workspace_bytes(p, h.OP_CSA_INDEX_TOPK) >= 131072 * 32768 * 4
    pd = _params(h, B=32, n_cap=65536)
    assert h.hcsa_workspace_bytes(pd, h.OP_CSA_DECODE_INDEX_TOPK) >= 32 * 65536 * 4
    assert h.hcsa_proj_cols(p, h.KIND_CSA) == 36960
    assert h.hcsa_proj_cols(p, h.KIND_HCA) == 2048 + 32768


def test_noalloc_refuses_requests_beyond_its_scratch(h):
    """The allocation-free decode indexer checks its fixed 8 MiB scratch before any launch: 32 sequences of
    65536 entries need 8 MiB of scores alone (plus the multi-block select's scratch)."""
    lib = h.load()
    V = ctypes.c_void_p
    p = _params(h, B=32, n_cap=65536)
    assert h.hcsa_workspace_bytes(p, h.OP_CSA_DECODE_INDEX_TOPK) > 8 << 20
    cache = h.make_cache(None, None, None)
    cache.entries = cache.win_kv = cache.ring_g = cache.idx_keys = cache.ring_ki = FAKE
    assert lib.csa_decode_index_topk_noalloc(ctypes.byref(p), ctypes.byref(cache), V(FAKE), V(FAKE), 2048,
                                             V(FAKE), 32, V(FAKE), None) == 5


def test_row_range_is_checked_before_launch(h):
    """Prefill row ranges: row0 a multiple of 128, row1 a multiple of 128 or T, row0 <= row1 <= T."""
    lib = h.load()
    V = ctypes.c_void_p
    for r0, r1 in [(64, 256), (0, 200), (256, 128), (0, 131072 + 128), (-128, 0)]:
        p = _params(h, row0=r0, row1=r1)
        assert lib.csa_compress(ctypes.byref(p), V(FAKE), 36960, V(FAKE), 36960, V(FAKE), 36960, V(FAKE),
                                V(FAKE), V(FAKE), None) == 2, (r0, r1)
        assert lib.hca_attend(ctypes.byref(p), V(FAKE), 36960, V(FAKE), 36960, V(FAKE), V(FAKE), None, 0,
                              None) == 2, (r0, r1)


def test_shard_and_lowprec_arguments_are_checked_before_launch(h):
    lib = h.load()
    V = ctypes.c_void_p
    cache = h.Cache(entries=FAKE, idx_keys=FAKE, win_kv=FAKE, ring_g=FAKE, ring_ki=FAKE)
    C = ctypes.byref(cache)
    # a non-zero entry offset on an unsharded cache
    p = _params(h, T=0, B=2, n_cap=1000, ent0=500)
    assert lib.hcsa_cache_append(ctypes.byref(p), C, V(FAKE), V(FAKE), 36960, V(FAKE), 36960, V(FAKE), 36960,
                                 V(FAKE), None) == 2
    # the *_shard calls need a sharded cache
    p = _params(h, T=0, B=2, n_cap=1000)
    assert lib.csa_decode_index_topk_shard(ctypes.byref(p), C, V(FAKE), V(FAKE), 36960, V(FAKE), 36960, V(FAKE),
                                           V(FAKE), V(FAKE), 1 << 30, None) == 2
    # the merge: candidates per row within 8192 and at least k
    p = _params(h, T=0, B=2, n_cap=1000)
    assert lib.csa_topk_merge(ctypes.byref(p), V(FAKE), V(FAKE), 9000, V(FAKE), None) == 8
    assert lib.csa_topk_merge(ctypes.byref(p), V(FAKE), V(FAKE), 100, V(FAKE), None) == 8   # fewer than k = 512
    assert lib.hcsa_merge_partials(ctypes.byref(p), V(FAKE), 2, V(FAKE), 12345, None) == 2
    # low precision: bf16 only, and not for the HCA prefill attention
    p = _params(h, lowprec=1, dtype=0)
    assert lib.hcsa_quantize_rows(ctypes.byref(p), 0, V(FAKE), 10, V(FAKE), None) == 8
    p = _params(h, lowprec=2)
    assert lib.hcsa_quantize_rows(ctypes.byref(p), 0, V(FAKE), 10, V(FAKE), None) == 2
    p = _params(h, lowprec=1)
    assert h.hcsa_entry_bytes(p, 10) == 10 * (1024 + 32) and h.hcsa_key_bytes(p, 10) == 10 * (32 + 2)
