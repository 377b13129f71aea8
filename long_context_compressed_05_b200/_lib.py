"""ctypes binding of libhcsa.so: same names as the C ABI (include/hca_csa.h).

Argument marshalling only: tensors become (pointer, leading dimension) pairs and
the current torch CUDA stream is passed along.  Every step runs in the CUDA
library; if it is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhcsa.so")

HCSA_F32, HCSA_BF16 = 0, 1
KIND_CSA, KIND_HCA = 0, 1
OP_PROJECT, OP_CSA_INDEX_TOPK, OP_CSA_ATTEND, OP_HCA_ATTEND = 0, 1, 2, 3
OP_CSA_DECODE_INDEX_TOPK, OP_CSA_DECODE_ATTEND, OP_HCA_DECODE_ATTEND = 4, 5, 6
OP_CSA_DECODE_INDEX_TOPK_SHARD, OP_CSA_DECODE_ATTEND_SHARD, OP_HCA_DECODE_ATTEND_SHARD = 7, 8, 9

STATUS = {0: "HCSA_OK", 1: "HCSA_ERR_NULL", 2: "HCSA_ERR_SHAPE", 3: "HCSA_ERR_DTYPE", 4: "HCSA_ERR_ALIGN",
          5: "HCSA_ERR_WORKSPACE", 6: "HCSA_ERR_CUDA", 7: "HCSA_ERR_TIMEOUT", 8: "HCSA_ERR_UNSUPPORTED",
          9: "HCSA_ERR_DEVICE"}

# every entry point the header declares (checked by the CPU export test)
EXPORTS = ["hcsa_version", "hcsa_status_string", "hcsa_workspace_bytes", "hcsa_proj_cols", "hcsa_project",
           "hcsa_out_project",
           "csa_compress", "hca_compress", "csa_index_topk", "csa_attend", "hca_attend", "hcsa_cache_append",
           "csa_decode_index_topk", "csa_decode_attend", "hca_decode_attend", "csa_decode_index_topk_noalloc",
           "hcsa_get_device_status", "hcsa_selftest_wait_timeout",
           "hcsa_launch_count", "hcsa_entry_bytes", "hcsa_key_bytes", "hcsa_quantize_rows",
           "csa_decode_index_topk_shard", "csa_topk_merge", "csa_decode_attend_shard", "hca_decode_attend_shard",
           "hcsa_merge_partials", "hcsa_project_append", "hcsa_project_compress"]
STORE_ENTRIES, STORE_KEYS = 0, 1


class HcsaError(RuntimeError):
    def __init__(self, fn, code):
        self.code = code
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")


class Params(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "T", "D", "m", "width", "C", "di", "Hi", "topk", "window",
                                              "H", "dh")] + [("scale", ctypes.c_float), ("dtype", ctypes.c_int32),
                                                             ("n_cap", ctypes.c_int32), ("row0", ctypes.c_int32),
                                                             ("row1", ctypes.c_int32), ("lowprec", ctypes.c_int32),
                                                             ("ent0", ctypes.c_int32), ("ent_shard", ctypes.c_int32)]


class Cache(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("entries", "idx_keys", "win_kv", "ring_g", "ring_ki")]


_lib = None


def load():
    """Load libhcsa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"CUDA library {LIB_PATH} is missing: build it with __graft_entry__.build()")
    lib = ctypes.CDLL(LIB_PATH)
    V, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    P = ctypes.POINTER(Params)
    CP = ctypes.POINTER(Cache)
    sig = {
        "hcsa_version": (I32, []),
        "hcsa_status_string": (ctypes.c_char_p, [I32]),
        "hcsa_workspace_bytes": (SZ, [P, I32]),
        "hcsa_proj_cols": (I64, [P, I32]),
        "hcsa_project": (I32, [P, I32, I64, V, V, V, V, SZ, V]),
        "hcsa_out_project": (I32, [P, I64, V, I64, V, V, I64, V, SZ, V]),
        "csa_compress": (I32, [P, V, I64, V, I64, V, I64, V, V, V, V]),
        "hca_compress": (I32, [P, V, I64, V, I64, V, V, V]),
        "csa_index_topk": (I32, [P, V, I64, V, I64, V, V, V, SZ, V]),
        "csa_attend": (I32, [P, V, I64, V, I64, V, V, V, V, SZ, V]),
        "hca_attend": (I32, [P, V, I64, V, I64, V, V, V, SZ, V]),
        "hcsa_cache_append": (I32, [P, CP, V, V, I64, V, I64, V, I64, V, V]),
        "csa_decode_index_topk": (I32, [P, CP, V, V, I64, V, I64, V, V, SZ, V]),
        "csa_decode_attend": (I32, [P, CP, V, V, I64, V, V, V, SZ, V]),
        "hca_decode_attend": (I32, [P, CP, V, V, I64, V, V, SZ, V]),
        "csa_decode_index_topk_noalloc": (I32, [P, CP, V, V, I64, V, I64, V, V]),
        "hcsa_get_device_status": (I32, [V]),
        "hcsa_selftest_wait_timeout": (I32, [V]),
        "hcsa_launch_count": (I64, [I32]),
        "hcsa_entry_bytes": (SZ, [P, I64]),
        "hcsa_key_bytes": (SZ, [P, I64]),
        "hcsa_quantize_rows": (I32, [P, I32, V, I64, V, V]),
        "csa_decode_index_topk_shard": (I32, [P, CP, V, V, I64, V, I64, V, V, V, SZ, V]),
        "csa_topk_merge": (I32, [P, V, V, I32, V, V]),
        "csa_decode_attend_shard": (I32, [P, CP, V, V, I64, V, I32, V, V, SZ, V]),
        "hca_decode_attend_shard": (I32, [P, CP, V, V, I64, I32, V, V, SZ, V]),
        "hcsa_merge_partials": (I32, [P, V, I32, V, I64, V]),
        "hcsa_project_append": (I32, [P, I32, CP, V, V, V, V, V, V, SZ, V]),
        "hcsa_project_compress": (I32, [P, I32, V, V, V, V, V, V, V, SZ, V]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _check(fn, code):
    if code != 0:
        raise HcsaError(fn, code)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _ld(t):
    return 0 if t is None else (t.stride(0) if t.dim() >= 2 else t.shape[-1])


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def make_params(*, T=0, D=0, m=4, width=8, C=0, di=0, Hi=0, topk=0, window=128, H=1, dh=0, scale=1.0,
                dtype="bf16", B=1, n_cap=0, row0=0, row1=0, lowprec=0, ent0=0, ent_shard=0) -> Params:
    return Params(B=B, T=T, D=D, m=m, width=width, C=C, di=di, Hi=Hi, topk=topk, window=window, H=H, dh=dh,
                  scale=scale, dtype=HCSA_BF16 if dtype == "bf16" else HCSA_F32, n_cap=n_cap, row0=row0,
                  row1=row1, lowprec=int(lowprec), ent0=ent0, ent_shard=int(ent_shard))


def make_cache(entries, win_kv, ring_g, idx_keys=None, ring_ki=None) -> Cache:
    return Cache(entries=_ptr(entries), idx_keys=_ptr(idx_keys), win_kv=_ptr(win_kv), ring_g=_ptr(ring_g),
                 ring_ki=_ptr(ring_ki))


# ---------------------------------------------------------------- entry points (same names as the C ABI)

def hcsa_version():
    return load().hcsa_version()


def hcsa_status_string(code):
    return load().hcsa_status_string(code).decode()


def hcsa_workspace_bytes(p: Params, op: int) -> int:
    return int(load().hcsa_workspace_bytes(ctypes.byref(p), op))


def hcsa_proj_cols(p: Params, kind: int) -> int:
    return int(load().hcsa_proj_cols(ctypes.byref(p), kind))


def hcsa_project(p, kind, x, W_cat, y, ws=None, stream=None):
    _check("hcsa_project", load().hcsa_project(ctypes.byref(p), kind, x.shape[0], _ptr(x), _ptr(W_cat), _ptr(y),
                                               _ptr(ws), 0 if ws is None else ws.numel() * ws.element_size(),
                                               _stream(stream)))


def hcsa_out_project(p, out, W_o, x, ws=None, stream=None):
    """x += out W_o in place (the residual update of a chained stack; bf16)."""
    _check("hcsa_out_project", load().hcsa_out_project(ctypes.byref(p), x.shape[0], _ptr(out), _ld(out), _ptr(W_o),
                                                       _ptr(x), _ld(x), _ptr(ws), _wsz(ws), _stream(stream)))


def csa_compress(p, kv, g, ki, bias, entries, idx_keys, stream=None):
    _check("csa_compress", load().csa_compress(ctypes.byref(p), _ptr(kv), _ld(kv), _ptr(g), _ld(g), _ptr(ki),
                                               _ld(ki), _ptr(bias), _ptr(entries), _ptr(idx_keys),
                                               _stream(stream)))


def hca_compress(p, kv, g, bias, entries, stream=None):
    _check("hca_compress", load().hca_compress(ctypes.byref(p), _ptr(kv), _ld(kv), _ptr(g), _ld(g), _ptr(bias),
                                               _ptr(entries), _stream(stream)))


def _wsz(ws):
    return 0 if ws is None else ws.numel() * ws.element_size()


def csa_index_topk(p, qi, w, idx_keys, sel, ws, stream=None):
    _check("csa_index_topk", load().csa_index_topk(ctypes.byref(p), _ptr(qi), _ld(qi), _ptr(w), _ld(w),
                                                   _ptr(idx_keys), _ptr(sel), _ptr(ws), _wsz(ws),
                                                   _stream(stream)))


def csa_attend(p, q, kv, entries, sel, out, ws=None, stream=None):
    _check("csa_attend", load().csa_attend(ctypes.byref(p), _ptr(q), _ld(q), _ptr(kv), _ld(kv), _ptr(entries),
                                           _ptr(sel), _ptr(out), _ptr(ws), _wsz(ws), _stream(stream)))


def hca_attend(p, q, kv, entries, out, ws=None, stream=None):
    _check("hca_attend", load().hca_attend(ctypes.byref(p), _ptr(q), _ld(q), _ptr(kv), _ld(kv), _ptr(entries),
                                           _ptr(out), _ptr(ws), _wsz(ws), _stream(stream)))


def hcsa_cache_append(p, cache: Cache, pos, kv, g, ki, bias, stream=None):
    _check("hcsa_cache_append", load().hcsa_cache_append(ctypes.byref(p), ctypes.byref(cache), _ptr(pos),
                                                         _ptr(kv), _ld(kv), _ptr(g), _ld(g), _ptr(ki), _ld(ki),
                                                         _ptr(bias), _stream(stream)))


def csa_decode_index_topk(p, cache: Cache, pos, qi, w, sel, ws, stream=None):
    _check("csa_decode_index_topk", load().csa_decode_index_topk(
        ctypes.byref(p), ctypes.byref(cache), _ptr(pos), _ptr(qi), _ld(qi), _ptr(w), _ld(w), _ptr(sel), _ptr(ws),
        _wsz(ws), _stream(stream)))


def csa_decode_attend(p, cache: Cache, pos, q, sel, out, ws=None, stream=None):
    _check("csa_decode_attend", load().csa_decode_attend(ctypes.byref(p), ctypes.byref(cache), _ptr(pos), _ptr(q),
                                                         _ld(q), _ptr(sel), _ptr(out), _ptr(ws), _wsz(ws),
                                                         _stream(stream)))


def hca_decode_attend(p, cache: Cache, pos, q, out, ws=None, stream=None):
    _check("hca_decode_attend", load().hca_decode_attend(ctypes.byref(p), ctypes.byref(cache), _ptr(pos), _ptr(q),
                                                         _ld(q), _ptr(out), _ptr(ws), _wsz(ws), _stream(stream)))


def csa_decode_index_topk_noalloc(p, cache: Cache, pos, qi, w, sel, stream=None):
    """csa_decode_index_topk with the scores in the library's fixed scratch array (no workspace)."""
    _check("csa_decode_index_topk_noalloc", load().csa_decode_index_topk_noalloc(
        ctypes.byref(p), ctypes.byref(cache), _ptr(pos), _ptr(qi), _ld(qi), _ptr(w), _ld(w), _ptr(sel),
        _stream(stream)))


def hcsa_get_device_status(stream=None) -> int:
    return int(load().hcsa_get_device_status(_stream(stream)))


def hcsa_selftest_wait_timeout(stream=None) -> None:
    """Enqueue the bounded-wait self-test kernel (see include/hca_csa.h)."""
    _check("hcsa_selftest_wait_timeout", load().hcsa_selftest_wait_timeout(_stream(stream)))


def hcsa_entry_bytes(p: Params, rows: int) -> int:
    return int(load().hcsa_entry_bytes(ctypes.byref(p), rows))


def hcsa_key_bytes(p: Params, rows: int) -> int:
    return int(load().hcsa_key_bytes(ctypes.byref(p), rows))


def hcsa_quantize_rows(p, what, src, dst, stream=None):
    """src: [rows, C] (entries) or [rows, di] (keys) bf16; dst: a byte buffer of the matching size."""
    _check("hcsa_quantize_rows", load().hcsa_quantize_rows(ctypes.byref(p), what, _ptr(src), src.shape[0],
                                                           _ptr(dst), _stream(stream)))


def hcsa_project_compress(p, kind, x, W_cat, bias, y, entries, idx_keys, ws=None, stream=None):
    _check("hcsa_project_compress", load().hcsa_project_compress(
        ctypes.byref(p), kind, _ptr(x), _ptr(W_cat), _ptr(bias), _ptr(y), _ptr(entries), _ptr(idx_keys), _ptr(ws),
        _wsz(ws), _stream(stream)))


def hcsa_project_append(p, kind, cache: Cache, pos, x, W_cat, bias, y, ws=None, stream=None):
    _check("hcsa_project_append", load().hcsa_project_append(
        ctypes.byref(p), kind, ctypes.byref(cache), _ptr(pos), _ptr(x), _ptr(W_cat), _ptr(bias), _ptr(y), _ptr(ws),
        _wsz(ws), _stream(stream)))


def csa_decode_index_topk_shard(p, cache: Cache, pos, qi, w, sel, sel_scores, ws, stream=None):
    _check("csa_decode_index_topk_shard", load().csa_decode_index_topk_shard(
        ctypes.byref(p), ctypes.byref(cache), _ptr(pos), _ptr(qi), _ld(qi), _ptr(w), _ld(w), _ptr(sel),
        _ptr(sel_scores), _ptr(ws), _wsz(ws), _stream(stream)))


def csa_topk_merge(p, cand_sel, cand_scores, sel, stream=None):
    """cand_sel / cand_scores: [B, n_cand] (one row per sequence); sel: [B, topk]."""
    _check("csa_topk_merge", load().csa_topk_merge(ctypes.byref(p), _ptr(cand_sel), _ptr(cand_scores),
                                                   cand_sel.shape[1], _ptr(sel), _stream(stream)))


def csa_decode_attend_shard(p, cache: Cache, pos, q, sel, with_window, part, ws=None, stream=None):
    _check("csa_decode_attend_shard", load().csa_decode_attend_shard(
        ctypes.byref(p), ctypes.byref(cache), _ptr(pos), _ptr(q), _ld(q), _ptr(sel), int(with_window), _ptr(part),
        _ptr(ws), _wsz(ws), _stream(stream)))


def hca_decode_attend_shard(p, cache: Cache, pos, q, with_window, part, ws=None, stream=None):
    _check("hca_decode_attend_shard", load().hca_decode_attend_shard(
        ctypes.byref(p), ctypes.byref(cache), _ptr(pos), _ptr(q), _ld(q), int(with_window), _ptr(part), _ptr(ws),
        _wsz(ws), _stream(stream)))


def hcsa_merge_partials(p, parts, n_parts, out, stream=None):
    """parts: n_parts consecutive partial blocks of B * H * (dh + 2) floats; out: [B, H * dh]."""
    _check("hcsa_merge_partials", load().hcsa_merge_partials(ctypes.byref(p), _ptr(parts), n_parts, _ptr(out),
                                                             _ld(out), _stream(stream)))


def hcsa_launch_count(reset: bool = False) -> int:
    return int(load().hcsa_launch_count(1 if reset else 0))
