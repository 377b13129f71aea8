"""fp64 CPU oracle for CSA / HCA -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check and the benchmark's CPU-baseline leg may import
this package.  It shares no code with the CUDA library and never imports it.

The arithmetic lives in hcsa_oracle.c (plain loops in double precision, see
its header for the definitions and the passages they follow).  This module
converts storage-format arrays to float64 (exact), runs the projections as a
float64 library matmul, and assembles the per-query key lists:
  * prefill: entries visible to query t are j < t // m (entry j is visible
    iff m*j + m <= t); the raw window is tokens (t - window, t] inside [0, T);
  * decode at position P (the new token): the cache holds entries formed by
    tokens < P, the window ring holds token p in slot p % window and the gate /
    indexer-key staging rings hold token p in slot p % width; the new token is
    written into the rings first, an entry whose last token is P is formed,
    and the query then sees entries j < P // m and tokens (P - window, P].
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hcsa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

ST_F64, ST_F32, ST_BF16 = 0, 1, 2

_dp = ctypes.POINTER(ctypes.c_double)


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        V, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.orc_round.argtypes = [V, I64, I]
        lib.orc_compress.argtypes = [I64, I, I, I, V, I64, V, I64, V, V, I64, I, V, V, I]
        lib.orc_pool_rows.argtypes = [I, I, V, I64, V, I64, V, I64, V, I]
        lib.orc_index_scores.argtypes = [I, I, I, V, V, V, I64, V, V]
        lib.orc_topk.argtypes = [I, V, I64, V, I, V, V, V]
        lib.orc_attend.argtypes = [I, I, I, ctypes.c_double, V, I64, V, I, V, I, V, V, I64, V, I, V, I]
        lib.orc_round_e4m3.argtypes = [V, I64]
        lib.orc_round_e2m1.argtypes = [V, I64]
        lib.orc_store_fp8_rows.argtypes = [V, I64, I, I, V]
        lib.orc_store_fp4_rows.argtypes = [V, I64, I, I, V]
        lib.orc_num_threads.argtypes = []
        lib.orc_num_threads.restype = ctypes.c_int
        for f in ("orc_round", "orc_compress", "orc_pool_rows", "orc_index_scores", "orc_topk", "orc_attend",
                  "orc_round_e4m3", "orc_round_e2m1", "orc_store_fp8_rows", "orc_store_fp4_rows"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data


def storage_code(dtype: str) -> int:
    return {"f64": ST_F64, "f32": ST_F32, "bf16": ST_BF16}[dtype]


def to_f64(a: np.ndarray) -> np.ndarray:
    """Exact float64 value of a storage array (float32, float64 or bfloat16 bits as uint16)."""
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def round_to(a: np.ndarray, st: int) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float64).copy()
    _load().orc_round(a.ctypes.data, a.size, st)
    return a


def round_e4m3(a: np.ndarray) -> np.ndarray:
    """Nearest OCP E4M3 value of each element (ties to even), saturating at +-448."""
    a = np.ascontiguousarray(a, dtype=np.float64).copy()
    _load().orc_round_e4m3(a.ctypes.data, a.size)
    return a


def round_e2m1(a: np.ndarray) -> np.ndarray:
    """Nearest OCP E2M1 value of each element (ties to the even mantissa), saturating at +-6."""
    a = np.ascontiguousarray(a, dtype=np.float64).copy()
    _load().orc_round_e2m1(a.ctypes.data, a.size)
    return a


def store_fp8_rows(a: np.ndarray, block: int = 32):
    """FP8 (E4M3) storage of the rows of a 2-D array in blocks of `block` channels, one power-of-two
    scale 2^e per block (e smallest with amax / 2^e <= 448).  Returns (stored values, exponents)."""
    a = np.ascontiguousarray(a, dtype=np.float64).copy()
    rows, cols = a.shape
    exps = np.empty((rows, -(-cols // block)), np.int32)
    _load().orc_store_fp8_rows(a.ctypes.data, rows, cols, block, exps.ctypes.data)
    return a, exps


def store_fp4_rows(a: np.ndarray, block: int = 32):
    """FP4 (E2M1) storage of the rows of a 2-D array in blocks of `block` channels, one power-of-two
    scale 2^e per block (e smallest with amax / 2^e <= 6).  Returns (stored values, exponents)."""
    a = np.ascontiguousarray(a, dtype=np.float64).copy()
    rows, cols = a.shape
    exps = np.empty((rows, -(-cols // block)), np.int32)
    _load().orc_store_fp4_rows(a.ctypes.data, rows, cols, block, exps.ctypes.data)
    return a, exps


# ---------------------------------------------------------------- building blocks

def project(x64: np.ndarray, W64: np.ndarray, st: int) -> np.ndarray:
    """y = x W in float64 (library matmul), rounded to storage."""
    return round_to(x64 @ W64, st)


def compress(T, C, m, width, kv, ld_kv, g, ld_g, bias, ki, ld_ki, di, st, kv_base=None):
    """Prefill pool over a sequence; kv/g/ki are float64 arrays (views via base + offsets)."""
    N = -(-T // m)
    entries = np.empty((N, C), np.float64)
    idx = np.empty((N, di), np.float64) if ki is not None else None
    _load().orc_compress(T, C, m, width, kv, ld_kv, g, ld_g, _p(bias), ki, ld_ki, di,
                         _p(entries), _p(idx), st)
    return entries, idx


def pool_rows(kv_tok, g_tok, b_tok, nch, st):
    n = kv_tok.shape[0]
    out = np.empty(nch, np.float64)
    kv_tok, g_tok, b_tok = (np.ascontiguousarray(a, np.float64) for a in (kv_tok, g_tok, b_tok))
    _load().orc_pool_rows(n, nch, _p(kv_tok), kv_tok.shape[1], _p(g_tok), g_tok.shape[1], _p(b_tok),
                          b_tok.shape[1], _p(out), st)
    return out


def index_scores(qi, w, keys, n_vis, Hi, di):
    qi = np.ascontiguousarray(qi, np.float64)
    w = np.ascontiguousarray(w, np.float64)
    keys = np.ascontiguousarray(keys, np.float64)
    n_vis = np.ascontiguousarray(n_vis, np.int64)
    nq, N = qi.shape[0], keys.shape[0]
    s = np.empty((nq, N), np.float64)
    _load().orc_index_scores(nq, Hi, di, _p(qi), _p(w), _p(keys), N, _p(n_vis), _p(s))
    return s


def topk(scores, n_vis, k):
    scores = np.ascontiguousarray(scores, np.float64)
    n_vis = np.ascontiguousarray(n_vis, np.int64)
    nq, N = scores.shape
    sel = np.empty((nq, k), np.int32)
    gap = np.empty(nq, np.float64)
    kth = np.empty(nq, np.float64)
    _load().orc_topk(nq, _p(scores), N, _p(n_vis), k, _p(sel), _p(gap), _p(kth))
    return sel, gap, kth


def attend(q, H, dh, scale, entries, sel, n_vis, raw, win_rows, st):
    """q[nq, H*dh]; entries[N, C]; sel[nq, k] (or None => all j < n_vis); raw[R, >=C]; win_rows[nq, w]."""
    q = np.ascontiguousarray(q, np.float64)
    entries = np.ascontiguousarray(entries, np.float64)
    raw = np.ascontiguousarray(raw, np.float64)
    win_rows = np.ascontiguousarray(win_rows, np.int64)
    nq = q.shape[0]
    C = entries.shape[1] if entries.ndim == 2 and entries.shape[0] else 2 * dh
    if entries.size == 0:
        entries = np.zeros((1, C), np.float64)
    out = np.empty((nq, H * dh), np.float64)
    if sel is not None:
        sel = np.ascontiguousarray(sel, np.int32)
        nsel = sel.shape[1]
        nv = None
    else:
        nsel = 0
        nv = np.ascontiguousarray(n_vis, np.int64)
    _load().orc_attend(nq, H, dh, float(scale), _p(q), q.shape[1], _p(entries), C, _p(sel), nsel, _p(nv),
                       _p(raw), raw.shape[1], _p(win_rows), win_rows.shape[1], _p(out), st)
    return out


def prefill_window_rows(tpos, window):
    tpos = np.asarray(tpos, np.int64)
    r = tpos[:, None] - window + 1 + np.arange(window, dtype=np.int64)[None, :]
    return np.where(r >= 0, r, -1)


def prefill_n_vis(tpos, m, N):
    return np.minimum(np.asarray(tpos, np.int64) // m, N)


# ---------------------------------------------------------------- whole layer

def _col_slices(spec):
    cols, off = {}, 0
    names = [("kv", spec.C), ("g", spec.C)]
    if spec.kind == "csa":
        names += [("ki", spec.di), ("qi", spec.Hi * spec.di), ("w", spec.Hi)]
    names += [("q", spec.H * spec.dh)]
    for n, w in names:
        cols[n] = slice(off, off + w)
        off += w
    return cols


def prefill(spec, inp, rows=None, chunk=8192, lowprec=False):
    """Run the whole layer on the oracle.

    inp: storage arrays x[T,D], W_cat[D,ncat], B[width,C] (as produced by synth).
    rows: query positions to evaluate (default: all).  Entries are always built
    for the whole sequence.  lowprec: store the compressed entries as FP8 (blocks of
    32 channels) and the indexer keys as FP4 (blocks of 32), see store_fp8_rows /
    store_fp4_rows; everything downstream reads the stored values.  Returns a dict of
    float64 arrays."""
    res = prefill_entries(spec, inp, chunk=chunk, lowprec=lowprec)
    return prefill_queries(spec, inp, res, rows)


def prefill_entries(spec, inp, chunk=8192, lowprec=False):
    """The sequence-wide half of prefill(): projections of the pooled columns (kv, g, ki) of every
    token, then the compressor (entries and indexer keys of the whole sequence)."""
    st = storage_code(spec.dtype)
    T, C, m = spec.T, spec.C, spec.m
    cols = _col_slices(spec)
    W = to_f64(inp["W_cat"])
    B = to_f64(inp["B"])
    csa = spec.kind == "csa"
    pool_end = cols["ki"].stop if csa else cols["g"].stop
    W_pool = np.ascontiguousarray(W[:, :pool_end])
    ypool = np.empty((T, pool_end), np.float64)
    for a in range(0, T, chunk):
        ypool[a:a + chunk] = project(to_f64(inp["x"][a:a + chunk]), W_pool, st)
    ld = pool_end
    base = ypool.ctypes.data
    ki_ptr = base + 8 * cols["ki"].start if csa else None
    entries, idx = compress(T, C, m, spec.width, base, ld, base + 8 * C, ld, B, ki_ptr, ld,
                            spec.di if csa else 0, st)
    if lowprec:
        entries = store_fp8_rows(entries, 32)[0]
        if csa:
            idx = store_fp4_rows(idx, 32)[0]
    return {"y_pool": ypool, "entries": entries, "idx_keys": idx, "W_q": np.ascontiguousarray(W[:, pool_end:]),
            "pool_end": pool_end}


def prefill_queries(spec, inp, ent, rows=None):
    """The per-query half of prefill() for the positions `rows` (default all), over the sequence-wide
    results `ent` of prefill_entries(): query projections (qi, w, q), indexer scores, top-k and
    attention.  Returns the dict prefill() documents."""
    st = storage_code(spec.dtype)
    m = spec.m
    cols = _col_slices(spec)
    csa = spec.kind == "csa"
    rows = np.arange(spec.T, dtype=np.int64) if rows is None else np.asarray(rows, np.int64)
    yq = project(to_f64(inp["x"][rows]), ent["W_q"], st)
    off = ent["pool_end"]
    qcols = {n: slice(s.start - off, s.stop - off) for n, s in cols.items() if s.start >= off}
    res = {"y_pool": ent["y_pool"], "entries": ent["entries"], "idx_keys": ent["idx_keys"], "rows": rows,
           "y_q": yq}
    N = ent["entries"].shape[0]
    n_vis = prefill_n_vis(rows, m, N)
    res["n_vis"] = n_vis
    if csa:
        scores = index_scores(yq[:, qcols["qi"]], yq[:, qcols["w"]], ent["idx_keys"], n_vis, spec.Hi, spec.di)
        sel, gap, kth = topk(scores, n_vis, spec.topk)
        res.update(scores=scores, sel=sel, gap=gap, kth=kth)
    else:
        sel = None
    res["out"] = attend_rows(spec, res, yq[:, qcols["q"]], sel)
    res["q"] = yq[:, qcols["q"]]
    return res


def num_threads() -> int:
    """OpenMP threads the oracle's loops use."""
    return int(_load().orc_num_threads())


def attend_rows(spec, res, q, sel):
    """Attention for res['rows'] given a selection (None = HCA dense); raw window = projected kv."""
    st = storage_code(spec.dtype)
    rows = res["rows"]
    ypool = res["y_pool"]
    win = prefill_window_rows(rows, spec.window)
    return attend(q, spec.H, spec.dh, spec.scale, res["entries"], sel, res["n_vis"], ypool, win, st)


def decode_step(spec, inp, P, seqs=None, lowprec=False):
    """One decode step of one layer.

    inp: storage arrays as produced by synth.decode_inputs: W_cat, B, x[Ball, D] and the cache
    entries[Ball,N,C], idx_keys[Ball,N,di], win_kv[Ball,win,C], ring_g[Ball,width,C], ring_ki[Ball,width,di].
    P: position of the new token, one int or one per batch row.  seqs: the batch rows to evaluate
    (default all).  lowprec: the cache holds its entries in FP8 and its indexer keys in FP4 (the
    given values are stored in those formats first, and an entry formed by this step is stored so too);
    the window ring stays in the layer's storage format.  Returns per-evaluated-row results (float64),
    in the order of seqs."""
    st = storage_code(spec.dtype)
    csa = spec.kind == "csa"
    m, Wd, win, C = spec.m, spec.width, spec.window, spec.C
    if win < Wd:
        raise ValueError("the window ring also stages the kv rows of the open pool: window >= width")
    cols = _col_slices(spec)
    nb_all = inp["x"].shape[0]
    seqs = list(range(nb_all)) if seqs is None else list(seqs)
    Pv = np.broadcast_to(np.asarray(P, np.int64), (nb_all,))
    Bm = to_f64(inp["B"])
    W = to_f64(inp["W_cat"])
    res = {"seqs": seqs, "y": [], "out": [], "win_kv": [], "ring_g": [], "ring_ki": [], "entries": [],
           "new_entry": [], "sel": [], "gap": [], "scores": []}
    for b in seqs:
        Pb = int(Pv[b])
        yb = project(to_f64(inp["x"][b:b + 1]), W, st)[0]
        win_kv = to_f64(inp["win_kv"][b]).copy()
        ring_g = to_f64(inp["ring_g"][b]).copy()
        ent_b = to_f64(inp["entries"][b])
        idx_b = to_f64(inp["idx_keys"][b]) if csa else None
        if lowprec:
            ent_b = store_fp8_rows(ent_b, 32)[0]
            if csa:
                idx_b = store_fp4_rows(idx_b, 32)[0]
        ring_ki = to_f64(inp["ring_ki"][b]).copy() if csa else None
        Ncap = ent_b.shape[0]
        # append: the new token enters the rings
        win_kv[Pb % win] = yb[cols["kv"]]
        ring_g[Pb % Wd] = yb[cols["g"]]
        if csa:
            ring_ki[Pb % Wd] = yb[cols["ki"]]
        new = None
        if (Pb + 1) % m == 0:       # the token closes entry j: pool tokens [m j - (width - m), m j + m)
            j = (Pb + 1) // m - 1
            lo = m * j - (Wd - m)
            toks = [i for i in range(lo, m * j + m) if i >= 0]
            kv_t = np.stack([win_kv[i % win] for i in toks])
            g_t = np.stack([ring_g[i % Wd] for i in toks])
            b_t = np.stack([Bm[i - lo] for i in toks])
            new = {"j": j, "entry": pool_rows(kv_t, g_t, b_t, C, st)}
            if lowprec:
                new["entry"] = store_fp8_rows(new["entry"][None], 32)[0][0]
            if csa:
                ki_t = np.stack([ring_ki[i % Wd] for i in toks])
                new["idx_key"] = pool_rows(ki_t, g_t, b_t, spec.di, st)
                if lowprec:
                    new["idx_key"] = store_fp4_rows(new["idx_key"][None], 32)[0][0]
            if j < Ncap:
                ent_b = ent_b.copy()
                ent_b[j] = new["entry"]
                if csa:
                    idx_b = idx_b.copy()
                    idx_b[j] = new["idx_key"]
        n_vis = np.array([min(Pb // m, Ncap)], np.int64)
        if csa:
            sc = index_scores(yb[cols["qi"]][None], yb[cols["w"]][None], idx_b, n_vis, spec.Hi, spec.di)
            sel, gap, _ = topk(sc, n_vis, spec.topk)
            res["sel"].append(sel[0])
            res["gap"].append(gap[0])
            res["scores"].append(sc[0])
        else:
            sel = None
        pos = Pb - win + 1 + np.arange(win)
        wrows = np.where(pos >= 0, pos % win, -1)[None, :]
        res["out"].append(attend(yb[cols["q"]][None], spec.H, spec.dh, spec.scale, ent_b, sel, n_vis,
                                 win_kv, wrows, st)[0])
        res["y"].append(yb)
        res["win_kv"].append(win_kv)
        res["ring_g"].append(ring_g)
        res["ring_ki"].append(ring_ki)
        res["entries"].append(ent_b)
        res["new_entry"].append(new)
        res["P"] = Pv
    res["out"] = np.stack(res["out"])
    if csa:
        res["sel"] = np.stack(res["sel"])
        res["gap"] = np.array(res["gap"])
    return res


def decode_stack(specs, layer_inputs, P, residual=True, lowprec=False):
    """Decode steps of a stack of layers for one batch.

    Layer l reads the hidden state x_l (x_0 = layer_inputs[0]["x"]).  With residual, the layers chain
    through the residual stream: x_{l+1} = x_l + out_l W_o,l, rounded once to the storage format (the
    pages define neither an output projection nor a normalisation; this is the reading taken for the
    V4-style schedule).  Without residual every layer reads x_0.  layer_inputs[l]: as for decode_step,
    plus W_o [H*dh, D] when residual.  Returns (the hidden state after the last layer, per-layer
    results of decode_step)."""
    x0 = to_f64(layer_inputs[0]["x"])
    x = x0
    results = []
    for spec, inp in zip(specs, layer_inputs):
        li = dict(inp)
        li["x"] = x
        r = decode_step(spec, li, P, lowprec=lowprec)
        results.append(r)
        if residual:
            x = round_to(x + r["out"] @ to_f64(inp["W_o"]), storage_code(spec.dtype))
    return x, results


def decode_attend_with_sel(spec, res, i, sel_row):
    """Recompute the i-th evaluated row of a decode_step result on a given selection (e.g. the GPU's)."""
    st = storage_code(spec.dtype)
    win = spec.window
    cols = _col_slices(spec)
    b = res["seqs"][i]
    Pb = int(res["P"][b])
    pos = Pb - win + 1 + np.arange(win)
    wrows = np.where(pos >= 0, pos % win, -1)[None, :]
    return attend(res["y"][i][cols["q"]][None], spec.H, spec.dh, spec.scale, res["entries"][i],
                  np.asarray(sel_row, np.int32)[None], None, res["win_kv"][i], wrows, st)[0]
