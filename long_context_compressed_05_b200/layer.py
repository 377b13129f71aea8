"""Layer-level helpers over the C ABI: allocate device buffers with torch and
issue the calls of one CSA / HCA layer (prefill) or one decode step, in order.

Nothing here computes: every step is a call into libhcsa.so.
"""
from __future__ import annotations

import torch

from . import _lib as L

__all__ = ["params_for", "torch_dtype", "row_ranges", "PrefillLayer", "DecodeLayer"]


def torch_dtype(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def params_for(spec, *, T=None, B=1, n_cap=0, row0=0, row1=0, lowprec=False, ent0=0, ent_shard=False) -> L.Params:
    """Params from any object with the layer fields (kind, D, m, width, C, di, Hi, topk, window, H, dh, scale, dtype).
    row0 / row1: the prefill row range (both 0: the whole sequence).  lowprec: FP8 entries, FP4 indexer keys."""
    return L.make_params(T=spec.T if T is None else T, D=spec.D, m=spec.m, width=spec.width, C=spec.C,
                         di=getattr(spec, "di", 0), Hi=getattr(spec, "Hi", 0), topk=getattr(spec, "topk", 0),
                         window=spec.window, H=spec.H, dh=spec.dh, scale=spec.scale, dtype=spec.dtype, B=B,
                         n_cap=n_cap, row0=row0, row1=row1, lowprec=lowprec, ent0=ent0, ent_shard=ent_shard)


def row_ranges(T, chunks):
    """At most `chunks` contiguous row ranges covering [0, T), each starting on a 128-row boundary (the
    prefill calls' row-range rule)."""
    step = -(-max(1, -(-T // max(1, chunks))) // 128) * 128
    return [(a, min(T, a + step)) for a in range(0, T, step)]


def _col_offsets(spec):
    names = [("kv", spec.C), ("g", spec.C)]
    if spec.kind == "csa":
        names += [("ki", spec.di), ("qi", spec.Hi * spec.di), ("w", spec.Hi)]
    names += [("q", spec.H * spec.dh)]
    off, out = 0, {}
    for n, w in names:
        out[n] = (off, off + w)
        off += w
    return out, off


class PrefillLayer:
    """One CSA or HCA layer over a sequence of T tokens, buffers allocated once."""

    def __init__(self, spec, device="cuda", lowprec=False):
        self.spec = spec
        self.csa = spec.kind == "csa"
        self.kind = L.KIND_CSA if self.csa else L.KIND_HCA
        self.lowprec = lowprec
        self.p = params_for(spec, lowprec=lowprec)
        dt = torch_dtype(spec.dtype)
        T, N = spec.T, -(-spec.T // spec.m)
        self.cols, ncols = _col_offsets(spec)
        assert ncols == L.hcsa_proj_cols(self.p, self.kind)
        self.y = torch.empty((T, ncols), dtype=dt, device=device)
        # FP8 / FP4 storage: byte arrays of codes followed by the block exponents
        self.entries = (torch.empty(L.hcsa_entry_bytes(self.p, N), dtype=torch.uint8, device=device) if lowprec
                        else torch.empty((N, spec.C), dtype=dt, device=device))
        self.out = torch.empty((T, spec.H * spec.dh), dtype=dt, device=device)
        self.ws_proj = self._ws(L.OP_PROJECT, device)
        if self.csa:
            self.idx_keys = (torch.empty(L.hcsa_key_bytes(self.p, N), dtype=torch.uint8, device=device) if lowprec
                             else torch.empty((N, spec.di), dtype=dt, device=device))
            self.sel = torch.empty((T, spec.topk), dtype=torch.int32, device=device)
            self.ws_index = self._ws(L.OP_CSA_INDEX_TOPK, device)
            self.ws_attend = self._ws(L.OP_CSA_ATTEND, device)
        else:
            self.ws_attend = self._ws(L.OP_HCA_ATTEND, device)

    def _ws(self, op, device):
        n = L.hcsa_workspace_bytes(self.p, op)
        return torch.empty(max(n, 16), dtype=torch.uint8, device=device) if n else None

    def view(self, name):
        a, b = self.cols[name]
        return self.y[:, a:b]

    def project(self, x, W_cat):
        L.hcsa_project(self.p, self.kind, x, W_cat, self.y, self.ws_proj)

    def compress(self, bias):
        if self.csa:
            L.csa_compress(self.p, self.view("kv"), self.view("g"), self.view("ki"), bias, self.entries,
                           self.idx_keys)
        else:
            L.hca_compress(self.p, self.view("kv"), self.view("g"), bias, self.entries)

    def index_topk(self):
        L.csa_index_topk(self.p, self.view("qi"), self.view("w"), self.idx_keys, self.sel, self.ws_index)

    def attend(self, sel=None, p=None):
        """Attention for all rows, or for the row range of `p` (params with row0 / row1 set)."""
        p = self.p if p is None else p
        if self.csa:
            L.csa_attend(p, self.view("q"), self.view("kv"), self.entries, self.sel if sel is None else sel,
                         self.out, self.ws_attend)
        else:
            L.hca_attend(p, self.view("q"), self.view("kv"), self.entries, self.out, self.ws_attend)

    def project_compress(self, x, W_cat, bias):
        """The projection with the compressor in its epilogue (one GEMM + a seam pass for CSA layers).  Same
        results as project + compress; at T = 131072 about 0.6 ms slower, so forward() keeps the two calls."""
        L.hcsa_project_compress(self.p, self.kind, x, W_cat, bias, self.y, self.entries,
                                self.idx_keys if self.csa else None, self.ws_proj)

    def forward(self, x, W_cat, bias):
        self.project(x, W_cat)
        self.compress(bias)
        if self.csa:
            self.index_topk()
        self.attend()
        return self.out

    def forward_host(self, x_host, W_cat, bias, out_host, chunks=8):
        """forward() with the input x and the output in (pinned) host memory.

        The attention runs in at most `chunks` row ranges (multiples of 128 rows), and each range's output
        rows go back on a copy stream as soon as they are written, so the device-to-host copy overlaps the
        rest of the attention.  The copies of one call also overlap the next call's input copy, projection,
        compressor and indexer; only its attention, which rewrites `out`, waits for them.  Call wait_host()
        before reading out_host."""
        T = self.spec.T
        if getattr(self, "_copy_stream", None) is None:
            self._copy_stream = torch.cuda.Stream(device=self.y.device)
            self._x = torch.empty(x_host.shape, dtype=x_host.dtype, device=self.y.device)
            self._copied = None
        cur = torch.cuda.current_stream(self.y.device)
        self._x.copy_(x_host, non_blocking=True)
        self.project(self._x, W_cat)
        self.compress(bias)
        if self.csa:
            self.index_topk()
        if self._copied is not None:
            cur.wait_event(self._copied)   # the previous call's copies have read `out`
        for a, b in row_ranges(T, chunks):
            self.attend(p=params_for(self.spec, row0=a, row1=b, lowprec=self.lowprec))
            done = torch.cuda.Event()
            done.record(cur)
            self._copy_stream.wait_event(done)
            with torch.cuda.stream(self._copy_stream):
                out_host[a:b].copy_(self.out[a:b], non_blocking=True)
        self._copied = torch.cuda.Event()
        self._copied.record(self._copy_stream)
        return out_host

    def wait_host(self):
        """Make the current stream wait for the output copies of the last forward_host() call."""
        if getattr(self, "_copied", None) is not None:
            torch.cuda.current_stream(self.y.device).wait_event(self._copied)


class DecodeLayer:
    """One layer's decode step for B sequences over a caller-provided cache."""

    def __init__(self, spec, B, n_cap, cache: dict, device="cuda", lowprec=False, fused_append=True):
        """cache: device tensors entries, win_kv, ring_g (+ idx_keys, ring_ki for CSA); with lowprec the
        entries and idx_keys are byte arrays in the FP8 / FP4 layout (hcsa_quantize_rows converts bf16 rows).
        fused_append: the projection and the cache append in one kernel (hcsa_project_append) instead of two."""
        self.fused_append = fused_append
        self.spec = spec
        self.csa = spec.kind == "csa"
        self.kind = L.KIND_CSA if self.csa else L.KIND_HCA
        self.lowprec = lowprec
        self.p = params_for(spec, T=0, B=B, n_cap=n_cap, lowprec=lowprec)
        dt = torch_dtype(spec.dtype)
        self.cols, ncols = _col_offsets(spec)
        self.cache_t = cache
        self.cache = L.make_cache(cache["entries"], cache["win_kv"], cache["ring_g"], cache.get("idx_keys"),
                                  cache.get("ring_ki"))
        self.y = torch.empty((B, ncols), dtype=dt, device=device)
        self.out = torch.empty((B, spec.H * spec.dh), dtype=dt, device=device)
        self.ws_proj = self._ws(L.OP_PROJECT, device)
        if self.csa:
            self.sel = torch.empty((B, spec.topk), dtype=torch.int32, device=device)
            self.ws_index = self._ws(L.OP_CSA_DECODE_INDEX_TOPK, device)
            self.ws_attend = self._ws(L.OP_CSA_DECODE_ATTEND, device)
        else:
            self.ws_attend = self._ws(L.OP_HCA_DECODE_ATTEND, device)

    def _ws(self, op, device):
        n = L.hcsa_workspace_bytes(self.p, op)
        return torch.empty(max(n, 16), dtype=torch.uint8, device=device) if n else None

    def view(self, name):
        a, b = self.cols[name]
        return self.y[:, a:b]

    def step(self, x, W_cat, bias, pos):
        if self.fused_append:
            L.hcsa_project_append(self.p, self.kind, self.cache, pos, x, W_cat, bias, self.y, self.ws_proj)
        else:
            L.hcsa_project(self.p, self.kind, x, W_cat, self.y, self.ws_proj)
            L.hcsa_cache_append(self.p, self.cache, pos, self.view("kv"), self.view("g"),
                                self.view("ki") if self.csa else None, bias)
        if self.csa:
            L.csa_decode_index_topk(self.p, self.cache, pos, self.view("qi"), self.view("w"), self.sel,
                                    self.ws_index)
            L.csa_decode_attend(self.p, self.cache, pos, self.view("q"), self.sel, self.out, self.ws_attend)
        else:
            L.hca_decode_attend(self.p, self.cache, pos, self.view("q"), self.out, self.ws_attend)
        return self.out

    def out_project(self, x, W_o):
        """Residual update of a chained stack: x += out W_o, in place."""
        L.hcsa_out_project(self.p, self.out, W_o, x, self.ws_proj)
        return x
