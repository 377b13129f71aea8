"""Sequence-sharded prefill and entry-sharded decode of one CSA / HCA layer over the ranks of a process group.

Prefill (ShardedPrefillLayer):

The sequence of T tokens is cut into 2R chunks of equal length (a multiple of 128; the last one takes the
remainder) and rank r of R takes chunks r and 2R - 1 - r: the zig-zag assignment, which gives every rank
the same causal work.  A rank

  1. projects the tokens of its chunks plus the window halo before each chunk (the raw keys of the first
     query of a chunk reach back window - 1 tokens; the compressor's pools reach back width - m <= that),
  2. forms the compressed entries (and indexer keys) whose pools end in its chunks,
  3. all-gathers the entries with one collective (the only exchange: every query may select any visible
     entry, and the entries are small: C values per m tokens),
  4. runs the indexer + top-k and the attention of its own queries.

Every step runs in libhcsa.so on the rank's own GPU through the calls' prefill row range (hcsa_params
row0 / row1: global token positions, full-length arrays, only the chunk's rows computed); torch.distributed
only moves the entries.  The arrays are allocated at full sequence length on every rank and filled where
the rank's rows are (simple, and the row arithmetic stays global).

The phases are separate methods (`compute_entries`, `exchange_entries`, `attend_local`) so that a caller
can overlap or replace the exchange; `forward` runs all three.
"""
from __future__ import annotations

import torch

from . import _lib as L
from .layer import PrefillLayer, _col_offsets, params_for, torch_dtype

__all__ = ["zigzag_chunks", "entry_range", "ShardedPrefillLayer", "ShardedDecodeLayer", "shard_cache"]

ALIGN = 128   # chunk boundaries: the library's row-range granularity


def zigzag_chunks(T: int, world: int, rank: int, align: int = ALIGN):
    """Token ranges [a, b) of rank `rank`: chunks rank and 2 world - 1 - rank of 2 world equal chunks whose
    length is a multiple of `align` (the last chunk ends at T; chunks past the end are empty)."""
    n = 2 * world
    L_ = -(-T // n)
    L_ = -(-L_ // align) * align
    out = []
    for c in (rank, n - 1 - rank):
        a, b = min(c * L_, T), min((c + 1) * L_, T)
        out.append((a, b))
    return out


def entry_range(a: int, b: int, T: int, m: int):
    """Entries whose pools end in token rows [a, b) of a sequence of T tokens: j in [a / m, ceil(b / m)),
    the same rule the library's compressor applies to a row range."""
    if b <= a:
        return a // m, a // m
    j1 = -(-T // m) if b == T else b // m
    return a // m, j1


class ShardedPrefillLayer(PrefillLayer):
    """One CSA or HCA layer over a sequence of T tokens, of which this rank computes its zig-zag chunks."""

    def __init__(self, spec, rank: int = 0, world: int = 1, device="cuda"):
        super().__init__(spec, device)
        self.rank, self.world = rank, world
        self.chunks = [(a, b) for a, b in zigzag_chunks(spec.T, world, rank) if b > a]
        self.halo = max(spec.window - 1, spec.width - spec.m)

    def _p(self, a, b):
        return params_for(self.spec, row0=a, row1=b)

    # ---------------------------------------------------------------- phase 1: own projections and entries
    def projected_rows(self):
        """Token ranges [h, b) this rank projects: each own chunk with the halo before it."""
        return [(max(0, a - self.halo), b) for a, b in self.chunks]

    def project_local(self, x, W_cat):
        for h, b in self.projected_rows():
            L.hcsa_project(self.p, self.kind, x[h:b], W_cat, self.y[h:b], self.ws_proj)

    def compress_local(self, bias):
        for a, b in self.chunks:
            p = self._p(a, b)
            if self.csa:
                L.csa_compress(p, self.view("kv"), self.view("g"), self.view("ki"), bias, self.entries,
                               self.idx_keys)
            else:
                L.hca_compress(p, self.view("kv"), self.view("g"), bias, self.entries)

    def compute_entries(self, x, W_cat, bias):
        self.project_local(x, W_cat)
        self.compress_local(bias)

    def local_entry_blocks(self):
        """(j0, j1) of the entries this rank formed, one block per chunk (always two: empty when the chunk is)."""
        T, m = self.spec.T, self.spec.m
        return [entry_range(a, b, T, m) for a, b in zigzag_chunks(T, self.world, self.rank)]

    # ---------------------------------------------------------------- phase 2: the exchange
    def exchange_entries(self, group=None):
        """All-gather every rank's entry blocks (and indexer keys) into this rank's full-length arrays: one
        collective per array over a padded [2, E, C] block per rank."""
        if self.world == 1:
            return
        import torch.distributed as dist
        T, m = self.spec.T, self.spec.m
        all_blocks = [[entry_range(a, b, T, m) for a, b in zigzag_chunks(T, self.world, r)]
                      for r in range(self.world)]
        E = max(j1 - j0 for blocks in all_blocks for j0, j1 in blocks)
        arrays = [self.entries] + ([self.idx_keys] if self.csa else [])
        for arr in arrays:
            send = torch.zeros((2, E, arr.shape[1]), dtype=arr.dtype, device=arr.device)
            for i, (j0, j1) in enumerate(all_blocks[self.rank]):
                send[i, :j1 - j0] = arr[j0:j1]
            recv = [torch.empty_like(send) for _ in range(self.world)]
            dist.all_gather(recv, send, group=group)
            for r in range(self.world):
                if r == self.rank:
                    continue
                for i, (j0, j1) in enumerate(all_blocks[r]):
                    arr[j0:j1] = recv[r][i, :j1 - j0]

    # ---------------------------------------------------------------- phase 3: own queries
    def attend_local(self):
        for a, b in self.chunks:
            p = self._p(a, b)
            if self.csa:
                L.csa_index_topk(p, self.view("qi"), self.view("w"), self.idx_keys, self.sel, self.ws_index)
                L.csa_attend(p, self.view("q"), self.view("kv"), self.entries, self.sel, self.out,
                             self.ws_attend)
            else:
                L.hca_attend(p, self.view("q"), self.view("kv"), self.entries, self.out, self.ws_attend)
        return self.out

    def forward(self, x, W_cat, bias, group=None):
        """The layer for this rank's rows: out[a:b] of each own chunk (other rows are not written)."""
        self.compute_entries(x, W_cat, bias)
        self.exchange_entries(group)
        return self.attend_local()


# ====================================================================================================== decode

def shard_cache(cache: dict, rank: int, world: int) -> dict:
    """This rank's shard of a decode cache: entries (and indexer keys) [ent0, ent0 + n_shard) of every
    sequence, n_shard = ceil(n_cap / world) (the last shard zero-padded); the rings are copied whole."""
    B, n_cap = cache["entries"].shape[:2]
    n_shard = -(-n_cap // world)
    a, b = rank * n_shard, min((rank + 1) * n_shard, n_cap)
    out = {}
    for k in ("entries", "idx_keys"):
        if k in cache:
            t = cache[k]
            sh = torch.zeros((B, n_shard) + tuple(t.shape[2:]), dtype=t.dtype, device=t.device)
            if b > a:
                sh[:, :b - a] = t[:, a:b]
            out[k] = sh
    for k in ("win_kv", "ring_g", "ring_ki"):
        if k in cache:
            out[k] = cache[k].clone()
    return out


class ShardedDecodeLayer:
    """One layer's decode step for B sequences whose compressed caches are split by entry index over the
    ranks: rank r holds entries [r n_shard, (r + 1) n_shard) of every sequence (shard_cache), every rank
    holds the rings and the weights.  A step:

      1. every rank projects the new token and appends it (the rings everywhere; a formed entry only on the
         rank that holds it);
      2. CSA: the indexer and an exact top-k over the rank's own entries, with their scores; one all-gather
         of the (index, score) candidates; the exact global top-k of their union on every rank (a global
         top-k entry is always in the top-k of its own shard);
      3. attention over the rank's part of the keys (its selected / visible entries; the raw window on rank
         0) as an unnormalized partial per head; one all-gather of the partials and their log-sum-exp merge.

    Every step runs in libhcsa.so; torch.distributed moves the candidates and the partials."""

    def __init__(self, spec, B, n_total, cache: dict, rank: int = 0, world: int = 1, device="cuda"):
        self.spec = spec
        self.csa = spec.kind == "csa"
        self.kind = L.KIND_CSA if self.csa else L.KIND_HCA
        self.rank, self.world = rank, world
        self.n_shard = -(-n_total // world)
        self.ent0 = rank * self.n_shard
        self.p = params_for(spec, T=0, B=B, n_cap=self.n_shard, ent0=self.ent0, ent_shard=True)
        self.cache_t = cache
        self.cache = L.make_cache(cache["entries"], cache["win_kv"], cache["ring_g"], cache.get("idx_keys"),
                                  cache.get("ring_ki"))
        dt = torch_dtype(spec.dtype)
        self.cols, ncols = _col_offsets(spec)
        self.y = torch.empty((B, ncols), dtype=dt, device=device)
        self.out = torch.empty((B, spec.H * spec.dh), dtype=dt, device=device)
        self.part = torch.empty(B * spec.H * (spec.dh + 2), dtype=torch.float32, device=device)
        self.ws_proj = self._ws(L.OP_PROJECT, device)
        if self.csa:
            self.sel_l = torch.empty((B, spec.topk), dtype=torch.int32, device=device)
            self.score_l = torch.empty((B, spec.topk), dtype=torch.float32, device=device)
            self.sel = torch.empty((B, spec.topk), dtype=torch.int32, device=device)
            self.ws_index = self._ws(L.OP_CSA_DECODE_INDEX_TOPK_SHARD, device)
            self.ws_attend = self._ws(L.OP_CSA_DECODE_ATTEND_SHARD, device)
        else:
            self.ws_attend = self._ws(L.OP_HCA_DECODE_ATTEND_SHARD, device)

    def _ws(self, op, device):
        n = L.hcsa_workspace_bytes(self.p, op)
        return torch.empty(max(n, 16), dtype=torch.uint8, device=device) if n else None

    def view(self, name):
        a, b = self.cols[name]
        return self.y[:, a:b]

    def _gather(self, t, group):
        if self.world == 1:
            return [t]
        import torch.distributed as dist
        bufs = [torch.empty_like(t) for _ in range(self.world)]
        dist.all_gather(bufs, t.contiguous(), group=group)
        return bufs

    def select(self, group=None):
        """Step 2: the global top-k of every sequence in self.sel."""
        L.csa_decode_index_topk_shard(self.p, self.cache, self.pos, self.view("qi"), self.view("w"), self.sel_l,
                                      self.score_l, self.ws_index)
        cs = torch.cat(self._gather(self.sel_l, group), dim=1)
        cv = torch.cat(self._gather(self.score_l, group), dim=1)
        L.csa_topk_merge(self.p, cs, cv, self.sel)

    def attend(self, group=None):
        """Step 3: this rank's partial, the all-gather and the merge into self.out."""
        if self.csa:
            L.csa_decode_attend_shard(self.p, self.cache, self.pos, self.view("q"), self.sel, self.rank == 0,
                                      self.part, self.ws_attend)
        else:
            L.hca_decode_attend_shard(self.p, self.cache, self.pos, self.view("q"), self.rank == 0, self.part,
                                      self.ws_attend)
        parts = torch.stack(self._gather(self.part, group))
        L.hcsa_merge_partials(self.p, parts, self.world, self.out)
        return self.out

    def step(self, x, W_cat, bias, pos, group=None):
        self.pos = pos
        L.hcsa_project(self.p, self.kind, x, W_cat, self.y, self.ws_proj)
        L.hcsa_cache_append(self.p, self.cache, pos, self.view("kv"), self.view("g"),
                            self.view("ki") if self.csa else None, bias)
        if self.csa:
            self.select(group)
        return self.attend(group)
