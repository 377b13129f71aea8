"""Workload shapes and the seeded inputs for each of them.

The five named workloads are the CSA/HCA configurations of the DeepSeek-V4
hybrid-attention write-ups (CSA m=4 over overlapping width-8 pools with a
lightning indexer and top-k; HCA m'=128; a 128-token raw window), at the
sizes used for parity and benchmarking.  Distributions: x ~ N(0,1);
projection weights ~ N(0, 1/D); position bias B ~ N(0, 0.1) (variance 0.1);
decode caches ~ N(0,1).

Tensor ids (the generator's stream selector) are fixed per layer:
  0 x | 1 W_kv | 2 W_g | 3 W_ki | 4 W_qi | 5 W_w | 6 W_q | 7 B
  8 entries cache | 9 indexer-key cache | 10 window ring | 11 gate ring | 12 indexer-key ring
  13 W_o (output projection of a residual-chained stack)
Layer L of a multi-layer stack adds 16*L to every id except x (id 0), which
all layers share.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = ["LayerSpec", "DecodeSpec", "PREFILL", "DECODE", "prefill_inputs", "decode_inputs",
           "storage_kind", "proj_columns"]


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    kind: str            # "csa" or "hca"
    T: int               # tokens (prefill) -- ignored for decode
    D: int
    m: int               # compression ratio
    width: int           # pool width Wc (8 for CSA, m for HCA)
    C: int               # compressed dim: key half C/2, value half C/2
    di: int = 0          # indexer dim (CSA)
    Hi: int = 0          # indexer heads (CSA)
    topk: int = 0        # (CSA)
    window: int = 128
    H: int = 8
    dh: int = 64
    scale: float = 0.125
    dtype: str = "bf16"  # "f32" or "bf16" storage
    seed: int = 0

    @property
    def n_entries(self) -> int:
        return -(-self.T // self.m)

    def replace(self, **kw) -> "LayerSpec":
        return dataclasses.replace(self, **kw)


@dataclasses.dataclass(frozen=True)
class DecodeSpec:
    layers: tuple        # LayerSpec per layer (T unused)
    B: int               # sequences
    P: int               # position of the new token (= prefix length)
    seed: int = 0
    residual: bool = False   # chain the layers: x_{l+1} = x_l + out_l W_o,l (W_o ~ N(0, 1/(H dh)))

    def n_cache_entries(self, layer: LayerSpec) -> int:
        # entries fully formed by the prefix [0, P): entry j is complete once token m*j+m-1 < P
        return self.P // layer.m


def proj_columns(s: LayerSpec) -> list[tuple[str, int]]:
    """Column blocks of the concatenated projection W_cat = [W_kv | W_g | W_ki | W_qi | W_w | W_q]."""
    cols = [("kv", s.C), ("g", s.C)]
    if s.kind == "csa":
        cols += [("ki", s.di), ("qi", s.Hi * s.di), ("w", s.Hi)]
    cols += [("q", s.H * s.dh)]
    return cols


def storage_kind(s: LayerSpec) -> int:
    from . import KIND_BF16, KIND_F32
    return KIND_F32 if s.dtype == "f32" else KIND_BF16


_CSA_BIG = dict(kind="csa", D=2048, m=4, width=8, C=1024, di=64, Hi=32, topk=512, window=128, H=64, dh=512,
                scale=1.0 / math.sqrt(512.0), dtype="bf16")

PREFILL = {
    # CSA layer forward, fp32 storage, T=2048 (the small correctness workload)
    "csa_f32_t2048": LayerSpec(kind="csa", T=2048, D=512, m=4, width=8, C=128, di=32, Hi=4, topk=64,
                               window=128, H=8, dh=64, scale=0.125, dtype="f32", seed=0),
    # HCA layer prefill, bf16, T=65536
    "hca_bf16_t65536": LayerSpec(kind="hca", T=65536, D=1024, m=128, width=128, C=256, window=128, H=16,
                                 dh=128, scale=1.0 / math.sqrt(128.0), dtype="bf16", seed=1),
    # CSA layer prefill, bf16, T=131072
    "csa_bf16_t131072": LayerSpec(T=131072, seed=2, **_CSA_BIG),
}

_HCA_BIG = dict(kind="hca", D=2048, m=128, width=128, C=1024, window=128, H=64, dh=512,
                scale=1.0 / math.sqrt(512.0), dtype="bf16")

DECODE = {
    # CSA decode step: 32 sequences with a 262144-token prefix (65536 entries)
    "csa_decode_b32_p262144": DecodeSpec(layers=(LayerSpec(T=0, seed=3, **_CSA_BIG),), B=32, P=262144, seed=3),
    # 8-layer CSA/HCA alternating decode: 4 sequences at 1M context, top-k 1024 in the CSA layers
    "hybrid_decode_b4_p1048576": DecodeSpec(
        layers=tuple(LayerSpec(T=0, seed=4, **dict(_CSA_BIG, topk=1024)) if i % 2 == 0
                     else LayerSpec(T=0, seed=4, **_HCA_BIG) for i in range(8)),
        B=4, P=1048576, seed=4),
    # V4-style schedule: two HCA layers, then CSA and HCA alternating, chained through the residual
    # stream by an output projection per layer; 4 sequences at 1M context
    "v4_decode_b4_p1048576": DecodeSpec(
        layers=tuple(LayerSpec(T=0, seed=5, **_HCA_BIG) if (i < 2 or i % 2 == 1)
                     else LayerSpec(T=0, seed=5, **dict(_CSA_BIG, topk=1024)) for i in range(8)),
        B=4, P=1048576, seed=5, residual=True),
}


def _weights(s: LayerSpec, seed: int, base: int, kind: int) -> dict:
    from . import normal
    wstd = 1.0 / math.sqrt(s.D)
    out = {"W_kv": normal(seed, base + 1, (s.D, s.C), wstd, kind),
           "W_g": normal(seed, base + 2, (s.D, s.C), wstd, kind)}
    if s.kind == "csa":
        out["W_ki"] = normal(seed, base + 3, (s.D, s.di), wstd, kind)
        out["W_qi"] = normal(seed, base + 4, (s.D, s.Hi * s.di), wstd, kind)
        out["W_w"] = normal(seed, base + 5, (s.D, s.Hi), wstd, kind)
    out["W_q"] = normal(seed, base + 6, (s.D, s.H * s.dh), wstd, kind)
    out["B"] = normal(seed, base + 7, (s.width, s.C), math.sqrt(0.1), kind)
    return out


def w_cat(s: LayerSpec, ws: dict) -> np.ndarray:
    names = {"kv": "W_kv", "g": "W_g", "ki": "W_ki", "qi": "W_qi", "w": "W_w", "q": "W_q"}
    return np.ascontiguousarray(np.concatenate([ws[names[n]] for n, _ in proj_columns(s)], axis=1))


def prefill_inputs(s: LayerSpec, rows=None) -> dict:
    """x[T,D], the weights, W_cat[D, sum(cols)] and B[width, C] in storage format."""
    from . import normal
    kind = storage_kind(s)
    out = _weights(s, s.seed, 0, kind)
    out["x"] = normal(s.seed, 0, (s.T, s.D), 1.0, kind)
    out["W_cat"] = w_cat(s, out)
    return out


def decode_inputs(d: DecodeSpec, layer_index: int, with_cache: bool = True, seqs=None, n_cap=None) -> dict:
    """Weights, new-token x[B,D] and (optionally) the cache of one layer of a decode workload.

    seqs restricts the cache to a subset of sequences; n_cap overrides the entry capacity
    (default: the P // m entries the prefix has formed)."""
    from . import normal
    s = d.layers[layer_index]
    kind = storage_kind(s)
    base = 16 * layer_index
    out = _weights(s, d.seed, base, kind)
    out["W_cat"] = w_cat(s, out)
    out["x"] = normal(d.seed, 0, (d.B, s.D), 1.0, kind)
    if d.residual:
        out["W_o"] = normal(d.seed, base + 13, (s.H * s.dh, s.D), 1.0 / math.sqrt(s.H * s.dh), kind)
    if with_cache:
        N = d.n_cache_entries(s) if n_cap is None else n_cap
        seqs = list(range(d.B)) if seqs is None else list(seqs)
        dt = out["x"].dtype
        nb = len(seqs)

        def per_seq(tid, row_shape):
            arr = np.empty((nb,) + row_shape, dtype=dt)
            per = int(np.prod(row_shape))
            for i, b in enumerate(seqs):
                normal(d.seed, base + tid, row_shape, 1.0, kind, offset=b * per, out=arr[i])
            return arr

        out["entries"] = per_seq(8, (N, s.C))
        out["win_kv"] = per_seq(10, (s.window, s.C))
        out["ring_g"] = per_seq(11, (s.width, s.C))
        if s.kind == "csa":
            out["idx_keys"] = per_seq(9, (N, s.di))
            out["ring_ki"] = per_seq(12, (s.width, s.di))
    return out
