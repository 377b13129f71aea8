"""The entry-sharded decode (cache split by entry index, candidate all-gather, exact merge of the top-k,
per-shard attention partials, log-sum-exp merge) on the CPU: gloo ranks run ShardedDecodeLayer.select and
.attend with the library calls replaced by fp64 stand-ins that keep the calls' contracts (global indices,
the shard's local rows, the window on one rank only, the partial layout).  The projections and the appended
cache come from the oracle's unsharded decode step, so the merged selection must equal the oracle's and
the merged output must match it to fp64 rounding."""
import os
import socket
import types

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import synth


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _partial(q, K, V, scale, H, dh):
    """Unnormalized softmax partial of one query over keys K / values V: acc [H, dh], (max, sum) [H, 2]."""
    acc = np.zeros((H, dh))
    ml = np.zeros((H, 2))
    ml[:, 0] = -np.inf
    if K.shape[0] == 0:
        return acc, ml
    lg = (q.reshape(H, dh) @ K.T) * scale               # [H, keys]
    m = lg.max(axis=1)
    e = np.exp(lg - m[:, None])
    return e @ V, np.stack([m, e.sum(axis=1)], axis=1)


def _stand_in(spec, ref):
    """Library stand-ins on CPU tensors; `ref` is the oracle's unsharded decode step (after the append)."""
    H, dh, m, W = spec.H, spec.dh, spec.m, spec.window

    def index_topk_shard(p, cache, pos, qi, w, sel, sel_scores, ws, stream=None):
        for b in range(p.B):
            P = int(pos[b])
            nv = min(max(P // m - p.ent0, 0), p.n_cap)
            keys = ref["idx_keys"][b][p.ent0:p.ent0 + p.n_cap]
            s = oracle.index_scores(qi[b:b + 1].double().numpy(), w[b:b + 1].double().numpy(), keys,
                                    np.array([nv]), spec.Hi, spec.di)
            sl, _, _ = oracle.topk(s, np.array([nv]), p.topk)
            sel[b] = torch.from_numpy(np.where(sl[0] >= 0, sl[0] + p.ent0, -1).astype(np.int32))
            sel_scores[b] = torch.from_numpy(np.where(sl[0] >= 0, s[0][np.maximum(sl[0], 0)], -np.inf))

    def topk_merge(p, cs, cv, sel, stream=None):
        for b in range(p.B):
            j, v = cs[b].numpy(), cv[b].numpy()
            ok = j >= 0
            order = np.lexsort((j[ok], -v[ok]))[:p.topk]       # score desc, then index asc
            pick = np.sort(j[ok][order])
            out = -np.ones(p.topk, np.int32)
            out[:len(pick)] = pick
            sel[b] = torch.from_numpy(out)

    def attend_shard(p, pos, q, sel, with_window, part):
        B = p.B
        acc = np.zeros((B, H, dh))
        ml = np.zeros((B, H, 2))
        for b in range(B):
            P = int(pos[b])
            ent = ref["entries"][b]
            if sel is not None:
                js = [int(j) for j in sel[b] if p.ent0 <= j < p.ent0 + p.n_cap]
            else:
                js = list(range(p.ent0, min(P // m, p.ent0 + p.n_cap)))
            rows = [ent[j] for j in js]
            if with_window:
                rows += [ref["win_kv"][b][t % W] for t in range(max(0, P - W + 1), P + 1)]
            R = np.array(rows).reshape(-1, spec.C)
            acc[b], ml[b] = _partial(q[b].double().numpy(), R[:, :dh], R[:, dh:], spec.scale, H, dh)
        part.copy_(torch.from_numpy(np.concatenate([acc.ravel(), ml.ravel()])))

    def merge(p, parts, n, out, stream=None):
        blk = p.B * H * dh
        a = parts.double().numpy().reshape(n, -1)
        acc = a[:, :blk].reshape(n, p.B, H, dh)
        ml = a[:, blk:].reshape(n, p.B, H, 2)
        M = ml[..., 0].max(axis=0)
        wgt = np.where(np.isfinite(ml[..., 0]), np.exp(ml[..., 0] - M), 0.0)
        Z = (wgt * ml[..., 1]).sum(axis=0)
        o = (wgt[..., None] * acc).sum(axis=0) / Z[..., None]
        out.copy_(torch.from_numpy(o.reshape(p.B, H * dh)))

    import long_context_compressed_05_b200._lib as real
    return types.SimpleNamespace(
        KIND_CSA=0, KIND_HCA=1, OP_PROJECT=0, OP_CSA_DECODE_INDEX_TOPK_SHARD=7, OP_CSA_DECODE_ATTEND_SHARD=8,
        OP_HCA_DECODE_ATTEND_SHARD=9, hcsa_workspace_bytes=lambda p, op: 0, make_params=real.make_params,
        make_cache=lambda *a, **k: None,
        csa_decode_index_topk_shard=index_topk_shard, csa_topk_merge=topk_merge,
        csa_decode_attend_shard=lambda p, c, pos, q, sel, ww, part, ws=None, stream=None:
            attend_shard(p, pos, q, sel, ww, part),
        hca_decode_attend_shard=lambda p, c, pos, q, ww, part, ws=None, stream=None:
            attend_shard(p, pos, q, None, ww, part),
        hcsa_merge_partials=merge)


def _worker(rank, world, port, spec, pos, n_cap, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    import long_context_compressed_05_b200.sharded as sh
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B = len(pos)
        d = synth.DecodeSpec(layers=(spec,), B=B, P=max(pos), seed=spec.seed)
        inp = synth.decode_inputs(d, 0, n_cap=n_cap)
        ref = oracle.decode_step(spec, inp, np.array(pos))
        if spec.kind == "csa":   # the indexer keys after the append
            ref["idx_keys"] = [oracle.to_f64(inp["idx_keys"][b]).copy() for b in range(B)]
            for b, ne in enumerate(ref["new_entry"]):
                if ne is not None and ne["j"] < n_cap:
                    ref["idx_keys"][b][ne["j"]] = ne["idx_key"]
        sh.L = _stand_in(spec, ref)
        cache = {k: torch.zeros(1) for k in ("entries", "win_kv", "ring_g")}
        lay = sh.ShardedDecodeLayer(spec, B, n_cap, cache, rank, world, device="cpu")
        lay.y = lay.y.double()
        lay.out = lay.out.double()
        lay.part = lay.part.double()
        lay.y.copy_(torch.from_numpy(np.stack(ref["y"])))   # the step's projections (oracle)
        lay.pos = torch.tensor(pos, dtype=torch.int32)
        if lay.csa:
            lay.score_l = lay.score_l.double()
            lay.select()
        lay.attend()
        results[rank] = (lay.sel.numpy().copy() if lay.csa else None, lay.out.numpy().copy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


CASES = {
    "csa": (synth.LayerSpec(kind="csa", T=0, D=32, m=4, width=8, C=32, di=8, Hi=2, topk=8, window=16, H=2, dh=16,
                            scale=0.25, dtype="f32", seed=95), [401, 203, 3, 60], 110),
    "hca": (synth.LayerSpec(kind="hca", T=0, D=32, m=16, width=16, C=32, window=16, H=2, dh=16, scale=0.25,
                            dtype="f32", seed=96), [511, 255, 5, 100], 40),
}


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("name", list(CASES))
def test_sharded_decode_matches_unsharded_oracle(name, world):
    spec, pos, n_cap = CASES[name]
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), spec, pos, n_cap, results), nprocs=world, join=True)
    d = synth.DecodeSpec(layers=(spec,), B=len(pos), P=max(pos), seed=spec.seed)
    ref = oracle.decode_step(spec, synth.decode_inputs(d, 0, n_cap=n_cap), np.array(pos))
    for r in range(world):
        sel, out = results[r]
        if sel is not None:
            np.testing.assert_array_equal(sel, ref["sel"])
        # fp64 partials against the oracle's output rounded to fp32 storage
        np.testing.assert_allclose(out, ref["out"], rtol=1e-6, atol=1e-7)
