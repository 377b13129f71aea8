"""The sequence-sharded prefill (zig-zag chunks, halos, entry all-gather) on the CPU: two gloo ranks run
ShardedPrefillLayer with the library calls replaced by an oracle-backed stand-in that honours the same row
range contract (global positions, full-length arrays, only the range's rows / entries computed).  Rows a
rank does not project are NaN, so a halo that is too short or an entry block gathered to the wrong place
shows up as NaN or as a mismatch.  Every rank's selections must equal the unsharded oracle layer's and
its outputs must match them to fp32 rounding."""
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


def _stand_in(spec):
    """A module with the binding's names: each call computes with the oracle on CPU tensors, rows or entries
    of the params' row range only (row0 = row1 = 0: everything)."""
    st = oracle.storage_code(spec.dtype)
    cols = oracle._col_slices(spec)
    B64 = None

    def rng(p):
        return (0, p.T) if p.row0 == 0 and p.row1 == 0 else (p.row0, p.row1)

    def f64(t):
        return t.detach().double().numpy()

    def proj_cols(p, kind):
        return sum(s.stop - s.start for s in cols.values())

    def project(p, kind, x, W, y, ws=None, stream=None):
        y.copy_(torch.from_numpy(oracle.project(f64(x), f64(W), st)))

    def compress(p, kv, g, ki, bias, entries, idx_keys, stream=None):
        a, b = rng(p)
        j0, j1 = a // p.m, (-(-p.T // p.m) if b == p.T else b // p.m)
        y = f64(kv.as_strided((p.T, kv.stride(0)), (kv.stride(0), 1)))   # the whole projection row
        base = y.ctypes.data
        ki_ptr = base + 8 * cols["ki"].start if ki is not None else None
        ent, idx = oracle.compress(p.T, p.C, p.m, p.width, base, y.shape[1], base + 8 * cols["g"].start,
                                   y.shape[1], f64(bias), ki_ptr, y.shape[1], p.di if ki is not None else 0, st)
        entries[j0:j1] = torch.from_numpy(ent[j0:j1])
        if ki is not None:
            idx_keys[j0:j1] = torch.from_numpy(idx[j0:j1])

    def index_topk(p, qi, w, idx_keys, sel, ws, stream=None):
        a, b = rng(p)
        rows = np.arange(a, b)
        N = idx_keys.shape[0]
        nv = oracle.prefill_n_vis(rows, p.m, N)
        s = oracle.index_scores(f64(qi[a:b]), f64(w[a:b]), f64(idx_keys), nv, p.Hi, p.di)
        sl, _, _ = oracle.topk(s, nv, p.topk)
        sel[a:b] = torch.from_numpy(sl)

    def attend(p, q, kv, entries, sel, out, dense):
        a, b = rng(p)
        rows = np.arange(a, b)
        N = entries.shape[0]
        raw = f64(kv.as_strided((p.T, p.C), (kv.stride(0), 1)))
        o = oracle.attend(f64(q[a:b]), p.H, p.dh, p.scale, f64(entries),
                          None if dense else sel[a:b].numpy(), oracle.prefill_n_vis(rows, p.m, N), raw,
                          oracle.prefill_window_rows(rows, p.window), st)
        out[a:b] = torch.from_numpy(o)

    return types.SimpleNamespace(
        KIND_CSA=0, KIND_HCA=1, OP_PROJECT=0, OP_CSA_INDEX_TOPK=1, OP_CSA_ATTEND=2, OP_HCA_ATTEND=3,
        hcsa_proj_cols=proj_cols, hcsa_workspace_bytes=lambda p, op: 0, hcsa_project=project,
        csa_compress=compress,
        hca_compress=lambda p, kv, g, bias, entries, stream=None: compress(p, kv, g, None, bias, entries, None),
        csa_index_topk=index_topk,
        csa_attend=lambda p, q, kv, entries, sel, out, ws=None, stream=None: attend(p, q, kv, entries, sel, out,
                                                                                  False),
        hca_attend=lambda p, q, kv, entries, out, ws=None, stream=None: attend(p, q, kv, entries, None, out, True),
        make_params=__import__("long_context_compressed_05_b200._lib", fromlist=["make_params"]).make_params)


def _worker(rank, world, port, spec, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    import long_context_compressed_05_b200.layer as layer_mod
    import long_context_compressed_05_b200.sharded as sh
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        fake = _stand_in(spec)
        layer_mod.L = fake
        sh.L = fake
        inp = synth.prefill_inputs(spec)
        lay = sh.ShardedPrefillLayer(spec, rank, world, device="cpu")
        for t in [lay.y, lay.entries, lay.out] + ([lay.idx_keys] if lay.csa else []):
            t.fill_(float("nan"))   # nothing this rank does not compute or receive may be read
        if lay.csa:
            lay.sel.fill_(-7)
        x = torch.from_numpy(oracle.to_f64(inp["x"])).to(lay.y.dtype)
        W = torch.from_numpy(oracle.to_f64(inp["W_cat"])).to(lay.y.dtype)
        Bb = torch.from_numpy(oracle.to_f64(inp["B"])).to(lay.y.dtype)
        lay.forward(x, W, Bb)
        rows = [(a, b) for a, b in lay.chunks]
        results[rank] = (rows, lay.out.double().numpy().copy(),
                         lay.sel.numpy().copy() if lay.csa else None)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("kind", ["csa", "hca"])
def test_sharded_prefill_matches_unsharded_oracle(kind):
    if kind == "csa":
        spec = synth.LayerSpec(kind="csa", T=2000, D=32, m=4, width=8, C=16, di=8, Hi=2, topk=8, window=128, H=2,
                               dh=8, scale=0.35, dtype="f32", seed=71)
    else:
        spec = synth.LayerSpec(kind="hca", T=2000, D=32, m=128, width=128, C=16, window=128, H=2, dh=8,
                               scale=0.35, dtype="f32", seed=72)
    world = 2
    mgr = mp.Manager()
    results = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), spec, results), nprocs=world, join=True)
    ref = oracle.prefill(spec, synth.prefill_inputs(spec))
    covered = np.zeros(spec.T, bool)
    for r in range(world):
        rows, out, sel = results[r]
        for a, b in rows:
            covered[a:b] = True
            # the stand-in projects row subsets, so a library matmul may round an fp64 sum differently
            np.testing.assert_allclose(out[a:b], ref["out"][a:b], rtol=1e-6, atol=1e-7)
            if sel is not None:
                np.testing.assert_array_equal(sel[a:b], ref["sel"][a:b])
    assert covered.all()
