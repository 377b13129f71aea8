"""The sequence-sharded prefill on one GPU: two ranks emulated in one process (the all-gather of the
entries replaced by copies between their buffers) must reproduce the unsharded GPU layer bit for bit on
every rank's rows -- selections and outputs -- since every row and every entry is computed by the same
kernels from the same inputs.  Covers the library's prefill row ranges in the projection, compressor,
indexer + top-k (tensor-core and CUDA-core paths) and attention kernels (CSA tensor-core and generic,
HCA tensor-core)."""
import numpy as np
import pytest
import torch

import synth
from tests._helpers import dev

pytestmark = pytest.mark.gpu

CASES = {
    "csa_small": synth.LayerSpec(kind="csa", T=1003, D=256, m=4, width=8, C=256, di=64, Hi=8, topk=64, window=128,
                                 H=8, dh=128, scale=128 ** -0.5, dtype="bf16", seed=61),
    "csa_tc": synth.LayerSpec(kind="csa", T=2600, D=256, m=4, width=8, C=1024, di=64, Hi=32, topk=128, window=128,
                              H=64, dh=512, scale=512 ** -0.5, dtype="bf16", seed=62),
    "hca_small": synth.LayerSpec(kind="hca", T=1500, D=256, m=128, width=128, C=256, window=128, H=4, dh=128,
                                 scale=128 ** -0.5, dtype="bf16", seed=63),
    "csa_f32": synth.PREFILL["csa_f32_t2048"].replace(T=1100, seed=64),
    "hca_f32": synth.LayerSpec(kind="hca", T=1300, D=128, m=128, width=128, C=128, window=128, H=4, dh=64,
                               scale=0.125, dtype="f32", seed=65),
}


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("name", list(CASES))
def test_sharded_prefill_emulated_ranks_match_unsharded(name, world):
    import long_context_compressed_05_b200 as h
    spec = CASES[name]
    inp = synth.prefill_inputs(spec)
    x, W, B = dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"])
    full = h.PrefillLayer(spec)
    full.forward(x, W, B)
    ranks = [h.ShardedPrefillLayer(spec, r, world) for r in range(world)]
    for lay in ranks:
        for t in [lay.y, lay.entries, lay.out] + ([lay.idx_keys] if lay.csa else []):
            t.fill_(float("nan"))   # nothing a rank neither computes nor receives may be read
        lay.project_local(x, W)
        for a, b in lay.projected_rows():
            # a GEMM over fewer rows may split K differently (the sum's rounding order): same tolerance as
            # the projection's own parity tests, then the full layer's rows so that the rest is bit-exact
            ref = full.y[a:b].float()
            err = (lay.y[a:b].float() - ref).abs()
            assert bool((err <= 2.0 ** -7 * ref.abs() + 1e-3).all()), (a, b, float(err.max()))
            lay.y[a:b] = full.y[a:b]
        lay.compress_local(B)
    # the all-gather, emulated: every rank receives the other ranks' entry blocks
    for r, lay in enumerate(ranks):
        for s, src in enumerate(ranks):
            if s == r:
                continue
            for j0, j1 in src.local_entry_blocks():
                lay.entries[j0:j1] = src.entries[j0:j1]
                if lay.csa:
                    lay.idx_keys[j0:j1] = src.idx_keys[j0:j1]
    torch.cuda.synchronize()
    covered = np.zeros(spec.T, int)
    for lay in ranks:
        assert torch.equal(lay.entries, full.entries)
        if lay.csa:
            assert torch.equal(lay.idx_keys, full.idx_keys)
        # no query of the rank's ranges sees an entry at or past (row1 - 1) / m of its last range: poisoned
        j_lim = max((b - 1) // spec.m for a, b in lay.chunks)
        lay.entries[j_lim:] = float("nan")
        if lay.csa:
            lay.idx_keys[j_lim:] = float("nan")
        lay.attend_local()
        torch.cuda.synchronize()
        assert h.hcsa_get_device_status() == 0
        for a, b in lay.chunks:
            covered[a:b] += 1
            assert torch.equal(lay.out[a:b], full.out[a:b]), (a, b)
            if lay.csa:
                assert torch.equal(lay.sel[a:b], full.sel[a:b]), (a, b)
    assert (covered == 1).all()
