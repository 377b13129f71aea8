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


# ---------------------------------------------------------------------------------------- entry-sharded decode
CSA_DEC = synth.LayerSpec(kind="csa", T=0, D=256, m=4, width=8, C=1024, di=64, Hi=32, topk=128, window=128, H=64,
                          dh=512, scale=512 ** -0.5, dtype="bf16", seed=91)
HCA_DEC = synth.LayerSpec(kind="hca", T=0, D=256, m=128, width=128, C=1024, window=128, H=64, dh=512,
                          scale=512 ** -0.5, dtype="bf16", seed=92)
DEC_CASES = {
    # positions closing entries in the first, middle and last shard; fewer visible than k; a window only
    "csa": (CSA_DEC, [7999, 4003, 300, 3], 2000),
    "csa_rows": (CSA_DEC.replace(seed=93), [279999, 140003], 70000),   # shards above 32768 entries
    "hca": (HCA_DEC, [12799, 6399, 1000, 50], 100),
}


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("name", list(DEC_CASES))
def test_sharded_decode_emulated_ranks(name, world):
    """Shards of the cache on one GPU, the all-gathers emulated by concatenation: the merged selection equals
    the unsharded layer's, the merged output matches the oracle on that selection."""
    import long_context_compressed_05_b200 as h
    import oracle
    from tests._helpers import check_out, check_selection, host64
    spec, pos, n_cap = DEC_CASES[name]
    if name == "csa_rows" and world == 3:
        pytest.skip("one sharded split of the long rows is enough")
    B = len(pos)
    d = synth.DecodeSpec(layers=(spec,), B=B, P=max(pos), seed=spec.seed)
    inp = synth.decode_inputs(d, 0, n_cap=n_cap)
    keys = ("entries", "win_kv", "ring_g", "idx_keys", "ring_ki")
    full = {k: dev(inp[k]) for k in keys if k in inp}
    x, W, Bb = dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"])
    pos_t = torch.tensor(pos, dtype=torch.int32, device="cuda")
    ref_layer = h.DecodeLayer(spec, B, n_cap, {k: v.clone() for k, v in full.items()})
    ref_layer.step(x, W, Bb, pos_t)
    ranks = [h.ShardedDecodeLayer(spec, B, n_cap, h.shard_cache(full, r, world), r, world) for r in range(world)]
    for lay in ranks:
        lay.pos = pos_t
        h.hcsa_project_append(lay.p, lay.kind, lay.cache, pos_t, x, W, Bb, lay.y, lay.ws_proj)
    if spec.kind == "csa":
        for lay in ranks:
            h.csa_decode_index_topk_shard(lay.p, lay.cache, pos_t, lay.view("qi"), lay.view("w"), lay.sel_l,
                                          lay.score_l, lay.ws_index)
        cs = torch.cat([lay.sel_l for lay in ranks], dim=1)
        cv = torch.cat([lay.score_l for lay in ranks], dim=1)
        for lay in ranks:
            h.csa_topk_merge(lay.p, cs, cv, lay.sel)
            h.csa_decode_attend_shard(lay.p, lay.cache, pos_t, lay.view("q"), lay.sel, lay.rank == 0, lay.part,
                                      lay.ws_attend)
    else:
        for lay in ranks:
            h.hca_decode_attend_shard(lay.p, lay.cache, pos_t, lay.view("q"), lay.rank == 0, lay.part, lay.ws_attend)
    parts = torch.stack([lay.part for lay in ranks])
    for lay in ranks:
        h.hcsa_merge_partials(lay.p, parts, world, lay.out)
    torch.cuda.synchronize()
    assert h.hcsa_get_device_status() == 0
    # the appended entries: on the rank that holds them, as in the unsharded cache
    for b, P in enumerate(pos):
        if (P + 1) % spec.m == 0:
            j = (P + 1) // spec.m - 1
            r = j // ranks[0].n_shard
            assert torch.equal(ranks[r].cache_t["entries"][b, j - ranks[r].ent0], ref_layer.cache_t["entries"][b, j])
    ref = oracle.decode_step(spec, inp, np.array(pos))
    for lay in ranks:
        assert torch.equal(lay.out, ranks[0].out)
    for b in range(B):
        if spec.kind == "csa":
            assert torch.equal(ranks[0].sel[b], ref_layer.sel[b])
            sel = ranks[0].sel[b].cpu().numpy()[None]
            nv = np.array([min(pos[b] // spec.m, n_cap)])
            check_selection(sel, ref["sel"][b:b + 1], ref["gap"][b:b + 1], ref["scores"][b][None], nv, spec.topk,
                            exact=False)
            ref_out = oracle.decode_attend_with_sel(spec, ref, b, sel[0])
        else:
            ref_out = ref["out"][b]
        check_out(host64(ranks[0].out[b]), ref_out, "bf16")
        # against the unsharded layer: the same keys, only the merge order differs
        np.testing.assert_allclose(host64(ranks[0].out[b]), host64(ref_layer.out[b]), rtol=2 ** -7, atol=2e-3)
