"""GPU parity of the decode path (cache append, indexer + top-k over the cache, split attention) against
the fp64 oracle, and decode <-> prefill consistency, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._helpers import check_out, check_selection, dev, host64

pytestmark = pytest.mark.gpu

CSA_D = synth.LayerSpec(kind="csa", T=0, D=256, m=4, width=8, C=256, di=64, Hi=8, topk=64, window=128, H=8, dh=128,
                        scale=128 ** -0.5, dtype="bf16", seed=31)
HCA_D = synth.LayerSpec(kind="hca", T=0, D=256, m=128, width=128, C=256, window=128, H=4, dh=128,
                        scale=128 ** -0.5, dtype="bf16", seed=32)
# the tensor-core attention shapes (64 heads of 512, key segments of 128 merged by the combine kernel)
CSA_TC = CSA_D.replace(C=1024, H=64, dh=512, Hi=32, topk=128, scale=512 ** -0.5, seed=35)
HCA_TC = HCA_D.replace(C=1024, H=64, dh=512, scale=512 ** -0.5, seed=36)


def gpu_step(spec, inp, pos, n_cap):
    from long_context_compressed_05_b200 import DecodeLayer, hcsa_get_device_status
    cache = {k: dev(inp[k]) for k in ("entries", "win_kv", "ring_g", "idx_keys", "ring_ki") if k in inp}
    B = inp["x"].shape[0]
    layer = DecodeLayer(spec, B, n_cap, cache)
    pos_t = torch.tensor(pos, dtype=torch.int32, device="cuda")
    layer.step(dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"]), pos_t)
    torch.cuda.synchronize()
    assert hcsa_get_device_status() == 0
    return layer, cache


def compare_step(spec, inp, layer, cache, P, seqs):
    ref = oracle.decode_step(spec, inp, P, seqs=seqs)
    f32 = spec.dtype == "f32"
    for i, b in enumerate(seqs):
        # cache side effects: the new token's rows and any completed entry
        Pb = int(ref["P"][b])
        np.testing.assert_allclose(host64(cache["win_kv"][b, Pb % spec.window]), ref["win_kv"][i][Pb % spec.window],
                                   rtol=1e-6 if f32 else 2 ** -7, atol=1e-6)
        ne = ref["new_entry"][i]
        if ne is not None:
            np.testing.assert_allclose(host64(cache["entries"][b, ne["j"]]), ne["entry"],
                                       rtol=1e-6 if f32 else 2 ** -6, atol=1e-3 if not f32 else 1e-7)
            if spec.kind == "csa":
                np.testing.assert_allclose(host64(cache["idx_keys"][b, ne["j"]]), ne["idx_key"],
                                           rtol=1e-6 if f32 else 2 ** -6, atol=1e-3 if not f32 else 1e-7)
        if spec.kind == "csa":
            sel = layer.sel[b].cpu().numpy()[None]
            nv = np.array([min(Pb // spec.m, inp["entries"].shape[1])])
            check_selection(sel, ref["sel"][i:i + 1], ref["gap"][i:i + 1], ref["scores"][i][None], nv, spec.topk,
                            exact=f32)
            ref_out = oracle.decode_attend_with_sel(spec, ref, i, sel[0])
        else:
            ref_out = ref["out"][i]
        check_out(host64(layer.out[b]), ref_out, spec.dtype)


@pytest.mark.parametrize("spec,pos,n_cap", [
    (CSA_D, [515, 1023, 2000], 520),             # two appends close an entry
    (CSA_D.replace(dtype="f32", seed=33), [7, 100, 403], 110),
    (CSA_D, [3, 130, 259], 80),                   # no entry visible / fewer than k visible
    (HCA_D, [255, 1000, 383], 16),                # HCA: 255 and 383 close entries 1 and 2
    (HCA_D.replace(dtype="f32", seed=34), [127, 500, 64], 8),
    (CSA_TC, [515, 1023, 60], 300),               # P = 60: 15 visible < k and a partial window
    (HCA_TC, [255, 3000, 100], 30),               # 255 closes entry 1; 100: window only
])
def test_decode_small(spec, pos, n_cap):
    d = synth.DecodeSpec(layers=(spec,), B=len(pos), P=max(pos), seed=spec.seed)
    inp = synth.decode_inputs(d, 0, n_cap=n_cap)
    layer, cache = gpu_step(spec, inp, pos, n_cap)
    compare_step(spec, inp, layer, cache, np.array(pos), list(range(len(pos))))


@pytest.mark.parametrize("kind,dtype", [("csa", "f32"), ("csa", "bf16"), ("hca", "bf16")])
def test_decode_matches_prefill(kind, dtype):
    """Decode steps over a cache built from a GPU prefill reproduce the GPU prefill of the longer sequence."""
    from long_context_compressed_05_b200 import DecodeLayer, PrefillLayer
    base = CSA_D if kind == "csa" else HCA_D.replace(m=16, width=16)
    spec = base.replace(dtype=dtype)
    P0, n = (301, 9) if kind == "csa" else (251, 8)
    full = spec.replace(T=P0 + n)
    inp = synth.prefill_inputs(full)
    pre = PrefillLayer(full)
    pre.forward(dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"]))
    n_cap = (P0 + n) // spec.m + 2
    dt = pre.entries.dtype
    cache = {"entries": torch.zeros((1, n_cap, spec.C), dtype=dt, device="cuda"),
             "win_kv": torch.zeros((1, spec.window, spec.C), dtype=dt, device="cuda"),
             "ring_g": torch.zeros((1, spec.width, spec.C), dtype=dt, device="cuda")}
    nc = P0 // spec.m
    cache["entries"][0, :nc] = pre.entries[:nc]
    for p in range(max(0, P0 - spec.window), P0):
        cache["win_kv"][0, p % spec.window] = pre.view("kv")[p]
    for p in range(max(0, P0 - spec.width), P0):
        cache["ring_g"][0, p % spec.width] = pre.view("g")[p]
    if kind == "csa":
        cache["idx_keys"] = torch.zeros((1, n_cap, spec.di), dtype=dt, device="cuda")
        cache["idx_keys"][0, :nc] = pre.idx_keys[:nc]
        cache["ring_ki"] = torch.zeros((1, spec.width, spec.di), dtype=dt, device="cuda")
        for p in range(max(0, P0 - spec.width), P0):
            cache["ring_ki"][0, p % spec.width] = pre.view("ki")[p]
    layer = DecodeLayer(spec, 1, n_cap, cache)
    W, Bb = dev(inp["W_cat"]), dev(inp["B"])
    x = dev(inp["x"])
    for s in range(n):
        P = P0 + s
        layer.step(x[P:P + 1].contiguous(), W, Bb, torch.tensor([P], dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        if kind == "csa":
            a, b = layer.sel[0].cpu().numpy(), pre.sel[P].cpu().numpy()
            if dtype == "f32":
                np.testing.assert_array_equal(a, b)
            else:   # the one-row projection may round a few bf16 values differently from the T-row one
                assert len(set(a.tolist()) ^ set(b.tolist())) <= 4
        got, want = host64(layer.out[0]), host64(pre.out[P])
        if dtype == "f32":
            np.testing.assert_allclose(got, want, rtol=0, atol=1e-6)
        else:
            assert np.abs(got - want).max() <= 2e-2
    # every entry completed during the steps equals the prefill's entry
    for j in range(nc, (P0 + n) // spec.m):
        np.testing.assert_allclose(host64(cache["entries"][0, j]), host64(pre.entries[j]), rtol=2 ** -6, atol=1e-3)


@pytest.mark.parametrize("name", ["csa_decode_b32_p262144", "hybrid_decode_b4_p1048576"])
def test_decode_full_size_sampled(name):
    """Full-size decode workloads (all layers, all sequences on the GPU); the oracle checks sampled sequences."""
    d = synth.DECODE[name]
    seqs = [0, d.B - 1] if d.B > 2 else [0]
    for li, spec in enumerate(d.layers):
        if li >= 2 and li < len(d.layers) - 2:
            continue   # the middle layers repeat the first two shapes; check first two and last two
        inp = synth.decode_inputs(d, li)
        n_cap = inp["entries"].shape[1]
        layer, cache = gpu_step(spec, inp, [d.P] * d.B, n_cap)
        compare_step(spec, inp, layer, cache, d.P, seqs)
        del layer, cache
        torch.cuda.empty_cache()


def test_decode_long_rows_select():
    """Decode rows longer than 32768 entries take the multi-CTA select: a full row, a ragged last slice,
    a row with fewer visible entries than k, and a row whose indexer keys repeat 50 distinct vectors (hundreds
    of scores tie at the threshold: lowest indices first, via the single-CTA fallback).  Besides oracle parity,
    the selection must be exactly the top-k of the kernel's own fp32 scores (a property of the select itself)."""
    spec = CSA_TC.replace(seed=37)
    n_cap = 40000
    pos = [4 * n_cap, 4 * 35001 + 1, 4 * 100, 4 * 39000 + 3]
    d = synth.DecodeSpec(layers=(spec,), B=len(pos), P=max(pos), seed=spec.seed)
    inp = synth.decode_inputs(d, 0, n_cap=n_cap)
    keys = inp["idx_keys"]
    keys[3] = keys[3][np.arange(n_cap) % 50]
    layer, cache = gpu_step(spec, inp, pos, n_cap)
    compare_step(spec, inp, layer, cache, np.array(pos), list(range(len(pos))))
    scores = layer.ws_index[: len(pos) * n_cap * 4].view(torch.float32).view(len(pos), n_cap).cpu().numpy()
    sel = layer.sel.cpu().numpy()
    for b, P in enumerate(pos):
        n = min(P // spec.m, n_cap)
        s = scores[b, :n].astype(np.float64)
        s[s == 0] = 0.0
        order = np.lexsort((np.arange(n), -s))[: min(spec.topk, n)]
        want = np.full(spec.topk, -1, dtype=np.int64)
        want[: len(order)] = np.sort(order)
        np.testing.assert_array_equal(sel[b], want)


def test_decode_residual_stack():
    """A V4-style stack (two HCA layers, then a CSA layer) chained through the residual stream: every layer's
    output against the oracle on the GPU's own hidden state, and every residual update x += out W_o against
    the fp64 update of the GPU's own output, rounded once to bf16."""
    from long_context_compressed_05_b200 import DecodeLayer, hcsa_get_device_status
    d = synth.DecodeSpec(layers=(HCA_D.replace(seed=41), HCA_D.replace(seed=41), CSA_D.replace(seed=41)), B=3,
                         P=1000, seed=41, residual=True)
    pos = torch.full((d.B,), d.P, dtype=torch.int32, device="cuda")
    x = None
    for li, spec in enumerate(d.layers):
        inp = synth.decode_inputs(d, li)
        if x is None:
            x = dev(inp["x"])
        cache = {k: dev(inp[k]) for k in ("entries", "win_kv", "ring_g", "idx_keys", "ring_ki") if k in inp}
        layer = DecodeLayer(spec, d.B, inp["entries"].shape[1], cache)
        x_in = host64(x)
        layer.step(x, dev(inp["W_cat"]), dev(inp["B"]), pos)
        torch.cuda.synchronize()
        assert hcsa_get_device_status() == 0
        compare_step(spec, dict(inp, x=x_in), layer, cache, np.full(d.B, d.P), list(range(d.B)))
        out = host64(layer.out)
        layer.out_project(x, dev(inp["W_o"]))
        torch.cuda.synchronize()
        want = oracle.round_to(x_in + out @ oracle.to_f64(inp["W_o"]), oracle.ST_BF16)
        np.testing.assert_allclose(host64(x), want, rtol=2 ** -7, atol=2 ** -10)


@pytest.mark.parametrize("spec,pos,n_cap,lowprec", [
    (CSA_D, [515, 1023, 2000, 3, 7], 520, False),
    (CSA_TC, [515, 1023, 60], 300, False),
    (CSA_TC, [515, 1023, 60], 300, True),
    (HCA_D, [255, 1000, 383], 16, False),
    (HCA_TC, [255, 3000, 100, 127], 30, True),
    (CSA_TC, list(range(3, 3 + 4 * 20, 4)), 40, False),   # 20 sequences: the 32-token tile
    (CSA_D, list(range(3, 3 + 4 * 40, 4)), 50, False),    # 40 sequences: the two separate kernels
])
def test_fused_projection_append_matches_separate_calls(spec, pos, n_cap, lowprec):
    """hcsa_project_append (the append in the projection's epilogue) writes exactly what hcsa_project then
    hcsa_cache_append write: the projections, the rings and the closed entries."""
    import long_context_compressed_05_b200 as h
    d = synth.DecodeSpec(layers=(spec,), B=len(pos), P=max(pos), seed=spec.seed)
    inp = synth.decode_inputs(d, 0, n_cap=n_cap)
    B = len(pos)
    p = h.params_for(spec, T=0, B=B, n_cap=n_cap, lowprec=lowprec)
    kind = h.KIND_CSA if spec.kind == "csa" else h.KIND_HCA

    def fresh():
        c = {k: dev(inp[k]) for k in ("entries", "win_kv", "ring_g", "idx_keys", "ring_ki") if k in inp}
        if lowprec:
            rows = B * n_cap
            for key, what, nb in (("entries", h.STORE_ENTRIES, h.hcsa_entry_bytes(p, rows)),
                                  ("idx_keys", h.STORE_KEYS, h.hcsa_key_bytes(p, rows))):
                if key in c:
                    buf = torch.empty(nb, dtype=torch.uint8, device="cuda")
                    h.hcsa_quantize_rows(p, what, c[key].reshape(rows, -1), buf)
                    c[key] = buf
        return c

    x, W, Bb = dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"])
    pos_t = torch.tensor(pos, dtype=torch.int32, device="cuda")
    ncols = h.hcsa_proj_cols(p, kind)
    c1, c2 = fresh(), fresh()
    y1 = torch.empty((B, ncols), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty_like(y1)
    h.hcsa_project(p, kind, x, W, y1)   # no workspace: no split-K, the fused kernel's summation order
    C = spec.C
    h.hcsa_cache_append(p, h.make_cache(c1["entries"], c1["win_kv"], c1["ring_g"], c1.get("idx_keys"),
                                        c1.get("ring_ki")), pos_t, y1[:, :C], y1[:, C:2 * C],
                        y1[:, 2 * C:2 * C + spec.di] if spec.kind == "csa" else None, Bb)
    h.hcsa_project_append(p, kind, h.make_cache(c2["entries"], c2["win_kv"], c2["ring_g"], c2.get("idx_keys"),
                                                c2.get("ring_ki")), pos_t, x, W, Bb, y2)
    torch.cuda.synchronize()
    assert h.hcsa_get_device_status() == 0
    assert torch.equal(y1, y2)
    for k in c1:
        assert torch.equal(c1[k], c2[k]), k
