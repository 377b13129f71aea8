"""GPU parity of the prefill path (projection, compressor, indexer + top-k, attention) against the
fp64 oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._helpers import check_out, check_selection, dev, host64, sample_rows

pytestmark = pytest.mark.gpu

CSA_SMALL = synth.LayerSpec(kind="csa", T=1003, D=256, m=4, width=8, C=256, di=64, Hi=8, topk=64, window=128, H=8,
                            dh=128, scale=128 ** -0.5, dtype="bf16", seed=21)
CSA_WIDE = synth.LayerSpec(kind="csa", T=700, D=512, m=4, width=8, C=1024, di=64, Hi=32, topk=128, window=128,
                           H=4, dh=512, scale=512 ** -0.5, dtype="bf16", seed=22)
HCA_SMALL = synth.LayerSpec(kind="hca", T=1500, D=256, m=128, width=128, C=256, window=128, H=4, dh=128,
                            scale=128 ** -0.5, dtype="bf16", seed=23)
HCA_F32 = HCA_SMALL.replace(dtype="f32", T=700, seed=24)
# the shapes of the tensor-core attention kernel (64 heads of 512, <= 640 keys), at small D and T
CSA_TC_K128 = synth.LayerSpec(kind="csa", T=900, D=256, m=4, width=8, C=1024, di=64, Hi=8, topk=128, window=128,
                              H=64, dh=512, scale=512 ** -0.5, dtype="bf16", seed=41)
CSA_TC_K512 = CSA_TC_K128.replace(T=2600, topk=512, seed=42)
# the same kernel over a dense entry list (64 heads of 512, pools of 8): units of 1 to 5 tiles as t grows
HCA_TC_DENSE = synth.LayerSpec(kind="hca", T=3500, D=128, m=8, width=8, C=1024, window=128, H=64, dh=512,
                               scale=512 ** -0.5, dtype="bf16", seed=46)

CASES = {
    "csa_f32_t2048": synth.PREFILL["csa_f32_t2048"],
    "csa_bf16_small": CSA_SMALL,
    "csa_bf16_wide": CSA_WIDE,
    "hca_bf16_small": HCA_SMALL,
    "hca_f32_small": HCA_F32,
    # edge cases: no visible entry at all, a ragged tail, fewer visible entries than k everywhere
    "csa_bf16_t3": CSA_SMALL.replace(T=3, seed=25),
    "csa_bf16_t1": CSA_SMALL.replace(T=1, seed=26),
    "csa_bf16_vis_lt_k": CSA_SMALL.replace(T=230, seed=27),
    "csa_f32_ragged": synth.PREFILL["csa_f32_t2048"].replace(T=517, seed=28),
    "hca_bf16_t100": HCA_SMALL.replace(T=100, seed=29),
    "csa_bf16_tc_k128": CSA_TC_K128,
    "csa_bf16_tc_k512": CSA_TC_K512,
    "csa_bf16_tc_t5": CSA_TC_K128.replace(T=5, seed=43),
    # units of 3 and 4 tiles (the window tile is the last one, outside the output accumulator's columns)
    "csa_bf16_tc_k256": CSA_TC_K128.replace(T=1400, topk=256, seed=44),
    "csa_bf16_tc_k384": CSA_TC_K128.replace(T=2000, topk=384, seed=45),
    "hca_bf16_tc_dense": HCA_TC_DENSE,
}
# query rows checked per case (default: all)
SAMPLED = {"csa_bf16_tc_k128": 48, "csa_bf16_tc_k512": 48, "csa_bf16_tc_k256": 48, "csa_bf16_tc_k384": 48,
           "hca_bf16_tc_dense": 64}


def run_gpu(spec):
    from long_context_compressed_05_b200 import PrefillLayer, hcsa_get_device_status
    inp = synth.prefill_inputs(spec)
    layer = PrefillLayer(spec)
    layer.forward(dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"]))
    torch.cuda.synchronize()
    assert hcsa_get_device_status() == 0
    return inp, layer


def compare(spec, inp, layer, rows, ref):
    f32 = spec.dtype == "f32"
    cols = layer.cols
    # projections (rounded storage): allow one storage ulp where accumulation order differs
    y = host64(layer.y[torch.from_numpy(rows).cuda()])
    pool_end = cols["ki"][1] if spec.kind == "csa" else cols["g"][1]
    ypool_ref = ref["y_pool"][rows]
    # fp32 accumulation error is absolute (~1e-6 for unit-scale terms); bf16 adds one storage ulp
    rt, at = (1e-6, 1e-6) if f32 else (2 ** -7, 1e-5)
    np.testing.assert_allclose(y[:, :pool_end], ypool_ref, rtol=rt, atol=at)
    np.testing.assert_allclose(y[:, pool_end:], ref["y_q"], rtol=rt, atol=at)
    # compressor, in isolation: the oracle pools the GPU's own projections; results may differ by one
    # rounding of the stored value (fp32 vs fp64 arithmetic before the final rounding)
    yg = host64(layer.y[:, :pool_end])
    base = yg.ctypes.data
    csa = spec.kind == "csa"
    ent_iso, idx_iso = oracle.compress(spec.T, spec.C, spec.m, spec.width, base, pool_end, base + 8 * spec.C,
                                       pool_end, oracle.to_f64(inp["B"]),
                                       base + 8 * cols["ki"][0] if csa else None, pool_end,
                                       spec.di if csa else 0, oracle.storage_code(spec.dtype))
    ent = host64(layer.entries)
    rt_iso = 1e-6 if f32 else 2 ** -7
    np.testing.assert_allclose(ent, ent_iso, rtol=rt_iso, atol=1e-6)
    # end to end against the oracle's own chain: a storage ulp of a unit-scale input may propagate
    rt, at = (1e-6, 1e-6) if f32 else (2 ** -6, 2 ** -5)
    np.testing.assert_allclose(ent, ref["entries"], rtol=rt, atol=at)
    if csa:
        np.testing.assert_allclose(host64(layer.idx_keys), idx_iso, rtol=rt_iso, atol=1e-6)
        np.testing.assert_allclose(host64(layer.idx_keys), ref["idx_keys"], rtol=rt, atol=at)
        sel = layer.sel.cpu().numpy()[rows]
        check_selection(sel, ref["sel"], ref["gap"], ref["scores"], ref["n_vis"], spec.topk, exact=f32,
                        label=f"{spec.kind} T={spec.T} k={spec.topk}")
        ref_out = oracle.attend_rows(spec, ref, ref["q"], sel)     # oracle on the GPU's own selection
    else:
        ref_out = ref["out"]
    out = host64(layer.out[torch.from_numpy(rows).cuda()])
    return check_out(out, ref_out, spec.dtype)


@pytest.mark.parametrize("name", list(CASES))
def test_prefill_parity(name):
    spec = CASES[name]
    inp, layer = run_gpu(spec)
    rows = np.arange(spec.T, dtype=np.int64)
    if name in SAMPLED:
        # dense layers: rows around the first change of tile count (t = 128 m) stand in for the top-k crossing
        rows = sample_rows(spec.T, spec.m, spec.topk or 128, n_random=SAMPLED[name], seed=spec.seed)
    ref = oracle.prefill(spec, inp, rows=rows)
    compare(spec, inp, layer, rows, ref)


def test_prefill_f32_sets_bit_exact_and_deterministic():
    spec = synth.PREFILL["csa_f32_t2048"]
    inp, layer = run_gpu(spec)
    sel1, out1 = layer.sel.clone(), layer.out.clone()
    layer.forward(dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"]))
    torch.cuda.synchronize()
    assert torch.equal(sel1, layer.sel) and torch.equal(out1, layer.out)
    ref = oracle.prefill(spec, inp)
    np.testing.assert_array_equal(layer.sel.cpu().numpy(), ref["sel"])


@pytest.mark.parametrize("name", ["hca_bf16_t65536", "csa_bf16_t131072"])
def test_prefill_full_size_sampled(name):
    """Full-size workloads in the benchmark's launch configuration; the oracle checks sampled query rows."""
    spec = synth.PREFILL[name]
    inp, layer = run_gpu(spec)
    rows = sample_rows(spec.T, spec.m, max(spec.topk, 1), n_random=24 if spec.kind == "csa" else 64)
    ref = oracle.prefill(spec, inp, rows=rows)
    compare(spec, inp, layer, rows, ref)


@pytest.mark.parametrize("name,lowprec", [("csa_bf16_small", False), ("csa_bf16_tc_k128", False),
                                          ("csa_bf16_tc_k128", True), ("csa_bf16_t3", False),
                                          ("csa_bf16_vis_lt_k", False), ("hca_bf16_small", False),
                                          ("csa_f32_ragged", False)])
def test_fused_projection_compressor_matches_separate_calls(name, lowprec):
    """hcsa_project_compress (the compressor in the projection's epilogue, seams after) writes exactly
    what hcsa_project then csa_compress / hca_compress write."""
    import long_context_compressed_05_b200 as h
    spec = CASES[name]
    for T in sorted({spec.T, 257, 640, 1023} if spec.T > 100 else {spec.T}):
        sp = spec.replace(T=T)
        inp = synth.prefill_inputs(sp)
        x, W, B = dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"])
        a, b = h.PrefillLayer(sp, lowprec=lowprec), h.PrefillLayer(sp, lowprec=lowprec)
        a.y.fill_(0)
        L = h
        L.hcsa_project(a.p, a.kind, x, W, a.y)                     # no workspace: no split-K
        a.compress(B)
        L.hcsa_project_compress(b.p, b.kind, x, W, B, b.y, b.entries, b.idx_keys if b.csa else None)
        torch.cuda.synchronize()
        assert h.hcsa_get_device_status() == 0
        assert torch.equal(a.y, b.y), T
        assert torch.equal(a.entries, b.entries), T
        if sp.kind == "csa":
            assert torch.equal(a.idx_keys, b.idx_keys), T


@pytest.mark.parametrize("name,chunks", [("csa_bf16_tc_k512", 3), ("csa_bf16_tc_t5", 8), ("hca_bf16_tc_dense", 5),
                                         ("csa_bf16_small", 7), ("hca_bf16_small", 8)])
def test_forward_host_matches_forward(name, chunks):
    """The host-buffer call (attention by row ranges, output rows copied back on a second stream) returns
    the device call's output; a second call, whose attention waits for the first call's copies, too.
    Per-token attention kernels are bit-exact by range; the HCA kernel for dh = 128 tiles the window from
    each query block's first token, so a range boundary inside a block may change rounding by an ulp."""
    spec = CASES[name]
    inp, layer = run_gpu(spec)
    ref = layer.out.detach().cpu().clone()
    W, B = dev(inp["W_cat"]), dev(inp["B"])
    xh = dev(inp["x"]).cpu().pin_memory()
    for _ in range(2):
        oh = torch.full(tuple(layer.out.shape), float("nan"), dtype=layer.out.dtype).pin_memory()
        layer.forward_host(xh, W, B, oh, chunks=chunks)
        layer.wait_host()
        torch.cuda.synchronize()
        if spec.kind == "hca" and spec.dh == 128:
            torch.testing.assert_close(oh.float(), ref.float(), rtol=2 ** -7, atol=2 ** -9)
        else:
            assert torch.equal(oh, ref)
