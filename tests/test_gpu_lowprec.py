"""GPU parity of the FP8-entry / FP4-indexer-key storage (section "FP8 y FP4" of the KV-cache page) against the
oracle's low-precision storage, through the C ABI.

The quantizers (compressor epilogue, cache append, hcsa_quantize_rows) must reproduce the oracle's
store_fp8_rows / store_fp4_rows bit for bit on the same bf16 values.  Every stored value is a bf16 number, so
the readers (tensor-core indexer over FP4 keys, tensor-core attention over FP8 entries) must then match the
oracle recomputed on the GPU's own stored cache under the same rules as the bf16 path."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._helpers import check_out, check_selection, dev, host64, sample_rows

pytestmark = pytest.mark.gpu

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])

CSA_TC = synth.LayerSpec(kind="csa", T=1500, D=256, m=4, width=8, C=1024, di=64, Hi=32, topk=128, window=128,
                         H=64, dh=512, scale=512 ** -0.5, dtype="bf16", seed=81)
CSA_SMALL = synth.LayerSpec(kind="csa", T=700, D=256, m=4, width=8, C=256, di=64, Hi=8, topk=64, window=128,
                            H=8, dh=128, scale=128 ** -0.5, dtype="bf16", seed=82)
HCA_SMALL = synth.LayerSpec(kind="hca", T=1100, D=256, m=128, width=128, C=256, window=128, H=4, dh=128,
                            scale=128 ** -0.5, dtype="bf16", seed=83)
CSA_DEC = synth.LayerSpec(kind="csa", T=0, D=256, m=4, width=8, C=1024, di=64, Hi=32, topk=128, window=128, H=64,
                          dh=512, scale=512 ** -0.5, dtype="bf16", seed=84)
HCA_DEC = synth.LayerSpec(kind="hca", T=0, D=256, m=128, width=128, C=1024, window=128, H=64, dh=512,
                          scale=512 ** -0.5, dtype="bf16", seed=85)


def decode_fp8(buf, rows, ch):
    """Host decode of an FP8 byte array (codes [rows, ch], then int8 exponents [rows, ch / 32])."""
    b = buf.detach().cpu()
    codes = b[:rows * ch].view(torch.float8_e4m3fn).to(torch.float64).numpy().reshape(rows, ch)
    e = b[rows * ch:rows * ch + rows * ch // 32].view(torch.int8).numpy().astype(np.int64).reshape(rows, ch // 32)
    return codes * np.ldexp(1.0, np.repeat(e, 32, axis=1)), e


def decode_fp4(buf, rows, ch):
    """Host decode of an FP4 byte array (code pairs [rows, ch / 2], low nibble first; then exponents)."""
    b = buf.detach().cpu().numpy()
    pairs = b[:rows * ch // 2].reshape(rows, ch // 2)
    codes = np.empty((rows, ch), np.int64)
    codes[:, 0::2] = pairs & 15
    codes[:, 1::2] = pairs >> 4
    e = b[rows * ch // 2:rows * ch // 2 + rows * ch // 32].view(np.int8).astype(np.int64).reshape(rows, ch // 32)
    return E2M1[codes] * np.ldexp(1.0, np.repeat(e, 32, axis=1)), e


def test_quantize_rows_matches_oracle_storage():
    import long_context_compressed_05_b200 as h
    g = torch.Generator().manual_seed(7)
    R = 300
    ent = torch.randn(R, 1024, generator=g, dtype=torch.float64) * torch.exp(torch.empty(R, 1).uniform_(-6, 6, generator=g))
    ent[3, 64:96] = 0.0                                   # an all-zero block
    ent[4] = 0.0                                          # an all-zero row
    keys = torch.randn(R, 64, generator=g, dtype=torch.float64) * torch.exp(torch.empty(R, 1).uniform_(-4, 4, generator=g))
    ent_b, keys_b = ent.to(torch.bfloat16), keys.to(torch.bfloat16)
    p = h.params_for(CSA_DEC, lowprec=True)
    e_buf = torch.empty(h.hcsa_entry_bytes(p, R), dtype=torch.uint8, device="cuda")
    k_buf = torch.empty(h.hcsa_key_bytes(p, R), dtype=torch.uint8, device="cuda")
    h.hcsa_quantize_rows(p, h.STORE_ENTRIES, ent_b.cuda(), e_buf)
    h.hcsa_quantize_rows(p, h.STORE_KEYS, keys_b.cuda(), k_buf)
    torch.cuda.synchronize()
    got, ge = decode_fp8(e_buf, R, 1024)
    want, we = oracle.store_fp8_rows(ent_b.to(torch.float64).numpy(), 32)
    np.testing.assert_array_equal(got, want)
    nz = np.abs(ent_b.to(torch.float64).numpy()).reshape(R, 32, 32).max(axis=2) > 0
    np.testing.assert_array_equal(ge[nz], we[nz])
    got, ge = decode_fp4(k_buf, R, 64)
    want, we = oracle.store_fp4_rows(keys_b.to(torch.float64).numpy(), 32)
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(ge, we)


def test_quantize_rows_refuses_bad_requests():
    import long_context_compressed_05_b200 as h
    p16 = h.params_for(CSA_DEC)                           # lowprec off
    src = torch.zeros(4, 1024, dtype=torch.bfloat16, device="cuda")
    dst = torch.empty(8192, dtype=torch.uint8, device="cuda")
    with pytest.raises(h.HcsaError) as e:
        h.hcsa_quantize_rows(p16, h.STORE_ENTRIES, src, dst)
    assert e.value.code == 8
    p = h.params_for(CSA_DEC, lowprec=True)
    with pytest.raises(h.HcsaError) as e:
        h.hcsa_quantize_rows(p, 7, src, dst)
    assert e.value.code == 2


@pytest.mark.parametrize("spec", [CSA_SMALL, HCA_SMALL, CSA_TC], ids=["csa_small", "hca_small", "csa_tc"])
def test_compressor_stores_the_bf16_entries_in_fp8_fp4(spec):
    """The compressor's FP8 / FP4 output is the oracle's storage of the entries the bf16 path writes."""
    from long_context_compressed_05_b200 import PrefillLayer
    inp = synth.prefill_inputs(spec)
    x, W, B = dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"])
    ref16 = PrefillLayer(spec)
    ref16.project(x, W)
    ref16.compress(B)
    low = PrefillLayer(spec, lowprec=True)
    low.project(x, W)
    low.compress(B)
    torch.cuda.synchronize()
    N = ref16.entries.shape[0]
    got, _ = decode_fp8(low.entries, N, spec.C)
    np.testing.assert_array_equal(got, oracle.store_fp8_rows(host64(ref16.entries), 32)[0])
    if spec.kind == "csa":
        got, _ = decode_fp4(low.idx_keys, N, spec.di)
        np.testing.assert_array_equal(got, oracle.store_fp4_rows(host64(ref16.idx_keys), 32)[0])


@pytest.mark.parametrize("spec,n_sample", [(CSA_TC, 64), (CSA_TC.replace(T=700, topk=512, seed=86), 48),
                                           (CSA_TC.replace(T=5, seed=87), 0)],
                         ids=["k128", "k512", "t5"])
def test_prefill_csa_lowprec(spec, n_sample):
    """Indexer over FP4 keys and attention over FP8 entries, against the oracle on the GPU's stored cache."""
    from long_context_compressed_05_b200 import PrefillLayer, hcsa_get_device_status
    inp = synth.prefill_inputs(spec)
    layer = PrefillLayer(spec, lowprec=True)
    layer.forward(dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"]))
    torch.cuda.synchronize()
    assert hcsa_get_device_status() == 0
    rows = np.arange(spec.T) if not n_sample else sample_rows(spec.T, spec.m, spec.topk, n_random=n_sample,
                                                              seed=spec.seed)
    N = -(-spec.T // spec.m)
    ent_gpu, _ = decode_fp8(layer.entries, N, spec.C)
    key_gpu, _ = decode_fp4(layer.idx_keys, N, spec.di)
    full = oracle.prefill_entries(spec, inp, lowprec=True)
    # end to end: the oracle's own FP8 / FP4 cache differs only where a bf16 entry differed by an ulp
    assert np.mean(ent_gpu != full["entries"]) < 1e-2 and np.mean(key_gpu != full["idx_keys"]) < 1e-2
    ref = oracle.prefill_queries(spec, inp, dict(full, entries=ent_gpu, idx_keys=key_gpu), rows=rows)
    sel = layer.sel.cpu().numpy()[rows]
    check_selection(sel, ref["sel"], ref["gap"], ref["scores"], ref["n_vis"], spec.topk, exact=False,
                    label=f"lowprec T={spec.T} k={spec.topk}")
    ref_out = oracle.attend_rows(spec, ref, ref["q"], sel)
    check_out(host64(layer.out[torch.from_numpy(rows).cuda()]), ref_out, "bf16")


def _lowprec_cache(spec, inp, p):
    import long_context_compressed_05_b200 as h
    cache = {k: dev(inp[k]) for k in ("win_kv", "ring_g", "ring_ki") if k in inp}
    ent = dev(inp["entries"])
    rows = ent.shape[0] * ent.shape[1]
    cache["entries"] = torch.empty(h.hcsa_entry_bytes(p, rows), dtype=torch.uint8, device="cuda")
    h.hcsa_quantize_rows(p, h.STORE_ENTRIES, ent.reshape(rows, -1), cache["entries"])
    if spec.kind == "csa":
        keys = dev(inp["idx_keys"])
        cache["idx_keys"] = torch.empty(h.hcsa_key_bytes(p, rows), dtype=torch.uint8, device="cuda")
        h.hcsa_quantize_rows(p, h.STORE_KEYS, keys.reshape(rows, -1), cache["idx_keys"])
    return cache


@pytest.mark.parametrize("spec,pos,n_cap", [
    (CSA_DEC, [515, 1023, 60], 300),      # 515 closes an entry; P = 60: fewer visible than k
    (CSA_DEC, [40003, 39999, 20000], 10001),
    (HCA_DEC, [255, 3000, 100], 30),      # 255 closes entry 1; 100: window only
    (HCA_DEC, [70000, 65535, 4000], 600),
])
def test_decode_lowprec(spec, pos, n_cap):
    from long_context_compressed_05_b200 import DecodeLayer, hcsa_get_device_status, params_for
    d = synth.DecodeSpec(layers=(spec,), B=len(pos), P=max(pos), seed=spec.seed)
    inp = synth.decode_inputs(d, 0, n_cap=n_cap)
    B = len(pos)
    p = params_for(spec, T=0, B=B, n_cap=n_cap, lowprec=True)
    cache = _lowprec_cache(spec, inp, p)
    layer = DecodeLayer(spec, B, n_cap, cache, lowprec=True)
    pos_t = torch.tensor(pos, dtype=torch.int32, device="cuda")
    layer.step(dev(inp["x"]), dev(inp["W_cat"]), dev(inp["B"]), pos_t)
    torch.cuda.synchronize()
    assert hcsa_get_device_status() == 0
    ref = oracle.decode_step(spec, inp, np.array(pos), lowprec=True)
    ent_gpu, _ = decode_fp8(cache["entries"], B * n_cap, spec.C)
    ent_gpu = ent_gpu.reshape(B, n_cap, spec.C)
    for b in range(B):
        ne = ref["new_entry"][b]
        if ne is not None and ne["j"] < n_cap:
            # the appended entry: the same FP8 storage, up to one code step where its bf16 value differed by an ulp
            amax = np.abs(ne["entry"]).max()
            np.testing.assert_allclose(ent_gpu[b, ne["j"]], ne["entry"], rtol=2 ** -3, atol=amax * 2.0 ** -12)
        if spec.kind == "csa":
            sel = layer.sel[b].cpu().numpy()[None]
            nv = np.array([min(pos[b] // spec.m, n_cap)])
            check_selection(sel, ref["sel"][b:b + 1], ref["gap"][b:b + 1], ref["scores"][b][None], nv, spec.topk,
                            exact=False)
            ref_out = oracle.decode_attend_with_sel(spec, ref, b, sel[0])
        else:
            ref_out = ref["out"][b]
        check_out(host64(layer.out[b]), ref_out, "bf16")


def test_lowprec_unsupported_paths_refuse():
    from long_context_compressed_05_b200 import HcsaError, PrefillLayer
    spec = HCA_SMALL
    inp = synth.prefill_inputs(spec)
    layer = PrefillLayer(spec, lowprec=True)
    layer.project(dev(inp["x"]), dev(inp["W_cat"]))
    layer.compress(dev(inp["B"]))
    with pytest.raises(HcsaError) as e:
        layer.attend()
    assert e.value.code == 8
