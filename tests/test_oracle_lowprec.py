"""Pins of the oracle's low-precision cache storage (FP8 E4M3 entries, FP4 E2M1 indexer keys; readings in
the oracle's header): the element rounding against independent references (torch's float8_e4m3fn cast; a
brute-force search over the E2M1 grid with the even-mantissa tie rule) and the block-scaling invariants."""
import numpy as np
import pytest
import torch

import oracle

E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_ODD = np.array([0, 1, 0, 1, 0, 1, 0, 1])   # mantissa bit of each grid value


def e2m1_brute(v):
    a = abs(v)
    if a >= 6.0:
        q = 6.0
    else:
        d = np.abs(E2M1_GRID - a)
        best = np.flatnonzero(d == d.min())
        q = E2M1_GRID[best[0]] if len(best) == 1 else E2M1_GRID[best[E2M1_ODD[best] == 0][0]]
    return -q if v < 0 else q


def test_e4m3_rounding_matches_torch_cast():
    rng = np.random.default_rng(1)
    # every E4M3 value, every midpoint between neighbours (ties), and random values, all exact in fp32
    codes = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    grid = np.unique(codes[np.isfinite(codes)])
    mids = (grid[:-1] + grid[1:]) / 2
    rnd = np.concatenate([rng.uniform(-448, 448, 4000), rng.standard_normal(4000) * 0.01,
                          rng.standard_normal(4000) * 2.0 ** -8])
    v = np.concatenate([grid, mids, rnd]).astype(np.float32)
    v = v[np.abs(v) <= 448]
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.round_e4m3(v.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_e4m3_known_values_and_saturation():
    got = oracle.round_e4m3(np.array([448.0, 500.0, -1e6, 2.0 ** -9, 2.0 ** -10, 1 + 1 / 16, 1 + 3 / 16, 0.0]))
    np.testing.assert_array_equal(got, [448.0, 448.0, -448.0, 2.0 ** -9, 0.0, 1.0, 1.25, 0.0])


def test_e2m1_rounding_matches_brute_force():
    rng = np.random.default_rng(2)
    v = np.concatenate([np.arange(-8 * 64, 8 * 64 + 1) / 64.0, rng.uniform(-7, 7, 3000)])
    got = oracle.round_e2m1(v)
    want = np.array([e2m1_brute(x) for x in v])
    np.testing.assert_array_equal(got, want)


def test_fp8_block_storage_invariants():
    rng = np.random.default_rng(3)
    a = rng.standard_normal((64, 1024)) * np.exp(rng.uniform(-6, 6, (64, 1)))   # rows of very different scales
    a[5, :32] = 0.0                                                              # an all-zero block
    q, e = oracle.store_fp8_rows(a, 32)
    blocks = a.reshape(64, 32, 32)
    amax = np.abs(blocks).max(axis=2)
    scale = np.ldexp(1.0, e)
    nz = amax > 0
    r = amax[nz] / scale[nz]
    assert np.all(r <= 448.0) and np.all(r > 224.0)     # the smallest power of two that clips nothing
    assert np.all(e[~nz] == 0)
    codes = q.reshape(64, 32, 32) / scale[..., None]
    # every stored value is 2^e x (an E4M3 value): exact in the E4M3 grid (the rounding itself is pinned
    # against torch's cast above), and the nearest one to x / 2^e (checked against torch on fp32-exact inputs)
    np.testing.assert_array_equal(oracle.round_e4m3(codes.ravel()).reshape(codes.shape), codes)
    assert np.all(q.reshape(64, 32, 32)[5, 0] == 0.0)
    # error: half a unit in the last place of E4M3 (3 mantissa bits) in the normal range
    with np.errstate(invalid="ignore", divide="ignore"):
        rel = np.abs(codes * scale[..., None] - blocks) / np.maximum(np.abs(blocks), 2.0 ** -6 * scale[..., None])
    assert np.nanmax(rel[nz]) <= 2.0 ** -4 + 1e-12
    # a stored value is a bf16 number (4 significant bits times a power of two)
    q32 = torch.from_numpy(q).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(q32, q)


def test_fp8_block_rounding_against_torch_on_exact_inputs():
    rng = np.random.default_rng(6)
    # bf16 inputs (the storage type the entries arrive in): x / 2^e is exact in fp32, so torch's cast is an
    # independent reference for the element rounding of a whole block
    a = torch.from_numpy(rng.standard_normal((16, 256)) * 3.0).to(torch.bfloat16).to(torch.float64).numpy()
    q, e = oracle.store_fp8_rows(a, 32)
    scale = np.repeat(np.ldexp(1.0, e), 32, axis=1)
    want = torch.from_numpy((a / scale).astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(q / scale, want)


def test_fp4_block_storage_invariants():
    rng = np.random.default_rng(4)
    a = rng.standard_normal((32, 64)) * np.exp(rng.uniform(-4, 4, (32, 1)))
    q, e = oracle.store_fp4_rows(a, 32)
    blocks = a.reshape(32, 2, 32)
    amax = np.abs(blocks).max(axis=2)
    scale = np.ldexp(1.0, e)
    r = amax / scale
    assert np.all(r <= 6.0) and np.all(r > 3.0)          # the smallest power of two that clips nothing
    codes = q.reshape(32, 2, 32) / scale[..., None]
    np.testing.assert_array_equal(oracle.round_e2m1(codes.ravel()).reshape(codes.shape), codes)
    np.testing.assert_array_equal(codes, np.vectorize(e2m1_brute)(blocks / scale[..., None]))


def test_lowprec_prefill_reads_the_stored_entries():
    import synth
    spec = synth.LayerSpec(kind="csa", T=200, D=64, m=4, width=8, C=128, di=64, Hi=4, topk=16, window=16, H=2,
                           dh=64, scale=64 ** -0.5, dtype="bf16", seed=5)
    inp = synth.prefill_inputs(spec)
    ref = oracle.prefill(spec, inp)
    low = oracle.prefill(spec, inp, lowprec=True)
    np.testing.assert_array_equal(low["entries"], oracle.store_fp8_rows(ref["entries"], 32)[0])
    np.testing.assert_array_equal(low["idx_keys"], oracle.store_fp4_rows(ref["idx_keys"], 32)[0])
    assert not np.array_equal(low["out"], ref["out"])
