"""GPU parity of the projection GEMM (tcgen05, through the C ABI) against the fp64 oracle's projection:
hcsa_project (y = x W_cat) over ragged shapes -- token counts that are not multiples of a tile, a
contraction that is not a multiple of 64, column counts whose last tile is partly or half empty -- and
hcsa_out_project (x += out W_o, one rounding) on both of its paths: a decode batch, where the long
contraction is split over CTAs and the last CTA of a tile reduces the partials, and many rows, where
every tile is one CTA.  Tolerance: one bf16 storage ulp of the rounded value (the oracle rounds the fp64
product once; the kernel rounds its fp32 accumulation once) plus the fp32 accumulation error, bounded per
element by 2^-20 (16 fp32 ulps) times the L1 mass sum_k |x_k W_kn| of its terms: the tensor cores add
each K = 16 slice into the fp32 accumulator, and over a contraction of 32768 that error reaches a few
1e-5 on unit-scale sums, which matters where the sum cancels to near zero."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._helpers import dev, host64

pytestmark = pytest.mark.gpu

RTOL = 2 ** -7


def _atol(x64, W64, res64=None):
    mass = np.abs(x64) @ np.abs(W64)
    if res64 is not None:
        mass = mass + np.abs(res64)
    return 2.0 ** -20 * mass + 1e-7


def _check(got, want, atol):
    err = np.abs(got - want)
    bad = err > RTOL * np.abs(want) + atol
    assert not bad.any(), f"{bad.sum()} elements out of tolerance, worst {err[bad].max()}"


def _params(h, C, H, D, T=0, B=1):
    spec = synth.LayerSpec(kind="hca", T=T, D=D, m=128, width=128, C=C, window=128, H=H, dh=C // 2,
                           scale=1.0, dtype="bf16", seed=0)
    return h.params_for(spec, T=T, B=B)


def _bf16(seed, tid, shape, std):
    return synth.normal(seed, tid, shape, std, synth.KIND_BF16)


@pytest.mark.parametrize("rows,D,C,H", [
    (1, 256, 16, 1),        # 40 columns: one tile, its second half empty
    (5, 200, 64, 2),        # K = 200 (not a multiple of 64), 192 columns: the last tile exactly half full
    (16, 256, 256, 8),
    (17, 512, 256, 8),
    (33, 256, 1024, 64),    # 34816 columns, decode-sized token count
    (100, 256, 256, 8),
    (257, 2048, 256, 8),    # two token tiles of 256, the second with one row
    (1003, 256, 1024, 4),
])
def test_project_matches_oracle(rows, D, C, H):
    import long_context_compressed_05_b200 as h
    p = _params(h, C, H, D, T=rows)
    nc = h.hcsa_proj_cols(p, h.KIND_HCA)
    x = _bf16(7, 1, (rows, D), 1.0)
    W = _bf16(7, 2, (D, nc), D ** -0.5)
    y = torch.full((rows, nc), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(h.hcsa_workspace_bytes(p, h.OP_PROJECT), dtype=torch.uint8, device="cuda")
    h.hcsa_project(p, h.KIND_HCA, dev(x), dev(W), y, ws)
    torch.cuda.synchronize()
    assert h.hcsa_get_device_status() == 0
    x64, W64 = oracle.to_f64(x), oracle.to_f64(W)
    want = oracle.project(x64, W64, oracle.ST_BF16)
    _check(host64(y), want, _atol(x64, W64))


@pytest.mark.parametrize("rows,T,HD,D", [
    (4, 0, 32768, 2048),     # decode batch at the benchmark's shapes: split-K with the last-CTA reduction
    (32, 0, 4096, 512),
    (300, 300, 1024, 512),   # many rows: one CTA per tile, residual added in the epilogue
])
def test_out_project_matches_oracle_and_is_deterministic(rows, T, HD, D):
    import long_context_compressed_05_b200 as h
    C = 2 * (HD // 64) if HD >= 64 else 16
    H = HD // (C // 2)
    p = _params(h, C, H, D, T=T, B=rows if T == 0 else 1)
    out = _bf16(8, 1, (rows, HD), 1.0)
    Wo = _bf16(8, 2, (HD, D), HD ** -0.5)
    x0 = _bf16(8, 3, (rows, D), 1.0)
    ws = torch.empty(h.hcsa_workspace_bytes(p, h.OP_PROJECT), dtype=torch.uint8, device="cuda")
    o64, W64, x64 = oracle.to_f64(out), oracle.to_f64(Wo), oracle.to_f64(x0)
    want = oracle.round_to(x64 + o64 @ W64, oracle.ST_BF16)
    atol = _atol(o64, W64, x64)
    got = []
    for _ in range(2):
        x = dev(x0)
        h.hcsa_out_project(p, dev(out), dev(Wo), x, ws)
        torch.cuda.synchronize()
        assert h.hcsa_get_device_status() == 0
        got.append(x.clone())
    _check(host64(got[0]), want, atol)
    assert torch.equal(got[0], got[1])
    # without a workspace the same result comes from one CTA per tile (no split)
    x = dev(x0)
    h.hcsa_out_project(p, dev(out), dev(Wo), x, None)
    torch.cuda.synchronize()
    _check(host64(x), want, atol)


def test_out_project_refuses_more_rows_than_the_batch():
    import long_context_compressed_05_b200 as h
    p = _params(h, 256, 8, 512, T=0, B=2)
    out = torch.zeros((3, 1024), dtype=torch.bfloat16, device="cuda")
    Wo = torch.zeros((1024, 512), dtype=torch.bfloat16, device="cuda")
    x = torch.zeros((3, 512), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(h.HcsaError) as e:
        h.hcsa_out_project(p, out, Wo, x)
    assert e.value.code == 2
