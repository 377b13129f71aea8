"""Input generator and golden-fixture checks (CPU only)."""
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
GOLD = os.path.join(HERE, "golden")


def test_splitmix64_published_outputs(syn):
    for line in open(os.path.join(GOLD, "splitmix64_state0.txt")):
        if line.startswith("#") or not line.strip():
            continue
        n, h = line.split()
        assert syn.splitmix64_nth(0, int(n)) == int(h, 16)


def test_normal_moments_and_counter_slices(syn):
    a = syn.normal(7, 3, (1 << 20,), 1.0, syn.KIND_F64)
    assert abs(a.mean()) < 5 / 1024 and abs(a.std() - 1) < 5 / 1024 * 1.5
    # kurtosis of a normal is 3
    assert abs(((a - a.mean()) ** 4).mean() / a.var() ** 2 - 3.0) < 0.05
    # any slice reproduces the same elements (counter based)
    b = syn.normal(7, 3, (1000,), 1.0, syn.KIND_F64, offset=4321)
    np.testing.assert_array_equal(b, a[4321:5321])
    # different tensor ids / seeds are different streams
    assert not np.array_equal(a[:100], syn.normal(7, 4, (100,), 1.0, syn.KIND_F64))
    assert not np.array_equal(a[:100], syn.normal(8, 3, (100,), 1.0, syn.KIND_F64))


def test_storage_formats_round_the_same_draws(syn):
    import torch
    a = syn.normal(1, 1, (5000,), 0.3, syn.KIND_F64)
    f = syn.normal(1, 1, (5000,), 0.3, syn.KIND_F32)
    np.testing.assert_array_equal(f, a.astype(np.float32))
    bf = syn.normal(1, 1, (5000,), 0.3, syn.KIND_BF16)
    # direct double -> bf16 RNE equals float32 -> bf16 whenever the float32 step is exact or far from a tie
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (bf == ref).mean() > 0.999
    assert np.array_equal(syn.round_bf16_bits(np.array([1.0, 1 + 2 ** -8, 1 + 3 * 2 ** -8, -2.5])),
                          np.array([0x3F80, 0x3F80, 0x3F82, 0xC020], np.uint16))


def test_compression_ratio_entry_counts(syn, orc):
    for line in open(os.path.join(GOLD, "compression_ratios.txt")):
        if line.startswith("#") or not line.strip():
            continue
        kind, m, T, n = line.split()
        m, T, n = int(m), int(T), int(n)
        spec = syn.LayerSpec(kind=kind, T=T, D=8, m=m, width=8 if kind == "csa" else m, C=2)
        assert spec.n_entries == n
        if T <= 4096:
            ent, _ = orc.compress(T, 2, m, spec.width, *([np.zeros((T, 2)).ctypes.data, 2] * 2),
                                  np.zeros((spec.width, 2)), None, 0, 0, 0)
            assert ent.shape[0] == n


def test_oracle_regression_snapshot(orc):
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(GOLD, "make_golden.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    got = mod.compute()
    ref = np.load(os.path.join(GOLD, "oracle_csa_tiny.npz"))
    for k in ref.files:
        np.testing.assert_array_equal(got[k], ref[k])


def test_v4_schedule_workload():
    """The residual-chained 1M-context workload: two HCA layers, then CSA and HCA alternating; every layer has
    its own output projection W_o ~ N(0, 1/(H dh)) drawn from a stream of its own."""
    import synth
    d = synth.DECODE["v4_decode_b4_p1048576"]
    assert d.residual and [s.kind for s in d.layers] == ["hca", "hca", "csa", "hca", "csa", "hca", "csa", "hca"]
    small = synth.DecodeSpec(layers=tuple(s.replace(D=64, C=32, H=2, dh=16, di=16, Hi=2, topk=8, window=8,
                                                    width=8 if s.kind == "csa" else 128) for s in d.layers[:3]),
                             B=2, P=300, seed=d.seed, residual=True)
    wo = [synth.decode_inputs(small, i, with_cache=False)["W_o"] for i in range(3)]
    from oracle import to_f64
    w0 = to_f64(wo[0])
    assert w0.shape == (32, 64)
    assert abs(w0.std() * (32 ** 0.5) - 1.0) < 0.1 and abs(w0.mean()) < 0.03
    assert not np.array_equal(wo[0], wo[1])          # per-layer streams
    plain = synth.DecodeSpec(layers=small.layers, B=2, P=300, seed=d.seed)
    assert "W_o" not in synth.decode_inputs(plain, 0, with_cache=False)
