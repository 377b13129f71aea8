"""The algorithmic work counts behind the benchmark's roofline fractions, against closed forms worked out
by hand (integer sums over the causal visibility pattern and the decode byte budget)."""
import bench
import synth


def test_csa_prefill_work_closed_form():
    spec = synth.PREFILL["csa_bf16_t131072"]
    T, m, k, win = spec.T, spec.m, spec.topk, spec.window
    q = T // m
    # sum_t floor(t / 4) = 4 * sum_{j < T/4} j  (every entry index is visible to 4 consecutive tokens)
    pairs = 4 * q * (q - 1) // 2
    assert pairs == 2_147_418_112
    # selected keys: floor(t/4) until it reaches k (t < 4k), then k; window keys: t + 1 until 128
    sel = 4 * k * (k - 1) // 2 + k * (T - 4 * k)
    wins = win * (win + 1) // 2 + win * (T - win)
    assert sel + wins == 83_352_640
    w = bench.prefill_work(spec)
    assert w["csa_index_topk"]["flops"] == pairs * spec.Hi * spec.di * 2
    assert w["attend"]["flops"] == (sel + wins) * spec.H * spec.dh * 4
    assert w["hcsa_project"]["flops"] == 2 * T * spec.D * 36960


def test_hca_prefill_work_closed_form():
    spec = synth.PREFILL["hca_bf16_t65536"]
    T, m, win = spec.T, spec.m, spec.window
    q = T // m
    ent = m * q * (q - 1) // 2                      # sum_t floor(t / 128)
    wins = win * (win + 1) // 2 + win * (T - win)
    w = bench.prefill_work(spec)
    assert w["attend"]["flops"] == (ent + wins) * spec.H * spec.dh * 4


def test_decode_bytes_closed_form():
    d = synth.DECODE["csa_decode_b32_p262144"]
    spec = d.layers[0]
    weights = 2048 * 36960 * 2
    keys = 32 * 65536 * 64 * 2
    rows = 32 * (512 + 128) * 1024 * 2
    qo = 32 * 64 * 512 * 2 * 2
    assert bench.decode_bytes(spec, 32, 65536) == weights + keys + rows + qo == 465_960_960
    h = synth.DECODE["hybrid_decode_b4_p1048576"]
    total = 0
    for s in h.layers:
        N = h.n_cache_entries(s)
        if s.kind == "csa":
            total += 2048 * 36960 * 2 + 4 * N * 64 * 2 + 4 * (1024 + 128) * 1024 * 2
        else:
            total += 2048 * (2 * 1024 + 64 * 512) * 2 + 4 * (N + 128) * 1024 * 2
        total += 4 * 64 * 512 * 2 * 2
    assert sum(bench.decode_bytes(s, 4, h.n_cache_entries(s)) for s in h.layers) == total
    assert 2.0e9 < total < 2.1e9
