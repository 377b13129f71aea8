"""The prefill indexer + top-k on score patterns that random data rarely produces, through the C ABI,
against the oracle's top-k (a stable sort on (-score, j)).

The indexer keys, queries and head weights are chosen so that every score is a bf16 value computed exactly
in fp32 (one head, one channel: s[t, j] = 1 * ReLU(1 * key_j), key_j >= 1), and the selections must
therefore be bit-exact:
  * scores that grow with j: the k best are the last visible entries of every row;
  * plateaus of equal scores that grow with j: the threshold cuts through a run of ties, which must go to
    the lowest j;
  * a permuted pattern with many ties: about N / 101 keys share each value, so the threshold bucket holds
    hundreds of equal keys.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests._helpers import dev

pytestmark = pytest.mark.gpu


def _bf16_bits(a):
    return (torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
            .view(np.uint16))


def _run(pattern, T, Hi, topk):
    import long_context_compressed_05_b200 as h
    di, m = 64, 4
    N = -(-T // m)
    j = np.arange(N)
    # bf16 bit patterns of channel 0 of every key, from 1.0 upward (every value is exact)
    if pattern == "strict":
        bits = 0x3F80 + j                  # strictly increasing with j
    elif pattern == "increasing":
        bits = 0x3F80 + j // 16            # runs of 16 equal scores, increasing
    else:
        bits = 0x3F80 + (j * 37) % 101     # 101 distinct values, permuted, ~N/101 ties each
    bits = bits.astype(np.uint16)
    spec = synth.LayerSpec(kind="csa", T=T, D=64, m=m, width=8, C=128, di=di, Hi=Hi, topk=topk, window=128, H=1,
                           dh=64, scale=0.1, dtype="bf16", seed=0)
    p = h.params_for(spec)
    keys = np.zeros((N, di), np.uint16)
    keys[:, 0] = bits
    qi = np.zeros((T, Hi * di), np.float32)
    qi[:, 0] = 1.0                              # head 0, channel 0
    w = np.zeros((T, Hi), np.float32)
    w[:, 0] = 1.0
    sel = torch.full((T, topk), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(h.hcsa_workspace_bytes(p, h.OP_CSA_INDEX_TOPK), dtype=torch.uint8, device="cuda")
    h.csa_index_topk(p, dev(_bf16_bits(qi)), dev(_bf16_bits(w)), dev(keys), sel, ws)
    torch.cuda.synchronize()
    assert h.hcsa_get_device_status() == 0
    scores_row = synth.bf16_bits_to_f64(bits)
    return sel.cpu().numpy(), scores_row, N, m


@pytest.mark.parametrize("pattern", ["strict", "increasing", "permuted"])
@pytest.mark.parametrize("Hi,topk", [(8, 64), (32, 512)])
def test_fused_topk_exact_on_adversarial_scores(pattern, Hi, topk):
    T = 16000 if Hi == 8 else 40000
    sel, srow, N, m = _run(pattern, T, Hi, topk)
    r = np.random.default_rng(3)
    rows = np.unique(np.concatenate([np.arange(0, 40), np.arange(T - 40, T), r.integers(0, T, 200),
                                     np.arange(m * topk - 8, m * topk + 8)]))
    rows = rows[(rows >= 0) & (rows < T)]
    nv = np.minimum(rows // m, N)
    scores = np.broadcast_to(srow, (len(rows), N)).copy()
    want, _, _ = oracle.topk(scores, nv, topk)
    np.testing.assert_array_equal(sel[rows], want)
