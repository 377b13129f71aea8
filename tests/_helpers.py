"""Shared helpers for the GPU parity tests: host <-> device marshalling and the comparison rules.

Comparison rules (the parity contract of the layer):
  fp32 storage : top-k index sets bit-exact; outputs within 1e-4 max-abs of the oracle.
  bf16 storage : index sets equal except where the oracle's k-th vs (k+1)-th score gap is below
                 1e-3 relative.  Every row with more visible entries than k must also be a valid
                 top-k up to eps = 1e-3 |s_(k)|: each selected entry scores >= s_(k) - eps and each
                 visible entry left out scores <= s_(k+1) + eps (s_(i) = the i-th best oracle score).
                 The output must match the oracle recomputed on the GPU's own selection to 2e-2
                 max-abs and 2e-3 mean-abs.
"""
import numpy as np
import torch

from long_context_compressed_05_b200.host import to_device as dev  # noqa: F401  (re-exported for the tests)

GAP_REL = 1e-3
BF16_MAX_ABS, BF16_MEAN_ABS = 2e-2, 2e-3
F32_MAX_ABS = 1e-4


def host64(t):
    return t.detach().float().cpu().numpy().astype(np.float64) if t.dtype == torch.bfloat16 else \
        t.detach().double().cpu().numpy()


def sample_rows(T, m, k, n_random=32, seed=0):
    r = np.random.default_rng(seed)
    rows = set(range(min(T, 16)))
    thr = m * k                                   # visible count crosses k here
    rows |= {t for t in range(max(0, thr - 40), min(T, thr + 40)) if t % m == m - 1}
    rows |= set(range(max(0, T - 8), T))
    rows |= set(int(x) for x in r.integers(0, T, n_random)) if T else set()
    return np.array(sorted(x for x in rows if 0 <= x < T), np.int64)


def check_selection(gpu_sel, ref_sel, gap, scores, n_vis, k, exact, label=""):
    """gpu_sel/ref_sel [nq, k]; scores [nq, N] oracle float64.

    Rows whose oracle gap is at least GAP_REL (and every row when `exact`) must equal the oracle's set.
    Every row with more visible entries than k must in addition be a valid top-k within eps of the
    oracle's order statistics, on both sides (selected >= s_(k) - eps, left out <= s_(k+1) + eps).
    Returns the number of waived rows (printed with `label` when given)."""
    waived = 0
    for q in range(gpu_sel.shape[0]):
        n = int(n_vis[q])
        take = min(k, n)
        g = gpu_sel[q]
        assert (g[take:] == -1).all(), f"row {q}: padding"
        gs = g[:take]
        assert (gs >= 0).all() and (gs < max(n, 1)).all(), f"row {q}: index out of the visible range"
        assert (np.diff(gs) > 0).all(), f"row {q}: not strictly ascending"
        if exact or n <= k or gap[q] >= GAP_REL:
            np.testing.assert_array_equal(gs, ref_sel[q, :take], err_msg=f"row {q} (n_vis {n}, gap {gap[q]})")
        else:
            waived += 1
        if n > k:
            s = scores[q, :n]
            srt = np.sort(s)[::-1]
            kth, k1th = srt[k - 1], srt[k]
            eps = GAP_REL * abs(kth)
            assert (s[gs] >= kth - eps).all(), f"row {q}: selected an entry far below the k-th score"
            left = np.ones(n, bool)
            left[gs] = False
            assert (s[left] <= k1th + eps).all(), f"row {q}: left out an entry far above the (k+1)-th score"
    if label:
        print(f"{label}: {waived} of {gpu_sel.shape[0]} rows under the gap waiver")
    return waived


def check_out(gpu, ref, dtype):
    d = np.abs(gpu - ref)
    if dtype == "f32":
        assert d.max() <= F32_MAX_ABS, f"max-abs {d.max()}"
    else:
        assert d.max() <= BF16_MAX_ABS, f"max-abs {d.max()}"
        assert d.mean() <= BF16_MEAN_ABS, f"mean-abs {d.mean()}"
    return float(d.max()), float(d.mean())
