"""Row ranges of the host-buffer prefill call (PrefillLayer.forward_host).  The prefill calls take a row
range only when it starts on a 128-row boundary and ends on one or at T; the ranges must cover every row
once, in order, and there must be no more of them than asked for."""
import pytest

from long_context_compressed_05_b200.layer import row_ranges


@pytest.mark.parametrize("T", [0, 1, 5, 127, 128, 129, 1003, 2600, 65535, 65536, 131071, 131072])
@pytest.mark.parametrize("chunks", [0, 1, 3, 8, 1000])
def test_row_ranges_cover_in_order_and_align(T, chunks):
    r = row_ranges(T, chunks)
    if T == 0:
        assert r == []
        return
    assert 1 <= len(r) <= max(1, chunks)
    assert r[0][0] == 0 and r[-1][1] == T
    assert all(b == c for (_, b), (c, _) in zip(r, r[1:]))
    assert all(a % 128 == 0 and b > a and (b % 128 == 0 or b == T) for a, b in r)


def test_row_ranges_split_the_benchmark_sequence_evenly():
    assert row_ranges(131072, 8) == [(a, a + 16384) for a in range(0, 131072, 16384)]
