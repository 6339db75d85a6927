"""StreamedScan's copy groups (host logic, CPU): every (row, token) covered exactly once, in order,
segments on chunk boundaries except the last of a row."""
import numpy as np
import pytest

from int8_quant_b200.runner import plan_groups


@pytest.mark.parametrize("batch,L,chunk,rows,seg", [
    (3, 1000, 256, 1, None), (3, 1000, 256, 2, None), (3, 1000, 256, 1, 512), (2, 333, 64, 1, 128),
    (1, 256, 64, 1, 256), (2, 0, 64, 1, None), (4, 8192, 256, 1, 1024),
])
def test_groups_cover_every_token_once(batch, L, chunk, rows, seg):
    groups, s = plan_groups(batch, L, chunk, rows, seg)
    seen = np.zeros((batch, max(L, 1)), dtype=int)
    for r0, n, t0, ln in groups:
        assert 1 <= n <= rows and 0 <= ln <= s
        seen[r0:r0 + n, t0:t0 + ln] += 1
        if t0 + ln < L:                                  # not a row's last segment: whole chunks
            assert ln % chunk == 0 and ln == s
    assert (seen[:, :L] == 1).all()
    # a row's segments are consecutive and in token order
    by_row = {}
    for r0, n, t0, ln in groups:
        by_row.setdefault(r0, []).append((t0, ln))
    for segs in by_row.values():
        ends = [t0 + ln for t0, ln in segs]
        assert [t0 for t0, _ in segs] == [0] + ends[:-1]


def test_segments_need_whole_chunks_and_single_rows():
    with pytest.raises(AssertionError):
        plan_groups(2, 1000, 256, 1, 300)
    with pytest.raises(AssertionError):
        plan_groups(2, 1000, 256, 2, 512)
