"""Host-side logic of the binding that runs without a GPU."""
import pytest

from gated_delta_rule_86_b200.ops import segment_bounds


@pytest.mark.parametrize("T", [1, 63, 64, 65, 1000, 4096, 65536, 70690])
@pytest.mark.parametrize("segments", [1, 2, 7, 8, 16, 64])
@pytest.mark.parametrize("chunk", [16, 32, 64])
def test_segment_bounds_cover_at_chunk_starts(T, segments, chunk):
    b = segment_bounds(T, segments, chunk)
    assert 1 <= len(b) <= segments
    assert b[0][0] == 0 and b[-1][1] == T
    for (a0, a1), (b0, _) in zip(b, b[1:]):
        assert a1 == b0   # contiguous, no overlap
    for a, e in b:
        assert a % chunk == 0 and a < e   # every segment starts on a chunk boundary and is not empty


def test_segment_bounds_empty():
    assert segment_bounds(0, 8, 64) == []
