"""The row segments of the host-buffer prefill (polar_attn_fwd_host), as the
library computes them: host logic only, checked on a machine without a GPU.
Every row is covered exactly once, from the last rows to the first, on 128-row
query-tile boundaries, the last segment to go is the lightest (at most 1024
rows), and short sequences go in one segment."""
import os

import pytest

from polar_attention_b200 import native


@pytest.fixture(scope="module")
def segments():
    if not os.path.exists(native.LIB_PATH):
        pytest.skip("library not built")
    return native.fwd_host_segments


@pytest.mark.parametrize("T", [1, 127, 128, 300, 1024, 2047, 2048, 2049, 4500, 8192, 16384,
                               16385, 65536, 131072, 262144])
def test_cover_every_row_once_last_rows_first(segments, T):
    seg = segments(T)
    assert len(seg) >= 1
    assert seg[0][1] == T and seg[-1][0] == 0
    for i, (lo, hi) in enumerate(seg):
        assert 0 <= lo < hi <= T
        assert lo % 128 == 0
        if i + 1 < len(seg):
            assert seg[i + 1][1] == lo          # contiguous, descending
    if T < 2048:
        assert len(seg) == 1
    else:
        assert seg[-1][1] - seg[-1][0] <= 1024  # the call ends on a light segment
        assert max(hi - lo for lo, hi in seg) <= (T + 3) // 4 + 128


def test_known_plans(segments):
    assert segments(16384) == [(12288, 16384), (8192, 12288), (4096, 8192), (2048, 4096),
                               (1024, 2048), (0, 1024)]
    assert segments(4500) == [(3456, 4500), (2304, 3456), (1152, 2304), (512, 1152), (0, 512)]
    assert segments(300) == [(0, 300)]


def test_cap_and_bad_arguments(segments):
    seg = segments(16384, cap=2)
    assert len(seg) == 2 and seg[0][1] == 16384 and seg[-1][0] == 0 and seg[1][1] == seg[0][0]
    with pytest.raises(ValueError):
        segments(-1)
    with pytest.raises(ValueError):
        segments(100, cap=0)
