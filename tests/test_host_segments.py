"""The row segments of the host-buffer prefill (polar_attn_fwd_host), as the
library computes them: host logic only, checked on a machine without a GPU.
Every row is covered exactly once, from the last rows to the first, on 128-row
query-tile boundaries, the last segment to go is the lightest (at most 1024
rows), and short sequences go in one segment."""
import ctypes
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "polar_attention_b200", "libpolar_attn.so")


@pytest.fixture(scope="module")
def segments():
    if not os.path.exists(LIB):
        pytest.skip("library not built")
    lib = ctypes.CDLL(LIB)
    f = lib.polar_attn_selftest_fwd_host_segments
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                  ctypes.c_int]

    def call(T, cap=64):
        lo = (ctypes.c_int * cap)()
        hi = (ctypes.c_int * cap)()
        n = f(T, lo, hi, cap)
        return n, list(lo[:max(n, 0)]), list(hi[:max(n, 0)])
    return call


@pytest.mark.parametrize("T", [1, 127, 128, 300, 1024, 2047, 2048, 2049, 4500, 8192, 16384,
                               16385, 65536, 131072, 262144])
def test_cover_every_row_once_last_rows_first(segments, T):
    n, lo, hi = segments(T)
    assert n >= 1
    assert hi[0] == T and lo[-1] == 0
    for i in range(n):
        assert 0 <= lo[i] < hi[i] <= T
        assert lo[i] % 128 == 0
        if i + 1 < n:
            assert hi[i + 1] == lo[i]          # contiguous, descending
    if T < 2048:
        assert n == 1
    else:
        assert hi[-1] - lo[-1] <= 1024         # the call ends on a light segment
        sizes = [h - l for l, h in zip(lo, hi)]
        assert max(sizes) <= (T + 3) // 4 + 128


def test_known_plans(segments):
    assert segments(16384)[1:] == ([12288, 8192, 4096, 2048, 1024, 0],
                                   [16384, 12288, 8192, 4096, 2048, 1024])
    assert segments(4500)[1:] == ([3456, 2304, 1152, 512, 0], [4500, 3456, 2304, 1152, 512])
    assert segments(300)[1:] == ([0], [300])


def test_cap_and_bad_arguments(segments):
    n, lo, hi = segments(16384, cap=2)
    assert n == 2 and hi[0] == 16384 and lo[-1] == 0 and hi[1] == lo[0]
    assert segments(-1)[0] == -1
    assert segments(100, cap=0)[0] == -1
