"""Which frames leave the window, on the host: nomas_kv_evicted_frames against the oracle.

The oracle's own rule is a set difference: the frames its slots hold before a
commit minus those they hold after it. The library computes the same range
from its counters. The commits below fill the window partly, wrap it, and
overrun it with a segment longer than the window. The descriptor uses fake
device addresses (no call here touches the device), and its counters are set
to the oracle's state before each commit, as a commit would leave them.
"""

import pytest

import oracle
import segment_causal_kv_b200 as nm
import synth

FAKE = 0x7F0000000000


def desc(mode, heads, gh, gw, window, cap):
    ks, vs = (FAKE + (2 << 30), FAKE + (3 << 30)) if mode == nm.NOMAS_CACHE_INT8 else (None, None)
    d = nm.NomasCacheDesc(mode, heads, 128, gh, gw, window, cap, 256.0, FAKE, FAKE + (1 << 30), ks, vs,
                          0, 0, 0, 0)
    assert nm.nomas_cache_reset(d) == nm.NOMAS_OK
    return d


@pytest.mark.parametrize("mode,window,cap,commits", [
    ("int8", 4, 4, [1, 2, 1, 3, 6, 2, 4, 1, 9]),
    ("int8", 18, 18, [3] * 9 + [20]),
    ("int8", 1, 1, [1, 2, 1, 1]),
    ("bf16", 3, 3, [2, 2, 5, 1]),
    ("bf16", 0, 12, [3, 4, 5]),  # full history: nothing ever leaves
])
def test_evicted_range_is_the_oracle_window_difference(mode, window, cap, commits):
    heads, gh, gw = 2, 2, 3
    m = nm.NOMAS_CACHE_INT8 if mode == "int8" else nm.NOMAS_CACHE_BF16
    orc = oracle.OracleCache(oracle.MODE_INT8 if mode == "int8" else oracle.MODE_BF16, heads, gh, gw, window, cap)
    d = desc(m, heads, gh, gw, window, cap)
    geo = synth.Geometry(heads, gh, gw)
    for s, n in enumerate(commits):
        before = set(orc.window_frames())
        k, v = synth.history_kv(geo, n, 5, s)
        orc.commit(k, v, n)
        expected = sorted(before - set(orc.window_frames()))
        rc, count, first = nm.nomas_kv_evicted_frames(d, n)
        assert rc == nm.NOMAS_OK
        assert list(range(first, first + count)) == expected, (s, n, first, count, expected)
        # the counters a commit of n frames leaves
        d.frames_committed = orc.frames_committed
        d.valid_frames = orc.valid_frames
        d.head_slot = orc.frames_committed % window if window else orc.frames_committed
    if window == 0:
        assert orc.window_frames() == list(range(sum(commits)))


def test_archive_host_checks_come_before_any_copy():
    d = desc(nm.NOMAS_CACHE_INT8, 2, 2, 3, 4, 4)
    d.frames_committed, d.valid_frames, d.head_slot = 6, 4, 2  # frames 2..5 in the window
    assert nm.nomas_kv_evicted_frames(d, -1)[0] == nm.NOMAS_ERR_ARG
    assert nm.nomas_kv_evicted_frames(d, 0) == (nm.NOMAS_OK, 0, 2)
    assert nm.nomas_kv_evicted_frames(d, 3) == (nm.NOMAS_OK, 3, 2)
    # too small a host archive: rejected, but the count is reported
    assert nm.nomas_kv_archive_evicted(d, 3, FAKE, FAKE, FAKE, FAKE, 2, None) == (nm.NOMAS_ERR_CAPACITY, 3, 2)
    # missing buffers when there is something to copy
    assert nm.nomas_kv_archive_evicted(d, 3, None, FAKE, FAKE, FAKE, 3, None)[0] == nm.NOMAS_ERR_ARG
    assert nm.nomas_kv_archive_evicted(d, 3, FAKE, FAKE, None, FAKE, 3, None)[0] == nm.NOMAS_ERR_ARG
    # nothing to copy: no buffers, no device needed
    assert nm.nomas_kv_archive_evicted(d, 0, None, None, None, None, 0, None) == (nm.NOMAS_OK, 0, 2)
    assert nm.nomas_kv_archive_evicted(d, 3, FAKE, FAKE, FAKE, FAKE, -1, None)[0] == nm.NOMAS_ERR_ARG
    # a changed configuration is caught first
    d.grid_w = 4
    assert nm.nomas_kv_evicted_frames(d, 1)[0] == nm.NOMAS_ERR_STATE
    assert nm.nomas_kv_archive_evicted(d, 1, FAKE, FAKE, FAKE, FAKE, 4, None)[0] == nm.NOMAS_ERR_STATE
    # BF16 windows need no scale buffers
    b = desc(nm.NOMAS_CACHE_BF16, 2, 2, 3, 2, 2)
    b.frames_committed, b.valid_frames, b.head_slot = 2, 2, 0
    assert nm.nomas_kv_archive_evicted(b, 1, FAKE, None, None, None, 1, None)[0] == nm.NOMAS_ERR_ARG
    assert nm.nomas_kv_evicted_frames(b, 1) == (nm.NOMAS_OK, 1, 0)

