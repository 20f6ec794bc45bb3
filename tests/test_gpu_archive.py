"""The archive of evicted frames on the GPU: copies out of the cache, bit for bit.

Every commit goes through a FrameArchive, which first enqueues
nomas_kv_archive_evicted on the commit's stream. Before each commit the oracle
records the stored rows of the frames that commit will drop (its window
before minus its window after); at the end the archive must hold exactly
those frames, each equal to the oracle's rows, and nothing else.
"""

import numpy as np
import pytest

import oracle
import synth
from harness import oracle_mode, to_dev

pytestmark = pytest.mark.gpu


def run(mode, heads, gh, gw, window, commits, seed):
    torch = __import__("torch")
    import segment_causal_kv_b200 as nm
    gpu = nm.KVCache(mode, heads, gh, gw, window, window)
    orc = oracle.OracleCache(oracle_mode(mode), heads, gh, gw, window, window)
    arch = nm.FrameArchive()
    geo = synth.Geometry(heads, gh, gw)
    expected = {}
    stream = torch.cuda.current_stream()
    for s, n in enumerate(commits):
        k, v = synth.history_kv(geo, n, seed, s)
        before = {f: orc.frame_rows(f) for f in orc.window_frames()}
        orc.commit(k, v, n)
        for f in set(before) - set(orc.window_frames()):
            expected[f] = before[f]
        gpu.commit(to_dev(k), to_dev(v), n, stream=stream, archive=arch)
    torch.cuda.synchronize()
    assert arch.frames() == sorted(expected)
    for f, (ek, ev, eks, evs) in expected.items():
        gk, gv, gks, gvs = arch.frame(f)
        if mode == "int8":
            assert np.array_equal(gk.numpy(), ek) and np.array_equal(gv.numpy(), ev), f
            assert np.array_equal(gks.numpy().view(np.uint32), eks.view(np.uint32)), f
            assert np.array_equal(gvs.numpy().view(np.uint32), evs.view(np.uint32)), f
        else:
            assert np.array_equal(gk.view(torch.int16).numpy().view(np.uint16), ek), f
            assert np.array_equal(gv.view(torch.int16).numpy().view(np.uint16), ev), f
            assert gks is None and gvs is None
    # what stays in the window is untouched by the copies
    if mode == "int8":
        assert np.array_equal(gpu.k.cpu().numpy(), orc.k_code)
        assert np.array_equal(gpu.k_scale.cpu().numpy().view(np.uint32), orc.k_scale.view(np.uint32))
    return arch


@pytest.mark.parametrize("mode", ["int8", "bf16"])
def test_archive_holds_every_evicted_frame_bit_exact(mode):
    # partial fill, wrap, a commit longer than the window, ragged commits
    run(mode, 3, 4, 8, 4, [1, 2, 1, 3, 6, 2, 4, 1], seed=21)


def test_archive_single_gpu_configuration():
    # 18-frame INT8 window of 16 heads x 880 tokens, then three 3-frame commits
    arch = run("int8", 16, 22, 40, 18, [3] * 6 + [3, 3, 3], seed=1)
    assert arch.frames() == list(range(9))
    assert arch.host_bytes() == 9 * 16 * 880 * (2 * 128 + 2 * 4)


def test_full_history_archives_nothing():
    import segment_causal_kv_b200 as nm
    gpu = nm.KVCache("bf16", 2, 4, 8, 0, 8)
    for n in (1, 3):
        assert gpu.evicted_frames(n)[1] == 0
        assert gpu.archive_evicted(n).count == 0
        gpu.commit(to_dev(np.zeros((n * 32, 2, 128), np.uint16)), to_dev(np.zeros((n * 32, 2, 128), np.uint16)), n)
