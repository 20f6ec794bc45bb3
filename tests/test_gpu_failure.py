"""Failure detection on the device, without a fault.

Every wait of the library's kernels is bounded: when a wait runs out the
kernel records a status bit in its workspace, raises the CTA's abort flag so
that the other roles stop waiting, and returns; the host learns of it from
nomas_device_status. nomas_selftest_bounded_wait runs that path for real: its
kernel waits on an mbarrier that nothing arrives on. No trap, bad address or
endless loop is involved, and the context must stay usable afterwards.
"""

import time

import numpy as np
import pytest

import synth
from harness import MAX_ABS, REL_L2, current_segment, errors, make_caches, to_dev, to_f64

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_the_context_stays_usable():
    torch = __import__("torch")
    import segment_causal_kv_b200 as nm

    ws = torch.zeros(64, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    t0 = time.monotonic()
    assert nm.nomas_selftest_bounded_wait(ws.data_ptr(), stream) == nm.NOMAS_OK
    rc = nm.nomas_device_status(ws.data_ptr(), stream)
    elapsed = time.monotonic() - t0
    assert rc == nm.NOMAS_ERR_DEVICE_TIMEOUT, nm.nomas_status_string(rc)
    words = ws.view(torch.int32)[:3].cpu().tolist()
    # word 0 was read and cleared by nomas_device_status; word 1: the first role gave up;
    # word 2: the second role returned on the abort flag
    assert words == [0, 1, 1], words
    # the wait gave up after its 2 s limit, not at once and not much later
    assert 1.5 < elapsed < 60.0, elapsed
    # the status was cleared by the read
    assert nm.nomas_device_status(ws.data_ptr(), stream) == nm.NOMAS_OK

    # the context still works: a small commit + attention matches the oracle
    w = dict(synth.WORKLOADS["tiny"])
    cache, orc = make_caches(w)
    q, k, v = current_segment(w)
    out = cache.seg_attn(to_dev(q), to_dev(k), to_dev(v), w["cur_frames"], w["n_text"])
    torch.cuda.synchronize()
    assert cache.device_status() == nm.NOMAS_OK
    ref, _ = orc.seg_attn(q, k, v, w["cur_frames"], w["n_text"])
    mx, rel = errors(to_f64(out), ref)
    assert np.isfinite(mx) and mx <= MAX_ABS and rel <= REL_L2, (mx, rel)


def test_selftest_rejects_a_bad_workspace():
    import segment_causal_kv_b200 as nm

    assert nm.nomas_selftest_bounded_wait(None, None) == nm.NOMAS_ERR_ARG
