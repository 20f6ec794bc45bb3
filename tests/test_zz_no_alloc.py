"""nomas_seg_attn_static: the entry point for callers that cannot allocate.

Some callers cannot hand nomas_seg_attn a device workspace -- an operator
plugin whose host framework passes it only inputs and outputs, or code that
runs where a cudaMalloc would synchronise the device or fail because all
device memory is reserved. nomas_seg_attn_static serves them from a fixed
scratch array in the library's device image. These checks call it through
the C ABI and require its output to equal, bit for bit, that of the
workspace entry point given a workspace of the same size on the same inputs
(the two run the same kernels with the same plan), on two calls in a row (the
array keeps the last call's contents, so the second call must not depend on
them); the single-GPU configuration (18-frame INT8 history) must run through
it and match the oracle; and a shape whose scratch exceeds the fixed size is
refused before anything runs.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes on its own.
"""

import numpy as np
import pytest

import synth
from harness import MAX_ABS, REL_L2, current_segment, errors, make_caches, sample_rows, to_dev, to_f64

pytestmark = pytest.mark.gpu


def _static_call(nm, cache, q, k, v, n_video_frames, n_text, out, lse):
    torch = __import__("torch")
    stream = torch.cuda.current_stream().cuda_stream
    return nm.nomas_seg_attn_static(cache.desc, q.data_ptr(), k.data_ptr(), v.data_ptr(), q.stride(0),
                                    n_video_frames, n_text, out.data_ptr(), lse.data_ptr(), stream)


@pytest.mark.parametrize("mode", ["int8", "bf16"])
def test_static_scratch_matches_the_workspace_entry_point(mode):
    torch = __import__("torch")
    import segment_causal_kv_b200 as nm

    # several KV tiles, ragged tails, and the split-KV merge path
    w = dict(heads=4, grid_h=16, grid_w=16, mode=mode, window=6 if mode == "int8" else 0,
             capacity=6 if mode == "int8" else 10, hist_commits=[2, 2, 2], cur_frames=3, n_text=100, seed=21,
             q_std=1.0, kv_std=1.0)
    cache, _ = make_caches(w, with_oracle=False)
    assert cache.workspace_bytes(3, 100) <= nm.NOMAS_STATIC_SCRATCH_BYTES
    q, k, v = (to_dev(x) for x in current_segment(w))
    nq = q.shape[0]

    _check_static_equals_workspace_call(nm, cache, q, k, v, 3, 100)


def _check_static_equals_workspace_call(nm, cache, q, k, v, n_video_frames, n_text):
    """Two static calls in a row, each bit-identical to nomas_seg_attn given a
    workspace of NOMAS_STATIC_SCRATCH_BYTES (the same plan, the same kernels)."""
    torch = __import__("torch")
    nq = q.shape[0]
    ws = torch.zeros(nm.NOMAS_STATIC_SCRATCH_BYTES, dtype=torch.uint8, device="cuda")
    ref_lse = torch.empty((cache.heads, nq), dtype=torch.float32, device="cuda")
    ref = cache.seg_attn(q, k, v, n_video_frames, n_text, lse=ref_lse, workspace=ws)
    torch.cuda.synchronize()
    assert cache.device_status() == nm.NOMAS_OK
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        rc = _static_call(nm, cache, q, k, v, n_video_frames, n_text, out, lse)
        assert rc == nm.NOMAS_OK, nm.nomas_status_string(rc)
        torch.cuda.synchronize()
        assert torch.equal(out, ref), call
        assert torch.equal(lse, ref_lse), call
    # no bounded wait of the static calls ran out
    assert nm.nomas_seg_attn_static_status(torch.cuda.current_stream().cuda_stream) == nm.NOMAS_OK
    return ref, ref_lse


def test_static_scratch_serves_the_single_gpu_configuration():
    """16 heads, 18-frame INT8 history, 3 frames + 256 text tokens: the plan is
    fitted inside the fixed scratch; bit-identical to the workspace call with
    the same byte budget and within the parity bar of the oracle."""
    import segment_causal_kv_b200 as nm

    w = synth.WORKLOADS["single_gpu_int8_18f"]
    cache, orc = make_caches(w)
    q_h, k_h, v_h = current_segment(w)
    q, k, v = (to_dev(x) for x in (q_h, k_h, v_h))
    assert cache.workspace_min_bytes(3, 256) <= nm.NOMAS_STATIC_SCRATCH_BYTES
    ref, _ = _check_static_equals_workspace_call(nm, cache, q, k, v, 3, 256)
    F = w["grid_h"] * w["grid_w"]
    rows = sample_rows(3 * F + 256, F, 3, per_head=48)
    want, _ = orc.seg_attn(q_h, k_h, v_h, 3, 256, rows=rows)
    mx, rel = errors(to_f64(ref)[rows], want)
    assert mx <= MAX_ABS and rel <= REL_L2, (mx, rel)


def test_static_scratch_refuses_shapes_beyond_its_size():
    torch = __import__("torch")
    import segment_causal_kv_b200 as nm

    w = dict(synth.WORKLOADS["tiny"])
    w.update(heads=16, grid_h=22, grid_w=40, hist_commits=[], capacity=1)
    cache, _ = make_caches(w, with_oracle=False)
    # 72 latent frames of 880 tokens: the rotated Q and K alone exceed the static scratch
    need = cache.workspace_bytes(72, 256)
    assert need > nm.NOMAS_STATIC_SCRATCH_BYTES
    small = torch.zeros((16, 16, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((16, 16), dtype=torch.float32, device="cuda")
    rc = _static_call(nm, cache, small, small, small, 72, 256, small, lse)
    assert rc == nm.NOMAS_ERR_WORKSPACE
