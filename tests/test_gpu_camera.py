"""Parity of nomas_camera_attn (per-latent-frame camera cross-attention, through
the C ABI) with the oracle: bit-exact where one camera token per chunk makes
the output that token's V, and within the attention bar (max-abs 2e-2,
relative L2 5e-3) against the fp64 oracle otherwise."""

import numpy as np
import pytest

import oracle
import synth
from harness import MAX_ABS, REL_L2, Guards, errors, to_dev, to_f64

pytestmark = pytest.mark.gpu


def inputs(heads, gh, gw, n_frames, n_cam, chunk, seed, q_std=1.0):
    geo = synth.Geometry(heads, gh, gw)
    q, _, _ = synth.segment_qkv(geo, n_frames, 0, seed, q_std=q_std)
    kc, vc = synth.camera_kv(geo, -(-n_frames // chunk), n_cam, seed)
    return q, kc, vc, geo.tokens_per_frame


@pytest.mark.parametrize("n_frames,chunk", [(3, 1), (72, 1), (5, 2)])
def test_one_camera_token_gives_its_value_exactly(n_frames, chunk):
    torch = __import__("torch")
    import segment_causal_kv_b200 as nm
    q, kc, vc, F = inputs(16, 22, 40, n_frames, 1, chunk, seed=31)
    g = Guards()  # canary bands around the output
    out = g.alloc(q.shape, torch.bfloat16, fill=0.0)
    nm.camera_attn(to_dev(q), to_dev(kc), to_dev(vc), n_frames, F, chunk, out=out)
    torch.cuda.synchronize()
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    want = vc[(np.arange(n_frames * F) // F) // chunk, 0]
    assert np.array_equal(got, want)
    g.check()


@pytest.mark.parametrize("heads,gh,gw,n_frames,n_cam,chunk,q_std", [
    (3, 4, 8, 5, 4, 2, 1.0),      # ragged last chunk
    (16, 22, 40, 3, 8, 1, 1.0),   # single-GPU segment, 8 camera tokens per frame
    (2, 3, 5, 7, 33, 3, 4.0),     # peaky softmax, odd sizes
    (1, 1, 1, 1, 1, 1, 1.0),      # one token, one head
])
def test_camera_attn_matches_the_oracle(heads, gh, gw, n_frames, n_cam, chunk, q_std):
    torch = __import__("torch")
    import segment_causal_kv_b200 as nm
    q, kc, vc, F = inputs(heads, gh, gw, n_frames, n_cam, chunk, seed=heads + n_cam, q_std=q_std)
    g = Guards()
    out = g.alloc(q.shape, torch.bfloat16, fill=float("nan"))
    nm.camera_attn(to_dev(q), to_dev(kc), to_dev(vc), n_frames, F, chunk, out=out)
    torch.cuda.synchronize()
    ref = oracle.camera_attn(q, n_frames, F, kc, vc, chunk)
    got = to_f64(out)
    assert np.isfinite(got).all()
    mx, rel = errors(got, ref)
    assert mx <= MAX_ABS and rel <= REL_L2, (mx, rel)
    g.check()


def test_padded_strides_touch_only_their_rows():
    torch = __import__("torch")
    import segment_causal_kv_b200 as nm
    heads, n_frames, n_cam = 4, 3, 3
    q, kc, vc, F = inputs(heads, 4, 8, n_frames, n_cam, 1, seed=5)
    nv = n_frames * F
    qbuf = torch.zeros((nv, heads + 2, 128), dtype=torch.bfloat16, device="cuda")
    qbuf[:, 1:1 + heads] = to_dev(q)
    obuf = torch.full((nv, heads + 3, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    nm.camera_attn(qbuf[:, 1:1 + heads], to_dev(kc), to_dev(vc), n_frames, F, 1, out=obuf[:, 2:2 + heads])
    torch.cuda.synchronize()
    ref = oracle.camera_attn(q, n_frames, F, kc, vc, 1)
    mx, rel = errors(to_f64(obuf[:, 2:2 + heads]), ref)
    assert mx <= MAX_ABS and rel <= REL_L2, (mx, rel)
    # rows outside the output view keep their fill
    assert bool((obuf[:, :2] == 7.0).all()) and bool((obuf[:, 2 + heads:] == 7.0).all())
