"""Pins of the oracle's per-latent-frame camera cross-attention (oracle.camera_attn).

Each check fixes the result by something other than the oracle's own formula:
  * one camera token per chunk: the softmax weight is exactly 1, so every video
    token of the chunk gets that token's V, exactly;
  * two camera tokens: the logistic closed form sigma(s1 - s2) v1 + sigma(s2 - s1) v2;
  * a library routine: PyTorch's fp64 scaled_dot_product_attention over all video
    tokens and all camera tokens with a block-diagonal mask (token i may see
    chunk (i / F) / chunk_frames only);
  * invariants: camera token order inside a chunk does not matter, and changing one
    chunk's K/V changes only the outputs of that chunk's video tokens.
A wrong chunk index, head index or transposed operand fails at least one.
"""

import numpy as np
import pytest

import oracle
import synth


def f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def case(heads=3, gh=2, gw=3, n_frames=5, n_cam=1, chunk=1, seed=0):
    geo = synth.Geometry(heads, gh, gw)
    F = geo.tokens_per_frame
    q, _, _ = synth.segment_qkv(geo, n_frames, 0, seed)
    n_chunks = -(-n_frames // chunk)
    kc, vc = synth.camera_kv(geo, n_chunks, n_cam, seed)
    return q, kc, vc, F


@pytest.mark.parametrize("chunk", [1, 2])
def test_one_camera_token_passes_its_value_through(chunk):
    q, kc, vc, F = case(n_frames=5, n_cam=1, chunk=chunk)
    out = oracle.camera_attn(q, 5, F, kc, vc, chunk)
    for i in range(q.shape[0]):
        c = (i // F) // chunk
        np.testing.assert_array_equal(out[i], f64(vc[c, 0]))


def test_two_camera_tokens_follow_the_logistic_form():
    q, kc, vc, F = case(n_frames=3, n_cam=2, seed=4)
    out = oracle.camera_attn(q, 3, F, kc, vc, 1)
    Q, K, V = f64(q), f64(kc), f64(vc)
    for i in range(q.shape[0]):
        c = i // F
        for h in range(q.shape[1]):
            s1 = Q[i, h] @ K[c, 0, h] / np.sqrt(128.0)
            s2 = Q[i, h] @ K[c, 1, h] / np.sqrt(128.0)
            w1 = 1.0 / (1.0 + np.exp(s2 - s1))
            np.testing.assert_allclose(out[i, h], w1 * V[c, 0, h] + (1.0 - w1) * V[c, 1, h], rtol=0, atol=1e-13)


@pytest.mark.parametrize("n_frames,n_cam,chunk", [(4, 3, 1), (5, 4, 2), (1, 7, 3)])
def test_block_diagonal_dense_attention_from_the_library(n_frames, n_cam, chunk):
    torch = pytest.importorskip("torch")
    q, kc, vc, F = case(n_frames=n_frames, n_cam=n_cam, chunk=chunk, seed=7)
    out = oracle.camera_attn(q, n_frames, F, kc, vc, chunk)
    H = q.shape[1]
    n_chunks = kc.shape[0]
    Q = torch.from_numpy(f64(q)).permute(1, 0, 2)                              # [H][Nv][128]
    K = torch.from_numpy(f64(kc)).reshape(n_chunks * n_cam, H, 128).permute(1, 0, 2)
    V = torch.from_numpy(f64(vc)).reshape(n_chunks * n_cam, H, 128).permute(1, 0, 2)
    tok_chunk = (torch.arange(n_frames * F) // F) // chunk
    key_chunk = torch.arange(n_chunks * n_cam) // n_cam
    mask = tok_chunk[:, None] == key_chunk[None, :]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=mask).permute(1, 0, 2).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_key_order_is_irrelevant_and_chunks_are_independent():
    q, kc, vc, F = case(n_frames=4, n_cam=5, seed=9)
    out = oracle.camera_attn(q, 4, F, kc, vc, 1)
    perm = np.array([3, 0, 4, 2, 1])
    out_p = oracle.camera_attn(q, 4, F, kc[:, perm], vc[:, perm], 1)
    np.testing.assert_allclose(out_p, out, rtol=0, atol=1e-14)
    kc2, vc2 = kc.copy(), vc.copy()
    kc2[2] ^= np.uint16(0x0040)  # perturb chunk 2 only
    vc2[2] ^= np.uint16(0x0040)
    out2 = oracle.camera_attn(q, 4, F, kc2, vc2, 1)
    changed = np.any(out2 != out, axis=(1, 2))
    assert not changed[:2 * F].any() and not changed[3 * F:].any() and changed[2 * F:3 * F].all()


def test_bad_arguments_are_rejected():
    q, kc, vc, F = case(n_frames=2, n_cam=1)
    with pytest.raises(AssertionError):
        oracle.camera_attn(q, 2, F, kc[:1], vc[:1], 1)  # one chunk short
