"""Bit-exact parity of nomas_kv_commit (CUDA, through the C ABI) with the
oracle's commit: INT8 codes, fp32 scales (as bit patterns), BF16 cache
values, slot placement and the host counters."""

import numpy as np
import pytest

import oracle
import synth
from harness import Guards, make_caches, to_dev

pytestmark = pytest.mark.gpu


def assert_cache_equal(gpu, orc):
    torch = __import__("torch")
    torch.cuda.synchronize()
    if gpu.mode == "int8":
        assert np.array_equal(gpu.k.cpu().numpy(), orc.k_code)
        assert np.array_equal(gpu.v.cpu().numpy(), orc.v_code)
        assert np.array_equal(gpu.k_scale.cpu().numpy().view(np.uint32), orc.k_scale.view(np.uint32))
        assert np.array_equal(gpu.v_scale.cpu().numpy().view(np.uint32), orc.v_scale.view(np.uint32))
    else:
        assert np.array_equal(gpu.k.cpu().view(torch.int16).numpy().view(np.uint16), orc.k_bf16)
        assert np.array_equal(gpu.v.cpu().view(torch.int16).numpy().view(np.uint16), orc.v_bf16)
    assert gpu.frames_committed == orc.frames_committed
    assert gpu.valid_frames == orc.valid_frames


def test_commit_int8_eighteen_frame_history_bit_exact():
    w = synth.WORKLOADS["single_gpu_int8_18f"]
    g = Guards()  # canary bands around the cache tensors
    gpu, orc = make_caches(w, guards=g)
    assert_cache_equal(gpu, orc)
    assert gpu.valid_frames == 18 and gpu.head_slot == 0
    g.check()


@pytest.mark.parametrize("mode", ["int8", "bf16"])
def test_commit_ring_wraps_and_long_commits(mode):
    W = 4
    geo = synth.Geometry(3, 5, 7)
    import segment_causal_kv_b200 as nm
    g = Guards()
    gpu = nm.KVCache(mode, 3, 5, 7, W, W, alloc=g.zeros)
    orc = oracle.OracleCache(oracle.MODE_INT8 if mode == "int8" else oracle.MODE_BF16, 3, 5, 7, W, W)
    for s, nf in enumerate([3, 2, 5, 1, 9, 4]):
        k, v = synth.history_kv(geo, nf, 90, s)
        gpu.commit(to_dev(k), to_dev(v), nf)
        orc.commit(k, v, nf)
        assert_cache_equal(gpu, orc)
        assert gpu.head_slot == gpu.frames_committed % W
    g.check()


def test_commit_bf16_full_history_and_capacity():
    geo = synth.Geometry(2, 4, 8)
    import segment_causal_kv_b200 as nm
    gpu = nm.KVCache("bf16", 2, 4, 8, 0, 6)
    orc = oracle.OracleCache(oracle.MODE_BF16, 2, 4, 8, 0, 6)
    for s, nf in enumerate([2, 3, 1]):
        k, v = synth.history_kv(geo, nf, 91, s)
        gpu.commit(to_dev(k), to_dev(v), nf)
        orc.commit(k, v, nf)
    assert_cache_equal(gpu, orc)
    k, v = synth.history_kv(geo, 1, 91, 9)
    with pytest.raises(nm.NomasError) as e:
        gpu.commit(to_dev(k), to_dev(v), 1)
    assert e.value.status == nm.NOMAS_ERR_CAPACITY


def test_commit_with_padded_token_stride_and_zero_rows():
    torch = __import__("torch")
    import segment_causal_kv_b200 as nm
    H, gh, gw = 4, 3, 6
    geo = synth.Geometry(H, gh, gw)
    k, v = synth.history_kv(geo, 2, 92, 0)
    k[5, 1, :] = 0          # an all-zero (token, head) row: scale 0, codes 0
    v[7, :, :] = 0
    k[9, 2, 3] = 0x8000     # negative zero
    n = k.shape[0]
    pad = 64
    kb = torch.zeros((n, H * 128 + pad), dtype=torch.bfloat16, device="cuda")
    vb = torch.zeros_like(kb)
    kb[:, :H * 128] = to_dev(k).reshape(n, H * 128)
    vb[:, :H * 128] = to_dev(v).reshape(n, H * 128)
    kv = kb[:, :H * 128].view(n, H, 128)
    vv = vb[:, :H * 128].view(n, H, 128)
    assert kv.stride(0) == H * 128 + pad
    gpu = nm.KVCache("int8", H, gh, gw, 3, 3)
    gpu.commit(kv, vv, 2)
    orc = oracle.OracleCache(oracle.MODE_INT8, H, gh, gw, 3, 3)
    orc.commit(k, v, 2)
    assert_cache_equal(gpu, orc)
    F = gh * gw
    assert gpu.k_scale[1, 5].item() == 0.0 and not gpu.k[1, 5].any()


def test_commit_large_segment_spans_several_launches():
    # 130 frames of a 2x2 grid: more frames than one launch's RoPE table holds
    import segment_causal_kv_b200 as nm
    geo = synth.Geometry(2, 2, 2)
    gpu = nm.KVCache("int8", 2, 2, 2, 0, 140)
    orc = oracle.OracleCache(oracle.MODE_INT8, 2, 2, 2, 0, 140)
    for s, nf in enumerate([5, 130]):
        k, v = synth.history_kv(geo, nf, 93, s)
        gpu.commit(to_dev(k), to_dev(v), nf)
        orc.commit(k, v, nf)
    assert_cache_equal(gpu, orc)


def test_commit_subnormal_tiny_and_large_rows():
    """Rows whose absmax is a BF16 subnormal (the row scale is then an fp32
    subnormal and 1/scale overflows), rows of the smallest normals, rows near
    2^97, and single-element rows: codes and scales stay bit-exact."""
    import segment_causal_kv_b200 as nm
    H, gh, gw, W = 2, 3, 4, 2
    geo = synth.Geometry(H, gh, gw)
    k, v = synth.history_kv(geo, 2, 94, 0)
    rng = np.random.default_rng(5)
    sign = (rng.integers(0, 2, size=128) << 15).astype(np.uint16)
    sub = (rng.integers(0, 0x80, size=128).astype(np.uint16) | sign)
    sub[::7] = 0
    k[0, 0] = sub                                   # subnormal row, with zeros and both signs
    v[1, 1] = sub
    one = np.zeros(128, np.uint16)
    one[17] = 0x0001                                # a single smallest subnormal
    k[2, 1] = one
    v[2, 0] = one | 0x8000
    k[3, 0] = (k[3, 0] & 0x807F) | 0x0080           # smallest normal exponent
    k[4, 1] = (k[4, 1] & 0x807F) | (0xE0 << 7)      # around 2^97
    v[5, 0] = (v[5, 0] & 0x807F) | (0xE0 << 7)
    gpu = nm.KVCache("int8", H, gh, gw, W, W)
    orc = oracle.OracleCache(oracle.MODE_INT8, H, gh, gw, W, W)
    gpu.commit(to_dev(k), to_dev(v), 2)
    orc.commit(k, v, 2)
    assert_cache_equal(gpu, orc)
    F = gh * gw
    # the subnormal row got a subnormal (nonzero) scale and non-trivial codes
    s = gpu.k_scale.cpu().numpy()[0, 0]
    assert 0.0 < s < 1.17549435e-38
    assert gpu.k[0, 0].abs().max().item() == 127


@pytest.mark.parametrize("mode,n_layers", [("int8", 3), ("bf16", 3), ("int8", 54), ("int8", 130)])
def test_layered_commit_matches_per_layer_commits(mode, n_layers):
    """nomas_kv_commit_layers writes into every layer cache exactly what the
    oracle's commit of that layer's segment writes (54 layers, the model's
    depth: one launch; 130 layers: two launches)."""
    import segment_causal_kv_b200 as nm
    H, gh, gw, W = 2, 3, 5, 4
    geo = synth.Geometry(H, gh, gw)
    om = oracle.MODE_INT8 if mode == "int8" else oracle.MODE_BF16
    g = Guards()
    gpus = [nm.KVCache(mode, H, gh, gw, W, W, alloc=g.zeros) for _ in range(n_layers)]
    orcs = [oracle.OracleCache(om, H, gh, gw, W, W) for _ in range(n_layers)]
    for s, nf in enumerate([3, 2, 4]):  # wraps the 4-frame ring
        kv = [synth.history_kv(geo, nf, 200 + layer, s) for layer in range(n_layers)]
        nm.commit_layers(gpus, [to_dev(k) for k, _ in kv], [to_dev(v) for _, v in kv], nf)
        for o, (k, v) in zip(orcs, kv):
            o.commit(k, v, nf)
        for gc, o in zip(gpus, orcs):
            assert_cache_equal(gc, o)
    g.check()



def _tie_row(scale_exp: int, rng) -> np.ndarray:
    """A 128-element row whose absmax is 127 * 2^e (so the fp32 scale is exactly
    2^e) and whose other elements sit exactly halfway between two codes
    (x / scale = k + 1/2), or 1/64 beside a small half (k < 3, where 1/64 is
    still a whole number of BF16 ulps). Dims 0-15 (the t block of
    RoPE) are zero, so the row passes the commit's rotation unchanged at grid
    cell (0, 0) of any frame. Returns the row as float64 (exact BF16 values)."""
    s = 2.0 ** scale_exp
    x = np.zeros(128, np.float64)
    x[16] = 127 * s
    x[17] = -127 * s
    fixed = np.array([0.5, 1.5, 2.5, 3.5, 62.5, 63.5, 64.5, 125.5, 126.5])
    fixed = np.concatenate([fixed, -fixed])
    x[18:36] = fixed * s
    k = rng.integers(0, 127, size=76)
    sgn = np.where(rng.integers(0, 2, size=76) == 1, 1.0, -1.0)
    x[36:112] = sgn * (k + 0.5) * s
    off = np.where(rng.integers(0, 2, size=16) == 1, 1.0, -1.0) / 64.0
    x[112:128] = (rng.integers(0, 3, size=16) + 0.5 + off) * s
    return x


def _bits(x: np.ndarray) -> np.ndarray:
    b = synth.f32_to_bf16_bits(x.astype(np.float32))
    assert np.array_equal(synth.bf16_bits_to_f32(b).astype(np.float64), x)  # exact in BF16
    return b


def test_commit_int8_round_half_even_ties():
    """Hand-built exact ties x / scale = k + 1/2 in K and V rows: the codes are
    round-half-to-even of the quotient (checked against the rule computed here
    from the constructed values, and bit for bit against the oracle's commit).
    K carries the ties at grid cell (0, 0) of each frame, whose h and w
    rotations are the identity; V carries them at every token. The scales are
    powers of two, so the kernel's reciprocal product is exact and every tie
    lies exactly on the rounding boundary its packed fast path must hand to the
    exact path."""
    import segment_causal_kv_b200 as nm
    H, gh, gw, W = 3, 4, 8, 4
    F = gh * gw
    geo = synth.Geometry(H, gh, gw)
    rng = np.random.default_rng(33)
    g = Guards()
    gpu = nm.KVCache("int8", H, gh, gw, W, W, alloc=g.zeros)
    orc = oracle.OracleCache(oracle.MODE_INT8, H, gh, gw, W, W)
    want = {}  # (tensor, head, slot row) -> (expected codes, expected scale)
    frame0 = 0
    for seg, nf in enumerate([2, 3]):  # the second segment wraps the 4-frame ring
        k, v = synth.history_kv(geo, nf, 95, seg)
        for f in range(nf):
            slot = (frame0 + f) % W
            for h in range(H):
                xk = _tie_row(-4 - h, rng)
                k[f * F, h] = _bits(xk)
                want[("k", h, slot * F)] = (np.rint(xk / 2.0 ** (-4 - h)), 2.0 ** (-4 - h))
                for t in range(f * F, (f + 1) * F):
                    xv = _tie_row(-6 + h, rng)
                    v[t, h] = _bits(xv)
                    want[("v", h, slot * F + t - f * F)] = (np.rint(xv / 2.0 ** (-6 + h)), 2.0 ** (-6 + h))
        gpu.commit(to_dev(k), to_dev(v), nf)
        orc.commit(k, v, nf)
        assert_cache_equal(gpu, orc)
        frame0 += nf
    codes = {"k": gpu.k.cpu().numpy(), "v": gpu.v.cpu().numpy()}
    scales = {"k": gpu.k_scale.cpu().numpy(), "v": gpu.v_scale.cpu().numpy()}
    # frames 1..4 are in the window; frame 0's slot was overwritten by frame 4
    live = {(1 + i) % W for i in range(W)}
    checked = 0
    for (t, h, row), (c, sc) in want.items():
        if row // F not in live:
            continue
        assert scales[t][h, row] == np.float32(sc)
        assert np.array_equal(codes[t][h, row].astype(np.float64), c), (t, h, row)
        checked += 1
    assert checked == H * W * (1 + F)
    # np.rint rounds half to even: the fixed ties landed on even codes
    assert np.all(codes["k"][0, F, 18:36] % 2 == 0)
    g.check()
