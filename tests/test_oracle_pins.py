"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: every expected value comes from
a closed form, exact rational arithmetic, a high-precision evaluation
(mpmath), a brute-force computation written separately, or a number printed
on the pages (tests/golden/page_constants.json).
"""

import json
import math
import os
from fractions import Fraction

import mpmath
import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
PAGE = json.load(open(os.path.join(GOLDEN, "page_constants.json")))
mpmath.mp.dps = 50


# ----------------------------------------------------------------------------
# exact helpers (independent of the oracle)
# ----------------------------------------------------------------------------

def round_f32(fr: Fraction) -> np.float32:
    """Round an exact rational to fp32, half to even (normal range only)."""
    if fr == 0:
        return np.float32(0.0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    assert e >= -126
    m = a * Fraction(2) ** (23 - e)
    q, r = divmod(m.numerator, m.denominator)
    rem = Fraction(r, m.denominator)
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and q % 2 == 1):
        q += 1
    return np.float32(sign * q * 2.0 ** (e - 23))


def F(x) -> Fraction:
    return Fraction(float(x))


def bf16_vals(bits):
    return synth.bf16_bits_to_f32(bits).astype(np.float64)


def axis_of_pair(p):
    """(axis, width, index) of dimension pair p under the split [16, 56, 56]."""
    t, h, w = PAGE["rope_split"]["value"]
    if p < t // 2:
        return 0, t, p
    if p < (t + h) // 2:
        return 1, h, p - t // 2
    return 2, w, p - (t + h) // 2


# ----------------------------------------------------------------------------
# page constants
# ----------------------------------------------------------------------------

def test_page_constants_are_self_consistent():
    assert sum(PAGE["rope_split"]["value"]) == PAGE["head_dim"]["value"]
    gh, gw = PAGE["grid_704x1280"]["value"]
    assert gh * gw == PAGE["tokens_per_frame_704x1280"]["value"]
    per_tok = PAGE["int8_kv_bytes_per_token_per_layer"]["value"]
    assert per_tok * PAGE["layers"]["value"] == PAGE["int8_kv_bytes_per_token_54_layers"]["value"]
    assert per_tok * PAGE["layers"]["value"] * 880 == PAGE["int8_kv_bytes_per_frame_54_layers"]["value"]


def test_int8_cache_code_bytes_match_the_pages():
    H, D = PAGE["heads"]["value"], PAGE["head_dim"]["value"]
    gh, gw = PAGE["grid_704x1280"]["value"]
    W = PAGE["history_budget_frames"]["value"]
    c = oracle.OracleCache(oracle.MODE_INT8, H, gh, gw, W, W)
    code_bytes = c.k_code.nbytes + c.v_code.nbytes
    per_frame_one_layer = PAGE["int8_kv_bytes_per_frame_54_layers"]["value"] // PAGE["layers"]["value"]
    assert code_bytes == W * per_frame_one_layer == 64_880_640
    assert code_bytes // (W * gh * gw) == PAGE["int8_kv_bytes_per_token_per_layer"]["value"]
    assert D == oracle.HEAD_DIM


# ----------------------------------------------------------------------------
# RoPE
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("pos", [0, 1, 5, 17, 123, 100003])
def test_rope_time_block_angles_closed_form(pos):
    # width 16, theta 256: theta^(-2j/16) = 2^(-j) exactly
    for j in range(8):
        assert oracle.rope_angle(16, j, pos, 256.0) == pos * 2.0 ** (-j)


def test_rope_spatial_block_angles_closed_form():
    # width 56, theta 256: theta^(-2j/56) = 2^(-2j/7); exact powers of two at j = 0, 7, 14, 21
    for j, want in [(0, 1.0), (7, 0.25), (14, 2.0 ** -4), (21, 2.0 ** -6)]:
        assert oracle.rope_angle(56, j, 1.0, 256.0) == want
        assert oracle.rope_angle(56, j, 39.0, 256.0) == 39.0 * want
    for j in range(28):
        want = float(mpmath.power(2, mpmath.mpf(-2 * j) / 7))
        assert oracle.rope_angle(56, j, 1.0, 256.0) == pytest.approx(want, rel=4e-16)


def test_rope_cos_sin_f32_are_rounded_high_precision_values():
    rng = np.random.default_rng(7)
    for _ in range(300):
        d = int(rng.choice([16, 56]))
        j = int(rng.integers(0, d // 2))
        pos = int(rng.integers(0, 500))
        a = oracle.rope_angle(d, j, pos, 256.0)  # pinned above
        c, s = oracle.rope_cs_f32(d, j, pos, 256.0)
        ma = mpmath.mpf(a)
        assert c == round_f32(Fraction(str(mpmath.nstr(mpmath.cos(ma), 45)))), (d, j, pos)
        assert s == round_f32(Fraction(str(mpmath.nstr(mpmath.sin(ma), 45)))), (d, j, pos)


def test_rope_split_places_each_pair_on_its_axis():
    pos = np.array([3.0, 7.0, 11.0])  # distinct t, h, w
    for p in range(64):
        ax, d, j = axis_of_pair(p)
        x = np.zeros(128)
        x[2 * p] = 1.0
        y = oracle.rope_rotate_f64(x, pos)
        ang = pos[ax] * float(mpmath.power(256, mpmath.mpf(-2 * j) / d))
        want = np.zeros(128)
        want[2 * p], want[2 * p + 1] = math.cos(ang), math.sin(ang)
        np.testing.assert_allclose(y, want, rtol=0, atol=1e-14)
        # the partner dimension rotates the other way round
        x = np.zeros(128)
        x[2 * p + 1] = 1.0
        y = oracle.rope_rotate_f64(x, pos)
        want = np.zeros(128)
        want[2 * p], want[2 * p + 1] = -math.sin(ang), math.cos(ang)
        np.testing.assert_allclose(y, want, rtol=0, atol=1e-14)


def test_rope_block_boundaries():
    # dims [0,16) follow t only, [16,72) h only, [72,128) w only
    rng = np.random.default_rng(1)
    x = rng.standard_normal(128)
    base = oracle.rope_rotate_f64(x, [2.0, 3.0, 4.0])
    only_t = oracle.rope_rotate_f64(x, [9.0, 3.0, 4.0])
    only_h = oracle.rope_rotate_f64(x, [2.0, 9.0, 4.0])
    only_w = oracle.rope_rotate_f64(x, [2.0, 3.0, 9.0])
    changed = lambda a: set(np.nonzero(np.abs(a - base) > 1e-12)[0].tolist())
    assert changed(only_t) <= set(range(0, 16)) and len(changed(only_t)) > 8
    assert changed(only_h) <= set(range(16, 72)) and len(changed(only_h)) > 40
    assert changed(only_w) <= set(range(72, 128)) and len(changed(only_w)) > 40


def test_rope_position_zero_is_identity_and_pairs_keep_their_norm():
    rng = np.random.default_rng(2)
    x = rng.standard_normal(128)
    assert np.array_equal(oracle.rope_rotate_f64(x, [0, 0, 0]), x)
    xf = x.astype(np.float32)
    assert np.array_equal(oracle.rope_rotate_f32(xf, [0, 0, 0]), xf)
    y = oracle.rope_rotate_f64(x, [13, 5, 29])
    np.testing.assert_allclose(np.hypot(y[0::2], y[1::2]), np.hypot(x[0::2], x[1::2]), rtol=1e-14)


def test_rope_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(3)
    for _ in range(20):
        q, k = rng.standard_normal(128), rng.standard_normal(128)
        p = rng.integers(0, 50, 3).astype(np.float64)
        pp = rng.integers(0, 50, 3).astype(np.float64)
        shift = rng.integers(-20, 300, 3).astype(np.float64)
        a = oracle.rope_rotate_f64(q, p) @ oracle.rope_rotate_f64(k, pp)
        b = oracle.rope_rotate_f64(q, p + shift) @ oracle.rope_rotate_f64(k, pp + shift)
        assert a == pytest.approx(b, rel=1e-11, abs=1e-11)


def test_rope_f32_commit_expression_is_exact():
    """y0 = fma(x0, c, -rn(x1*s)), y1 = fma(x0, s, rn(x1*c)), checked with exact rationals."""
    rng = np.random.default_rng(4)
    for _ in range(40):
        xb = synth.f32_to_bf16_bits(rng.standard_normal(128).astype(np.float32) * 3)
        x = synth.bf16_bits_to_f32(xb)
        pos = rng.integers(0, 400, 3).astype(np.float64)
        y = oracle.rope_rotate_f32(x, pos)
        for p in range(64):
            ax, d, j = axis_of_pair(p)
            c, s = oracle.rope_cs_f32(d, j, pos[ax])
            x0, x1 = F(x[2 * p]), F(x[2 * p + 1])
            x1s = round_f32(x1 * F(s))
            x1c = round_f32(x1 * F(c))
            assert y[2 * p] == round_f32(x0 * F(c) - F(x1s))
            assert y[2 * p + 1] == round_f32(x0 * F(s) + F(x1c))


# ----------------------------------------------------------------------------
# BF16 rounding and INT8 quantisation
# ----------------------------------------------------------------------------

def test_bf16_rounding_ties_go_to_even():
    # 1 + 2^-8 lies halfway between bf16 1.0 (0x3F80) and 1 + 2^-7 (0x3F81): even is 0x3F80
    assert oracle.f32_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3*2^-8 lies halfway between 0x3F81 and 0x3F82: even is 0x3F82
    assert oracle.f32_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert oracle.f32_to_bf16(-(1.0 + 2.0 ** -8)) == 0xBF80
    assert oracle.f32_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -20) == 0x3F81  # above the tie
    rng = np.random.default_rng(5)
    for v in rng.standard_normal(2000).astype(np.float32):
        b = oracle.f32_to_bf16(v)
        lo = np.array([b & 0xFFFF], np.uint16)
        assert abs(float(synth.bf16_bits_to_f32(lo)[0]) - float(v)) <= abs(float(v)) * 2.0 ** -8


def test_quantize_codes_range_absmax_and_error_bound():
    rng = np.random.default_rng(6)
    for _ in range(200):
        x = (rng.standard_normal(128) * rng.uniform(0.01, 50)).astype(np.float32)
        code, scale = oracle.quantize_row(x)
        amax = np.abs(x).max()
        assert scale == round_f32(F(amax) / 127)           # IEEE fp32 division
        assert code.min() >= -127 and code.max() <= 127
        i = int(np.argmax(np.abs(x)))
        assert code[i] == (127 if x[i] > 0 else -127)
        err = np.abs(code.astype(np.float64) * float(scale) - x.astype(np.float64))
        assert err.max() <= float(scale) / 2 * (1 + 1e-6)
        # every code is the round-half-even of the exact fp32 quotient
        for e in range(0, 128, 17):
            qt = round_f32(F(x[e]) / F(scale))
            assert code[e] == np.clip(np.rint(qt), -127, 127)


def test_quantize_ties_round_half_to_even():
    x = np.zeros(128, np.float32)
    x[0] = 127 * 2.0 ** -4          # absmax -> scale exactly 2^-4
    halves = [0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 125.5, -126.5]
    want = [0, 2, 2, 0, -2, -2, 126, -126]
    for i, hv in enumerate(halves):
        x[1 + i] = hv * 2.0 ** -4
    code, scale = oracle.quantize_row(x)
    assert scale == np.float32(2.0 ** -4)
    assert code[0] == 127
    assert code[1:1 + len(halves)].tolist() == want


def test_quantize_zero_row():
    code, scale = oracle.quantize_row(np.zeros(128, np.float32))
    assert scale == 0.0 and not code.any()


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------

def _empty_cache(heads=2, gh=2, gw=2, mode=oracle.MODE_BF16, window=0, cap=4):
    return oracle.OracleCache(mode, heads, gh, gw, window, cap)


def test_single_key_returns_v_exactly():
    c = _empty_cache()
    geo = synth.Geometry(2, 2, 2)
    q, k, v = synth.segment_qkv(geo, 0, 1, seed=11)
    out, lse = c.seg_attn(q, k, v, 0, 1)
    assert np.array_equal(out[0], bf16_vals(v[0]))
    s = bf16_vals(q[0]) * bf16_vals(k[0])
    np.testing.assert_allclose(lse[:, 0], s.sum(-1) / math.sqrt(128), rtol=1e-13)


def test_two_keys_closed_form():
    c = _empty_cache()
    geo = synth.Geometry(2, 2, 2)
    q, k, v = synth.segment_qkv(geo, 0, 2, seed=12)
    out, _ = c.seg_attn(q, k, v, 0, 2)
    for h in range(2):
        for i in range(2):
            s0 = float(np.dot(bf16_vals(q[i, h]), bf16_vals(k[0, h]))) / math.sqrt(128)
            s1 = float(np.dot(bf16_vals(q[i, h]), bf16_vals(k[1, h]))) / math.sqrt(128)
            w0 = 1.0 / (1.0 + math.exp(s1 - s0))
            want = w0 * bf16_vals(v[0, h]) + (1 - w0) * bf16_vals(v[1, h])
            np.testing.assert_allclose(out[i, h], want, rtol=1e-12, atol=1e-14)


def test_constant_values_give_constant_output():
    c = _empty_cache(heads=1)
    geo = synth.Geometry(1, 2, 2)
    q, k, v = synth.segment_qkv(geo, 2, 3, seed=13)
    v[:] = v[0, 0]
    out, _ = c.seg_attn(q, k, v, 2, 3)
    np.testing.assert_allclose(out, np.broadcast_to(bf16_vals(v[0, 0]), out.shape), rtol=1e-14)


def _rotated_segment(x, nv_frames, n_text, t0, gh, gw):
    """fp64 rotation of a segment's tokens with oracle.rope_rotate_f64 (pinned above)."""
    n, H, _ = x.shape
    out = bf16_vals(x).copy()
    F_ = gh * gw
    for i in range(nv_frames * F_):
        pos = [t0 + i // F_, (i % F_) // gw, (i % F_) % gw]
        for h in range(H):
            out[i, h] = oracle.rope_rotate_f64(out[i, h], pos)
    return out


@pytest.mark.parametrize("mode", [oracle.MODE_BF16, oracle.MODE_INT8])
def test_brute_force_softmax_long_double(mode):
    w = synth.WORKLOADS["tiny"]
    c = oracle.OracleCache(mode, w["heads"], w["grid_h"], w["grid_w"], 0, 4)
    oracle.build_history(c, [1, 1], seed=21)
    geo = synth.Geometry(w["heads"], w["grid_h"], w["grid_w"])
    q, k, v = synth.segment_qkv(geo, 1, 5, seed=22)
    out, lse = c.seg_attn(q, k, v, 1, 5)
    kc, vc = c.dequantized()
    nc = c.visible_cache_tokens()
    qr = _rotated_segment(q, 1, 5, c.frames_committed, w["grid_h"], w["grid_w"])
    kr = _rotated_segment(k, 1, 5, c.frames_committed, w["grid_h"], w["grid_w"])
    vv = bf16_vals(v)
    for h in range(w["heads"]):
        keys = np.concatenate([kc[h, :nc], kr[:, h]]).astype(np.longdouble)
        vals = np.concatenate([vc[h, :nc], vv[:, h]]).astype(np.longdouble)
        for i in range(q.shape[0]):
            s = keys @ qr[i, h].astype(np.longdouble) / np.sqrt(np.longdouble(128))
            e = np.exp(s)  # no max subtraction: scores are small here
            want = (e[:, None] * vals).sum(0) / e.sum()
            np.testing.assert_allclose(out[i, h], want.astype(np.float64), rtol=1e-12, atol=1e-13)
            assert lse[h, i] == pytest.approx(float(np.log(e.sum())), rel=1e-12, abs=1e-12)


def test_permuting_cache_tokens_leaves_output_unchanged():
    w = synth.WORKLOADS["tiny"]
    c = oracle.OracleCache(oracle.MODE_INT8, w["heads"], w["grid_h"], w["grid_w"], 3, 3)
    oracle.build_history(c, [2, 2], seed=31)  # 4 frames through a 3-frame window: ring has wrapped
    geo = synth.Geometry(w["heads"], w["grid_h"], w["grid_w"])
    q, k, v = synth.segment_qkv(geo, 1, 4, seed=32)
    ref, _ = c.seg_attn(q, k, v, 1, 4)
    rng = np.random.default_rng(0)
    perm = rng.permutation(c.k_code.shape[1])
    c.k_code[:] = c.k_code[:, perm]
    c.v_code[:] = c.v_code[:, perm]
    c.k_scale[:] = c.k_scale[:, perm]
    c.v_scale[:] = c.v_scale[:, perm]
    out, _ = c.seg_attn(q, k, v, 1, 4)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------
# causality, cache equivalence, sliding window
# ----------------------------------------------------------------------------

def _session(geo, frames, texts, seed):
    return [synth.segment_qkv(geo, nf, nt, seed, segment=s) + (nf, nt) for s, (nf, nt) in
            enumerate(zip(frames, texts))]


def _incremental(mode, geo, segs, target, window, cap):
    c = oracle.OracleCache(mode, geo.heads, geo.grid_h, geo.grid_w, window, cap)
    F_ = geo.tokens_per_frame
    for s in range(target):
        q, k, v, nf, nt = segs[s]
        c.commit(k[:nf * F_], v[:nf * F_], nf)
    q, k, v, nf, nt = segs[target]
    return c.seg_attn(q, k, v, nf, nt), c


def test_incremental_cache_equals_masked_full_sequence():
    geo = synth.Geometry(2, 3, 4)
    segs = _session(geo, [2, 1, 3, 2], [5, 0, 3, 4], seed=41)
    for target in range(4):
        (out, lse), _ = _incremental(oracle.MODE_F64, geo, segs, target, 0, 16)
        ref, ref_lse = oracle.full_seq_attn(segs, 2, 3, 4, 0, target)
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_later_segments_do_not_change_earlier_outputs():
    geo = synth.Geometry(2, 3, 4)
    segs = _session(geo, [2, 2, 2], [3, 3, 3], seed=42)
    ref, _ = oracle.full_seq_attn(segs, 2, 3, 4, 0, 1)
    q, k, v, nf, nt = segs[2]
    segs[2] = (q ^ 0x1234, k ^ 0x0F0F, v ^ 0x00FF, nf, nt)
    out, _ = oracle.full_seq_attn(segs, 2, 3, 4, 0, 1)
    assert np.array_equal(out, ref)
    # while a change inside the visible history does change the output
    q, k, v, nf, nt = segs[0]
    segs[0] = (q, k ^ 0x0040, v, nf, nt)
    out2, _ = oracle.full_seq_attn(segs, 2, 3, 4, 0, 1)
    assert not np.allclose(out2, ref)


def test_sliding_window_keeps_exactly_the_last_frames():
    W = 4
    geo = synth.Geometry(2, 2, 3)
    c = oracle.OracleCache(oracle.MODE_INT8, 2, 2, 3, W, W)
    total = 0
    for s, nf in enumerate([3, 2, 5, 1, 4, 7]):
        k, v = synth.history_kv(geo, nf, 51, s)
        c.commit(k, v, nf)
        total += nf
        held = sorted(int(f) for f in c.slot_frame if f >= 0)
        assert held == list(range(max(0, total - W), total))
        assert c.valid_frames == min(total, W) and c.frames_committed == total
        for slot, f in enumerate(c.slot_frame):
            if f >= 0:
                assert f % W == slot


def test_sliding_window_attention_equals_explicit_last_frames():
    W = 3
    geo = synth.Geometry(2, 2, 3)
    frames, texts = [2, 2, 3, 1, 2], [2, 2, 2, 2, 5]
    segs = _session(geo, frames, texts, seed=52)
    for target in [1, 2, 3, 4]:
        (out, lse), c = _incremental(oracle.MODE_F64, geo, segs, target, W, W)
        ref, ref_lse = oracle.full_seq_attn(segs, 2, 2, 3, W, target)
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
        assert c.visible_cache_tokens() == min(sum(frames[:target]), W) * geo.tokens_per_frame


@pytest.mark.parametrize("mode,tol", [(oracle.MODE_BF16, 1e-2), (oracle.MODE_INT8, 3e-2)])
def test_stored_cache_modes_stay_close_to_exact_history(mode, tol):
    """BF16 / INT8 storage differs from the exact fp64 cache only by storage rounding."""
    geo = synth.Geometry(2, 4, 8)
    segs = _session(geo, [2, 2, 2], [16, 16, 16], seed=61)
    (ref, _), _ = _incremental(oracle.MODE_F64, geo, segs, 2, 0, 8)
    (out, _), _ = _incremental(mode, geo, segs, 2, 0, 8)
    rel = np.linalg.norm(out - ref) / np.linalg.norm(ref)
    assert rel < tol
    assert rel > 0


def test_commit_stores_rotated_quantised_rows_at_their_slots():
    """Composition check of commit: slot, head and token position of each stored row."""
    geo = synth.Geometry(3, 2, 3)
    W = 2
    c = oracle.OracleCache(oracle.MODE_INT8, 3, 2, 3, W, W)
    k0, v0 = synth.history_kv(geo, 1, 71, 0)
    c.commit(k0, v0, 1)
    k1, v1 = synth.history_kv(geo, 2, 71, 1)
    c.commit(k1, v1, 2)  # frames 1, 2 -> slots 1, 0
    F_ = geo.tokens_per_frame
    for fi, frame in enumerate([1, 2]):
        slot = frame % W
        for r in range(F_):
            n = fi * F_ + r
            pos = [frame, r // 3, r % 3]
            for h in range(3):
                rk = oracle.rope_rotate_f32(synth.bf16_bits_to_f32(k1[n, h]), pos)
                code, scale = oracle.quantize_row(rk)
                assert np.array_equal(c.k_code[h, slot * F_ + r], code)
                assert c.k_scale[h, slot * F_ + r] == scale
                vcode, vscale = oracle.quantize_row(synth.bf16_bits_to_f32(v1[n, h]))
                assert np.array_equal(c.v_code[h, slot * F_ + r], vcode)
                assert c.v_scale[h, slot * F_ + r] == vscale


def test_full_history_overflow_is_rejected():
    geo = synth.Geometry(1, 1, 2)
    c = oracle.OracleCache(oracle.MODE_BF16, 1, 1, 2, 0, 3)
    k, v = synth.history_kv(geo, 2, 81, 0)
    c.commit(k, v, 2)
    k, v = synth.history_kv(geo, 2, 81, 1)
    with pytest.raises(ValueError):
        c.commit(k, v, 2)
