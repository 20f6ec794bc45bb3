"""C ABI checks that need no GPU: the library loads, exports every function
include/nomas.h declares, agrees with the header on the descriptor layout,
and rejects bad arguments on the host before any CUDA call."""

import ctypes
import os
import re
import subprocess

import pytest

import segment_causal_kv_b200 as nm
from segment_causal_kv_b200 import build as nm_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "nomas.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    nm_build.build()
    yield


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nomas_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(nm.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = nm.lib()
    for name in declared_functions():
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", nm.LIB_PATH], capture_output=True, text=True).stdout
    for name in declared_functions():
        assert re.search(rf"\bT {name}$", out, re.M), name


def test_descriptor_layout_matches_the_header(tmp_path):
    fields = [f for f, _ in nm.NomasCacheDesc._fields_]
    src = tmp_path / "probe.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "nomas.h"\nint main(void){\n'
                   + "".join(f'printf("%zu\\n", offsetof(nomas_cache, {f}));\n' for f in fields)
                   + 'printf("%zu\\n", sizeof(nomas_cache));\nreturn 0;}\n')
    exe = tmp_path / "probe"
    subprocess.check_call(["gcc", "-std=c11", "-I", os.path.join(ROOT, "include"), "-o", str(exe), str(src)])
    got = [int(x) for x in subprocess.check_output([str(exe)]).split()]
    want = [getattr(nm.NomasCacheDesc, f).offset for f in fields] + [ctypes.sizeof(nm.NomasCacheDesc)]
    assert got == want


def test_status_strings():
    for code in range(-8, 1):
        s = nm.nomas_status_string(code)
        assert s.startswith("NOMAS_")
    assert "unknown" in nm.nomas_status_string(-99)


# fake device addresses: validation never dereferences them
FAKE = 0x7F0000000000


def desc(mode=nm.NOMAS_CACHE_INT8, heads=16, head_dim=128, gh=22, gw=40, window=18, cap=18, theta=256.0,
         k=FAKE, v=FAKE + (1 << 30), ks=FAKE + (2 << 30), vs=FAKE + (3 << 30)):
    if mode == nm.NOMAS_CACHE_BF16:
        ks = vs = None
    return nm.NomasCacheDesc(mode, heads, head_dim, gh, gw, window, cap, theta, k, v, ks, vs, 0, 0, 0, 0)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), nm.NOMAS_ERR_ARG),
    (dict(heads=0), nm.NOMAS_ERR_ARG),
    (dict(mode=7), nm.NOMAS_ERR_ARG),
    (dict(window=18, cap=20), nm.NOMAS_ERR_ARG),
    (dict(window=-1), nm.NOMAS_ERR_ARG),
    (dict(gh=60, gw=40), nm.NOMAS_ERR_ARG),
    (dict(theta=0.0), nm.NOMAS_ERR_ARG),
    (dict(ks=None), nm.NOMAS_ERR_ARG),
    (dict(k=None), nm.NOMAS_ERR_ARG),
    (dict(k=FAKE + 8), nm.NOMAS_ERR_ALIGN),
    (dict(vs=FAKE + 4), nm.NOMAS_ERR_ALIGN),
])
def test_reset_rejects_bad_descriptors(kw, code):
    assert nm.nomas_cache_reset(desc(**kw)) == code


def test_bf16_mode_must_not_carry_scales():
    d = desc(mode=nm.NOMAS_CACHE_BF16, window=0, cap=8)
    d.k_scale = FAKE
    assert nm.nomas_cache_reset(d) == nm.NOMAS_ERR_ARG


def test_reset_sets_state():
    d = desc()
    d.frames_committed, d.valid_frames, d.head_slot = 5, 3, 2
    assert nm.nomas_cache_reset(d) == nm.NOMAS_OK
    assert (d.frames_committed, d.valid_frames, d.head_slot) == (0, 0, 0)
    assert d.check != 0


def test_calls_on_an_unreset_or_changed_descriptor_fail():
    d = desc()
    assert nm.nomas_kv_commit(d, FAKE, FAKE, 2048, 3, None) == nm.NOMAS_ERR_STATE
    assert nm.nomas_seg_attn(d, FAKE, FAKE, FAKE, 2048, 3, 256, FAKE, None, FAKE, 1 << 30, None) == \
        nm.NOMAS_ERR_STATE
    assert nm.nomas_cache_reset(d) == nm.NOMAS_OK
    d.grid_w = 41  # configuration changed after reset
    assert nm.nomas_kv_commit(d, FAKE, FAKE, 2048, 3, None) == nm.NOMAS_ERR_STATE
    assert nm.nomas_seg_attn_workspace_bytes(d, 3, 256) == 0


def test_commit_argument_checks():
    d = desc()
    assert nm.nomas_cache_reset(d) == nm.NOMAS_OK
    assert nm.nomas_kv_commit(d, FAKE, FAKE, 2048, 0, None) == nm.NOMAS_OK  # no-op
    assert nm.nomas_kv_commit(d, FAKE, FAKE, 2048, -1, None) == nm.NOMAS_ERR_ARG
    assert nm.nomas_kv_commit(d, None, FAKE, 2048, 3, None) == nm.NOMAS_ERR_ARG
    assert nm.nomas_kv_commit(d, FAKE, FAKE, 2047, 3, None) == nm.NOMAS_ERR_ARG
    assert nm.nomas_kv_commit(d, FAKE, FAKE, 2052, 3, None) == nm.NOMAS_ERR_ARG
    assert nm.nomas_kv_commit(d, FAKE + 2, FAKE, 2048, 3, None) == nm.NOMAS_ERR_ALIGN
    assert d.frames_committed == 0  # nothing changed by the failed calls


def test_full_history_capacity_is_enforced_before_launch():
    d = desc(mode=nm.NOMAS_CACHE_BF16, window=0, cap=4)
    assert nm.nomas_cache_reset(d) == nm.NOMAS_OK
    assert nm.nomas_kv_commit(d, FAKE, FAKE, 2048, 5, None) == nm.NOMAS_ERR_CAPACITY
    assert d.frames_committed == 0


def test_seg_attn_argument_checks():
    d = desc()
    assert nm.nomas_cache_reset(d) == nm.NOMAS_OK
    need = nm.nomas_seg_attn_workspace_min_bytes(d, 3, 256)
    assert need > 2 * 16 * 2896 * 128 * 2  # holds at least rotated Q and K
    call = lambda **kw: nm.nomas_seg_attn(d, kw.get("q", FAKE), FAKE, FAKE, kw.get("ts", 2048), kw.get("nv", 3),
                                          kw.get("nt", 256), kw.get("out", FAKE), kw.get("lse", None),
                                          kw.get("ws", FAKE), kw.get("wsb", need), None)
    assert call(nv=0, nt=0) == nm.NOMAS_OK  # empty segment: nothing to do
    assert call(nv=-1) == nm.NOMAS_ERR_ARG
    assert call(q=None) == nm.NOMAS_ERR_ARG
    assert call(ts=1000) == nm.NOMAS_ERR_ARG
    assert call(out=FAKE + 8) == nm.NOMAS_ERR_ALIGN
    assert call(lse=FAKE + 2) == nm.NOMAS_ERR_ALIGN
    assert call(ws=None) == nm.NOMAS_ERR_WORKSPACE
    assert call(wsb=need - 1) == nm.NOMAS_ERR_WORKSPACE
    assert call(ws=FAKE + 16) == nm.NOMAS_ERR_ALIGN


def test_workspace_size_is_a_function_of_the_shape():
    d = desc()
    assert nm.nomas_cache_reset(d) == nm.NOMAS_OK
    a = nm.nomas_seg_attn_workspace_bytes(d, 3, 256)
    b = nm.nomas_seg_attn_workspace_bytes(d, 3, 256)
    assert a == b and a % 256 == 0
    assert nm.nomas_seg_attn_workspace_bytes(d, 6, 256) > a
    assert nm.nomas_seg_attn_workspace_bytes(d, -1, 0) == 0


def test_workspace_plans_between_the_minimum_and_the_full_size():
    d = desc()
    assert nm.nomas_cache_reset(d) == nm.NOMAS_OK
    d.valid_frames = 18  # as after 18 committed frames (state is not part of the stamp)
    full = nm.nomas_seg_attn_workspace_bytes(d, 3, 256)
    low = nm.nomas_seg_attn_workspace_min_bytes(d, 3, 256)
    # the minimum is the one-split plan: the 256-byte status header, the rotated FP16 Q
    # and K (16 heads x 2896 tokens x 256 B each), the tile records (16 heads x (124
    # cache + 23 current tiles) x 16 B) and the Q row factors (16 x 2896 x 4 B), each
    # rounded up to 256 bytes
    up = lambda x: -(-x // 256) * 256
    qk = up(16 * 2896 * 128 * 2)
    assert low == 256 + 2 * qk + up(16 * (124 + 23) * 16) + up(16 * 2896 * 4)
    # the full plan adds the FP16 copy of the INT8 window (2 x 16 heads x 15,840 tokens x
    # 256 B) and the KV-split partials: per split, 16 heads x 12 Q-tile pairs x 256 rows
    # of 128 FP16 values and an fp32 (max, sum, 2^e, 0) record, and one counter per unit
    copy = 2 * 16 * 18 * 880 * 256
    per_split = 16 * 12 * 256 * (128 * 2 + 16)
    assert full - low >= copy + 2 * per_split and full % 256 == 0
    call = lambda wsb: nm.nomas_seg_attn(d, FAKE, FAKE, FAKE, 2048, 3, 256, FAKE, None, FAKE, wsb, None)
    assert call(low - 1) == nm.NOMAS_ERR_WORKSPACE
    # the minimum, the full size and any size in between (a plan with fewer splits)
    # pass validation; without a GPU the call then stops at the device check
    for wsb in (low, (low + full) // 2, full):
        assert call(wsb) in (nm.NOMAS_ERR_DEVICE, nm.NOMAS_ERR_CUDA)


def test_layered_commit_argument_checks():
    ds = [desc(k=FAKE + (i << 32), v=FAKE + (i << 32) + (1 << 30), ks=FAKE + (i << 32) + (2 << 30),
               vs=FAKE + (i << 32) + (3 << 30)) for i in range(3)]
    for d in ds:
        assert nm.nomas_cache_reset(d) == nm.NOMAS_OK
    ptrs = [FAKE] * 3
    c = lambda dd, k=ptrs, v=ptrs, ts=2048, nf=3: nm.nomas_kv_commit_layers(dd, k, v, ts, nf, None)
    assert c(ds, nf=0) == nm.NOMAS_OK  # no-op
    assert c(ds, nf=-1) == nm.NOMAS_ERR_ARG
    assert c([ds[0], ds[1], ds[0]]) == nm.NOMAS_ERR_ARG  # one cache twice
    assert c(ds, k=[FAKE, None, FAKE]) == nm.NOMAS_ERR_ARG
    assert c(ds, v=[FAKE, FAKE, FAKE + 8]) == nm.NOMAS_ERR_ALIGN
    assert c(ds, ts=2052) == nm.NOMAS_ERR_ARG
    ds[2].grid_w = 41  # changed configuration: the stamp no longer matches
    assert c(ds) == nm.NOMAS_ERR_STATE
    ds[2].grid_w = 40
    ds[1].valid_frames = 2  # same configuration, different ring state
    assert c(ds) == nm.NOMAS_ERR_STATE
    ds[1].valid_frames = 0
    other = desc(window=9, cap=9, k=FAKE + (7 << 32))
    assert nm.nomas_cache_reset(other) == nm.NOMAS_OK
    assert c([ds[0], other, ds[2]]) == nm.NOMAS_ERR_STATE
    assert all(d.frames_committed == 0 for d in ds)
    assert nm.nomas_kv_commit_layers([], [], [], 2048, 3, None) == nm.NOMAS_ERR_ARG


def test_camera_attn_argument_checks():
    A = FAKE
    ok = dict(q=A, qs=16 * 128, nf=3, tpf=880, h=16, kc=A, vc=A, m=1, ch=1, o=A, os=16 * 128)

    def call(**kw):
        a = dict(ok, **kw)
        return nm.nomas_camera_attn(a["q"], a["qs"], a["nf"], a["tpf"], a["h"], a["kc"], a["vc"], a["m"], a["ch"],
                                    a["o"], a["os"], None)

    assert call(nf=0) == nm.NOMAS_OK  # nothing to do, no device touched
    assert call(nf=-1) == nm.NOMAS_ERR_ARG
    assert call(m=0) == nm.NOMAS_ERR_ARG
    assert call(m=4097) == nm.NOMAS_ERR_ARG
    assert call(ch=0) == nm.NOMAS_ERR_ARG
    assert call(h=0) == nm.NOMAS_ERR_ARG
    assert call(tpf=0) == nm.NOMAS_ERR_ARG
    assert call(q=None) == nm.NOMAS_ERR_ARG
    assert call(o=None) == nm.NOMAS_ERR_ARG
    assert call(qs=15 * 128) == nm.NOMAS_ERR_ARG
    assert call(os=16 * 128 - 8) == nm.NOMAS_ERR_ARG
    assert call(qs=16 * 128 + 4) == nm.NOMAS_ERR_ALIGN
    assert call(q=A + 8) == nm.NOMAS_ERR_ALIGN
    assert call(vc=A + 2) == nm.NOMAS_ERR_ALIGN
    assert call(nf=1 << 20, tpf=1 << 10, h=16) == nm.NOMAS_ERR_ARG  # rows beyond 31 bits


def test_div127_selftest_rejects_bad_pointers_before_any_cuda_call():
    assert nm.nomas_selftest_div127(None, None) == nm.NOMAS_ERR_ARG
    assert nm.nomas_selftest_div127(FAKE + 4, None) == nm.NOMAS_ERR_ARG
