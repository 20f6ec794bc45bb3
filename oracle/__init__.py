"""Python handle on the CPU oracle (``oracle/nomas_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library in
``segment_causal_kv_b200/``. The C source is compiled here with gcc into
``oracle/liboracle.so`` (``build()``), with ``-ffp-contract=off`` so that the
fp32 commit expression is evaluated exactly as written.

What each C function follows is cited in the C file's header; the readings
taken where the pages are silent are listed there.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nomas_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

MODE_BF16, MODE_INT8, MODE_F64 = 0, 1, 2
HEAD_DIM = 128


def build(force: bool = False) -> str:
    """Compile the oracle into a shared library with the host C compiler."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


class _OrcCache(ctypes.Structure):
    _fields_ = [
        ("mode", ctypes.c_int32),
        ("heads", ctypes.c_int32),
        ("grid_h", ctypes.c_int32),
        ("grid_w", ctypes.c_int32),
        ("window_frames", ctypes.c_int32),
        ("capacity_frames", ctypes.c_int32),
        ("theta", ctypes.c_double),
        ("k_bf16", ctypes.c_void_p),
        ("v_bf16", ctypes.c_void_p),
        ("k_code", ctypes.c_void_p),
        ("v_code", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p),
        ("k_f64", ctypes.c_void_p),
        ("v_f64", ctypes.c_void_p),
        ("slot_frame", ctypes.c_void_p),
        ("frames_committed", ctypes.c_int64),
        ("valid_frames", ctypes.c_int32),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        _lib.orc_cache_reset.argtypes = [ctypes.POINTER(_OrcCache)]
        _lib.orc_commit.argtypes = [ctypes.POINTER(_OrcCache), P, P, ctypes.c_int64, ctypes.c_int]
        _lib.orc_seg_attn.argtypes = [ctypes.POINTER(_OrcCache), P, P, P, ctypes.c_int64, ctypes.c_int,
                                      ctypes.c_int, P, ctypes.c_int64, P, P, ctypes.c_int]
        _lib.orc_visible_cache_tokens.argtypes = [ctypes.POINTER(_OrcCache)]
        _lib.orc_visible_cache_tokens.restype = ctypes.c_int64
        _lib.orc_full_seq_attn.argtypes = [ctypes.c_int, P, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_int, P, P,
                                           ctypes.c_int]
        _lib.orc_rope_angle.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double]
        _lib.orc_rope_angle.restype = ctypes.c_double
        _lib.orc_rope_cs_f32.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double, P, P]
        _lib.orc_rope_rotate_f64.argtypes = [P, P, ctypes.c_double, P]
        _lib.orc_rope_rotate_f32.argtypes = [P, P, ctypes.c_double, P]
        _lib.orc_quantize_row.argtypes = [P, P, P]
        _lib.orc_camera_attn.argtypes = [P, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P,
                                         ctypes.c_int, ctypes.c_int, P]
        _lib.orc_f32_to_bf16.argtypes = [ctypes.c_float]
        _lib.orc_f32_to_bf16.restype = ctypes.c_uint16
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


class OracleCache:
    """Host mirror of one layer's K/V cache, committed by the oracle's rules."""

    def __init__(self, mode: int, heads: int, grid_h: int, grid_w: int, window: int, capacity: int,
                 theta: float = 256.0):
        self.mode, self.heads, self.grid_h, self.grid_w = mode, heads, grid_h, grid_w
        self.window, self.capacity, self.theta = window, capacity, float(theta)
        F = grid_h * grid_w
        rows = heads * capacity * F
        self.k_bf16 = self.v_bf16 = self.k_code = self.v_code = None
        self.k_scale = self.v_scale = self.k_f64 = self.v_f64 = None
        if mode == MODE_BF16:
            self.k_bf16 = np.zeros((heads, capacity * F, HEAD_DIM), np.uint16)
            self.v_bf16 = np.zeros_like(self.k_bf16)
        elif mode == MODE_INT8:
            self.k_code = np.zeros((heads, capacity * F, HEAD_DIM), np.int8)
            self.v_code = np.zeros_like(self.k_code)
            self.k_scale = np.zeros((heads, capacity * F), np.float32)
            self.v_scale = np.zeros_like(self.k_scale)
        elif mode == MODE_F64:
            self.k_f64 = np.zeros((heads, capacity * F, HEAD_DIM), np.float64)
            self.v_f64 = np.zeros_like(self.k_f64)
        else:
            raise ValueError(mode)
        del rows
        self.slot_frame = np.full(capacity, -1, np.int64)
        self._c = _OrcCache(mode, heads, grid_h, grid_w, window, capacity, self.theta,
                            _ptr(self.k_bf16), _ptr(self.v_bf16), _ptr(self.k_code), _ptr(self.v_code),
                            _ptr(self.k_scale), _ptr(self.v_scale), _ptr(self.k_f64), _ptr(self.v_f64),
                            _ptr(self.slot_frame), 0, 0)
        rc = lib().orc_cache_reset(ctypes.byref(self._c))
        if rc != 0:
            raise ValueError(f"oracle cache reset rejected the descriptor ({rc})")

    @property
    def tokens_per_frame(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def frames_committed(self) -> int:
        return int(self._c.frames_committed)

    @property
    def valid_frames(self) -> int:
        return int(self._c.valid_frames)

    def visible_cache_tokens(self) -> int:
        return int(lib().orc_visible_cache_tokens(ctypes.byref(self._c)))

    def commit(self, k_bits: np.ndarray, v_bits: np.ndarray, n_frames: int) -> None:
        k_bits = np.ascontiguousarray(k_bits, np.uint16)
        v_bits = np.ascontiguousarray(v_bits, np.uint16)
        assert k_bits.shape == (n_frames * self.tokens_per_frame, self.heads, HEAD_DIM)
        rc = lib().orc_commit(ctypes.byref(self._c), _ptr(k_bits), _ptr(v_bits), self.heads * HEAD_DIM, n_frames)
        if rc != 0:
            raise ValueError(f"oracle commit rejected ({rc})")

    def seg_attn(self, q, k, v, n_video_frames: int, n_text: int, rows=None, nthreads: int | None = None):
        """fp64 attention. Returns (out [n_rows][H][128], lse [H][n_rows]), natural-log LSE."""
        q = np.ascontiguousarray(q, np.uint16)
        k = np.ascontiguousarray(k, np.uint16)
        v = np.ascontiguousarray(v, np.uint16)
        nq = n_video_frames * self.tokens_per_frame + n_text
        assert q.shape == (nq, self.heads, HEAD_DIM) and k.shape == q.shape and v.shape == q.shape
        if rows is None:
            n_rows, rows_arr = nq, None
        else:
            rows_arr = np.ascontiguousarray(rows, np.int64)
            assert rows_arr.min(initial=0) >= 0 and rows_arr.max(initial=0) < max(nq, 1)
            n_rows = len(rows_arr)
        out = np.zeros((n_rows, self.heads, HEAD_DIM), np.float64)
        lse = np.zeros((self.heads, n_rows), np.float64)
        rc = lib().orc_seg_attn(ctypes.byref(self._c), _ptr(q), _ptr(k), _ptr(v), self.heads * HEAD_DIM,
                                n_video_frames, n_text, _ptr(rows_arr), n_rows, _ptr(out), _ptr(lse),
                                nthreads or default_threads())
        if rc != 0:
            raise MemoryError(f"oracle attention failed ({rc})")
        return out, lse

    def window_frames(self) -> list[int]:
        """Absolute indices of the frames the cache holds now, read from the slots' frame labels.

        A frame leaves the window exactly when a commit overwrites its slot, so the
        frames a commit evicts are window_frames() before it minus window_frames() after it."""
        return sorted(int(f) for f in self.slot_frame if f >= 0)

    def frame_rows(self, f: int):
        """Stored rows of absolute frame f: (k, v, k_scale, v_scale) as [H][F][128] codes or
        BF16 bits and [H][F] fp32 scales (None in BF16 mode), copied."""
        slots = np.nonzero(self.slot_frame == f)[0]
        if len(slots) != 1:
            raise KeyError(f)
        F = self.tokens_per_frame
        r = slice(int(slots[0]) * F, (int(slots[0]) + 1) * F)
        if self.mode == MODE_INT8:
            return (self.k_code[:, r].copy(), self.v_code[:, r].copy(), self.k_scale[:, r].copy(),
                    self.v_scale[:, r].copy())
        if self.mode == MODE_BF16:
            return self.k_bf16[:, r].copy(), self.v_bf16[:, r].copy(), None, None
        return self.k_f64[:, r].copy(), self.v_f64[:, r].copy(), None, None

    def dequantized(self):
        """fp64 K and V of every slot row, [H][cap*F][128] (oracle dequantisation rule)."""
        if self.mode == MODE_BF16:
            f = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
            return f(self.k_bf16), f(self.v_bf16)
        if self.mode == MODE_INT8:
            return (self.k_code.astype(np.float64) * self.k_scale[..., None].astype(np.float64),
                    self.v_code.astype(np.float64) * self.v_scale[..., None].astype(np.float64))
        return self.k_f64.copy(), self.v_f64.copy()


def camera_attn(q, n_frames: int, tpf: int, k_cam, v_cam, chunk_frames: int = 1) -> np.ndarray:
    """fp64 per-latent-frame camera cross-attention (orc_camera_attn).

    q: BF16 bits [n_frames * tpf][heads][128] (video tokens); k_cam, v_cam: BF16 bits
    [n_chunks][n_cam][heads][128]. Returns out [n_frames * tpf][heads][128] fp64."""
    q = np.ascontiguousarray(q, np.uint16)
    k_cam = np.ascontiguousarray(k_cam, np.uint16)
    v_cam = np.ascontiguousarray(v_cam, np.uint16)
    heads = q.shape[1]
    n_chunks, n_cam = k_cam.shape[0], k_cam.shape[1]
    assert q.shape == (n_frames * tpf, heads, HEAD_DIM) and v_cam.shape == k_cam.shape
    assert k_cam.shape[2:] == (heads, HEAD_DIM) and n_chunks == -(-n_frames // chunk_frames)
    out = np.zeros(q.shape, np.float64)
    rc = lib().orc_camera_attn(_ptr(q), heads * HEAD_DIM, n_frames, tpf, heads, _ptr(k_cam), _ptr(v_cam), n_cam,
                               chunk_frames, _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle camera attention rejected its arguments ({rc})")
    return out


def full_seq_attn(segments, heads: int, grid_h: int, grid_w: int, window: int, target: int,
                  theta: float = 256.0, nthreads: int | None = None):
    """Masked full-sequence attention of segment ``target`` (no cache involved).

    ``segments``: list of (q, k, v, n_video_frames, n_text) with BF16 bits
    token-major [N_s][heads][128]. Returns (out [N_target][H][128], lse [H][N_target]).
    """
    n = len(segments)
    keep = [tuple(np.ascontiguousarray(a, np.uint16) for a in s[:3]) for s in segments]
    arr = lambda i: (ctypes.c_void_p * n)(*[keep[s][i].ctypes.data for s in range(n)])
    nv = np.array([s[3] for s in segments], np.int32)
    nt = np.array([s[4] for s in segments], np.int32)
    nq = int(nv[target]) * grid_h * grid_w + int(nt[target])
    out = np.zeros((nq, heads, HEAD_DIM), np.float64)
    lse = np.zeros((heads, nq), np.float64)
    qa, ka, va = arr(0), arr(1), arr(2)
    rc = lib().orc_full_seq_attn(n, ctypes.cast(qa, ctypes.c_void_p), ctypes.cast(ka, ctypes.c_void_p),
                                 ctypes.cast(va, ctypes.c_void_p), _ptr(nv), _ptr(nt), heads, grid_h, grid_w,
                                 float(theta), window, target, _ptr(out), _ptr(lse), nthreads or default_threads())
    if rc != 0:
        raise MemoryError(f"oracle full-sequence attention failed ({rc})")
    return out, lse


def rope_angle(d: int, j: int, pos: float, theta: float = 256.0) -> float:
    return float(lib().orc_rope_angle(d, j, float(pos), float(theta)))


def rope_cs_f32(d: int, j: int, pos: float, theta: float = 256.0):
    c = np.zeros(1, np.float32)
    s = np.zeros(1, np.float32)
    lib().orc_rope_cs_f32(d, j, float(pos), float(theta), _ptr(c), _ptr(s))
    return c[0], s[0]


def rope_rotate_f64(x: np.ndarray, pos, theta: float = 256.0) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float64)
    p = np.ascontiguousarray(pos, np.float64)
    y = np.zeros(HEAD_DIM, np.float64)
    lib().orc_rope_rotate_f64(_ptr(x), _ptr(p), float(theta), _ptr(y))
    return y


def rope_rotate_f32(x: np.ndarray, pos, theta: float = 256.0) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32)
    p = np.ascontiguousarray(pos, np.float64)
    y = np.zeros(HEAD_DIM, np.float32)
    lib().orc_rope_rotate_f32(_ptr(x), _ptr(p), float(theta), _ptr(y))
    return y


def quantize_row(x: np.ndarray):
    x = np.ascontiguousarray(x, np.float32)
    code = np.zeros(HEAD_DIM, np.int8)
    scale = np.zeros(1, np.float32)
    lib().orc_quantize_row(_ptr(x), _ptr(code), _ptr(scale))
    return code, scale[0]


def f32_to_bf16(x: float) -> int:
    """BF16 bits of an fp32 value by the oracle's round-half-to-even rule."""
    return int(lib().orc_f32_to_bf16(float(np.float32(x))))


def build_history(cache: OracleCache, commits, seed: int, kv_std: float = 1.0):
    """Commit synthetic finished segments (synth.history_kv) into ``cache``."""
    import synth
    geo = synth.Geometry(cache.heads, cache.grid_h, cache.grid_w)
    for s, nf in enumerate(commits):
        k, v = synth.history_kv(geo, nf, seed, s, kv_std)
        cache.commit(k, v, nf)
