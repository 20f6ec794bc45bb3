"""Seeded synthetic inputs shared by the oracle and the CUDA path.

This module only draws numbers. It holds none of the attention, RoPE or
quantisation arithmetic: both the CPU oracle (``oracle/``) and the CUDA
library (``segment_causal_kv_b200``) receive the very same BF16 bit patterns
from here, so a parity test compares two computations on identical bytes.

Generator (counter based, thread-count independent):

* SplitMix64 finaliser (Steele, Lea, Flood, "Fast splittable pseudorandom
  number generators", OOPSLA 2014; the 64-bit mix published with Java's
  ``SplittableRandom``) applied to ``key + (counter + 1) * golden_gamma``.
  ``key`` mixes the seed and a tensor id, so every tensor of a workload has
  its own stream and element ``i`` of a tensor never depends on how many
  elements were drawn before it.
* Box-Muller (Box and Muller, 1958) in double precision turns two uniforms
  (counters ``2i`` and ``2i+1``) into one standard normal.
* The normal is scaled by ``std``, rounded to fp32, then to BF16 with
  round-half-to-even: the library's inputs are BF16, so the fp32 draw of
  the small workload is consumed as its BF16 rounding by both sides.

Workload shapes follow the pages: 16 heads of 128 dims (model card
"Model Architecture" table), 22x40 = 880 tokens per latent frame at
704x1280 with 32x spatial compression (blog "Step 3: The Video Latent"),
an 18-frame history budget (model card "Single-GPU Low-Memory Inference").
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# tensor ids: one stream per role
TID_Q, TID_K, TID_V = 1, 2, 3
TID_HIST_K, TID_HIST_V = 4, 5
TID_CAM_K, TID_CAM_V = 6, 7


def _mix(z: np.ndarray) -> np.ndarray:
    z = z.astype(np.uint64, copy=True)
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def stream_key(seed: int, tensor_id: int, segment: int = 0) -> np.uint64:
    """Key of one tensor's stream: mix of (seed, tensor id, segment index)."""
    with np.errstate(over="ignore"):
        base = np.array([(seed * 0x100000001B3 + tensor_id * 0x1F123BB5 + segment * 0x5851F42D4C957F2D)
                         & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64)
        return _mix(base)[0]


def uniform_u64(key: np.uint64, start: int, n: int) -> np.ndarray:
    """64-bit outputs for counters start .. start+n-1 of the stream ``key``."""
    with np.errstate(over="ignore"):
        ctr = np.arange(start, start + n, dtype=np.uint64) + np.uint64(1)
        return _mix(key + ctr * _GAMMA)


def normal_f64(key: np.uint64, n: int) -> np.ndarray:
    """n standard normals (double) from counters 0 .. 2n-1."""
    r = uniform_u64(key, 0, 2 * n)
    r1, r2 = r[0::2], r[1::2]
    u1 = ((r1 >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)  # (0, 1]
    u2 = (r2 >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)          # [0, 1)
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """BF16 bit patterns (uint16) of fp32 values, round-half-to-even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_normal_numpy(seed: int, tensor_id: int, shape, std: float = 1.0, segment: int = 0) -> np.ndarray:
    """Pure-numpy statement of the generator (slow; the C version below is used)."""
    n = int(np.prod(shape))
    z = normal_f64(stream_key(seed, tensor_id, segment), n) * std
    return f32_to_bf16_bits(z.astype(np.float32)).reshape(shape)


_HERE = os.path.dirname(os.path.abspath(__file__))
_CLIB = None


def _clib():
    """gen.c compiled with gcc (same generator, multi-threaded)."""
    global _CLIB
    if _CLIB is None:
        src = os.path.join(_HERE, "gen.c")
        so = os.path.join(_HERE, "libsynth.so")
        if not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(src):
            tmp = so + f".{os.getpid()}.tmp"
            subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, src, "-lm", "-lpthread"])
            os.replace(tmp, so)
        lib = ctypes.CDLL(so)
        lib.synth_bf16_normal.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p,
                                          ctypes.c_int]
        _CLIB = lib
    return _CLIB


def bf16_normal(seed: int, tensor_id: int, shape, std: float = 1.0, segment: int = 0) -> np.ndarray:
    """BF16 bits (uint16 array of ``shape``) of N(0, std^2) draws."""
    n = int(np.prod(shape))
    out = np.empty(n, np.uint16)
    key = int(stream_key(seed, tensor_id, segment))
    _clib().synth_bf16_normal(key, n, float(std), out.ctypes.data_as(ctypes.c_void_p), os.cpu_count() or 1)
    return out.reshape(shape)


class Geometry:
    """Token geometry of one workload (heads x 128, grid_h x grid_w tokens per latent frame)."""

    def __init__(self, heads: int, grid_h: int, grid_w: int, head_dim: int = 128):
        self.heads, self.grid_h, self.grid_w, self.head_dim = heads, grid_h, grid_w, head_dim

    @property
    def tokens_per_frame(self) -> int:
        return self.grid_h * self.grid_w


def segment_qkv(geo: Geometry, n_video_frames: int, n_text: int, seed: int, segment: int = 0,
                q_std: float = 1.0, kv_std: float = 1.0):
    """Q, K, V BF16 bits, token-major [n_video*F + n_text][heads][128], video tokens first."""
    n = n_video_frames * geo.tokens_per_frame + n_text
    shape = (n, geo.heads, geo.head_dim)
    return (bf16_normal(seed, TID_Q, shape, q_std, segment),
            bf16_normal(seed, TID_K, shape, kv_std, segment),
            bf16_normal(seed, TID_V, shape, kv_std, segment))


def history_kv(geo: Geometry, n_frames: int, seed: int, segment: int, kv_std: float = 1.0):
    """K, V BF16 bits of a finished segment to commit, token-major [n_frames*F][heads][128]."""
    shape = (n_frames * geo.tokens_per_frame, geo.heads, geo.head_dim)
    return (bf16_normal(seed, TID_HIST_K, shape, kv_std, segment),
            bf16_normal(seed, TID_HIST_V, shape, kv_std, segment))


def camera_kv(geo: Geometry, n_chunks: int, n_cam: int, seed: int, segment: int = 0, std: float = 1.0):
    """Projected camera K, V BF16 bits [n_chunks][n_cam][heads][128] (n_cam tokens per camera chunk)."""
    shape = (n_chunks, n_cam, geo.heads, geo.head_dim)
    return (bf16_normal(seed, TID_CAM_K, shape, std, segment),
            bf16_normal(seed, TID_CAM_V, shape, std, segment))


# ---------------------------------------------------------------------------
# Workloads (shapes and value distributions from the pages)
# ---------------------------------------------------------------------------

WORKLOADS = {
    # correctness-sized: 2 heads, 4x8 grid, 2-frame segment + 16 text, 2-frame BF16 history
    "tiny": dict(heads=2, grid_h=4, grid_w=8, mode="bf16", window=0, capacity=4,
                 hist_commits=[2], cur_frames=2, n_text=16, seed=0, q_std=1.0, kv_std=1.0),
    # single-GPU configuration: 18-frame INT8 history built from six 3-frame commits
    "single_gpu_int8_18f": dict(heads=16, grid_h=22, grid_w=40, mode="int8", window=18, capacity=18,
                                hist_commits=[3] * 6, cur_frames=3, n_text=256, seed=1,
                                q_std=1.0, kv_std=1.0),
    # full-history BF16: four prior 72-frame segments, current 72 frames
    "full_history_bf16": dict(heads=16, grid_h=22, grid_w=40, mode="bf16", window=0, capacity=360,
                              hist_commits=[72] * 4, cur_frames=72, n_text=256, seed=2,
                              q_std=0.5, kv_std=1.0),
}


def sweep_workload(hist_frames: int) -> dict:
    """History sweep: INT8 cache whose window equals the history length."""
    commits = []
    left = hist_frames
    while left > 0:
        commits.append(min(3, left))
        left -= commits[-1]
    return dict(heads=16, grid_h=22, grid_w=40, mode="int8", window=hist_frames, capacity=hist_frames,
                hist_commits=commits, cur_frames=3, n_text=256, seed=3, q_std=1.0, kv_std=1.0)
