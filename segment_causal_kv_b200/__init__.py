"""Python binding of the sm_100a segment-causal attention library (``libnomas.so``).

Argument marshalling only: every step of the hot path runs in the library's
CUDA kernels, reached through the C ABI declared in ``include/nomas.h``. The
functions keep the C names (``nomas_cache_reset``, ``nomas_kv_commit``,
``nomas_seg_attn``, ...); ``KVCache`` is a convenience wrapper that owns the
cache tensors (PyTorch is used for device memory and streams only).

There is no fallback: if ``libnomas.so`` has not been built (``python
segment_causal_kv_b200/build.py`` or ``__graft_entry__.build()``), importing
the library raises.
"""

from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnomas.so")

NOMAS_OK = 0
NOMAS_ERR_ARG = -1
NOMAS_ERR_ALIGN = -2
NOMAS_ERR_STATE = -3
NOMAS_ERR_CAPACITY = -4
NOMAS_ERR_WORKSPACE = -5
NOMAS_ERR_CUDA = -6
NOMAS_ERR_DEVICE = -7
NOMAS_ERR_DEVICE_TIMEOUT = -8

NOMAS_CACHE_BF16 = 0
NOMAS_CACHE_INT8 = 1
HEAD_DIM = 128

# exported symbols (checked against include/nomas.h by the tests)
EXPORTS = ("nomas_cache_reset", "nomas_kv_commit", "nomas_kv_commit_layers", "nomas_seg_attn_workspace_bytes",
           "nomas_seg_attn_workspace_min_bytes", "nomas_seg_attn",
           "nomas_device_status", "nomas_status_string", "nomas_seg_attn_static", "nomas_selftest_bounded_wait",
           "nomas_kv_evicted_frames", "nomas_kv_archive_evicted", "nomas_camera_attn", "nomas_selftest_div127",
           "nomas_seg_attn_static_status")
NOMAS_STATIC_SCRATCH_BYTES = 64 << 20


class NomasCacheDesc(ctypes.Structure):
    """Mirror of ``struct nomas_cache``."""

    _fields_ = [
        ("mode", ctypes.c_int32),
        ("heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("grid_h", ctypes.c_int32),
        ("grid_w", ctypes.c_int32),
        ("window_frames", ctypes.c_int32),
        ("capacity_frames", ctypes.c_int32),
        ("rope_theta", ctypes.c_float),
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("v_scale", ctypes.c_void_p),
        ("frames_committed", ctypes.c_int64),
        ("valid_frames", ctypes.c_int32),
        ("head_slot", ctypes.c_int32),
        ("check", ctypes.c_uint64),
    ]


class NomasError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {nomas_status_string(status)} ({status})" if what else nomas_status_string(status))


_lib = None


def lib():
    """Load ``libnomas.so`` (raises ImportError when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python {os.path.join(HERE, 'build.py')}`")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        D = ctypes.POINTER(NomasCacheDesc)
        L.nomas_cache_reset.argtypes = [D]
        L.nomas_cache_reset.restype = ctypes.c_int
        L.nomas_kv_commit.argtypes = [D, P, P, I64, I32, P]
        L.nomas_kv_commit.restype = ctypes.c_int
        L.nomas_kv_commit_layers.argtypes = [ctypes.POINTER(D), ctypes.POINTER(P), ctypes.POINTER(P), I64, I32, I32, P]
        L.nomas_kv_commit_layers.restype = ctypes.c_int
        L.nomas_seg_attn_workspace_bytes.argtypes = [D, I32, I32]
        L.nomas_seg_attn_workspace_bytes.restype = ctypes.c_size_t
        L.nomas_seg_attn_workspace_min_bytes.argtypes = [D, I32, I32]
        L.nomas_seg_attn_workspace_min_bytes.restype = ctypes.c_size_t
        L.nomas_seg_attn.argtypes = [D, P, P, P, I64, I32, I32, P, P, P, ctypes.c_size_t, P]
        L.nomas_seg_attn.restype = ctypes.c_int
        L.nomas_device_status.argtypes = [P, P]
        L.nomas_device_status.restype = ctypes.c_int
        L.nomas_seg_attn_static.argtypes = [D, P, P, P, I64, I32, I32, P, P, P]
        L.nomas_seg_attn_static.restype = ctypes.c_int
        L.nomas_selftest_bounded_wait.argtypes = [P, P]
        L.nomas_selftest_bounded_wait.restype = ctypes.c_int
        L.nomas_seg_attn_static_status.argtypes = [P]
        L.nomas_seg_attn_static_status.restype = ctypes.c_int
        L.nomas_selftest_div127.argtypes = [P, P]
        L.nomas_selftest_div127.restype = ctypes.c_int
        L.nomas_kv_evicted_frames.argtypes = [D, I32, ctypes.POINTER(I32), ctypes.POINTER(I64)]
        L.nomas_kv_evicted_frames.restype = ctypes.c_int
        L.nomas_kv_archive_evicted.argtypes = [D, I32, P, P, P, P, I32, ctypes.POINTER(I32), ctypes.POINTER(I64), P]
        L.nomas_kv_archive_evicted.restype = ctypes.c_int
        L.nomas_camera_attn.argtypes = [P, I64, I32, I32, I32, P, P, I32, I32, P, I64, P]
        L.nomas_camera_attn.restype = ctypes.c_int
        L.nomas_status_string.argtypes = [ctypes.c_int]
        L.nomas_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


# ---------------------------------------------------------------- raw C ABI

def nomas_status_string(status: int) -> str:
    return lib().nomas_status_string(int(status)).decode()


def nomas_cache_reset(desc: NomasCacheDesc) -> int:
    return lib().nomas_cache_reset(ctypes.byref(desc))


def nomas_kv_commit(desc: NomasCacheDesc, k_ptr: int, v_ptr: int, token_stride: int, n_frames: int,
                    stream: int | None) -> int:
    return lib().nomas_kv_commit(ctypes.byref(desc), k_ptr, v_ptr, token_stride, n_frames, stream)


def nomas_kv_commit_layers(descs, k_ptrs, v_ptrs, token_stride: int, n_frames: int, stream: int | None) -> int:
    """Commit one segment into several layer caches in one call (descs: NomasCacheDesc objects)."""
    n = len(descs)
    if not (len(k_ptrs) == len(v_ptrs) == n):
        raise ValueError("one K and one V pointer per cache")
    D = ctypes.POINTER(NomasCacheDesc)
    darr = (D * n)(*[ctypes.pointer(d) for d in descs])
    karr = (ctypes.c_void_p * n)(*k_ptrs)
    varr = (ctypes.c_void_p * n)(*v_ptrs)
    return lib().nomas_kv_commit_layers(darr, karr, varr, token_stride, n, n_frames, stream)


def nomas_kv_evicted_frames(desc: NomasCacheDesc, n_frames: int) -> tuple[int, int, int]:
    """(status, count, first_frame) of the frames the next commit of n_frames drops from the window."""
    count, first = ctypes.c_int32(-1), ctypes.c_int64(-1)
    rc = lib().nomas_kv_evicted_frames(ctypes.byref(desc), n_frames, ctypes.byref(count), ctypes.byref(first))
    return rc, int(count.value), int(first.value)


def nomas_kv_archive_evicted(desc: NomasCacheDesc, n_frames: int, hk: int | None, hv: int | None,
                             hks: int | None, hvs: int | None, max_frames: int,
                             stream: int | None) -> tuple[int, int, int]:
    """(status, count, first_frame); enqueues the device-to-host copies of those frames."""
    count, first = ctypes.c_int32(-1), ctypes.c_int64(-1)
    rc = lib().nomas_kv_archive_evicted(ctypes.byref(desc), n_frames, hk, hv, hks, hvs, max_frames,
                                        ctypes.byref(count), ctypes.byref(first), stream)
    return rc, int(count.value), int(first.value)


def nomas_camera_attn(q_ptr: int, q_stride: int, n_frames: int, tokens_per_frame: int, heads: int, kc_ptr: int,
                      vc_ptr: int, n_cam: int, chunk_frames: int, out_ptr: int, out_stride: int,
                      stream: int | None) -> int:
    return lib().nomas_camera_attn(q_ptr, q_stride, n_frames, tokens_per_frame, heads, kc_ptr, vc_ptr, n_cam,
                                   chunk_frames, out_ptr, out_stride, stream)


def camera_attn(q, k_cam, v_cam, n_frames: int, tokens_per_frame: int, chunk_frames: int = 1, out=None,
                stream=None):
    """Per-latent-frame camera cross-attention of the video tokens q [n_frames*F][heads][128]
    (BF16, any token stride) over k_cam, v_cam [n_chunks][n_cam][heads][128]. Returns out."""
    torch = _torch()
    heads = k_cam.shape[2]
    nv = n_frames * tokens_per_frame
    assert q.dtype == torch.bfloat16 and k_cam.dtype == q.dtype and v_cam.dtype == q.dtype
    assert q.shape[0] == nv and q.shape[1] == heads and q.stride(1) == HEAD_DIM and q.stride(2) == 1
    assert k_cam.is_contiguous() and v_cam.is_contiguous() and k_cam.shape == v_cam.shape
    if out is None:
        out = torch.empty((nv, heads, HEAD_DIM), dtype=torch.bfloat16, device=q.device)
    assert out.shape == (nv, heads, HEAD_DIM) and out.stride(1) == HEAD_DIM and out.stride(2) == 1
    _check(nomas_camera_attn(q.data_ptr(), q.stride(0), n_frames, tokens_per_frame, heads, k_cam.data_ptr(),
                             v_cam.data_ptr(), k_cam.shape[1], chunk_frames, out.data_ptr(), out.stride(0),
                             _stream_handle(stream)), "nomas_camera_attn")
    return out


def commit_layers(caches, ks, vs, n_frames: int, stream=None) -> None:
    """nomas_kv_commit_layers for KVCache objects and per-layer BF16 K/V tensors sharing one layout."""
    assert len(caches) == len(ks) == len(vs) and len(caches) > 0
    torch = _torch()
    for k, v in zip(ks, vs):
        assert k.dtype == torch.bfloat16 and v.dtype == k.dtype and k.stride() == v.stride() == ks[0].stride()
    _check(nomas_kv_commit_layers([c.desc for c in caches], [k.data_ptr() for k in ks], [v.data_ptr() for v in vs],
                                  ks[0].stride(0), n_frames, _stream_handle(stream)), "nomas_kv_commit_layers")


def nomas_seg_attn_workspace_bytes(desc: NomasCacheDesc, n_video_frames: int, n_text: int) -> int:
    return int(lib().nomas_seg_attn_workspace_bytes(ctypes.byref(desc), n_video_frames, n_text))


def nomas_seg_attn_workspace_min_bytes(desc: NomasCacheDesc, n_video_frames: int, n_text: int) -> int:
    return int(lib().nomas_seg_attn_workspace_min_bytes(ctypes.byref(desc), n_video_frames, n_text))


def nomas_seg_attn(desc: NomasCacheDesc, q_ptr: int, k_ptr: int, v_ptr: int, token_stride: int,
                   n_video_frames: int, n_text: int, out_ptr: int, lse_ptr: int | None, ws_ptr: int | None,
                   ws_bytes: int, stream: int | None) -> int:
    return lib().nomas_seg_attn(ctypes.byref(desc), q_ptr, k_ptr, v_ptr, token_stride, n_video_frames, n_text,
                                out_ptr, lse_ptr, ws_ptr, ws_bytes, stream)


def nomas_seg_attn_static(desc: NomasCacheDesc, q_ptr: int, k_ptr: int, v_ptr: int, token_stride: int,
                          n_video_frames: int, n_text: int, out_ptr: int, lse_ptr: int | None,
                          stream: int | None) -> int:
    """nomas_seg_attn with the library's static scratch, for callers that cannot allocate a workspace."""
    return lib().nomas_seg_attn_static(ctypes.byref(desc), q_ptr, k_ptr, v_ptr, token_stride, n_video_frames,
                                       n_text, out_ptr, lse_ptr, stream)


def nomas_seg_attn_static_status(stream: int | None) -> int:
    """Synchronise and read/clear the status header of nomas_seg_attn_static's fixed array."""
    return lib().nomas_seg_attn_static_status(stream)


def nomas_selftest_bounded_wait(ws_ptr: int, stream: int | None) -> int:
    """Enqueue the bounded-wait self-test (a wait on a barrier nothing arrives on gives up after 2 s)."""
    return lib().nomas_selftest_bounded_wait(ws_ptr, stream)


def nomas_selftest_div127(result_ptr: int, stream: int | None) -> int:
    """Enqueue the exhaustive check of the commit's division by 127 (two uint32 result words)."""
    return lib().nomas_selftest_div127(result_ptr, stream)


def nomas_device_status(ws_ptr: int, stream: int | None) -> int:
    return lib().nomas_device_status(ws_ptr, stream)


def _check(rc: int, what: str) -> None:
    if rc != NOMAS_OK:
        raise NomasError(rc, what)


# ---------------------------------------------------------------- convenience

def _torch():
    import torch
    return torch


def _stream_handle(stream) -> int | None:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


class KVCache:
    """One layer's lifelong K/V cache in device memory, driven through the C ABI.

    mode: "int8" (codes + fp32 per-(token, head) scales) or "bf16".
    window: history budget in latent frames (0 = full history).
    alloc: optional allocator (shape, dtype, device) -> zero-filled tensor for the
    cache and workspace buffers (default torch.zeros); the tests pass one that
    surrounds every buffer with canary bands.
    """

    def __init__(self, mode: str, heads: int, grid_h: int, grid_w: int, window: int, capacity: int,
                 theta: float = 256.0, device=None, alloc=None):
        torch = _torch()
        self.device = torch.device(device if device is not None else "cuda")
        zeros = alloc or (lambda shape, dtype, dev: torch.zeros(shape, dtype=dtype, device=dev))
        self._zeros = zeros
        self.mode = mode
        self.heads, self.grid_h, self.grid_w = heads, grid_h, grid_w
        self.window, self.capacity = window, capacity
        F = grid_h * grid_w
        if mode == "int8":
            self.k = zeros((heads, capacity * F, HEAD_DIM), torch.int8, self.device)
            self.v = zeros((heads, capacity * F, HEAD_DIM), torch.int8, self.device)
            self.k_scale = zeros((heads, capacity * F), torch.float32, self.device)
            self.v_scale = zeros((heads, capacity * F), torch.float32, self.device)
            m = NOMAS_CACHE_INT8
        elif mode == "bf16":
            self.k = zeros((heads, capacity * F, HEAD_DIM), torch.bfloat16, self.device)
            self.v = zeros((heads, capacity * F, HEAD_DIM), torch.bfloat16, self.device)
            self.k_scale = self.v_scale = None
            m = NOMAS_CACHE_BF16
        else:
            raise ValueError(mode)
        self.desc = NomasCacheDesc(m, heads, HEAD_DIM, grid_h, grid_w, window, capacity, theta,
                                   self.k.data_ptr(), self.v.data_ptr(),
                                   self.k_scale.data_ptr() if self.k_scale is not None else None,
                                   self.v_scale.data_ptr() if self.v_scale is not None else None, 0, 0, 0, 0)
        self._ws = None
        self.reset()

    @property
    def tokens_per_frame(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def frames_committed(self) -> int:
        return int(self.desc.frames_committed)

    @property
    def valid_frames(self) -> int:
        return int(self.desc.valid_frames)

    @property
    def head_slot(self) -> int:
        return int(self.desc.head_slot)

    def reset(self) -> None:
        _check(nomas_cache_reset(self.desc), "nomas_cache_reset")

    def commit(self, k, v, n_frames: int, stream=None, archive: "FrameArchive | None" = None) -> None:
        """k, v: BF16 [n_frames * F][heads][128] (token stride taken from the tensor).

        With an archive, the frames this commit drops from the window are first
        copied into it (on the same stream, so before they are overwritten)."""
        if archive is not None:
            archive.add(self.archive_evicted(n_frames, stream=stream))
        assert k.dtype == _torch().bfloat16 and v.dtype == k.dtype and k.stride() == v.stride()
        assert k.shape[0] >= n_frames * self.tokens_per_frame and k.stride(2) == 1 and k.stride(1) == HEAD_DIM
        _check(nomas_kv_commit(self.desc, k.data_ptr(), v.data_ptr(), k.stride(0), n_frames,
                               _stream_handle(stream)), "nomas_kv_commit")

    def evicted_frames(self, n_frames: int) -> tuple[int, int]:
        """(first_frame, count): the frames the next commit of n_frames drops from the window."""
        rc, count, first = nomas_kv_evicted_frames(self.desc, n_frames)
        _check(rc, "nomas_kv_evicted_frames")
        return first, count

    def archive_evicted(self, n_frames: int, stream=None) -> "ArchivedFrames":
        """Enqueue device-to-host copies of the frames the next commit of n_frames drops.

        Returns pinned host tensors that hold them once `stream` has passed this point."""
        torch = _torch()
        first, count = self.evicted_frames(n_frames)
        F = self.tokens_per_frame
        code_t = torch.int8 if self.mode == "int8" else torch.bfloat16
        host = lambda shape, dt: torch.empty(shape, dtype=dt, pin_memory=count > 0)
        k = host((count, self.heads, F, HEAD_DIM), code_t)
        v = host((count, self.heads, F, HEAD_DIM), code_t)
        ks = vs = None
        if self.mode == "int8":
            ks = host((count, self.heads, F), torch.float32)
            vs = host((count, self.heads, F), torch.float32)
        ptr = lambda t: t.data_ptr() if t is not None and t.numel() else None
        rc, got, first2 = nomas_kv_archive_evicted(self.desc, n_frames, ptr(k), ptr(v), ptr(ks), ptr(vs), count,
                                                   _stream_handle(stream))
        _check(rc, "nomas_kv_archive_evicted")
        assert (got, first2) == (count, first)
        return ArchivedFrames(first, k, v, ks, vs)

    def workspace_bytes(self, n_video_frames: int, n_text: int) -> int:
        return nomas_seg_attn_workspace_bytes(self.desc, n_video_frames, n_text)

    def workspace_min_bytes(self, n_video_frames: int, n_text: int) -> int:
        return nomas_seg_attn_workspace_min_bytes(self.desc, n_video_frames, n_text)

    def workspace(self, n_video_frames: int, n_text: int):
        """A cached device workspace for the fastest form of this call (status header zeroed)."""
        torch = _torch()
        need = self.workspace_bytes(n_video_frames, n_text)
        if self._ws is None or self._ws.numel() < need:
            self._ws = self._zeros((max(need, 256),), torch.uint8, self.device)
        return self._ws

    def seg_attn(self, q, k, v, n_video_frames: int, n_text: int, out=None, lse=None, workspace=None,
                 stream=None):
        """Segment attention; q, k, v BF16 [Nq][heads][128] sharing one token stride. Returns out."""
        torch = _torch()
        nq = n_video_frames * self.tokens_per_frame + n_text
        for t in (q, k, v):
            assert t.dtype == torch.bfloat16 and t.shape[0] == nq and t.stride() == q.stride()
        assert q.stride(2) == 1 and q.stride(1) == HEAD_DIM
        if out is None:
            out = torch.empty((nq, self.heads, HEAD_DIM), dtype=torch.bfloat16, device=q.device)
        ws = workspace if workspace is not None else self.workspace(n_video_frames, n_text)
        _check(nomas_seg_attn(self.desc, q.data_ptr(), k.data_ptr(), v.data_ptr(), q.stride(0), n_video_frames,
                              n_text, out.data_ptr(), lse.data_ptr() if lse is not None else None, ws.data_ptr(),
                              ws.numel() * ws.element_size(), _stream_handle(stream)), "nomas_seg_attn")
        return out

    def device_status(self, stream=None) -> int:
        """Synchronise and read/clear the workspace status header (NOMAS_OK or NOMAS_ERR_DEVICE_TIMEOUT)."""
        if self._ws is None:
            return NOMAS_OK
        return nomas_device_status(self._ws.data_ptr(), _stream_handle(stream))


class ArchivedFrames:
    """Frames [first, first + count) copied out of a cache's window, frame-major in the
    cache's encoding: k, v [count][heads][F][128] (int8 codes or BF16), k_scale,
    v_scale [count][heads][F] fp32 (INT8 mode, else None). Pinned host tensors."""

    def __init__(self, first: int, k, v, k_scale, v_scale):
        self.first, self.k, self.v, self.k_scale, self.v_scale = first, k, v, k_scale, v_scale

    @property
    def count(self) -> int:
        return int(self.k.shape[0])


class FrameArchive:
    """Host archive of every frame dropped from a cache's window (pass it to KVCache.commit).

    It grows without bound, one entry per archived frame; frame(f) returns the
    stored (k, v, k_scale, v_scale) of absolute frame f. Read it only after the
    stream of the commits has been synchronised."""

    def __init__(self):
        self._chunks: list[ArchivedFrames] = []
        self._index: dict[int, tuple[int, int]] = {}

    def add(self, chunk: ArchivedFrames) -> None:
        if chunk.count == 0:
            return
        self._chunks.append(chunk)
        for i in range(chunk.count):
            self._index[chunk.first + i] = (len(self._chunks) - 1, i)

    def frames(self) -> list[int]:
        return sorted(self._index)

    def frame(self, f: int):
        c, i = self._index[f]
        ch = self._chunks[c]
        pick = lambda t: t[i] if t is not None else None
        return pick(ch.k), pick(ch.v), pick(ch.k_scale), pick(ch.v_scale)

    def host_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for ch in self._chunks
                   for t in (ch.k, ch.v, ch.k_scale, ch.v_scale) if t is not None)
