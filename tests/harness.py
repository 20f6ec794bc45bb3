"""Shared helpers of the GPU parity tests: build the same cache on the GPU
(through the C ABI) and in the oracle from identical synthetic inputs, and
compare attention outputs with the tolerances the targets state."""

from __future__ import annotations

import numpy as np

import oracle
import synth

# Attention parity bar: max-abs error 2e-2 and relative L2 error 5e-3
# against the fp64 oracle.
MAX_ABS = 2e-2
REL_L2 = 5e-3


def torch_mod():
    import torch
    return torch


def to_dev(bits: np.ndarray, device="cuda"):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def to_f64(t) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def oracle_mode(mode: str) -> int:
    return oracle.MODE_INT8 if mode == "int8" else oracle.MODE_BF16


class Guards:
    """Device buffers with canary bands before and after them (a stand-in for a
    memory checker, which is not available on the GPU pool): every buffer is
    the interior of a larger allocation whose first and last PAD bytes hold the
    pattern PAT; check() asserts that no kernel wrote into a band."""

    PAD = 4096
    PAT = 0xA5

    def __init__(self):
        self.bufs = []

    def alloc(self, shape, dtype, device="cuda", fill=0.0):
        torch = torch_mod()
        el = torch.empty((), dtype=dtype).element_size()
        n = int(np.prod(shape)) * el
        raw = torch.full((n + 2 * self.PAD,), self.PAT, dtype=torch.uint8, device=device)
        inner = raw[self.PAD:self.PAD + n].view(dtype).view(shape)
        inner.fill_(fill)
        self.bufs.append((raw, n))
        return inner

    def zeros(self, shape, dtype, device):
        return self.alloc(shape, dtype, device, 0)

    def check(self):
        torch = torch_mod()
        torch.cuda.synchronize()
        for i, (raw, n) in enumerate(self.bufs):
            lo = raw[:self.PAD]
            hi = raw[self.PAD + n:]
            assert bool((lo == self.PAT).all()), f"buffer {i}: bytes written before its start"
            assert bool((hi == self.PAT).all()), f"buffer {i}: bytes written past its end"


def make_caches(w: dict, with_oracle: bool = True, device="cuda", guards: Guards | None = None):
    import segment_causal_kv_b200 as nm
    gpu = nm.KVCache(w["mode"], w["heads"], w["grid_h"], w["grid_w"], w["window"], w["capacity"], device=device,
                     alloc=guards.zeros if guards is not None else None)
    orc = oracle.OracleCache(oracle_mode(w["mode"]), w["heads"], w["grid_h"], w["grid_w"], w["window"],
                             w["capacity"]) if with_oracle else None
    geo = synth.Geometry(w["heads"], w["grid_h"], w["grid_w"])
    for s, nf in enumerate(w["hist_commits"]):
        k, v = history_segment(w, geo, s, nf)
        gpu.commit(to_dev(k, device), to_dev(v, device), nf)
        if orc is not None:
            orc.commit(k, v, nf)
    return gpu, orc


def history_segment(w: dict, geo, s: int, nf: int):
    """K/V of history segment s; with w["kv_ramp"] = r, K of segment s is scaled by
    r^s (then rounded to BF16), so scores rise from segment to segment."""
    k, v = synth.history_kv(geo, nf, w["seed"], s, w.get("kv_std", 1.0))
    r = w.get("kv_ramp")
    if r:
        k = synth.f32_to_bf16_bits((synth.bf16_bits_to_f32(k).astype(np.float64) * r ** s).astype(np.float32))
    return k, v


def current_segment(w: dict):
    geo = synth.Geometry(w["heads"], w["grid_h"], w["grid_w"])
    return synth.segment_qkv(geo, w["cur_frames"], w["n_text"], w["seed"], segment=len(w["hist_commits"]),
                             q_std=w.get("q_std", 1.0), kv_std=w.get("kv_std", 1.0))


def errors(got: np.ndarray, ref: np.ndarray):
    d = got - ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))


def sample_rows(nq: int, tpf: int, n_video_frames: int, per_head: int, seed: int = 0) -> np.ndarray:
    """Query rows covering first/last video frame, tile tails and text tokens, plus random rows."""
    nv = n_video_frames * tpf
    fixed = {0, 1, min(127, nq - 1), min(128, nq - 1), nq - 1, max(nq - 2, 0)}
    if nv > 0:
        fixed |= {nv - 1, max(nv - tpf, 0), min(nv, nq - 1)}
    fixed |= {min(nq - 1, (nq // 128) * 128 - 1), min(nq - 1, (nq // 128) * 128)}
    rng = np.random.default_rng(seed)
    rest = rng.choice(nq, size=min(nq, max(per_head - len(fixed), 0)), replace=False)
    return np.array(sorted(fixed | set(int(x) for x in rest)), dtype=np.int64)
