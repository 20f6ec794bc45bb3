"""The multi-rank path on the host: world_size-2 process groups over gloo.

segment_causal_kv_b200.shard splits a layer-step by head (no exchange) or, for
token-sharded inputs, exchanges token shards for head shards and back
(Ulysses-style all-to-all). These tests run that code as two spawned CPU ranks
over gloo on 127.0.0.1:
  * the exchange is exact and its inverse restores every rank's shard, for
    even and uneven token and head splits;
  * attention computed per head shard by the oracle, between the two
    exchanges, equals the oracle's attention over all heads, and the per-shard
    caches hold exactly the full cache's codes and scales of their heads;
  * the max-over-ranks reduction the benchmark times with.
The per-rank attention here is the oracle (test infrastructure, CPU); on a GPU
the same exchanges wrap the library's kernels (bench.py --shard ulysses).
"""

from __future__ import annotations

import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(fn, world: int = 2, *args):
    torch = pytest.importorskip("torch")
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_entry, args=(world, port, fn, args), nprocs=world, join=True, start_method="spawn")
    del torch


def _entry(rank: int, world: int, port: int, fn, args):
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from datetime import timedelta
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        fn(rank, world, *args)
        dist.barrier()
    finally:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# rank bodies (module level so that spawned ranks can import them)
# ---------------------------------------------------------------------------

def _exchange_body(rank, world, heads, n_tokens):
    import torch
    from segment_causal_kv_b200 import shard
    g = torch.Generator().manual_seed(7)
    full = torch.randint(-32768, 32767, (n_tokens, heads, 128), generator=g, dtype=torch.int32)
    full = full.to(torch.int16).view(torch.bfloat16)
    counts = shard.split_counts(n_tokens, world)
    t0, n_r = shard.split_range(n_tokens, world, rank)
    h0, nh = shard.head_range(heads, world, rank)
    x = full[t0:t0 + n_r].clone()
    y = shard.seq_to_heads(x, heads, counts)
    assert y.dtype == torch.bfloat16 and tuple(y.shape) == (n_tokens, nh, 128)
    assert torch.equal(y.view(torch.int16), full[:, h0:h0 + nh].view(torch.int16)), "head shard differs"
    back = shard.heads_to_seq(y, heads, counts)
    assert torch.equal(back.view(torch.int16), x.view(torch.int16)), "round trip differs"
    # float64 payloads (the oracle's outputs) take the same route
    # (compared as bits: random BF16 bit patterns include NaNs)
    z = shard.heads_to_seq(full[:, h0:h0 + nh].double(), heads, counts)
    assert torch.equal(z.view(torch.int64), x.double().view(torch.int64))


def _max_body(rank, world):
    from segment_causal_kv_b200 import shard
    got = shard.max_over_ranks([float(rank), 10.0 - rank, 3.5])
    assert got == [float(world - 1), 10.0, 3.5], got


def _oracle_ulysses_body(rank, world, w):
    import torch
    import oracle
    import synth
    from segment_causal_kv_b200 import shard

    H = w["heads"]
    geo = synth.Geometry(H, w["grid_h"], w["grid_w"])
    F = geo.tokens_per_frame
    h0, nh = shard.head_range(H, world, rank)
    mode = oracle.MODE_INT8 if w["mode"] == "int8" else oracle.MODE_BF16
    ref = oracle.OracleCache(mode, H, w["grid_h"], w["grid_w"], w["window"], w["capacity"])
    mine = oracle.OracleCache(mode, nh, w["grid_h"], w["grid_w"], w["window"], w["capacity"])
    as_t = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    for s, nf in enumerate(w["hist_commits"]):
        k, v = synth.history_kv(geo, nf, w["seed"], s)
        ref.commit(k, v, nf)
        # the finished segment arrives token-sharded; exchange it for this rank's heads
        counts = shard.split_counts(nf * F, world)
        t0, n_r = shard.split_range(nf * F, world, rank)
        kh = shard.seq_to_heads(as_t(k[t0:t0 + n_r]), H, counts).numpy().view(np.uint16)
        vh = shard.seq_to_heads(as_t(v[t0:t0 + n_r]), H, counts).numpy().view(np.uint16)
        mine.commit(kh, vh, nf)
    # the per-shard cache holds exactly the full cache's rows of its heads
    if mode == oracle.MODE_INT8:
        assert np.array_equal(mine.k_code, ref.k_code[h0:h0 + nh]) and np.array_equal(mine.v_code, ref.v_code[h0:h0 + nh])
        assert np.array_equal(mine.k_scale.view(np.uint32), ref.k_scale[h0:h0 + nh].view(np.uint32))
        assert np.array_equal(mine.v_scale.view(np.uint32), ref.v_scale[h0:h0 + nh].view(np.uint32))
    else:
        assert np.array_equal(mine.k_bf16, ref.k_bf16[h0:h0 + nh]) and np.array_equal(mine.v_bf16, ref.v_bf16[h0:h0 + nh])

    q, k, v = synth.segment_qkv(geo, w["cur_frames"], w["n_text"], w["seed"], segment=len(w["hist_commits"]))
    nq = q.shape[0]
    counts = shard.split_counts(nq, world)
    t0, n_r = shard.split_range(nq, world, rank)
    qh, kh, vh = (shard.seq_to_heads(as_t(x[t0:t0 + n_r]), H, counts).numpy().view(np.uint16) for x in (q, k, v))
    o_heads, _ = mine.seg_attn(qh, kh, vh, w["cur_frames"], w["n_text"], nthreads=2)
    o_tokens = shard.heads_to_seq(torch.from_numpy(o_heads), H, counts).numpy()
    o_ref, _ = ref.seg_attn(q, k, v, w["cur_frames"], w["n_text"], nthreads=2)
    d = np.abs(o_tokens - o_ref[t0:t0 + n_r]).max()
    assert d <= 1e-12, d


# ---------------------------------------------------------------------------

def test_split_counts_cover_the_range_in_order():
    from segment_causal_kv_b200 import shard
    for n in (0, 1, 7, 80, 2896):
        for world in (1, 2, 3, 8):
            c = shard.split_counts(n, world)
            assert sum(c) == n and max(c) - min(c) <= 1 and c == sorted(c, reverse=True)
            starts = [shard.split_range(n, world, r)[0] for r in range(world)]
            assert starts == [sum(c[:r]) for r in range(world)]
    assert shard.head_range(16, 8, 7) == (14, 2)
    assert shard.head_range(16, 3, 0) == (0, 6) and shard.head_range(16, 3, 2) == (11, 5)
    with pytest.raises(ValueError):
        shard.head_range(2, 4, 0)


def test_single_rank_exchange_is_the_identity():
    torch = pytest.importorskip("torch")
    from segment_causal_kv_b200 import shard
    x = torch.arange(5 * 3 * 128, dtype=torch.int16).view(5, 3, 128).view(torch.bfloat16)
    assert shard.seq_to_heads(x, 3, [5]) is x
    assert shard.heads_to_seq(x, 3, [5]) is x
    assert shard.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]


@pytest.mark.parametrize("heads,n_tokens", [(16, 80), (3, 81), (2, 7), (4, 1)])  # (4, 1): rank 1 holds no token
def test_exchange_is_exact_and_invertible_over_two_gloo_ranks(heads, n_tokens):
    _run(_exchange_body, 2, heads, n_tokens)


def test_max_over_two_gloo_ranks():
    _run(_max_body, 2)


@pytest.mark.parametrize("variant", ["tiny_bf16", "int8_window_3_heads"])
def test_ulysses_attention_matches_the_all_heads_oracle_over_two_gloo_ranks(variant):
    import synth
    w = dict(synth.WORKLOADS["tiny"])
    if variant == "int8_window_3_heads":
        # uneven head split (2 + 1), INT8 ring with eviction
        w.update(heads=3, mode="int8", window=2, capacity=2, hist_commits=[1, 2, 1])
    _run(_oracle_ulysses_body, 2, w)
