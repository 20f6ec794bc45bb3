"""Head shards on one GPU: the head-split layer-step, one shard after another.

A rank of the head-sharded layer-step owns a cache of its heads and calls the
library on strided views of its heads' inputs (token stride = all heads x 128,
so the attention reads Q, K and V with a padded stride). No call waits on
another, so one GPU runs the shards of 2 and 3 ranks in turn. Each shard's
commits must equal the oracle's cache rows of its heads bit for bit, and the
shards' outputs, side by side, must meet the attention bar against the oracle
over all heads.
"""

import numpy as np
import pytest

import oracle
import synth
from harness import MAX_ABS, REL_L2, errors, oracle_mode, to_dev, to_f64

pytestmark = pytest.mark.gpu


def workload(mode):
    # 8 heads, 128 tokens per frame; 3-frame segment + 16 text (Nq = 400, a ragged
    # last tile); INT8: a 4-frame window the history wraps; BF16: 5 frames of full history
    w = dict(heads=8, grid_h=8, grid_w=16, mode=mode, hist_commits=[2, 2, 1], cur_frames=3, n_text=16, seed=11)
    if mode == "int8":
        w.update(window=4, capacity=4)
    else:
        w.update(window=0, capacity=8)
    return w


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("mode", ["int8", "bf16"])
def test_head_shards_match_the_all_heads_oracle(mode, world):
    torch = __import__("torch")
    import segment_causal_kv_b200 as nm
    from segment_causal_kv_b200 import shard

    w = workload(mode)
    H = w["heads"]
    geo = synth.Geometry(H, w["grid_h"], w["grid_w"])
    orc = oracle.OracleCache(oracle_mode(mode), H, w["grid_h"], w["grid_w"], w["window"], w["capacity"])
    caches = []
    for r in range(world):
        h0, nh = shard.head_range(H, world, r)
        caches.append((h0, nh, nm.KVCache(mode, nh, w["grid_h"], w["grid_w"], w["window"], w["capacity"])))
    for s, nf in enumerate(w["hist_commits"]):
        k, v = synth.history_kv(geo, nf, w["seed"], s)
        orc.commit(k, v, nf)
        kd, vd = to_dev(k), to_dev(v)
        for h0, nh, c in caches:
            c.commit(kd[:, h0:h0 + nh], vd[:, h0:h0 + nh], nf)
    torch.cuda.synchronize()
    for h0, nh, c in caches:
        sl = slice(h0, h0 + nh)
        if mode == "int8":
            assert np.array_equal(c.k.cpu().numpy(), orc.k_code[sl])
            assert np.array_equal(c.v.cpu().numpy(), orc.v_code[sl])
            assert np.array_equal(c.k_scale.cpu().numpy().view(np.uint32), orc.k_scale[sl].view(np.uint32))
            assert np.array_equal(c.v_scale.cpu().numpy().view(np.uint32), orc.v_scale[sl].view(np.uint32))
        else:
            assert np.array_equal(c.k.cpu().view(torch.int16).numpy().view(np.uint16), orc.k_bf16[sl])
            assert np.array_equal(c.v.cpu().view(torch.int16).numpy().view(np.uint16), orc.v_bf16[sl])
        assert c.valid_frames == orc.valid_frames and c.frames_committed == orc.frames_committed

    q, k, v = synth.segment_qkv(geo, w["cur_frames"], w["n_text"], w["seed"], segment=len(w["hist_commits"]))
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    outs = []
    for h0, nh, c in caches:
        outs.append(c.seg_attn(qd[:, h0:h0 + nh], kd[:, h0:h0 + nh], vd[:, h0:h0 + nh], w["cur_frames"], w["n_text"]))
    torch.cuda.synchronize()
    for _, _, c in caches:
        assert c.device_status() == nm.NOMAS_OK
    got = to_f64(torch.cat(outs, dim=1))
    ref, _ = orc.seg_attn(q, k, v, w["cur_frames"], w["n_text"])
    assert np.isfinite(got).all()
    mx, rel = errors(got, ref)
    assert mx <= MAX_ABS and rel <= REL_L2, (mx, rel)
