"""bench.py's CPU side: the reference arm (the oracle on host cores) prints one
JSON line with the contract's keys and the same workload config keys as the
GPU arm."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == "seg_attn_tflops" and d["unit"] == "TFLOP/s"
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    sys.path.insert(0, ROOT)
    try:
        import bench
        import synth
        want = bench.workload_config(synth.WORKLOADS[bench.WORKLOAD])
    finally:
        sys.path.remove(ROOT)
    for k, v in want.items():
        assert d["config"][k] == v, k


def test_algorithmic_work_figures():
    """The FLOP and byte counts bench.py divides by: 4*H*D*Nq*Nk for attention (QK^T + PV, unpadded,
    nothing masked); K, V BF16 read plus INT8 codes and fp32 scales written for a commit."""
    sys.path.insert(0, ROOT)
    try:
        import bench
        import synth
        w = synth.WORKLOADS[bench.WORKLOAD]
        F, nq, nc, nk, flop = bench.workload_shape(w)
        assert (F, nq, nc, nk) == (880, 3 * 880 + 256, 18 * 880, 18 * 880 + 3 * 880 + 256)
        assert flop == 4 * 16 * 128 * 2896 * 18736 == 444_493_463_552
        # 3 frames x 880 tokens x 16 heads x (K, V) x (256 B read + 128 B codes + 4 B scale written)
        assert bench.commit_bytes(w) == 3 * 880 * 16 * 2 * (256 + 128 + 4) == 32_778_240
    finally:
        sys.path.remove(ROOT)
