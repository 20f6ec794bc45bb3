"""The INT8 commit's row scale is absmax / 127, correctly rounded to fp32
(IEEE division, as the oracle computes it). The kernel reaches it without a
division instruction, by Markstein's method (a product with RN(1/127), an
exact fma remainder, one correction), which is exact only where nothing
underflows. This test has the device compare that function with its own
IEEE division for all 2^31 non-negative fp32 bit patterns, zero, subnormals,
infinity and NaNs included."""

import pytest

pytestmark = pytest.mark.gpu


def test_div127_matches_ieee_division_for_every_nonnegative_float():
    torch = __import__("torch")
    import segment_causal_kv_b200 as nm
    res = torch.zeros(2, dtype=torch.int32, device="cuda")
    rc = nm.nomas_selftest_div127(res.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == nm.NOMAS_OK, nm.nomas_status_string(rc)
    torch.cuda.synchronize()
    mismatches, first = (int(x) & 0xFFFFFFFF for x in res.cpu().tolist())
    assert mismatches == 0, f"{mismatches} inputs differ, first pattern {first:#010x}"
    assert first == 0xFFFFFFFF
