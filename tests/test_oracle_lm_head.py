"""Pin for oracle O2 (LM-head logits, EAGLE summary section 3 "Draft model"):
logits = hidden W^T equals numpy's float64 matmul of the same exact input values."""
import numpy as np
import pytest

import workloads as wl


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_lm_head_matches_numpy(orc, dtype):
    rng = np.random.default_rng(2)
    M, H, V = 13, 96, 77
    h = rng.standard_normal((M, H)).astype(np.float32)
    w = (rng.standard_normal((V, H)) / np.sqrt(H)).astype(np.float32)
    if dtype == "bf16":
        h, w = wl.round_to_bf16_bits(h), wl.round_to_bf16_bits(w)
    got = orc.lm_head(h, w)
    ref = wl.as_f32(h, dtype).astype(np.float64) @ wl.as_f32(w, dtype).astype(np.float64).T
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)
    rows = np.array([12, 0, 5])
    np.testing.assert_array_equal(orc.lm_head(h, w, rows=rows), got[rows])


def test_lm_head_bf16_decoding_exact(orc):
    # 1.5 and -0.25 are exact in bf16: 0x3FC0 and 0xBE80
    h = np.array([[0x3FC0, 0xBE80]], dtype=np.uint16)
    w = np.array([[0x3FC0, 0x3FC0], [0xBE80, 0x3F80]], dtype=np.uint16)
    got = orc.lm_head(h, w)
    np.testing.assert_array_equal(got, [[1.5 * 1.5 - 0.25 * 1.5, -1.5 * 0.25 - 0.25]])
