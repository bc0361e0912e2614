"""The shared input module: seeded, reproducible, and its bf16 rounding agrees
with torch's own fp32 -> bf16 conversion (round to nearest even)."""
import numpy as np
import pytest

import workloads as W


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    a = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 7
    a[:4] = [0.0, -0.0, 1.0 + 2**-8, 1.0 + 3 * 2**-8]        # ties go to even
    ours = W.bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_draws_are_reproducible_and_distinct():
    a = W.normal((64, 32), 1.0, 1234, W.TAG_Q, "bf16")
    b = W.normal((64, 32), 1.0, 1234, W.TAG_Q, "bf16")
    c = W.normal((64, 32), 1.0, 1234, W.TAG_K, "bf16")
    np.testing.assert_array_equal(a, b)
    assert not np.array_equal(a, c)
    assert np.array_equal(W.round_to(a, "bf16"), a)      # already representable


def test_workload_table():
    assert W.STACK720P.N == 21 * 23 * 40 and W.STACK720P.D == 3072 and W.STACK720P.L == 24
    assert W.STACK480P.N == 21 * 15 * 26 and W.STACK480P.D == 2048
    assert W.LONG4.N == 41 * 23 * 40
    assert W.HYBRID4_F32.attnres_block == 0 and W.HYBRID4_F32.dtype == "f32"
    assert [w.seed for w in W.STACKS.values()] == [1234, 1235, 1236, 1237]
