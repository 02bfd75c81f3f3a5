"""The by-value evaluation of the oracle that the full-size GPU parity tests use
(tests/_helpers.py, OracleExpertByValue) gives exactly what the oracle's
direct evaluation gives (OracleExpert): absmax, scale, every code, the packed
stream and the dequantized matrices, on whole experts with outliers, zeros of
both signs, subnormals and every width; and a non-finite master still raises."""
import numpy as np
import pytest

import synth
from oracle import quantize as oq

from _helpers import OracleExpert, OracleExpertByValue


def _same(master, H, F, b):
    a = OracleExpert(master, H, F, b)
    v = OracleExpertByValue(master, H, F, b)
    assert v.m == a.m
    assert v.s == a.s and np.float32(v.s).tobytes() == np.float32(a.s).tobytes()
    assert np.array_equal(v.codes(), a.k)
    assert np.array_equal(v.stream(), a.stream())
    for x, y in zip(v.mats(), a.mats()):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("b", [3, 4, 8])
def test_by_value_equals_direct_on_workload_experts(b):
    wl = synth.WORKLOADS[1]
    for e in (0, 5):
        _same(synth.expert_weights(wl, e).numpy(), wl.H, wl.F, b)
    # the outlier recipe of the Mixtral-shaped layer, at a small size
    wl2 = synth.scaled(synth.WORKLOADS[2], H=256, F=512)
    m2 = synth.expert_weights(wl2, 3).numpy()
    assert np.abs(m2.astype(np.float64)).max() == float(np.float16(0.2))
    _same(m2, wl2.H, wl2.F, b)


@pytest.mark.parametrize("b", [3, 4, 8])
def test_by_value_equals_direct_on_edge_values(b):
    H, F = 256, 128  # 98,304 weights: room for all 63,488 finite values
    rng = np.random.default_rng(b)
    # every finite fp16 value at least once (ties, subnormals, both zeros),
    # then random finite patterns
    finite = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    finite = finite[np.isfinite(finite.view(np.float16))]
    n = 3 * H * F
    pats = np.concatenate([finite, rng.choice(finite, n - finite.size)])
    rng.shuffle(pats)
    _same(pats.view(np.float16), H, F, b)
    # a small absmax: most of the grid lies in the subnormals
    small = (pats.view(np.float16).astype(np.float64) * 2.0 ** -20).astype(np.float16)
    _same(small, H, F, b)
    zero = np.zeros(n, dtype=np.float16)
    zero[::7] = -0.0
    _same(zero, H, F, b)


def test_by_value_rejects_non_finite_master():
    m = synth.expert_weights(synth.WORKLOADS[1], 0).numpy().copy()
    m[1234] = np.float16(np.inf)
    with pytest.raises(oq.NonFiniteMaster):
        OracleExpertByValue(m, 256, 512, 4)
    m[1234] = np.float16(np.nan)
    with pytest.raises(oq.NonFiniteMaster):
        OracleExpertByValue(m, 256, 512, 4)
