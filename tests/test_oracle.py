"""The fp64 oracle against its pins (CPU only)."""
import math

import numpy as np
import pytest

from oracle import brute
from tests import oracle_pins


@pytest.mark.parametrize("name", sorted(oracle_pins.PINS))
def test_pin(name, oracle_lib):
    oracle_pins.PINS[name](oracle_lib)


def test_partition_merge_equals_direct_softmax():
    """Splitting the context into partitions, taking (max, exp-sum,
    normalised partial output) per partition and merging them with
    M = max m_p, w_p = l_p exp(m_p - M) gives the single-pass softmax
    attention (the blocked softmax of "PagedAttention：大模型KV Cache分页管理
    优化实践" §5.1 with partitions in place of blocks)."""
    rng = np.random.Generator(np.random.PCG64(17))
    for n, cuts in ((1000, [0, 512, 1000]), (37, [0, 1, 2, 36, 37]), (2048, [0, 512, 1024, 1536, 2048])):
        x = rng.standard_normal(n) * 4
        v = rng.standard_normal((n, 16))
        w = np.exp(x - x.max())
        direct = (w[:, None] * v).sum(0) / w.sum()
        parts = brute.partition_scores(x, v, list(zip(cuts[:-1], cuts[1:])))
        merged = brute.partition_merge(parts)
        assert np.max(np.abs(merged - direct)) < 1e-12


def test_partition_merge_single_partition_is_identity():
    rng = np.random.Generator(np.random.PCG64(18))
    x, v = rng.standard_normal(20), rng.standard_normal((20, 4))
    (m, l, o), = brute.partition_scores(x, v, [(0, 20)])
    assert np.allclose(brute.partition_merge([(m, l, o)]), o, rtol=0, atol=0)
    assert math.isclose(m, x.max())
