"""The package's vectorised threshold calibration against the oracle's
loop-by-loop one ("Block Sparse Flash Attention", section "Gating Mechanism
and Threshold Calibration"), on random block maxima of several sequences,
causal and not, for k from 0 to past the number of candidates."""
import numpy as np
import pytest

import oracle
from blockwise_attn_ffn_b200 import bsfa


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("k", [0, 1, 2, 5, 9, 12])
def test_calibrate_matches_oracle(causal, k):
    rng = np.random.default_rng(k + 10 * causal)
    S, h, nb = 3, 2, 9
    bm = rng.normal(2.0, 1.0, size=(S, h, nb, nb))
    if causal:
        bm = np.where(np.tril(np.ones((nb, nb), bool)), bm, -np.inf)
    want = oracle.calibrate_thresholds(list(bm), k, causal).astype(np.float32)
    got = bsfa.calibrate(bm, k, causal)
    np.testing.assert_array_equal(got, want)


def test_calibrate_rejects_negative_k():
    with pytest.raises(ValueError):
        bsfa.calibrate(np.zeros((1, 1, 2, 2)), -1, True)
