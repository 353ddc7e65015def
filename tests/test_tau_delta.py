"""tau = delta / N, the pages' length-adaptive skip threshold (host-side mapping)."""
import math

import pytest

import block_sparse_long_14_b200 as cosa


def test_delta_minus_one_turns_skipping_off():
    assert cosa.tau_from_delta(-1, 131072) == 0.0


@pytest.mark.parametrize("delta", [200, 1000, 2000])
@pytest.mark.parametrize("n", [4096, 32768, 131072])
def test_tau_is_delta_over_tokens(delta, n):
    tau = cosa.tau_from_delta(delta, n)
    assert tau == delta / n
    assert 0.0 <= tau < 1.0
    # the skip test compares against ln(tau): longer sequences skip more readily
    assert math.log(tau) < 0


def test_longer_sequences_get_smaller_tau():
    taus = [cosa.tau_from_delta(1000, n) for n in (4096, 16384, 65536, 131072)]
    assert taus == sorted(taus, reverse=True)


@pytest.mark.parametrize("delta,n", [(5000, 4096), (-2, 1024), (10, 0)])
def test_out_of_range_is_rejected(delta, n):
    with pytest.raises(ValueError):
        cosa.tau_from_delta(delta, n)
