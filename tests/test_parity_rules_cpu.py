"""The set comparison the GPU parity tests use (tests/parity.py: check_sets),
checked on the CPU against the oracle on a tiny case with an exact tie at
the k-th score.  A valid alternative set inside the tie band passes; sets
that are wrong in ways a kernel could plausibly get wrong -- the initial
block dropped, a set one entry short, padding moved, a block after the
query, a repeat, an unsorted list, a block from below the band -- fail."""
import numpy as np
import pytest

import oracle
from block_sparse_long_sparda_b200 import workloads as W
from tests.parity import candidate_range, check_sets, scores_f64

NB, K, N_INIT, N_LOCAL = 16, 4, 1, 2
T = NB * 64


def _case():
    # F = e0, so block j scores kc[j][0]; blocks 4, 5 and 7 tie at 3.0, the
    # fourth-best score, so the oracle keeps 4 and 5 (lower index wins) and 7
    # is an equally valid choice
    kc = np.zeros((1, 1, NB, 128), np.float32)
    kc[0, 0, :, 0] = [9, 5, -2, 4, 3, 3, 0, 3, -1, 1, 2, -3, -4, 1, 8, 7]
    F = np.zeros((1, 1, 1, 1, 128), np.float32)
    F[..., 0] = 1.0
    Fb, kcb = W.f32_to_bf16_bits(F), W.f32_to_bf16_bits(kc)
    ora, kth, kth1 = oracle.select(Fb, kcb, K, N_INIT, N_LOCAL, T - 1)
    return ora, kth, kth1, scores_f64(Fb, kcb)


def _check(got, ora, kth, kth1, sc):
    return check_sets(np.asarray(got, np.int32).reshape(1, 1, 1, -1), ora, kth, kth1, sc, "tiny",
                      q_pos=T - 1, n_init=N_INIT, n_local=N_LOCAL)


def test_oracle_set_and_tie_of_the_case():
    ora, kth, kth1, _ = _case()
    assert ora.reshape(-1).tolist() == [0, 1, 3, 4, 5, 14, 15]
    assert kth.item() == 3.0 and kth1.item() == 3.0
    assert candidate_range(T - 1, N_INIT, N_LOCAL) == (15, 1, 14)


def test_identical_and_valid_alternative_sets_pass():
    ora, kth, kth1, sc = _case()
    assert _check(ora.reshape(-1), ora, kth, kth1, sc) == 1
    assert _check([0, 1, 3, 4, 7, 14, 15], ora, kth, kth1, sc) == 0   # 7 for 5: same score


@pytest.mark.parametrize("got,why", [
    ([1, 3, 4, 5, 7, 14, 15], "initial block dropped for a tied block"),
    ([0, 1, 3, 4, 7, 15, 13], "local block replaced (and unsorted)"),
    ([0, 1, 3, 4, 7, 13, 15], "local block replaced by a candidate"),
    ([0, 1, 3, 4, 14, 15, -1], "one entry short"),
    ([-1, 0, 1, 3, 4, 14, 15], "padding moved to the front"),
    ([0, 1, 3, 4, 5, 15, 16], "a block after the query's own"),
    ([0, 1, 3, 4, 4, 14, 15], "a repeated block"),
    ([0, 1, 4, 3, 7, 14, 15], "not ascending"),
    ([0, 1, 3, 4, 6, 14, 15], "a block from below the band (score 0)"),
    ([0, 3, 4, 5, 7, 14, 15], "a block from above the band dropped (score 5)"),
])
def test_planted_mistakes_fail(got, why):
    ora, kth, kth1, sc = _case()
    with pytest.raises(AssertionError):
        _check(got, ora, kth, kth1, sc)


def test_a_clear_gap_demands_identical_sets():
    ora, kth, kth1, sc = _case()
    kc_clear = kth.copy()
    kth1_clear = kth1 - 1.0        # as if the (k+1)-th score were clearly lower
    with pytest.raises(AssertionError):
        _check([0, 1, 3, 4, 7, 14, 15], ora, kc_clear, kth1_clear, sc)
