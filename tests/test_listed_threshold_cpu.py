"""The exactness argument of the prefill ranking's listed threshold, checked
on the CPU with numpy on rows of the shapes the kernel takes (1024-2048
keys, k <= 64, entry e held by lane e % 32).

t0 is the least over the 32 lanes of each lane's second-largest key.  Every
lane then holds two keys >= t0, so at least 64 keys pass it; the k-th
largest key is therefore >= t0, and every key the set keeps (all keys above
the k-th, and the lowest-index ones equal to it) lies among the listed keys.
These tests check that claim on rows drawn from several distributions, and
that on Gaussian rows the list is short (about six keys per lane, none
past the kernel's 24 slots) while the
patterns the kernel hands to the full search do trip their conditions."""
import numpy as np
import pytest

LANES, CAP = 32, 24


def t0_of(keys):
    """keys: 1-D array of one row (entry e in lane e % 32)."""
    n = len(keys)
    pad = np.full(((n + LANES - 1) // LANES) * LANES, -np.inf)
    pad[:n] = keys
    per_lane = pad.reshape(-1, LANES).T          # [lane][q]
    second = np.sort(per_lane, axis=1)[:, -2]    # each lane's second-largest
    return second.min()


def top_k(keys, k):
    """The exact set: k largest, ties to the lower index."""
    order = np.lexsort((np.arange(len(keys)), -keys))
    return np.sort(order[:k])


def rows(kind, n, count, rng):
    if kind == "gauss":
        return rng.normal(0, 1.4, (count, n))
    if kind == "heavy":
        return rng.standard_t(2.0, (count, n))
    if kind == "recency":  # scores rising toward the end of the row
        return rng.normal(0, 1.0, (count, n)) + np.linspace(0, 4, n)[None, :]
    if kind == "ties":
        return rng.integers(0, 4, (count, n)).astype(np.float64)
    if kind == "lane":  # one lane's entries all high
        x = rng.normal(0, 1.0, (count, n))
        x[:, 5::LANES] += 6.0
        return x
    raise ValueError(kind)


@pytest.mark.parametrize("kind", ["gauss", "heavy", "recency", "ties", "lane"])
@pytest.mark.parametrize("n", [1024, 1500, 2045, 2048])
def test_the_kept_set_lies_among_the_listed_keys(kind, n):
    rng = np.random.default_rng(n + len(kind))
    for x in rows(kind, n, 40, rng):
        t0 = t0_of(x)
        listed = x >= t0
        assert listed.sum() >= 2 * LANES
        for k in (1, 8, 33, 64):
            keep = top_k(x, k)
            assert listed[keep].all(), (kind, n, k)
            # the k-th largest is >= t0, and every key equal to it is listed
            kth = np.sort(x)[-k]
            assert kth >= t0 and listed[x == kth].all()


def test_gaussian_rows_list_a_few_keys_per_lane():
    rng = np.random.default_rng(7)
    fracs, over = [], 0
    for x in rows("gauss", 2045, 400, rng):
        listed = x >= t0_of(x)
        fracs.append(listed.mean())
        per_lane = np.bincount(np.nonzero(listed)[0] % LANES, minlength=LANES)
        over += int(per_lane.max() > CAP)
    assert 0.06 < np.mean(fracs) < 0.12      # ~9 % of the row, ~6 keys per lane
    assert over == 0                          # no lane past its 24 slots (16: ~2 % of rows)


def test_the_patterns_handed_to_the_full_search_trip_their_conditions():
    rng = np.random.default_rng(11)
    # one lane's entries all high: that lane lists more than 24 keys
    x = rows("lane", 2045, 1, rng)[0]
    listed = np.nonzero(x >= t0_of(x))[0]
    assert np.bincount(listed % LANES, minlength=LANES).max() > CAP
    # four distinct values: keys equal to the k-th are only partly kept
    x = rows("ties", 2045, 1, rng)[0]
    k = 64
    kth = np.sort(x)[-k]
    assert (x > kth).sum() < k < (x >= kth).sum()
