"""The filtering score sweep's bucket test, checked on the CPU.

The top-k buckets are read from the order-preserving score key (a monotone, non-increasing
function of the score with 256 buckets per octave of |s|).  The filtering sweep of the bracketed
prefill selection does not form the key of every score: it keeps a key iff its score exceeds a
per-row float bound derived from the bracket bucket b_hi, -F with bits(F) = (b_hi + first + 1)
<< 15 (first = the bucket base, bits(0.25) >> 15).  This test restates the key and the bucket
from their definitions in numpy and checks that the two tests agree for every bucket and for
scores around every bucket edge, zero, the clamped ends, infinities and NaN (which rank below
every score and are never candidates unless the whole pool is).
"""
import numpy as np

FIRST = 125 << 8          # bits(0.25) >> 15
BINS = 2048


def score_key(s):
    b = np.asarray(s, np.float32).view(np.uint32).astype(np.uint64)
    s = np.asarray(s, np.float32)
    b = np.where(s == 0, 0, b)                       # -0 -> +0
    k = np.where(b & 0x80000000, (~b) & 0xFFFFFFFF, b | 0x80000000)
    return np.where(np.isnan(s), 0, k).astype(np.uint64)


def score_bin(key):
    v = ((0x7FFFFFFF - key.astype(np.int64)) >> 15) - FIRST   # arithmetic shift of a signed value
    return np.clip(v, 0, BINS - 1)


def bound(b_hi):
    if b_hi >= BINS - 1:
        return np.float32(-np.inf)
    return -np.uint32((b_hi + FIRST + 1) << 15).view(np.float32)


def scores():
    edges = []
    for b in range(0, BINS + 2):
        f = np.uint32((b + FIRST) << 15).view(np.float32)
        for x in (f, np.nextafter(f, np.float32(0)), np.nextafter(f, np.float32(np.inf))):
            edges += [-x, x]
    rng = np.random.default_rng(0)
    extra = [0.0, -0.0, 1e-30, -1e-30, 0.1, -0.1, -0.25, -64.0, -64.5, -1e30, np.inf, -np.inf, np.nan]
    return np.concatenate([np.float32(edges), np.float32(extra),
                           (-np.exp2(rng.uniform(-4, 8, 200000))).astype(np.float32)])


def test_bound_matches_the_bucket_for_every_bracket():
    s = scores()
    bins = score_bin(score_key(s))
    for b_hi in list(range(0, BINS, 7)) + [BINS - 2, BINS - 1]:
        take = s > bound(b_hi)
        want = bins <= b_hi
        if b_hi == BINS - 1:   # the whole pool: every score but NaN and -inf
            want = want & ~np.isnan(s) & ~np.isneginf(s)
        np.testing.assert_array_equal(take, want, err_msg=f"b_hi={b_hi}")


def test_bucket_is_monotone_in_the_score():
    s = np.sort(scores()[~np.isnan(scores())])
    bins = score_bin(score_key(s))
    assert np.all(np.diff(bins) <= 0)
