"""Host model of the per-token top-k selection the routing kernels and the one-kernel decode
layer run (one warp per token; expert e sits in lane e % 32, slot e // 32), checked against
the oracle's top-k (Reading R4: the k largest float32 logits, equal logits by the lower
expert id).

The kernel first takes a threshold, the k-th largest of the 32 lane maxima: at least k logits
reach it, so every logit of the top k is among the candidates at or above it. At most 32
candidates are gathered one per lane and each is ranked against the others (equal keys by the
lower id); with more candidates the kernel falls back to k rounds of a warp arg-max, which is
the sorted order by definition. This model follows those steps on the same float32 bit keys,
so a wrong threshold, a candidate lost or a wrong tie rule shows up as a difference from the
oracle. Both zeros map to the key of +0.0, so logits of -0.0 and +0.0 tie like equal values.
"""
import numpy as np
import pytest

from oracle import moe as omoe

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _keys(row_f32):
    r = row_f32.astype(np.float32)
    r = np.where(r == 0.0, np.float32(0.0), r)  # -0.0 -> +0.0
    u = r.view(np.uint32).astype(np.uint64)
    neg = (u >> 31) == 1
    return np.where(neg, (~u) & 0xFFFFFFFF, u | 0x80000000).astype(np.uint64)


def _threshold_select(row_f32, k):
    """Returns (picks in order, number of candidates); picks is None when the kernel would
    take its fallback (more than 32 candidates)."""
    E = row_f32.size
    key = _keys(row_f32)
    lanes = [[(int(key[e]), e) for e in range(lane, E, 32)] for lane in range(32)]
    lmax = [max((kk for kk, _ in l), default=0) for l in lanes]
    above = [sum(1 for o in range(32) if o != l and lmax[o] > lmax[l]) for l in range(32)]
    th = min(lmax[l] for l in range(32) if above[l] < k)
    cand = [(kk, e) for l in range(32) for kk, e in lanes[l] if kk >= th]
    if len(cand) > 32:
        return None, len(cand)
    rank = [sum(1 for (ok, oe) in cand if ok > ck or (ok == ck and oe < ce)) for (ck, ce) in cand]
    picks = [None] * k
    for (ck, ce), r in zip(cand, rank):
        if r < k:
            picks[r] = ce
    return picks, len(cand)


def _check_rows(rows, k):
    want = omoe.topk(rows, k)
    n_fallback = 0
    for t in range(rows.shape[0]):
        picks, _ = _threshold_select(rows[t], k)
        if picks is None:
            n_fallback += 1
            continue
        assert picks == list(want[t]), f"row {t}: {picks} != {list(want[t])}"
    return n_fallback


@pytest.mark.parametrize("E,k", [(8, 2), (64, 8), (256, 8), (512, 10), (512, 32), (1024, 8), (40, 32)])
def test_threshold_selection_random_rows(E, k):
    rng = np.random.default_rng(E * 100 + k)
    rows = rng.standard_normal((64, E)).astype(np.float32)
    n_fallback = _check_rows(rows, k)
    if k <= 16:
        # independent logits almost never put more than 32 candidates over the threshold
        assert n_fallback <= 2
    # with k near 32 the threshold sinks to the smallest lane maximum and the k rounds of the
    # fallback do the selection (the model then checks nothing for those rows)


def test_threshold_candidate_count_is_small():
    """The reason the fast path is the usual one: for 512 independent logits and k = 10 the
    candidates number about k + 2."""
    rng = np.random.default_rng(5)
    counts = [_threshold_select(rng.standard_normal(512).astype(np.float32), 10)[1] for _ in range(200)]
    assert 10 <= min(counts) and np.mean(counts) < 16 and max(counts) <= 32


@pytest.mark.parametrize("levels", [2, 5, 40])
def test_threshold_selection_with_ties(levels):
    """Logits on a few levels: many equal keys, so the tie rule (lower id first) decides."""
    rng = np.random.default_rng(levels)
    rows = rng.integers(0, levels, size=(48, 512)).astype(np.float32) - levels / 2
    fallback = 0
    for t in range(rows.shape[0]):
        picks, n = _threshold_select(rows[t], 10)
        if picks is None:
            fallback += 1
            continue
        assert picks == list(omoe.topk(rows[t:t + 1], 10)[0])
    if levels == 2:
        assert fallback == rows.shape[0]  # half the experts tie at the top: fallback every time


def test_threshold_selection_top_values_in_one_lane():
    """The k largest logits all in lane 0 (experts 0, 32, 64, ...): the lane maxima see only
    one of them, and the threshold must still keep all of them as candidates."""
    E, k = 512, 10
    rows = np.random.default_rng(3).standard_normal((8, E)).astype(np.float32)
    for t in range(rows.shape[0]):
        rows[t, 0:32 * k:32] = 10.0 + np.arange(k, dtype=np.float32) + t
    assert _check_rows(rows, k) == 0


def test_threshold_selection_small_E():
    """E < 32: lanes without experts hold key 0 and never reach the threshold."""
    rng = np.random.default_rng(11)
    for E in (1, 3, 17, 31):
        for k in range(1, E + 1, max(1, E // 4)):
            rows = rng.standard_normal((4, E)).astype(np.float32)
            assert _check_rows(rows, k) == 0


def test_threshold_selection_signed_zeros():
    """Logits of exactly -0.0 and +0.0 around the k-th place are equal values: the oracle
    takes the lower expert ids first, and so do the kernels' keys (both zeros share one key)."""
    E, k = 64, 8
    rng = np.random.default_rng(21)
    rows = -np.abs(rng.standard_normal((16, E))).astype(np.float32) - 1.0
    for t in range(rows.shape[0]):
        zeros = rng.choice(E, 12, replace=False)
        rows[t, zeros] = np.where(rng.random(12) < 0.5, np.float32(-0.0), np.float32(0.0))
        rows[t, rng.choice(np.setdiff1d(np.arange(E), zeros), 3, replace=False)] = 1.0
    assert _check_rows(rows, k) == 0
