"""Host model of how the one-kernel decode layer gives each CTA its units, checked against the
plain definition the decode FFN's preparation kernel uses (CPU only).

Definition: slots are the shared expert (if any) followed by the experts some token chose, in
id order; unit ug is slice ug % (I/64) of slot ug // (I/64); CTA b runs units b, b + G, ...

The kernel instead keeps a bitmap of chosen experts (one 32-bit word per lane), takes an
inclusive popcount scan over the words, finds for each of its units the first word whose count
exceeds the unit's rank among the chosen experts (binary lifting over the scan, steps 16, 8,
4, 2, 1), and the rank-th set bit inside that word. This model runs those steps as the warp
does, lane by lane, so a wrong bound in the lifting or an off-by-one in the bit count shows up
as a different unit.
"""
import numpy as np
import pytest


def _units_by_definition(chosen, E, has_shared, nt1, G, b):
    slots = ([E] if has_shared else []) + sorted(set(int(e) for e in chosen))
    n_units = len(slots) * nt1
    return [(slots[ug // nt1], ug % nt1) for ug in range(b, n_units, G)]


def _units_by_bitmap(chosen, E, has_shared, nt1, G, b):
    words = [0] * 32
    for e in chosen:
        words[int(e) >> 5] |= 1 << (int(e) & 31)
    nwd = (E + 31) >> 5
    word = [words[l] if l < nwd else 0 for l in range(32)]
    incl = list(np.cumsum([bin(w).count("1") for w in word]))
    nslots = incl[31] + has_shared
    nunits = nslots * nt1
    n = (nunits - 1 - b) // G + 1 if b < nunits else 0
    out = []
    for lane in range(n):
        ug = b + lane * G
        rnk = ug // nt1 - has_shared
        lo = 0
        for step in (16, 8, 4, 2, 1):
            if incl[lo + step - 1] <= rnk:
                lo += step
        wd = word[lo]
        below = incl[lo - 1] if lo > 0 else 0
        if rnk < 0:
            e = E
        else:
            for _ in range(rnk - below):
                wd &= wd - 1
            e = 32 * lo + (wd & -wd).bit_length() - 1
        out.append((e, ug % nt1))
    return out


@pytest.mark.parametrize("E,T,k,I,has_shared", [
    (512, 8, 10, 512, 1), (512, 1, 10, 512, 1), (512, 4, 10, 512, 0), (256, 8, 8, 2048, 1),
    (8, 3, 2, 64, 1), (1024, 8, 32, 64, 1), (40, 8, 32, 192, 0), (1, 2, 1, 64, 1)])
def test_bitmap_units_match_the_definition(E, T, k, I, has_shared):
    rng = np.random.default_rng(E + 7 * T + 13 * k)
    G, nt1 = 147, I // 64
    for trial in range(20):
        if trial % 4 == 0:  # skewed: a few experts take most choices
            p = 1.0 / np.arange(1, E + 1) ** 1.2
            chosen = np.concatenate([rng.choice(E, size=k, replace=False, p=p / p.sum()) for _ in range(T)])
        else:
            chosen = np.concatenate([rng.choice(E, size=k, replace=False) for _ in range(T)])
        for b in range(G):
            assert _units_by_bitmap(chosen, E, has_shared, nt1, G, b) == \
                _units_by_definition(chosen, E, has_shared, nt1, G, b), (trial, b)


def test_bitmap_units_extremes():
    """Every expert chosen (all 32 words full), and only the last expert chosen."""
    G, nt1, E = 147, 8, 1024
    for chosen in (np.arange(E), np.array([E - 1])):
        for b in (0, 1, 146):
            assert _units_by_bitmap(chosen, E, 1, nt1, G, b) == _units_by_definition(chosen, E, 1, nt1, G, b)
