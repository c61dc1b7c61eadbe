"""CPU check of the selection steps the routing kernel's quad form (four
lanes per token) takes, restated in Python and compared with the oracle's
routing, bit for bit:

* tau, the k-th largest of the E/4 piece maxima, found by sorting each lane's
  maxima (Batcher's odd-even merge sort) and merging the four lanes' lists
  with two butterfly steps (the k largest of two sorted lists A, B are
  max(A_i, B_(k-1-i))), is a lower bound on the k-th largest logit;
* ranking the candidates (logits >= tau) by 64-bit keys (order key of the
  value, then ~expert) puts the k largest in slot order with ties to the lower
  expert; so does taking them one per round when there are too many.

This pins the mathematics of those steps (the CUDA kernel itself is checked by
the GPU routing tests); it shares no code with the library.
"""
import numpy as np
import pytest

from oracle import moe_oracle as O


def order_key(v):
    v = np.float32(v)
    if v == 0:
        v = np.float32(0.0)  # -0 ties with +0
    u = int(np.array(v, dtype=np.float32).view(np.uint32))
    return (~u & 0xFFFFFFFF) if u >> 31 else (u | 0x80000000)


def odd_even_merge_sort_desc(g):
    """Batcher's odd-even merge sort network of the next power of two, with the
    comparators that touch an index >= len(g) dropped."""
    n = len(g)
    P = 1
    while P < n:
        P *= 2
    g = list(g)
    p = 1
    while p < P:
        k = p
        while k >= 1:
            j = k % p
            while j + k < P:
                for i in range(k):
                    a, b = i + j, i + j + k
                    if b < n and a // (2 * p) == b // (2 * p):
                        g[a], g[b] = max(g[a], g[b]), min(g[a], g[b])
                j += 2 * k
            k >>= 1
        p <<= 1
    return g


def bitonic_sort_desc(c):
    n = len(c)
    if n & (n - 1):
        return odd_even_merge_sort_desc(c)
    c = list(c)
    s = n // 2
    while s >= 1:
        for j in range(n):
            if not j & s:
                c[j], c[j + s] = max(c[j], c[j + s]), min(c[j], c[j + s])
        s //= 2
    return c


def quad_select(row, k, cap=16, low_word=lambda e: ~e & 0xFFFFFFFF):
    """The quad form's steps for one token: lane q holds the 4-logit pieces
    q, q+4, ...; tau from the sorted piece maxima merged over the lanes by two
    butterfly steps; candidates >= tau; slots by rank (at most cap candidates),
    else the k largest one per round.  Returns (experts in slot order, number
    of candidates, tau of each lane)."""
    E = len(row)
    E4 = E // 4
    nv = 2 if E <= 32 else 4 if E <= 64 else 8
    neg = np.float32(-np.inf)
    lst = []
    for q in range(4):
        gm = [max(row[4 * (q + 4 * i):4 * (q + 4 * i) + 4]) if q + 4 * i < E4 else neg for i in range(nv)]
        gm = odd_even_merge_sort_desc(gm)
        lst.append([gm[j] if j < nv else neg for j in range(k)])
    mrg = [bitonic_sort_desc([max(lst[q][j], lst[q ^ 1][k - 1 - j]) for j in range(k)]) for q in range(4)]
    taus = [min(max(mrg[q][j], mrg[q ^ 2][k - 1 - j]) for j in range(k)) for q in range(4)]
    tau = taus[0]
    cand = [16 * i + 4 * q + c for q in range(4) for i in range(nv) if q + 4 * i < E4 for c in range(4)
            if row[16 * i + 4 * q + c] >= tau]
    key = {e: (order_key(row[e]) << 32) | low_word(e) for e in cand}
    if len(cand) <= cap:
        slots = [None] * k
        for e in cand:
            r = sum(1 for f in cand if key[f] > key[e])
            if r < k:
                slots[r] = e
    else:
        rem, slots = set(cand), []
        for _ in range(k):
            best = max(rem, key=lambda e: key[e])
            slots.append(best)
            rem.remove(best)
    return slots, len(cand), taus


@pytest.mark.parametrize("n", [1, 2, 3, 4, 5, 6, 7, 8])
def test_quad_sorting_networks(n):
    rng = np.random.default_rng(n)
    for _ in range(400):
        g = [float(v) for v in rng.integers(0, 4, n)]
        assert odd_even_merge_sort_desc(g) == sorted(g, reverse=True)
        a = sorted(rng.integers(0, 9, n), reverse=True)
        b = sorted(rng.integers(0, 9, n), reverse=True)
        c = [max(a[j], b[n - 1 - j]) for j in range(n)]  # the k largest of a and b, bitonic
        assert sorted(c, reverse=True) == sorted(list(a) + list(b), reverse=True)[:n]
        assert bitonic_sort_desc(c) == sorted(c, reverse=True)


@pytest.mark.parametrize("E,k", [(128, 8), (96, 4), (32, 8), (8, 2), (64, 8), (120, 5), (112, 7), (24, 3), (128, 1),
                                 (4, 1), (16, 4)])
def test_quad_selection_steps_match_the_oracle(E, k):
    rng = np.random.default_rng(E * 10 + k + 7)
    over_cap = 0
    for trial in range(150):
        row = rng.standard_normal(E).astype(np.float32)
        if trial % 3 == 0:
            row = (np.round(row * 2) / 2).astype(np.float32)  # many ties
        if trial % 7 == 0:
            row[:] = np.float32(0.5)                          # a fully tied row
        if trial % 11 == 0:
            row[::3] = np.float32(-0.0)
            row[1::5] = np.float32(0.0)
        slots, n, taus = quad_select([np.float32(v) for v in row], k)
        assert len(set(taus)) == 1  # the four lanes agree on tau
        assert n >= k
        over_cap += n > 16
        ref, _ = O.route(row[None, :], k)
        assert slots == list(ref[0]), (E, k, trial)
    if E >= 32:
        assert over_cap > 0  # the one-per-round path is taken too


def test_quad_bound_leaves_few_candidates():
    # on Gaussian logits (E = 128, k = 8) about 9 candidates, never more than 16
    rng = np.random.default_rng(1)
    n = [quad_select([np.float32(v) for v in rng.standard_normal(128).astype(np.float32)], 8)[1]
         for _ in range(300)]
    assert 8 <= np.mean(n) < 10.5 and max(n) <= 16


def test_quad_planted_mistake_rank_ties_to_the_higher_expert():
    # a key whose low word is the expert itself (not ~expert) ranks equal
    # values the wrong way round
    rng = np.random.default_rng(9)
    row = [np.float32(v) for v in (np.round(rng.standard_normal(128) * 2) / 2)]
    ref, _ = O.route(np.array(row, dtype=np.float32)[None, :], 8)
    assert quad_select(row, 8)[0] == list(ref[0])
    assert quad_select(row, 8, low_word=lambda e: e)[0] != list(ref[0])
    assert quad_select(row, 8, cap=0, low_word=lambda e: e)[0] != list(ref[0])
