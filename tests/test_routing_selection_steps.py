"""CPU check of the selection steps the lane-per-token routing kernel takes,
restated in Python and compared with the oracle's routing, bit for bit:

* tau, the k-th largest of NG group maxima (NG = 2k when E is a multiple of 8k,
  else k), by sorting two halves of the maxima and merging them with
  max_i min(A_i, B_(k-i)), is a lower bound on the k-th largest logit;
* inserting the logits >= tau in expert order into k sorted slots, a strictly
  larger order key moving ahead, leaves the k largest in slot order with ties to
  the lower expert.

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


def kth_largest_of_maxima(g, k):
    g = list(g)
    if len(g) == k:
        return min(g)
    halves = [sorted(g[:k], reverse=True), sorted(g[k:], reverse=True)]
    a, b = halves
    t = max(a[k - 1], b[k - 1])
    for i in range(1, k):
        t = max(t, min(a[i - 1], b[k - 1 - i]))
    return t


def select(row, k, strict=True):
    E = len(row)
    ng = 2 * k if E % (8 * k) == 0 else k
    gs = E // ng
    tau = kth_largest_of_maxima([max(row[g * gs:(g + 1) * gs]) for g in range(ng)], k)
    cand = [e for e in range(E) if row[e] >= tau]
    assert len(cand) >= k  # tau is a lower bound on the k-th largest
    keys, idx = [0] * k, [0] * k
    for e in cand:  # expert order
        x = order_key(row[e])
        gt = [(x > keys[j]) if strict else (x >= keys[j]) for j in range(k)]
        nk, ni = keys[:], idx[:]
        for j in range(k - 1, 0, -1):
            nk[j] = keys[j - 1] if gt[j - 1] else (x if gt[j] else keys[j])
            ni[j] = idx[j - 1] if gt[j - 1] else (e if gt[j] else idx[j])
        nk[0] = x if gt[0] else keys[0]
        ni[0] = e if gt[0] else idx[0]
        keys, idx = nk, ni
    return idx, len(cand)


@pytest.mark.parametrize("E,k", [(128, 8), (96, 4), (32, 8), (8, 2), (64, 8), (120, 5), (112, 7), (24, 3), (128, 1)])
def test_selection_steps_match_the_oracle(E, k):
    rng = np.random.default_rng(E * 10 + k)
    for trial in range(150):
        row = rng.standard_normal(E).astype(np.float32)
        if trial % 3 == 0:
            row = (np.round(row * 2) / 2).astype(np.float32)  # many ties
        if trial % 7 == 0:
            row[:] = np.float32(0.5)                          # a fully tied row
        if trial % 11 == 0:
            row[::3] = np.float32(-0.0)
            row[1::5] = np.float32(0.0)
        idx, _ = select([np.float32(v) for v in row], k)
        ref, _ = O.route(row[None, :], k)
        assert idx == list(ref[0]), (E, k, trial)


def test_tighter_bound_leaves_fewer_candidates():
    # on Gaussian logits the 2k-group bound leaves about 10 candidates for
    # E = 128, k = 8, against about 20 for the k-group bound
    rng = np.random.default_rng(0)
    n = []
    for _ in range(200):
        n.append(select([np.float32(v) for v in rng.standard_normal(128).astype(np.float32)], 8)[1])
    assert 8 <= np.mean(n) < 13


def test_planted_mistake_ties_to_the_higher_expert():
    # a non-strict comparison lets a later (higher) expert pass an equal key
    rng = np.random.default_rng(5)
    row = (np.round(rng.standard_normal(64) * 2) / 2).astype(np.float32)
    ref, _ = O.route(row[None, :], 8)
    assert select([np.float32(v) for v in row], 8)[0] == list(ref[0])
    assert select([np.float32(v) for v in row], 8, strict=False)[0] != list(ref[0])
