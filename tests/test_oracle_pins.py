"""Pins for the CPU oracle: each test checks it against something other than itself.

Kinds of pin used here:
  * brute force on tiny inputs (Python loops, sorted() with an explicit key,
    every expert on every token);
  * closed forms (identity-weight experts, k = E with equal logits, identical
    experts, a hand-worked 2-d example);
  * invariants (counts sum to T*k, perm is a bijection, inv inverts it,
    ascending tokens inside an expert, weights sum to one);
  * central finite differences of the forward for every gradient.
The planted-mistake tests at the end perturb the oracle on the CPU and check
that at least one pin then fails.
"""
import math

import numpy as np
import pytest

from oracle import moe_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ----------------------------------------------------------------------------
# helpers written independently of the oracle (scalar Python)
# ----------------------------------------------------------------------------
def py_sigmoid(z):
    return 1.0 / (1.0 + math.exp(-z)) if z > -700 else 0.0


def py_silu(z):
    return z * py_sigmoid(z)


def py_expert(xrow, wgu_e, wd_e):
    """One expert on one token with explicit loops (no numpy products)."""
    twoI, d = len(wgu_e), len(xrow)
    I = twoI // 2
    h = [sum(wgu_e[r][c] * xrow[c] for c in range(d)) for r in range(twoI)]
    a = [py_silu(h[i]) * h[I + i] for i in range(I)]
    return [sum(wd_e[r][i] * a[i] for i in range(I)) for r in range(len(wd_e))]


def py_topk(row, k):
    order = sorted(range(len(row)), key=lambda e: (-float(row[e]), e))
    return order[:k]


def rand_layer(rng, T, d, E, k, I, wscale=0.3):
    x = rng.standard_normal((T, d))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wgu = rng.standard_normal((E, 2 * I, d)) * wscale
    wd = rng.standard_normal((E, d, I)) * wscale
    gout = rng.standard_normal((T, d))
    return x, logits, wgu, wd, gout


def spaced_logits(rng, T, E, gap=0.37):
    """Logits whose sorted values differ by at least ``gap`` within each row."""
    base = np.arange(E, dtype=np.float64) * gap
    rows = [rng.permutation(base) + rng.uniform(0, 0.01) for _ in range(T)]
    return np.asarray(rows, dtype=np.float32)


# ----------------------------------------------------------------------------
# routing
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("T,E,k", [(64, 8, 2), (40, 16, 4), (17, 5, 5), (9, 7, 1), (33, 128, 8)])
def test_route_matches_sorted_bruteforce(T, E, k):
    rng = np.random.default_rng(T * 100 + E)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    # force many exact ties: round half of the rows to multiples of 0.25
    logits[::2] = np.round(logits[::2] * 4) / 4
    logits[3 % T, :] = 0.5          # a fully tied row -> experts 0..k-1
    logits[5 % T, :E // 2] = -0.0   # signed zeros compare equal
    logits[5 % T, E // 2:] = 0.0
    idx, w = O.route(logits, k)
    for t in range(T):
        assert list(idx[t]) == py_topk(logits[t], k), t
    assert list(idx[3 % T]) == list(range(k))
    # weights: exp(l_j - l_max) / sum over the chosen set, written per token
    for t in range(T):
        sel = [float(logits[t, e]) for e in idx[t]]
        m = max(float(v) for v in logits[t])
        ex = [math.exp(v - m) for v in sel]
        s = sum(ex)
        for j in range(k):
            assert w[t, j] == pytest.approx(ex[j] / s, rel=1e-13, abs=1e-300)
    assert np.allclose(w.sum(1), 1.0, atol=1e-14)
    if k == 1:
        assert np.all(w == 1.0)


def test_dispatch_invariants_and_bruteforce():
    rng = np.random.default_rng(7)
    T, E, k = 50, 12, 3
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[:, 4] -= 100.0  # expert 4 never chosen -> an empty group
    idx, _ = O.route(logits, k)
    counts, offsets, perm, inv = O.dispatch(idx, E)
    assert counts.sum() == T * k
    assert counts[4] == 0
    # brute-force construction: experts ascending, then tokens ascending
    bf = [t * k + j for e in range(E) for t in range(T) for j in range(k) if idx[t, j] == e]
    assert list(perm) == bf
    assert sorted(perm.tolist()) == list(range(T * k))
    for q in range(T * k):
        assert inv.reshape(-1)[perm[q]] == q
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(idx.reshape(-1)[seg] == e)
        assert np.all(np.diff(seg // k) > 0)
        assert offsets[e + 1] - offsets[e] == sum(1 for t in range(T) for j in range(k) if idx[t, j] == e)


# ----------------------------------------------------------------------------
# forward
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("T,d,E,k,I", [(24, 8, 6, 2, 5), (16, 6, 4, 4, 3), (10, 4, 3, 1, 2)])
def test_sparse_equals_dense_bruteforce(T, d, E, k, I):
    rng = np.random.default_rng(T + d + E)
    x, logits, wgu, wd, _ = rand_layer(rng, T, d, E, k, I)
    sparse = O.forward(x, logits, wgu, wd, k)["out"]
    dense = O.dense_forward(x, logits, wgu, wd, k)
    assert np.max(np.abs(sparse - dense)) <= 1e-12


def test_forward_matches_scalar_loops():
    rng = np.random.default_rng(11)
    T, d, E, k, I = 7, 5, 4, 2, 3
    x, logits, wgu, wd, _ = rand_layer(rng, T, d, E, k, I)
    out = O.forward(x, logits, wgu, wd, k)["out"]
    for t in range(T):
        order = py_topk(logits[t], k)
        m = max(float(v) for v in logits[t])
        ex = [math.exp(float(logits[t, e]) - m) for e in order]
        ref = [0.0] * d
        for j, e in enumerate(order):
            y = py_expert(list(x[t]), wgu[e].tolist(), wd[e].tolist())
            for c in range(d):
                ref[c] += ex[j] / sum(ex) * y[c]
        assert np.allclose(out[t], ref, rtol=1e-12, atol=1e-12)


def test_identity_experts_closed_form():
    """W_gate = W_up = Id, W_down = Id  =>  out = silu(x) * x for any routing."""
    rng = np.random.default_rng(3)
    T, d, E, k = 12, 6, 5, 3
    x = rng.standard_normal((T, d)) * 2
    logits = rng.standard_normal((T, E)).astype(np.float32)
    eye = np.eye(d)
    wgu = np.stack([np.concatenate([eye, eye])] * E)
    wd = np.stack([eye] * E)
    out = O.forward(x, logits, wgu, wd, k)["out"]
    ref = np.array([[py_silu(v) * v for v in row] for row in x])
    assert np.allclose(out, ref, rtol=1e-13, atol=1e-14)
    # backward closed form: dx = gout * (silu'(x) x + silu(x)), dlogits = 0
    gout = rng.standard_normal((T, d))
    g = O.backward(x, logits, wgu, wd, k, gout)
    ref_dx = np.array([[gout[t, c] * ((py_sigmoid(v) * (1 + v * (1 - py_sigmoid(v)))) * v + py_silu(v))
                        for c, v in enumerate(row)] for t, row in enumerate(x)])
    assert np.allclose(g["dx"], ref_dx, rtol=1e-12, atol=1e-13)
    assert np.max(np.abs(g["dlogits"])) <= 1e-12


def test_uniform_scores_all_experts_is_mean():
    """k = E and equal logits: idx = 0..E-1, w = 1/E, out = mean of expert outputs."""
    rng = np.random.default_rng(5)
    T, d, E, I = 6, 4, 5, 3
    x, _, wgu, wd, _ = rand_layer(rng, T, d, E, E, I)
    logits = np.full((T, E), 0.75, dtype=np.float32)
    f = O.forward(x, logits, wgu, wd, E)
    assert np.all(f["idx"] == np.arange(E)[None, :])
    assert np.allclose(f["w"], 1.0 / E, rtol=0, atol=1e-16)
    for t in range(T):
        ys = [py_expert(list(x[t]), wgu[e].tolist(), wd[e].tolist()) for e in range(E)]
        mean = [sum(y[c] for y in ys) / E for c in range(d)]
        assert np.allclose(f["out"][t], mean, rtol=1e-12, atol=1e-13)


def test_handworked_two_dim_example():
    """A worked example small enough to do by hand (gate rows first, W_down [d, I]).

    d = 2, I = 1, E = 2, k = 2.  x = (1, 2).  Expert 0: gate row (3, 4), up row
    (5, 6), W_down column (7, 8).  Expert 1: gate (-1, 1), up (2, 0), W_down (1, -1).
    Logits (0.5, 0): w0 = e^0.5 / (e^0.5 + 1), w1 = 1 / (e^0.5 + 1).
    Expert 0: g = 3 + 8 = 11, u = 5 + 12 = 17, a = silu(11) 17, y = (7a, 8a).
    Expert 1: g = -1 + 2 = 1, u = 2, a = 2 silu(1), y = (a, -a).
    """
    x = np.array([[1.0, 2.0]])
    wgu = np.array([[[3.0, 4.0], [5.0, 6.0]], [[-1.0, 1.0], [2.0, 0.0]]])
    wd = np.array([[[7.0], [8.0]], [[1.0], [-1.0]]])
    logits = np.array([[0.5, 0.0]], dtype=np.float32)
    f = O.forward(x, logits, wgu, wd, 2)
    w0 = math.exp(0.5) / (math.exp(0.5) + 1.0)
    w1 = 1.0 / (math.exp(0.5) + 1.0)
    a0 = 11.0 / (1.0 + math.exp(-11.0)) * 17.0
    a1 = 2.0 * (1.0 / (1.0 + math.exp(-1.0)))
    expect = [w0 * 7 * a0 + w1 * a1, w0 * 8 * a0 - w1 * a1]
    assert list(f["idx"][0]) == [0, 1]
    assert np.allclose(f["out"][0], expect, rtol=1e-14)
    # dscore[j] = <gout, y_j>; with gout = (1, 0): (7 a0, a1)
    g = O.backward(x, logits, wgu, wd, 2, np.array([[1.0, 0.0]]))
    assert np.allclose(g["dscore"][0], [7 * a0, a1], rtol=1e-14)
    # dW_down[0] = w0 * gout (x) a0 = [[w0 a0], [0]]
    assert np.allclose(g["dwd"][0], [[w0 * a0], [0.0]], rtol=1e-14)


# ----------------------------------------------------------------------------
# backward: central finite differences of the forward, loss = <out, gout>
# ----------------------------------------------------------------------------
def _fd(f, arr, index, eps=1e-6):
    old = arr[index]
    arr[index] = old + eps
    lp = f()
    arr[index] = old - eps
    lm = f()
    arr[index] = old
    return (lp - lm) / (2 * eps)


@pytest.fixture(scope="module")
def fd_case():
    rng = np.random.default_rng(21)
    T, d, E, k, I = 10, 6, 5, 3, 4
    x, _, wgu, wd, gout = rand_layer(rng, T, d, E, k, I, wscale=0.5)
    logits = spaced_logits(rng, T, E)
    return x, logits, wgu, wd, gout, k


def test_finite_differences_x_and_weights(fd_case):
    x, logits, wgu, wd, gout, k = fd_case
    x, wgu, wd = x.copy(), wgu.copy(), wd.copy()
    g = O.backward(x, logits, wgu, wd, k, gout)
    loss = lambda: float(np.sum(O.forward(x, logits, wgu, wd, k)["out"] * gout))  # noqa: E731
    rng = np.random.default_rng(0)
    for arr, grad in ((x, g["dx"]), (wgu, g["dwgu"]), (wd, g["dwd"])):
        for _ in range(12):
            index = tuple(int(rng.integers(0, s)) for s in arr.shape)
            assert _fd(loss, arr, index) == pytest.approx(grad[index], rel=1e-6, abs=1e-8)


def test_finite_differences_logits(fd_case):
    x, logits, wgu, wd, gout, k = fd_case
    lg = logits.astype(np.float64)
    g = O.backward(x, logits, wgu, wd, k, gout)

    def loss():
        # route on the (fixed) ordering but weights from the perturbed fp64 logits
        return float(np.sum(O.forward(x, lg, wgu, wd, k)["out"] * gout))

    T, E = lg.shape
    for t in range(T):
        for e in range(E):
            assert _fd(loss, lg, (t, e), eps=1e-6) == pytest.approx(g["dlogits"][t, e], rel=1e-6, abs=1e-8)


def test_finite_differences_dscore(fd_case):
    x, logits, wgu, wd, gout, k = fd_case
    f = O.forward(x, logits, wgu, wd, k)
    g = O.backward(x, logits, wgu, wd, k, gout, f)
    idx, w = f["idx"], f["w"].copy()
    loss = lambda: float(np.sum(O.combine_forward(x, idx, w, wgu, wd) * gout))  # noqa: E731
    for t in range(w.shape[0]):
        for j in range(k):
            assert _fd(loss, w, (t, j)) == pytest.approx(g["dscore"][t, j], rel=1e-7, abs=1e-9)


def test_identical_experts_routing_grad_vanishes():
    rng = np.random.default_rng(4)
    T, d, E, k, I = 8, 5, 6, 3, 4
    x, logits, wgu, wd, gout = rand_layer(rng, T, d, E, k, I)
    wgu[:] = wgu[0]
    wd[:] = wd[0]
    g = O.backward(x, logits, wgu, wd, k, gout)
    assert np.max(np.abs(g["dlogits"])) <= 1e-12
    assert np.allclose(g["dscore"], g["dscore"][:, :1], rtol=1e-12, atol=1e-12)


def test_empty_expert_has_exact_zero_weight_grads():
    rng = np.random.default_rng(9)
    T, d, E, k, I = 20, 6, 5, 2, 3
    x, logits, wgu, wd, gout = rand_layer(rng, T, d, E, k, I)
    logits[:, 2] = -50.0
    g = O.backward(x, logits, wgu, wd, k, gout)
    assert np.all(g["dwgu"][2] == 0.0) and np.all(g["dwd"][2] == 0.0)


def test_sampled_variants_agree_with_full():
    rng = np.random.default_rng(12)
    T, d, E, k, I = 30, 8, 6, 3, 5
    x, logits, wgu, wd, gout = rand_layer(rng, T, d, E, k, I)
    f = O.forward(x, logits, wgu, wd, k)
    g = O.backward(x, logits, wgu, wd, k, gout, f)
    toks = [0, 7, 29]
    ft = O.forward_tokens(x, logits, wgu, wd, k, toks)
    assert np.allclose(ft["out"], f["out"][toks], rtol=1e-12, atol=1e-13)
    bt = O.backward_tokens(x, logits, wgu, wd, k, gout, toks)
    for key in ("dx", "dscore", "dlogits"):
        assert np.allclose(bt[key], g[key][toks], rtol=1e-12, atol=1e-13)
    be = O.backward_experts(x, logits, wgu, wd, k, gout, [1, 4])
    for e in (1, 4):
        assert np.allclose(be[e][0], g["dwgu"][e], rtol=1e-12, atol=1e-13)
        assert np.allclose(be[e][1], g["dwd"][e], rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------
# the skewed workload's recipe
# ----------------------------------------------------------------------------
def test_zipf_skew_gives_about_ten_empty_experts():
    from grouped_gemm_route_b200 import inputs as IN
    cfg = IN.WORKLOADS["qwen3_30b_a3b_skew"]
    lg = IN.make_logits(cfg["T"], cfg["E"], seed=0, zipf_s=cfg["zipf_s"]).numpy()
    idx, _ = O.route(lg, cfg["k"])
    c = np.bincount(idx.ravel(), minlength=cfg["E"])
    assert 8 <= int((c == 0).sum()) <= 12
    assert c.max() > 8 * cfg["T"] * cfg["k"] // cfg["E"]


# ----------------------------------------------------------------------------
# planted mistakes: a plausible slip in the oracle must fail a pin
# ----------------------------------------------------------------------------
def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def test_planted_mistake_silu_grad(monkeypatch, fd_case):
    monkeypatch.setattr(O, "silu_grad", lambda z: O.sigmoid(z))  # dropped term
    assert _fails(test_finite_differences_x_and_weights, fd_case)


def test_planted_mistake_gate_up_swap(monkeypatch):
    def swapped(xe, wgu_e, wd_e, limit=0.0):
        I = wd_e.shape[1]
        h = xe @ wgu_e.T
        a = O.silu(h[:, I:]) * h[:, :I]
        return h, a, a @ wd_e.T
    monkeypatch.setattr(O, "expert_forward", swapped)
    assert _fails(test_handworked_two_dim_example)


def test_planted_mistake_no_renormalisation(monkeypatch):
    real = O.route

    def unnormalised(logits, k):
        idx, w = real(logits, k)
        lo = np.asarray(logits, dtype=np.float64)
        p = np.exp(lo - lo.max(1, keepdims=True))
        p /= p.sum(1, keepdims=True)
        return idx, np.take_along_axis(p, idx.astype(np.int64), 1)
    monkeypatch.setattr(O, "route", unnormalised)
    assert _fails(test_forward_matches_scalar_loops)


def test_planted_mistake_routing_grad_sign(monkeypatch, fd_case):
    monkeypatch.setattr(O, "routing_backward", lambda w, ds: -np.asarray(w) * (np.asarray(ds) - np.sum(w * ds, 1, keepdims=True)))
    assert _fails(test_finite_differences_logits, fd_case)
