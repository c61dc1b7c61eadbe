"""The C++ fp64 oracle against the numpy oracle and against the pins that do
not depend on either (CPU only).

Both oracles state the same definitions independently (different language,
loops vs library products, different summation orders), so agreement to
~1e-12 on shapes with ragged and empty expert groups is itself a check of each.
The dense brute force and the closed forms pin the C++ side directly.
"""
import numpy as np
import pytest

from oracle import cpp_oracle as C
from oracle import moe_oracle as O


def rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(np.asarray(b)), 1e-300)


def random_layer(seed, T, d, E, k, I, scale=0.2):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, d))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wgu = rng.standard_normal((E, 2 * I, d)) * scale
    wd = rng.standard_normal((E, d, I)) * scale
    gout = rng.standard_normal((T, d))
    return x, logits, wgu, wd, gout


@pytest.mark.parametrize("seed,T,E,k", [(0, 37, 6, 2), (1, 64, 8, 8), (2, 5, 16, 3), (3, 50, 4, 1)])
def test_routing_and_dispatch_bit_exact(seed, T, E, k):
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    logits[: T // 2] = np.round(logits[: T // 2] * 4) / 4  # many exact ties
    logits[0] = 0.5  # an all-equal row: experts 0..k-1
    i1, w1 = C.route(logits, k)
    i2, w2 = O.route(logits, k)
    assert np.array_equal(i1, i2)
    assert np.array_equal(i1[0], np.arange(k))
    assert np.allclose(w1, w2, rtol=1e-14, atol=0)
    for a, b in zip(C.dispatch(i1, E), O.dispatch(i2, E)):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("seed,T,d,E,k,I,threads", [(0, 24, 32, 6, 2, 16, 1), (1, 40, 64, 9, 3, 32, 4),
                                                     (2, 16, 32, 16, 4, 16, 3)])
def test_forward_backward_agree_with_numpy_oracle(seed, T, d, E, k, I, threads):
    x, logits, wgu, wd, gout = random_layer(seed, T, d, E, k, I)
    f1 = C.forward(x, logits, wgu, wd, k, nthreads=threads)
    f2 = O.forward(x, logits, wgu, wd, k)
    assert np.array_equal(f1["idx"], f2["idx"])
    assert rel(f1["out"], f2["out"]) < 1e-13
    assert rel(f1["h"], f2["h"]) < 1e-13 and rel(f1["a"], f2["a"]) < 1e-13
    b1 = C.backward(x, logits, wgu, wd, k, gout, nthreads=threads)
    b2 = O.backward(x, logits, wgu, wd, k, gout, f2)
    for key in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
        assert rel(b1[key], b2[key]) < 1e-12, key


def test_thread_count_does_not_change_results():
    x, logits, wgu, wd, gout = random_layer(5, 30, 32, 7, 2, 16)
    a = C.backward(x, logits, wgu, wd, 2, gout, nthreads=1)
    b = C.backward(x, logits, wgu, wd, 2, gout, nthreads=5)
    for key in a:
        assert np.array_equal(a[key], b[key]), key


def test_dense_brute_force_pins_cpp_forward():
    x, logits, wgu, wd, _ = random_layer(7, 20, 32, 6, 2, 16)
    assert rel(C.forward(x, logits, wgu, wd, 2)["out"], O.dense_forward(x, logits, wgu, wd, 2)) < 1e-12


def test_identity_experts_closed_form():
    # I = d, W_gate = W_up = Id, W_down = Id: out = silu(x) * x for any routing
    rng = np.random.default_rng(8)
    T, d, E, k = 12, 16, 5, 3
    x = rng.standard_normal((T, d))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    eye = np.eye(d)
    wgu = np.broadcast_to(np.concatenate([eye, eye], axis=0), (E, 2 * d, d)).copy()
    wd = np.broadcast_to(eye, (E, d, d)).copy()
    out = C.forward(x, logits, wgu, wd, k)["out"]
    assert np.allclose(out, O.silu(x) * x, rtol=1e-13, atol=1e-14)
    # identical experts: dlogits = 0 and dscore equal across slots
    b = C.backward(x, logits, wgu, wd, k, rng.standard_normal((T, d)))
    assert np.max(np.abs(b["dlogits"])) < 1e-12
    assert np.allclose(b["dscore"], b["dscore"][:, :1], rtol=1e-12, atol=1e-13)


def test_empty_expert_gets_zero_weight_gradients():
    x, logits, wgu, wd, gout = random_layer(9, 20, 32, 6, 2, 16)
    logits[:, 4] = -50.0  # expert 4 never chosen
    b = C.backward(x, logits, wgu, wd, 2, gout)
    assert np.all(b["dwgu"][4] == 0.0) and np.all(b["dwd"][4] == 0.0)


def test_central_differences_pin_cpp_backward():
    rng = np.random.default_rng(10)
    T, d, E, k, I = 4, 8, 4, 2, 4
    x = rng.standard_normal((T, d))
    logits = np.array([[3.0, 1.0, -1.0, -3.0], [-3.0, 2.0, 0.0, 4.0], [0.5, -2.5, 2.5, -0.5],
                       [1.5, 3.5, -1.5, 0.0]], dtype=np.float32)  # top-2 gaps >> step
    wgu = rng.standard_normal((E, 2 * I, d)) * 0.5
    wd = rng.standard_normal((E, d, I)) * 0.5
    gout = rng.standard_normal((T, d))
    b = C.backward(x, logits, wgu, wd, k, gout)
    L = lambda xx, ww, vv: float(np.sum(C.forward(xx, logits, ww, vv, k, keep_intermediates=False)["out"] * gout))
    h = 1e-6
    for (t, c) in [(0, 0), (2, 5), (3, 7)]:
        xp, xm = x.copy(), x.copy()
        xp[t, c] += h
        xm[t, c] -= h
        assert abs((L(xp, wgu, wd) - L(xm, wgu, wd)) / (2 * h) - b["dx"][t, c]) < 1e-7
    for (e, r, c) in [(0, 1, 2), (3, 6, 0)]:
        wp, wm = wgu.copy(), wgu.copy()
        wp[e, r, c] += h
        wm[e, r, c] -= h
        assert abs((L(x, wp, wd) - L(x, wm, wd)) / (2 * h) - b["dwgu"][e, r, c]) < 1e-7
    for (e, o, i) in [(1, 3, 1), (2, 7, 3)]:
        vp, vm = wd.copy(), wd.copy()
        vp[e, o, i] += h
        vm[e, o, i] -= h
        assert abs((L(x, wgu, vp) - L(x, wgu, vm)) / (2 * h) - b["dwd"][e, o, i]) < 1e-7


@pytest.mark.parametrize("limit", [0.3, 1.0])
def test_clamped_swiglu_agrees_with_numpy_oracle(limit):
    rng = np.random.default_rng(31)
    T, d, E, k, I = 40, 32, 6, 2, 16
    x = rng.standard_normal((T, d))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wgu = rng.standard_normal((E, 2 * I, d)) * 0.3
    wd = rng.standard_normal((E, d, I)) * 0.3
    gout = rng.standard_normal((T, d))
    ref_f = O.forward(x, logits, wgu, wd, k, limit=limit)
    assert np.any(ref_f["h"][:, :I] > limit) and np.any(np.abs(ref_f["h"][:, I:]) > limit)
    f = C.forward(x, logits, wgu, wd, k, nthreads=3, limit=limit)
    assert np.allclose(f["out"], ref_f["out"], rtol=1e-12, atol=1e-12)
    ref_b = O.backward(x, logits, wgu, wd, k, gout, limit=limit)
    b = C.backward(x, logits, wgu, wd, k, gout, nthreads=3, limit=limit)
    for key in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
        assert np.allclose(b[key], ref_b[key], rtol=1e-11, atol=1e-12), key
