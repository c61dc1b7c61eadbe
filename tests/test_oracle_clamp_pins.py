"""Pins for the oracle's clamped SwiGLU (a = silu(min(g, L)) * clip(u, -L, L), L > 0).

* identity experts (W_gate = W_up = Id, W_down = Id) give, for any routing
  (the weights sum to one), out = silu(min(x, L)) * clip(x, -L, L) elementwise
  and dx = gout * d/dx of that, written here with scalar math;
* a limit above every pre-activation gives the plain layer bit for bit;
* central finite differences of the clamped forward for every gradient, on
  inputs whose pre-activations stay well away from the clamps' corners;
* the side of a clamp is decided on h rounded to bfloat16: bf16_round is
  pinned against torch's float32 -> bfloat16 conversion and hand-worked ties,
  and swiglu_backward against points just inside and outside a clamp;
* a planted mistake (the gate clamped from below instead of above) fails the
  closed form.
"""
import math

import numpy as np
import pytest

from oracle import moe_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def py_sigmoid(z):
    return 1.0 / (1.0 + math.exp(-z)) if z > -700 else 0.0


def py_silu(z):
    return z * py_sigmoid(z)


def py_act(v, L):
    """silu(min(v, L)) * clip(v, -L, L) for gate = up = v."""
    gc = v if v <= L else L
    uc = -L if v < -L else (L if v > L else v)
    return py_silu(gc) * uc


def py_act_grad(v, L):
    """d/dv of py_act: the gate term where v <= L, the up term where |v| <= L."""
    gc = v if v <= L else L
    uc = -L if v < -L else (L if v > L else v)
    s = py_sigmoid(gc)
    dg = s * (1 + gc * (1 - s)) * uc if v <= L else 0.0
    du = py_silu(gc) if -L <= v <= L else 0.0
    return dg + du


def identity_layer(rng, L, T=14, d=7, E=5):
    x = rng.standard_normal((T, d)) * 2.5
    near = np.abs(np.abs(x) - L) < 0.05  # keep |x| clear of L by more than a bf16 spacing
    x[near] += 0.1
    logits = rng.standard_normal((T, E)).astype(np.float32)
    eye = np.eye(d)
    wgu = np.stack([np.concatenate([eye, eye])] * E)
    wd = np.stack([eye] * E)
    return x, logits, wgu, wd


@pytest.mark.parametrize("L", [0.5, 1.5, 3.0])
def test_identity_experts_closed_form(L):
    rng = np.random.default_rng(int(L * 10))
    x, logits, wgu, wd = identity_layer(rng, L)
    assert np.any(x > L) and np.any(x < -L)  # both clamps active somewhere
    out = O.forward(x, logits, wgu, wd, 3, limit=L)["out"]
    ref = np.array([[py_act(v, L) for v in row] for row in x])
    assert np.allclose(out, ref, rtol=1e-13, atol=1e-14)
    gout = rng.standard_normal(x.shape)
    g = O.backward(x, logits, wgu, wd, 3, gout, limit=L)
    ref_dx = np.array([[gout[t, c] * py_act_grad(v, L) for c, v in enumerate(row)] for t, row in enumerate(x)])
    assert np.allclose(g["dx"], ref_dx, rtol=1e-12, atol=1e-13)
    assert np.max(np.abs(g["dlogits"])) <= 1e-12  # identical experts


def test_limit_above_every_preactivation_is_the_plain_layer():
    rng = np.random.default_rng(7)
    T, d, E, k, I = 12, 16, 4, 2, 8
    x = rng.standard_normal((T, d))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wgu = rng.standard_normal((E, 2 * I, d)) * 0.3
    wd = rng.standard_normal((E, d, I)) * 0.3
    gout = rng.standard_normal((T, d))
    plain_f = O.forward(x, logits, wgu, wd, k)
    assert np.max(np.abs(plain_f["h"])) < 1e3
    big_f = O.forward(x, logits, wgu, wd, k, limit=1e3)
    assert np.array_equal(plain_f["out"], big_f["out"])
    plain_b = O.backward(x, logits, wgu, wd, k, gout, plain_f)
    big_b = O.backward(x, logits, wgu, wd, k, gout, big_f, limit=1e3)
    for key in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
        assert np.array_equal(plain_b[key], big_b[key]), key


def _fd(f, arr, index, eps=1e-6):
    old = arr[index]
    arr[index] = old + eps
    lp = f()
    arr[index] = old - eps
    lm = f()
    arr[index] = old
    return (lp - lm) / (2 * eps)


@pytest.fixture(scope="module")
def clamp_case():
    """A small layer with both clamps active and every pre-activation at least
    0.02 away from the corners (g = L, u = +-L), so that steps of 1e-6 in any
    input never cross one."""
    T, d, E, k, I, L = 10, 6, 4, 2, 5, 0.6
    for seed in range(200):
        rng = np.random.default_rng(1000 + seed)
        x = rng.standard_normal((T, d))
        base = np.arange(E, dtype=np.float64) * 0.37
        logits = np.asarray([rng.permutation(base) + rng.uniform(0, 0.01) for _ in range(T)], dtype=np.float32)
        wgu = rng.standard_normal((E, 2 * I, d)) * 0.5
        wd = rng.standard_normal((E, d, I)) * 0.5
        h = O.forward(x, logits, wgu, wd, k)["h"]
        g, u = h[:, :I], h[:, I:]
        if (np.min(np.abs(g - L)) > 0.02 and np.min(np.abs(np.abs(u) - L)) > 0.02 and np.any(g > L)
                and np.any(np.abs(u) > L)):
            return x, logits, wgu, wd, rng.standard_normal((T, d)), k, L
    raise AssertionError("no case with clear clamp margins")


def test_finite_differences_clamped(clamp_case):
    x, logits, wgu, wd, gout, k, L = clamp_case
    x, wgu, wd = x.copy(), wgu.copy(), wd.copy()
    g = O.backward(x, logits, wgu, wd, k, gout, limit=L)
    loss = lambda: float(np.sum(O.forward(x, logits, wgu, wd, k, limit=L)["out"] * gout))  # noqa: E731
    rng = np.random.default_rng(0)
    for arr, grad in ((x, g["dx"]), (wgu, g["dwgu"]), (wd, g["dwd"])):
        for _ in range(16):
            index = tuple(int(rng.integers(0, s)) for s in arr.shape)
            assert _fd(loss, arr, index) == pytest.approx(grad[index], rel=1e-6, abs=1e-8)


def test_finite_differences_clamped_dscore(clamp_case):
    x, logits, wgu, wd, gout, k, L = clamp_case
    f = O.forward(x, logits, wgu, wd, k, limit=L)
    g = O.backward(x, logits, wgu, wd, k, gout, f, limit=L)
    idx, w = f["idx"], f["w"].copy()
    loss = lambda: float(np.sum(O.combine_forward(x, idx, w, wgu, wd, limit=L) * gout))  # noqa: E731
    for t in range(w.shape[0]):
        for j in range(k):
            assert _fd(loss, w, (t, j)) == pytest.approx(g["dscore"][t, j], rel=1e-7, abs=1e-9)


def test_clamped_mx_layer_without_quantisation_is_the_clamped_layer(monkeypatch):
    rng = np.random.default_rng(9)
    T, d, E, k, I, L = 20, 64, 5, 2, 32, 0.4
    x = rng.standard_normal((T, d))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wgu = rng.standard_normal((E, 2 * I, d)) * 0.2
    wd = rng.standard_normal((E, d, I)) * 0.2
    gout = rng.standard_normal((T, d))
    ref_f = O.forward(x, logits, wgu, wd, k, limit=L)
    ref_b = O.backward(x, logits, wgu, wd, k, gout, ref_f, limit=L)
    monkeypatch.setattr(O, "mx_qdq_blocks", lambda v, axis: np.asarray(v, dtype=np.float64))
    f = O.forward_mx(x, logits, wgu, wd, k, limit=L)
    b = O.backward_mx(x, logits, wgu, wd, k, gout, f, limit=L)
    assert np.allclose(f["out"], ref_f["out"], rtol=1e-12, atol=1e-12)
    for key in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
        assert np.allclose(b[key], ref_b[key], rtol=1e-11, atol=1e-12), key


def test_planted_mistake_gate_clamped_from_below(monkeypatch):
    def wrong(g, u, limit):
        g, u = np.asarray(g, dtype=np.float64), np.asarray(u, dtype=np.float64)
        return (np.maximum(g, -limit), np.clip(u, -limit, limit)) if limit > 0 else (g, u)
    monkeypatch.setattr(O, "_clamps", wrong)
    with pytest.raises(AssertionError):
        test_identity_experts_closed_form(1.5)


def test_bf16_round_matches_torch_conversion():
    import torch
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.standard_normal(4000) * np.exp(rng.uniform(-20, 20, 4000)),
                        [0.0, -0.0, 1.0, 0.2, 0.1875, -3.75e-3]]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.bf16_round(v.astype(np.float64)), ref)
    # hand-worked ties: halfway values go to the even 8-bit significand
    assert O.bf16_round(1.0 + 2.0 ** -8) == 1.0
    assert O.bf16_round(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert O.bf16_round(-(1.0 + 3 * 2.0 ** -8)) == -(1.0 + 2.0 ** -6)


def test_clamp_side_is_decided_on_bf16_h():
    L = 0.25  # a bfloat16 value; the bf16 spacing just above it is 2^-9
    g = np.array([L + 1e-6, L + 2.0 ** -9, L - 1e-6, 0.1])
    u = np.array([0.1, 0.1, 0.1, -(L + 1e-6)])
    dg, du = O.swiglu_backward(g, u, np.ones(4), L)
    assert dg[0] != 0.0  # rounds to L: inside
    assert dg[1] == 0.0  # the next bf16 value: outside
    assert dg[2] != 0.0 and dg[3] != 0.0
    assert du[3] != 0.0  # -(L + 1e-6) rounds to -L: inside
    assert np.all(du[:3] != 0.0)
