"""Pins for the oracle's clamped SwiGLU (a = silu(min(g, L)) * clip(u, -L, L), L > 0).

* identity experts (W_gate = W_up = Id, W_down = Id) give, for any routing
  (the weights sum to one), out = silu(min(x, L)) * clip(x, -L, L) elementwise
  and dx = gout * d/dx of that, written here with scalar math;
* a limit above every pre-activation gives the plain layer bit for bit;
* central finite differences of the clamped forward for every gradient, on
  inputs whose pre-activations stay well away from the clamps' corners;
* the side of a clamp is decided on the exact pre-activation, with the end
  points of the closed interval inside: a closed form on experts whose gate
  pre-activation lands exactly on the limit, or a quarter of a bfloat16 step
  above it (where a rule that rounded h to bfloat16 first would put it
  inside), written with scalar math;
* planted mistakes fail the closed forms: the gate clamped from below instead
  of above, the side decided on h rounded to bfloat16, and an open interval.
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


def _bf16(v):
    """float64 -> nearest bfloat16 -> float64, through torch (used only to plant a mistake)."""
    import torch
    return torch.from_numpy(np.asarray(v, dtype=np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


SIDE_L = 0.5
SIDE_EPS = 2.0 ** -10  # weight of the neighbouring input in the gate rows


def side_layer():
    """One expert (E = k = 1, so w = 1), d = I = 4: W_gate = Id + eps * S with S
    the cyclic shift (g_i = x_i + eps * x_(i+1 mod 4)), W_up = Id, W_down = Id.

    Token 0: g_0 = L + eps / 4 = L + 2^-12, a quarter of the bfloat16 spacing
    (2^-8) above L: outside the gate's interval, although bfloat16 rounding
    would give exactly L.  Token 1: g_0 = L exactly and u_2 = -L exactly: both
    on the closed interval's end points, inside.  Token 2: u_1 = L + 2^-12,
    just outside the up clamp (bfloat16 rounding would again give L)."""
    L, eps, d = SIDE_L, SIDE_EPS, 4
    x = np.array([[L, 0.25, 0.1, -0.3],
                  [L, 0.0, -L, 0.2],
                  [0.1, L + 2.0 ** -12, 0.0, 0.05]])
    shift = np.roll(np.eye(d), 1, axis=1)  # (S x)_i = x_(i+1 mod d)
    wgu = np.concatenate([np.eye(d) + eps * shift, np.eye(d)])[None]
    wd = np.eye(d)[None]
    logits = np.zeros((x.shape[0], 1), dtype=np.float32)
    gout = np.array([[1.0, -0.5, 0.25, 2.0], [0.75, 1.5, -1.0, 0.5], [-2.0, 1.25, 0.3, 0.9]])
    return x, logits, wgu, wd, gout


def side_closed_form(x, gout):
    """out and dx of side_layer by scalar math: gate g_i = x_i + eps x_(i+1),
    up u_i = x_i; a_i = silu(min(g_i, L)) clip(u_i, -L, L); out = a;
    dx_j = dg_j + eps dg_(j-1) + du_j, with dg_i = gout_i clip(u_i) silu'(min(g_i, L))
    where g_i <= L (else 0) and du_i = gout_i silu(min(g_i, L)) where |u_i| <= L (else 0)."""
    L, eps = SIDE_L, SIDE_EPS
    T, d = x.shape
    out = np.zeros((T, d))
    dx = np.zeros((T, d))
    for t in range(T):
        dg, du = [0.0] * d, [0.0] * d
        for i in range(d):
            g = x[t, i] + eps * x[t, (i + 1) % d]
            u = x[t, i]
            gc = g if g <= L else L
            uc = -L if u < -L else (L if u > L else u)
            out[t, i] = py_silu(gc) * uc
            s = py_sigmoid(gc)
            dg[i] = gout[t, i] * uc * s * (1 + gc * (1 - s)) if g <= L else 0.0
            du[i] = gout[t, i] * py_silu(gc) if -L <= u <= L else 0.0
        for j in range(d):
            dx[t, j] = dg[j] + eps * dg[(j - 1) % d] + du[j]
    return out, dx


def test_clamp_side_closed_form():
    x, logits, wgu, wd, gout = side_layer()
    ref_out, ref_dx = side_closed_form(x, gout)
    f = O.forward(x, logits, wgu, wd, 1, limit=SIDE_L)
    g = O.backward(x, logits, wgu, wd, 1, gout, f, limit=SIDE_L)
    assert np.allclose(f["out"], ref_out, rtol=1e-13, atol=1e-15)
    assert np.allclose(g["dx"], ref_dx, rtol=1e-13, atol=1e-15)
    # the cases the layer was built for do occur in the oracle's own h
    h = f["h"]
    assert h[0, 0] > SIDE_L and _bf16(h[0, 0]) == SIDE_L
    assert h[1, 0] == SIDE_L and h[1, 4 + 2] == -SIDE_L
    assert h[2, 4 + 1] > SIDE_L and _bf16(h[2, 4 + 1]) == SIDE_L


def test_clamp_side_closed_form_cpp():
    from oracle import cpp_oracle as C
    x, logits, wgu, wd, gout = side_layer()
    _, ref_dx = side_closed_form(x, gout)
    g = C.backward(x, logits, wgu, wd, 1, gout, nthreads=1, limit=SIDE_L)
    assert np.allclose(g["dx"], ref_dx, rtol=1e-13, atol=1e-15)


def _planted_backward(decide):
    """swiglu_backward with the clamp side taken by `decide(g, u, limit)`."""
    def backward(g, u, da, limit=0.0):
        g, u = np.asarray(g, dtype=np.float64), np.asarray(u, dtype=np.float64)
        gc, uc = O._clamps(g, u, limit)
        da = np.asarray(da, dtype=np.float64)
        dg, du = da * uc * O.silu_grad(gc), da * O.silu(gc)
        if limit > 0:
            keep_g, keep_u = decide(g, u, limit)
            dg, du = np.where(keep_g, dg, 0.0), np.where(keep_u, du, 0.0)
        return dg, du
    return backward


@pytest.mark.parametrize("rule", ["bf16_side", "open_interval"])
def test_planted_wrong_side_rule_fails_closed_form(monkeypatch, rule):
    if rule == "bf16_side":
        decide = lambda g, u, L: (_bf16(g) <= L, np.abs(_bf16(u)) <= L)  # noqa: E731
    else:
        decide = lambda g, u, L: (g < L, np.abs(u) < L)  # noqa: E731
    monkeypatch.setattr(O, "swiglu_backward", _planted_backward(decide))
    with pytest.raises(AssertionError):
        test_clamp_side_closed_form()


def test_planted_right_side_rule_passes(monkeypatch):
    """The planting harness itself: with the definition's rule it passes."""
    monkeypatch.setattr(O, "swiglu_backward", _planted_backward(lambda g, u, L: (g <= L, np.abs(u) <= L)))
    test_clamp_side_closed_form()
