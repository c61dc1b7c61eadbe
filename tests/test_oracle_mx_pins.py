"""Pins for the oracle's MXFP8 operand quantisation and its MXFP8 layer.

* the E4M3 grid is rebuilt from the format's bit fields (sign, 4 exponent
  bits with bias 7, 3 mantissa bits, subnormals, 448 as the largest finite
  magnitude): every code is a fixed point of e4m3_round, midpoints go to the
  even code, larger magnitudes saturate;
* the block scale exponent is checked against a brute-force search;
* qdq is idempotent, scale-equivariant by powers of two and block-local;
* with quantisation switched off, forward_mx / backward_mx reproduce the
  pinned bf16 forward / backward (so their GEMM decomposition is right).
"""
import math

import numpy as np
import pytest

from oracle import moe_oracle as O

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def e4m3_codes():
    """All finite non-negative E4M3 values from the bit fields (S.EEEE.MMM, bias 7)."""
    vals = set()
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue  # the NaN code
            if e == 0:
                v = (m / 8.0) * 2.0 ** (1 - 7)
            else:
                v = (1 + m / 8.0) * 2.0 ** (e - 7)
            vals.add(v)
    return sorted(vals)


def test_e4m3_codes_are_fixed_points_and_max_is_448():
    codes = e4m3_codes()
    assert max(codes) == 448.0 and len(codes) == 127
    arr = np.array(codes + [-c for c in codes])
    assert np.array_equal(O.e4m3_round(arr), arr)


def test_e4m3_midpoints_round_to_even_code():
    codes = e4m3_codes()
    for lo, hi in zip(codes[:-1], codes[1:]):
        mid = (lo + hi) / 2.0
        # even code = even mantissa field; consecutive codes alternate parity
        lo_code = codes.index(lo)
        expect = lo if lo_code % 2 == 0 else hi
        assert O.e4m3_round(np.array([mid]))[0] == expect, (lo, hi)
        assert O.e4m3_round(np.array([math.nextafter(mid, 0)]))[0] == lo
        assert O.e4m3_round(np.array([math.nextafter(mid, 1e9)]))[0] == hi


def test_e4m3_saturates():
    assert np.array_equal(O.e4m3_round(np.array([449.0, 1e6, -500.0])), [448.0, 448.0, -448.0])


def test_scale_exponent_bruteforce():
    rng = np.random.default_rng(1)
    amax = np.concatenate([rng.lognormal(0, 6, 500), [448.0, 448.0 * 2 ** 3, 448.0 * 2 ** -5, 1e-30, 0.0]])
    got = O.mx_scale_exponent(amax)
    for a, s in zip(amax, got):
        if a == 0:
            assert s == 0
            continue
        best = next(t for t in range(-127, 128) if a <= 448.0 * 2.0 ** t)
        assert s == best, (a, s, best)


def test_qdq_idempotent_equivariant_blocklocal():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((6, 96)) * np.exp(rng.standard_normal((6, 1)) * 3)
    q = O.mx_qdq_blocks(v, axis=1)
    assert np.array_equal(O.mx_qdq_blocks(q, axis=1), q)
    assert np.array_equal(O.mx_qdq_blocks(v * 2.0 ** 5, axis=1), q * 2.0 ** 5)
    v2 = v.copy()
    v2[:, 32:64] *= 1000.0  # only the middle block's scale changes
    q2 = O.mx_qdq_blocks(v2, axis=1)
    assert np.array_equal(q2[:, :32], q[:, :32]) and np.array_equal(q2[:, 64:], q[:, 64:])
    # the block maximum of a block whose amax is 448 * 2^s is kept exactly
    w = rng.standard_normal(32) * 0.1
    w[7] = 448.0 * 2.0 ** -6
    assert O.mx_qdq_blocks(w[None, :], axis=1)[0, 7] == w[7]
    # relative error per element is at most half an E4M3 spacing (2^-4) above the subnormal range
    big = np.abs(v) > 2.0 ** -6 * np.max(np.abs(v))
    assert np.max(np.abs(q - v)[big] / np.abs(v)[big]) <= 2.0 ** -4 + 1e-12


def test_mx_layer_without_quantisation_is_the_bf16_layer(monkeypatch):
    rng = np.random.default_rng(3)
    T, d, E, k, I = 20, 64, 5, 2, 32
    x = rng.standard_normal((T, d))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wgu = rng.standard_normal((E, 2 * I, d)) * 0.2
    wd = rng.standard_normal((E, d, I)) * 0.2
    gout = rng.standard_normal((T, d))
    ref_f = O.forward(x, logits, wgu, wd, k)
    ref_b = O.backward(x, logits, wgu, wd, k, gout, ref_f)
    monkeypatch.setattr(O, "mx_qdq_blocks", lambda v, axis: np.asarray(v, dtype=np.float64))
    f = O.forward_mx(x, logits, wgu, wd, k)
    b = O.backward_mx(x, logits, wgu, wd, k, gout, f)
    assert np.allclose(f["out"], ref_f["out"], rtol=1e-12, atol=1e-12)
    for key in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
        assert np.allclose(b[key], ref_b[key], rtol=1e-11, atol=1e-12), key


def test_mx_layer_close_to_bf16_layer():
    rng = np.random.default_rng(4)
    T, d, E, k, I = 40, 64, 4, 2, 32
    x = rng.standard_normal((T, d))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wgu = rng.standard_normal((E, 2 * I, d)) * 0.1
    wd = rng.standard_normal((E, d, I)) * 0.1
    gout = rng.standard_normal((T, d))
    f = O.forward_mx(x, logits, wgu, wd, k)
    ref = O.forward(x, logits, wgu, wd, k)
    rel = np.linalg.norm(f["out"] - ref["out"]) / np.linalg.norm(ref["out"])
    assert 1e-3 < rel < 0.1  # quantised, but only at E4M3 precision
    b = O.backward_mx(x, logits, wgu, wd, k, gout, f)
    rb = O.backward(x, logits, wgu, wd, k, gout, ref)
    for key in ("dx", "dwgu", "dwd"):
        rel = np.linalg.norm(b[key] - rb[key]) / np.linalg.norm(rb[key])
        assert rel < 0.1, key


def test_planted_mistake_scale_off_by_one(monkeypatch):
    real = O.mx_scale_exponent
    monkeypatch.setattr(O, "mx_scale_exponent", lambda a: real(a) - 1)  # would saturate block maxima
    with pytest.raises(AssertionError):
        test_scale_exponent_bruteforce()


def test_sampled_mx_variants_agree_with_full():
    rng = np.random.default_rng(6)
    T, d, E, k, I = 48, 64, 5, 3, 32
    x = rng.standard_normal((T, d))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wgu = rng.standard_normal((E, 2 * I, d)) * 0.2
    wd = rng.standard_normal((E, d, I)) * 0.2
    gout = rng.standard_normal((T, d))
    f = O.forward_mx(x, logits, wgu, wd, k)
    b = O.backward_mx(x, logits, wgu, wd, k, gout, f)
    toks = [0, 5, 47]
    ft = O.forward_tokens_mx(x, logits, wgu, wd, k, toks)
    assert np.allclose(ft["out"], f["out"][toks], rtol=1e-12, atol=1e-12)
    bt = O.backward_tokens_mx(x, logits, wgu, wd, k, gout, toks)
    for key in ("dx", "dscore", "dlogits"):
        assert np.allclose(bt[key], b[key][toks], rtol=1e-11, atol=1e-12), key
    be = O.backward_experts_mx(x, logits, wgu, wd, k, gout, [0, 3])
    for e in (0, 3):
        assert np.allclose(be[e][0], b["dwgu"][e], rtol=1e-11, atol=1e-12)
        assert np.allclose(be[e][1], b["dwd"][e], rtol=1e-11, atol=1e-12)


def test_backward_on_given_h():
    """backward(h=...) uses the given pre-activations: the forward's own h gives
    the plain backward bit for bit; the MXFP8 forward's h gives the bf16 backward
    that follows an MXFP8 forward (and differs from the plain one)."""
    rng = np.random.default_rng(8)
    T, d, E, k, I = 24, 64, 5, 2, 32
    x = rng.standard_normal((T, d))
    logits = rng.standard_normal((T, E)).astype(np.float32)
    wgu = rng.standard_normal((E, 2 * I, d)) * 0.2
    wd = rng.standard_normal((E, d, I)) * 0.2
    gout = rng.standard_normal((T, d))
    f = O.forward(x, logits, wgu, wd, k)
    b = O.backward(x, logits, wgu, wd, k, gout, f)
    bh = O.backward(x, logits, wgu, wd, k, gout, f, h=f["h"])
    for key in ("dx", "dwgu", "dwd", "dscore", "dlogits"):
        assert np.array_equal(b[key], bh[key]), key
    fm = O.forward_mx(x, logits, wgu, wd, k)
    bm = O.backward(x, logits, wgu, wd, k, gout, fm, h=fm["h"])
    rel = np.linalg.norm(bm["dscore"] - b["dscore"]) / np.linalg.norm(b["dscore"])
    assert 1e-4 < rel < 0.1


# ----------------------------------------------------------------------------
# Where the weight-gradient blocks start.  Reading: the K dimension of a weight
# gradient is one expert's own tokens, in dispatch order (tokens ascending), and
# its blocks of 32 start at that expert's first token -- a property of the
# expert alone, not of where its group sits among the other experts' pairs.
# ----------------------------------------------------------------------------
def _block_origin_case(split):
    """k = 1, E = 3.  Tokens 37..99 go to expert 1 in both variants; tokens
    0..split-1 go to expert 0 and split..36 to expert 2, so expert 1's first
    sorted position is `split` while its own token sequence stays the same."""
    rng = np.random.default_rng(5)
    T, d, E, I = 100, 64, 3, 32
    x = rng.standard_normal((T, d))
    gout = rng.standard_normal((T, d))
    # a large row at expert 1's 29th token: which rows share its block (and so
    # its scale) depends on where the blocks start
    gout[37 + 28] *= 64.0
    wgu = rng.standard_normal((E, 2 * I, d)) * 0.2
    wd = rng.standard_normal((E, d, I)) * 0.2
    choice = np.where(np.arange(T) < split, 0, np.where(np.arange(T) < 37, 2, 1))
    logits = np.full((T, E), -4.0, dtype=np.float32)
    logits[np.arange(T), choice] = 4.0
    logits += rng.uniform(0, 0.5, (T, E)).astype(np.float32)  # weights vary per token
    logits[np.arange(T), choice] += 4.0
    return x, logits, wgu, wd, gout


def _qdq32_loop(rows):
    """Blocks of 32 consecutive rows, the first starting at row 0, each column
    of a block quantised with its own scale: a plain loop over the blocks."""
    rows = np.asarray(rows, dtype=np.float64)
    out = np.zeros_like(rows)
    for b0 in range(0, rows.shape[0], 32):
        blk = rows[b0:b0 + 32]
        for c in range(rows.shape[1]):
            col = blk[:, c]
            amax = float(np.max(np.abs(col)))
            s = 0
            if amax > 0:
                s = -127
                while amax > 448.0 * 2.0 ** s:
                    s += 1
            out[b0:b0 + 32, c] = O.e4m3_round(col / 2.0 ** s) * 2.0 ** s
    return out


def test_wgrad_blocks_start_at_the_experts_first_token():
    dws = []
    for split in (37, 30):
        x, logits, wgu, wd, gout = _block_origin_case(split)
        f = O.forward_mx(x, logits, wgu, wd, 1)
        assert int(f["offsets"][1]) == split and int(f["counts"][1]) == 63
        b = O.backward_mx(x, logits, wgu, wd, 1, gout, f)
        dws.append(b["dwd"][1])
        # brute force on expert 1's own token sequence (tokens 37..99 ascending)
        pairs = f["perm"][f["offsets"][1]:f["offsets"][2]].astype(np.int64)
        assert np.array_equal(pairs, np.arange(37, 100))
        ref = _qdq32_loop(gout[pairs]).T @ _qdq32_loop(f["aw"][pairs])
        assert np.allclose(b["dwd"][1], ref, rtol=1e-13, atol=1e-13)
    # expert 1's gradient does not move when its group's start among the sorted pairs moves
    assert np.array_equal(dws[0], dws[1])


def test_wgrad_block_origin_pin_discriminates():
    """Blocks aligned to the global sorted position instead (origin 0 of all
    pairs) give a different dW_down for the expert that starts at 37."""
    x, logits, wgu, wd, gout = _block_origin_case(37)
    f = O.forward_mx(x, logits, wgu, wd, 1)
    b = O.backward_mx(x, logits, wgu, wd, 1, gout, f)
    lo, hi = int(f["offsets"][1]), int(f["offsets"][2])
    pairs = f["perm"][lo:hi].astype(np.int64)
    pad = lo % 32  # rows of the global block that belong to expert 0: zeros here
    g = np.concatenate([np.zeros((pad, gout.shape[1])), gout[pairs]])
    a = np.concatenate([np.zeros((pad, f["aw"].shape[1])), f["aw"][pairs]])
    glob = _qdq32_loop(g).T @ _qdq32_loop(a)
    assert not np.allclose(b["dwd"][1], glob, rtol=1e-6, atol=1e-9)
