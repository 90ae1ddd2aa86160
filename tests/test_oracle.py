"""Pins for the CPU oracle: checks against what the pages and mathematics fix.

None of these re-types the oracle's formulas: each compares it with a printed
value, a hand-worked example, an independent routine (scipy's normal quantile,
torch's bf16 rounding, exact rational arithmetic, Python triple loops), a
closed form or an invariant.
"""
from fractions import Fraction

import numpy as np
import pytest
from scipy.stats import norm

from oracle import nf4_oracle as O
from tests.conftest import golden_path, read_golden
from qlora_linear_layers_nf4_b200 import workloads as WL


def _printed_levels():
    vals = []
    with open(golden_path("nf4_levels_printed.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                vals.append(float(line))
    return np.array(vals)


# --------------------------------------------------------------------------- levels

def test_levels_match_printed_table():
    printed = _printed_levels()
    assert printed.size == 16
    lv = O.nf4_levels().astype(np.float64)
    assert np.max(np.abs(lv - printed)) <= 5e-4 + 1e-12


def test_levels_invariants():
    lv = O.nf4_levels()
    assert lv.dtype == np.float32
    assert lv[0] == np.float32(-1.0) and lv[15] == np.float32(1.0)
    assert lv[7] == 0.0 and np.sum(lv == 0.0) == 1
    assert np.all(np.diff(lv) > 0)
    assert np.sum(lv < 0) == 7 and np.sum(lv > 0) == 8


def test_levels_against_scipy_quantiles():
    # Independent normal quantile routine (scipy's ndtri) for the same construction.
    delta = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0)
    pos = norm.ppf(np.linspace(delta, 0.5, 9)[:-1])
    neg = -norm.ppf(np.linspace(delta, 0.5, 8)[:-1])
    ref = np.sort(np.concatenate([pos, neg, [0.0]]))
    ref = ref / np.max(np.abs(ref))
    assert np.max(np.abs(ref - O.nf4_levels_f64())) < 1e-12
    # the fp32 table is far from any rounding boundary, so both routines give it bit for bit
    assert np.array_equal(ref.astype(np.float32).view(np.uint32), O.nf4_levels().view(np.uint32))


def test_levels_equally_likely_on_each_side():
    # Page: levels at quantiles so each is equally likely.  Undo the normalisation
    # and check the normal CDF of the raw positive / negative levels is evenly spaced.
    lv = O.nf4_levels_f64()
    scale = norm.ppf(1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0))
    p_pos = norm.cdf(lv[7:] * scale)           # 0 and the 8 positive levels
    p_neg = norm.cdf(-lv[:8] * scale)          # 0 and the 7 negative levels, mirrored
    assert np.allclose(np.diff(p_pos), np.diff(p_pos)[0], rtol=1e-9, atol=1e-12)
    assert np.allclose(np.diff(np.sort(p_neg)), np.diff(np.sort(p_neg))[0], rtol=1e-9, atol=1e-12)


# --------------------------------------------------------------------------- encode

def _exact_nearest(v32: np.float32) -> int:
    """Nearest level by exact rational arithmetic, lowest index on a tie."""
    v = Fraction(float(v32))
    best, best_d = None, None
    for i, lev in enumerate(O.nf4_levels()):
        d = abs(v - Fraction(float(lev)))
        if best_d is None or d < best_d:
            best, best_d = i, d
    return best


def _midpoint_neighbourhood():
    lv = [Fraction(float(x)) for x in O.nf4_levels()]
    vals = [np.float32(0.0), np.float32(-0.0)]
    for i in range(15):
        m = (lv[i] + lv[i + 1]) / 2
        f = np.float32(float(m))
        cand = [f]
        up, dn = f, f
        for _ in range(3):
            up = np.nextafter(up, np.float32(2), dtype=np.float32)
            dn = np.nextafter(dn, np.float32(-2), dtype=np.float32)
            cand += [up, dn]
        vals += cand
    return np.array(vals, dtype=np.float32)


def test_encode_matches_exact_arithmetic_at_midpoints():
    vals = _midpoint_neighbourhood()
    got = O.nearest_code(vals)
    want = np.array([_exact_nearest(v) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_exact_ties_go_to_lower_code():
    lv = [Fraction(float(x)) for x in O.nf4_levels()]
    ties = 0
    for i in range(15):
        m = (lv[i] + lv[i + 1]) / 2
        f = np.float32(float(m))
        if Fraction(float(f)) == m:          # midpoint representable in fp32: an exact tie
            ties += 1
            assert O.nearest_code(np.array([f]))[0] == i
    assert ties == 4                         # four of the fifteen midpoints are fp32 numbers


def test_levels_round_trip_to_own_code():
    assert np.array_equal(O.nearest_code(O.nf4_levels()), np.arange(16, dtype=np.uint8))


def test_worked_example_block():
    g = read_golden("nf4_worked_example.txt")
    w = np.array([float(v) for v in g["w"]], dtype=np.float32)
    q = O.quantize(w, block_size=8)
    assert q["absmax"][0] == np.float32(g["absmax"][0])
    assert np.array_equal(O.unpack_codes(q["codes"]), np.array([int(c) for c in g["codes"]]))
    assert np.array_equal(q["codes"], np.array([int(c, 16) for c in g["packed"]], dtype=np.uint8))


def test_pack_unpack_lossless():
    rng = np.random.default_rng(11)
    c = rng.integers(0, 16, size=4096, dtype=np.uint8)
    assert np.array_equal(O.unpack_codes(O.pack_codes(c)), c)
    p = rng.integers(0, 256, size=1024, dtype=np.uint8)
    assert np.array_equal(O.pack_codes(O.unpack_codes(p)), p)


def _reciprocal_failures(n=64):
    """fp32 values a with fp32(a * fp32(1/a)) != 1 (multiplying by a reciprocal is wrong here)."""
    rng = np.random.default_rng(5)
    a = (rng.random(200000, dtype=np.float32) * np.float32(0.1) + np.float32(1e-3)).astype(np.float32)
    bad = a[(a * (np.float32(1.0) / a)).astype(np.float32) != np.float32(1.0)]
    assert bad.size >= n
    return bad[:n]


def test_absmax_element_maps_to_pm_one_exactly():
    bad = _reciprocal_failures()
    rng = np.random.default_rng(3)
    blocks = rng.standard_normal((bad.size, 64)).astype(np.float32) * np.float32(0.001)
    idx = rng.integers(0, 64, size=bad.size)
    sign = np.where(rng.random(bad.size) < 0.5, -1.0, 1.0).astype(np.float32)
    blocks[np.arange(bad.size), idx] = sign * bad
    q = O.quantize(blocks, 64)
    codes = O.unpack_codes(q["codes"]).reshape(bad.size, 64)
    got = codes[np.arange(bad.size), idx]
    assert np.array_equal(got, np.where(sign > 0, 15, 0))
    deq = O.dequantize(q).reshape(bad.size, 64)
    assert np.array_equal(deq[np.arange(bad.size), idx], sign * bad)


def test_all_zero_tensor_quantizes():
    # export.rs unit tests quantize an all-zeros tensor and expect success.
    q = O.quantize(np.zeros((32, 32), np.float32), 64, double=True)
    assert np.all(q["codes"] == 0x77)
    assert np.all(q["absmax"] == 0) and q["absmax_scale"] == 0 and np.all(q["absmax_q"] == 0)
    d = O.dequantize(q)
    assert np.all(d == 0) and not np.any(np.signbit(d))


def test_scaled_levels_reproduce_exactly():
    lv = O.nf4_levels()
    rng = np.random.default_rng(2)
    blocks = []
    for e in range(-8, 4):
        perm = rng.permutation(np.concatenate([np.arange(16)] * 4))
        blocks.append((lv[perm] * np.float32(2.0 ** e)).astype(np.float32))
    w = np.stack(blocks)
    q = O.quantize(w, 64)
    assert np.array_equal(O.dequantize(q), w)


def test_round_trip_error_bound():
    w = WL.draw_weight((256, 512), seed=9)
    for double in (False, True):
        q = O.quantize(w, 64, double=double)
        d = O.dequantize(q)
        lv = O.nf4_levels().astype(np.float64)
        half_gap = np.max(np.diff(lv)) / 2           # 0.1519, between -1 and -0.696
        assert abs(half_gap - 0.15190359) < 1e-6
        absmax = np.repeat(q["absmax"], 64).reshape(w.shape).astype(np.float64)
        bound = absmax * half_gap * (1 + 1e-6)
        if double:
            scale = np.repeat(O.block_scales(q), 64).reshape(w.shape).astype(np.float64)
            bound = bound + np.abs(scale - absmax) + 1e-12
        assert np.all(np.abs(w.astype(np.float64) - d) <= bound + 1e-12)


def test_refuses_bad_shapes_and_nonfinite():
    with pytest.raises(ValueError):
        O.quantize(np.zeros(64, np.float32), 63)
    w = np.zeros(64, np.float32)
    w[3] = np.inf
    with pytest.raises(ValueError):
        O.quantize(w, 64)


# --------------------------------------------------------------------------- double quant

def test_double_quant_invariants():
    w = WL.draw_weight((512, 256), seed=4)
    q = O.quantize(w, 64, double=True)
    absmax = q["absmax"].astype(np.float64)
    s_g = float(q["absmax_scale"])
    assert q["absmax_q"][np.argmax(absmax)] == 255
    assert abs(s_g - absmax.max() / 255) <= 1e-7 * s_g
    dec = O.block_scales(q).astype(np.float64)
    assert np.all(np.abs(dec - absmax) <= s_g / 2 + 4 * np.spacing(absmax.astype(np.float32)))
    order = np.argsort(absmax, kind="stable")
    assert np.all(np.diff(q["absmax_q"][order].astype(int)) >= 0)       # monotone


def test_double_quant_half_even_rounding():
    # absmax values chosen so absmax / s_g lands exactly on k + 0.5 for small k.
    s_g = np.float32(255.0) / np.float32(255.0)
    absmax = np.array([255.0, 0.5, 1.5, 2.5, 3.5, 254.5], dtype=np.float32)
    q, sg = O.double_quant(absmax)
    assert sg == s_g
    assert list(q) == [255, 0, 2, 2, 4, 254]


# --------------------------------------------------------------------------- dequant rounding

def test_bf16_round_matches_torch():
    import torch
    rng = np.random.default_rng(8)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * np.float32(0.02),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1e-40], dtype=np.float32),
    ])
    u = rng.integers(0, 2 ** 16, size=5000, dtype=np.uint32) << 16 | np.uint32(0x8000)
    x = np.concatenate([x, u.view(np.float32)[np.isfinite(u.view(np.float32))]])
    ours = O.bf16_round(x)
    theirs = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, theirs)


def _weight_with_scales(scales):
    # One block per scale, the 16 codes twice each: every level times every scale.
    codes = np.tile(np.arange(16, dtype=np.uint8), 4)
    q = {"codes": O.pack_codes(np.tile(codes, len(scales))),
         "absmax": np.asarray(scales, dtype=np.float32), "shape": (len(scales), 64),
         "block_size": 64}
    return q


def test_f16_dequant_matches_torch_half():
    # The F16 dequant is the fp32 product rounded to binary16, nearest, ties to
    # even.  Checked against torch's own fp32 -> f16 conversion on scales that
    # put products on f16 halfway points (both tie directions), past the f16
    # maximum (overflow to inf, and the 65520 tie that rounds to inf), into
    # the subnormal range (including the tie at half the smallest subnormal,
    # which rounds to zero) and on ordinary random scales.
    import torch
    lv = O.nf4_levels()
    ties = [1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11, 2.0 ** -14 * (1 + 2.0 ** -11)]
    big = [65504.0, 65519.0, 65520.0, 70000.0, 3.0e38]
    tiny = [2.0 ** -25, 3 * 2.0 ** -25, 1e-6, 6.0e-8, 2.0 ** -24, 1e-30]
    rand = list(np.random.default_rng(12).uniform(0.001, 2.0, 200))
    # scales that make a level land exactly on an f16 tie: level * s = 1 + 2^-11 etc.
    on_tie = [np.float32(t / float(lv[c])) for t in (1.0 + 2.0 ** -11, 2.0 ** -25) for c in (9, 12, 14)]
    scales = np.array(ties + big + tiny + rand + on_tie, dtype=np.float32)
    q = _weight_with_scales(scales)
    w32 = O.dequantize(q, "f32")
    with np.errstate(over="ignore"):       # overflow to inf is one of the cases
        ours = O.dequantize(q, "f16")
    theirs = torch.from_numpy(w32).half().numpy()
    assert ours.dtype == np.float16
    assert np.array_equal(ours.view(np.uint16), theirs.view(np.uint16))
    # the classes really occur: infinities, subnormals, zeros from nonzero products, exact ties
    assert np.any(np.isinf(ours)) and np.any((ours != 0) & (np.abs(ours) < np.float16(6.104e-5)))
    assert np.any((ours == 0) & (w32 != 0))
    assert ours[0, 15] == np.float16(1.0) and ours[1, 15] == np.float16(1.0 + 2.0 ** -9)


def test_dequant_single_product_per_element():
    lv = O.nf4_levels()
    rng = np.random.default_rng(1)
    w = WL.draw_weight((64, 128), seed=21)
    q = O.quantize(w, 64)
    d = O.dequantize(q)
    codes = O.unpack_codes(q["codes"]).reshape(64, 128)
    # element by element in Python floats rounded once to fp32
    for _ in range(200):
        i, j = rng.integers(0, 64), rng.integers(0, 128)
        s = q["absmax"][(i * 128 + j) // 64]
        assert d[i, j] == np.float32(float(lv[codes[i, j]]) * float(s))


# --------------------------------------------------------------------------- forward / backward

def test_worked_linear_example():
    g = read_golden("qlora_worked_example.txt")
    f = lambda k: np.array([float(v) for v in g[k]])
    x, w, a, b = f("x")[None, :], f("w")[None, :], f("a")[None, :], f("b")[None, :]
    alpha = float(g["alpha"][0])
    y, t = O.qlora_forward(x, w, a, b, alpha)
    assert y[0, 0] == float(g["y"][0]) and t[0, 0] == float(g["t"][0])
    d_a, d_b, d_x = O.qlora_backward(x, w, a, b, alpha, f("dy")[None, :])
    assert np.array_equal(d_b.ravel(), f("dB"))
    assert np.array_equal(d_a.ravel(), f("dA"))
    assert np.array_equal(d_x.ravel(), f("dx"))
    # the same example with a bias on the output feature
    yb, tb = O.qlora_forward(x, w, a, b, alpha, bias=f("bias"))
    assert yb[0, 0] == float(g["y_bias"][0]) and tb[0, 0] == float(g["t"][0])


def test_bias_adds_once_per_output_feature():
    # Brute force with a bias: every row of y gains exactly the bias vector.
    inp, w_hat, x, a, b, dy = _tiny()
    bias = np.random.default_rng(5).standard_normal(w_hat.shape[0]) * 0.1
    y0, _ = O.qlora_forward(x, w_hat, a, b, inp.case.alpha)
    y1, _ = O.qlora_forward(x, w_hat, a, b, inp.case.alpha, bias=bias)
    s = inp.case.alpha / inp.case.r
    y_bf = (O.matmul_bruteforce(x, w_hat.T) + s * O.matmul_bruteforce(O.matmul_bruteforce(x, a.T), b.T)
            + np.repeat(bias[None, :], x.shape[0], axis=0))
    assert np.max(np.abs(y1 - y_bf)) <= 1e-12 * np.max(np.abs(y_bf))
    # a bias of all zeros changes nothing, and adding one is a per-column shift
    assert np.array_equal(O.qlora_forward(x, w_hat, a, b, inp.case.alpha, bias=np.zeros_like(bias))[0], y0)
    assert np.allclose(y1 - y0, np.broadcast_to(bias, y0.shape), rtol=0, atol=1e-12)


def _tiny():
    inp = WL.draw_linear(WL.TINY)
    q = O.quantize(inp.w, 64)
    w_hat = O.bf16_to_f32(O.dequantize(q, "bf16"))
    f = WL.bf16_bits_to_f32
    return inp, w_hat, f(inp.x), f(inp.a), f(inp.b), f(inp.dy)


def test_forward_matches_bruteforce():
    inp, w_hat, x, a, b, dy = _tiny()
    y, t = O.qlora_forward(x, w_hat, a, b, inp.case.alpha)
    s = inp.case.alpha / inp.case.r
    t_bf = O.matmul_bruteforce(x, a.T)
    y_bf = O.matmul_bruteforce(x, w_hat.T) + s * O.matmul_bruteforce(t_bf, b.T)
    assert np.max(np.abs(y - y_bf)) <= 1e-12 * np.max(np.abs(y_bf))
    assert np.max(np.abs(t - t_bf)) <= 1e-12 * np.max(np.abs(t_bf))


def test_merge_identity():
    # Equation 6.3.6: x (W' + (alpha/r) B A)^T equals the adapter-on-base forward.
    inp, w_hat, x, a, b, dy = _tiny()
    y, _ = O.qlora_forward(x, w_hat, a, b, inp.case.alpha)
    merged = w_hat.astype(np.float64) + (inp.case.alpha / inp.case.r) * O.matmul_bruteforce(b, a)
    y2 = O.matmul_bruteforce(x, merged.T)
    assert np.max(np.abs(y - y2)) <= 1e-11 * np.max(np.abs(y))


def test_special_cases():
    inp, w_hat, x, a, b, dy = _tiny()
    alpha = inp.case.alpha
    # B = 0: the base matmul alone
    y0, _ = O.qlora_forward(x, w_hat, a, np.zeros_like(b), alpha)
    assert np.array_equal(y0, x.astype(np.float64) @ w_hat.T.astype(np.float64))
    # zero base weight: only the adapter term remains
    q0 = O.quantize(np.zeros_like(inp.w), 64)
    w0 = O.bf16_to_f32(O.dequantize(q0, "bf16"))
    assert np.all(w0 == 0)
    ya, t = O.qlora_forward(x, w0, a, b, alpha)
    assert np.allclose(ya, (alpha / inp.case.r) * O.matmul_bruteforce(O.matmul_bruteforce(x, a.T), b.T),
                       rtol=1e-12, atol=1e-15)
    # A = 0: dB vanishes
    d_a, d_b, d_x = O.qlora_backward(x, w_hat, np.zeros_like(a), b, alpha, dy)
    assert np.all(d_b == 0)


def test_finite_difference_gradients():
    inp, w_hat, x, a, b, dy = _tiny()
    alpha = inp.case.alpha
    x, a, b, dy = (v.astype(np.float64) for v in (x, a, b, dy))
    d_a, d_b, d_x = O.qlora_backward(x, w_hat, a, b, alpha, dy)

    def loss(xx, aa, bb):
        return float(np.sum(dy * O.qlora_forward(xx, w_hat, aa, bb, alpha)[0]))

    h = 1e-3
    rng = np.random.default_rng(0)
    for i in range(a.shape[0]):
        for j in range(0, a.shape[1], 7):
            ap, am = a.copy(), a.copy()
            ap[i, j] += h
            am[i, j] -= h
            fd = (loss(x, ap, b) - loss(x, am, b)) / (2 * h)
            assert abs(fd - d_a[i, j]) <= 1e-8 * max(1.0, abs(d_a[i, j]))
    for i in range(0, b.shape[0], 5):
        for j in range(b.shape[1]):
            bp, bm = b.copy(), b.copy()
            bp[i, j] += h
            bm[i, j] -= h
            fd = (loss(x, a, bp) - loss(x, a, bm)) / (2 * h)
            assert abs(fd - d_b[i, j]) <= 1e-8 * max(1.0, abs(d_b[i, j]))
    for _ in range(256):
        i, j = rng.integers(0, x.shape[0]), rng.integers(0, x.shape[1])
        xp, xm = x.copy(), x.copy()
        xp[i, j] += h
        xm[i, j] -= h
        fd = (loss(xp, a, b) - loss(xm, a, b)) / (2 * h)
        assert abs(fd - d_x[i, j]) <= 1e-8 * max(1.0, abs(d_x[i, j]))


# --------------------------------------------------------------------------- merge

def _tiny_q():
    inp, w_hat, x, a, b, dy = _tiny()
    q = O.quantize(inp.w, 64, double=inp.case.double_quant)
    return inp, q, x, a, b


def test_merge_equals_forward_on_the_fp32_base():
    # Equation 6.3.6 with the fp32 dequant as the base: the merged weight
    # applied to x equals the adapter-on-base forward (an independent path).
    inp, q, x, a, b = _tiny_q()
    m = O.merge(q, a, b, inp.case.alpha, "f64")
    w32 = O.dequantize(q, "f32")
    y, _ = O.qlora_forward(x, w32, a, b, inp.case.alpha)
    y2 = O.matmul_bruteforce(x, m.T)
    assert np.max(np.abs(y - y2)) <= 1e-11 * np.max(np.abs(y))


def test_merge_matches_bruteforce_and_rounds_once():
    inp, q, x, a, b = _tiny_q()
    s = inp.case.alpha / inp.case.r
    want = O.dequantize(q, "f32").astype(np.float64) + s * O.matmul_bruteforce(b, a)
    m = O.merge(q, a, b, inp.case.alpha, "f64")
    assert np.max(np.abs(m - want)) <= 1e-13 * np.max(np.abs(want))
    # f32: the nearest fp32 of the exact sum (checked with exact rationals on a sample)
    m32 = O.merge(q, a, b, inp.case.alpha, "f32")
    rng = np.random.default_rng(0)
    for idx in rng.integers(0, m32.size, 64):
        exact = Fraction(float(want.flat[idx]))
        got = Fraction(float(m32.flat[idx]))
        lo = np.nextafter(m32.flat[idx], np.float32(-np.inf))
        hi = np.nextafter(m32.flat[idx], np.float32(np.inf))
        assert abs(got - exact) <= abs(Fraction(float(lo)) - exact)
        assert abs(got - exact) <= abs(Fraction(float(hi)) - exact)
    # bf16: the fp32 value rounded to bf16 (torch's rounding as the independent routine)
    import torch
    mb = O.merge(q, a, b, inp.case.alpha, "bf16")
    tb = torch.from_numpy(m32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mb, tb)


def test_merge_special_cases():
    inp, q, x, a, b = _tiny_q()
    # B = 0: the merge is the plain dequant, bit for bit in both dtypes
    assert np.array_equal(O.merge(q, a, np.zeros_like(b), inp.case.alpha, "bf16"),
                          O.dequantize(q, "bf16"))
    assert np.array_equal(O.merge(q, a, np.zeros_like(b), inp.case.alpha, "f32").view(np.uint32),
                          O.dequantize(q, "f32").view(np.uint32))
    # zero base: only the low-rank update remains
    q0 = O.quantize(np.zeros_like(inp.w), 64)
    s = inp.case.alpha / inp.case.r
    assert np.allclose(O.merge(q0, a, b, inp.case.alpha, "f64"), s * O.matmul_bruteforce(b, a),
                       rtol=1e-13, atol=0)


def test_bf16_and_f16_widening_is_exact():
    # The typed quantizer's definition rests on widening bf16 / f16 to fp32
    # exactly; checked against torch's conversions on every bf16 pattern and
    # a sweep of f16 values.
    import torch
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    mine = WL.bf16_bits_to_f32(bits)
    theirs = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    same = (mine.view(np.uint32) == theirs.view(np.uint32)) | (np.isnan(mine) & np.isnan(theirs))
    assert np.all(same)
    h = bits.view(np.float16)
    assert np.all((h.astype(np.float32) == torch.from_numpy(h).float().numpy()) | np.isnan(h))


# --------------------------------------------------------------------------- tail blocks (R19)

def test_tail_block_is_its_own_quantization():
    # The short last block must come out exactly as that block quantized on its
    # own (a full-block quantization with block size = its length, an
    # independent path), and the full blocks as before.
    rng = np.random.default_rng(8)
    for n, bs in [(100, 64), (1000, 64), (130, 32), (37, 8), (65, 64)]:
        w = (rng.standard_normal(n) * 0.02).astype(np.float32)
        q = O.quantize(w, bs)
        full = (n // bs) * bs
        t = n - full
        codes = O.unpack_codes(q["codes"])[:n]
        if full:
            qf = O.quantize(w[:full], bs)
            assert np.array_equal(codes[:full], O.unpack_codes(qf["codes"]))
            assert np.array_equal(q["absmax"][:-1], qf["absmax"])
        if t % 2 == 0:
            qt = O.quantize(w[full:], t)
            assert np.array_equal(codes[full:], O.unpack_codes(qt["codes"]))
            assert q["absmax"][-1] == qt["absmax"][0]
        assert q["absmax"][-1] == np.max(np.abs(w[full:]))       # its own elements only
        assert q["codes"].size == (n + 1) // 2
        if n % 2:
            assert q["codes"][-1] & 0x0F == 7                      # the pad nibble
        # round trip within the largest half gap of the block's absmax
        d = O.dequantize(q, "f32")
        scale = np.repeat(q["absmax"], bs)[:n]
        assert np.all(np.abs(d - w) <= scale * 0.1519 + 1e-12)


def test_tail_block_double_quant_counts_every_block():
    w = WL.draw_weight((1, 1000), seed=12).reshape(-1)
    q = O.quantize(w, 64, double=True)
    assert q["absmax_q"].size == 16                   # 15 full blocks + the tail
    assert q["absmax_q"].max() == 255


# --------------------------------------------------------------------------- a part of a tensor (R6)

def test_double_quant_of_a_part_uses_the_whole_max():
    # One scale of scales per tensor: the blocks of a part, encoded against the
    # tensor's max, are exactly those blocks of the whole tensor's encoding.
    w = WL.draw_weight((48, 256), seed=21)
    w[40:] *= np.float32(6.0)                              # the max lies in the last part
    whole = O.quantize(w, 64, double=True)
    g = np.float32(whole["absmax"].max())
    parts = [w[:16], w[16:40], w[40:]]
    qs, ss = [], []
    for part in parts:
        qp = O.quantize(part, 64, double=False)
        q, s = O.double_quant(qp["absmax"], g=g)
        qs.append(q)
        ss.append(s)
    assert np.array_equal(np.concatenate(qs), whole["absmax_q"])
    assert all(s == np.float32(whole["absmax_scale"]) for s in ss)
    # a part encoded against its own max differs: the exchange is needed
    own, _ = O.double_quant(O.quantize(parts[0], 64)["absmax"])
    assert not np.array_equal(own, qs[0])
    # the default max is the part's own
    a = O.quantize(parts[1], 64)["absmax"]
    q_default, s_default = O.double_quant(a)
    q_given, s_given = O.double_quant(a, g=a.max())
    assert np.array_equal(q_default, q_given) and s_default == s_given


def test_merge_f16_is_the_f16_rounding_of_the_fp32_merge():
    """The merge's f16 output (R16 with the F16 compute dtype) is the
    round-to-nearest-even f16 of the fp32 merged value, overflow to inf."""
    import torch
    rng = np.random.default_rng(77)
    w = (rng.standard_normal((8, 128)) * 0.02).astype(np.float32)
    w[0, :64] *= 5e6                  # one block whose merged values pass 65504
    q = O.quantize(w, 64, double=False)
    a = rng.standard_normal((8, 128)) * 0.1
    b = rng.standard_normal((8, 8)) * 0.01
    m32 = O.merge(q, a, b, 16.0, "f32")
    want = torch.from_numpy(m32).half().numpy()
    got = O.merge(q, a, b, 16.0, "f16")
    assert got.dtype == np.float16
    assert np.array_equal(got.view(np.uint16), want.view(np.uint16))
    assert np.isinf(got[0, :64]).any()
