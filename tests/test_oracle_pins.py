"""Pins of the CPU oracle against what the pages and mathematics fix (no GPU).

Each test checks the oracle against something other than itself:
  * IEEE conversions done by a library (numpy's float16 / rint),
  * exact rational arithmetic (fractions.Fraction),
  * brute-force nearest-code search over every admissible code,
  * closed forms (constant weights, ones / one-hot activations, g = 0, a
    boosted head row, lowest-index ties),
  * the bundle sizes the pages print (tests/golden/bundle_sizes.txt).
A plausible slip in the oracle -- a dropped term, a wrong sign or index, a
transposed operand, a truncating instead of rounding conversion -- fails one
of these.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from int4_quantized_decode_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f16_np(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def np_f16_bits(x32):
    return np.asarray(x32, dtype=np.float32).astype(np.float16).view(np.uint16)


# ------------------------------------------------------------------ fp16 ---

def _f32_probe_values():
    rng = np.random.default_rng(7)
    vals = []
    allh = np.arange(0, 0x7C00, dtype=np.uint16)          # every finite positive fp16
    h64 = allh.view(np.float16).astype(np.float64)
    mids = (h64[:-1] + h64[1:]) / 2                         # exact ties (12 bits)
    vals += [h64, mids]
    mids32 = mids.astype(np.float32)
    vals += [np.nextafter(mids32, np.float32(np.inf)).astype(np.float64),
             np.nextafter(mids32, np.float32(0)).astype(np.float64)]
    for sc in (1e-9, 1e-7, 3e-6, 6e-5, 1e-3, 0.02, 1.0, 300.0, 6e4):
        vals.append(rng.normal(0, sc, 4000))
    vals.append(np.array([65504.0, 65519.0, 65519.996, 65520.0, 65536.0, 1e9,
                          2.0**-24, 2.0**-25, 2.0**-25 * 1.0000001, 3 * 2.0**-26,
                          2.0**-14, 2.0**-14 - 2.0**-25, 1e-40, 0.0]))
    v = np.concatenate(vals).astype(np.float32)
    return np.concatenate([v, -v])


def test_f32_to_f16_matches_ieee_library_conversion():
    x = _f32_probe_values()
    ours = oracle.f32_to_f16_bits(x)
    ref = np_f16_bits(x)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first x={x[bad[:5]]}"


def test_f32_to_f16_specials():
    f = oracle.lib().orc_f32_to_f16
    assert f(float("inf")) == 0x7C00
    assert f(float("-inf")) == 0xFC00
    h = f(float("nan"))
    assert (h & 0x7C00) == 0x7C00 and (h & 0x3FF) != 0
    assert f(-0.0) == 0x8000
    assert f(65520.0) == 0x7C00           # rounds up to Inf (tie to even)
    assert f(65519.0) == 0x7BFF           # stays at fp16 max


def test_f16_to_f64_every_bit_pattern():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_bits_to_f64(allbits)
    ref = f16_np(allbits)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_rint_half_even_matches_library():
    rng = np.random.default_rng(3)
    xs = np.concatenate([np.arange(-260, 260) * 0.5, rng.uniform(-300, 300, 5000),
                         np.nextafter(np.float32(2.5), np.float32(3)) * np.ones(1),
                         np.nextafter(np.float32(-2.5), np.float32(-3)) * np.ones(1)])
    xs = xs.astype(np.float32)
    for x in xs:
        assert oracle.rint_half_even(x) == float(np.rint(x)), x


# ------------------------------------------------------ int8 block-32 -----

def _brute_int8(w, s):
    """Exact nearest code in [-127, 127] to w / s (ties -> even code), fp64."""
    cand = np.arange(-127, 128, dtype=np.float64)
    d = np.abs(w[..., None] - cand * s[..., None])          # exact in fp64
    dmin = d.min(axis=-1, keepdims=True)
    tie = d == dmin
    even = (np.abs(cand) % 2 == 0)
    pick_even = tie & even
    has_even = pick_even.any(axis=-1, keepdims=True)
    chosen = np.where(has_even, pick_even, tie)
    return cand[np.argmax(chosen, axis=-1)]


def _near_half_integer(ratio32, ulps=1):
    """True where w/s lies within `ulps` fp32 ulps of a half-integer."""
    r = ratio32.astype(np.float64)
    frac = np.abs(r - np.floor(r) - 0.5)
    return frac <= ulps * np.spacing(np.abs(ratio32)).astype(np.float64)


@pytest.mark.parametrize("seed", range(100))
def test_block32_brute_force_4x64(seed):
    rng = np.random.default_rng(seed)
    w = rng.normal(0, 0.02, (4, 64)).astype(np.float32)
    codes, scales = oracle.quantize_block32(w)
    s = np.repeat(f16_np(scales), 32, axis=1)
    # scale: fp32 absmax / 127, rounded to fp16 by the library conversion
    absmax = np.abs(w).reshape(4, 2, 32).max(-1)
    ref_s = np_f16_bits(absmax.astype(np.float32) / np.float32(127.0))
    assert np.array_equal(scales, ref_s)
    best = _brute_int8(w.astype(np.float64), s)
    window = _near_half_integer((w / s.astype(np.float32)).astype(np.float32))
    mism = codes.astype(np.float64) != best
    assert not (mism & ~window).any(), "code is not the nearest multiple of s"
    assert mism.sum() == 0
    # round trip |w - q s| <= s/2 (every scale here is a normal fp16)
    assert (np.abs(w - codes * s) <= s / 2).all()
    # absmax element maps to +-127 with its sign
    wb = w.reshape(4, 2, 32)
    qb = codes.reshape(4, 2, 32)
    arg = np.abs(wb).argmax(-1)
    qa = np.take_along_axis(qb, arg[..., None], -1)[..., 0]
    wa = np.take_along_axis(wb, arg[..., None], -1)[..., 0]
    assert np.array_equal(qa, (np.sign(wa) * 127).astype(np.int8))


def test_block32_special_blocks():
    w = np.zeros((3, 96), dtype=np.float32)
    w[0, 32:64] = 0.37                      # constant positive block
    w[0, 64:96] = -1.25                     # constant negative block
    w[1, :32] = 1e-4 * np.linspace(-1, 1, 32)   # absmax/127 ~ 7.9e-7: subnormal fp16 scale
    w[2, :] = np.random.default_rng(0).normal(0, 50.0, 96)
    codes, scales = oracle.quantize_block32(w)
    assert scales[0, 0] == 0 and (codes[0, :32] == 0).all()      # zero block
    assert (codes[0, 32:64] == 127).all() and (codes[0, 64:96] == -127).all()
    assert scales[0, 1] == np_f16_bits(np.float32(0.37) / np.float32(127))
    assert (codes >= -127).all() and (codes <= 127).all()
    sub = f16_np(scales[1, 0])
    assert 0 < sub < 2.0**-14                # subnormal scale is kept
    assert np.array_equal(np.sign(codes[1, :32]), np.sign(np.round(w[1, :32] / sub)))


def test_block32_constant_weight_closed_form():
    k = 2048
    for c in (0.02, -0.013, 1.7):
        w = np.full((2, k), c, dtype=np.float32)
        codes, scales = oracle.quantize_block32(w)
        s = f16_np(np_f16_bits(np.float32(abs(c)) / np.float32(127)))
        assert (codes == int(np.sign(c)) * 127).all()
        ones = np.full(k, 0x3C00, dtype=np.uint16)        # fp16 1.0
        y, mag = oracle.matvec(0, codes, scales, None, ones)
        assert np.all(y == 127 * s * k * np.sign(c))
        assert np.all(mag == 127 * s * k)


# --------------------------------------------------- int4 group-64 --------

@pytest.mark.parametrize("seed", range(50))
def test_int4_brute_force_4x64(seed):
    rng = np.random.default_rng(1000 + seed)
    w = rng.normal(0, 0.02, (4, 128)).astype(np.float32)
    codes, scales, biases = oracle.quantize_int4_g64(w)
    lo = (codes & 0x0F).astype(np.int64)
    hi = (codes >> 4).astype(np.int64)
    q = np.empty((4, 128), dtype=np.int64)
    q[:, 0::2], q[:, 1::2] = lo, hi                       # low nibble = even k
    s = np.repeat(f16_np(scales), 64, axis=1)
    b = np.repeat(f16_np(biases), 64, axis=1)
    wg = w.reshape(4, 2, 64)
    mx, mn = wg.max(-1), wg.min(-1)
    assert np.array_equal(scales, np_f16_bits((mx - mn).astype(np.float32) / np.float32(15)))
    assert np.array_equal(biases, np_f16_bits(mn))
    cand = np.arange(16, dtype=np.float64)
    d = np.abs(w.astype(np.float64)[..., None] - (cand * s[..., None] + b[..., None]))
    dmin = d.min(-1, keepdims=True)
    tie = d == dmin
    pick = np.where((tie & (cand % 2 == 0)).any(-1, keepdims=True), tie & (cand % 2 == 0), tie)
    best = cand[np.argmax(pick, -1)]
    ratio = ((w - b.astype(np.float32)) / s.astype(np.float32)).astype(np.float32)
    window = _near_half_integer(ratio, ulps=2)
    mism = q != best
    assert not (mism & ~window).any()
    # round trip |w - (q s + b)| <= s/2 + |min - b|
    err = np.abs(w - (q * s + b))
    lim = s / 2 + np.repeat(np.abs(mn - f16_np(biases)), 64, axis=1)
    assert (err <= lim * (1 + 1e-6)).all()
    # min -> 0 and max -> 15
    qg = q.reshape(4, 2, 64)
    assert np.array_equal(np.take_along_axis(qg, wg.argmin(-1)[..., None], -1)[..., 0],
                          np.zeros((4, 2), dtype=np.int64))
    assert np.array_equal(np.take_along_axis(qg, wg.argmax(-1)[..., None], -1)[..., 0],
                          np.full((4, 2), 15))


def test_int4_packing_and_constant_group():
    # a ramp over one group hits each code 0..15 in order; the even k goes in
    # the low nibble
    k = 128
    ramp = np.repeat(np.arange(16, dtype=np.float32), 4) * np.float32(0.25) - 1.0
    w = np.zeros((1, k), dtype=np.float32)
    w[0, :64] = ramp
    w[0, 64:] = 0.5                                       # constant group
    codes, scales, biases = oracle.quantize_int4_g64(w)
    expect_q = np.repeat(np.arange(16), 4)
    assert np.array_equal(codes[0, :32], (expect_q[0::2] | (expect_q[1::2] << 4)).astype(np.uint8))
    assert f16_np(scales[0, 0]) == 0.25 and f16_np(biases[0, 0]) == -1.0
    assert scales[0, 1] == 0 and (codes[0, 32:] == 0).all()
    assert f16_np(biases[0, 1]) == 0.5


# ------------------------------------------------------ dequant / matvec --

def _np_dequant_i8(codes, scales):
    return codes.astype(np.float64) * np.repeat(f16_np(scales), 32, axis=1)


def _np_dequant_i4(codes, scales, biases):
    q = np.empty((codes.shape[0], codes.shape[1] * 2))
    q[:, 0::2] = codes & 0x0F
    q[:, 1::2] = codes >> 4
    return q * np.repeat(f16_np(scales), 64, 1) + np.repeat(f16_np(biases), 64, 1)


def test_dequant_matches_independent_decode():
    rng = np.random.default_rng(11)
    w = rng.normal(0, 0.02, (5, 192)).astype(np.float32)
    c8, s8 = oracle.quantize_block32(w)
    assert np.array_equal(oracle.dequant_i8(c8, s8), _np_dequant_i8(c8, s8))
    c4, s4, b4 = oracle.quantize_int4_g64(w)
    assert np.array_equal(oracle.dequant_i4(c4, s4, b4), _np_dequant_i4(c4, s4, b4))


@pytest.mark.parametrize("fmt", [0, 1])
def test_matvec_exact_rational(fmt):
    rng = np.random.default_rng(5 + fmt)
    n, k = 3, 128
    w = rng.normal(0, 0.02, (n, k)).astype(np.float32)
    xb = np_f16_bits(rng.normal(0, 1, k))
    if fmt == 0:
        c, s = oracle.quantize_block32(w)
        b = None
        wdq = _np_dequant_i8(c, s)
    else:
        c, s, b = oracle.quantize_int4_g64(w)
        wdq = _np_dequant_i4(c, s, b)
    y, mag = oracle.matvec(fmt, c, s, b, xb)
    xs = f16_np(xb)
    for r in range(n):
        exact = sum(Fraction(float(wdq[r, j])) * Fraction(float(xs[j])) for j in range(k))
        exact_mag = sum(abs(Fraction(float(wdq[r, j])) * Fraction(float(xs[j]))) for j in range(k))
        assert abs(Fraction(float(y[r])) - exact) <= Fraction(k) * Fraction(2) ** -53 * exact_mag
        assert abs(Fraction(float(mag[r])) - exact_mag) <= Fraction(k) * Fraction(2) ** -53 * exact_mag


def test_matvec_ones_and_one_hot_closed_forms():
    rng = np.random.default_rng(2)
    n, k = 6, 256
    w = rng.normal(0, 0.02, (n, k)).astype(np.float32)
    c, s = oracle.quantize_block32(w)
    sf = f16_np(s)
    ones = np.full(k, 0x3C00, dtype=np.uint16)
    y, _ = oracle.matvec(0, c, s, None, ones)
    for r in range(n):
        exact = sum(Fraction(float(sf[r, b])) * int(c[r, 32 * b:32 * b + 32].astype(np.int64).sum())
                    for b in range(k // 32))
        assert Fraction(float(y[r])) == exact
    for j in (0, 31, 32, 200, 255):
        e = np.zeros(k, dtype=np.uint16)
        e[j] = 0x3C00
        y, _ = oracle.matvec(0, c, s, None, e)
        assert np.array_equal(y, c[:, j].astype(np.float64) * sf[:, j // 32])


def test_tied_head_is_embedding_times_x():
    """A tied LM head is the embedding table E [V, H] quantized as a head:
    logits = E_dq x, i.e. x times the transposed embedding (non-square V != H
    so a transposed operand cannot pass)."""
    rng = np.random.default_rng(9)
    V, H = 96, 64
    E = rng.normal(0, 0.02, (V, H)).astype(np.float32)
    xb = np_f16_bits(rng.normal(0, 1, H))
    c, s = oracle.quantize_block32(E)
    logits, _ = oracle.matvec(0, c, s, None, xb)
    ref = f16_np(xb) @ _np_dequant_i8(c, s).T
    np.testing.assert_allclose(logits, ref, rtol=1e-12, atol=1e-15)


def test_matvec_fp16_weights_tied_head():
    """Plain fp16 weights (the int8lin bundle's tied fp16 head): w_dq is the
    fp16 value itself.  Exact rational sums, the ones / one-hot closed forms,
    and logits = x E^T against numpy's own fp16 decode on a non-square table."""
    rng = np.random.default_rng(31)
    V, H = 72, 160
    E = np_f16_bits(rng.normal(0, 0.02, (V, H)))
    ef = f16_np(E)
    xb = np_f16_bits(rng.normal(0, 1, H))
    xs = f16_np(xb)
    y, mag = oracle.matvec(oracle.FMT_F16, E, None, None, xb)
    np.testing.assert_allclose(y, ef.astype(np.float64) @ xs.astype(np.float64),
                               rtol=1e-12, atol=1e-15)
    for r in (0, 37, V - 1):
        exact = sum(Fraction(float(ef[r, j])) * Fraction(float(xs[j])) for j in range(H))
        exact_mag = sum(abs(Fraction(float(ef[r, j])) * Fraction(float(xs[j]))) for j in range(H))
        assert abs(Fraction(float(y[r])) - exact) <= Fraction(H) * Fraction(2) ** -53 * exact_mag
        assert abs(Fraction(float(mag[r])) - exact_mag) <= Fraction(H) * Fraction(2) ** -53 * exact_mag
    ones = np.full(H, 0x3C00, dtype=np.uint16)
    y1, _ = oracle.matvec(oracle.FMT_F16, E, None, None, ones)
    for r in range(V):
        assert abs(Fraction(float(y1[r])) - sum(Fraction(float(v)) for v in ef[r])) <= \
            Fraction(H) * Fraction(2) ** -53 * sum(abs(Fraction(float(v))) for v in ef[r])
    for j in (0, 1, 77, H - 1):
        e = np.zeros(H, dtype=np.uint16)
        e[j] = 0x3C00
        yj, _ = oracle.matvec(oracle.FMT_F16, E, None, None, e)
        assert np.array_equal(yj, ef[:, j].astype(np.float64))


# --------------------------------------------------------- SwiGLU ---------

def test_silu_and_grad():
    assert oracle.silu(0.0) == 0.0
    for g in np.linspace(-30, 30, 241):
        ref = g / (1 + math.exp(-g))
        assert oracle.silu(g) == pytest.approx(ref, rel=1e-14, abs=1e-300)
        h = 1e-6
        num = (oracle.silu(g + h) - oracle.silu(g - h)) / (2 * h)
        assert oracle.silu_grad(g) == pytest.approx(num, rel=1e-6, abs=1e-9)
    assert oracle.silu(40.0) == pytest.approx(40.0)
    assert abs(oracle.silu(-40.0)) < 1e-15


def test_swiglu_closed_forms_and_bound():
    g = np.array([0.0, 1.0, -2.0, 5.0])
    u = np.array([3.0, 2.0, 0.5, -1.0])
    h, bound = oracle.swiglu(g, u, np.ones(4), np.ones(4), 2e-3)
    assert h[0] == 0.0                                     # g = 0 gives h = 0
    for i in range(1, 4):
        assert h[i] == pytest.approx(g[i] / (1 + math.exp(-g[i])) * u[i], rel=1e-15)
    assert (bound >= 0.5 * 2.0**-24).all()


def _swiglu_first_order(g, u, mg, mu, tol):
    """The largest first-order change of silu(g) u over the box |dg| <= tol mg,
    |du| <= tol mu, found by evaluating the function itself at the box's four
    corners with a tolerance small enough that second-order terms vanish
    (brute force: no formula of the bound is retyped)."""
    h0 = oracle.silu(g) * u
    worst = 0.0
    for sg in (-1.0, 1.0):
        for su in (-1.0, 1.0):
            worst = max(worst, abs(oracle.silu(g + sg * tol * mg) * (u + su * tol * mu) - h0))
    return worst


def test_swiglu_bound_pinned_by_perturbation():
    """The SwiGLU bound's propagated part is the worst case of silu(g) u over
    the box of gate and up errors allowed by the GEMV bound: checked against
    the function perturbed at the box corners, term by term and mixed.  A
    dropped term, silu in place of its derivative, or a missing |u| fails."""
    rng = np.random.default_rng(17)
    tiny = 1e-7
    cases = [(0.0, 2.5, 3.0, 0.0), (0.0, -1.5, 0.0, 4.0), (1.3, 0.7, 2.0, 0.0),
             (-2.2, 1.1, 0.0, 5.0), (4.0, -3.0, 1.0, 2.0), (-0.4, 0.0, 3.0, 1.5)]
    cases += [(float(rng.normal(0, 3)), float(rng.normal(0, 2)), float(rng.uniform(0, 5)),
               float(rng.uniform(0, 5))) for _ in range(200)]
    for g, u, mg, mu in cases:
        h, b = oracle.swiglu(np.array([g]), np.array([u]), np.array([mg]), np.array([mu]), tiny)
        e = b[0] - 0.5 * oracle.ulp_f16(abs(h[0]) + (b[0] - 0.5 * oracle.ulp_f16(abs(h[0]))))
        ref = _swiglu_first_order(g, u, mg, mu, tiny)
        assert e == pytest.approx(ref, rel=1e-5, abs=1e-18), (g, u, mg, mu)


def test_swiglu_bound_closed_forms():
    """g = 0: silu = 0 and silu' = 1/2, so the propagated part is tol mg |u| / 2
    (the up error cannot move h); with no GEMV error at all (mg = mu = 0) the
    bound is half an fp16 ulp of h (the output rounding alone), numpy's
    spacing; large g: silu' -> 1 and silu(g) -> g."""
    tol = 2e-3
    h, b = oracle.swiglu(np.array([0.0]), np.array([3.0]), np.array([5.0]), np.array([7.0]), tol)
    assert h[0] == 0.0
    assert b[0] == pytest.approx(tol * 0.5 * 5.0 * 3.0 + 0.5 * float(np.spacing(np.float16(
        tol * 0.5 * 5.0 * 3.0))), rel=1e-12)
    for g, u in [(0.7, -2.0), (-3.0, 0.25), (6.0, 1.0)]:
        h, b = oracle.swiglu(np.array([g]), np.array([u]), np.zeros(1), np.zeros(1), tol)
        assert b[0] == 0.5 * float(np.spacing(np.float16(abs(h[0]))))
    g, u, mg, mu = 60.0, 2.0, 1.0, 1.0
    h, b = oracle.swiglu(np.array([g]), np.array([u]), np.array([mg]), np.array([mu]), tol)
    e = tol * (mg * abs(u) + abs(g) * mu)
    assert b[0] == pytest.approx(e + 0.5 * float(np.spacing(np.float16(abs(h[0]) + e))), rel=1e-9)


def test_ulp_f16_matches_library_spacing():
    for v in [2.0**-24, 1e-5, 2.0**-14, 0.1, 0.5, 1.0, 1.5, 1000.0, 40000.0]:
        assert oracle.ulp_f16(v) == float(np.spacing(np.float16(v))), v


# --------------------------------------------------------- argmax ---------

def test_argmax_lowest_index_on_ties_and_boosted_row():
    assert oracle.argmax(np.array([1.0, 3.0, 3.0, 2.0])) == 1
    assert oracle.argmax(np.array([-5.0, -5.0])) == 0
    rng = np.random.default_rng(4)
    logits = rng.normal(0, 1, 5000)
    for v in (0, 17, 4999):
        l2 = logits.copy()
        l2[v] = logits.max() + 1.0
        assert oracle.argmax(l2) == v


def test_argmax_margin_rule():
    l = np.array([0.0, 1.0, 1.0 - 5e-4, 0.2])
    assert oracle.argmax_ok(1, l)
    assert oracle.argmax_ok(2, l)          # within the 1e-3 tie margin
    assert not oracle.argmax_ok(3, l)
    assert not oracle.argmax_ok(7, l)


# ------------------------------------------- byte format vs page sizes ----

def _bytes_per_weight_i8():
    c, s = oracle.quantize_block32(np.ones((1, 32), dtype=np.float32))
    return (c.nbytes + s.nbytes) / 32


def test_byte_formats():
    assert _bytes_per_weight_i8() == 1.0625
    c, s, b = oracle.quantize_int4_g64(np.ones((1, 64), dtype=np.float32))
    assert (c.nbytes + s.nbytes + b.nbytes) / 64 == 0.5625


def _bundle_gib(dec, head, bpw):
    body = dec.weight_count(include_head=False) * bpw
    emb = dec.vocab * dec.hidden * 2                      # fp16 embedding table
    if head == "int8":
        return (body + dec.vocab * dec.hidden * bpw + emb) / 2**30
    assert head == "fp16-tied"                            # embedding doubles as head
    return (body + emb) / 2**30


def _size_matches(computed, printed):
    """The printed size is rounded to 0.1; the bundle also carries a tokenizer,
    metadata and norm vectors (tens of MB) that the computed weight bytes leave
    out, so the computed size may fall up to 0.03 GiB further below."""
    return printed - 0.05 - 0.03 <= computed <= printed + 0.05


def test_bundle_sizes_printed_on_pages():
    rows = []
    with open(os.path.join(GOLDEN, "bundle_sizes.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                name, head, size, _cite = [p.strip() for p in line.split("|", 3)]
                rows.append((wl.DECODERS[name], head, float(size)))
    assert len(rows) == 4
    bpw = _bytes_per_weight_i8()
    for dec, head, printed in rows:
        got = _bundle_gib(dec, head, bpw)
        assert _size_matches(got, printed), (dec.name, head, got, printed)
    # fp32 scales (1.125 B/weight) would not reproduce any int8-head size
    for dec, head, printed in rows:
        if head == "int8":
            assert not _size_matches(_bundle_gib(dec, head, 1.125), printed)


def test_int4_signed_zero_group_gives_positive_zero_side_data():
    """A group of +0 and -0 has min = max = 0; its scale and bias are +0."""
    w = np.zeros((1, 64), dtype=np.float32)
    w[0, 1::2] = -0.0
    codes, scales, biases = oracle.quantize_int4_g64(w)
    assert scales[0, 0] == 0 and biases[0, 0] == 0 and (codes == 0).all()
    w2 = -np.zeros((1, 64), dtype=np.float32)
    codes, scales, biases = oracle.quantize_int4_g64(w2)
    assert scales[0, 0] == 0 and biases[0, 0] == 0


# --------------------------------------------------------- RMSNorm --------

def test_f64_to_f16_matches_ieee_library_conversion():
    rng = np.random.default_rng(41)
    vals = np.concatenate([
        rng.normal(0, 1, 20000), rng.normal(0, 1e-5, 5000), rng.normal(0, 3e4, 5000),
        np.ldexp(rng.uniform(1, 2, 5000), rng.integers(-30, 17, 5000)),
        [0.0, -0.0, 65504.0, 65519.99, 65520.0, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26,
         2.0 ** -14, 2.0 ** -14 - 2.0 ** -25, 1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11]])
    # midpoints between consecutive fp16 values and one fp64 ulp either side
    f = np.arange(0x0000, 0x7BFF, 97, dtype=np.uint16).view(np.float16).astype(np.float64)
    g = (np.arange(0x0000, 0x7BFF, 97, dtype=np.uint16) + 1).view(np.float16).astype(np.float64)
    mid = (f + g) / 2
    vals = np.concatenate([vals, mid, np.nextafter(mid, 0), np.nextafter(mid, np.inf), -mid])
    ours = oracle.f64_to_f16_bits(vals)
    ref = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_rmsnorm_closed_forms():
    k = 64
    rng = np.random.default_rng(43)
    gam = np_f16_bits(rng.normal(1, 0.1, k))
    # constant h = c, eps = 0: h / rms = sign(c) exactly, so x = +-gamma
    for c in (0.75, -3.0, 1e-3):
        x, _ = oracle.rmsnorm(np.full(k, c, np.float32), gam, 0.0)
        assert np.array_equal(x, gam ^ (0x8000 if c < 0 else 0))
    # scale invariance with eps = 0: h * 2^m gives the same bits
    h = rng.normal(0, 1, k).astype(np.float32)
    x0, _ = oracle.rmsnorm(h, gam, 0.0)
    for m in (-7, 3, 20):
        xm, _ = oracle.rmsnorm(h * np.float32(2.0 ** m), gam, 0.0)
        assert np.array_equal(xm, x0)
    # one-hot h = a e_j: rms = |a| / sqrt(k), so x_j = sign(a) sqrt(k) gamma_j = 8 gamma_j
    for j, a in ((0, 2.5), (37, -0.125)):
        e = np.zeros(k, np.float32)
        e[j] = a
        x, _ = oracle.rmsnorm(e, gam, 0.0)
        want = np.zeros(k, np.uint16)
        want[j] = oracle.f64_to_f16_bits(np.sign(a) * 8.0 * f16_np(gam[j:j + 1]).astype(np.float64))[0]
        assert np.array_equal(x, want)
    # eps only matters against a tiny mean square: h = 0 gives x = 0
    x, _ = oracle.rmsnorm(np.zeros(k, np.float32), gam, 1e-6)
    assert not np.any(x & 0x7FFF)


def test_rmsnorm_matches_independent_numpy():
    rng = np.random.default_rng(47)
    for k in (128, 2048, 5120):
        h = (rng.normal(0, 1, k) * rng.uniform(0.1, 30)).astype(np.float32)
        gam = np_f16_bits(rng.normal(1, 0.2, k))
        x, xe = oracle.rmsnorm(h, gam, 1e-6)
        hd = h.astype(np.float64)
        ref = hd * f16_np(gam).astype(np.float64) / np.sqrt(np.mean(hd * hd) + 1e-6)
        np.testing.assert_allclose(xe, ref, rtol=1e-13, atol=0)
        near_tie = np.abs(ref * 2.0 ** (10 - np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -14))))
                          % 1 - 0.5) < 1e-9
        assert np.array_equal(x[~near_tie], ref.astype(np.float16).view(np.uint16)[~near_tie])


# ------------------------------------------------------ decode attention ---
THETA = 5e6   # rope theta of the pages' Qwen3-VL decoders


def test_rope_closed_forms():
    rng = np.random.default_rng(51)
    x = rng.normal(0, 1, 128)
    assert np.array_equal(oracle.rope(x, 0, THETA), x)              # position 0: identity
    # d = 2: one pair at frequency theta^0 = 1, the textbook rotation by pos radians
    for pos in (1, 7, 1000):
        r = oracle.rope(np.array([0.6, -0.8]), pos, THETA)
        c, s = math.cos(pos), math.sin(pos)
        np.testing.assert_allclose(r, [0.6 * c + 0.8 * s, -0.8 * c + 0.6 * s], rtol=0, atol=1e-14)
    # pairs are (i, i + d/2) and each rotation keeps its pair's length
    r = oracle.rope(x, 12345, THETA)
    np.testing.assert_allclose(r[:64] ** 2 + r[64:] ** 2, x[:64] ** 2 + x[64:] ** 2, rtol=1e-12)
    # a unit vector on dimension 64 + i turns into dimension i with -sin
    e = np.zeros(128)
    e[64 + 5] = 1.0
    r = oracle.rope(e, 3, THETA)
    a = 3 * THETA ** (-2 * 5 / 128)
    np.testing.assert_allclose([r[5], r[64 + 5]], [-math.sin(a), math.cos(a)], atol=1e-15)
    assert np.count_nonzero(r) == 2


def test_rope_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(52)
    q, k = rng.normal(0, 1, 128), rng.normal(0, 1, 128)
    s0 = oracle.rope(q, 40, THETA) @ oracle.rope(k, 15, THETA)
    for shift in (1, 100, 5000):
        s = oracle.rope(q, 40 + shift, THETA) @ oracle.rope(k, 15 + shift, THETA)
        assert abs(s - s0) <= 1e-9 * (np.abs(q) @ np.abs(k))
    # and not on the absolute one: moving only the key changes the score
    assert abs(oracle.rope(q, 40, THETA) @ oracle.rope(k, 16, THETA) - s0) > 1e-6


def _attn_inputs(rng, hq, hkv, d, l_max, pos):
    qkv = rng.normal(0, 1, (hq + 2 * hkv) * d).astype(np.float32)
    kc = np_f16_bits(rng.normal(0, 1, (hkv, l_max, d)))
    vc = np_f16_bits(rng.normal(0, 1, (hkv, l_max, d)))
    return qkv, kc, vc


def test_attention_first_token_returns_its_value():
    """pos = 0: one key, softmax weight 1, so every head returns its kv head's
    (fp16) value row; the appended key is fp16(RoPE(k)) = fp16(k) at position 0."""
    rng = np.random.default_rng(53)
    hq, hkv, d = 16, 8, 128
    qkv, kc, vc = _attn_inputs(rng, hq, hkv, d, 4, 0)
    o, mag, kn, vn = oracle.decode_attention(qkv, hq, hkv, d, kc, vc, 0, THETA)
    k = qkv[hq * d:(hq + hkv) * d]
    v = qkv[(hq + hkv) * d:]
    assert np.array_equal(kn, np_f16_bits(k.astype(np.float64)))
    assert np.array_equal(vn, np_f16_bits(v.astype(np.float64)))
    vrow = f16_np(vn).astype(np.float64).reshape(hkv, d)
    np.testing.assert_array_equal(o.reshape(hq, d), np.repeat(vrow, hq // hkv, axis=0))
    np.testing.assert_array_equal(mag.reshape(hq, d), np.abs(np.repeat(vrow, hq // hkv, axis=0)))


def test_attention_zero_query_is_the_mean_and_pins_the_head_groups():
    """q = 0: every score is 0, the weights uniform, so head h returns the
    mean of its kv head's value rows (kv head h // (hq/hkv))."""
    rng = np.random.default_rng(54)
    hq, hkv, d, l_max, pos = 32, 8, 128, 12, 9
    qkv, kc, vc = _attn_inputs(rng, hq, hkv, d, l_max, pos)
    qkv[:hq * d] = 0.0
    o, _, _, vn = oracle.decode_attention(qkv, hq, hkv, d, kc, vc, pos, THETA)
    rows = f16_np(vc).astype(np.float64)[:, :pos, :]
    allv = np.concatenate([rows, f16_np(vn).astype(np.float64).reshape(hkv, 1, d)], axis=1)
    want = np.repeat(allv.mean(axis=1), hq // hkv, axis=0)
    np.testing.assert_allclose(o.reshape(hq, d), want, rtol=0, atol=1e-14)


def test_attention_matches_numpy_softmax_brute_force():
    rng = np.random.default_rng(55)
    for hq, hkv, d, l_max, pos in ((4, 2, 8, 9, 6), (16, 8, 128, 40, 33), (6, 3, 16, 5, 4)):
        qkv, kc, vc = _attn_inputs(rng, hq, hkv, d, l_max, pos)
        o, mag, kn, vn = oracle.decode_attention(qkv, hq, hkv, d, kc, vc, pos, THETA)
        K = f16_np(kc).astype(np.float64).copy()
        V = f16_np(vc).astype(np.float64).copy()
        K[:, pos, :] = f16_np(kn).astype(np.float64).reshape(hkv, d)
        V[:, pos, :] = f16_np(vn).astype(np.float64).reshape(hkv, d)
        for h in range(hq):
            g = h // (hq // hkv)
            q = oracle.rope(qkv[h * d:(h + 1) * d].astype(np.float64), pos, THETA)
            s = K[g, :pos + 1] @ q / math.sqrt(d)
            p = np.exp(s - s.max())
            p /= p.sum()
            np.testing.assert_allclose(o[h * d:(h + 1) * d], p @ V[g, :pos + 1], rtol=1e-12,
                                       atol=1e-13)
            np.testing.assert_allclose(mag[h * d:(h + 1) * d], p @ np.abs(V[g, :pos + 1]),
                                       rtol=1e-12, atol=1e-13)


def test_attention_scale_and_dominant_key():
    """Two positions with scores a and b give weights e^a / (e^a + e^b): with
    q = c e_0 at position 0 (no rotation) and keys e_0, 0 the first weight is
    1 / (1 + e^(-c/sqrt(d))), pinning the 1/sqrt(d) scale; a large c makes the
    matching key dominate."""
    hq, hkv, d, l_max = 2, 1, 128, 4
    for c in (3.0, 1000.0):
        qkv = np.zeros((hq + 2 * hkv) * d, np.float32)
        qkv[0] = qkv[d] = c                           # both query heads: c e_0
        qkv[(hq + hkv) * d:] = 0.25                   # the new token's value row
        kc = np.zeros((hkv, l_max, d), np.uint16)
        vc = np.zeros((hkv, l_max, d), np.uint16)
        kc[0, 0, 0] = np_f16_bits(np.array([1.0]))[0]  # key of position 0: e_0
        vc[0, 0, :] = np_f16_bits(np.array([-1.0]))[0]
        # pos = 1: the new key is fp16(RoPE(0)) = 0, score 0; position 0 scores
        # RoPE(c e_0, 1) . e_0 / sqrt(d) = c cos(1) / sqrt(d)
        o, _, _, _ = oracle.decode_attention(qkv, hq, hkv, d, kc, vc, 1, THETA)
        a = c * math.cos(1.0) / math.sqrt(d)
        w0 = 1.0 / (1.0 + math.exp(-a))
        np.testing.assert_allclose(o[:d], np.full(d, w0 * -1.0 + (1 - w0) * 0.25), rtol=1e-13)
    assert abs(o[0] + 1.0) < 1e-15                    # c = 1000: position 0 dominates
