"""Pins for the CPU oracle: facts fixed by the BitNet model page's scheme and by
mathematics, checked against the oracle without retyping its arithmetic.

Each ``pin_*`` function raises AssertionError when the oracle disagrees.  They
are run by ``test_oracle_pins.py`` against the real oracle and by
``test_oracle_mutants.py`` against copies of the oracle with planted mistakes
(each mutant must fail at least one pin).

Kinds of pin used:
  * a hand-worked example (every value derived by hand, bit patterns included);
  * hand-built special cases (exact ties, power-of-two scales, zero rows);
  * invariants that hold for any input (ranges, argmax -> +-127, error bounds);
  * closed forms for Gaussian latents (E mean|W|, zero fraction of W_q);
  * independent library routines (exact summation, numpy integer matmul).
"""
import math
from fractions import Fraction

import numpy as np

import oracle
import synth


def _f32_bits(v):
    return int(np.asarray(v, np.float32).view(np.uint32))


# --------------------------------------------------------------------------
# Hand-worked example.
#   x = [0.5, -1, 0.25, 2] (bf16-exact)
#   max|x| = 2, s = 127/2 = 63.5 (0x427E0000, exact)
#   x*s = [31.75, -63.5, 15.875, 127] -> x_q = [32, -64 (tie -> even), 16, 127]
#   W = [[0.03, -0.01, 0, -0.05], [0.02, 0.04, -0.02, 0.01]] (fp32)
#   mean|W| of the fp32 values = 0.0224999998... -> gamma = 0x3CB851EB
#   d = gamma + 1e-5 = 0x3CB866E4
#   W/d = [[1.333, -0.444, 0, -2.221], [0.888, 1.777, -0.888, 0.444]]
#     -> W_q = [[1, 0, 0, -1], [1, 1, -1, 0]]
#   acc = [32 + (-127), 32 - 64 - 16] = [-95, -48]
#   y = acc * gamma / s = [-0.0336614..., -0.0170078...]
# --------------------------------------------------------------------------
WX = [0.5, -1.0, 0.25, 2.0]
WW = [[0.03, -0.01, 0.0, -0.05], [0.02, 0.04, -0.02, 0.01]]


def pin_worked_example_quant():
    x = np.array([WX], np.float32)
    x_q, s, rs = oracle.quant_act(x)
    assert _f32_bits(s[0]) == 0x427E0000, hex(_f32_bits(s[0]))
    assert x_q.tolist() == [[32, -64, 16, 127]], x_q
    assert int(rs[0]) == 111


def pin_worked_example_weights():
    w = np.array(WW, np.float32)
    g = oracle.gamma(w)
    assert _f32_bits(g) == 0x3CB851EB, hex(_f32_bits(g))
    w_q = oracle.ternarize(w, g)
    assert w_q.tolist() == [[1, 0, 0, -1], [1, 1, -1, 0]], w_q


def pin_worked_example_forward():
    w = np.array(WW, np.float32)
    # pad K to 16 with zero weights / zero activations (does not change acc)
    w16 = np.zeros((2, 16), np.float32)
    w16[:, :4] = w
    x16 = np.zeros((1, 16), np.float32)
    x16[0, :4] = WX
    g = oracle.gamma(w)           # gamma of the 2x4 matrix, as derived above
    w_q = oracle.ternarize(w16, g)
    packed = oracle.pack(w_q)
    # row 0 codes [2,1,1,0, 1 x 12]: byte b = c[b] | c[4+b]<<2 | c[8+b]<<4 | c[12+b]<<6
    assert packed[0, :4].tolist() == [0x56, 0x55, 0x55, 0x54], packed[0, :4]
    # row 1 codes [2,2,0,1, 1 x 12]
    assert packed[1, :4].tolist() == [0x56, 0x56, 0x54, 0x55], packed[1, :4]
    y, acc, x_q, s = oracle.bitlinear(x16, packed, g, 16)
    assert acc.tolist() == [[-95, -48]], acc
    # hand-derived: -95 * 0.0224999990314245 / 63.5 and -48 * ... / 63.5
    expect = [-95 * 0.022499999031424522 / 63.5, -48 * 0.022499999031424522 / 63.5]
    assert np.allclose(y[0], expect, rtol=1e-12, atol=0), (y, expect)
    # the same values printed to 8 digits (the fp32 results the GPU epilogue gives)
    assert abs(y[0, 0] / -0.033661418 - 1) < 1e-7 and abs(y[0, 1] / -0.017007872 - 1) < 1e-7


def pin_bf16_conversion():
    bits = np.array([0x3F80, 0xC000, 0x4049, 0x0001, 0x8000, 0x7F7F], np.uint16)
    f = oracle.bf16_to_f32(bits)
    assert f[0] == 1.0 and f[1] == -2.0 and f[2] == 3.140625
    assert f[3] == np.float32(2.0 ** -133) and f[4] == 0.0 and np.signbit(f[4])
    assert f[5] == np.float32(3.3895313892515355e38)


def pin_relu2_values():
    g = np.array([0.5, -0.25, 0.0, 2.0, 3.0])
    u = np.array([3.0, 7.0, 5.0, -1.0, 0.5])
    h = oracle.relu2_gate(g, u)
    # 0.25*3, gate<0 -> 0, gate=0 -> 0, 4*(-1), 9*0.5
    assert h.tolist() == [0.75, 0.0, 0.0, -4.0, 4.5], h


# --------------------------------------------------------------------------
# Activation quantiser: hand-built exact cases.
# --------------------------------------------------------------------------
def pin_quant_ties_unit_scale():
    # max|x| = 127 -> s = 1 exactly; ties go to the even integer
    x = np.array([[127.0, 2.5, -2.5, 3.5, 0.5, -0.5, 1.5, -126.5]], np.float32)
    x_q, s, rs = oracle.quant_act(x)
    assert float(s[0]) == 1.0
    assert x_q.tolist() == [[127, 2, -2, 4, 0, 0, 2, -126]], x_q
    assert int(rs[0]) == 127 + 2 - 2 + 4 + 0 + 0 + 2 - 126


def pin_quant_half_scale():
    # max|x| = 254 -> s = 0.5 exactly
    x = np.array([[1.0, 3.0, -5.0, -254.0, 7.0]], np.float32)
    x_q, s, _ = oracle.quant_act(x)
    assert float(s[0]) == 0.5
    assert x_q.tolist() == [[0, 2, -2, -127, 4]], x_q


def pin_quant_zero_row():
    x = np.zeros((2, 32), np.float32)
    x[1, 3] = 1.0
    x_q, s, rs = oracle.quant_act(x)
    assert not x_q[0].any() and int(rs[0]) == 0
    assert float(s[0]) == float(np.float32(127.0) / np.float32(1e-5))
    assert x_q[1, 3] == 127 and int(rs[1]) == 127


def pin_quant_per_token():
    # each row scaled by its own max; permuting rows permutes everything
    x = synth.bf16_bits_to_f32(synth.activations(6, 64, 11, "student_t_rows"))
    x_q, s, rs = oracle.quant_act(x)
    perm = np.array([3, 0, 5, 1, 4, 2])
    x_q2, s2, rs2 = oracle.quant_act(x[perm])
    assert (x_q2 == x_q[perm]).all() and (s2 == s[perm]).all() and (rs2 == rs[perm]).all()
    # columns: permuting columns permutes x_q and leaves s alone
    cp = np.random.default_rng(3).permutation(64)
    x_q3, s3, _ = oracle.quant_act(x[:, cp])
    assert (x_q3 == x_q[:, cp]).all() and (s3 == s).all()


def pin_quant_power_of_two_invariance():
    # scaling a row by 2^e is exact, so s scales by 2^-e and x_q is unchanged
    x = synth.bf16_bits_to_f32(synth.activations(4, 256, 12))
    x_q, s, _ = oracle.quant_act(x)
    for e in (-3, 5):
        x_q2, s2, _ = oracle.quant_act(x * np.float32(2.0 ** e))
        assert (x_q2 == x_q).all()
        assert (s2 == s * np.float32(2.0 ** -e)).all()


def pin_quant_invariants_random():
    for seed, kind in ((21, "normal"), (22, "outliers"), (23, "student_t_rows")):
        x = synth.bf16_bits_to_f32(synth.activations(16, 2560, seed, kind))
        x_q, s, rs = oracle.quant_act(x)
        assert x_q.min() >= -127 and x_q.max() <= 127          # -128 never produced
        amax = np.abs(x).max(axis=1)
        arg = np.abs(x).argmax(axis=1)
        for m in range(x.shape[0]):                             # row max -> +-127
            assert x_q[m, arg[m]] == (127 if x[m, arg[m]] > 0 else -127)
        # s = 127 / max|x| to within one fp32 rounding
        assert np.all(np.abs(s.astype(np.float64) * amax - 127.0) <= 127.0 * 2.0 ** -23)
        # rounding error: |x*s - x_q| <= 1/2 (+ one rounding of the product)
        err = np.abs(x.astype(np.float64) * s[:, None] - x_q)
        assert err.max() <= 0.5 + 127.0 * 2.0 ** -23, err.max()
        # signs agree or x_q is zero
        assert np.all((np.sign(x_q) == np.sign(x)) | (x_q == 0))
        assert (rs == x_q.astype(np.int64).sum(axis=1)).all()


# --------------------------------------------------------------------------
# Weight ternariser and gamma.
# --------------------------------------------------------------------------
def pin_gamma_simple_means():
    assert float(oracle.gamma(np.array([[1, 2], [3, 4]], np.float32))) == 2.5
    assert float(oracle.gamma(np.array([[-1, 2], [-3, -4]], np.float32))) == 2.5
    assert float(oracle.gamma(np.full((3, 16), -0.25, np.float32))) == 0.25
    # asymmetric shape: rows and columns both count
    w = np.zeros((2, 16), np.float32)
    w[1, 15] = 32.0
    assert float(oracle.gamma(w)) == 1.0


def pin_gamma_exact_sum():
    # mean|W| rounded to fp32 equals the correctly rounded exact mean
    for (n, k, seed) in ((64, 256, 31), (300, 320, 32), (7, 2560, 33)):
        w = synth.latent_weights(n, k, seed)
        exact = Fraction(math.fsum(np.abs(w.astype(np.float64)).ravel())) / (n * k)
        assert oracle.gamma(w) == np.float32(float(exact))
        assert abs(oracle.absmean_f64(w) - float(exact)) <= 1e-12 * float(exact)


def pin_ternarize_constructed():
    g = np.float32(1.0)
    d = np.float32(g + np.float32(1e-5))
    w = np.array([[0.5 * d, -0.5 * d, d, -d, 2 * d, -3 * d, 0.0, 0.4,
                   0.51, -0.51, 1.45, -1.55, 100.0, -1e-30, 0.6, -0.6]], np.float32)
    w_q = oracle.ternarize(w, g)
    assert w_q.tolist() == [[0, 0, 1, -1, 1, -1, 0, 0, 1, -1, 1, -1, 1, 0, 1, -1]], w_q


def pin_ternarize_threshold_random():
    w = synth.latent_weights(128, 512, 41)
    g = oracle.gamma(w)
    w_q = oracle.ternarize(w, g)
    assert set(np.unique(w_q).tolist()) <= {-1, 0, 1}
    r = w.astype(np.float64) / (float(g) + 1e-5)
    far = np.abs(np.abs(r) - 0.5) > 1e-5           # away from the rounding boundary
    expect = np.where(np.abs(r) > 0.5, np.sign(r), 0)
    assert (w_q[far] == expect[far]).all()


def pin_ternary_closed_forms():
    # Gaussian latents N(0, s): E|W| = s*sqrt(2/pi); P(|W| < gamma/2) = 2*Phi(sqrt(2/pi)/2) - 1
    n, k = 2560, 6912
    w = synth.latent_weights(n, k, 42)
    g = float(oracle.gamma(w))
    e_abs = 0.02 * math.sqrt(2.0 / math.pi)
    assert abs(g / e_abs - 1.0) < 1e-3, g
    w_q = oracle.ternarize(w, np.float32(g))
    frac0 = float((w_q == 0).mean())
    p0 = math.erf(0.5 * math.sqrt(2.0 / math.pi) / math.sqrt(2.0))
    sd = math.sqrt(p0 * (1 - p0) / (n * k))
    assert abs(frac0 - p0) < 6 * sd + 2e-4, (frac0, p0)   # + finite-gamma wiggle
    fp, fm = float((w_q == 1).mean()), float((w_q == -1).mean())
    assert abs(fp - fm) < 6 * math.sqrt(0.35 / (n * k)) * 2, (fp, fm)


# --------------------------------------------------------------------------
# Packing.
# --------------------------------------------------------------------------
def pin_pack_single_weight_probes():
    base = np.zeros((1, 32), np.int8)
    assert oracle.pack(base).tolist() == [[0x55] * 8]
    w = base.copy()
    w[0, 5] = 1          # group 0, k%16 = 5 -> j = 1, b = 1: byte 1 bits 2..3 = 0b10
    assert oracle.pack(w).tolist() == [[0x55, 0x59, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55]]
    w = base.copy()
    w[0, 18] = -1        # group 1, k%16 = 2 -> j = 0, b = 2: byte 4+2 bits 0..1 = 0b00
    assert oracle.pack(w).tolist() == [[0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x54, 0x55]]
    w = base.copy()
    w[0, 31] = 1         # group 1, k%16 = 15 -> j = 3, b = 3: byte 7 bits 6..7 = 0b10
    assert oracle.pack(w).tolist() == [[0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x55, 0x95]]
    w = np.zeros((2, 16), np.int8)
    w[1, 0] = -1         # second row starts at byte K/4 = 4
    assert oracle.pack(w).tolist() == [[0x55] * 4, [0x54, 0x55, 0x55, 0x55]]


def pin_pack_roundtrip():
    r = np.random.default_rng(51)
    for (n, k) in ((3, 16), (17, 64), (40, 2560)):
        w_q = r.integers(-1, 2, size=(n, k)).astype(np.int8)
        packed = oracle.pack(w_q)
        assert packed.shape == (n, k // 4)
        back, bad = oracle.unpack(packed, k)
        assert bad == 0 and (back == w_q).all()
    planted = oracle.pack(np.zeros((1, 16), np.int8))
    planted[0, 2] |= 0x30                  # code 3 at k = 2*4 + 2 = 10
    _, bad = oracle.unpack(planted, 16)
    assert bad == 1


# --------------------------------------------------------------------------
# Integer contraction and epilogue.
# --------------------------------------------------------------------------
def pin_int_matmul_vs_numpy():
    r = np.random.default_rng(61)
    for (m, n, k) in ((1, 7, 64), (5, 33, 256), (4, 256, 320)):
        a = r.integers(-128, 128, size=(m, k)).astype(np.int8)
        b = r.integers(-1, 2, size=(n, k)).astype(np.int8)
        acc = oracle.int_matmul(a, b)
        assert (acc == a.astype(np.int64) @ b.astype(np.int64).T).all()
        mi = r.integers(0, m, size=20)
        ni = r.integers(0, n, size=20)
        assert (oracle.int_dot_samples(a, b, mi, ni) == acc[mi, ni]).all()


def pin_dequant_special_values():
    acc = np.array([[0, 1, -7, 877824]], np.int64)
    s = np.array([1.0], np.float32)
    y = oracle.dequant(acc, s, np.float32(1.0))
    assert y.tolist() == [[0.0, 1.0, -7.0, 877824.0]]
    s = np.array([0.5], np.float32)
    y = oracle.dequant(acc, s, np.float32(0.25))          # gamma/s = 0.5
    assert y.tolist() == [[0.0, 0.5, -3.5, 438912.0]]
    # row m uses s[m]
    acc2 = np.array([[4, 8], [4, 8]], np.int64)
    y2 = oracle.dequant(acc2, np.array([2.0, 4.0], np.float32), np.float32(1.0))
    assert y2.tolist() == [[2.0, 4.0], [1.0, 2.0]]


def pin_forward_error_bound():
    # y approximates x . (gamma W_q)^T; the only gap is activation rounding:
    # |y - x.(gamma W_q)^T| <= gamma * sum_k |W_q| * (1/2 + eps') / s
    x = synth.bf16_bits_to_f32(synth.activations(6, 256, 71, "outliers"))
    w = synth.latent_weights(48, 256, 72)
    packed, g, w_q = oracle.pack_weights(w)
    y, acc, x_q, s = oracle.bitlinear(x, packed, g, 256)
    ref = x.astype(np.float64) @ (float(g) * w_q.astype(np.float64)).T
    bound = float(g) * np.abs(w_q).sum(axis=1)[None, :] * (0.5 + 1e-4) / s[:, None].astype(np.float64)
    assert np.all(np.abs(y - ref) <= bound + 1e-12)
    assert np.all((y == 0) == (acc == 0)) and np.all(np.sign(y) == np.sign(acc))


def pin_ffn_composition():
    x = synth.bf16_bits_to_f32(synth.activations(3, 64, 81))
    pg, gg, _ = oracle.pack_weights(synth.latent_weights(32, 64, 82))
    pu, gu, _ = oracle.pack_weights(synth.latent_weights(32, 64, 83))
    h, ag, au, _, s = oracle.ffn_gate_up(x, pg, gg, pu, gu, 64)
    yg = oracle.dequant(ag, s, gg)
    yu = oracle.dequant(au, s, gu)
    assert np.all(h[yg <= 0] == 0)
    pos = yg > 0
    assert np.allclose(h[pos], (yg[pos] ** 2) * yu[pos], rtol=1e-15, atol=0)


# ---------------------------------------------------------------- RMS normalisation (subln) prologue
def pin_rmsnorm_exact_integer_sum():
    """x_k = k + 1: the sum of squares is n(n+1)(2n+1)/6 exactly (every partial and pairing
    step is an exact integer in binary64); r follows from it by one division and one root."""
    for n in (64, 512, 2560, 6912):
        x = np.arange(1, n + 1, dtype=np.float32)
        exact = n * (n + 1) * (2 * n + 1) // 6
        assert oracle.sumsq(x) == float(exact)
        y, r = oracle.rmsnorm(x[None, :], np.ones(n, np.float32))
        want = np.float32(1.0 / math.sqrt(exact / n + oracle.RMS_EPS))
        assert r[0] == want
        # y_k = fl(k * r): monotone, last element = fl(n * r)
        assert y[0, -1] == np.float32(np.float32(n) * want)


def pin_rmsnorm_eps_dominates_tiny_rows():
    """mean(x^2) << eps: y = x / sqrt(mean + eps) ~ x / sqrt(eps) (eps = 1e-5 must be present)."""
    x = (synth.activations_f32(3, 256, 301) * np.float32(1e-4)).astype(np.float32)
    y, r = oracle.rmsnorm(x, np.ones(256, np.float32))
    ms = np.mean(x.astype(np.float64) ** 2, axis=1)
    want = 1.0 / np.sqrt(ms + 1e-5)
    assert np.all(np.abs(r.astype(np.float64) - want) <= 2 ** -23 * want)
    assert np.all(ms < 1e-6)
    # the result is far from x / rms(x), which a dropped eps would give
    assert np.all(r.astype(np.float64) < 0.5 / np.sqrt(ms))


def pin_rmsnorm_constant_row_quantises_to_127():
    """x = c everywhere, g = 1: every y_k equals c * r, so every code is +-127."""
    for c in (0.75, -3.0, 1e3):
        x = np.full((1, 320), c, np.float32)
        x_q, s, rs, y, r = oracle.rmsnorm_quant_act(x, np.ones(320, np.float32))
        assert abs(float(r[0]) - 1.0 / math.sqrt(c * c + 1e-5)) <= 2 ** -23 / math.sqrt(c * c + 1e-5)
        assert np.all(y == y[0, 0])
        assert np.all(x_q == (127 if c > 0 else -127))
        assert rs[0] == 320 * (127 if c > 0 else -127)


def pin_rmsnorm_power_of_two_invariance():
    """With eps = 0, scaling x by 2^j scales the sum of squares by 4^j exactly and r by 2^-j
    exactly, so y is bit-identical."""
    x = synth.bf16_bits_to_f32(synth.activations(4, 2560, 302))
    g = synth.activations_f32(1, 2560, 303)[0]
    y0, r0 = oracle.rmsnorm(x, g, eps=0.0)
    for j in (-3, 5):
        y1, r1 = oracle.rmsnorm((x * np.float32(2.0 ** j)).astype(np.float32), g, eps=0.0)
        assert np.array_equal(y0.view(np.uint32), y1.view(np.uint32))
        assert np.array_equal(r1, (r0 * np.float32(2.0 ** -j)).astype(np.float32))


def pin_rmsnorm_weight_per_feature():
    """y with weight g equals fl(y with unit weight * g_k) element by element."""
    x = synth.bf16_bits_to_f32(synth.activations(5, 320, 304))
    g = (synth.activations_f32(1, 320, 305)[0] * np.float32(0.1) + np.float32(1.0)).astype(np.float32)
    y1, _ = oracle.rmsnorm(x, np.ones(320, np.float32))
    yg, _ = oracle.rmsnorm(x, g)
    assert np.array_equal(yg, (y1 * g[None, :]).astype(np.float32))


def _sq_terms(p):
    """binary32 values whose squares add up to exactly 2^p."""
    return [2.0 ** (p // 2)] if p % 2 == 0 else [2.0 ** ((p - 1) // 2)] * 2


def _exact_sumsq(row):
    return sum(Fraction(float(v)) ** 2 for v in row)


def _sumsq_rows():
    """Rows for the sum-of-squares pins: the workloads' rows, wide dynamic ranges, subnormals,
    one large value among many tiny ones, and exact ties between two binary64 neighbours."""
    rows = list(synth.bf16_bits_to_f32(synth.activations(4, 2560, 306, "outliers")))
    rows += list(synth.bf16_bits_to_f32(synth.activations(2, 6912, 307)))
    rows += list(synth.bf16_bits_to_f32(synth.activations(8, 333, 309, "student_t_rows"))[6:])
    rng = np.random.default_rng(310)
    for n in (64, 700, 2560, 6912):
        rows.append((rng.standard_normal(n) * 2.0 ** rng.integers(-60, 61, n)).astype(np.float32))
    rows.append((rng.standard_normal(300) * 2.0 ** rng.integers(-149, -126, 300)).astype(np.float32))
    rows.append(np.array([2.0 ** -149, 3 * 2.0 ** -149, 2.0 ** -126], np.float32))
    rows.append(np.array([1.0] + [2.0 ** -27] * 4095, np.float32))
    rows.append(np.array([2.0 ** 100, 2.0 ** -100, -(2.0 ** 60)], np.float32))
    for v0 in rng.uniform(1.0, 2.0, 6).astype(np.float32):
        e = math.frexp(float(v0) * float(v0))[1] - 1  # binary64 ulp of v0^2 is 2^(e - 52)
        rows.append(np.array([v0] + _sq_terms(e - 53), np.float32))                        # tie, even below
        rows.append(np.array([v0] + _sq_terms(e - 52) + _sq_terms(e - 53), np.float32))    # tie, odd below
        rows.append(np.array([v0] + _sq_terms(e - 53) + [2.0 ** -40], np.float32))         # just above a tie
        rows.append(np.array([-v0] + _sq_terms(e - 54), np.float32))                       # below a tie
    return rows


def pin_rmsnorm_sumsq_correctly_rounded():
    """The sum of squares is the exact sum rounded once to the nearest binary64, ties to even:
    equal to the exact rational sum converted by Python and to math.fsum of the (exact) squares,
    two correctly rounded sums that share nothing with the oracle.  The rows include ones on
    which a binary64 sum in list order, in reverse order or by strided partials gives another
    value, so no fixed summation order passes."""
    rows = _sumsq_rows()
    wrong = {"forward": 0, "reverse": 0, "strided": 0}
    for row in rows:
        want = float(_exact_sumsq(row))
        assert math.fsum(float(v) * float(v) for v in row) == want
        assert oracle.sumsq(row) == want
        sq = [float(v) * float(v) for v in row]
        fwd = 0.0
        for q in sq:
            fwd += q
        rev = 0.0
        for q in reversed(sq):
            rev += q
        part = [0.0] * 256
        for i, q in enumerate(sq):
            part[i % 256] += q
        strided = 0.0
        for q in part:
            strided += q
        wrong["forward"] += fwd != want
        wrong["reverse"] += rev != want
        wrong["strided"] += strided != want
    assert all(v > 0 for v in wrong.values()), wrong


def pin_rmsnorm_sumsq_ties_hand_cases():
    """Hand-worked rounding of 1 + small squares: 1 + 2^-53 is the midpoint between 1 and
    1 + 2^-52 and goes to the even 1; anything above it goes up; (1 + 2^-23)^2 is exact."""
    cases = [([1.0, 2.0 ** -27, 2.0 ** -27], 1.0),
             ([1.0, 2.0 ** -27, 2.0 ** -27, 2.0 ** -60], 1.0 + 2.0 ** -52),
             ([1.0, 2.0 ** -26, 2.0 ** -27, 2.0 ** -27], 1.0 + 2.0 ** -51),
             ([1.0 + 2.0 ** -23], 1.0 + 2.0 ** -22 + 2.0 ** -46),
             ([2.0 ** -149], 2.0 ** -298),
             ([0.0, -0.0], 0.0)]
    for row, want in cases:
        assert oracle.sumsq(np.array(row, np.float32)) == want, row


def pin_rmsnorm_output_mean_square():
    """The mean square of the normalised row is mean(x^2) / (mean(x^2) + eps) to fp32 accuracy."""
    for n, seed in ((2560, 306), (6912, 307), (100, 308), (333, 309)):
        x = synth.bf16_bits_to_f32(synth.activations(2, n, seed, "outliers"))
        y, _ = oracle.rmsnorm(x, np.ones(n, np.float32))
        ms = np.mean(x.astype(np.float64) ** 2, axis=1)
        got = np.mean(y.astype(np.float64) ** 2, axis=1)
        assert np.all(np.abs(got - ms / (ms + 1e-5)) <= 1e-6)


# --------------------------------------------------------------------------
# Output stage: bf16 rounding, the fp32 epilogue value, emitted row maxima and
# the quantiser fed a maximum from outside.
# --------------------------------------------------------------------------
def _bits_to_f32(b):
    return np.array([b], np.uint32).view(np.float32)


def pin_bf16_round_hand_cases():
    """Bit patterns worked by hand: bf16 keeps the upper 16 bits of binary32;
    the dropped half decides (above 0x8000 up, below down, exactly 0x8000 to
    the even upper half)."""
    cases = [
        (0x3F800000, 0x3F80),  # 1.0 exact
        (0x3F808000, 0x3F80),  # 1 + 2^-8: tie, upper 0x3F80 is even -> stays
        (0x3F818000, 0x3F82),  # 1 + 3*2^-8: tie, upper 0x3F81 odd -> up
        (0x3F808001, 0x3F81),  # just above the tie -> up
        (0x3F807FFF, 0x3F80),  # just below the tie -> down
        (0xBF808000, 0xBF80),  # negative tie: magnitude rounds like the positive one
        (0xBF818000, 0xBF82),
        (0x3F80FFFF, 0x3F81),
        (0x7F7FFFFF, 0x7F80),  # largest finite binary32 rounds up to +inf
        (0x00008000, 0x0000),  # subnormal tie to the even zero
        (0x00018000, 0x0002),  # subnormal tie, odd upper -> up
        (0x80000000, 0x8000),  # -0 keeps its sign
        (0x7F800000, 0x7F80),  # +inf
    ]
    src = np.concatenate([_bits_to_f32(a) for a, _ in cases])
    got = oracle.f32_to_bf16(src)
    for (a, want), g in zip(cases, got.tolist()):
        assert g == want, (hex(a), hex(g), hex(want))
    # a NaN whose payload sits only in the dropped half must stay a NaN
    for a in (0x7F800001, 0xFF800001, 0x7FC00000):
        g = int(oracle.f32_to_bf16(_bits_to_f32(a))[0])
        assert (g & 0x7F80) == 0x7F80 and (g & 0x007F) != 0, (hex(a), hex(g))


def pin_bf16_round_vs_torch():
    """Against torch's own binary32 -> bfloat16 conversion (round to nearest even)
    on random finite values of every magnitude, including constructed ties."""
    import torch
    rng = np.random.default_rng(77)
    bits = rng.integers(0, 2**32, 20000, dtype=np.uint64).astype(np.uint32)
    bits = bits[(bits & 0x7F800000) != 0x7F800000]  # finite only
    ties = (rng.integers(0, 2**16, 2000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    ties = ties[(ties & 0x7F800000) != 0x7F800000]
    v = np.concatenate([bits, ties]).view(np.float32)
    want = torch.from_numpy(v.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.f32_to_bf16(v)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(hex(int(v.view(np.uint32)[i])), hex(int(got[i])), hex(int(want[i]))) for i in bad[:5]]


def pin_row_absmax_hand():
    v = np.array([[1.0, -3.0, 2.0], [-0.5, 0.25, 0.0], [0.0, -0.0, 0.0], [-7.0, -8.0, -1.0]], np.float32)
    assert oracle.row_absmax(v).tolist() == [3.0, 0.5, 0.0, 8.0]


def _rne32(q):
    """Exact rational -> nearest binary32 value (ties to even), as a Fraction.
    Normal range only (the pins below stay far from under/overflow)."""
    if q == 0:
        return Fraction(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    # a = m * 2^(e-23) with 2^23 <= m < 2^24
    m = a / Fraction(2) ** (e - 23)
    lo = m.numerator // m.denominator
    rem = m - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return sign * Fraction(lo) * Fraction(2) ** (e - 23)


def pin_epilogue_f32_exact_rounding():
    """y32 = fl32(acc * fl32(gamma / s)) evaluated in exact rational arithmetic
    with its own round-to-nearest-even, on triples where rounding gamma / s
    first changes the result against the single rounding of the exact product
    (so a fused or binary64 product would fail), plus the gated form
    h32 = fl32(fl32(p * p) * u32)."""
    triples = [(3, 0.75, 42.33333206176758), (3, 0.75, 181.42857360839844),
               (7, 0.75, 42.33333206176758), (100, 0.75, 181.42857360839844),
               (12345, 0.75, 42.33333206176758), (-12345, 0.75, 42.33333206176758),
               (1, 0.5, 127.0), (0, 0.8, 3.0)]
    acc = np.array([[t[0] for t in triples]], np.int64)
    for gam in sorted({t[1] for t in triples}):
        for s in sorted({t[2] for t in triples}):
            s32 = np.float32(s)
            y = oracle.epilogue_f32(acc, np.array([s32], np.float32), np.float32(gam))[0]
            r = _rne32(Fraction(float(np.float32(gam))) / Fraction(float(s32)))
            for a, got in zip(acc[0].tolist(), y.tolist()):
                want = _rne32(a * r)
                assert Fraction(got) == want, (a, gam, s, got, float(want))
    # at least one triple separates the two-rounding value from the exact product's
    s32 = np.float32(42.33333206176758)
    r = _rne32(Fraction(0.75) / Fraction(float(s32)))
    assert _rne32(3 * r) != _rne32(3 * Fraction(0.75) / Fraction(float(s32)))
    # gated: acc_g, acc_u pairs, signs of both
    ag = np.array([[5, -5, 17, 100, 0, 33]], np.int64)
    au = np.array([[7, 7, -9, 3, 4, -1]], np.int64)
    sg, gg, gu = np.float32(42.33333206176758), np.float32(0.75), np.float32(0.3)
    h = oracle.epilogue_f32(ag, np.array([sg], np.float32), gg, au, gu)[0]
    rg = _rne32(Fraction(float(gg)) / Fraction(float(sg)))
    ru = _rne32(Fraction(float(gu)) / Fraction(float(sg)))
    for a, b, got in zip(ag[0].tolist(), au[0].tolist(), h.tolist()):
        g32 = _rne32(a * rg)
        u32 = _rne32(b * ru)
        p = g32 if g32 > 0 else Fraction(0)
        want = _rne32(_rne32(p * p) * u32)
        assert Fraction(got) == want, (a, b, got, float(want))


def pin_epilogue_f32_error_bound():
    """fp32 epilogue within its rounding bound of the binary64 forward: two
    roundings (2u) for y, eight (8u) for the gated h, u = 2^-24."""
    rng = np.random.default_rng(91)
    m, n, k = 5, 40, 512
    acc_g = rng.integers(-127 * k // 4, 127 * k // 4, (m, n)).astype(np.int64)
    acc_u = rng.integers(-127 * k // 4, 127 * k // 4, (m, n)).astype(np.int64)
    s = (127.0 / rng.uniform(0.01, 30.0, m)).astype(np.float32)
    gg, gu = np.float32(0.0213), np.float32(0.0377)
    u = 2.0 ** -24
    y = oracle.epilogue_f32(acc_g, s, gg).astype(np.float64)
    y64 = oracle.dequant(acc_g, s, gg)
    assert np.all(np.abs(y - y64) <= 2.0001 * u * np.abs(y64))
    h = oracle.epilogue_f32(acc_g, s, gg, acc_u, gu).astype(np.float64)
    h64 = oracle.relu2_gate(y64, oracle.dequant(acc_u, s, gu))
    assert np.all(np.abs(h - h64) <= 8.001 * u * np.abs(h64))
    assert np.all(h[acc_g <= 0] == 0)


def pin_quant_given_amax():
    """The quantiser with a supplied maximum: the true maximum changes nothing;
    a larger one A gives the codes of the same row with one more element equal
    to A (whose own code is 127)."""
    rng = np.random.default_rng(93)
    x = rng.standard_normal((6, 96)).astype(np.float32)
    x[2] *= 1e-7  # below the 1e-5 floor
    x[3, 5] = 41.0
    true_max = np.abs(x).max(axis=1).astype(np.float32)
    q0, s0, r0 = oracle.quant_act(x)
    q1, s1, r1 = oracle.quant_act(x, true_max)
    assert np.array_equal(q0, q1) and np.array_equal(s0, s1) and np.array_equal(r0, r1)
    big = (true_max * np.float32(3.5) + np.float32(0.25)).astype(np.float32)
    qa, sa, ra = oracle.quant_act(x, big)
    qb, sb, rb = oracle.quant_act(np.concatenate([x, big[:, None]], axis=1))
    assert np.array_equal(qa, qb[:, :-1]) and np.array_equal(sa, sb)
    assert np.array_equal(ra.astype(np.int64), rb.astype(np.int64) - qb[:, -1]) and np.all(qb[:, -1] == 127)


def pin_bitlinear_ex_output_forms():
    """bf16 output = the bf16 rounding of the fp32 output; the emitted maxima
    are the maxima of the stored values; chaining through the emitted maximum
    equals recomputing it."""
    rng = np.random.default_rng(95)
    k, n, m = 128, 32, 4
    w = synth.latent_weights(n, k, 5)
    packed, g, _ = oracle.pack_weights(w)
    wu = synth.latent_weights(n, k, 6)
    packed_u, gu_, _ = oracle.pack_weights(wu)
    x = rng.standard_normal((m, k)).astype(np.float32)
    y32, a32 = oracle.bitlinear_ex(x, packed, g, k, "f32")
    yb, ab = oracle.bitlinear_ex(x, packed, g, k, "bf16")
    assert np.array_equal(yb, oracle.f32_to_bf16(y32))
    widened = (yb.astype(np.uint32) << 16).view(np.float32)
    assert np.array_equal(ab, np.abs(widened).max(axis=1)) and np.array_equal(a32, np.abs(y32).max(axis=1))
    y64 = oracle.bitlinear(x, packed, g, k)[0]
    assert np.all(np.abs(y32 - y64) <= 2.0001 * 2.0 ** -24 * np.abs(y64))
    h32, _ = oracle.bitlinear_ex(x, packed, g, k, "f32", packed_u=packed_u, gamma_u=gu_)
    h64 = oracle.ffn_gate_up(x, packed, g, packed_u, gu_, k)[0]
    assert np.all(np.abs(h32 - h64) <= 8.001 * 2.0 ** -24 * np.abs(h64))
    # next layer: quantising y through the emitted maximum
    p2, g2, _ = oracle.pack_weights(np.ascontiguousarray(synth.latent_weights(16, n, 8)))
    z_a, _ = oracle.bitlinear_ex(widened, p2, g2, n, "f32", x_amax=ab)
    z_b, _ = oracle.bitlinear_ex(widened, p2, g2, n, "f32")
    assert np.array_equal(z_a, z_b)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
