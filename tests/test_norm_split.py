"""The centroid norm enters the assign kernel's accumulator through one extra K = 16 MMA
step against the norm's three bf16 pieces (csrc/prep_row.cuh): hi = RN_bf16(c2),
mid = RN_bf16(c2 - hi), lo = RN_bf16(c2 - hi - mid).  What the split guarantees, checked
here on the host with bf16 round-to-nearest-even written out in integer arithmetic, over
every fp32 mantissa at several exponents, random fp32 values and the edge cases:
  - each piece is a bf16 value, and hi + mid + lo = c2 exactly, for every norm from 2^-110
    up to the largest that does not round hi to infinity (below 2^-110 lo's low bits fall
    under bf16's smallest subnormal, 2^-133, which bounds the error there);
  - adding the pieces in fp32 gives c2 exactly in every order that adds hi and mid before
    lo (and whenever hi did not round up); adding hi and lo first can round, by at most
    one ulp of c2.  The ISA fixes no order for the products of one MMA step, so the
    folded norm is c2 to within one fp32 ulp: 6e-8 relative, inside the screening
    window's allowance for the norm step's own fp32 accumulation (17 units of 2^-23 of
    its partial sums, as for every MMA step) and far inside the 1e-4 tie window."""
import itertools

import numpy as np

TINY = np.float32(2.0 ** -110)  # exact from here up
ULP_FLOOR = 2.0 ** -133          # bf16's smallest subnormal
# the largest fp32 norm whose hi piece stays finite: below the rounding midpoint between
# the largest finite bf16 (0x7f7f) and infinity
TOP = np.array([(0x7F7F << 16) | 0x7FFF], dtype=np.uint32).view(np.float32)[0]


def rn_bf16(x32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (round to nearest, ties to even), returned widened to fp32."""
    b = x32.astype(np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def pieces(c2: np.ndarray):
    c2 = c2.astype(np.float32)
    h = rn_bf16(c2)
    r1 = (c2 - h).astype(np.float32)
    m = rn_bf16(r1)
    l = rn_bf16((r1 - m).astype(np.float32))
    return c2, h, m, l


def ulp(x32: np.ndarray) -> np.ndarray:
    e = (x32.view(np.uint32) >> 23).astype(np.int64)
    return np.ldexp(1.0, np.maximum(e, 1) - 150)


def check(c2):
    c2, h, m, l = pieces(c2)
    assert np.isfinite(h).all()
    for p in (h, m, l):
        assert np.array_equal(rn_bf16(p), p)
    # the three pieces add up to the fp32 norm exactly
    assert np.array_equal(h.astype(np.float64) + m + l, c2.astype(np.float64))
    hi_rounded_up = h > c2
    for a, b, c, name in ((h, m, l, "hm"), (m, h, l, "hm"), (m, l, h, "ml"),
                          (l, m, h, "ml"), (h, l, m, "hl"), (l, h, m, "hl")):
        s = ((a + b).astype(np.float32) + c).astype(np.float32)
        if name != "hl":
            assert np.array_equal(s, c2), name  # hi and mid (or mid and lo) first: exact
        else:
            # hi and lo first: exact unless hi rounded up, and then within one ulp
            assert np.array_equal(s[~hi_rounded_up], c2[~hi_rounded_up])
            err = np.abs(s.astype(np.float64) - c2.astype(np.float64))
            assert (err <= ulp(c2)).all()


def check_tiny(c2):
    """Norms below 2^-110: the pieces add up to within bf16's smallest subnormal."""
    c2, h, m, l = pieces(c2)
    err = np.abs(h.astype(np.float64) + m + l - c2.astype(np.float64))
    assert (err <= ULP_FLOOR).all(), err.max()


def test_every_mantissa_at_several_exponents():
    mant = np.arange(1 << 23, dtype=np.uint32)
    for e in (17, 64, 127, 127 + 20, 200, 254):  # 2^-110 to the top binade
        v = ((np.uint32(e) << 23) | mant).view(np.float32)
        check(v[v <= TOP])
    for e in (0, 1, 9, 16):  # subnormals and the binades below 2^-110
        check_tiny(((np.uint32(e) << 23) | mant).view(np.float32))


def test_random_norms_and_edges():
    rng = np.random.default_rng(0)
    v = rng.integers(0, 0x7F7FFFFF, size=2_000_000, dtype=np.uint32).view(np.float32)
    check(v[(v >= TINY) & (v <= TOP)])
    check_tiny(v[v < TINY])
    check(np.array([0.0, 2.0 ** -110, 1.0, 3.0, 65536.0, TOP,
                    np.float32(1) + np.float32(2.0 ** -23)], dtype=np.float32))
    check_tiny(np.array([1e-40, 1.17549435e-38, 1e-35], dtype=np.float32))


def test_hi_and_lo_first_does_round_sometimes():
    # the one-ulp allowance above is needed: the order hi + lo first is not always exact
    mant = np.arange(1 << 23, dtype=np.uint32)
    c2, h, m, l = pieces(((np.uint32(127) << 23) | mant).view(np.float32))
    s = ((h + l).astype(np.float32) + m).astype(np.float32)
    assert 0 < (s != c2).sum() < len(c2) // 100


def test_padding_piece_is_the_largest_finite_bf16():
    # a padding centroid's first piece 0x7f7f: finite, at least every real norm's hi
    pad = np.array([0x7F7F << 16], dtype=np.uint32).view(np.float32)[0]
    assert np.isfinite(pad) and pad > 3.38e38
    assert rn_bf16(np.array([TOP], dtype=np.float32))[0] <= pad
