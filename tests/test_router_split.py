"""The prefill router's exactness argument, checked on the CPU: every fp32 weight w with
|w| >= 2^-100 (so that its last piece is still a normal number) equals hi + mid + lo exactly with hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid) (round to
nearest even; each difference is exact in fp32), and a bf16 activation times a bf16 piece is
exact in fp32.  So three bf16 x bf16 products per weight give the fp32 dot product's terms
exactly; only the accumulation rounds."""
import numpy as np


def bf16_rne(a: np.ndarray) -> np.ndarray:
    """fp32 -> nearest bf16 (ties to even), returned as fp32."""
    u = a.astype(np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return r.astype(np.uint32).view(np.float32)


def split3(w: np.ndarray):
    hi = bf16_rne(w)
    r1 = (w - hi).astype(np.float32)
    mid = bf16_rne(r1)
    r2 = (r1 - mid).astype(np.float32)
    lo = bf16_rne(r2)
    return hi, mid, lo, r1, r2


def test_three_bf16_pieces_reconstruct_every_fp32_weight_exactly():
    rng = np.random.default_rng(7)
    w = np.concatenate([
        rng.standard_normal(200_000).astype(np.float32) * np.float32(0.02),      # router-like weights
        # every binade whose last piece (about 2^-16 of w) is still a normal number
        rng.uniform(-1, 1, 200_000).astype(np.float32) * np.float32(2.0) ** rng.integers(-100, 100, 200_000).astype(np.float32),
        np.array([0.0, -0.0, 1.0, -1.0, 3.0e38, -3.0e38, 1.17549435e-38 * 2 ** 10], dtype=np.float32),
    ]).astype(np.float32)
    w = w[(np.abs(w) >= np.float32(2.0 ** -100)) | (w == 0)]
    hi, mid, lo, r1, r2 = split3(w)
    # each residual is exact (float64 reference) and the pieces sum back exactly
    w64 = w.astype(np.float64)
    assert np.array_equal(r1.astype(np.float64), w64 - hi.astype(np.float64))
    assert np.array_equal(r2.astype(np.float64), r1.astype(np.float64) - mid.astype(np.float64))
    assert np.array_equal(lo, r2)                              # the last piece needs no rounding
    assert np.array_equal(hi.astype(np.float64) + mid.astype(np.float64) + lo.astype(np.float64), w64)


def test_bf16_times_bf16_is_exact_in_fp32():
    rng = np.random.default_rng(8)
    a = bf16_rne(rng.standard_normal(100_000).astype(np.float32))
    b = bf16_rne(rng.standard_normal(100_000).astype(np.float32) * np.float32(0.02))
    p32 = (a * b).astype(np.float32)
    assert np.array_equal(p32.astype(np.float64), a.astype(np.float64) * b.astype(np.float64))


def test_split_is_what_a_single_bf16_would_lose():
    # a bf16 copy of the router weights alone would not be exact: the split is needed
    rng = np.random.default_rng(9)
    w = rng.standard_normal(10_000).astype(np.float32) * np.float32(0.02)
    hi, mid, lo, _, _ = split3(w)
    assert np.count_nonzero(mid) > 9_000
    assert np.count_nonzero(lo) > 1_000


def test_tiny_weights_lose_at_most_a_subnormal_remainder():
    # below 2^-100 the third piece can fall under bf16's normal range; what is lost is below
    # 2^-133 in absolute value -- immaterial next to any logit, but not exact
    w = np.float32(2.0) ** -np.arange(101, 126, dtype=np.float32) * np.float32(1.2345678)
    hi, mid, lo, _, _ = split3(w)
    err = np.abs(hi.astype(np.float64) + mid.astype(np.float64) + lo.astype(np.float64) - w.astype(np.float64))
    assert np.all(err <= 2.0 ** -133)
