"""The prefill router runs on the bf16 tensor cores with the FP32 router weights written as three
bf16 planes, hi + mid + lo, each rounding (to nearest, ties to even) what the planes before it
left. The router stays an FP32 computation because that decomposition is exact for every finite
FP32 weight of magnitude at least 2^-110 (24 significand bits in three bf16 significands of 8,
each residual exact in FP32 by Sterbenz) and off by less than 2^-133 below that, where the last
plane's bits fall under bf16's subnormal step. This checks the claim on the host with its own
bf16 rounding, independent of the CUDA sources; the GPU parity tests check the router's outputs."""
import numpy as np


def bf16_rne(v: np.ndarray) -> np.ndarray:
    """FP32 -> nearest bf16 (ties to even), returned as FP32 values."""
    b = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> 16) & 1
    r = ((b + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32)


def split3(v: np.ndarray):
    v = np.asarray(v, dtype=np.float32)
    hi = bf16_rne(v)
    r1 = (v - hi).astype(np.float32)
    mid = bf16_rne(r1)
    r2 = (r1 - mid).astype(np.float32)
    lo = bf16_rne(r2)
    return hi, mid, lo, r1, r2


def _check(v):
    v = np.asarray(v, dtype=np.float32)
    tiny = np.abs(v) < np.float32(2.0 ** -110)
    hi, mid, lo, _, _ = split3(v[tiny])
    err = np.abs(hi.astype(np.float64) + mid.astype(np.float64) + lo.astype(np.float64) - v[tiny].astype(np.float64))
    assert np.all(err < 2.0 ** -133)
    v = v[~tiny]
    hi, mid, lo, r1, r2 = split3(v)
    v64 = v.astype(np.float64)
    # the residuals are exact in FP32 ...
    assert np.array_equal(r1.astype(np.float64), v64 - hi.astype(np.float64))
    assert np.array_equal(r2.astype(np.float64), r1.astype(np.float64) - mid.astype(np.float64))
    # ... the last plane holds the last residual without rounding ...
    assert np.array_equal(lo, r2)
    # ... and the three planes add up to the weight exactly
    assert np.array_equal(hi.astype(np.float64) + mid.astype(np.float64) + lo.astype(np.float64), v64)
    # every plane is a bf16 value (low 16 bits zero)
    for p in (hi, mid, lo):
        assert not np.any(p.view(np.uint32) & 0xFFFF)


def test_bf16_rounding_reference():
    # exact bf16 values stay; a halfway case rounds to even; a carry into the exponent
    v = np.array([1.0, -2.5, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 1.9999999], dtype=np.float32)
    r = bf16_rne(v)
    assert r[0] == 1.0 and r[1] == -2.5
    assert r[2] == 1.0                      # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: even is 1
    assert r[3] == np.float32(1.0 + 2.0 ** -6)   # halfway between 1 + 2^-7 and 1 + 2^-6: even is the latter
    assert r[4] == 2.0


def test_split_is_exact_on_router_like_weights():
    rng = np.random.default_rng(11)
    _check((rng.standard_normal(200_000) / np.sqrt(2816.0)).astype(np.float32))


def test_split_is_exact_on_random_bit_patterns():
    rng = np.random.default_rng(12)
    bits = rng.integers(0, 2 ** 32, size=400_000, dtype=np.uint64).astype(np.uint32)
    v = bits.view(np.float32)
    v = v[np.isfinite(v)]
    # keep the planes away from overflow: |v| below the largest bf16-rounding-safe value
    v = v[np.abs(v) < np.float32(3.0e38)]
    _check(v)


def test_split_edge_values():
    v = np.array([0.0, -0.0, 1.0, -1.0, np.float32(np.finfo(np.float32).tiny), np.float32(1.4e-45),
                  np.float32(1.0 + 2.0 ** -23), np.float32(-(1.0 + 2.0 ** -23)), np.float32(3.3333333),
                  np.float32(1.0 - 2.0 ** -24), np.float32(2.0 ** 100 * (1 + 2.0 ** -9 + 2.0 ** -17))],
                 dtype=np.float32)
    _check(v)
