"""The rounding of the decode's INT4 p.v in offset form, emulated on the host in binary32.

The CUDA-core engine multiplies p * v_scale by 0.5 + code/256 (the nibble placed as mantissa bits
under the exponent of 0.5, exact) instead of by (code - zp); after every tile a lane subtracts
0.5 * sum(p * v_scale) over its rows from its accumulators and collects v_scale * zp * sum(p) in a
separate sum, and the segment's end forms 256 * acc - zsum. These tests replay that sequence of
binary32 operations (each fused multiply-add rounded once) for one lane and check the error of
the normalised output against binary64, next to the per-code form it replaced, on inputs chosen
to make the offset's share large: flat attention over a long segment, one dominant tile, and
codes at the zero point (where 256 * acc and zsum cancel).
"""
import numpy as np
import pytest

F32 = np.float32
TPL = 8  # rows of a tile held by one lane (32-token tile, 4 row groups)


def fma32(a, b, c):
    """a * b + c rounded once to binary32 (the product is exact in binary64)."""
    return F32(np.float64(F32(a)) * np.float64(F32(b)) + np.float64(F32(c)))


def lane_sums(p, vs, codes, zp, offset):
    """p, vs, zp: [T, TPL] per row (vs and zp constant within a half-tile); codes: [T, TPL].
    Returns the lane's sum of p * vs * (code - zp) as the kernel forms it in binary32."""
    acc, zsum = F32(0), F32(0)
    for t in range(p.shape[0]):
        pv = [F32(F32(p[t, i]) * F32(vs[t, i])) for i in range(TPL)]
        for i in range(TPL):
            if offset:
                v = F32(0.5 + codes[t, i] / 256.0)  # exact
            else:
                v = F32(float(codes[t, i]) - float(zp[t, i]))  # exact
            acc = fma32(pv[i], v, acc)
        if offset:
            s1 = [F32(0), F32(0)]
            for i in range(TPL):
                s1[i * 2 // TPL] = F32(s1[i * 2 // TPL] + pv[i])
            acc = F32(acc + F32(F32(-0.5) * F32(s1[0] + s1[1])))
            zsum = fma32(zp[t, 0], s1[0], zsum)
            zsum = fma32(zp[t, TPL - 1], s1[1], zsum)
    if offset:
        return F32(fma32(acc, 256.0, -zsum))
    return acc


def exact_sum(p, vs, codes, zp):
    pv = np.float32(p).astype(np.float64) * np.float32(vs).astype(np.float64)
    return float(np.sum(pv * (codes - zp)))


def make(rng, T, kind):
    vs = np.repeat(rng.uniform(0.05, 1.0, size=(T, 2)), TPL // 2, axis=1)
    zp = np.repeat(rng.integers(0, 16, size=(T, 2)), TPL // 2, axis=1).astype(np.float64)
    codes = rng.integers(0, 16, size=(T, TPL)).astype(np.float64)
    if kind == "flat":  # every weight at the running max
        p = np.ones((T, TPL))
    elif kind == "dominant":  # one tile carries nearly all the weight
        p = rng.uniform(0, 1e-3, size=(T, TPL))
        p[T // 2] = 1.0
    elif kind == "at_zero_point":  # codes equal to the zero point: a result near 0 from two large sums
        p = np.ones((T, TPL))
        codes = zp.copy()
        codes[:, 0] = np.minimum(zp[:, 0] + 1, 15)
    else:
        p = np.exp2(-rng.uniform(0, 8, size=(T, TPL)))
    return p, vs, codes, zp


@pytest.mark.parametrize("kind", ["flat", "dominant", "at_zero_point", "random"])
def test_offset_form_error_within_its_bound(kind):
    rng = np.random.default_rng(7)
    T = 300  # 2400 rows of one lane: a long stream-K segment
    p, vs, codes, zp = make(rng, T, kind)
    ref = exact_sum(p, vs, codes, zp)
    l = float(np.sum(np.float32(p).astype(np.float64)))
    got_off = float(lane_sums(p, vs, codes, zp, offset=True))
    got_exact = float(lane_sums(p, vs, codes, zp, offset=False))
    err_off = abs(got_off - ref) / l
    err_exact = abs(got_exact - ref) / l
    vmax = float(vs.max())
    # the offset adds at most 2^-12.8 of the weight per tile, i.e. 1.4e-4 * v_scale on the output,
    # on top of the running-sum rounding of the per-code form
    assert err_off <= 1.4e-4 * vmax + 4 * err_exact + 1e-7
    # either way far inside the decode's 2e-3 bound on outputs of unit-variance data
    assert err_off < 2e-4


def test_offset_values_are_exact_and_linear():
    # 0x3F000000 | c << 16 is 0.5 + c/256 for every nibble c (exponent of 0.5, mantissa bits 16..19)
    for c in range(16):
        bits = np.uint32(0x3F000000 | (c << 16))
        assert float(bits.view(np.float32)) == 0.5 + c / 256.0
