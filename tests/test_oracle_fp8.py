"""Pins of the oracle's E4M3 block quantiser (the FP8 forward's inputs).

The decode is written from the format definition (1 sign, 4 exponent bits with
bias 7, 3 mantissa bits, subnormals at exponent 0, NaN at S.1111.111, largest
finite 448) and checked here against hand values; the encode (torch's
float8_e4m3fn conversion) against a brute-force nearest-code search with ties
to the even code; the block quantiser against its defining invariants."""
import numpy as np
import pytest

import oracle


def test_e4m3_decode_hand_values():
    d = oracle.e4m3_decode(np.array([0x00, 0x80, 0x38, 0xB8, 0x7E, 0xFE, 0x01, 0x08, 0x07, 0x3C, 0x40, 0x7F, 0xFF],
                                    dtype=np.uint8))
    assert d[0] == 0.0 and d[1] == 0.0 and np.signbit(d[1])
    assert d[2] == 1.0 and d[3] == -1.0          # 0.0111.000 = 2^0
    assert d[4] == 448.0 and d[5] == -448.0      # 0.1111.110 = 1.75 * 2^8
    assert d[6] == 2.0 ** -9                     # smallest subnormal
    assert d[7] == 2.0 ** -6                     # smallest normal
    assert d[8] == 7 / 8 * 2.0 ** -6             # largest subnormal
    assert d[9] == 1.5 and d[10] == 2.0
    assert np.isnan(d[11]) and np.isnan(d[12])


def _nearest_code(x, finite_codes, finite_vals):
    """Brute force: the finite code nearest to x; a tie goes to the code with
    an even mantissa (the last bit of the code)."""
    err = np.abs(finite_vals - x)
    best = err.min()
    cand = finite_codes[err == best]
    if cand.size > 1:
        even = cand[(cand & 1) == 0]
        cand = even if even.size else cand
    return int(cand[0])


def test_e4m3_encode_is_nearest_with_ties_to_even():
    codes = np.arange(256, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    fin = ~np.isnan(vals)
    fc, fv = codes[fin], vals[fin]
    rng = np.random.default_rng(4)
    # random magnitudes over the whole range, the exact midpoints between
    # neighbouring codes, and the codes themselves
    pos = np.sort(np.unique(fv[fv >= 0]))
    mids = (pos[:-1] + pos[1:]) / 2
    xs = np.concatenate([rng.uniform(-448, 448, 3000), np.exp(rng.uniform(-12, 6, 2000)) * rng.choice([-1, 1], 2000),
                         mids, -mids, pos]).astype(np.float32)
    got = oracle.e4m3_encode(xs)
    want = np.array([_nearest_code(float(x), fc, fv) for x in xs], dtype=np.uint8)
    # +0 and -0 both decode to zero: compare decoded values, and codes elsewhere
    dv_got, dv_want = oracle.e4m3_decode(got), oracle.e4m3_decode(want)
    assert np.array_equal(dv_got, dv_want)


@pytest.mark.parametrize("rows,n", [(4, 32), (4, 30), (128, 300), (8, 7)])
def test_block_quantiser_invariants(rows, n):
    rng = np.random.default_rng(rows * 1000 + n)
    X = (rng.standard_normal((2, n, 16)) * np.exp(rng.uniform(-3, 3, (2, n, 1)))).astype(np.float32)
    X[1, :min(rows, n)] = 0.0  # one all-zero block
    codes, sc = oracle.quantize_e4m3_rows(X, rows)
    nb = -(-n // rows)
    assert codes.shape == X.shape and codes.dtype == np.uint8 and sc.shape == (2, nb)
    for b in range(2):
        for j in range(nb):
            blk = X[b, j * rows:(j + 1) * rows]
            amax = np.abs(blk).max()
            cb = codes[b, j * rows:(j + 1) * rows]
            v = oracle.e4m3_decode(cb)
            if amax == 0:
                assert sc[b, j] == 1.0 and np.all(v == 0)
                continue
            assert sc[b, j] == np.float32(amax / np.float32(448.0))
            # the block's largest element takes the largest code
            assert np.abs(v).max() == 448.0
            # every element within half a code step (relative 2^-4 for normals,
            # absolute 2^-10 in code units for subnormals)
            y = blk.astype(np.float64) * float(np.float32(448.0) / np.float32(amax))
            tol = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) * 1.0001
            assert np.all(np.abs(v - y) <= tol)
    Xd = oracle.dequantize_e4m3_rows(codes, sc, rows)
    assert np.all(np.abs(Xd - X) <= np.abs(X) * 2.0 ** -4 * 1.0001 + 2.0 ** -10 * np.repeat(sc, rows, axis=-1)[..., :n, None])
