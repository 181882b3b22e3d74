"""The two-part binary16 split the tensor-core GEMM relies on is exact.

The M > 16 path feeds every weight w = q * d (q the signed code: q - 8 of a
Q4_0 nibble, or a Q8_0 byte; d any finite binary16 scale) to the MMA as
main = RN16(w) plus rest = RN16(w - main).  w has at most 4 + 11 (Q4_0) or
8 + 11 (Q8_0) significant bits and is a multiple of d's last bit, so the
remainder is representable and main + rest == w exactly, unless main
overflows.  Checked here for every finite binary16 d and every code, in exact
fp64 arithmetic (each product and difference is exact in fp64).
"""
import numpy as np
import pytest

D = np.arange(0x10000, dtype=np.uint32).astype(np.uint16).view(np.float16)
D = D[np.isfinite(D)].astype(np.float64)


@pytest.mark.parametrize("codes,dmax", [(range(-8, 8), 8188.0), (range(-128, 128), 511.75)])
def test_main_plus_rest_is_exact(codes, dmax):
    for q in codes:
        w = q * D
        with np.errstate(over="ignore", invalid="ignore"):
            main = w.astype(np.float16).astype(np.float64)
            rest = (w - main).astype(np.float16).astype(np.float64)
        fin = np.isfinite(main)
        assert np.array_equal(main[fin] + rest[fin], w[fin]), q
        # overflow only where |w| rounds beyond the binary16 range
        assert np.all(np.abs(w[~fin]) >= 65520.0), q
    # the largest scale for which no code overflows
    big = np.max(np.abs(np.array(list(codes))))
    with np.errstate(over="ignore"):
        ok = np.isfinite((big * D).astype(np.float16))
    assert np.max(np.abs(D[ok])) == dmax
