"""The argument the GPU quantizer rests on, checked on the CPU: for r > 0 and
an approximate reciprocal inv within 2^-22 of 1/r, p = RN(x * inv); when
RN(p (1 - 2^-18)) and RN(p (1 + 2^-18)) have the same E2M1 code, that is the
code of the IEEE quotient RN(x / r).  Values are drawn uniformly, on every
E2M1 rounding boundary of r and within a few ulps of it, with reciprocals
perturbed to the edges of the allowed error.  numpy float32 multiply and
divide are IEEE round-to-nearest; codes come from the oracle's encoder."""
import numpy as np

import oracle

LO, HI = np.float32(1 - 2.0 ** -18), np.float32(1 + 2.0 ** -18)
MIDS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def _codes(v):
    return oracle.e2m1_encode(np.asarray(v, np.float32))


def test_bracket_agreement_implies_the_exact_code():
    rng = np.random.default_rng(5)
    agreed = 0
    for _ in range(40):
        r = np.float32(rng.uniform(1e-3, 10.0))
        xs = [np.float32(rng.uniform(-7.0, 7.0) * r) for _ in range(40)]
        for m in MIDS:
            v = np.float32(m * np.float64(r))
            for k in range(-3, 4):
                w = v
                for _ in range(abs(k)):
                    w = np.nextafter(w, np.float32(np.inf) if k > 0 else np.float32(0))
                xs += [w, -w]
        x = np.array(xs, np.float32)
        exact = _codes(x / r)                                   # RN(x / r), then E2M1
        for eps in (-2.0 ** -22, 0.0, 2.0 ** -22):              # reciprocal at the edges of its error
            inv = np.float32((1.0 / np.float64(r)) * (1.0 + eps))
            p = (x * inv).astype(np.float32)
            c_lo, c_hi = _codes(p * LO), _codes(p * HI)
            same = c_lo == c_hi
            assert (c_hi[same] == exact[same]).all()
            agreed += int(same.sum())
    # the uniformly drawn elements are nearly all decided by the bracket; the
    # ones placed within a few ulps of a boundary are left to the division
    assert agreed >= 0.95 * 40 * 3 * 40
