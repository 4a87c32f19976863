"""Helpers shared by the GPU parity tests."""
import numpy as np

# Floating-point parity bar: per element
#   e_i = |y_i - r_i| / max(|r_i|, 1e-2 * max_j |r_j|)  must stay <= 2e-3.
# A plain per-element relative error is ill-posed for outputs near zero (dot
# products of random data cross zero), so the denominator is floored at 1% of
# the output's scale.
REL_TOL = 2e-3
FLOOR = 1e-2


def rel_err(y, ref):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    scale = np.abs(ref).max()
    if scale == 0.0:
        return float(np.abs(y).max())
    den = np.maximum(np.abs(ref), FLOOR * scale)
    return float((np.abs(y - ref) / den).max())


def assert_close(y, ref, tol=REL_TOL, what=""):
    e = rel_err(y, ref)
    assert e <= tol, "%s: max relative error %.3e > %.1e" % (what, e, tol)
    return e


def f16_bits(t):
    """torch float16 tensor -> numpy uint16 bit patterns."""
    return t.detach().cpu().contiguous().numpy().view(np.uint16)


def f16_values(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def to_dev_f16(bits, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits, dtype=np.uint16).view(np.float16).copy()).to(device)


def assert_close_rows(y, ref, tol=REL_TOL, what=""):
    """assert_close over the whole output and over each row (batch element,
    token) on its own scale."""
    y = np.atleast_2d(np.asarray(y))
    ref = np.atleast_2d(np.asarray(ref))
    assert_close(y, ref, tol, what)
    for i in range(y.shape[0]):
        assert_close(y[i], ref[i], tol, "%s, row %d" % (what, i))



def assert_close_f16(y16, ref64, ref16, tol=REL_TOL, what=""):
    """An fp16 output against the oracle where some outputs exceed the fp16
    range: +-inf exactly where the oracle's own fp16 rounding (ref16, bit
    patterns) gives +-inf, the finite outputs within the tolerance on the
    scale of the finite reference values."""
    y = np.asarray(y16, dtype=np.float16).astype(np.float64)
    want = np.asarray(ref16, dtype=np.uint16).view(np.float16).astype(np.float64)
    inf = np.isinf(want)
    assert np.array_equal(np.isinf(y), inf), "%s: infinities differ from the oracle's" % what
    assert np.array_equal(np.sign(y[inf]), np.sign(want[inf])), "%s: signs of inf" % what
    fin = ~inf
    if fin.any():
        assert_close(y[fin], np.asarray(ref64)[fin], tol, what)
