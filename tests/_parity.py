"""Comparison helpers for GPU-vs-oracle parity tests (test infrastructure)."""
import numpy as np

from oracle import qvla_oracle as O

# bf16 output tolerance: |gpu - ref| <= ATOL + RTOL * |ref|
Y_ATOL = 2e-2
Y_RTOL = 1e-2
# end-to-end activation codes: a code may differ by 1 only where x'/s lies
# within BOUNDARY of a rounding boundary j + 1/2, on at most MAX_FLIP_FRAC of
# the elements
BOUNDARY = 1e-5
MAX_FLIP_FRAC = 1e-4
# 8-bit codes: the same fp32 rotation error, measured in code units, is 127/7
# times larger (codes span +-127 instead of +-7), so the window scales with it
BOUNDARY_8BIT = 2e-4


def unpack(b):
    return O.unpack_nibbles(np.asarray(b))


def check_codes_near_boundary(q_gpu, q_ref, xr_ref, s_ref, what="codes", boundary=BOUNDARY):
    """Returns the number of allowed flips; raises AssertionError otherwise."""
    q_gpu = np.asarray(q_gpu, np.int64)
    q_ref = np.asarray(q_ref, np.int64)
    d = q_gpu - q_ref
    bad = d != 0
    n = int(bad.sum())
    if n == 0:
        return 0
    assert np.abs(d[bad]).max() == 1, f"{what}: a code differs by more than 1"
    s = np.broadcast_to(np.asarray(s_ref, np.float64).reshape(-1, 1), q_ref.shape)
    t = np.asarray(xr_ref, np.float64)[bad] / s[bad]
    dist = np.abs(t - (np.floor(t) + 0.5))
    assert (dist < boundary).all(), (
        f"{what}: {int((dist >= boundary).sum())} flips away from a rounding boundary "
        f"(max distance {dist.max():.3g})")
    assert n <= MAX_FLIP_FRAC * q_ref.size, f"{what}: {n} flips of {q_ref.size} elements"
    return n


def check_y(y_gpu, y_ref, what="y"):
    y_gpu = np.asarray(y_gpu, np.float64)
    y_ref = np.asarray(y_ref, np.float64)
    err = np.abs(y_gpu - y_ref)
    lim = Y_ATOL + Y_RTOL * np.abs(y_ref)
    worst = float((err - lim).max()) if err.size else 0.0
    assert (err <= lim).all(), f"{what}: {int((err > lim).sum())} outputs outside tolerance " \
                               f"(worst excess {worst:.3g})"


def check_gptq_flips(q_gpu, q_ref, t_ref, boundary, max_frac, what="GPTQ codes"):
    """GPTQ codes from a factor that differs from the oracle's by rounding.

    The error feedback carries a flipped code along its row, so only the
    first flip of each row is a rounding decision of its own: it must differ
    by 1 and lie where the oracle's quotient w/s is within `boundary` of a
    half-integer.  Later flips in that row follow from it.  Returns the
    number of flipped codes (at most max_frac of them, and at least 1
    allowed)."""
    q_gpu = np.asarray(q_gpu, np.int64)
    q_ref = np.asarray(q_ref, np.int64)
    d = q_gpu - q_ref
    n = int((d != 0).sum())
    for r in np.nonzero((d != 0).any(axis=1))[0]:
        j = int(np.argmax(d[r] != 0))
        t = float(t_ref[r, j])
        dist = abs(t - (np.floor(t) + 0.5))
        assert abs(int(d[r, j])) == 1, f"{what}: row {r} first flip differs by {d[r, j]}"
        assert dist < boundary, (f"{what}: row {r} first flip at column {j} is {dist:.3g} "
                                 f"from a rounding boundary")
    assert n <= max(1, max_frac * q_ref.size), f"{what}: {n} flips of {q_ref.size}"
    return n
