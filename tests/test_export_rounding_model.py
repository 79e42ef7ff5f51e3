"""The export kernels' rounding shortcut, checked on the CPU.

Per row the int8 code of x is rne(fl(x / s)), s = fl(a / 127), a = max|x|.
The GPU kernels instead take p = fl(x * fl(1 / s)), round it by adding
1.5 * 2^23 (the integer then sits in the low mantissa bits, ties to even),
and use that whenever every value of the lane lies more than 1e-4 from a
half-integer (|p - rint(p)| <= 0.4999); otherwise the lane recomputes its
values from fl(x / s).  p is within about 2^-23 |x/s| <= 1.6e-5 of x/s and
fl(x/s) within 2^-24 |x/s|, so both round the same way outside that margin.

This test restates those steps with numpy binary32 arithmetic (the same IEEE
round-to-nearest operations as the kernels' __fmul_rn / __frcp_rn / __fadd_rn /
__fdiv_rn) and checks them against rne(fl(x / s)) on random rows of many
magnitudes and on rows built to land on and next to half-integers.
"""
import numpy as np

F = np.float32
MAGIC = F(12582912.0)  # 1.5 * 2^23


def rne_magic(v):
    y = (v + MAGIC).astype(np.float32)
    return (y.view(np.int32) - np.int32(0x4B400000)), (y - MAGIC).astype(np.float32)


def codes_like_the_kernel(x, lane_width=16):
    """x: float32 [rows][D]; the lane groups are lane_width consecutive values."""
    a = np.abs(x).max(axis=1).astype(np.float32)
    s = (a / F(127.0)).astype(np.float32)
    with np.errstate(divide="ignore", over="ignore"):
        rcp = (F(1.0) / s).astype(np.float32)
    fast = np.isfinite(rcp) & (a != 0)
    with np.errstate(over="ignore", invalid="ignore"):
        p = (x * rcp[:, None]).astype(np.float32)
    t, r = rne_magic(np.where(np.isfinite(p), p, F(0)))
    amb = (np.abs(p - r) > F(0.4999)) | ~np.isfinite(p)
    rows, D = x.shape
    lane_amb = amb.reshape(rows, D // lane_width, lane_width).any(axis=2)
    lane_amb |= ~fast[:, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (x / s[:, None]).astype(np.float32)
    t_slow, _ = rne_magic(np.where(np.isfinite(q), q, F(0)))
    use_slow = np.repeat(lane_amb, lane_width, axis=1)
    out = np.where(use_slow, t_slow, t)
    out = np.clip(out, -127, 127)
    out[a == 0] = 0
    return out.astype(np.int8), s


def codes_by_definition(x):
    a = np.abs(x).max(axis=1).astype(np.float32)
    s = (a / F(127.0)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = (x / s[:, None]).astype(np.float32)
    out = np.clip(np.rint(q.astype(np.float64)), -127, 127)  # rint: half to even
    out[a == 0] = 0
    return out.astype(np.int8), s


def test_random_rows_of_many_magnitudes():
    rng = np.random.default_rng(0)
    rows, D = 20000, 64
    scale = F(10.0) ** rng.uniform(-38, 38, size=(rows, 1)).astype(np.float32)
    x = (rng.standard_normal((rows, D)) * scale).astype(np.float32)
    x[::97] = 0
    got, s1 = codes_like_the_kernel(x)
    want, s2 = codes_by_definition(x)
    assert np.array_equal(s1.view(np.uint32), s2.view(np.uint32))
    assert np.array_equal(got, want)


def test_rows_on_and_next_to_half_integers():
    rng = np.random.default_rng(1)
    rows, D = 20000, 64
    a = (F(10.0) ** rng.uniform(-30, 30, size=rows)).astype(np.float32)
    a[::61] = F(3e-42)  # subnormal absmax: subnormal scale, no finite reciprocal
    s = (a / F(127.0)).astype(np.float32)
    k = rng.integers(-127, 127, size=(rows, D)).astype(np.float32)
    x = ((k + F(0.5)) * s[:, None]).astype(np.float32)
    nudge = rng.integers(-3, 4, size=(rows, D))
    for n in (-3, -2, -1, 1, 2, 3):
        sel = nudge == n
        toward = np.float32(np.inf) if n > 0 else np.float32(-np.inf)
        for _ in range(abs(n)):
            x[sel] = np.nextafter(x[sel], toward)
    x[:, 0] = a  # the absmax element
    got, _ = codes_like_the_kernel(x)
    want, _ = codes_by_definition(x)
    assert np.array_equal(got, want)
    # the shortcut really is bypassed here: many lanes take the quotient
    with np.errstate(over="ignore", divide="ignore", invalid="ignore"):
        p = (x * (F(1.0) / s)[:, None]).astype(np.float32)
    _, r = rne_magic(np.where(np.isfinite(p), p, F(0)))
    assert (np.abs(p - r) > F(0.4999)).mean() > 0.1


def test_a_looser_guard_would_be_wrong():
    """Without the guard (always the product), some codes differ: the guard is
    what makes the shortcut exact."""
    rng = np.random.default_rng(2)
    rows, D = 20000, 64
    a = (F(10.0) ** rng.uniform(-20, 20, size=rows)).astype(np.float32)
    s = (a / F(127.0)).astype(np.float32)
    k = rng.integers(-127, 127, size=(rows, D)).astype(np.float32)
    x = ((k + F(0.5)) * s[:, None]).astype(np.float32)
    x[:, 0] = a
    with np.errstate(over="ignore", divide="ignore"):
        p = (x * (F(1.0) / s)[:, None]).astype(np.float32)
    p = np.where(np.isfinite(p), p, F(0))
    t, _ = rne_magic(p)
    want, _ = codes_by_definition(x)
    assert (np.clip(t, -127, 127).astype(np.int8) != want).any()
