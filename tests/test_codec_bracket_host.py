"""The codec's fast path, checked on the host with IEEE fp32 arithmetic.

The GPU codec does not divide: it takes r = an approximate reciprocal of the
scale S (within 1 ulp of 1/S), forms r_lo = fl32(r (1 - 2^-20)) and
r_hi = fl32(r (1 + 2^-20)), and multiplies x by both. It keeps the code of
fl32(x r_lo) when fl32(x r_hi) encodes to the same code, and divides only
otherwise. That is exact because the two products lie strictly on either side
of fl32(x / S) (and rounding onto the E2M1 or E4M3 grid is monotone). This
test checks the bracket with numpy's fp32 multiply and divide (both correctly
rounded, like mul.rn.f32 and div.rn.f32) for every reciprocal within 1 ulp of
1/S, over bf16 inputs of all binades and scales across the fast path's range
[2^-126, 2^100]."""
import numpy as np

F32 = np.float32
LO = F32(1.0 - 2.0 ** -20)
HI = F32(1.0 + 2.0 ** -20)


def _bf16_values(rng, n):
    """Random bf16 bit patterns (finite, nonzero), widened to fp32."""
    exp = rng.integers(1, 255, n, dtype=np.uint32)
    man = rng.integers(0, 128, n, dtype=np.uint32)
    sign = rng.integers(0, 2, n, dtype=np.uint32)
    bits = (sign << 31) | (exp << 23) | (man << 16)
    return bits.view(np.float32)


def _check(x, S):
    q = (x / S).astype(F32)  # fl32(x / S)
    r0 = (F32(1.0) / S).astype(F32)
    for r in (np.nextafter(r0, F32(0)), r0, np.nextafter(r0, F32(np.inf))):
        r_lo = (r * LO).astype(F32)
        r_hi = (r * HI).astype(F32)
        lo = (x * r_lo).astype(F32)
        hi = (x * r_hi).astype(F32)
        # keep quotients in the normal fp32 range (smaller ones are code 0 on
        # either side of the bracket; larger ones saturate)
        keep = (np.abs(q) >= F32(2.0 ** -120)) & (np.abs(q) <= F32(2.0 ** 120))
        pos = keep & (x > 0)
        neg = keep & (x < 0)
        assert np.all(lo[pos] < q[pos]) and np.all(q[pos] < hi[pos])
        assert np.all(hi[neg] < q[neg]) and np.all(q[neg] < lo[neg])
        assert keep.sum() > len(x) // 4


def test_bracket_holds_over_scales_and_binades():
    rng = np.random.default_rng(2024)
    with np.errstate(over="ignore", under="ignore"):
        for _ in range(40):
            n = 50_000
            x = _bf16_values(rng, n)
            # scales as the codec meets them: E4M3 block scale times a global
            # scale, over the whole fast-path range
            S = np.ldexp(rng.uniform(1.0, 2.0, n), rng.integers(-126, 100, n)).astype(F32)
            _check(x, S)


def test_bracket_at_exact_quotients_and_ties():
    """x / S exactly on the E2M1 grid, on its rounding thresholds and one
    bf16 step either side: the bracket still encloses fl32(x / S)."""
    rng = np.random.default_rng(7)
    grid = np.array([0.25, 0.5, 0.75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6], F32)
    e4m3 = np.ldexp(np.arange(8, 16, dtype=np.float64) / 8, np.arange(-6, 9)[:, None]).ravel()
    with np.errstate(over="ignore", under="ignore"):
        for g in (1.0, 0.37, 2.0 ** -40, 2.0 ** 60, 1.0 / 2688):
            S = (e4m3.astype(F32) * F32(g)).astype(F32)
            S = np.repeat(S, grid.size)
            xv = (np.tile(grid, e4m3.size) * S).astype(F32)
            xb = (xv.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)
            for step in (-1, 0, 1):
                x = (xb.view(np.uint32).astype(np.int64) + step * (1 << 16)).astype(np.uint32).view(np.float32)
                sgn = np.where(rng.random(x.size) < 0.5, F32(-1), F32(1))
                _check((x * sgn).astype(F32), S)
