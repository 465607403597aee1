"""Inputs on which the two plausible operation orders of the 4-bit quantizers
give different codes (test fixtures, CPU only).

The pages name the formats ("Nunchaku Lite" docs, "Supported quantization
types" table: nvfp4 with group 16, int4 with group 64) but not the order of
the divisions inside the quantizer.  A value v can be divided by its block
scale d directly, fl(v / d), or multiplied by the block scale's reciprocal,
fl(v * fl(1 / d)).  The two differ by at most a couple of fp32 units in the
last place, so they give different codes only where v / d lies within that
distance of a rounding midpoint of the target grid.  The searches below put
v (or the group maximum a) right next to such midpoints, for a fixed
per-tensor scale s, and keep the inputs whose codes differ between the two
orders.  Every product and quotient is a single IEEE fp32 operation (numpy
float32 scalars), and the grids come from the format decoders.
"""
import numpy as np

from oracle import formats as F

E2M1_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def f32(v):
    return np.float32(v)


def _neighbours(v0, k):
    """v0 and its k fp32 neighbours on each side."""
    out = [f32(v0)]
    lo = hi = f32(v0)
    for _ in range(k):
        lo = np.nextafter(lo, f32(-np.inf))
        hi = np.nextafter(hi, f32(np.inf))
        out += [lo, hi]
    return out


def _e2m1(v):
    return int(F.e2m1_encode(np.array([v], np.float32))[0])


def _e4m3(t):
    return int(F.e4m3_encode_nonneg(np.array([t], np.float32))[0])


def nvfp4_code_cases(s, count, seed=0):
    """(a, v, sb, code_recip, code_div) with a group maximum a whose scale
    byte is sb and an element v whose E2M1 code differs between
    v * fl(1/d) and v / d, d = fl(E4M3(sb) * s)."""
    rng = np.random.default_rng(seed)
    s = f32(s)
    six_s = f32(f32(6.0) * s)
    inv6s = f32(f32(1.0) / six_s)
    cases = []
    for _ in range(20000):
        sb = int(rng.integers(0x20, 0x70))
        val = f32(F.E4M3_VALUE[sb])
        a = f32(val * six_s)                     # t = fl(a * inv6s) lands next to val
        if _e4m3(f32(a * inv6s)) != sb:
            continue
        d = f32(val * s)
        r = f32(f32(1.0) / d)
        m = E2M1_MIDPOINTS[int(rng.integers(len(E2M1_MIDPOINTS)))]
        sign = f32(-1.0) if rng.integers(2) else f32(1.0)
        for v in _neighbours(f32(f32(m) * d), 3):
            v = f32(sign * v)
            if not abs(v) < a:
                continue
            c_rec, c_div = _e2m1(f32(v * r)), _e2m1(f32(v / d))
            if c_rec != c_div:
                cases.append((a, v, sb, c_rec, c_div))
                break
        if len(cases) == count:
            break
    return cases


def nvfp4_scale_cases(s, count, seed=0):
    """(a, sb_recip, sb_div): group maxima a whose E4M3 scale byte differs
    between fl(a * fl(1/fl(6s))) and fl(a / fl(6s))."""
    rng = np.random.default_rng(seed)
    s = f32(s)
    six_s = f32(f32(6.0) * s)
    inv6s = f32(f32(1.0) / six_s)
    cases = []
    for _ in range(20000):
        b = int(rng.integers(0x10, 0x7D))                   # normal bytes with a normal neighbour above
        mid = f32((F.E4M3_VALUE[b] + F.E4M3_VALUE[b + 1]) / 2)
        for a in _neighbours(f32(mid * six_s), 3):
            sr, sd = _e4m3(f32(a * inv6s)), _e4m3(f32(a / six_s))
            if sr != sd:
                cases.append((a, sr, sd))
                break
        if len(cases) == count:
            break
    return cases


def int4_code_cases(count, seed=0):
    """(a, v, sc, q_recip, q_div): a group maximum a (scale sc = bf16(a / 7))
    and an element v whose rint differs between v * fl(1/sc) and v / sc."""
    rng = np.random.default_rng(seed)
    cases = []
    for _ in range(20000):
        a = f32(np.exp(rng.uniform(-4, 4)))
        sc = f32(F.bf16_round(np.array([f32(a / f32(7.0))], np.float32))[0])
        if sc == 0 or np.frexp(sc)[0] == 0.5:               # powers of two have exact reciprocals
            continue
        r = f32(f32(1.0) / sc)
        k = int(rng.integers(-7, 7))
        for v in _neighbours(f32(f32(k + 0.5) * sc), 3):
            if not abs(v) < a:
                continue
            q_rec = int(np.clip(np.rint(f32(v * r)), -8, 7))
            q_div = int(np.clip(np.rint(f32(v / sc)), -8, 7))
            if q_rec != q_div:
                cases.append((a, v, sc, q_rec, q_div))
                break
        if len(cases) == count:
            break
    return cases


def nvfp4_rows(s, n_code=48, n_scale=48, seed=0):
    """Rows of 16-element groups that hold the NVFP4 cases: a code case
    [a, v, 0, ...] or a scale case [a, 0, ...] per group.  Returns
    (rows fp32 [R, 16 * G], list of (row, group, kind, case))."""
    codes = nvfp4_code_cases(s, n_code, seed)
    scales = nvfp4_scale_cases(s, n_scale, seed + 1)
    groups = []
    for c in codes:
        g = np.zeros(16, np.float32)
        g[0], g[1] = c[0], c[1]
        groups.append((g, "code", c))
    for c in scales:
        g = np.zeros(16, np.float32)
        g[0] = c[0]
        groups.append((g, "scale", c))
    per_row = 16
    n_rows = (len(groups) + per_row - 1) // per_row
    rows = np.zeros((n_rows, 16 * per_row), np.float32)
    where = []
    for i, (g, kind, c) in enumerate(groups):
        r, j = divmod(i, per_row)
        rows[r, 16 * j:16 * j + 16] = g
        where.append((r, j, kind, c))
    return rows, where


def int4_rows(count=32, seed=0):
    """Rows of 64-element groups [a, v, 0, ...] holding the INT4 cases."""
    cases = int4_code_cases(count, seed)
    per_row = 8
    n_rows = (len(cases) + per_row - 1) // per_row
    rows = np.zeros((n_rows, 64 * per_row), np.float32)
    where = []
    for i, c in enumerate(cases):
        r, j = divmod(i, per_row)
        rows[r, 64 * j] = c[0]
        rows[r, 64 * j + 1] = c[1]
        where.append((r, j, c))
    return rows, where
