"""The error bounds behind the two fp16 tensor-core scorers, checked on the CPU.

Two kernels score with fp16 mma.sync and keep exactness by re-scoring, in
fp32, everything a proven bound cannot decide: the k-means assignment and
the row-max block selection.  Both bounds are checked here.

k-means.  km_assign_mma_kernel (csrc/kmeans.cu) computes D = |mu|^2 - 2 x~.mu~ with an
mma.sync m16n8k16: x and -2 mu rounded to fp16, the accumulator seeded with
the exact path's fp32 |mu|^2.  It decides a key only when the other groups'
smallest D exceeds its smallest D by more than 2E, with

    E = 1.125 * 2^-9 |x| M + 2^-16 M^2 + 2^-20 (|x| + M),   M = max_c |mu_c|

(|x| and M as the kernel computes them in fp32), and re-scores every other
key with the exact path: |mu|^2 and x.mu as fp32 fma chains in dimension
order, then fma(-2, x.mu, |mu|^2).  The assignment is the exact path's only
if |D - exact| <= E for every key and centroid.

The tensor core's accumulation order and rounding are not documented, so
this test computes D under several accumulation models (one rounding of the
exact sum; a chain in dimension order rounded to nearest or toward zero at
every step; a pairwise tree rounded to nearest or toward zero), all in exact
rational arithmetic with explicit fp32 rounding, and the exact path with a
correctly rounded fma.  Inputs are adversarial: magnitudes from fp16's
subnormal range up to the kernel's limits (|x| < 30000, M <= 8192),
components placed on fp16 half-way points, mixed scales and near-cancelling
distances.  Every model must stay within E.

Row-max selection.  block_select_rowmax_kernel (csrc/select.cu) scores the
rows u_i of a query block against candidate centroids c_j as fp16 MMAs of
su u (su a power of two putting every entry below 2^14) and c, accumulated
from zero in fp32, and keeps for exact re-scoring every candidate whose
approximate row maximum lies within 2E of the k-th, with
    E = 2^-9 max|su u_i| max|c_j| + 2^-22 (max|su u_i| + max|c_j|)
(the maxima as the kernel forms them in fp32, with a 1.001 factor).  The
exact score is u_i . c_j in two fp32 fma chains of eight ranks, then their
sum; each approximate product must lie within E of su times it.
"""

from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

R = 16  # rank of the projected keys


def round32(v: Fraction, toward_zero: bool = False) -> Fraction:
    """v rounded to the nearest fp32 value (ties to even), or toward zero."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = -v if v < 0 else v
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    e = max(e, -126)  # subnormals share the smallest normal exponent
    scale = Fraction(2) ** (e - 23)
    q, rem = divmod(a / scale, 1)
    q = int(q)
    if not toward_zero and (rem > Fraction(1, 2) or (rem == Fraction(1, 2) and q % 2 == 1)):
        q += 1
    out = q * scale
    assert out < Fraction(2) ** 128, "fp32 overflow"
    return sign * out


def F(v) -> Fraction:
    return v if isinstance(v, Fraction) else Fraction(float(v))


def fma32(a, b, c):
    return round32(F(a) * F(b) + F(c))


def to_f16(x: float) -> Fraction:
    """fp32 -> fp16, round to nearest even (numpy's conversion)."""
    h = np.float16(np.float32(x))
    assert np.isfinite(h)
    return Fraction(float(h))


def exact_path(x, mu):
    """The kernel's fp32 distance (exact_assign / exact_dist)."""
    sq = Fraction(0)
    for d in range(R):
        sq = fma32(mu[d], mu[d], sq)
    dot = Fraction(0)
    for d in range(R):
        dot = fma32(x[d], mu[d], dot)
    return fma32(-2.0, dot, sq), sq


def mma_models(x, mu, nrm):
    """D under several accumulation models of the tensor core."""
    p = [to_f16(x[d]) * to_f16(-2.0 * float(mu[d])) for d in range(R)]  # products are exact
    c = Fraction(nrm)
    out = {"exact_sum": round32(c + sum(p))}
    for tz in (False, True):
        acc = c
        for v in p:
            acc = round32(acc + v, tz)
        out[f"chain_{'rz' if tz else 'rn'}"] = acc
        level = p
        while len(level) > 1:
            level = [round32(level[i] + level[i + 1], tz) for i in range(0, len(level), 2)]
        out[f"tree_{'rz' if tz else 'rn'}"] = round32(level[0] + c, tz)
    return out


def kernel_xnorm(x):
    """|x| as the kernel forms it: per lane fma over dims (2q, 2q+1, 2q+8,
    2q+9), then the quad's four partial sums added by shuffles, in fp32."""
    part = []
    for q in range(4):
        lo0, lo1, hi0, hi1 = (np.float32(x[i]) for i in (2 * q, 2 * q + 1, 2 * q + 8, 2 * q + 9))
        t = round32(F(hi1) * F(hi1))
        t = fma32(hi0, hi0, t)
        t = fma32(lo1, lo1, t)
        t = fma32(lo0, lo0, t)
        part.append(t)
    s01 = [round32(part[0] + part[1]), round32(part[2] + part[3])]
    s = round32(s01[0] + s01[1])
    return math.sqrt(float(s))


def bound(xn, M):
    return 1.125 * 2.0 ** -9 * xn * M + 2.0 ** -16 * M * M + 2.0 ** -20 * (xn + M)


def f16_halfway(rng, n, exp_lo, exp_hi):
    """fp32 values on (or one fp32 ulp off) the midpoint between two fp16 values."""
    e = rng.integers(exp_lo, exp_hi, n)
    m = rng.integers(0, 1024, n)
    v = ((1.0 + (m + 0.5) / 1024.0) * np.exp2(e.astype(np.float64))).astype(np.float32)
    nudge = rng.integers(-1, 2, n)
    up, down = np.nextafter(v, np.float32(np.inf)), np.nextafter(v, np.float32(-np.inf))
    v = np.where(nudge > 0, up, np.where(nudge < 0, down, v)).astype(np.float32)
    return v * rng.choice(np.array([-1.0, 1.0], dtype=np.float32), n)


def cases(rng):
    out = []
    for sx, sm in [(1.0, 1.0), (1e-3, 1.0), (1.0, 1e-3), (1e-6, 1e-6), (2e-5, 3.0), (50.0, 40.0), (1500.0, 1500.0)]:
        for _ in range(6):
            out.append((rng.standard_normal(R).astype(np.float32) * np.float32(sx),
                        rng.standard_normal((8, R)).astype(np.float32) * np.float32(sm)))
    for lo, hi in [(-24, -14), (-14, -4), (-2, 4), (8, 11)]:  # subnormal fp16 range up to large values
        for _ in range(6):
            out.append((f16_halfway(rng, R, lo, hi), f16_halfway(rng, 8 * R, lo, hi).reshape(8, R)))
    for _ in range(6):  # near the limits: |x| just below 30000, M just below 8192
        x = rng.standard_normal(R)
        x = (x / np.linalg.norm(x) * 29990.0).astype(np.float32)
        mu = rng.standard_normal((8, R))
        mu = (mu / np.linalg.norm(mu, axis=1, keepdims=True) * 8180.0).astype(np.float32)
        out.append((x, mu))
    # coherent worst case: every component one fp32 ulp above the midpoint
    # (1 + 2^-11) 2^e, so every fp16 rounding goes up by almost 2^-11 relative,
    # and x parallel to mu, so the product errors add up instead of cancelling
    def up(e):
        return np.nextafter(np.float32((1.0 + 2.0 ** -11) * 2.0 ** e), np.float32(np.inf))
    for ex, em in [(0, 0), (10, 10), (-5, 3), (12, 11), (-13, -13), (6, -2)]:
        out.append((np.full(R, up(ex), np.float32), np.full((8, R), up(em), np.float32)))
    for _ in range(6):  # near-cancelling distances: mu close to 2x along x, |mu|^2 ~ 2 x.mu
        x = (rng.standard_normal(R) * 40.0).astype(np.float32)
        mu = np.stack([2 * x + rng.standard_normal(R).astype(np.float32) * np.float32(1e-3) for _ in range(8)])
        out.append((x, mu.astype(np.float32)))
    return out


def test_tensor_core_distance_stays_within_the_bound():
    rng = np.random.default_rng(2024)
    worst, checked = 0.0, 0
    for x, mus in cases(rng):
        xn = kernel_xnorm(x)
        nrms = [exact_path(x, mu)[1] for mu in mus]
        M = math.sqrt(float(max(nrms)))
        if not (xn < 30000.0 and M <= 8192.0):  # the kernel leaves such keys to the exact path
            continue
        checked += 1
        E = bound(xn, M)
        for mu, nrm in zip(mus, nrms):
            ex, _ = exact_path(x, mu)
            for name, D in mma_models(x, mu, nrm).items():
                err = abs(float(D - ex))
                worst = max(worst, err / E)
                assert err <= E, (name, err, E, xn, M)
    print(f"largest |D - exact| / E: {worst:.3f} over {checked} keys x 8 centroids")
    assert checked >= 76 and worst > 0.5  # the coherent cases come close to the bound


def test_round32_matches_numpy():
    rng = np.random.default_rng(5)
    for v in np.concatenate([rng.standard_normal(200) * np.exp2(rng.integers(-140, 120, 200)),
                             [1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24, 2.0 ** -149 * 1.5, 2.0 ** -149 * 2.5]]):
        assert float(round32(Fraction(float(v)))) == float(np.float32(v))


# ------------------------------------------------------------ row-max scores


def two_chains(u, c):
    """score16_two_chains: ranks 0-7 and 8-15 in two fp32 fma chains, then added."""
    s0 = round32(F(u[0]) * F(c[0]))
    s1 = round32(F(u[8]) * F(c[8]))
    for d in range(1, 8):
        s0 = fma32(u[d], c[d], s0)
        s1 = fma32(u[8 + d], c[8 + d], s1)
    return round32(s0 + s1)


def rowmax_scale_and_bound(U, Cs):
    """su, and E in the scaled unit, as block_select_rowmax_kernel forms them."""
    un2 = []
    for u in U:
        t = Fraction(0)
        for d in range(R):
            t = fma32(u[d], u[d], t)
        un2.append(t)
    umax = np.float32(math.sqrt(float(max(un2)))) * np.float32(1.001)
    _, ue = math.frexp(float(umax))
    su = 2.0 ** (14 - ue) if umax > 0 else 1.0
    cn2 = [sum(float(np.float32(c[d]) * np.float32(c[d])) for d in range(R)) for c in Cs]
    cmax = float(np.float32(math.sqrt(max(cn2))) * np.float32(1.001))
    sumax = su * float(umax)
    return su, 2.0 ** -9 * sumax * cmax + 2.0 ** -22 * (sumax + cmax), cmax


def mma_models_from_zero(a, b):
    """sum_d fp16(a_d) fp16(b_d) accumulated from zero under the same models."""
    p = [to_f16(a[d]) * to_f16(b[d]) for d in range(R)]
    out = {"exact_sum": round32(sum(p))}
    for tz in (False, True):
        acc = Fraction(0)
        for v in p:
            acc = round32(acc + v, tz)
        out[f"chain_{'rz' if tz else 'rn'}"] = acc
        level = p
        while len(level) > 1:
            level = [round32(level[i] + level[i + 1], tz) for i in range(0, len(level), 2)]
        out[f"tree_{'rz' if tz else 'rn'}"] = level[0]
    return out


def rowmax_cases(rng):
    out = []
    for su_, sc in [(1.0, 1.0), (1e-4, 3.0), (30.0, 1e-3), (1e-7, 1e-7), (500.0, 2000.0)]:
        for _ in range(5):
            out.append(((rng.standard_normal((4, R)) * su_).astype(np.float32),
                        (rng.standard_normal((6, R)) * sc).astype(np.float32)))
    for lo, hi in [(-24, -14), (-6, 2), (6, 12)]:
        for _ in range(5):
            out.append((f16_halfway(rng, 4 * R, lo, hi).reshape(4, R), f16_halfway(rng, 6 * R, lo, hi).reshape(6, R)))

    def up(e):
        return np.nextafter(np.float32((1.0 + 2.0 ** -11) * 2.0 ** e), np.float32(np.inf))
    for eu, ec in [(0, 0), (-9, 5), (7, -3), (3, 12)]:  # coherent: every fp16 rounding upward
        out.append((np.full((4, R), up(eu), np.float32), np.full((6, R), up(ec), np.float32)))
    return out


def test_rowmax_approximate_scores_stay_within_the_bound():
    rng = np.random.default_rng(77)
    worst, checked = 0.0, 0
    for U, Cs in rowmax_cases(rng):
        su, E, cmax = rowmax_scale_and_bound(U, Cs)
        if not cmax < 32768.0:  # the kernel then scores every candidate exactly
            continue
        checked += 1
        for u in U:
            su_u = [np.float32(su * float(u[d])) for d in range(R)]
            assert max(abs(float(v)) for v in su_u) < 2.0 ** 14
            for c in Cs:
                ex = Fraction(su) * two_chains(u, c)  # scaling by a power of two is exact
                for name, D in mma_models_from_zero(su_u, c).items():
                    err = abs(float(D - ex))
                    worst = max(worst, err / E)
                    assert err <= E, (name, err, E)
    print(f"row-max: largest |a - su s| / E: {worst:.3f} over {checked} blocks")
    assert checked >= 35 and worst > 0.3  # the coherent cases come close to half the bound
