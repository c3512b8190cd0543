"""The certified error bound of the selection's tensor-core scores, checked
on the host by emulating the arithmetic it covers (no GPU).

The score kernel forms S~ = q_hi.k_hi + q_hi.k_lo + q_lo.k_hi from a
two-term bf16 split of each float64 block mean (f = float32(m),
hi = bf16(f), lo = bf16(f - hi)) and accumulates the 3d exact products in
float32; the selection trusts
    |S~ - S| <= E = (3.1 2^-16 + 3.09 d 2^-23) |q| |k|    (times 1.05)
with S the float64 dot product of the means.  Here the products are summed
in float32 in several orders (sequential, reversed, pairwise, by channel
groups), with rounding to nearest and toward zero, on means of mixed
magnitude and with heavy cancellation, and every error must stay under E.
"""
import numpy as np
import pytest


def bf16_rn(x32):
    """float32 -> bf16 (round to nearest even), returned as float32."""
    b = np.asarray(x32, np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32)


def split(m64):
    f = m64.astype(np.float32)
    hi = bf16_rn(f)
    lo = bf16_rn((f - hi).astype(np.float32))
    return hi, lo


def toward_zero32(x64):
    """float64 -> float32 rounded toward zero."""
    f = np.float32(x64)
    if abs(np.float64(f)) > abs(x64):
        f = np.nextafter(f, np.float32(0))
    return f


def sums32(terms):
    """float32 sums of the exact float64 terms in several orders/roundings."""
    out = []
    for order in (terms, terms[::-1], np.sort(terms), np.sort(terms)[::-1]):
        acc = np.float32(0)
        for t in order:                       # sequential, round to nearest
            acc = np.float32(np.float64(acc) + np.float64(np.float32(t)))
        out.append(acc)
        acc = np.float32(0)
        for t in order:                       # sequential, toward zero
            acc = toward_zero32(np.float64(acc) + np.float64(np.float32(t)))
        out.append(acc)
    v = terms.astype(np.float32)              # pairwise tree, round to nearest
    while len(v) > 1:
        if len(v) % 2:
            v = np.append(v, np.float32(0))
        v = (v[0::2].astype(np.float64) + v[1::2].astype(np.float64)).astype(np.float32)
    out.append(v[0])
    return out


def bound(d, qn, kn):
    return (3.1 * 2.0 ** -16 + 3.09 * d * 2.0 ** -23) * 1.05 * qn * kn


@pytest.mark.parametrize("d", [64, 128])
def test_split_score_error_within_bound(d):
    rng = np.random.default_rng(d)
    worst = 0.0
    for trial in range(60):
        scale = 10.0 ** rng.uniform(-3, 3, size=d)            # mixed magnitudes
        q = rng.standard_normal(d) * scale
        k = rng.standard_normal(d) * scale[rng.permutation(d)]
        if trial % 3 == 0:                                    # heavy cancellation
            k = k - q * (q @ k) / (q @ q)
        qh, ql = split(q)
        kh, kl = split(k)
        # Products of bf16 values are exact in float64 (and in float32).
        terms = np.concatenate([qh.astype(np.float64) * kh, qh.astype(np.float64) * kl,
                                ql.astype(np.float64) * kh])
        assert np.array_equal(terms.astype(np.float32).astype(np.float64), terms)
        exact = float(q @ k)
        E = bound(d, np.linalg.norm(q), np.linalg.norm(k))
        for s in sums32(terms):
            err = abs(float(s) - exact)
            assert err <= E, (trial, err, E)
            worst = max(worst, err / E)
    assert worst > 1e-4          # the bound is not vacuous: errors reach a visible fraction


def test_split_reconstructs_the_mean():
    # |m - (hi + lo)| <= 1.004 2^-16 |m|: the per-element step of the bound.
    # Worst cases sit just below a power of two in the remainder's binade.
    rng = np.random.default_rng(1)
    m = rng.standard_normal(100000) * 10.0 ** rng.uniform(-20, 20, size=100000)
    worst = np.float64(1.0) + 2.0 ** -8 * (1 - 2.0 ** -8)     # r at a bf16 rounding tie
    m = np.concatenate([m, [worst, -worst * 3.0, 1.0 + 2.0 ** -9 + 2.0 ** -17]])
    hi, lo = split(m)
    rel = np.abs(hi.astype(np.float64) + lo - m) / np.abs(m)
    assert rel.max() <= 1.004 * 2.0 ** -16
    assert rel.max() > 2.0 ** -18          # and the old 2^-18 claim would not hold
