"""The compress kernel decides q != 0 without dividing:

    fl(|x'| / scale) >= 1/2   <=>   |x'| >= T,
    T = least fp32 value >= scale * (1/2 - 2^-26)   (product exact in fp64).

This checks the identity against IEEE fp32 division (numpy) on the CPU, for
scales across the whole fp32 range (subnormals included) and for |x'| at,
just below and just above T, and at random points of [0, scale].
"""
from __future__ import annotations

import numpy as np

import synth


def threshold(scale: np.float32) -> np.float32:
    t64 = float(scale) * (0.5 - 2.0 ** -26)          # exact: 24 + 25 significant bits
    t = np.float32(t64)
    if float(t) < t64:
        t = np.nextafter(t, np.float32(np.inf))
    return t


def by_division(xa, scale):
    with np.errstate(divide="ignore", invalid="ignore", under="ignore"):
        return (xa / scale) >= np.float32(0.5)


def test_identity_near_the_threshold():
    key = synth.key_for(31, 0)
    u = synth.uniforms(key, 4000)
    # scales from subnormal to near FLT_MAX/2, plus exact powers of two
    expo = (u * 250 - 148).astype(np.int64)
    mant = 1.0 + synth.uniforms(synth.key_for(31, 1), 4000)
    scales = [np.float32(np.ldexp(m, int(e))) for m, e in zip(mant, expo)]
    scales += [np.float32(2.0 ** k) for k in range(-149, 127)]
    scales += [np.float32(np.ldexp(1.5, -149)), np.float32(1.9990234375)]
    checked = 0
    for sc in scales:
        if not np.isfinite(sc) or sc == 0:
            continue
        t = threshold(sc)
        xs = [t, np.nextafter(t, np.float32(0)), np.nextafter(t, np.float32(np.inf)),
              np.float32(sc), np.float32(sc * np.float32(0.5))]
        xa = np.array([v for v in xs if 0 <= v <= sc], np.float32)
        assert np.array_equal(xa >= t, by_division(xa, sc))
        checked += xa.size
    assert checked > 15000


def test_identity_on_random_values():
    for seed in range(6):
        key = synth.key_for(900 + seed, 0)
        sc = np.float32(np.ldexp(1.0 + synth.uniforms(key, 1)[0], int(seed * 20 - 60)))
        xa = (synth.uniforms(synth.key_for(key, 1), 200000) * float(sc)).astype(np.float32)
        xa = np.minimum(xa, sc)
        assert np.array_equal(xa >= threshold(sc), by_division(xa, sc))


def test_plain_half_scale_comparison_fails_on_subnormal_scales():
    """|x'| >= fl(scale/2) agrees with the division for normal scales (no fp32
    value lies between scale*(1/2 - 2^-26) and scale/2 there), but not when
    scale/2 rounds: at scale = 2^-149 it rounds to 0 and would make q != 0
    for x' = 0.  The threshold T has no such case."""
    sc = np.float32(np.ldexp(1.0, -149))
    xa = np.array([0.0, sc], np.float32)
    naive = xa >= sc / np.float32(2)
    exact = by_division(xa, sc)
    assert exact.tolist() == [False, True]
    assert naive.tolist() == [True, True]
    assert (xa >= threshold(sc)).tolist() == exact.tolist()
