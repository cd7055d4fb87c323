"""The 8-bit kernel's quantization by slices of |x|, checked on the CPU.

The kernel finds the code of the map value nearest to x without a search:
|x| in [2^-23, 1] falls in one of 24 binades x 128 slices (the exponent and
the top 7 fraction bits), each slice holds at most one threshold between
neighbouring map values, and its entry gives the code at the slice's bottom
plus one if |x| is above that threshold; negative x in the signed map use the
mirror code 254 - c (one lower at an exact midpoint); |x| below 2^-23 takes
the code of 0.  These tests rebuild that rule from the pinned oracle map and
check its premises and its result against the oracle's brute-force nearest
code, over random values, every threshold and its neighbours, and exact ties.
"""
import numpy as np
import pytest


def _thresholds(qmap):
    mid = (qmap[:-1].astype(np.float64) + qmap[1:].astype(np.float64)) / 2
    t = mid.astype(np.float32)
    t = np.where(t.astype(np.float64) > mid, np.nextafter(t, np.float32(-np.inf)), t)   # round down
    return t.astype(np.float32), t.astype(np.float64) == mid


def _slices(qmap):
    thr, exact = _thresholds(qmap)
    lo_bits = ((np.arange(24)[:, None] + 127 - 23) << 23 | (np.arange(128)[None, :] << 16)).reshape(-1)
    lo = lo_bits.astype(np.uint32).view(np.float32)
    hi = (lo_bits + (1 << 16)).astype(np.uint32).view(np.float32)
    base = np.searchsorted(thr, lo, side="left")              # thresholds strictly below lo
    inside = [(thr >= a) & (thr < b) for a, b in zip(lo, hi)]
    return thr, exact, lo, hi, base, inside


def _code(qmap, slices, x, signed):
    thr, exact, lo, hi, base, inside = slices
    out = []
    for v in np.asarray(x, np.float32):
        a = abs(float(v))
        if a < 2.0 ** -23:
            out.append(127 if signed else 0)
            continue
        bits = int(np.float32(a).view(np.uint32))
        s = ((bits >> 23) - (127 - 23)) * 128 + ((bits >> 16) & 0x7F)
        c = int(base[s])
        t = thr[c] if c < 255 and thr[c] < hi[s] else np.float32(np.inf)
        tie = c < 255 and thr[c] < hi[s] and bool(exact[c]) and a == float(t)
        c += 1 if a > float(t) else 0
        if signed and v < 0:
            c = max(0, 254 - c - (1 if tie else 0))
        out.append(c)
    return np.array(out, np.uint8)


@pytest.mark.parametrize("signed", [True, False])
def test_every_slice_holds_at_most_one_threshold(oracle_mod, signed):
    qmap = oracle_mod.quant_map(signed)
    *_, inside = _slices(qmap)
    assert max(int(m.sum()) for m in inside) <= 1
    thr, _ = _thresholds(qmap)
    pos = thr[thr > 0]
    assert pos.min() > 2.0 ** -23          # below 2^-23 the nearest value is 0


@pytest.mark.parametrize("signed", [True, False])
def test_slice_rule_gives_the_nearest_code(oracle_mod, signed):
    qmap = oracle_mod.quant_map(signed)
    sl = _slices(qmap)
    thr, exact = _thresholds(qmap)
    g = np.random.Generator(np.random.Philox(71))
    lo = -1.0 if signed else 0.0
    xs = [g.uniform(lo, 1.0, 3000), np.sign(g.uniform(lo, 1.0, 3000)) * 10.0 ** g.uniform(-9, 0, 3000),
          qmap, thr, np.nextafter(thr, np.float32(2)), np.nextafter(thr, np.float32(-2)),
          np.array([0.0, 1.0, 2.0 ** -23, np.nextafter(np.float32(2.0 ** -23), np.float32(0))])]
    if signed:
        xs += [-thr, -np.nextafter(thr, np.float32(2)), -qmap, np.array([-1.0, -(2.0 ** -23)])]
    x = np.concatenate([np.asarray(a, np.float64) for a in xs]).astype(np.float32)
    x = x[(x >= -1) & (x <= 1)]
    assert np.array_equal(_code(qmap, sl, x, signed), oracle_mod.quantize(qmap, x))
    assert exact.sum() > 50                 # exact ties are among the cases
