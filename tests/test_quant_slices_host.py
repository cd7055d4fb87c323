"""The 8-bit kernel's quantization by slices of x, checked on the CPU.

The kernel finds the code of the map value nearest to x without a search:
the exponent of x picks a row (below 2^-23, where the nearest value is 0;
one row per binade up to 2^0; NaN), the top 7 fraction bits a slice of the
row; every slice holds at most one threshold between neighbouring map
values, t the low 16 bits of its magnitude.  The code is the code at the
slice's low end (in value order) plus (low16(x) > t) for x >= 0 or
(low16(x) < t) for x < 0; the entry stores that base in its high half and
0xFFFF - t (x >= 0) or t (x < 0) in its low half, so that the code is
(entry + key) >> 16 with key = low16(x), complemented for x < 0 (a table per
sign; 0 in the low half of a slice without a threshold).  These
tests rebuild that rule from the pinned oracle map and check its premises
and its result against the oracle's brute-force nearest code, over random
values, every threshold and its neighbours, and exact ties.  They also check
the margin the kernel's fast quotient relies on: RN32(m * RN32(1/N)) is within
3 ulp of RN32(m / N).
"""
import numpy as np
import pytest

ROWS = 26


def _thresholds(qmap):
    mid = (qmap[:-1].astype(np.float64) + qmap[1:].astype(np.float64)) / 2
    t = mid.astype(np.float32)
    t = np.where(t.astype(np.float64) > mid, np.nextafter(t, np.float32(-np.inf)), t)   # round down
    return t.astype(np.float32)


def _bits(x):
    return int(np.float32(x).view(np.uint32))


def _table(qmap, neg):
    thr = _thresholds(qmap)
    zero = int(np.nonzero(qmap == 0)[0][0])
    tab = []
    for i in range(ROWS * 128):
        r, k = divmod(i, 128)
        if r == 0:
            tab.append(zero << 16)
            continue
        if r == ROWS - 1:
            tab.append(0)
            continue
        lo_bits = ((r - 1 + 127 - 23) << 23) | (k << 16)
        lo = np.uint32(lo_bits).view(np.float32)
        hi = np.uint32(lo_bits + (1 << 16)).view(np.float32)
        c = 0
        if not neg:
            base = int(np.searchsorted(thr, lo, side="left"))        # thresholds < lo
            if base < 255 and thr[base] < hi:
                c = 0xFFFF - (_bits(thr[base]) & 0xFFFF)
        else:
            base = int(np.searchsorted(thr, -hi, side="right"))      # thresholds <= -hi
            if base < 255 and thr[base] < -lo:
                c = _bits(-thr[base]) & 0xFFFF
        tab.append((base << 16) | c)
    return tab


def _inside_counts(qmap):
    thr = _thresholds(qmap)
    counts = []
    for i in range(128, (ROWS - 1) * 128):
        r, k = divmod(i, 128)
        lo_bits = ((r - 1 + 127 - 23) << 23) | (k << 16)
        lo = np.uint32(lo_bits).view(np.float32)
        hi = np.uint32(lo_bits + (1 << 16)).view(np.float32)
        counts.append(int(((thr >= lo) & (thr < hi)).sum()))
        counts.append(int(((thr > -hi) & (thr < -lo)).sum()))
    return counts


def _slice(b, signed):
    """The kernel's slice number of x's bits b: the exponent and the top 7
    fraction bits, clamped to the table; the unsigned map keeps the sign bit
    in, so any x with it set lands in the last (NaN) slice."""
    top = (b >> 16) & 0x7FFF if signed else b >> 16
    return min(max(top - (127 - 24) * 128, 0), ROWS * 128 - 1)


def _code(tabs, x, signed):
    out = []
    for v in np.asarray(x, np.float32):
        b = _bits(v)
        i = _slice(b, signed)
        neg = signed and (b >> 31) == 1
        q = tabs[1 if neg else 0][i]
        key = (b & 0xFFFF) ^ (0xFFFF if neg else 0)
        out.append((q + key) >> 16)
    return np.array(out, np.uint8)


@pytest.mark.parametrize("signed", [True, False])
def test_every_slice_holds_at_most_one_threshold(oracle_mod, signed):
    qmap = oracle_mod.quant_map(signed)
    assert max(_inside_counts(qmap)) <= 1
    thr = _thresholds(qmap)
    assert np.abs(thr[thr != 0]).min() > 2.0 ** -23     # below 2^-23 the nearest value is 0


@pytest.mark.parametrize("signed", [True, False])
def test_slice_rule_gives_the_nearest_code(oracle_mod, signed):
    qmap = oracle_mod.quant_map(signed)
    tabs = (_table(qmap, False), _table(qmap, True))
    thr = _thresholds(qmap)
    g = np.random.Generator(np.random.Philox(71))
    lo = -1.0 if signed else 0.0
    xs = [g.uniform(lo, 1.0, 3000), np.sign(g.uniform(lo, 1.0, 3000)) * 10.0 ** g.uniform(-9, 0, 3000),
          qmap, thr, np.nextafter(thr, np.float32(2)), np.nextafter(thr, np.float32(-2)),
          np.array([0.0, -0.0, 1.0, 2.0 ** -23, np.nextafter(np.float32(2.0 ** -23), np.float32(0)), np.nan,
                    -np.nan])]
    if signed:
        xs += [-thr, -np.nextafter(thr, np.float32(2)), -qmap, np.array([-1.0, -(2.0 ** -23), -0.0])]
    x = np.concatenate([np.asarray(a, np.float64) for a in xs]).astype(np.float32)
    x = x[np.isnan(x) | ((x >= -1) & (x <= 1))]
    assert np.array_equal(_code(tabs, x, signed), oracle_mod.quantize(qmap, x))


def test_fast_quotient_is_within_three_ulp():
    """RN32(m * RN32(1/N)) against RN32(m / N), for |m| <= N over many
    magnitudes: at most 3 ulp of the exact quotient apart."""
    g = np.random.Generator(np.random.Philox(73))
    n = (10.0 ** g.uniform(-30, 30, 200_000)).astype(np.float32)
    m = (n * g.uniform(-1, 1, n.size).astype(np.float32)).astype(np.float32)
    exact = (m / n).astype(np.float32)
    fast = (m * (np.float32(1) / n)).astype(np.float32)
    ok = np.isfinite(fast) & (np.abs(exact) >= 2.0 ** -126)
    ulp = np.spacing(np.abs(exact[ok])).astype(np.float64)
    assert np.max(np.abs(fast[ok].astype(np.float64) - exact[ok].astype(np.float64)) / ulp) <= 3


def test_library_tables_are_the_rule(oracle_mod):
    """The tables the library uploads with every 8-bit plan (built on the
    host, opt2s_api8.cpp) equal the pinned oracle maps and the slice rule
    rebuilt here from them."""
    from elementwise_optimizer_b200 import _build
    from elementwise_optimizer_b200 import binding as B
    _build.build()
    smap, umap, spos, sneg, upos = B.testing_quant_tables()
    qs, qu = oracle_mod.quant_map(True), oracle_mod.quant_map(False)
    assert np.array_equal(smap.view(np.uint32), qs.view(np.uint32))
    assert np.array_equal(umap.view(np.uint32), qu.view(np.uint32))
    assert np.array_equal(spos, np.array(_table(qs, False), np.uint32))
    assert np.array_equal(sneg, np.array(_table(qs, True), np.uint32))
    assert np.array_equal(upos, np.array(_table(qu, False), np.uint32))


def _device_code(tabs, m, n, signed):
    """The kernel's decision, restated: the code of the fast quotient
    RN32(m * RN32(1/n)) unless its key lies within 4 of the slice's threshold
    (mod 2^16, so within 4 of either edge of a slice without one), else the
    code of the exact quotient."""
    fast = (m * (np.float32(1) / n)).astype(np.float32)
    exact = (m.astype(np.float64) / n.astype(np.float64)).astype(np.float32)
    out = []
    for f, e in zip(fast, exact):
        b = _bits(f)
        neg = signed and (b >> 31) == 1
        q = tabs[1 if neg else 0][_slice(b, signed)]
        key = (b & 0xFFFF) ^ (0xFFFF if neg else 0)
        s = q + key
        if ((s + 5) & 0xFFFF) <= 8:
            out.append(int(_code(tabs, np.array([e], np.float32), signed)[0]))
        else:
            out.append(s >> 16)
    return np.array(out, np.uint8), exact


@pytest.mark.parametrize("signed", [True, False])
def test_fast_quotient_with_decision_test_gives_the_exact_code(oracle_mod, signed):
    """Over random (m, absmax) pairs and pairs whose exact quotient lands on,
    next to, or within a few ulp of every threshold, the kernel's fast path
    with its decision test gives the nearest code of RN32(m / absmax)."""
    qmap = oracle_mod.quant_map(signed)
    tabs = (_table(qmap, False), _table(qmap, True))
    thr = _thresholds(qmap)
    g = np.random.Generator(np.random.Philox(79))
    n = (10.0 ** g.uniform(-20, 20, 20_000)).astype(np.float32)
    lo = -1.0 if signed else 0.0
    m = (n * g.uniform(lo, 1, n.size).astype(np.float32)).astype(np.float32)
    # quotients at the thresholds: m = RN32(T * n) for every threshold T (and its negative),
    # then nudged by up to 3 ulp of m
    t_all = np.concatenate([thr, -thr]) if signed else thr
    nt = (10.0 ** g.uniform(-20, 20, t_all.size)).astype(np.float32)
    mt = (t_all.astype(np.float64) * nt.astype(np.float64)).astype(np.float32)
    steps = g.integers(-3, 4, mt.size)
    mt = np.array([np.float32(x).view(np.int32) + int(k) for x, k in zip(mt, steps)], np.int32).view(np.float32)
    m = np.concatenate([m, mt])
    n = np.concatenate([n, nt])
    keep = np.isfinite(m) & (np.abs(m) <= n)
    m, n = m[keep], n[keep]
    codes, exact = _device_code(tabs, m, n, signed)
    assert np.array_equal(codes, oracle_mod.quantize(qmap, exact))


@pytest.mark.parametrize("signed", [True, False])
def test_no_threshold_sits_near_an_edge_shared_with_another_threshold(oracle_mod, signed):
    """The kernel needs no separate slice-boundary test because of two
    properties of the maps: a threshold within 8 ulp of an edge of its slice
    never faces a slice that holds a threshold across that edge (so a fast
    quotient that crosses an edge from a slice holding a threshold crosses no
    threshold), and every threshold lies more than 8 ulp above 2^-23, the edge
    of the row of values whose code is that of 0."""
    thr = _thresholds(oracle_mod.quant_map(signed))
    for side in ((1, -1) if signed else (1,)):
        mags = np.abs(thr[thr * side > 0]).astype(np.float32)
        bits = mags.view(np.uint32).astype(np.int64)
        slices = [_slice(int(b), True) for b in bits]
        holders = set(slices)
        for b, sl in zip(bits, slices):
            low = int(b) & 0xFFFF
            assert not (low <= 8 and sl - 1 in holders), (side, sl, low)
            assert not (0x10000 - low <= 8 and sl + 1 in holders), (side, sl, low)
        assert bits.min() > np.float32(2.0 ** -23).view(np.uint32) + 8


def _codes_vec(tabs, bits, signed):
    """The slice rule over an array of bit patterns (uint32), vectorised."""
    bits = bits.astype(np.int64)
    top = ((bits >> 16) & 0x7FFF) if signed else (bits >> 16)
    idx = np.clip(top - (127 - 24) * 128, 0, ROWS * 128 - 1)
    neg = ((bits >> 31) == 1) & signed
    pos_t, neg_t = (np.array(t, np.int64) for t in tabs)
    q = np.where(neg, neg_t[idx], pos_t[idx])
    key = (bits & 0xFFFF) ^ np.where(neg, 0xFFFF, 0)
    return q + key, key


@pytest.mark.parametrize("signed", [True, False])
def test_decision_test_around_every_edge_and_threshold(oracle_mod, signed):
    """Every fast quotient within 3 ulp of an exact one, the exact one within
    4 ulp of any slice edge or threshold of the map (both signs for the signed
    map): the kernel's decision -- the fast quotient's code unless
    (entry + key + 5) mod 2^16 <= 8, else the exact quotient's code -- gives
    the exact quotient's nearest code."""
    qmap = oracle_mod.quant_map(signed)
    tabs = (_table(qmap, False), _table(qmap, True))
    thr = _thresholds(qmap)
    edges = np.arange((127 - 23) << 7, (127 << 7) + 1, dtype=np.int64) << 16     # every slice start, 2^-23 .. 1
    anchors = np.concatenate([edges, np.abs(thr[thr != 0]).astype(np.float32).view(np.uint32).astype(np.int64)])
    exact = (anchors[:, None] + np.arange(-4, 5)[None, :]).reshape(-1)
    exact = exact[(exact > 0) & (exact <= np.float32(1.0).view(np.uint32))]
    signs = (0, 1 << 31) if signed else (0,)
    for sgn in signs:
        e_bits = (exact | sgn).astype(np.uint32)
        want = oracle_mod.quantize(qmap, e_bits.view(np.float32))
        for d in range(-3, 4):
            f_mag = np.clip(exact + d, 0, np.float32(1.0).view(np.uint32) + 3)
            f_bits = (f_mag | sgn).astype(np.uint32)
            s_f, _ = _codes_vec(tabs, f_bits, signed)
            s_e, _ = _codes_vec(tabs, e_bits, signed)
            redo = ((s_f + 5) & 0xFFFF) <= 8
            got = np.where(redo, s_e >> 16, s_f >> 16).astype(np.uint8)
            bad = np.nonzero(got != want)[0]
            assert bad.size == 0, (sgn, d, e_bits[bad[:5]], f_bits[bad[:5]], got[bad[:5]], want[bad[:5]])
