"""Property tests of the host logic of the C ABI, against brute force (no GPU).

Hypothesis draws collections whose fake buffers are packed into a small
address window, so that overlaps are frequent, and checks each host routine
against a plain restatement of its rule:

  * the overlap check: a call is rejected with OPT2S_ERR_ALIAS exactly when
    some buffer that the step writes (param, state1, state2) shares a byte
    with any other buffer of the call (two gradients may share memory,
    since neither is written);
  * the chunk-table builder: every element of every tensor in exactly one
    chunk, chunks in descriptor order, none longer than the chunk length;
  * the chunk-length chooser: the power of two c in [128, 2048] that
    minimises (waves of chunks over the resident warps) x (c / 32 + 8), the
    longest on ties, where a plan with 16-bit tensors takes 128 only when it
    fits in one wave;
  * the shard partition: consecutive, 8-element aligned, covering the buffer;
  * the bounded-update-norm tables: 2,048-element norm blocks per tensor,
    groups of at most 64 consecutive blocks of one tensor covering each
    tensor's blocks in order, and each chunk's tensor.

Pointers are fake addresses: nothing is dereferenced.
"""
import ctypes

import pytest
from hypothesis import HealthCheck, given, settings, strategies as st

from elementwise_optimizer_b200 import binding as B

SETTINGS = settings(max_examples=300, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow])
DT = {"f32": 4, "f16": 2, "bf16": 2}
BASE = 1 << 32


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from elementwise_optimizer_b200 import _build
    _build.build()
    B.lib()


@st.composite
def crowded_collections(draw):
    """Records whose four buffers start at 4-byte aligned offsets in a
    window a few times larger than the data, so that they often overlap."""
    algo = draw(st.sampled_from(["adam", "ademamix"]))
    count = draw(st.integers(1, 6))
    recs = []
    for _ in range(count):
        n = draw(st.integers(0, 64))
        dt = draw(st.sampled_from(sorted(DT)))
        window = 4 * 64 * 4 * count
        addr = [BASE + 4 * draw(st.integers(0, window // 4)) for _ in range(4)]
        recs.append((addr[0], addr[1], addr[2], addr[3], n, B.DTYPES[dt]))
    return algo, recs


def byte_ranges(rec, algo):
    p, g, s1, s2, n, dt = rec
    es = 4 if dt == B.DTYPES["f32"] else 2
    s1n = 2 * n if algo == "ademamix" else n
    return [(p, p + n * es, True), (g, g + n * es, False),
            (s1, s1 + 4 * s1n, True), (s2, s2 + 4 * n, True)]


def aliases_by_brute_force(recs, algo):
    rs = [r for rec in recs if rec[4] > 0 for r in byte_ranges(rec, algo)]
    for i in range(len(rs)):
        for j in range(i + 1, len(rs)):
            a, b = rs[i], rs[j]
            if (a[2] or b[2]) and a[0] < b[1] and b[0] < a[1]:
                return True
    return False


def hyper(algo):
    return (B.make_hyper("ademamix", beta3=0.999, alpha=5.0) if algo == "ademamix"
            else B.make_hyper("adam"))


@SETTINGS
@given(crowded_collections())
def test_overlap_check_equals_brute_force(case):
    algo, recs = case
    status = B.testing_validate(B.TensorList(recs), hyper(algo), 1)
    expect = -2 if aliases_by_brute_force(recs, algo) else 0
    assert status == expect


@SETTINGS
@given(crowded_collections())
def test_no_alloc_entry_point_applies_the_same_overlap_rule(case):
    """opt2s_step_noalloc has its own allocation-free validation; it must
    reject exactly the same collections.  Only rejected collections are
    passed to it (they return before any CUDA call), so fake pointers never
    reach a kernel."""
    algo, recs = case
    if not aliases_by_brute_force(recs, algo):
        return
    tl = B.TensorList(recs)
    h = hyper(algo)
    assert B.lib().opt2s_step_noalloc(ctypes.byref(tl.desc), ctypes.byref(h), 1, None) == -2


@st.composite
def collections(draw):
    sizes = draw(st.lists(st.one_of(st.integers(0, 40), st.integers(0, 20_000),
                                    st.sampled_from([255, 256, 257, 2047, 2048, 2049, 1 << 20])),
                          min_size=0, max_size=30))
    dts = draw(st.lists(st.sampled_from(sorted(DT)), min_size=len(sizes), max_size=len(sizes)))
    recs, addr = [], BASE
    for n, dt in zip(sizes, dts):
        rec = []
        for nbytes in (n * DT[dt], n * DT[dt], 4 * n, 4 * n):
            rec.append(addr)
            addr += (nbytes + 255) // 256 * 256 + 256
        recs.append((*rec, n, B.DTYPES[dt]))
    return sizes, dts, recs


@SETTINGS
@given(collections(), st.sampled_from([0, 1, 8, 64, 256, 1000, 2048, 8192]))
def test_chunk_table_covers_each_element_once(coll, chunk):
    sizes, dts, recs = coll
    chunks = B.testing_build_chunks(B.TensorList(recs), "adam", chunk)
    ce = chunk or B.lib().opt2s_testing_default_chunk_elems()
    pos = {}
    last_t = -1
    for t, s, n, dt in chunks:
        assert t >= last_t                   # descriptor order
        last_t = t
        assert 1 <= n <= ce and dt == B.DTYPES[dts[t]]
        assert s == pos.get(t, 0)            # contiguous, no gap, no overlap
        pos[t] = s + n
    for i, n in enumerate(sizes):
        assert pos.get(i, 0) == n


def chosen_by_brute_force(sizes, dts, warps):
    all_f32 = not any(n > 0 and dt != "f32" for n, dt in zip(sizes, dts))
    best, best_cost = None, None
    for c in (2048, 1024, 512, 256, 128):
        chunks = sum(-(-n // c) for n in sizes)
        waves = -(-chunks // warps)
        if c == 128 and not all_f32 and waves > 1:
            continue
        cost = waves * (c // 32 + 8)
        if best_cost is None or cost < best_cost:
            best, best_cost = c, cost
    return best


@SETTINGS
@given(collections(), st.integers(1, 148 * 64))
def test_chunk_length_minimises_the_wave_model(coll, warps):
    sizes, dts, recs = coll
    got = B.testing_choose_chunk_elems(B.TensorList(recs), warps)
    assert got == chosen_by_brute_force(sizes, dts, warps)


@SETTINGS
@given(st.integers(0, 1 << 40), st.integers(1, 8))
def test_shard_partition(numel, world):
    pos = 0
    for r in range(world):
        start, n = B.opt2s_shard_range(numel, world, r)
        assert start == pos and n >= 0
        assert start % 8 == 0 or n == 0
        pos += n
    assert pos == numel


@SETTINGS
@given(collections(), st.sampled_from([0, 128, 256, 1000, 2048, 8192]))
def test_norm_tables_group_each_tensors_blocks_in_order(coll, chunk):
    sizes, dts, recs = coll
    tl = B.TensorList(recs)
    t = B.testing_unorm_tables(tl, "adam", chunk)
    nb = [-(-n // 2048) for n in sizes]
    assert t["nblocks"] == sum(nb)
    ranges = list(zip(t["ranges"][0::2], t["ranges"][1::2]))
    first = t["first_group"]
    assert len(first) == len(sizes) + 1 and first[0] == 0 and first[-1] == len(ranges)
    block0 = 0
    for i, n in enumerate(nb):
        mine = ranges[first[i]:first[i + 1]]
        pos = block0
        for lo, hi in mine:                    # contiguous, in order, 1..64 blocks each
            assert lo == pos and 1 <= hi - lo <= 64
            pos = hi
        assert pos == block0 + n
        block0 += n
    chunks = B.testing_build_chunks(tl, "adam", chunk)
    assert t["chunk_tensor"] == [c[0] for c in chunks]
