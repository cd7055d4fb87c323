"""Host-side tests of the C ABI (no GPU needed).

They check that libopt2s.so loads, that it exports exactly the entry points
include/*.h declares, that the ctypes mirrors have the C layout, and the
host logic every call runs before touching CUDA: argument validation (every
record checked before any launch, so an argument error never leaves a partial
update) and the chunk-table builder (every element covered exactly once).
Pointers here are fake addresses: nothing is dereferenced on the host.
"""
import ctypes
import os
import re
import subprocess
import sys
import tempfile

import pytest

from elementwise_optimizer_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INCLUDE = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def L():
    from elementwise_optimizer_b200 import _build
    _build.build()
    return B.lib()


def declared_functions():
    names = set()
    for h in ("opt2s.h", "opt2s_testing.h"):
        src = open(os.path.join(INCLUDE, h)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"^[A-Za-z_][\w \t\*]*?\b(opt2s_\w+)\s*\(", src, flags=re.M))
    return names


def _exported(path):
    out = subprocess.run(["nm", "-D", "--defined-only", path], check=True,
                         capture_output=True, text=True).stdout
    return {l.split()[-1] for l in out.splitlines() if " T " in l and "opt2s_" in l}


def test_exports_match_headers(L):
    """The test build exports every function the headers declare; the
    product exports all of them but the forcing knobs, the fault injection
    and the division check, which exist only in the test build."""
    decl = declared_functions()
    assert "opt2s_step" in decl and "opt2s_plan_create" in decl
    assert B.TESTING_ONLY <= decl
    assert _exported(B.TESTING_LIB_PATH) == decl, (_exported(B.TESTING_LIB_PATH) ^ decl)
    product = _exported(B.LIB_PATH)
    assert product == decl - B.TESTING_ONLY, (product ^ (decl - B.TESTING_ONLY))
    for name in decl - B.TESTING_ONLY:
        assert getattr(L, name) is not None
    assert set(B.EXPORTS) == decl
    with pytest.raises(RuntimeError):         # knobs need the test build
        B.testing_set_launch(0, 0)


def test_struct_layout_matches_c(L):
    prog = r"""
    #include <stddef.h>
    #include <stdio.h>
    #include "opt2s_testing.h"
    int main(void) {
      printf("%zu %zu %zu %zu %zu %zu\n", sizeof(opt2s_tensor), offsetof(opt2s_tensor, numel),
             offsetof(opt2s_tensor, dtype), sizeof(TensorListDesc), sizeof(Hyper),
             offsetof(Hyper, skip_zeros));
      printf("%zu %zu\n", sizeof(opt2s_testing_chunk), offsetof(opt2s_testing_chunk, dtype));
      printf("%zu %zu %zu %zu %zu\n", sizeof(opt2s_step_scalars), offsetof(opt2s_step_scalars, decay),
             offsetof(opt2s_step_scalars, inv_bc2), offsetof(opt2s_step_scalars, rcp_bc1_hi),
             offsetof(opt2s_step_scalars, rcp_bc2_lo));
      return 0;
    }"""
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "p.c")
        open(c, "w").write(prog)
        exe = os.path.join(d, "p")
        cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
        subprocess.run(["gcc", "-std=c11", "-I", INCLUDE, "-I", cuda_inc, "-o", exe, c], check=True)
        lines = subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split("\n")
    a = list(map(int, lines[0].split()))
    assert a == [ctypes.sizeof(B.opt2s_tensor), B.opt2s_tensor.numel.offset,
                 B.opt2s_tensor.dtype.offset, ctypes.sizeof(B.TensorListDesc),
                 ctypes.sizeof(B.Hyper), B.Hyper.skip_zeros.offset]
    b = list(map(int, lines[1].split()))
    assert b == [ctypes.sizeof(B.opt2s_testing_chunk), B.opt2s_testing_chunk.dtype.offset]
    c = list(map(int, lines[2].split()))
    assert c == [ctypes.sizeof(B.opt2s_step_scalars), B.opt2s_step_scalars.decay.offset,
                 B.opt2s_step_scalars.inv_bc2.offset, B.opt2s_step_scalars.rcp_bc1_hi.offset,
                 B.opt2s_step_scalars.rcp_bc2_lo.offset]


def test_abi_version(L):
    assert L.opt2s_abi_version() == 2


def test_error_strings(L):
    for code in B.STATUS:
        s = L.opt2s_error_string(code).decode()
        assert s and s != "unknown status"
    assert L.opt2s_error_string(12345).decode() == "unknown status"


# --------------------------------------------------------------------------
# Fake device buffers: disjoint address ranges, 256-byte aligned
# --------------------------------------------------------------------------

class Arena:
    def __init__(self, base=1 << 40):
        self.next = base

    def alloc(self, nbytes, align=256, offset=0):
        a = (self.next + align - 1) // align * align + offset
        self.next = a + nbytes + 4096
        return a


def records(sizes, dtypes=None, algo="adam", arena=None):
    arena = arena or Arena()
    dtypes = dtypes or ["f32"] * len(sizes)
    recs = []
    for n, dt in zip(sizes, dtypes):
        es = 4 if dt == "f32" else 2
        s1n = 2 * n if algo == "ademamix" else n
        recs.append((arena.alloc(n * es), arena.alloc(n * es), arena.alloc(4 * s1n),
                     arena.alloc(4 * n), n, B.DTYPES[dt]))
    return recs


H = B.make_hyper("adam")


def validate(recs, hyper=H, step=1):
    return B.testing_validate(B.TensorList(recs), hyper, step)


def test_valid_collection_passes(L):
    assert validate(records([1, 7, 4096, 100000], ["f32", "f16", "bf16", "f32"])) == 0
    assert validate([]) == 0


@pytest.mark.parametrize("field,value", [
    ("algo", 2), ("algo", -1), ("skip_zeros", 2), ("lr", float("nan")),
    ("lr", float("inf")), ("beta1", 1.0), ("beta1", -0.1), ("beta2", 1.5),
    ("eps", -1e-8), ("eps", float("inf")), ("weight_decay", float("nan"))])
def test_bad_hyper_rejected(L, field, value):
    h = B.make_hyper("adam")
    setattr(h, field, value)
    assert validate(records([16]), h) == -1


def test_ademamix_hyper_checked_only_for_ademamix(L):
    h = B.make_hyper("adam", beta3=2.0, alpha=float("nan"))
    assert validate(records([16]), h) == 0
    h = B.make_hyper("ademamix", beta3=1.0, alpha=5.0)
    assert validate(records([16], algo="ademamix"), h) == -1
    h = B.make_hyper("ademamix", beta3=0.999, alpha=float("inf"))
    assert validate(records([16], algo="ademamix"), h) == -1


@pytest.mark.parametrize("step", [0, -1, -(2 ** 31)])
def test_step_below_one_rejected(L, step):
    assert validate(records([16]), step=step) == -1


def test_bad_records_rejected(L):
    good = records([64])
    p, g, s1, s2, n, dt = good[0]
    assert validate([(p, g, s1, s2, -1, dt)]) == -1            # negative numel
    assert validate([(p, g, s1, s2, n, 7)]) == -1              # bad dtype
    assert validate([(0, g, s1, s2, n, dt)]) == -1             # null param
    assert validate([(p, 0, s1, s2, n, dt)]) == -1             # null grad
    assert validate([(p, g, 0, s2, n, dt)]) == -1              # null state1
    assert validate([(p, g, s1, 0, n, dt)]) == -1              # null state2
    assert validate([(p + 2, g, s1, s2, n, dt)]) == -1         # fp32 param not 4-aligned
    assert validate([(p, g, s1 + 1, s2, n, dt)]) == -1         # state not 4-aligned
    assert validate([(0, 0, 0, 0, 0, dt)]) == 0                # empty record: skipped
    tl = B.TensorList(good)
    tl._arr[0].reserved = 1
    assert B.testing_validate(tl, H, 1) == -1
    null_desc = B.TensorListDesc(None, 3)
    assert B.lib().opt2s_testing_validate(ctypes.byref(null_desc), ctypes.byref(H), 1) == -1
    neg = B.TensorListDesc(None, -1)
    assert B.lib().opt2s_testing_validate(ctypes.byref(neg), ctypes.byref(H), 1) == -1


def test_half_storage_needs_only_2_byte_alignment(L):
    p, g, s1, s2, n, _ = records([64], ["f16"])[0]
    assert validate([(p + 2, g + 6, s1 + 4, s2 + 12, n, B.DTYPES["f16"])]) == 0
    assert validate([(p + 1, g, s1, s2, n, B.DTYPES["f16"])]) == -1


def test_aliasing_rejected(L):
    p, g, s1, s2, n, dt = records([1024])[0]
    assert validate([(p, p, s1, s2, n, dt)]) == -2                     # grad is param
    assert validate([(p, g, s1, s1, n, dt)]) == -2                     # m is v
    assert validate([(p, g, s1, s1 + 4 * 1023, n, dt)]) == -2          # partial overlap
    assert validate([(p, g, p + 4 * 512, s2, n, dt)]) == -2            # state inside param
    a, b = records([100, 100])
    assert validate([a, (b[0], b[1], a[2], b[3], 100, dt)]) == -2      # states shared across tensors
    # two tensors reading the same gradient is fine (it is never written)
    assert validate([a, (b[0], a[1], b[2], b[3], 100, dt)]) == 0


def test_ademamix_state1_is_twice_numel(L):
    arena = Arena()
    n = 256
    p, g = arena.alloc(4 * n), arena.alloc(4 * n)
    s1 = arena.alloc(4 * n, align=4096)      # room for n floats only ...
    s2 = s1 + 4 * n                          # ... v starts right after m
    adam_ok = validate([(p, g, s1, s2, n, 0)], B.make_hyper("adam"))
    ademamix = validate([(p, g, s1, s2, n, 0)], B.make_hyper("ademamix", beta3=0.999, alpha=5))
    assert adam_ok == 0 and ademamix == -2   # m2 = state1[n:2n] would overlap v


# --------------------------------------------------------------------------
# Chunk-table builder
# --------------------------------------------------------------------------

@pytest.mark.parametrize("chunk", [0, 8, 64, 4096, 8192])
def test_chunks_cover_every_element_once(L, chunk):
    sizes = [1, 2, 31, 32, 33, 255, 256, 257, 1023, 1024, 1025, 4095, 4096, 4097,
             8191, 8192, 8193, 0, 100003]
    dts = [("f32", "f16", "bf16")[i % 3] for i in range(len(sizes))]
    tl = B.TensorList(records(sizes, dts))
    chunks = B.testing_build_chunks(tl, "adam", chunk)
    ce = chunk or B.lib().opt2s_testing_default_chunk_elems()
    cover = {i: [] for i in range(len(sizes))}
    for t, s, n, dt in chunks:
        assert 1 <= n <= ce and s % ce == 0
        assert dt == B.DTYPES[dts[t]]
        cover[t].append((s, n))
    for i, n in enumerate(sizes):
        segs = cover[i]
        assert sum(x[1] for x in segs) == n
        pos = 0
        for s, k in segs:                     # contiguous, in order, no overlap
            assert s == pos
            pos += k
    # launch order follows descriptor order
    assert [c[0] for c in chunks] == sorted(c[0] for c in chunks)


def test_chunk_count_for_large_tensor(L):
    tl = B.TensorList(records([268_435_456]))
    ce = B.lib().opt2s_testing_default_chunk_elems()
    assert len(B.testing_build_chunks(tl, "adam")) == 268_435_456 // ce


def test_build_chunks_validates_first(L):
    p, g, s1, s2, n, dt = records([64])[0]
    with pytest.raises(B.Opt2sError) as e:
        B.testing_build_chunks(B.TensorList([(p, p, s1, s2, n, dt)]), "adam")
    assert e.value.status == -2


@pytest.mark.usefixtures("testing_lib")
def test_testing_knobs_validate(L):
    with pytest.raises(B.Opt2sError):
        B.testing_set_launch(33, 0)
    with pytest.raises(B.Opt2sError):
        B.testing_set_launch(2048, 0)
    B.testing_set_launch(0, 0)
    prev = B.testing_set_chunk_elems(0)
    assert B.testing_set_chunk_elems(prev) == 0


# --------------------------------------------------------------------------
# The step entry point without a GPU: argument errors come first, no crash
# --------------------------------------------------------------------------

def _cuda_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.mark.skipif(_cuda_available(), reason="checks the no-device path")
def test_step_without_device(L):
    tl = B.TensorList(records([64]))
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step(tl, H, 1, stream=0)
    assert e.value.status == -4                       # CUDA: no device
    p, g, s1, s2, n, dt = records([64])[0]
    with pytest.raises(B.Opt2sError) as e:            # argument errors still first
        B.opt2s_step(B.TensorList([(p, p, s1, s2, n, dt)]), H, 1, stream=0)
    assert e.value.status == -2
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step(tl, H, 0, stream=0)
    assert e.value.status == -1
    B.opt2s_step(B.TensorList([]), H, 1, stream=0)    # empty collection: no-op
    B.opt2s_step(B.TensorList([(0, 0, 0, 0, 0, 0)]), H, 1, stream=0)


def test_max_unorm_argument_checks(L):
    """The bound must be finite and positive; this is checked before any
    CUDA call, so it holds with or without a device."""
    tl = B.TensorList(records([64]))
    for mu in (0.0, -1.0, float("nan"), float("inf"), float("-inf")):
        with pytest.raises(B.Opt2sError) as e:
            B.opt2s_step_max_unorm(tl, H, mu, 1, stream=0)
        assert e.value.status == -1, mu
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step_max_unorm(tl, H, 1.0, 0, stream=0)
    assert e.value.status == -1
    B.opt2s_step_max_unorm(B.TensorList([]), H, 1.0, 1, stream=0)   # empty: no-op


@pytest.mark.skipif(_cuda_available(), reason="checks the no-device path")
def test_max_unorm_step_without_device(L):
    tl = B.TensorList(records([64, 3000], ["f32", "bf16"]))
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step_max_unorm(tl, H, 1.0, 1, stream=0)
    assert e.value.status == -4                       # CUDA: no device
    p, g, s1, s2, n, dt = records([64])[0]
    with pytest.raises(B.Opt2sError) as e:            # argument errors still first
        B.opt2s_step_max_unorm(B.TensorList([(p, g, s1, s1, n, dt)]), H, 1.0, 1, stream=0)
    assert e.value.status == -2


def test_lamb_argument_checks(L):
    """LAMB takes Adam moments: AdEMAMix is rejected, as are a bad step and
    bad hyper-parameters, before any CUDA call."""
    tl = B.TensorList(records([64]))
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step_lamb(tl, B.make_hyper("ademamix", beta3=0.9, alpha=1.0), 1, stream=0)
    assert e.value.status == -1
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step_lamb(tl, H, 0, stream=0)
    assert e.value.status == -1
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step_lamb(tl, B.make_hyper("adam", eps=-1.0), 1, stream=0)
    assert e.value.status == -1
    B.opt2s_step_lamb(B.TensorList([]), H, 1, stream=0)   # empty: no-op


@pytest.mark.skipif(_cuda_available(), reason="checks the no-device path")
def test_lamb_step_without_device(L):
    tl = B.TensorList(records([64, 3000], ["f32", "bf16"]))
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step_lamb(tl, H, 1, stream=0)
    assert e.value.status == -4                       # CUDA: no device
    p, g, s1, s2, n, dt = records([64])[0]
    with pytest.raises(B.Opt2sError) as e:            # argument errors still first
        B.opt2s_step_lamb(B.TensorList([(p, g, s1, s1, n, dt)]), H, 1, stream=0)
    assert e.value.status == -2


def _rec8(arena, n, dt="f32", bits=8, algo="adam"):
    es = 4 if dt == "f32" else 2
    two = 2 if algo == "ademamix" else 1
    sb = 1 if bits == 8 else 4
    nb = (n + 2047) // 2048
    a1 = arena.alloc(4 * two * nb) if bits == 8 else 0
    a2 = arena.alloc(4 * nb) if bits == 8 else 0
    return (arena.alloc(n * es), arena.alloc(n * es), arena.alloc(two * n * sb), arena.alloc(n * sb),
            a1, a2, n, B.DTYPES[dt], bits)


def test_8bit_routing_and_argument_checks(L):
    """Routing by min_8bit_size, and every record checked before any CUDA
    call: state_bits in {8, 32}, absmax pointers exactly for 8-bit records,
    and no overlap of written codes or absmaxes with another buffer."""
    assert B.state_bits_for(4095) == 32 and B.state_bits_for(4096) == 8
    assert B.state_bits_for(10, 8) == 8 and B.state_bits_for(7, 8) == 32
    assert B.state_bits_for(4096, 0) == 8            # <= 0: the default threshold
    ar = Arena()
    good = _rec8(ar, 5000)
    small = _rec8(ar, 100, bits=32)
    cases = []
    p, g, s1, s2, a1, a2, n, dt, bits = good
    cases.append(((p, g, s1, s2, 0, a2, n, dt, 8), -1))        # missing absmax1
    cases.append(((p, g, s1, s2, a1, a2, n, dt, 16), -1))      # bad state_bits
    cases.append(((p, g, s1, s1, a1, a2, n, dt, 8), -2))       # codes of m and v overlap
    cases.append(((p, g, s1, s2, a1, a1, n, dt, 8), -2))       # absmaxes overlap
    cases.append(((p, g, s1, s2, a1, a2, n, 7, 8), -1))        # bad dtype
    sp, sg, ss1, ss2, _, _, sn, sdt, _ = small
    cases.append(((sp, sg, ss1, ss2, a1, 0, sn, sdt, 32), -1))  # absmax on a 32-bit record
    cases.append(((sp, sg, ss1 + 2, ss2, 0, 0, sn, sdt, 32), -1))  # misaligned fp32 state
    for rec, want in cases:
        with pytest.raises(B.Opt2sError) as e:
            B.opt2s_step_8bit(B.TensorList8([good if rec[0] != p else small, rec]), H, 1, stream=0)
        assert e.value.status == want, rec
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step_8bit(B.TensorList8([good]), H, 0, stream=0)
    assert e.value.status == -1
    B.opt2s_step_8bit(B.TensorList8([]), H, 1, stream=0)                         # empty: no-op
    # AdEMAMix state1 holds [m1 | m2] codes (2n bytes) and 2 x blocks absmaxes
    ar2 = Arena()
    rec = _rec8(ar2, 4096, algo="ademamix")
    q = list(rec)
    q[3] = q[2] + 4096                  # v codes inside m2's half of state1
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step_8bit(B.TensorList8([tuple(q)]), B.make_hyper("ademamix", beta3=0.9, alpha=1.0),
                          1, stream=0)
    assert e.value.status == -2


@pytest.mark.skipif(_cuda_available(), reason="checks the no-device path")
def test_8bit_step_without_device(L):
    ar = Arena()
    tl = B.TensorList8([_rec8(ar, 5000), _rec8(ar, 100, bits=32)])
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step_8bit(tl, H, 1, stream=0)
    assert e.value.status == -4                       # CUDA: no device


def test_missing_library_fails_loudly(tmp_path):
    code = ("import elementwise_optimizer_b200.binding as b; b.LIB_PATH='/nonexistent/x.so'\n"
            "try:\n  b.lib()\nexcept RuntimeError as e:\n  print('RAISED', e)\n")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True,
                         text=True, check=True).stdout
    assert out.startswith("RAISED") and "no CPU fallback" in out


# --------------------------------------------------------------------------
# Per-step scalar tables (host only)
# --------------------------------------------------------------------------

def test_step_scalar_table_matches_the_definitions(L, oracle_mod):
    """The table a captured graph reads holds the same per-step scalars the
    oracle computes: bc = 1 - beta^t and decay = 1 - lr*wd in double rounded
    once, 1 - beta in fp32, and the binary64 reciprocals of bc1, bc2."""
    import numpy as np
    h = B.make_hyper("ademamix", lr=3e-3, beta1=0.9, beta2=0.999, eps=1e-8,
                     weight_decay=0.1, beta3=0.9999, alpha=5.0)
    raw = B.fill_step_scalars(h, 7, 20)
    arr = (B.opt2s_step_scalars * 20).from_buffer_copy(raw)
    f32 = np.float32
    for k, s in enumerate(arr):
        t = 7 + k
        assert s.bc1 == oracle_mod.bias_correction(0.9, t)
        assert s.bc2 == oracle_mod.bias_correction(0.999, t)
        assert s.decay == oracle_mod.decay_factor(3e-3, 0.1)
        assert s.one_minus_beta1 == f32(1) - f32(0.9)
        assert s.one_minus_beta3 == f32(1) - f32(0.9999)
        assert s.inv_bc1 == 1.0 / float(f32(s.bc1)) and s.inv_bc2 == 1.0 / float(f32(s.bc2))
        for inv, hi, lo in ((s.inv_bc1, s.rcp_bc1_hi, s.rcp_bc1_lo), (s.inv_bc2, s.rcp_bc2_hi, s.rcp_bc2_lo)):
            assert hi == float(f32(inv)) and lo == float(f32(inv - hi))
            # the pair carries the reciprocal to about 2^-48 relative
            assert abs(hi + lo - inv) <= 2.0 ** -47 * inv
        assert (s.lr, s.alpha) == (f32(3e-3), f32(5.0))


def test_step_scalar_table_rejects_bad_arguments(L):
    h = B.make_hyper("adam")
    out = (B.opt2s_step_scalars * 2)()
    p = ctypes.cast(out, ctypes.c_void_p)
    assert L.opt2s_fill_step_scalars(ctypes.byref(h), 0, 2, p) == -1        # step 0
    assert L.opt2s_fill_step_scalars(ctypes.byref(h), 1, -1, p) == -1       # negative count
    assert L.opt2s_fill_step_scalars(ctypes.byref(h), 2 ** 31 - 1, 2, p) == -1   # step overflow
    assert L.opt2s_fill_step_scalars(ctypes.byref(h), 1, 2, None) == -1
    h.beta1 = 1.0
    assert L.opt2s_fill_step_scalars(ctypes.byref(h), 1, 2, p) == -1
    assert L.opt2s_plan_step_table(None, 0, None, 1, None, None) == -1


def test_chunk_length_follows_collection_size(L):
    """Large collections get the longest chunk (2,048); a 2,000-tensor
    collection of 64..1,024 elements gets 256-element chunks so that every
    resident warp has work and no warp walks a whole tensor alone; a small
    tensor gets 128-element chunks (4 elements per lane).  A plan with 16-bit
    tensors takes 128 only when it fits in one wave of warps (the short-chunk
    path pays only there); an all-fp32 one whenever the model says so."""
    from elementwise_optimizer_b200 import synth
    W = 148 * 20
    big = B.TensorList(records([268_435_456]))
    assert B.testing_choose_chunk_elems(big, W) == 2048
    w = synth.small_collection()
    small = B.TensorList(records(w.sizes, w.dtypes))
    assert B.testing_choose_chunk_elems(small, W) == 256
    assert B.testing_choose_chunk_elems(B.TensorList(records([1024])), W) == 128
    assert B.testing_choose_chunk_elems(B.TensorList(records([1024], ["bf16"])), W) == 128
    assert B.testing_choose_chunk_elems(B.TensorList(records([1024, 64], ["f32", "f16"])), W) == 128
    # ten 100-element tensors over 4 warps: three waves whatever the length
    assert B.testing_choose_chunk_elems(B.TensorList(records([100] * 10)), 4) == 128
    assert B.testing_choose_chunk_elems(B.TensorList(records([100] * 10, ["f16"] * 10)), 4) == 256
    for tl in (big, small):
        c = B.testing_choose_chunk_elems(tl, W)
        assert c in (128, 256, 512, 1024, 2048)
    assert B.testing_choose_chunk_elems(B.TensorList([]), W) == 2048


# --------------------------------------------------------------------------
# Sharded step: partition and validation (host only)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("numel", [0, 1, 7, 8, 9, 1000, 1000003, 268_435_456])
@pytest.mark.parametrize("world", [1, 2, 3, 5, 8])
def test_shard_ranges_partition_the_buffer(L, numel, world):
    ranges = [B.opt2s_shard_range(numel, world, r) for r in range(world)]
    pos = 0
    for start, n in ranges:
        assert start == pos and n >= 0 and start % 8 == 0 or n == 0
        pos = start + n
    assert pos == numel
    sizes = [n for _, n in ranges]
    assert max(sizes) - min(sizes) <= 8 + (numel % 8)


def test_shard_range_rejects_bad_arguments(L):
    for args in ((10, 0, 0), (10, 9, 0), (10, 2, 2), (10, 2, -1), (-1, 1, 0)):
        with pytest.raises(B.Opt2sError):
            B.opt2s_shard_range(*args)


def test_shard_step_validation(L):
    arena = Arena()
    n, world = 4096, 2
    params = [arena.alloc(4 * n) for _ in range(world)]
    grads = [arena.alloc(4 * n) for _ in range(world)]
    k = B.opt2s_shard_range(n, world, 0)[1]
    s1, s2 = arena.alloc(4 * k), arena.alloc(4 * k)
    h = B.make_hyper("adam")

    def run(**kw):
        d = B.make_shard_desc(world, 0, n, 0, params, grads, s1, s2)
        for key, val in kw.items():
            if key in ("params", "grads"):
                for q, x in enumerate(val):
                    getattr(d, key)[q] = x
            else:
                setattr(d, key, val)
        return L.opt2s_shard_step(ctypes.byref(d), ctypes.byref(h), 1, None)

    assert run(world=0) == -1 and run(world=9) == -1 and run(rank=2) == -1
    assert run(dtype=5) == -1 and run(reserved=1) == -1
    assert run(params=[params[0], 0]) == -1                        # missing peer buffer
    assert run(grads=[grads[0], params[1]]) == -2                  # a grad is a param buffer
    assert run(params=[params[0], params[0]]) == -2                # two ranks, one buffer
    assert run(state1=params[0] + 64) == -2                        # state inside a param buffer
    assert run(state2=0) == -1
    assert L.opt2s_shard_step(None, ctypes.byref(h), 1, None) == -1


def test_host_sources_compile_with_nvtx_ranges():
    """The optional NVTX ranges (-DOPT2S_NVTX) compile in every host source
    that marks a step entry point."""
    import shutil
    import subprocess
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("no g++")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    csrc = os.path.join(root, "elementwise_optimizer_b200", "csrc")
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    for src in ("opt2s_api.cpp", "opt2s_api8.cpp"):
        r = subprocess.run([gxx, "-std=c++17", "-fsyntax-only", "-DOPT2S_NVTX",
                            "-I", os.path.join(root, "include"), "-I", csrc, "-I", cuda_inc,
                            os.path.join(csrc, src)], capture_output=True, text=True)
        assert r.returncode == 0, r.stderr
