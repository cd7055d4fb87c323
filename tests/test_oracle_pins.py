"""Pins for the CPU oracle: each check is fixed by something other than the
oracle itself -- a library optimizer or conversion, a closed form, an
invariant, or an exact special case -- so that a plausible slip in the oracle
(a dropped term, a wrong index, a swapped operand or a wrong rounding) fails
at least one of them.

The method is the 32-bit two-state update of the bitsandbytes issue
"Investigate a 256-thread SM103 path for small 32-bit optimizer tensors"
(sections "Problem", "Scope", "Correctness oracle"), with the standard
definitions of Adam (Kingma & Ba 2015, Algorithm 1), AdamW (Loshchilov &
Hutter 2019, Algorithm 2) and AdEMAMix (Pagliardini et al. 2024, Algorithm 1).
"""
import math

import numpy as np
import pytest
import torch

from elementwise_optimizer_b200 import synth

F32_EPS = 2.0 ** -23


def ulp32(x):
    """Spacing of float32 at |x| (at least the smallest subnormal)."""
    x = np.abs(np.asarray(x, np.float32))
    return np.spacing(x).astype(np.float64)


# --------------------------------------------------------------------------
# Storage conversions vs numpy / ml_dtypes / torch (IEEE 754 roundTiesToEven)
# --------------------------------------------------------------------------

def _conversion_probe(n=1 << 20, seed=7):
    g = np.random.Generator(np.random.Philox(seed))
    bits = g.integers(0, 1 << 32, n, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    # values near the fp16/bf16 rounding boundaries, overflow and subnormals
    special = np.array([0.0, -0.0, 1.0, -1.0, 65504.0, 65519.99, 65520.0,
                        65536.0, 6.1035156e-05, 5.9604645e-08, 2.9802322e-08,
                        2.9802326e-08, 1e-45, -1e-45, 3.4028235e38, np.inf,
                        -np.inf, np.nan, 1.0 + 2 ** -11, 1.0 + 3 * 2 ** -11,
                        1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.1754944e-38,
                        1.1754942e-38], np.float32)
    # exact ties: odd multiples of half a bf16/fp16 quantum around 1..2
    k = np.arange(0, 4096, dtype=np.uint32)
    ties_bf16 = ((np.uint32(0x3F800000) + (k << 16) + np.uint32(0x8000))).view(np.float32)
    ties_f16 = ((np.uint32(0x3F800000) + (k << 13) + np.uint32(0x1000))).view(np.float32)
    return np.concatenate([x, special, ties_bf16, ties_f16]).astype(np.float32)


def _same_bits_or_both_nan(a_bits, b_bits, a_val, b_val):
    nan = np.isnan(a_val) & np.isnan(b_val)
    return np.all((a_bits == b_bits) | nan)


def test_f16_narrowing_matches_numpy(oracle_mod):
    x = _conversion_probe()
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16)
    got = oracle_mod.narrow(x, "f16")
    assert _same_bits_or_both_nan(got, ref.view(np.uint16),
                                  got.view(np.float16), ref)


def test_bf16_narrowing_matches_ml_dtypes_and_torch(oracle_mod):
    import ml_dtypes
    x = _conversion_probe(seed=8)
    ref = x.astype(ml_dtypes.bfloat16)
    got = oracle_mod.narrow(x, "bf16")
    assert _same_bits_or_both_nan(got, ref.view(np.uint16),
                                  got.view(ml_dtypes.bfloat16).astype(np.float32),
                                  ref.astype(np.float32))
    tref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert _same_bits_or_both_nan(got, tref, x, x)


def test_widening_exhaustive(oracle_mod):
    import ml_dtypes
    allbits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f16 = oracle_mod.widen(allbits, "f16")
    ref16 = allbits.view(np.float16).astype(np.float32)
    assert np.array_equal(f16.view(np.uint32)[~np.isnan(ref16)],
                          ref16.view(np.uint32)[~np.isnan(ref16)])
    assert np.array_equal(np.isnan(f16), np.isnan(ref16))
    bf = oracle_mod.widen(allbits, "bf16")
    refb = allbits.view(ml_dtypes.bfloat16).astype(np.float32)
    assert np.array_equal(np.isnan(bf), np.isnan(refb))
    ok = ~np.isnan(refb)
    assert np.array_equal(bf.view(np.uint32)[ok], refb.view(np.uint32)[ok])


# --------------------------------------------------------------------------
# The float64 shadow vs torch.optim (an independent library implementation)
# --------------------------------------------------------------------------

HYPERS = [
    dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0),
    dict(lr=1e-2, beta1=0.8, beta2=0.95, eps=1e-3, weight_decay=0.1),
    dict(lr=3e-2, beta1=0.5, beta2=0.7, eps=1e-6, weight_decay=0.5),
]


def _torch_reference(p0, grads, hyper, cls=torch.optim.AdamW):
    p = torch.tensor(p0, dtype=torch.float64, requires_grad=True)
    opt = cls([p], lr=hyper["lr"], betas=(hyper["beta1"], hyper["beta2"]),
              eps=hyper["eps"], weight_decay=hyper["weight_decay"],
              foreach=False, fused=False)
    for g in grads:
        p.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
    st = opt.state[p]
    return (p.detach().numpy(), st["exp_avg"].numpy(), st["exp_avg_sq"].numpy())


@pytest.mark.parametrize("hyper", HYPERS)
def test_shadow_adamw_matches_torch(oracle_mod, hyper):
    n, steps = 4096, 12
    g = np.random.Generator(np.random.Philox(11))
    p0 = g.standard_normal(n)
    grads = [g.standard_normal(n) * 10.0 ** g.uniform(-6, 1, n) for _ in range(steps)]
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    for t, gr in enumerate(grads, 1):
        oracle_mod.step_f64(p, gr, m, v, algo="adam", step=t, **hyper)
    tp, tm, tv = _torch_reference(p0, grads, hyper)
    # m can cancel; bound its difference by the EMA of |g| (its magnitude scale)
    scale = np.zeros(n)
    for gr in grads:
        scale = hyper["beta1"] * scale + (1 - hyper["beta1"]) * np.abs(gr)
    assert np.all(np.abs(m - tm) <= 1e-14 * scale)
    np.testing.assert_allclose(v, tv, rtol=1e-13, atol=1e-300)
    np.testing.assert_allclose(p, tp, rtol=1e-12, atol=1e-15)


def test_shadow_adam_without_decay_matches_torch_adam(oracle_mod):
    hyper = dict(HYPERS[0])
    n = 1000
    g = np.random.Generator(np.random.Philox(12))
    p0 = g.standard_normal(n)
    grads = [g.standard_normal(n) * 1e-2 for _ in range(5)]
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    for t, gr in enumerate(grads, 1):
        oracle_mod.step_f64(p, gr, m, v, algo="adam", step=t, **hyper)
    tp, _, _ = _torch_reference(p0, grads, hyper, cls=torch.optim.Adam)
    np.testing.assert_allclose(p, tp, rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("alpha,wd", [(5.0, 0.0), (2.0, 0.1), (0.5, 0.3)])
def test_shadow_ademamix_reduces_to_torch_adam(oracle_mod, alpha, wd):
    """With beta1 = beta3 = 0 the slow EMA is the gradient itself and the bias
    correction of m1 is 1, so AdEMAMix(lr, alpha, wd) steps exactly like Adam
    with beta1 = 0, learning rate lr*(1+alpha) and weight decay wd/(1+alpha)
    (the decay factor 1 - lr*wd is unchanged)."""
    n, steps, lr = 2048, 8, 1e-2
    g = np.random.Generator(np.random.Philox(13))
    p0 = g.standard_normal(n)
    grads = [g.standard_normal(n) * 10.0 ** g.uniform(-4, 1, n) for _ in range(steps)]
    p, m, v, m2 = p0.copy(), np.zeros(n), np.zeros(n), np.zeros(n)
    for t, gr in enumerate(grads, 1):
        oracle_mod.step_f64(p, gr, m, v, m2, algo="ademamix", step=t, lr=lr,
                            beta1=0.0, beta2=0.99, beta3=0.0, alpha=alpha,
                            eps=1e-8, weight_decay=wd)
    lib = dict(lr=lr * (1 + alpha), beta1=0.0, beta2=0.99, eps=1e-8,
               weight_decay=wd / (1 + alpha))
    tp, _, _ = _torch_reference(p0, grads, lib)
    np.testing.assert_allclose(p, tp, rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(m2, grads[-1])


# --------------------------------------------------------------------------
# The fp32 oracle vs the float64 shadow, one step from identical state
# --------------------------------------------------------------------------

def _random_state(seed, n, dtype, algo):
    g = np.random.Generator(np.random.Philox(seed))
    p = synth.to_storage(g.standard_normal(n).astype(np.float32), dtype)
    gr = synth.to_storage((g.standard_normal(n) * 10.0 ** g.uniform(-5, 1, n)).astype(np.float32), dtype)
    m = (g.standard_normal(n) * 1e-2).astype(np.float32)
    m2 = (g.standard_normal(n) * 1e-2).astype(np.float32)
    v = (g.random(n) * 1e-3).astype(np.float32)
    s1 = np.concatenate([m, m2]) if algo == "ademamix" else m
    return p, gr, s1, v


@pytest.mark.parametrize("algo", ["adam", "ademamix"])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("hi", range(len(HYPERS)))
@pytest.mark.parametrize("t", [1, 2, 10, 1000])
def test_f32_oracle_one_step_within_rounding_of_shadow(oracle_mod, algo, dtype, hi, t):
    """From the same state and the same (fp32) hyper-parameters, the fp32
    oracle stays within a rounding-error bound of the float64 shadow.  Each
    fp32 operation errs by at most 2^-24 of its result, so every bound below
    is a small multiple of 2^-24 times the magnitudes of the terms that feed
    the result (which also covers cancellation in m and in p)."""
    hyper = {k: float(np.float32(x)) for k, x in dict(HYPERS[hi], beta3=0.999, alpha=3.0).items()}
    n = 20000
    p, gr, s1, v = _random_state(100 + hi, n, dtype, algo)
    pf = synth.from_storage(p, dtype).astype(np.float64)
    gf = synth.from_storage(gr, dtype).astype(np.float64)
    m_old = s1[:n].astype(np.float64)
    m2_old = s1[n:].astype(np.float64) if algo == "ademamix" else None
    v_old = v.astype(np.float64)
    p64, m64, v64 = pf.copy(), m_old.copy(), v_old.copy()
    m2_64 = m2_old.copy() if m2_old is not None else None
    oracle_mod.step_f64(p64, gf, m64, v64, m2_64, algo=algo, step=t, **hyper)
    p32, s1_32, v32 = p.copy(), s1.copy(), v.copy()
    oracle_mod.step_f32(p32, gr, s1_32, v32, dtype=dtype, algo=algo, step=t, **hyper)

    u = 2.0 ** -24
    tiny = 1e-44
    b1, b2, b3 = hyper["beta1"], hyper["beta2"], hyper["beta3"]
    m_scale = np.abs(b1 * m_old) + np.abs((1 - b1) * gf)
    assert np.all(np.abs(s1_32[:n] - m64) <= 4 * u * m_scale + tiny)
    assert np.all(np.abs(v32 - v64) <= 8 * u * v64 + tiny)
    num_scale = m_scale / (1 - b1 ** t)
    if algo == "ademamix":
        m2_scale = np.abs(b3 * m2_old) + np.abs((1 - b3) * gf)
        assert np.all(np.abs(s1_32[n:] - m2_64) <= 4 * u * m2_scale + tiny)
        num_scale = num_scale + hyper["alpha"] * m2_scale
    den = np.sqrt(v64 / (1 - b2 ** t)) + hyper["eps"]
    lr, wd = hyper["lr"], hyper["weight_decay"]
    p_scale = np.abs(pf * (1 - lr * wd)) + lr * num_scale / den
    got = synth.from_storage(p32, dtype).astype(np.float64)
    bound = 24 * u * p_scale + tiny
    if dtype == "f16":        # one more rounding, to binary16
        bound = bound + 2.0 ** -11 * np.abs(p64) + 2.0 ** -25
    elif dtype == "bf16":     # one more rounding, to bfloat16
        bound = bound + 2.0 ** -8 * np.abs(p64) + 1e-40
    assert np.all(np.abs(got - p64) <= bound)


# --------------------------------------------------------------------------
# Closed forms
# --------------------------------------------------------------------------

@pytest.mark.parametrize("algo", ["adam", "ademamix"])
def test_step_one_closed_form(oracle_mod, algo):
    """At t = 1 from zero state m/bc1 = g and v/bc2 = g^2 exactly (real
    arithmetic), and m2 = (1-beta3) g, so
    p1 = p0*(1-lr*wd) - lr*(g + alpha*(1-beta3)*g)/(|g| + eps)."""
    n = 50000
    g = np.random.Generator(np.random.Philox(21))
    p0 = g.standard_normal(n).astype(np.float32)
    gr = (g.standard_normal(n) * 10.0 ** g.uniform(-9, 1, n)).astype(np.float32)
    hyper = dict(lr=1e-2, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1,
                 beta3=0.99, alpha=4.0)
    p, s1 = p0.copy(), np.zeros(2 * n if algo == "ademamix" else n, np.float32)
    v = np.zeros(n, np.float32)
    oracle_mod.step_f32(p, gr, s1, v, dtype="f32", algo=algo, step=1, **hyper)
    gd = gr.astype(np.float64)
    num = gd + (hyper["alpha"] * (1 - hyper["beta3"]) * gd if algo == "ademamix" else 0)
    exact = p0 * (1 - 1e-2 * 0.1) - 1e-2 * num / (np.abs(gd) + 1e-8)
    step = 1e-2 * np.abs(num) / (np.abs(gd) + 1e-8)
    assert np.all(np.abs(p - exact) <= 2 * ulp32(exact) + 16 * F32_EPS * step)


def test_step_one_unit_gradient_is_exactly_minus_lr(oracle_mod):
    """p0 = 0, g = 1: m/bc1 = v/bc2 = 1 exactly in fp32 (Sterbenz), and
    1 + 1e-8 rounds to 1, so p1 is the fp32 value of -lr exactly."""
    p = np.zeros(1, np.float32)
    s1, v = np.zeros(1, np.float32), np.zeros(1, np.float32)
    oracle_mod.step_f32(p, np.ones(1, np.float32), s1, v, dtype="f32",
                        algo="adam", step=1, lr=1e-3, beta1=0.9, beta2=0.999,
                        eps=1e-8)
    assert p[0] == np.float32(-1e-3)


@pytest.mark.parametrize("algo", ["adam", "ademamix"])
@pytest.mark.parametrize("wd", [0.0, 0.05])
def test_constant_gradient_closed_form(oracle_mod, algo, wd):
    """A constant gradient g keeps m/bc1 = g and v/bc2 = g^2 at every step,
    while m2_k = g (1 - beta3^k), so with d = 1 - lr*wd
    p_T = p0 d^T - lr * sum_k d^(T-k) (g + alpha g (1-beta3^k)) / (|g| + eps).
    """
    T, lr, b3, alpha, eps = 1000, 1e-3, 0.999, 5.0, 1e-8
    gvals = np.array([0.5, -0.5, 2e-3, -7.0, 1e-6, 30.0], np.float32)
    p0 = np.array([2.0, -2.0, 3.0, 5.0, -4.0, 3.0], np.float32)
    n = gvals.size
    p = p0.copy()
    s1 = np.zeros(2 * n if algo == "ademamix" else n, np.float32)
    v = np.zeros(n, np.float32)
    for t in range(1, T + 1):
        oracle_mod.step_f32(p, gvals, s1, v, dtype="f32", algo=algo, step=t,
                            lr=lr, beta1=0.9, beta2=0.999, eps=eps, beta3=b3,
                            alpha=alpha, weight_decay=wd)
    gd = gvals.astype(np.float64)
    d = 1 - lr * wd
    k = np.arange(1, T + 1, dtype=np.float64)
    mix = (alpha * (1 - b3 ** k)) if algo == "ademamix" else np.zeros(T)
    w = d ** (T - k)
    total = (w[None, :] * (1 + mix[None, :])).sum(axis=1)
    exact = p0 * d ** T - lr * total * gd / (np.abs(gd) + eps)
    # each step adds O(1) rounding of |p|; T steps -> T-ish ulps
    np.testing.assert_allclose(p, exact, rtol=2e-4)
    if algo == "ademamix":
        np.testing.assert_allclose(s1[n:], gd * (1 - b3 ** T), rtol=1e-4)


# --------------------------------------------------------------------------
# Invariants and exact special cases
# --------------------------------------------------------------------------

@pytest.mark.parametrize("algo", ["adam", "ademamix"])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_zero_gradient_fixed_point(oracle_mod, algo, dtype):
    """g = 0 from zero state: nothing moves without decay; with decay only
    p *= d each step (p_T = p0 d^T), moments stay zero."""
    n = 513
    p0 = synth.to_storage(np.linspace(-3, 3, n).astype(np.float32), dtype)
    z = synth.to_storage(np.zeros(n, np.float32), dtype)
    for wd in (0.0, 0.1):
        p = p0.copy()
        s1 = np.zeros(2 * n if algo == "ademamix" else n, np.float32)
        v = np.zeros(n, np.float32)
        for t in range(1, 11):
            oracle_mod.step_f32(p, z, s1, v, dtype=dtype, algo=algo, step=t,
                                lr=1e-2, beta1=0.9, beta2=0.999, eps=1e-8,
                                beta3=0.999, alpha=5.0, weight_decay=wd)
        assert not s1.any() and not v.any()
        if wd == 0.0:
            assert np.array_equal(p.view(np.uint8), p0.view(np.uint8))
        else:
            exact = synth.from_storage(p0, dtype).astype(np.float64) * (1 - 1e-3) ** 10
            got = synth.from_storage(p, dtype).astype(np.float64)
            tol = {"f32": 12 * F32_EPS, "f16": 12 * 2 ** -11, "bf16": 12 * 2 ** -8}[dtype]
            assert np.all(np.abs(got - exact) <= tol * np.abs(exact) + 1e-30)


@pytest.mark.parametrize("algo", ["adam", "ademamix"])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_skip_zeros(oracle_mod, algo, dtype):
    """skip_zeros leaves every zero-gradient element wholly untouched (also
    without decay) and treats the others exactly as the plain step does."""
    n = 4097
    p, gr, s1, v = _random_state(31, n, dtype, algo)
    gvals = synth.from_storage(gr, dtype)
    zero = np.arange(n) % 3 == 0
    gvals[zero] = 0.0
    gvals[np.arange(n) % 6 == 0] = -0.0
    gr = synth.to_storage(gvals, dtype)
    kw = dict(dtype=dtype, algo=algo, step=5, lr=1e-2, beta1=0.9, beta2=0.999,
              eps=1e-8, beta3=0.999, alpha=5.0, weight_decay=0.1)
    a = [x.copy() for x in (p, s1, v)]
    oracle_mod.step_f32(a[0], gr, a[1], a[2], skip_zeros=True, **kw)
    b = [x.copy() for x in (p, s1, v)]
    oracle_mod.step_f32(b[0], gr, b[1], b[2], skip_zeros=False, **kw)
    zi = np.concatenate([zero, zero]) if algo == "ademamix" else zero
    assert np.array_equal(a[0][zero].view(np.uint8), p[zero].view(np.uint8))
    assert np.array_equal(a[1][zi], s1[zi]) and np.array_equal(a[2][zero], v[zero])
    nz = ~zero
    nzi = ~zi
    assert np.array_equal(a[0][nz].view(np.uint8), b[0][nz].view(np.uint8))
    assert np.array_equal(a[1][nzi], b[1][nzi]) and np.array_equal(a[2][nz], b[2][nz])
    # and without skip_zeros the zero-gradient elements do decay
    assert not np.array_equal(b[0][zero & (synth.from_storage(p, dtype) != 0)],
                              p[zero & (synth.from_storage(p, dtype) != 0)])


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_ademamix_alpha_zero_equals_adam_bitwise(oracle_mod, dtype):
    """alpha = 0 adds an exact +0 to m/bc1, so param, m1 and v match Adam."""
    n = 3000
    p, gr, s1, v = _random_state(41, n, dtype, "ademamix")
    kw = dict(dtype=dtype, step=7, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8,
              weight_decay=0.01)
    pa, s1a, va = p.copy(), s1.copy(), v.copy()
    oracle_mod.step_f32(pa, gr, s1a, va, algo="ademamix", beta3=0.9, alpha=0.0, **kw)
    pb, mb, vb = p.copy(), s1[:n].copy(), v.copy()
    oracle_mod.step_f32(pb, gr, mb, vb, algo="adam", **kw)
    assert np.array_equal(pa.view(np.uint8), pb.view(np.uint8))
    assert np.array_equal(s1a[:n], mb) and np.array_equal(va, vb)


def test_gradient_is_never_written(oracle_mod):
    n = 1025
    for dtype in ("f32", "f16", "bf16"):
        p, gr, s1, v = _random_state(51, n, dtype, "adam")
        keep = gr.copy()
        oracle_mod.step_f32(p, gr, s1, v, dtype=dtype, algo="adam", step=3,
                            lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8)
        assert np.array_equal(keep.view(np.uint8), gr.view(np.uint8))


def test_rejects_step_zero(oracle_mod):
    p = np.zeros(4, np.float32)
    with pytest.raises(ValueError):
        oracle_mod.step_f32(p, p.copy(), p.copy(), p.copy(), dtype="f32",
                            algo="adam", step=0, lr=1e-3, beta1=0.9,
                            beta2=0.999, eps=1e-8)


def test_bias_correction_and_decay_round_once(oracle_mod):
    """bc = 1 - beta^t and d = 1 - lr*wd are exact in double for these inputs
    up to one double rounding, then rounded to fp32 once."""
    assert oracle_mod.bias_correction(0.5, 3) == np.float32(0.875)
    assert oracle_mod.bias_correction(0.0, 1) == np.float32(1.0)
    assert oracle_mod.decay_factor(0.5, 0.25) == np.float32(0.875)
    b = np.float32(0.9)
    assert oracle_mod.bias_correction(float(b), 2) == np.float32(1 - float(b) ** 2)


def test_golden_traces(oracle_mod):
    """Single-element trajectories stored by tests/golden/make_golden.py; the
    first seven agree with an independent hand computation (see the file)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "traces.txt")
    rows = [l.split() for l in open(path) if l.strip() and not l.startswith("#")]
    assert rows
    from tests.golden.make_golden import run_trace
    for r in rows:
        case, t, hexbits = r[0], int(r[1]), r[2]
        got = run_trace(case)[t - 1]
        assert got == hexbits, (case, t, got, hexbits)


# --------------------------------------------------------------------------
# Data-parallel pieces: rank-order mean of gradients, fp32-gradient step
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("world", [1, 2, 3, 5, 8])
def test_average_grads_within_rounding_of_exact_mean(oracle_mod, dtype, world):
    """Each of the world-1 additions and the division rounds once, so the
    fp32 mean is within (world+1)*2^-24 * sum|g|/world of the exact mean."""
    n = 20000
    g = np.random.Generator(np.random.Philox(61))
    grads = [synth.to_storage((g.standard_normal(n) * 10.0 ** g.uniform(-6, 2, n)).astype(np.float32), dtype)
             for _ in range(world)]
    avg = oracle_mod.average_grads(grads, dtype)
    vals = np.stack([synth.from_storage(x, dtype).astype(np.float64) for x in grads])
    exact = vals.mean(axis=0)
    bound = (world + 1) * 2.0 ** -24 * np.abs(vals).sum(axis=0) / world + 1e-45
    assert np.all(np.abs(avg - exact) <= bound)
    if world == 1:
        assert np.array_equal(avg, vals[0].astype(np.float32))


@pytest.mark.parametrize("world", [2, 4, 8])
def test_average_of_identical_grads_is_exact(oracle_mod, world):
    """world identical copies (world a power of two) of values with at most
    20 significant bits: every partial sum k*x (k <= 8) is exact, and so is
    the division by world."""
    g = np.random.Generator(np.random.Philox(62))
    mant = g.integers(-(1 << 20) + 1, 1 << 20, 4096).astype(np.float64)
    x = (mant * 2.0 ** g.integers(-60, 10, 4096)).astype(np.float32)
    assert np.array_equal(oracle_mod.average_grads([x] * world, "f32"), x)


@pytest.mark.parametrize("algo", ["adam", "ademamix"])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_fp32_gradient_step_reduces_to_the_storage_step(oracle_mod, algo, dtype):
    """A float32 gradient whose values are representable in the storage dtype
    steps exactly like the storage-dtype gradient."""
    n = 3001
    p, gr, s1, v = _random_state(71, n, dtype, algo)
    kw = dict(dtype=dtype, algo=algo, step=4, lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8,
              beta3=0.99, alpha=5.0, weight_decay=0.01, skip_zeros=True)
    a = [x.copy() for x in (p, s1, v)]
    oracle_mod.step_f32(a[0], gr, a[1], a[2], **kw)
    b = [x.copy() for x in (p, s1, v)]
    oracle_mod.step_f32_fgrad(b[0], synth.from_storage(gr, dtype), b[1], b[2], **kw)
    for x, y in zip(a, b):
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8))


# --------------------------------------------------------------------------
# max_unorm: the update norm of a tensor clipped to max_unorm x its weight
# norm (the reading the oracle states; the pages name the option only)
# --------------------------------------------------------------------------

UNORM_HYPER = dict(lr=0.1, beta1=0.9, beta2=0.999, eps=1e-8, beta3=0.999, alpha=3.0)


@pytest.mark.parametrize("algo", ["adam", "ademamix"])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("skip", [False, True])
def test_max_unorm_above_the_norm_is_the_plain_step(oracle_mod, algo, dtype, skip):
    """A bound no update reaches leaves every bit of the plain step."""
    n = 5000
    p, gr, s1, v = _random_state(300, n, dtype, algo)
    gr[::7] = 0
    a = (p.copy(), s1.copy(), v.copy())
    b = (p.copy(), s1.copy(), v.copy())
    h = dict(UNORM_HYPER, weight_decay=0.01)
    oracle_mod.step_f32(a[0], gr, a[1], a[2], dtype=dtype, algo=algo, step=7, skip_zeros=skip, **h)
    s = oracle_mod.step_f32_max_unorm(b[0], gr, b[1], b[2], dtype=dtype, algo=algo, step=7,
                                      skip_zeros=skip, max_unorm=1e30, **h)
    assert s == 1.0
    for x, y in zip(a, b):
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8))


@pytest.mark.parametrize("algo", ["adam", "ademamix"])
def test_max_unorm_step_one_closed_form(oracle_mod, algo):
    """Every element equal: p0 = 0.5, g = 0.25.  At t = 1 every element has
    the same update u (1 for Adam, 1 + alpha(1-beta3) for AdEMAMix, up to
    eps), so |u| sqrt(n) against max_unorm * 0.5 sqrt(n) decides: a bound
    below |u| / 0.5 clips every element to p1 = p0 - lr*max_unorm*p0, a bound
    above it leaves p1 = p0 - lr*u."""
    n = 4096
    p0, g0 = 0.5, 0.25
    u = 1.0 + (UNORM_HYPER["alpha"] * (1 - UNORM_HYPER["beta3"]) if algo == "ademamix" else 0.0)
    for mu, want in ((0.1, p0 - UNORM_HYPER["lr"] * 0.1 * p0),
                     (10.0, p0 - UNORM_HYPER["lr"] * u)):
        p = np.full(n, p0, np.float32)
        g = np.full(n, g0, np.float32)
        s1 = np.zeros(2 * n if algo == "ademamix" else n, np.float32)
        v = np.zeros(n, np.float32)
        oracle_mod.step_f32_max_unorm(p, g, s1, v, dtype="f32", algo=algo, step=1,
                                      max_unorm=mu, **UNORM_HYPER)
        assert np.all(p == p[0])
        assert abs(float(p[0]) - want) <= 8 * float(ulp32(want)), (mu, float(p[0]), want)


@pytest.mark.parametrize("algo", ["adam", "ademamix"])
@pytest.mark.parametrize("wd", [0.0, 0.5])
@pytest.mark.parametrize("t", [1, 10, 1000])
def test_max_unorm_bounds_the_applied_update(oracle_mod, algo, wd, t):
    """The update actually applied, p1 - p0*decay (one fp32 product rounded
    as the step rounds it), has norm lr*max_unorm*||p0|| when the bound
    binds, and the plain step's update otherwise; skipped elements add
    nothing.  Checked on random states against norms taken in float64."""
    n = 20000
    for skip in (False, True):
        p, gr, s1, v = _random_state(400 + t, n, "f32", algo)
        if skip:
            gr[::3] = 0
        h = dict(UNORM_HYPER, weight_decay=wd)
        decay = np.float32(oracle_mod.decay_factor(h["lr"], wd))
        plain = (p.copy(), s1.copy(), v.copy())
        oracle_mod.step_f32(plain[0], gr, plain[1], plain[2], dtype="f32", algo=algo, step=t,
                            skip_zeros=skip, **h)
        base = (p * decay).astype(np.float64)          # rounded to fp32 like the step
        d_plain = plain[0].astype(np.float64) - base
        if skip:
            d_plain[gr == 0] = 0.0
        pn = float(np.linalg.norm(p.astype(np.float64)))
        free = float(np.linalg.norm(d_plain)) / (h["lr"] * pn)  # the unclipped ratio
        for mu in (0.25 * free, 0.8 * free, 4.0 * free):
            q, m_, v_ = p.copy(), s1.copy(), v.copy()
            s = oracle_mod.step_f32_max_unorm(q, gr, m_, v_, dtype="f32", algo=algo, step=t,
                                              skip_zeros=skip, max_unorm=float(np.float32(mu)), **h)
            d = q.astype(np.float64) - base
            if skip:
                assert np.array_equal(q[gr == 0], p[gr == 0])
                d[gr == 0] = 0.0
            norm = float(np.linalg.norm(d))
            if mu < free:
                assert s < 1.0
                assert norm == pytest.approx(h["lr"] * float(np.float32(mu)) * pn, rel=2e-4)
            else:
                assert s == 1.0
                assert np.array_equal(q, plain[0])
            # the moments never depend on the bound
            assert np.array_equal(m_, plain[1]) and np.array_equal(v_, plain[2])


def test_max_unorm_must_be_positive(oracle_mod):
    p, gr, s1, v = _random_state(500, 16, "f32", "adam")
    for mu in (0.0, -1.0, float("nan")):
        with pytest.raises(ValueError):
            oracle_mod.step_f32_max_unorm(p, gr, s1, v, dtype="f32", algo="adam", step=1,
                                          max_unorm=mu, **UNORM_HYPER)


# --------------------------------------------------------------------------
# LAMB (You et al. 2020, Algorithm 2): per tensor, the Adam direction plus
# lambda*p, scaled by the trust ratio ||p|| / ||direction + lambda*p||.
# --------------------------------------------------------------------------

LAMB_HYPER = dict(lr=0.01, beta1=0.9, beta2=0.999, eps=1e-6)


def _lamb_state(seed, n, dtype):
    p, gr, m, v = _random_state(seed, n, dtype, "adam")
    return p, gr, m, v


@pytest.mark.parametrize("p0,wd", [(0.5, 0.0), (-4.0, 0.5), (3.0, 0.1)])
def test_lamb_step_one_closed_form(oracle_mod, p0, wd):
    """Every element equal: p0 and g = 0.25 at t = 1 give every element the
    same direction u = g/(|g| + eps) (m/bc1 = g and sqrt(v/bc2) = |g| in
    exact arithmetic), so w = u + wd*p0 for all of them and the trust
    ratio is |p0| / |w|: each element moves by lr*|p0| against the sign of w.
    (p0 = -4 with wd = 0.5 gives w = -1: the decay term inside w decides the
    direction.)"""
    n = 4096
    p = np.full(n, p0, np.float32)
    g = np.full(n, 0.25, np.float32)
    m = np.zeros(n, np.float32)
    v = np.zeros(n, np.float32)
    r = oracle_mod.step_f32_lamb(p, g, m, v, dtype="f32", step=1, weight_decay=wd, **LAMB_HYPER)
    u = 0.25 / (0.25 + LAMB_HYPER["eps"])
    w = u + wd * p0
    want = p0 - LAMB_HYPER["lr"] * abs(p0) * math.copysign(1.0, w)
    assert r == pytest.approx(abs(p0) / abs(w), rel=1e-6)
    assert np.all(p == p[0])
    assert abs(float(p[0]) - want) <= 8 * float(ulp32(want)), (float(p[0]), want)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("wd", [0.0, 0.01, 0.3])
@pytest.mark.parametrize("t", [1, 10, 1000])
def test_lamb_update_is_the_trust_ratio_times_the_decayed_direction(oracle_mod, dtype, wd, t):
    """Against the float64 shadow: the Adam direction u of every element is
    taken from the shadow step (pinned to torch.optim.Adam) run with lr = 1
    and no decay, w = u + wd*p0 and the trust ratio ||p0|| / ||w|| in float64.
    The oracle's applied update p1 - p0 must equal -lr*ratio*w elementwise up
    to fp32 rounding, and its norm must be lr*||p0||; skipped elements do
    not move and add nothing to ||w||; the moments are the plain step's."""
    n = 20000
    for skip in (False, True):
        p, gr, m, v = _lamb_state(600 + t, n, dtype)
        if skip:
            gr[::3] = 0
        pf = synth.from_storage(p, dtype).astype(np.float64)
        gf = synth.from_storage(gr, dtype).astype(np.float64)
        sh_p, sh_m, sh_v = pf.copy(), m.astype(np.float64), v.astype(np.float64)
        h32 = {k: float(np.float32(x)) for k, x in LAMB_HYPER.items()}
        oracle_mod.step_f64(sh_p, gf, sh_m, sh_v, algo="adam", step=t, lr=1.0,
                            beta1=h32["beta1"], beta2=h32["beta2"], eps=h32["eps"],
                            skip_zeros=skip)
        u = pf - sh_p
        w = u + float(np.float32(wd)) * pf
        live = ~((gr.view(np.uint16 if dtype != "f32" else np.uint32) << 1) == 0) if skip else \
            np.ones(n, bool)
        w[~live] = 0.0
        ratio = np.linalg.norm(pf) / np.linalg.norm(w)
        q, m1, v1 = p.copy(), m.copy(), v.copy()
        r = oracle_mod.step_f32_lamb(q, gr, m1, v1, dtype=dtype, step=t, weight_decay=wd,
                                     skip_zeros=skip, **LAMB_HYPER)
        assert r == pytest.approx(ratio, rel=1e-5)
        d = synth.from_storage(q, dtype).astype(np.float64) - pf
        want = -LAMB_HYPER["lr"] * ratio * w
        # each element: fp32 rounding of w (relative to |u| + |wd p|), of the
        # products and of the final subtraction (one ulp of p in storage)
        quantum = np.spacing(np.abs(synth.from_storage(q, dtype)).astype(np.float32)).astype(np.float64)
        if dtype == "bf16":
            quantum = quantum * 2.0 ** 16
        slack = (LAMB_HYPER["lr"] * ratio * (np.abs(u) + abs(wd) * np.abs(pf)) * 1e-5 + quantum)
        assert np.all(np.abs(d - want) <= slack)
        if dtype == "f32":
            assert np.linalg.norm(d) == pytest.approx(LAMB_HYPER["lr"] * np.linalg.norm(pf), rel=1e-4)
        assert np.array_equal(q[~live], p[~live])
        plain_p, plain_m, plain_v = p.copy(), m.copy(), v.copy()
        oracle_mod.step_f32(plain_p, gr, plain_m, plain_v, dtype=dtype, algo="adam", step=t,
                            skip_zeros=skip, **LAMB_HYPER)
        assert np.array_equal(m1, plain_m) and np.array_equal(v1, plain_v)


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_lamb_zero_weights_take_ratio_one(oracle_mod, dtype):
    """||p0|| = 0 takes trust ratio 1, so from p0 = 0 the LAMB step is
    p1 = 0 - lr*u, bit for bit the plain Adam step from p0 = 0 without decay
    (0*decay - lr*u)."""
    n = 3000
    _, gr, m, v = _lamb_state(700, n, dtype)
    p = synth.to_storage(np.zeros(n, np.float32), dtype)
    a = (p.copy(), m.copy(), v.copy())
    b = (p.copy(), m.copy(), v.copy())
    r = oracle_mod.step_f32_lamb(a[0], gr, a[1], a[2], dtype=dtype, step=5, weight_decay=0.2,
                                 **LAMB_HYPER)
    oracle_mod.step_f32(b[0], gr, b[1], b[2], dtype=dtype, algo="adam", step=5, **LAMB_HYPER)
    assert r == 1.0
    for x, y in zip(a, b):
        assert np.array_equal(x.view(np.uint8), y.view(np.uint8))


def test_lamb_zero_gradient_closed_forms(oracle_mod):
    """From zero moments and g = 0: the direction is u = 0, so w = wd*p.
    Without decay W = 0 and the ratio is 1, leaving p unchanged; with decay
    W = wd*||p||, the ratio 1/wd, and every element becomes p*(1 - lr) up to
    rounding."""
    n = 5000
    p, _, _, _ = _lamb_state(800, n, "f32")
    g = np.zeros(n, np.float32)
    q = p.copy()
    r = oracle_mod.step_f32_lamb(q, g, np.zeros(n, np.float32), np.zeros(n, np.float32),
                                 dtype="f32", step=3, weight_decay=0.0, **LAMB_HYPER)
    assert r == 1.0 and np.array_equal(q, p)
    q = p.copy()
    wd = 0.25
    r = oracle_mod.step_f32_lamb(q, g, np.zeros(n, np.float32), np.zeros(n, np.float32),
                                 dtype="f32", step=3, weight_decay=wd, **LAMB_HYPER)
    assert r == pytest.approx(1.0 / wd, rel=1e-6)
    want = p.astype(np.float64) * (1.0 - LAMB_HYPER["lr"])
    assert np.all(np.abs(q - want) <= 4 * ulp32(want))


def test_lamb_rejects_step_zero(oracle_mod):
    p, gr, m, v = _lamb_state(900, 16, "f32")
    with pytest.raises(ValueError):
        oracle_mod.step_f32_lamb(p, gr, m, v, dtype="f32", step=0, **LAMB_HYPER)


# --------------------------------------------------------------------------
# 8-bit blockwise state (Dettmers, Lewis, Shleifer & Zettlemoyer, "8-bit
# Optimizers via Block-wise Quantization", ICLR 2022, sections 2.1-2.3).
# --------------------------------------------------------------------------

from fractions import Fraction


def _rn32(fr: Fraction) -> np.float32:
    """The binary32 value nearest to the exact rational fr (ties to an even
    significand), found by comparing exact distances to the neighbours."""
    c = np.float32(float(fr))
    cands = [c, np.nextafter(c, np.float32(np.inf)), np.nextafter(c, np.float32(-np.inf))]
    best = min(cands, key=lambda x: (abs(Fraction(float(x)) - fr),
                                     int(np.array(x).view(np.uint32)) & 1))
    return np.float32(best)


def _map_from_bits(signed: bool) -> np.ndarray:
    """Every 8-bit pattern of the data type decoded from its fields, as the
    paper describes them: [sign,] E zero bits (decimal exponent 10^-E), an
    indicator bit 1, then F fraction bits f of a linear quantization of
    [0.1, 1] (the midpoint of the f-th of 2^F equal bins).  Patterns without
    an indicator are 0, except one spare pattern, read as 1.0."""
    vals = []
    body = 7 if signed else 8                      # bits after the sign
    for pattern in range(256):
        sign = -1 if (signed and pattern >> 7) else 1
        bits = pattern & ((1 << body) - 1)
        if bits == 0 or (not signed and bits == 1):   # no indicator among the 7 leading bits
            vals.append(None)
            continue
        width = body if signed else body - 1            # the unsigned last bit is a fraction bit
        lead = bits if signed else bits >> 1
        E = width - lead.bit_length()                   # zero bits before the indicator
        if E > 6:
            vals.append(None)
            continue
        F = (body - 1 - E)                              # remaining bits after the indicator
        f = bits & ((1 << F) - 1)
        value = Fraction(1, 10 ** E) * (Fraction(1, 10) + Fraction(9, 10) * Fraction(2 * f + 1, 2 ** (F + 1)))
        vals.append(sign * value)
    exact = sorted(set(v for v in vals if v is not None))
    assert len(exact) == 254, len(exact)
    out = np.array([_rn32(v) for v in exact] + [np.float32(0.0), np.float32(1.0)], np.float32)
    return np.sort(out)


@pytest.mark.parametrize("signed", [True, False])
def test_quant_map_is_the_papers_data_type(oracle_mod, signed):
    want = _map_from_bits(signed)
    got = oracle_mod.quant_map(signed)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    # structure: strictly ascending, 0 and 1 present, 2^F values per decade
    assert np.all(np.diff(got.astype(np.float64)) > 0)
    assert 0.0 in got and got[-1] == 1.0
    pos = got[(got > 0) & (got < 1)].astype(np.float64)
    for E in range(7):
        F = (6 if signed else 7) - E
        inside = pos[(pos >= 0.1 * 10.0 ** -E) & (pos < 10.0 ** -E)]
        assert len(inside) == 2 ** F, (E, len(inside))
        if len(inside) > 1:      # a linear fraction: equal steps of 0.9*10^-E/2^F
            assert np.allclose(np.diff(inside), 0.9 * 10.0 ** -E / 2 ** F, rtol=1e-5)
    if signed:                   # symmetric apart from the spare 1.0
        assert got[127] == 0.0 and np.array_equal(got[:127], -got[128:255][::-1])
    else:
        assert got[0] == 0.0 and np.all(got >= 0)


def _nearest_codes(qmap, x):
    """Brute force: the index of the nearest map value (float64 distances,
    first index on a tie, i.e. the lower code)."""
    d = np.abs(x.astype(np.float64)[:, None] - qmap.astype(np.float64)[None, :])
    return np.argmin(d, axis=1).astype(np.uint8)


@pytest.mark.parametrize("signed", [True, False])
def test_quantize_is_the_nearest_code(oracle_mod, signed):
    qmap = oracle_mod.quant_map(signed)
    g = np.random.Generator(np.random.Philox(31))
    lo = -1.0 if signed else 0.0
    xs = [g.uniform(lo, 1.0, 4000).astype(np.float32),
          (np.sign(g.uniform(lo, 1.0, 4000)) * 10.0 ** g.uniform(-9, 0, 4000)).astype(np.float32),
          qmap]
    a, b = qmap[:-1].astype(np.float64), qmap[1:].astype(np.float64)
    mid = ((a + b) / 2).astype(np.float32)
    exact_ties = mid[mid.astype(np.float64) == (a + b) / 2]
    assert exact_ties.size > 100
    xs += [exact_ties, np.nextafter(mid, np.float32(2)), np.nextafter(mid, np.float32(-2)),
           np.array([0.0, -0.0, 1.0, 1e-45, 1e-30, 5e-8], np.float32)]
    if signed:
        xs.append(np.array([-1.0, -1e-45], np.float32))
    x = np.concatenate(xs)
    assert np.array_equal(oracle_mod.quantize(qmap, x), _nearest_codes(qmap, x))
    assert np.array_equal(oracle_mod.quantize(qmap, qmap), np.arange(256, dtype=np.uint8))
    # every exact tie goes to the lower of its two codes
    codes = oracle_mod.quantize(qmap, exact_ties)
    assert np.all(qmap[codes] < exact_ties)


def _block_quantize(qmap, x, block=2048):
    """Reference block quantization: per block the absmax in float32, the
    normalised values x/absmax (float32 division), brute-force nearest codes;
    the code of 0 where the absmax is 0."""
    n = x.size
    nb = (n + block - 1) // block
    codes = np.empty(n, np.uint8)
    amax = np.zeros(nb, np.float32)
    zc = int(np.nonzero(qmap == 0.0)[0][0])
    for b in range(nb):
        seg = x[b * block:(b + 1) * block]
        a = np.float32(np.max(np.abs(seg))) if seg.size else np.float32(0)
        amax[b] = a
        if a > 0:
            codes[b * block:(b + 1) * block] = _nearest_codes(qmap, (seg / a).astype(np.float32))
        else:
            codes[b * block:(b + 1) * block] = zc
    return codes, amax


def _dequant(qmap, codes, amax, block=2048):
    return (qmap[codes] * np.repeat(amax, block)[:codes.size]).astype(np.float32)


def _eightbit_reference(oracle_mod, algo, dtype, p, gr, q1, q2, a1, a2, step, hyper, skip):
    """The 8-bit step composed from pinned parts: dequantize (map value times
    block absmax), the plain fp32 oracle step (pinned to torch.optim), and the
    reference block quantization above."""
    smap, umap = oracle_mod.quant_map(True), oracle_mod.quant_map(False)
    n = p.size
    nb = (n + 2047) // 2048
    m = _dequant(smap, q1[:n], a1[:nb])
    v = _dequant(umap, q2, a2)
    s1 = m
    if algo == "ademamix":
        s1 = np.concatenate([m, _dequant(smap, q1[n:], a1[nb:])])
    p = p.copy()
    oracle_mod.step_f32(p, gr, s1, v, dtype=dtype, algo=algo, step=step, skip_zeros=skip, **hyper)
    c1, b1 = _block_quantize(smap, s1[:n])
    c2, b2 = _block_quantize(umap, v)
    if algo == "ademamix":
        c3, b3 = _block_quantize(smap, s1[n:])
        c1, b1 = np.concatenate([c1, c3]), np.concatenate([b1, b3])
    return p, c1, c2, b1, b2


EIGHT_HYPER = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, beta3=0.9999, alpha=5.0,
                   weight_decay=0.01)


@pytest.mark.parametrize("algo", ["adam", "ademamix"])
@pytest.mark.parametrize("dtype", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("t", [1, 2, 10, 1000])
def test_8bit_step_is_dequantize_update_quantize(oracle_mod, algo, dtype, t):
    """Random 8-bit states (codes and block absmaxes; zero state at t = 1),
    a ragged last block, with and without skip_zeros: param bits, codes and
    absmaxes equal the composition of the pinned parts."""
    n = 3 * 2048 + 777
    nb = 4
    two = algo == "ademamix"
    g = np.random.Generator(np.random.Philox(900 + t))
    for skip in (False, True):
        p = synth.to_storage(g.standard_normal(n).astype(np.float32), dtype)
        gr = synth.to_storage((g.standard_normal(n) * 10.0 ** g.uniform(-5, 0, n)).astype(np.float32),
                              dtype)
        if skip:
            gr[::5] = 0
        if t == 1:
            q1 = np.zeros(2 * n if two else n, np.uint8)
            q2 = np.zeros(n, np.uint8)
            a1 = np.zeros(2 * nb if two else nb, np.float32)
            a2 = np.zeros(nb, np.float32)
        else:
            q1 = g.integers(0, 256, 2 * n if two else n).astype(np.uint8)
            q2 = g.integers(0, 256, n).astype(np.uint8)
            a1 = (g.random(2 * nb if two else nb) * 1e-2).astype(np.float32)
            a2 = (g.random(nb) * 1e-4).astype(np.float32)
        want = _eightbit_reference(oracle_mod, algo, dtype, p, gr, q1, q2, a1, a2, t,
                                   EIGHT_HYPER, skip)
        got = [p.copy(), q1.copy(), q2.copy(), a1.copy(), a2.copy()]
        oracle_mod.step_8bit(got[0], gr, got[1], got[2], got[3], got[4], dtype=dtype, algo=algo,
                             step=t, skip_zeros=skip, **EIGHT_HYPER)
        for k, (x, y) in enumerate(zip(got, want)):
            assert np.array_equal(x.view(np.uint8), y.view(np.uint8)), (skip, k)


@pytest.mark.parametrize("algo", ["adam", "ademamix"])
def test_8bit_first_step_equals_the_32bit_step(oracle_mod, algo):
    """From zero state the dequantized moments are exactly 0, so the first
    8-bit update of the param is the 32-bit step's, bit for bit; and each
    block's stored absmax is the largest |m| of the 32-bit step's moments in
    that block."""
    n = 5000
    g = np.random.Generator(np.random.Philox(77))
    p = g.standard_normal(n).astype(np.float32)
    gr = (g.standard_normal(n) * 1e-2).astype(np.float32)
    two = algo == "ademamix"
    a = [p.copy(), np.zeros(2 * n if two else n, np.uint8), np.zeros(n, np.uint8),
         np.zeros(6 if two else 3, np.float32), np.zeros(3, np.float32)]
    oracle_mod.step_8bit(a[0], gr, a[1], a[2], a[3], a[4], dtype="f32", algo=algo, step=1,
                         **EIGHT_HYPER)
    b = [p.copy(), np.zeros(2 * n if two else n, np.float32), np.zeros(n, np.float32)]
    oracle_mod.step_f32(b[0], gr, b[1], b[2], dtype="f32", algo=algo, step=1, **EIGHT_HYPER)
    assert np.array_equal(a[0], b[0])
    for blk in range(3):
        sl = slice(2048 * blk, min(n, 2048 * (blk + 1)))
        assert a[3][blk] == np.max(np.abs(b[1][:n][sl]))
        assert a[4][blk] == np.max(b[2][sl])


def test_8bit_zero_gradient_keeps_zero_state(oracle_mod):
    """g = 0 everywhere from zero state without decay: the moments stay 0, every
    absmax stays 0 and every code is the code of 0; the param is unchanged."""
    n = 4097
    p = np.linspace(-1, 1, n).astype(np.float32)
    q1 = np.zeros(n, np.uint8)
    q2 = np.zeros(n, np.uint8)
    a1 = np.zeros(3, np.float32)
    a2 = np.zeros(3, np.float32)
    h = dict(EIGHT_HYPER, weight_decay=0.0)
    q = p.copy()
    oracle_mod.step_8bit(q, np.zeros(n, np.float32), q1, q2, a1, a2, dtype="f32", algo="adam",
                         step=1, **h)
    smap, umap = oracle_mod.quant_map(True), oracle_mod.quant_map(False)
    assert np.array_equal(q, p)
    assert np.all(a1 == 0) and np.all(a2 == 0)
    assert np.all(smap[q1] == 0) and np.all(umap[q2] == 0)
