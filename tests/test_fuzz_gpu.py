"""Seeded random collections through the C ABI, bitwise against the oracle.

Each case draws, from its own seed, a collection (1 to 40 tensors whose sizes
mix empty, single-element, ragged and chunk-boundary lengths with a few
larger ones), storage dtypes (mixed, or one 16-bit dtype so that the
specialised Adam kernel runs), the algorithm, skip_zeros, hyper-parameters
(learning rate over four decades, beta1 including 0, weight decay on or off),
the gradient recipe, the storage layout (separate allocations, packed back to
back, or padded so that most tensors start misaligned), the starting step,
for half the cases a forced chunk length and launch shape, for a third of
them a max_unorm bound (opt2s_step_max_unorm against the oracle's bounded
step), and for some of the other Adam cases the LAMB step (opt2s_step_lamb
against the oracle's).  After every step, param, state1 and state2 must hold the oracle's
bits and the gradients must be untouched.
"""
import numpy as np
import pytest

import oracle
from elementwise_optimizer_b200 import binding as B
from elementwise_optimizer_b200 import synth
from tests.gpu_support import Harness

pytestmark = pytest.mark.gpu

CASES = 32


def draw_case(case):
    r = np.random.default_rng([synth.SEED_BASE, 9100, case])
    count = int(r.integers(1, 41))
    sizes = []
    for _ in range(count):
        kind = r.random()
        if kind < 0.15:
            sizes.append(int(r.integers(0, 3)))
        elif kind < 0.45:
            sizes.append(int(r.integers(3, 300)))
        elif kind < 0.70:
            base = int(r.choice([256, 512, 1024, 2048, 4096, 8192]))
            sizes.append(base + int(r.integers(-9, 10)))
        elif kind < 0.95:
            sizes.append(int(r.integers(300, 70_000)))
        else:
            sizes.append(int(r.integers(1 << 19, 1 << 21)))
    algo = str(r.choice(["adam", "ademamix"]))
    if r.random() < 0.3:
        dtypes = [str(r.choice(["f16", "bf16"]))] * count
    else:
        dtypes = [str(r.choice(["f32", "f16", "bf16"])) for _ in range(count)]
    hyper = dict(lr=float(10 ** r.uniform(-5, -1)),
                 beta1=float(r.choice([0.0, 0.5, 0.9, 0.95])),
                 beta2=float(r.choice([0.9, 0.99, 0.999, 0.9999])),
                 eps=float(r.choice([1e-12, 1e-8, 1e-6, 1e-3])),
                 weight_decay=float(r.choice([0.0, 1e-2, 0.1])),
                 beta3=float(r.choice([0.999, 0.9999])) if algo == "ademamix" else 0.0,
                 alpha=float(r.choice([2.0, 5.0, 8.0])) if algo == "ademamix" else 0.0)
    w = synth.Workload(f"fuzz{case}", sizes, dtypes, algo, hyper, 3,
                       synth.SEED_BASE + 9100 + case,
                       str(r.choice(["normal", "sparse_mixture", "mixed_magnitude"])),
                       skip_zeros=bool(r.random() < 0.5))
    layout = str(r.choice(["separate", "packed", "padded"]))
    pad = int(r.integers(1, 6))
    first_step = int(r.choice([1, 11, 1001]))
    steps = int(r.integers(1, 4))
    geometry = None
    if r.random() < 0.5:
        geometry = (int(r.choice([32, 64, 128, 256])), int(r.choice([0, 1, 3, 7])),
                    int(r.choice([0, 8, 256, 1000, 4096])))
    max_unorm = float(np.float32(10 ** r.uniform(-2, 1))) if r.random() < 1 / 3 else 0.0
    # LAMB takes Adam moments; drawn last, so the draws above are unchanged
    lamb = algo == "adam" and max_unorm == 0.0 and r.random() < 0.4
    return w, layout, pad, first_step, steps, geometry, max_unorm, lamb


@pytest.mark.usefixtures("testing_lib")
@pytest.mark.parametrize("case", range(CASES))
def test_random_collection_matches_oracle(case):
    w, layout, pad, first_step, steps, geometry, max_unorm, lamb = draw_case(case)
    if geometry is not None:
        B.opt2s_release_cache()
        prev = B.testing_set_chunk_elems(geometry[2])
        B.testing_set_launch(geometry[0], geometry[1])
    try:
        h = Harness(w, layout=layout, pad=pad)
        for t in range(first_step, first_step + steps):
            if max_unorm > 0.0:
                h.load_grads(t)
                B.opt2s_step_max_unorm(h.tl, h.hyper, max_unorm, t)
                for i, dt in enumerate(w.dtypes):
                    oracle.step_f32_max_unorm(h.h_p[i], h._h_g[i], h.h_s1[i], h.h_s2[i], dtype=dt,
                                              algo=w.algo, step=t, skip_zeros=w.skip_zeros,
                                              max_unorm=max_unorm, **w.hyper)
            elif lamb:
                h.load_grads(t)
                B.opt2s_step_lamb(h.tl, h.hyper, t)
                hy = {k: w.hyper[k] for k in ("lr", "beta1", "beta2", "eps", "weight_decay")}
                for i, dt in enumerate(w.dtypes):
                    oracle.step_f32_lamb(h.h_p[i], h._h_g[i], h.h_s1[i], h.h_s2[i], dtype=dt, step=t,
                                         skip_zeros=w.skip_zeros, **hy)
            else:
                h.step_both(t)
            worst = h.max_ulps()
            assert worst == {"param": 0, "state1": 0, "state2": 0}, (t, worst, w.sizes, w.dtypes)
            assert h.grads_unchanged()
    finally:
        if geometry is not None:
            B.testing_set_launch(0, 0)
            B.testing_set_chunk_elems(prev)
            B.opt2s_release_cache()
