"""Seeded random collections through the 8-bit-state step, bitwise against
the oracle.

Each case draws, from its own seed, a collection of 1 to 24 tensors whose
sizes mix small fp32-state tensors (below min_8bit_size = 4,096) with 8-bit
ones of ragged, block-boundary and larger lengths; the storage dtypes; the
algorithm; skip_zeros; hyper-parameters (learning rate over four decades,
beta1 including 0, beta2, eps and weight decay over their ranges, AdEMAMix's
beta3 and alpha); the gradient recipe; the layout (separate allocations, or
packed buffers where most arrays start misaligned); and the starting step.
After every step, params, codes, absmaxes and fp32 states must hold the
oracle's bits and the gradients must be untouched.
"""
import numpy as np
import pytest
import torch

from elementwise_optimizer_b200 import binding as B
from elementwise_optimizer_b200 import synth
from tests.gpu_support import Harness8

pytestmark = pytest.mark.gpu

CASES = 24


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from elementwise_optimizer_b200 import _build
    _build.build()
    B.lib()
    yield
    B.opt2s_release_cache()


def draw_case(case):
    r = np.random.default_rng([synth.SEED_BASE, 9800, case])
    count = int(r.integers(1, 25))
    sizes = []
    for _ in range(count):
        kind = r.random()
        if kind < 0.3:
            sizes.append(int(r.integers(1, 4096)))                       # fp32 state
        elif kind < 0.55:
            sizes.append(int(r.choice([4096, 6144, 8192, 10240])) + int(r.integers(-3, 4)))
        elif kind < 0.95:
            sizes.append(int(r.integers(4096, 40_000)))
        else:
            sizes.append(int(r.integers(100_000, 300_000)))
    algo = str(r.choice(["adam", "ademamix"]))
    dtypes = [str(r.choice(["f32", "f16", "bf16"])) for _ in range(count)]
    hyper = dict(lr=float(10 ** r.uniform(-5, -1)),
                 beta1=float(r.choice([0.0, 0.5, 0.9, 0.95])),
                 beta2=float(r.choice([0.9, 0.99, 0.999, 0.9999])),
                 eps=float(r.choice([1e-12, 1e-8, 1e-6, 1e-3])),
                 weight_decay=float(r.choice([0.0, 1e-2, 0.1])),
                 beta3=float(r.choice([0.999, 0.9999])) if algo == "ademamix" else 0.0,
                 alpha=float(r.choice([2.0, 5.0, 8.0])) if algo == "ademamix" else 0.0)
    w = synth.Workload(f"fuzz8_{case}", sizes, dtypes, algo, hyper, 3, synth.SEED_BASE + 9800 + case,
                       str(r.choice(["normal", "sparse_mixture", "mixed_magnitude"])),
                       skip_zeros=bool(r.random() < 0.5))
    layout = str(r.choice(["separate", "packed"]))
    first_step = int(r.choice([1, 11, 1001]))
    steps = int(r.integers(1, 4))
    return w, layout, first_step, steps


@pytest.mark.parametrize("case", range(CASES))
def test_random_8bit_collection_matches_oracle(case):
    w, layout, first_step, steps = draw_case(case)
    h = Harness8(w, layout=layout)
    for t in range(first_step, first_step + steps):
        h.step_both(t)
        assert h.mismatches() == [], (t, w.sizes, w.dtypes, w.algo, w.skip_zeros, layout)
        assert h.grads_unchanged()
