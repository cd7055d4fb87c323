"""opt2s_step_noalloc: the step for callers that cannot let the library
allocate device memory (a runtime that owns every byte of device memory
through its own pool, or a deployment whose footprint is fixed at start-up).

It runs the same kernel and arithmetic as opt2s_step with another launch
geometry (fixed 8,192-element chunks, 128-thread blocks), and launch geometry
must not change a bit of the result.  So on two calls in a row -- the second
call reuses the fixed device table the first one left behind -- its results
must equal the oracle's bit for bit and opt2s_step's bit for bit, each call
must count exactly one launch, and a collection larger than its fixed table
must be rejected before any work (no launch, no update).

This file is collected last on purpose, and it holds no state of its own
between tests, so it passes both alone in a fresh process and after the rest
of the suite.
"""
import numpy as np
import pytest
import torch

from elementwise_optimizer_b200 import binding as B
from elementwise_optimizer_b200 import synth
from tests.gpu_support import Harness, storage_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from elementwise_optimizer_b200 import _build
    _build.build()
    B.lib()


def _workload(algo):
    sizes = [1, 33, 64, 1000, 4097, 8192, 8193, 100_003, 1 << 20]
    dtypes = [("f32", "f16", "bf16")[i % 3] for i in range(len(sizes))]
    hyper = dict(synth.ADEMAMIX_HYPER if algo == "ademamix" else synth.ADAM_HYPER,
                 weight_decay=0.01)
    return synth.Workload(f"noalloc_{algo}", sizes, dtypes, algo, hyper, 2,
                          synth.SEED_BASE + 30, "mixed_magnitude", skip_zeros=(algo == "adam"))


@pytest.mark.parametrize("layout", ["separate", "packed"])
@pytest.mark.parametrize("algo", ["adam", "ademamix"])
def test_noalloc_matches_oracle_and_opt2s_step_on_two_calls(algo, layout):
    w = _workload(algo)
    a = Harness(w, layout=layout)          # stepped by opt2s_step_noalloc, checked against the oracle
    b = Harness(w, layout=layout)          # stepped by opt2s_step
    for t in (1, 2):
        a.load_grads(t)
        b.load_grads(t)
        before = B.launch_count()
        B.opt2s_step_noalloc(a.tl, a.hyper, t)
        assert B.launch_count() == before + 1
        B.opt2s_step(b.tl, b.hyper, t)
        a.oracle_step(t)
        torch.cuda.synchronize()
        assert a.max_ulps() == {"param": 0, "state1": 0, "state2": 0}, t
        assert a.grads_unchanged()
        for i in range(len(w.sizes)):
            assert np.array_equal(storage_bits(a.params[i]), storage_bits(b.params[i]))
            assert np.array_equal(storage_bits(a.s1[i]), storage_bits(b.s1[i]))
            assert np.array_equal(storage_bits(a.s2[i]), storage_bits(b.s2[i]))


def test_noalloc_rejects_a_collection_beyond_its_table():
    cap = B.noalloc_max_chunks()
    assert cap == 65536
    dev = torch.device("cuda")
    # one more single-chunk tensor than the table holds, all views of one buffer
    n = cap + 1
    p = torch.zeros(2 * n, device=dev)
    g = torch.ones(2 * n, device=dev)
    s = torch.zeros(4 * n, device=dev)
    recs = [(p.data_ptr() + 8 * i, g.data_ptr() + 8 * i, s.data_ptr() + 16 * i,
             s.data_ptr() + 16 * i + 8, 1, B.DTYPES["f32"]) for i in range(n)]
    before = B.launch_count()
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step_noalloc(B.TensorList(recs), B.make_hyper("adam"), 1)
    assert e.value.status == -6                      # OPT2S_ERR_TOO_LARGE
    torch.cuda.synchronize()
    assert B.launch_count() == before
    assert not p.any().item()
