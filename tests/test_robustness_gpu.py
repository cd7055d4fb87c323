"""Failure handling and concurrency of the C ABI on a GPU, with faults made
on the host only (nothing here faults, traps or hangs the device):

* an injected out-of-memory during plan creation returns OPT2S_ERR_NO_MEMORY,
  updates nothing, leaves no cache entry behind, and the next call works;
* argument errors leave every tensor untouched (validation precedes any
  launch);
* several host threads stepping their own collections on their own streams
  through the shared plan cache produce the same bits as sequential runs.
"""
import threading

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


def _workload(seed, sizes=(1, 33, 1000, 4097, 70001)):
    return synth.Workload(f"robust_{seed}", list(sizes), ["f32", "f16", "bf16", "f32", "bf16"][:len(sizes)],
                          "ademamix", dict(synth.ADEMAMIX_HYPER, weight_decay=0.01), 3,
                          synth.SEED_BASE + seed, "mixed_magnitude")


def _snapshot(h):
    torch.cuda.synchronize()
    return [tuple(storage_bits(x) for x in (p, s1, s2)) for p, s1, s2 in zip(h.params, h.s1, h.s2)]


@pytest.mark.usefixtures("testing_lib")
def test_injected_out_of_memory_leaves_no_trace():
    B.opt2s_release_cache()
    h = Harness(_workload(80))
    h.load_grads(1)
    before = _snapshot(h)
    n0 = B.launch_count()
    B.testing_fail_allocs(1)
    with pytest.raises(B.Opt2sError) as e:
        h.gpu_step(1)
    assert e.value.status == -3                       # OPT2S_ERR_NO_MEMORY
    assert B.launch_count() == n0
    after = _snapshot(h)
    for x, y in zip(before, after):
        for a, b in zip(x, y):
            assert np.array_equal(a, b)
    B.testing_fail_allocs(1)
    with pytest.raises(B.Opt2sError):
        B.Plan(h.tl, h.w.algo)
    # the failure was not cached: the next call builds the plan and steps
    h.gpu_step(1)
    h.oracle_step(1)
    torch.cuda.synchronize()
    assert h.max_ulps() == {"param": 0, "state1": 0, "state2": 0}


def test_argument_errors_update_nothing():
    h = Harness(_workload(81))
    h.load_grads(1)
    h.gpu_step(1)
    before = _snapshot(h)
    bad = B.make_hyper("ademamix", beta1=1.5, beta3=0.999, alpha=5.0)
    with pytest.raises(B.Opt2sError):
        B.opt2s_step(h.tl, bad, 2)
    with pytest.raises(B.Opt2sError):
        B.opt2s_step(h.tl, h.hyper, 0)
    recs = [(h.params[0].data_ptr(), h.params[0].data_ptr(), h.s1[0].data_ptr(),
             h.s2[0].data_ptr(), 1, B.DTYPES["f32"])]
    with pytest.raises(B.Opt2sError):                 # grad aliases param
        B.opt2s_step(B.TensorList(recs), h.hyper, 2)
    after = _snapshot(h)
    for x, y in zip(before, after):
        for a, b in zip(x, y):
            assert np.array_equal(a, b)


def test_concurrent_threads_and_streams():
    workloads = [_workload(90 + k) for k in range(4)]
    seq = []
    for w in workloads:
        h = Harness(w)
        for t in (1, 2, 3):
            h.load_grads(t)
            h.gpu_step(t)
        seq.append(_snapshot(h))
    B.opt2s_release_cache()
    hs = [Harness(w) for w in workloads]
    grads = {}
    for k, h in enumerate(hs):           # stage every step's grads up front
        for t in (1, 2, 3):
            h.load_grads(t)
            grads[(k, t)] = [g.clone() for g in h.grads]
    torch.cuda.synchronize()
    errors = []

    def worker(k):
        try:
            h = hs[k]
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                for t in (1, 2, 3):
                    for g, src in zip(h.grads, grads[(k, t)]):
                        g.copy_(src)
                    B.opt2s_step(h.tl, h.hyper, t, stream=stream)
            stream.synchronize()
        except Exception as exc:  # pragma: no cover - reported below
            errors.append(exc)

    threads = [threading.Thread(target=worker, args=(k,)) for k in range(len(hs))]
    for th in threads:
        th.start()
    for th in threads:
        th.join(timeout=120)
    assert not errors, errors
    for k, h in enumerate(hs):
        for x, y in zip(seq[k], _snapshot(h)):
            for a, b in zip(x, y):
                assert np.array_equal(a, b)
