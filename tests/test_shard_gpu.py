"""The fused sharded step on one GPU with emulated ranks.

Each emulated rank q owns a flat param buffer and a flat grad buffer on the
same GPU; the step of rank r reads every rank's gradient, updates its shard
and writes every rank's param buffer.  Ranks never wait on one another, so
launching the ranks' steps one after another is a faithful emulation (their
writes are disjoint and grads are read only).  The result must equal, bit for
bit, the CPU oracle stepping the whole buffer with the rank-order mean of the
gradients -- and with one rank, the plain opt2s_step.
"""
import numpy as np
import pytest
import torch

from elementwise_optimizer_b200 import binding as B
from elementwise_optimizer_b200 import shard, synth
from tests.gpu_support import TORCH, storage_bits, to_device_storage

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from elementwise_optimizer_b200 import _build
    _build.build()
    B.lib()


HYPER = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, beta3=0.999, alpha=5.0, weight_decay=0.01)


def _setup(world, n, dtype, algo, offset=0):
    p0 = synth.normal(synth.SEED_BASE + 60, (n,), n, 1.0)
    p0 = synth.from_storage(synth.to_storage(p0, dtype), dtype)
    bufs = [to_device_storage(np.concatenate([np.zeros(offset, np.float32), p0]), dtype, "cuda")
            for _ in range(world)]
    params = [b[offset:] for b in bufs]
    gbufs = [torch.empty(n + offset, dtype=TORCH[dtype], device="cuda") for _ in range(world)]
    grads = [g[offset:] for g in gbufs]
    steps = [shard.ShardedStep(params, grads, r, algo) for r in range(world)]
    return p0, bufs, params, gbufs, grads, steps


def _grad_values(q, t, n, dtype):
    g = synth.mixed_magnitude(synth.SEED_BASE + 61, (q, t, n), n, zero_frac=0.05)
    return synth.from_storage(synth.to_storage(g, dtype), dtype)


@pytest.mark.parametrize("offset", [0, 1])
@pytest.mark.parametrize("algo,skip", [("adam", False), ("ademamix", True)])
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("world,n", [(1, 100_003), (2, 1_000_003), (3, 100_003), (8, 1_000_003),
                                     (8, 37)])
def test_sharded_step_equals_oracle(world, n, dtype, algo, skip, offset):
    import oracle
    p0, bufs, params, gbufs, grads, steps = _setup(world, n, dtype, algo, offset)
    hyper = B.make_hyper(algo, skip_zeros=skip, **HYPER)
    hp = synth.to_storage(p0, dtype)
    hs1 = np.zeros(2 * n if algo == "ademamix" else n, np.float32)
    hs2 = np.zeros(n, np.float32)
    for t in range(1, 4):
        host_grads = []
        for q in range(world):
            gv = _grad_values(q, t, n, dtype)
            grads[q].copy_(to_device_storage(gv, dtype, "cuda"))
            host_grads.append(synth.to_storage(gv, dtype))
        for r in range(world):                      # emulated ranks, one after another
            steps[r].step(hyper, t)
        avg = oracle.average_grads(host_grads, dtype)
        oracle.step_f32_fgrad(hp, avg, hs1, hs2, dtype=dtype, algo=algo, step=t,
                              skip_zeros=skip, **HYPER)
    torch.cuda.synchronize()
    want = hp.view(np.uint32 if dtype == "f32" else np.uint16)
    for q in range(world):
        assert np.array_equal(storage_bits(params[q]), want), q
        if offset:
            assert np.array_equal(storage_bits(bufs[q][:offset]), np.zeros(offset, want.dtype))
    for r, st in enumerate(steps):
        a, k = st.start, st.length
        m = hs1[a:a + k]
        if algo == "ademamix":
            m = np.concatenate([m, hs1[n + a:n + a + k]])
        assert np.array_equal(st.state1.cpu().numpy(), m), r
        assert np.array_equal(st.state2.cpu().numpy(), hs2[a:a + k]), r


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_one_rank_equals_the_plain_step(dtype):
    n = 300_001
    p0, bufs, params, gbufs, grads, steps = _setup(1, n, dtype, "ademamix")
    hyper = B.make_hyper("ademamix", **HYPER)
    ref_p = params[0].clone()
    ref_g = grads[0]
    s1 = torch.zeros(2 * n, device="cuda")
    s2 = torch.zeros(n, device="cuda")
    tl = B.TensorList.from_tensors([ref_p], [ref_g], [s1], [s2])
    for t in range(1, 4):
        grads[0].copy_(to_device_storage(_grad_values(0, t, n, dtype), dtype, "cuda"))
        steps[0].step(hyper, t)
        B.opt2s_step(tl, hyper, t)
    torch.cuda.synchronize()
    assert torch.equal(params[0].view(torch.uint8), ref_p.view(torch.uint8))
    assert torch.equal(steps[0].state1, s1) and torch.equal(steps[0].state2, s2)
