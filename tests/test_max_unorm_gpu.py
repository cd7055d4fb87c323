"""The bounded-update-norm step (opt2s_step_max_unorm) against the oracle.

Per tensor, the oracle's oracle_step_f32_max_unorm takes the update norm and
the weight norm as plain binary64 sums in index order; the CUDA path sums in
a fixed tree.  The scale s is rounded to fp32, so the two agree bit for bit
unless a ratio falls within a few binary64 ulp of an fp32 rounding boundary
(never on these inputs): every case asserts 0 ulp on param, state1 and
state2, and untouched gradients.  The bounds are chosen so that every
tensor, some tensors or no tensor is clipped.
"""
import numpy as np
import pytest
import torch

import oracle
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
    yield
    B.opt2s_release_cache()


def _workload(algo, skip, dtypes=("f32", "f16", "bf16"), sizes=None, seed=21):
    sizes = sizes or [1, 2, 31, 33, 255, 257, 1000, 2047, 2048, 2049, 4097, 70_001, 1 << 20]
    hy = dict(synth.ADEMAMIX_HYPER if algo == "ademamix" else synth.ADAM_HYPER, weight_decay=0.01)
    return synth.Workload("unorm", sizes, [dtypes[i % len(dtypes)] for i in range(len(sizes))],
                          algo, hy, 3, synth.SEED_BASE + seed, "mixed_magnitude", skip_zeros=skip)


def _oracle_step(h, step, max_unorm):
    w = h.w
    for i, dt in enumerate(w.dtypes):
        oracle.step_f32_max_unorm(h.h_p[i], h._h_g[i], h.h_s1[i], h.h_s2[i], dtype=dt,
                                  algo=w.algo, step=step, skip_zeros=w.skip_zeros,
                                  max_unorm=max_unorm, **w.hyper)


def _final(h):
    torch.cuda.synchronize()
    return [(storage_bits(p), storage_bits(s1), storage_bits(s2))
            for p, s1, s2 in zip(h.params, h.s1, h.s2)]


def _same(a, b):
    assert len(a) == len(b)
    for i, (x, y) in enumerate(zip(a, b)):
        for k in range(3):
            assert np.array_equal(x[k], y[k]), (i, k)


@pytest.mark.parametrize("max_unorm", [0.01, 1.0, 1e6])
@pytest.mark.parametrize("skip", [False, True])
@pytest.mark.parametrize("algo", ["adam", "ademamix"])
def test_matches_oracle(algo, skip, max_unorm):
    h = Harness(_workload(algo, skip))
    for t in (1, 2, 3):
        h.load_grads(t)
        B.opt2s_step_max_unorm(h.tl, h.hyper, max_unorm, t)
        _oracle_step(h, t, max_unorm)
        torch.cuda.synchronize()
        assert h.max_ulps() == {"param": 0, "state1": 0, "state2": 0}, (t, h.max_ulps())
        assert h.grads_unchanged()


@pytest.mark.parametrize("algo", ["adam", "ademamix"])
def test_bound_above_every_norm_is_the_plain_step(algo):
    w = _workload(algo, True)
    a = Harness(w)
    b = Harness(w)
    for t in (1, 2):
        a.load_grads(t)
        b.load_grads(t)
        B.opt2s_step(a.tl, a.hyper, t)
        B.opt2s_step_max_unorm(b.tl, b.hyper, 1e30, t)
    _same(_final(a), _final(b))


def _run(w, max_unorm, steps=2, layout="separate", pad=0, per_tensor=False):
    h = Harness(w, layout=layout, pad=pad)
    for t in range(1, steps + 1):
        h.load_grads(t)
        if per_tensor:
            for i in range(len(w.sizes)):
                one = B.TensorList.from_tensors([h.params[i]], [h.grads[i]], [h.s1[i]], [h.s2[i]])
                B.opt2s_step_max_unorm(one, h.hyper, max_unorm, t)
        else:
            B.opt2s_step_max_unorm(h.tl, h.hyper, max_unorm, t)
    return _final(h)


@pytest.mark.usefixtures("testing_lib")
def test_geometry_and_alignment_do_not_change_the_result():
    """The norms are summed over fixed 2,048-element blocks in a fixed order,
    so neither the plan's chunk length, the block width, a per-tensor launch
    nor the storage alignment changes a bit."""
    w = _workload("ademamix", True)
    ref = _run(w, 1.0)
    _same(ref, _run(w, 1.0, per_tensor=True))
    _same(ref, _run(w, 1.0, layout="padded", pad=3))
    _same(ref, _run(w, 1.0, layout="packed"))
    for bt, blocks, chunk in ((64, 0, 8), (256, 3, 1000), (128, 1, 0), (512, 0, 4096)):
        B.opt2s_release_cache()
        prev = B.testing_set_chunk_elems(chunk)
        B.testing_set_launch(bt, blocks)
        try:
            got = _run(w, 1.0)
        finally:
            B.testing_set_launch(0, 0)
            B.testing_set_chunk_elems(prev)
            B.opt2s_release_cache()
        _same(ref, got)


def test_large_tensor_matches_oracle():
    """Two tensors of 2^24 fp32 elements (the norm spans 8,192 blocks each)."""
    n = 1 << 24
    w = synth.Workload("unorm_large", [n, n], ["f32", "bf16"], "adam",
                       dict(synth.ADAM_HYPER, weight_decay=0.01), 2, synth.SEED_BASE + 23,
                       "normal", ring_threshold=1 << 26)
    h = Harness(w)
    for t in (1, 2):
        h.load_grads(t)
        B.opt2s_step_max_unorm(h.tl, h.hyper, 0.5, t)
        _oracle_step(h, t, 0.5)
        torch.cuda.synchronize()
        assert h.max_ulps() == {"param": 0, "state1": 0, "state2": 0}, (t, h.max_ulps())


def test_four_launches_per_step():
    h = Harness(_workload("adam", False))
    h.load_grads(1)
    B.opt2s_step_max_unorm(h.tl, h.hyper, 1.0, 1)
    torch.cuda.synchronize()
    before = B.launch_count()
    h.load_grads(2)
    B.opt2s_step_max_unorm(h.tl, h.hyper, 1.0, 2)
    assert B.launch_count() - before == 4


def _params(seed):
    gen = torch.Generator(device="cpu").manual_seed(seed)
    shapes = [(64, 33), (33,), (33, 7), (7,), (1000,), (5, 200), (3000,)]
    dts = [torch.float32, torch.float32, torch.bfloat16, torch.bfloat16, torch.float16,
           torch.float32, torch.bfloat16]
    return [torch.nn.Parameter(torch.randn(s, generator=gen).to(d).cuda()) for s, d in zip(shapes, dts)]


def _set_grads(ps, step):
    gen = torch.Generator(device="cpu").manual_seed(5000 + step)
    for p in ps:
        g = (torch.randn(p.shape, generator=gen) * 1e-2).to(p.dtype).cuda()
        if p.grad is None:
            p.grad = g
        else:
            p.grad.copy_(g)        # flat layout: keep the views


@pytest.mark.parametrize("algo", ["adamw", "ademamix"])
def test_optimizer_max_unorm_matches_oracle_and_flat_layout(algo):
    """optim classes with max_unorm: per parameter the oracle's bounded step;
    the flat layout (one record per parameter into flat buffers, AdEMAMix
    state kept [m1 | m2] per parameter) gives the same bits."""
    from elementwise_optimizer_b200 import optim
    cls = optim.AdEMAMix32bit if algo == "ademamix" else optim.AdamW32bit
    pa, pb = _params(11), _params(11)
    oa = cls(pa, lr=1e-2, max_unorm=0.02)
    ob = cls(pb, lr=1e-2, max_unorm=0.02, flatten=True)
    dt = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}
    bits = {torch.float32: torch.int32, torch.float16: torch.int16, torch.bfloat16: torch.int16}
    hosts = []
    for p in pa:
        n = p.numel()
        hosts.append(dict(p=p.detach().cpu().view(bits[p.dtype]).numpy().reshape(-1).copy(),
                          s1=np.zeros(2 * n if oa.algo == "ademamix" else n, np.float32),
                          s2=np.zeros(n, np.float32)))
    g = oa.param_groups[0]
    for t in range(1, 5):
        _set_grads(pa, t)
        _set_grads(pb, t)
        oa.step()
        ob.step()
        for h, p in zip(hosts, pa):
            gr = p.grad.detach().cpu().view(bits[p.dtype]).numpy().reshape(-1)
            oracle.step_f32_max_unorm(h["p"], gr, h["s1"], h["s2"], dtype=dt[p.dtype],
                                      algo=oa.algo, step=t, lr=g["lr"], beta1=g["betas"][0],
                                      beta2=g["betas"][1], eps=g["eps"], beta3=g["beta3"],
                                      alpha=g["alpha"], weight_decay=g["weight_decay"],
                                      max_unorm=0.02)
    torch.cuda.synchronize()
    for h, a, b in zip(hosts, pa, pb):
        got = a.detach().cpu().view(bits[a.dtype]).numpy().reshape(-1)
        assert np.array_equal(got, h["p"])
        assert torch.equal(a.detach().view(torch.uint8), b.detach().view(torch.uint8))
        sa, sb = oa.state[a], ob.state[b]
        assert np.array_equal(sa["state2"].cpu().numpy(), h["s2"])
        assert torch.equal(sa["state2"].reshape(-1), sb["exp_avg_sq"].reshape(-1))
        n = a.numel()
        assert torch.equal(sa["state1"][:n], sb["exp_avg"].reshape(-1))
        if oa.algo == "ademamix":
            assert torch.equal(sa["state1"][n:], sb["exp_avg_slow"].reshape(-1))
