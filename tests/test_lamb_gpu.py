"""The LAMB step (opt2s_step_lamb) against the oracle.

Per tensor, the oracle's oracle_step_f32_lamb takes the weight norm and the
norm of the decayed direction w = u + weight_decay*p as plain binary64 sums
in index order; the CUDA path sums in a fixed tree of binary64 sums.  The
trust ratio is rounded to fp32, so the two agree bit for bit unless a ratio
falls within a few binary64 ulp of an fp32 rounding boundary (never on these
inputs): every case asserts 0 ulp on param, state1 and state2, and untouched
gradients.
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


def _workload(skip, wd, dtypes=("f32", "f16", "bf16"), sizes=None, seed=41):
    sizes = sizes or [1, 2, 31, 33, 255, 257, 1000, 2047, 2048, 2049, 4097, 70_001, 1 << 20]
    hy = dict(synth.ADAM_HYPER, weight_decay=wd)
    return synth.Workload("lamb", sizes, [dtypes[i % len(dtypes)] for i in range(len(sizes))],
                          "adam", hy, 3, synth.SEED_BASE + seed, "mixed_magnitude", skip_zeros=skip)


def _oracle_step(h, step):
    w = h.w
    hy = {k: v for k, v in w.hyper.items() if k not in ("beta3", "alpha")}
    for i, dt in enumerate(w.dtypes):
        oracle.step_f32_lamb(h.h_p[i], h._h_g[i], h.h_s1[i], h.h_s2[i], dtype=dt, step=step,
                             skip_zeros=w.skip_zeros, **hy)


def _final(h):
    torch.cuda.synchronize()
    return [(storage_bits(p), storage_bits(s1), storage_bits(s2))
            for p, s1, s2 in zip(h.params, h.s1, h.s2)]


def _same(a, b):
    assert len(a) == len(b)
    for i, (x, y) in enumerate(zip(a, b)):
        for k in range(3):
            assert np.array_equal(x[k], y[k]), (i, k)


@pytest.mark.parametrize("wd", [0.0, 0.01, 0.3])
@pytest.mark.parametrize("skip", [False, True])
def test_matches_oracle(skip, wd):
    h = Harness(_workload(skip, wd))
    for t in (1, 2, 3):
        h.load_grads(t)
        B.opt2s_step_lamb(h.tl, h.hyper, t)
        _oracle_step(h, t)
        torch.cuda.synchronize()
        assert h.max_ulps() == {"param": 0, "state1": 0, "state2": 0}, (t, h.max_ulps())
        assert h.grads_unchanged()


def test_zero_weights_move_like_the_plain_step():
    """A zero-initialised tensor has weight norm 0 and takes trust ratio 1:
    its first LAMB step is the plain Adam step without decay, bit for bit."""
    w = synth.Workload("lamb_zero", [4097, 33, 70_001], ["f32", "bf16", "f16"], "adam",
                       dict(synth.ADAM_HYPER), 2, synth.SEED_BASE + 42, "mixed_magnitude")
    a = Harness(w)
    b = Harness(w)
    for h in (a, b):
        for p in h.params:
            p.zero_()
    a.load_grads(1)
    b.load_grads(1)
    B.opt2s_step_lamb(a.tl, B.make_hyper("adam", weight_decay=0.5, **{
        k: v for k, v in w.hyper.items() if k != "weight_decay"}), 1)
    B.opt2s_step(b.tl, b.hyper, 1)
    _same(_final(a), _final(b))


def _run(w, steps=2, layout="separate", pad=0, per_tensor=False):
    h = Harness(w, layout=layout, pad=pad)
    for t in range(1, steps + 1):
        h.load_grads(t)
        if per_tensor:
            for i in range(len(w.sizes)):
                one = B.TensorList.from_tensors([h.params[i]], [h.grads[i]], [h.s1[i]], [h.s2[i]])
                B.opt2s_step_lamb(one, h.hyper, t)
        else:
            B.opt2s_step_lamb(h.tl, h.hyper, t)
    return _final(h)


@pytest.mark.usefixtures("testing_lib")
def test_geometry_and_alignment_do_not_change_the_result():
    """The norms are summed over fixed 2,048-element blocks in a fixed order,
    so neither the plan's chunk length, the block width, a per-tensor launch
    nor the storage alignment changes a bit."""
    w = _workload(True, 0.05)
    ref = _run(w)
    _same(ref, _run(w, per_tensor=True))
    _same(ref, _run(w, layout="padded", pad=3))
    _same(ref, _run(w, layout="packed"))
    for bt, blocks, chunk in ((64, 0, 8), (256, 3, 1000), (128, 1, 0), (512, 0, 4096)):
        B.opt2s_release_cache()
        prev = B.testing_set_chunk_elems(chunk)
        B.testing_set_launch(bt, blocks)
        try:
            got = _run(w)
        finally:
            B.testing_set_launch(0, 0)
            B.testing_set_chunk_elems(prev)
            B.opt2s_release_cache()
        _same(ref, got)


def test_large_tensor_matches_oracle():
    """Two tensors of 2^24 elements (the norms span 8,192 blocks each)."""
    n = 1 << 24
    w = synth.Workload("lamb_large", [n, n], ["f32", "bf16"], "adam",
                       dict(synth.ADAM_HYPER, weight_decay=0.01), 2, synth.SEED_BASE + 43,
                       "normal", ring_threshold=1 << 26)
    h = Harness(w)
    for t in (1, 2):
        h.load_grads(t)
        B.opt2s_step_lamb(h.tl, h.hyper, t)
        _oracle_step(h, t)
        torch.cuda.synchronize()
        assert h.max_ulps() == {"param": 0, "state1": 0, "state2": 0}, (t, h.max_ulps())


def test_lamb_and_max_unorm_share_the_plan_and_launch_four_kernels():
    h = Harness(_workload(False, 0.01))
    h.load_grads(1)
    B.opt2s_step_max_unorm(h.tl, h.hyper, 1.0, 1)
    torch.cuda.synchronize()
    before = B.launch_count()
    h.load_grads(2)
    B.opt2s_step_lamb(h.tl, h.hyper, 2)
    assert B.launch_count() - before == 4


def test_ademamix_is_rejected_before_any_work():
    w = _workload(False, 0.01)
    h = Harness(w)
    before = [storage_bits(p) for p in h.params]
    bad = B.make_hyper("ademamix", beta3=0.9999, alpha=5.0)
    with pytest.raises(B.Opt2sError) as e:
        B.opt2s_step_lamb(h.tl, bad, 1)
    assert e.value.status == -1
    torch.cuda.synchronize()
    for x, p in zip(before, h.params):
        assert np.array_equal(x, storage_bits(p))


def _params(seed):
    gen = torch.Generator(device="cpu").manual_seed(seed)
    shapes = [(64, 33), (33,), (33, 7), (7,), (1000,), (5, 200), (3000,)]
    dts = [torch.float32, torch.float32, torch.bfloat16, torch.bfloat16, torch.float16,
           torch.float32, torch.bfloat16]
    return [torch.nn.Parameter(torch.randn(s, generator=gen).to(d).cuda()) for s, d in zip(shapes, dts)]


def _set_grads(ps, step):
    gen = torch.Generator(device="cpu").manual_seed(7000 + step)
    for p in ps:
        g = (torch.randn(p.shape, generator=gen) * 1e-2).to(p.dtype).cuda()
        if p.grad is None:
            p.grad = g
        else:
            p.grad.copy_(g)        # flat layout: keep the views


def test_optimizer_lamb_matches_oracle_and_flat_layout():
    """LAMB32bit: per parameter the oracle's LAMB step; the flat layout (one
    record per parameter into flat buffers) gives the same bits."""
    from elementwise_optimizer_b200 import optim
    pa, pb = _params(13), _params(13)
    oa = optim.LAMB32bit(pa, lr=1e-2, weight_decay=0.05)
    ob = optim.LAMB32bit(pb, lr=1e-2, weight_decay=0.05, flatten=True)
    dt = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}
    bits = {torch.float32: torch.int32, torch.float16: torch.int16, torch.bfloat16: torch.int16}
    hosts = []
    for p in pa:
        n = p.numel()
        hosts.append(dict(p=p.detach().cpu().view(bits[p.dtype]).numpy().reshape(-1).copy(),
                          s1=np.zeros(n, np.float32), s2=np.zeros(n, np.float32)))
    g = oa.param_groups[0]
    for t in range(1, 5):
        _set_grads(pa, t)
        _set_grads(pb, t)
        oa.step()
        ob.step()
        for h, p in zip(hosts, pa):
            gr = p.grad.detach().cpu().view(bits[p.dtype]).numpy().reshape(-1)
            oracle.step_f32_lamb(h["p"], gr, h["s1"], h["s2"], dtype=dt[p.dtype], step=t,
                                 lr=g["lr"], beta1=g["betas"][0], beta2=g["betas"][1],
                                 eps=g["eps"], weight_decay=g["weight_decay"])
    torch.cuda.synchronize()
    for h, a, b in zip(hosts, pa, pb):
        got = a.detach().cpu().view(bits[a.dtype]).numpy().reshape(-1)
        assert np.array_equal(got, h["p"])
        assert torch.equal(a.detach().view(torch.uint8), b.detach().view(torch.uint8))
        sa, sb = oa.state[a], ob.state[b]
        assert np.array_equal(sa["state2"].cpu().numpy(), h["s2"])
        assert torch.equal(sa["state2"].reshape(-1), sb["exp_avg_sq"].reshape(-1))
        assert torch.equal(sa["state1"], sb["exp_avg"].reshape(-1))
