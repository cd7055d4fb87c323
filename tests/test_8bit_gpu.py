"""The 8-bit blockwise-state step (opt2s_step_8bit) against the oracle.

A collection mixes tensors of at least min_8bit_size = 4,096 elements, whose
state is stored in 8 bits (Dettmers et al. 2022: 2,048-element blocks, one
absmax each, dynamic tree / dynamic quantization maps), with smaller ones
whose state stays fp32 -- the routing of the issue's section "Problem" --
and steps them in one launch.  The oracle steps each tensor on its own
(oracle_step_8bit or oracle_step_f32).  Every case asserts bitwise equality
of params, codes, absmaxes and fp32 states, and untouched gradients.
"""
import numpy as np
import pytest
import torch

import oracle
from elementwise_optimizer_b200 import binding as B
from elementwise_optimizer_b200 import synth
from tests.gpu_support import Harness8, storage_bits, to_device_storage

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


# bias/norm/LoRA-like tensors below the routing threshold, the threshold's
# neighbours, ragged and whole 8-bit blocks, and a larger weight
SIZES = [1, 64, 100, 333, 512, 1000, 1024, 4095, 4096, 4097, 6144, 8191, 70_001, 1 << 20]


def _workload(algo, skip, wd=0.01, grad_kind="mixed_magnitude", seed=51, sizes=SIZES):
    dtypes = [("f32", "bf16", "f16")[i % 3] for i in range(len(sizes))]
    hy = dict(synth.ADEMAMIX_HYPER if algo == "ademamix" else synth.ADAM_HYPER, weight_decay=wd)
    return synth.Workload("eightbit", sizes, dtypes, algo, hy, 3, synth.SEED_BASE + seed, grad_kind,
                          skip_zeros=skip)


@pytest.mark.parametrize("layout", ["separate", "packed"])
@pytest.mark.parametrize("skip", [False, True])
@pytest.mark.parametrize("algo", ["adam", "ademamix"])
def test_matches_oracle(algo, skip, layout):
    h = Harness8(_workload(algo, skip), layout=layout)
    assert 8 in h.bits and 32 in h.bits
    for t in (1, 2, 3):
        h.step_both(t)
        assert h.mismatches() == [], t
        assert h.grads_unchanged()


@pytest.mark.parametrize("algo", ["adam", "ademamix"])
def test_normal_gradients_many_steps(algo):
    """Ten steps of N(0, 1e-2) gradients: the quantized state evolves over
    many requantizations and stays bitwise on the oracle's."""
    h = Harness8(_workload(algo, False, grad_kind="normal", seed=52,
                           sizes=[300, 4096, 10_000, 65_536 + 5]))
    for t in range(1, 11):
        h.step_both(t)
    assert h.mismatches() == []


def test_one_launch_for_a_mixed_collection():
    h = Harness8(_workload("adam", False))
    h.load_grads(1)
    h.gpu_step(1)
    torch.cuda.synchronize()
    before = B.launch_count()
    h.load_grads(2)
    h.gpu_step(2)
    assert B.launch_count() - before == 1


def test_per_tensor_launches_equal_one_launch():
    """Stepping each tensor by its own call gives the bits of one call for
    the whole collection (each block is stepped by one CTA either way)."""
    w = _workload("ademamix", True, seed=53)
    a = Harness8(w)
    b = Harness8(w)
    for t in (1, 2):
        a.load_grads(t)
        b.load_grads(t)
        a.gpu_step(t)
        for i in range(len(w.sizes)):
            one = B.TensorList8.from_tensors([b.params[i]], [b.grads[i]], [b.s1[i]], [b.s2[i]],
                                             [b.a1[i]], [b.a2[i]])
            B.opt2s_step_8bit(one, b.hyper, t)
    torch.cuda.synchronize()
    for i in range(len(w.sizes)):
        for x, y in ((a.params[i], b.params[i]), (a.s1[i], b.s1[i]), (a.s2[i], b.s2[i])):
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), i
        if a.a1[i] is not None:
            assert torch.equal(a.a1[i], b.a1[i]) and torch.equal(a.a2[i], b.a2[i])


def test_all_32bit_collection_equals_opt2s_step():
    """With every tensor routed to fp32 state, the 8-bit entry point gives
    opt2s_step's bits (the same element arithmetic)."""
    from tests.gpu_support import Harness
    w = _workload("adam", False, sizes=[1, 64, 1000, 4095, 70_001], seed=54)
    a = Harness8(w, min_8bit_size=1 << 30)
    b = Harness(w)
    for t in (1, 2):
        a.load_grads(t)
        b.load_grads(t)
        a.gpu_step(t)
        b.gpu_step(t)
    torch.cuda.synchronize()
    for i in range(len(w.sizes)):
        assert np.array_equal(storage_bits(a.params[i]), storage_bits(b.params[i]))
        assert np.array_equal(storage_bits(a.s1[i]), storage_bits(b.s1[i]))
        assert np.array_equal(storage_bits(a.s2[i]), storage_bits(b.s2[i]))


def test_large_tensor_sampled_blocks():
    """One 2^24-element bf16 AdEMAMix tensor with 8-bit state: blocks are
    independent, so sampled blocks (first, last, and every 97th) are checked
    against the oracle stepping just those blocks."""
    n = 1 << 24
    nb = n // 2048
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev).manual_seed(55)
    p = (torch.randn(n, device=dev, generator=gen)).to(torch.bfloat16)
    q1 = torch.zeros(2 * n, dtype=torch.uint8, device=dev)
    q2 = torch.zeros(n, dtype=torch.uint8, device=dev)
    a1 = torch.zeros(2 * nb, device=dev)
    a2 = torch.zeros(nb, device=dev)
    h = B.make_hyper("ademamix", weight_decay=0.1, beta3=0.9999, alpha=5.0)
    hy = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, beta3=0.9999, alpha=5.0, weight_decay=0.1)
    sample = np.unique(np.concatenate([np.arange(0, nb, 97), [nb - 1]]))
    bits = lambda t: t.view(torch.int16).cpu().numpy().view(np.uint16)
    hp = bits(p)[np.concatenate([np.arange(b * 2048, (b + 1) * 2048) for b in sample])]
    k = sample.size
    hq1, hq2 = np.zeros(2 * k * 2048, np.uint8), np.zeros(k * 2048, np.uint8)
    ha1, ha2 = np.zeros(2 * k, np.float32), np.zeros(k, np.float32)
    for t in (1, 2, 3):
        g = (torch.randn(n, device=dev, generator=gen) * 1e-2).to(torch.bfloat16)
        tl = B.TensorList8.from_tensors([p], [g], [q1], [q2], [a1], [a2])
        B.opt2s_step_8bit(tl, h, t)
        hg = bits(g)
        # the sampled blocks, stepped by the oracle one block at a time
        for j, b in enumerate(sample):
            sl = slice(b * 2048, (b + 1) * 2048)
            js = slice(j * 2048, (j + 1) * 2048)
            m1 = hq1[2 * j * 2048:(2 * j + 1) * 2048]
            m2 = hq1[(2 * j + 1) * 2048:(2 * j + 2) * 2048]
            qq1 = np.concatenate([m1, m2])
            aa1 = np.array([ha1[2 * j], ha1[2 * j + 1]], np.float32)
            aa2 = ha2[j:j + 1].copy()
            pp = hp[js].copy()
            qq2 = hq2[js].copy()
            oracle.step_8bit(pp, hg[sl].copy(), qq1, qq2, aa1, aa2, dtype="bf16", algo="ademamix",
                             step=t, **hy)
            hp[js], hq2[js] = pp, qq2
            m1[:], m2[:] = qq1[:2048], qq1[2048:]
            ha1[2 * j], ha1[2 * j + 1], ha2[j] = aa1[0], aa1[1], aa2[0]
    torch.cuda.synchronize()
    idx = np.concatenate([np.arange(b * 2048, (b + 1) * 2048) for b in sample])
    ti = torch.from_numpy(idx).to(dev)
    assert np.array_equal(bits(p[ti]), hp)
    assert np.array_equal(q2[ti].cpu().numpy(), hq2)
    got1 = np.concatenate([np.concatenate([q1[:n][b * 2048:(b + 1) * 2048].cpu().numpy(),
                                           q1[n:][b * 2048:(b + 1) * 2048].cpu().numpy()])
                           for b in sample])
    assert np.array_equal(got1, hq1)
    ts = torch.from_numpy(sample).to(dev)
    assert np.array_equal(a2[ts].cpu().numpy(), ha2)
    assert np.array_equal(torch.stack([a1[:nb][ts], a1[nb:][ts]], 1).reshape(-1).cpu().numpy(), ha1)


def test_rejects_bad_records_before_any_work():
    w = _workload("adam", False, sizes=[64, 5000], seed=56)
    h = Harness8(w)
    before = [storage_bits(p) for p in h.params]
    p, g = h.params[1], h.grads[1]
    bad = [
        (p.data_ptr(), g.data_ptr(), h.s1[1].data_ptr(), h.s2[1].data_ptr(), 0, 0, 5000,
         B.DTYPES["bf16"], 8),                                    # 8-bit without absmax
        (p.data_ptr(), g.data_ptr(), h.s1[1].data_ptr(), h.s2[1].data_ptr(),
         h.a1[1].data_ptr(), h.a2[1].data_ptr(), 5000, B.DTYPES["bf16"], 16),   # bad state_bits
        (p.data_ptr(), g.data_ptr(), h.s1[1].data_ptr(), h.s1[1].data_ptr(),
         h.a1[1].data_ptr(), h.a2[1].data_ptr(), 5000, B.DTYPES["bf16"], 8),    # codes overlap
        (p.data_ptr(), g.data_ptr(), h.s1[1].data_ptr(), h.s2[1].data_ptr(),
         h.a1[1].data_ptr(), h.a1[1].data_ptr(), 5000, B.DTYPES["bf16"], 8),    # absmax overlap
    ]
    for rec, status in zip(bad, (-1, -1, -2, -2)):
        with pytest.raises(B.Opt2sError) as e:
            h.load_grads(1)
            B.opt2s_step_8bit(B.TensorList8([rec]), h.hyper, 1)
        assert e.value.status == status, rec
    torch.cuda.synchronize()
    for x, q in zip(before, h.params):
        assert np.array_equal(x, storage_bits(q))
