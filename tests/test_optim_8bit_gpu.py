"""The torch.optim front end with 8-bit blockwise state (optim.AdamW8bit,
Adam8bit, AdEMAMix8bit): parameters of at least min_8bit_size elements keep
uint8 codes and per-block absmaxes, smaller ones fp32 state, all of a group
in one launch; every step must equal the oracle's bit for bit.  Also
state_dict round trips, which must keep the state's own dtypes (torch.optim's
loader alone would cast it to each parameter's dtype)."""
import copy

import numpy as np
import pytest
import torch

import oracle
from elementwise_optimizer_b200 import binding as B
from elementwise_optimizer_b200 import optim

pytestmark = pytest.mark.gpu

DT = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}
BITS = {torch.float32: torch.int32, torch.float16: torch.int16, torch.bfloat16: torch.int16}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from elementwise_optimizer_b200 import _build
    _build.build()


def _params(seed):
    """Bias/norm-like tensors below the routing threshold, the threshold's
    neighbours, and tensors of several blocks with a ragged last block."""
    gen = torch.Generator(device="cpu").manual_seed(seed)
    shapes = [(33,), (64, 63), (4095,), (4096,), (3, 2049), (1000, 9), (20000,)]
    dts = [torch.float32, torch.bfloat16, torch.float16, torch.float32, torch.bfloat16, torch.float32,
           torch.float16]
    return [torch.nn.Parameter(torch.randn(s, generator=gen).to(d).cuda()) for s, d in zip(shapes, dts)]


def _bits(t):
    return t.detach().cpu().view(BITS[t.dtype]).numpy().reshape(-1).copy()


def _grads(ps, gen):
    for p in ps:
        p.grad = (torch.randn(p.shape, generator=gen) * 1e-2).to(p.dtype).cuda()


def _host_mirror(ps, algo, min_8bit_size):
    two = algo == "ademamix"
    out = []
    for p in ps:
        n = p.numel()
        h = {"p": _bits(p), "bits": B.state_bits_for(n, min_8bit_size)}
        if h["bits"] == 8:
            nb = (n + B.BLOCK8 - 1) // B.BLOCK8
            h["s1"] = np.full((2 if two else 1) * n, 127, np.uint8)     # the code of 0, signed map
            h["s2"] = np.zeros(n, np.uint8)                             # and unsigned map
            h["a1"] = np.zeros((2 if two else 1) * nb, np.float32)
            h["a2"] = np.zeros(nb, np.float32)
        else:
            h["s1"] = np.zeros((2 if two else 1) * n, np.float32)
            h["s2"] = np.zeros(n, np.float32)
        out.append(h)
    return out


def _oracle_step(hosts, ps, algo, t, hy):
    for h, p in zip(hosts, ps):
        g = _bits(p.grad)
        if h["bits"] == 8:
            oracle.step_8bit(h["p"], g, h["s1"], h["s2"], h["a1"], h["a2"], dtype=DT[p.dtype], algo=algo,
                             step=t, **hy)
        else:
            oracle.step_f32(h["p"], g, h["s1"], h["s2"], dtype=DT[p.dtype], algo=algo, step=t, **hy)


def _assert_equal(opt, ps, hosts):
    torch.cuda.synchronize()
    for i, (h, p) in enumerate(zip(hosts, ps)):
        st = opt.state[p]
        assert np.array_equal(_bits(p), h["p"]), (i, "param")
        s1, s2 = st["state1"].cpu().numpy(), st["state2"].cpu().numpy()
        if h["bits"] == 8:
            assert st["state1"].dtype == torch.uint8 and st["state2"].dtype == torch.uint8
            assert np.array_equal(s1, h["s1"]) and np.array_equal(s2, h["s2"]), (i, "codes")
            assert np.array_equal(st["absmax1"].cpu().numpy().view(np.uint32), h["a1"].view(np.uint32)), i
            assert np.array_equal(st["absmax2"].cpu().numpy().view(np.uint32), h["a2"].view(np.uint32)), i
        else:
            assert st["state1"].dtype == torch.float32
            assert np.array_equal(s1.view(np.uint32), h["s1"].view(np.uint32)), (i, "state1")
            assert np.array_equal(s2.view(np.uint32), h["s2"].view(np.uint32)), (i, "state2")


@pytest.mark.parametrize("cls,algo", [(optim.AdamW8bit, "adam"), (optim.Adam8bit, "adam"),
                                      (optim.AdEMAMix8bit, "ademamix")])
def test_8bit_optimizer_matches_the_oracle(cls, algo):
    ps = _params(31)
    opt = cls(ps, lr=3e-3)
    g = opt.param_groups[0]
    hy = dict(lr=g["lr"], beta1=g["betas"][0], beta2=g["betas"][1], eps=g["eps"],
              weight_decay=g["weight_decay"])
    if algo == "ademamix":
        hy.update(beta3=g["beta3"], alpha=g["alpha"])
    hosts = _host_mirror(ps, algo, opt.min_8bit_size)
    assert [h["bits"] for h in hosts] == [32, 32, 32, 8, 8, 8, 8]
    gen = torch.Generator(device="cpu").manual_seed(7)
    for t in range(1, 5):
        _grads(ps, gen)
        before = B.launch_count()
        opt.step()
        assert B.launch_count() - before == 1          # the whole group, mixed state, one launch
        _oracle_step(hosts, ps, algo, t, hy)
    _assert_equal(opt, ps, hosts)


def test_min_8bit_size_routes_the_state():
    ps = _params(33)
    opt = optim.AdamW8bit(ps, min_8bit_size=2049)
    _grads(ps, torch.Generator(device="cpu").manual_seed(3))
    opt.step()
    kinds = [opt.state[p]["state1"].dtype for p in ps]
    assert kinds == [torch.float32, torch.uint8, torch.uint8, torch.uint8, torch.uint8, torch.uint8,
                     torch.uint8]
    with pytest.raises(ValueError):
        optim.AdamW8bit(ps, min_8bit_size=0)


@pytest.mark.parametrize("make", [lambda ps: optim.AdamW8bit(ps, lr=3e-3),
                                  lambda ps: optim.AdEMAMix8bit(ps, lr=3e-3),
                                  lambda ps: optim.AdamW32bit(ps, lr=3e-3)])
def test_state_dict_round_trip_keeps_state_bits(make):
    """Two steps, save; a fresh optimizer over copies of the parameters loads
    the state; one more step on both gives the same bits everywhere, and the
    loaded state keeps its dtypes (uint8 codes, fp32 moments of bf16/fp16
    parameters)."""
    ps = _params(35)
    opt = make(ps)
    gen = torch.Generator(device="cpu").manual_seed(9)
    for _ in range(2):
        _grads(ps, gen)
        opt.step()
    saved = copy.deepcopy(opt.state_dict())
    qs = [torch.nn.Parameter(p.detach().clone()) for p in ps]
    opt2 = make(qs)
    opt2.load_state_dict(saved)
    for p, q in zip(ps, qs):
        for k, v in opt.state[p].items():
            if isinstance(v, torch.Tensor) and k != "step":
                assert opt2.state[q][k].dtype == v.dtype, k
    _grads(ps, gen)
    for p, q in zip(ps, qs):
        q.grad = p.grad.clone()
    opt.step()
    opt2.step()
    torch.cuda.synchronize()
    for p, q in zip(ps, qs):
        assert np.array_equal(_bits(p), _bits(q))
        for k, v in opt.state[p].items():
            if isinstance(v, torch.Tensor) and k != "step":
                assert torch.equal(v.view(torch.uint8), opt2.state[q][k].view(torch.uint8)), k


@pytest.mark.parametrize("cls", [optim.AdamW32bit, optim.AdEMAMix32bit])
def test_flat_layout_state_dict_round_trip(cls):
    """With flatten=True the steps read the flat state buffers: a loaded
    state must land in them (and in the step count), not only in the state
    dict, so that the next step continues exactly."""
    ps = _params(37)
    opt = cls(ps, lr=3e-3, flatten=True)
    gen = torch.Generator(device="cpu").manual_seed(11)

    def grads_in_place(params, values=None):
        out = []
        for i, p in enumerate(params):
            v = values[i] if values is not None else (torch.randn(p.shape, generator=gen) * 1e-2).to(p.dtype)
            p.grad.copy_(v.cuda())              # flat layout: gradients stay views of one buffer
            out.append(v)
        return out

    for _ in range(3):
        grads_in_place(ps)
        opt.step()
    saved = copy.deepcopy(opt.state_dict())
    qs = [torch.nn.Parameter(p.detach().clone()) for p in ps]
    opt2 = cls(qs, lr=3e-3, flatten=True)
    opt2.load_state_dict(saved)
    vals = grads_in_place(ps)
    grads_in_place(qs, vals)
    opt.step()
    opt2.step()
    torch.cuda.synchronize()
    for p, q in zip(ps, qs):
        assert np.array_equal(_bits(p), _bits(q))
        for k, v in opt.state[p].items():
            if isinstance(v, torch.Tensor) and k != "step":
                assert torch.equal(v, opt2.state[q][k]), k
        assert int(opt2.state[q]["step"]) == 4
