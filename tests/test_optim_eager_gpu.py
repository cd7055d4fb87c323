"""The eager optimizer path without flattening: the group's launch records
are refreshed in place every step (csrc/opt2s_marshal.cpp) and the results
must stay bitwise the oracle's whatever happens to the tensors between
steps -- gradients zeroed in place, replaced by new tensors, dropped for one
step, or a parameter's storage swapped with ``p.data = ...``."""
import numpy as np
import pytest
import torch

import oracle
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
    gen = torch.Generator(device="cpu").manual_seed(seed)
    shapes = [(64, 33), (33,), (1000,), (7,), (4096,), (5, 200)]
    dts = [torch.float32, torch.bfloat16, torch.float16, torch.float32, torch.bfloat16, torch.float32]
    return [torch.nn.Parameter(torch.randn(s, generator=gen).to(d).cuda()) for s, d in zip(shapes, dts)]


def _bits(t):
    return t.detach().cpu().view(BITS[t.dtype]).numpy().reshape(-1).copy()


def test_marshalling_helper_is_built():
    assert optim._marshal_module() is not None


@pytest.mark.parametrize("mode", ["in_place", "replace", "drop_one", "swap_data"])
def test_eager_steps_follow_the_tensors(mode):
    ps = _params(21)
    opt = optim.AdamW32bit(ps, lr=1e-2, weight_decay=0.05)
    g = opt.param_groups[0]
    host = [dict(p=_bits(p), s1=np.zeros(p.numel(), np.float32), s2=np.zeros(p.numel(), np.float32))
            for p in ps]
    gen = torch.Generator(device="cpu").manual_seed(5)
    for t in range(1, 6):
        for i, p in enumerate(ps):
            grad = (torch.randn(p.shape, generator=gen) * 1e-2).to(p.dtype).cuda()
            if mode == "in_place" and p.grad is not None:
                p.grad.copy_(grad)                     # same tensor, same address
            else:
                p.grad = grad                          # a new tensor
        if mode == "drop_one" and t == 3:
            ps[2].grad = None                          # not stepped this time
        if mode == "swap_data" and t == 3:
            with torch.no_grad():
                fresh = ps[0].detach().clone()         # same values, new storage
            ps[0].data = fresh
        opt.step()
        for i, (h, p) in enumerate(zip(host, ps)):
            if p.grad is None:
                continue
            # a group shares one step count (one launch, one set of bias
            # corrections): a parameter left out of a step still counts it
            oracle.step_f32(h["p"], _bits(p.grad), h["s1"], h["s2"], dtype=DT[p.dtype], algo="adam",
                            step=t, lr=g["lr"], beta1=g["betas"][0], beta2=g["betas"][1],
                            eps=g["eps"], weight_decay=g["weight_decay"])
        if mode == "in_place":
            opt.zero_grad()                            # in place by default
            assert all(p.grad is not None and not p.grad.any() for p in ps)
    torch.cuda.synchronize()
    for h, p in zip(host, ps):
        assert np.array_equal(_bits(p), h["p"])
        st = opt.state[p]
        assert np.array_equal(st["state1"].cpu().numpy(), h["s1"])
        assert np.array_equal(st["state2"].cpu().numpy(), h["s2"])


def test_flat_layout_refuses_replaced_gradients():
    """flatten=True steps its flat gradient buffer; gradients set to None and
    made anew by a backward would leave it stale, so the step refuses.  New
    groups after flattening are refused too."""
    ps = _params(23)
    opt = optim.AdamW32bit(ps, lr=1e-3, flatten=True)
    for p in ps:
        p.grad.normal_()
    opt.step()                                   # gradients are the flat views: fine
    for p in ps:
        p.grad = None                            # what module.zero_grad() does by default
    for p in ps:
        p.grad = torch.ones_like(p)              # a backward makes new tensors
    with pytest.raises(RuntimeError):
        opt.step()
    with pytest.raises(ValueError):
        opt.add_param_group({"params": [torch.nn.Parameter(torch.zeros(4, device="cuda"))]})
