"""Steps that a captured CUDA graph can replay, and the torch.optim front end.

The bitsandbytes issue "Investigate a 256-thread SM103 path for small 32-bit
optimizer tensors" asks that the launch path stay safe for CUDA graph capture
(section "Scope") and includes a graph-compatible direct-call collection
(section "B300 benchmark and acceptance").  opt2s_plan_step_table reads the
per-step scalars from a device table at a device index, so each replay of a
captured step performs the next step; these tests require its results to be
bitwise equal to eager opt2s_step calls (and so to the oracle).
"""
import numpy as np
import pytest
import torch

from elementwise_optimizer_b200 import binding as B
from elementwise_optimizer_b200 import optim, synth
from tests.gpu_support import Harness, storage_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from elementwise_optimizer_b200 import _build
    _build.build()
    B.lib()


def _workload(algo="ademamix", skip=True):
    sizes = [1, 33, 640, 4097, 100_003]
    dtypes = ["f32", "f16", "bf16", "f32", "bf16"]
    hyper = dict(synth.ADEMAMIX_HYPER if algo == "ademamix" else synth.ADAM_HYPER,
                 weight_decay=0.01)
    return synth.Workload(f"graph_{algo}", sizes, dtypes, algo, hyper, 10, synth.SEED_BASE + 40,
                          "mixed_magnitude", skip_zeros=skip)


def _state(h):
    torch.cuda.synchronize()
    return [tuple(storage_bits(x) for x in (p, s1, s2)) for p, s1, s2 in zip(h.params, h.s1, h.s2)]


def _same(a, b):
    for x, y in zip(a, b):
        for u, v in zip(x, y):
            assert np.array_equal(u, v)


def _table(hyper, first, count):
    raw = B.fill_step_scalars(hyper, first, count)
    return torch.frombuffer(bytearray(raw), dtype=torch.uint8).cuda()


@pytest.mark.parametrize("algo,skip", [("adam", False), ("ademamix", True)])
def test_table_steps_equal_eager_steps(algo, skip):
    w = _workload(algo, skip)
    eager, tab = Harness(w), Harness(w)
    plan = B.Plan(tab.tl, w.algo)
    table = _table(tab.hyper, 1, 6)
    index = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(1, 6):
        eager.load_grads(t)
        tab.load_grads(t)
        B.opt2s_step(eager.tl, eager.hyper, t)
        plan.step_table(skip, table.data_ptr(), 6, index.data_ptr())
    _same(_state(eager), _state(tab))
    assert int(index.item()) == 5
    plan.step_table(skip, table.data_ptr(), 6, index.data_ptr())     # entry 5 = step 6
    assert int(index.item()) == -1                                   # table used up
    before = _state(tab)
    plan.step_table(skip, table.data_ptr(), 6, index.data_ptr())     # no update now
    _same(before, _state(tab))
    plan.close()


def test_captured_graph_replays_successive_steps():
    w = _workload()
    eager, g = Harness(w), Harness(w)
    plan = B.Plan(g.tl, w.algo)
    table = _table(g.hyper, 1, 16)
    index = torch.zeros(1, dtype=torch.int32, device="cuda")
    # one eager step first (plan built, attributes queried), then capture
    eager.load_grads(1)
    g.load_grads(1)
    B.opt2s_step(eager.tl, eager.hyper, 1)
    plan.step_table(True, table.data_ptr(), 16, index.data_ptr())
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        plan.step_table(True, table.data_ptr(), 16, index.data_ptr())
    torch.cuda.synchronize()
    assert int(index.item()) == 1              # capture itself ran nothing
    n0 = B.launch_count()
    for t in range(2, 11):
        eager.load_grads(t)
        g.load_grads(t)
        B.opt2s_step(eager.tl, eager.hyper, t)
        graph.replay()
    _same(_state(eager), _state(g))
    assert int(index.item()) == 10
    assert B.launch_count() == n0 + 9          # replays launch without the library's host code
    # and the replayed trajectory equals the oracle's
    for t in range(1, 11):
        g.load_grads(t)
        g.oracle_step(t)
    assert g.max_ulps() == {"param": 0, "state1": 0, "state2": 0}
    del graph
    plan.close()


def _torch_params(seed, dtypes=("f32", "f16", "bf16", "f32"), sizes=(7, 1000, 4097, 65536)):
    gen = torch.Generator(device="cpu").manual_seed(seed)
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
    ps = []
    for n, d in zip(sizes, dtypes):
        ps.append(torch.randn(n, generator=gen).to(tdt[d]).cuda().requires_grad_(True))
    return ps


def _grads(ps, step, seed):
    gen = torch.Generator(device="cpu").manual_seed(seed * 1000 + step)
    for p in ps:
        p.grad = (torch.randn(p.numel(), generator=gen) * 1e-2).to(p.dtype).cuda()


@pytest.mark.parametrize("cls,kw", [(optim.AdamW32bit, {}), (optim.Adam32bit, {}),
                                    (optim.AdEMAMix32bit, dict(weight_decay=0.1)),
                                    (optim.AdamW32bit, dict(skip_zeros=True))])
def test_optimizer_classes_match_the_oracle(cls, kw):
    import oracle
    ps = _torch_params(3)
    opt = cls(ps, lr=2e-3, **kw)
    hosts = [dict(p=(p.detach().cpu().view(torch.int16 if p.dtype != torch.float32 else torch.int32)
                     .numpy().copy())) for p in ps]
    for h, p in zip(hosts, ps):
        n = p.numel()
        h["s1"] = np.zeros(2 * n if opt.algo == "ademamix" else n, np.float32)
        h["s2"] = np.zeros(n, np.float32)
    dt = {torch.float32: "f32", torch.float16: "f16", torch.bfloat16: "bf16"}
    group = opt.param_groups[0]
    for t in range(1, 6):
        _grads(ps, t, 3)
        opt.step()
        for h, p in zip(hosts, ps):
            g = p.grad.detach().cpu()
            g = g.view(torch.int16 if p.dtype != torch.float32 else torch.int32).numpy()
            oracle.step_f32(h["p"], g, h["s1"], h["s2"], dtype=dt[p.dtype], algo=opt.algo,
                            step=t, lr=group["lr"], beta1=group["betas"][0],
                            beta2=group["betas"][1], eps=group["eps"], beta3=group["beta3"],
                            alpha=group["alpha"], weight_decay=group["weight_decay"],
                            skip_zeros=group["skip_zeros"])
    torch.cuda.synchronize()
    for h, p in zip(hosts, ps):
        got = p.detach().cpu().view(torch.int16 if p.dtype != torch.float32 else torch.int32).numpy()
        assert np.array_equal(got, h["p"])
        st = opt.state[p]
        assert np.array_equal(st["state1"].cpu().numpy(), h["s1"])
        assert np.array_equal(st["state2"].cpu().numpy(), h["s2"])
        assert st["step"] == 5


def test_optimizer_capturable_graph_equals_eager():
    pa, pb = _torch_params(4), _torch_params(4)
    eager = optim.AdEMAMix32bit(pa, lr=1e-3)
    cap = optim.AdEMAMix32bit(pb, lr=1e-3, capturable=True, table_len=8)
    _grads(pa, 1, 4)
    _grads(pb, 1, 4)
    eager.step()
    cap.step()                        # eager first step: builds plan and table
    torch.cuda.synchronize()
    static_grads = [p.grad for p in pb]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cap.step()
    for t in range(2, 8):
        _grads(pa, t, 4)
        _grads(pb, t, 4)
        for sg, p in zip(static_grads, pb):       # same buffers the graph reads
            sg.copy_(p.grad)
            p.grad = sg
        eager.step()
        graph.replay()
    torch.cuda.synchronize()
    assert cap.steps_left() == 1
    for a, b in zip(pa, pb):
        assert torch.equal(a.detach().view(torch.uint8), b.detach().view(torch.uint8))
        assert torch.equal(eager.state[a]["state1"], cap.state[b]["state1"])
        assert torch.equal(eager.state[a]["state2"], cap.state[b]["state2"])
    del graph


@pytest.mark.parametrize("cls", [optim.AdamW32bit, optim.AdEMAMix32bit])
def test_flattened_optimizer_equals_per_tensor_optimizer(cls):
    """A small model trained a few steps with real backward passes: the flat
    layout (params, grads and state in one buffer per dtype) gives the same
    bits as the per-tensor layout."""
    def model_params(seed):
        gen = torch.Generator(device="cpu").manual_seed(seed)
        shapes = [(64, 33), (33,), (33, 7), (7,), (1000,), (5, 200)]
        dts = [torch.float32, torch.float32, torch.bfloat16, torch.bfloat16, torch.float16,
               torch.float32]
        return [torch.nn.Parameter(torch.randn(s, generator=gen).to(d).cuda()) for s, d in zip(shapes, dts)]

    def loss_of(ps, x):
        h = torch.tanh(x @ ps[0].float() + ps[1].float())
        y = h @ ps[2].float() + ps[3].float()
        return (y ** 2).mean() + (ps[4].float() ** 2).sum() * 1e-3 + ps[5].float().pow(2).mean()

    pa, pb = model_params(7), model_params(7)
    oa, ob = cls(pa, lr=1e-2), cls(pb, lr=1e-2, flatten=True)
    gen = torch.Generator(device="cpu").manual_seed(8)
    for _ in range(5):
        x = torch.randn(16, 64, generator=gen).cuda()
        for ps, o in ((pa, oa), (pb, ob)):
            o.zero_grad()
            loss_of(ps, x).backward()
            o.step()
    torch.cuda.synchronize()
    for a, b in zip(pa, pb):
        assert torch.equal(a.detach().view(torch.uint8), b.detach().view(torch.uint8))
    # the flat layout really is flat: one plan per (group, dtype)
    assert len(ob._flat) == 3
    assert all(p.grad.data_ptr() >= f["grad"].data_ptr() for f in ob._flat for p in f["params"])
