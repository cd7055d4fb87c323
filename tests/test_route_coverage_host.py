"""The GPU parity workloads exercise both division routes of the grouped
update.

The 8-bit kernel, the norm pass and the scaled step divide a group's moments
by bc1 and bc2 with the fp32 route when every value of the group lies in
[2^-40, 2^96), else with the binary64 route for the whole group; both are
exact, so the parity tests can only show that each path is right if their
inputs send some groups down each.  These checks, on the CPU, take the
first step's moments of the workloads of tests/test_8bit_gpu.py and
tests/test_max_unorm_gpu.py (m = (1-b1) g, v = (1-b2) g^2 from zero state,
in fp32) and count the groups of 4 and of 8 consecutive elements that take
each route.  No kernel arithmetic is involved: only which path a group takes.
"""
import numpy as np
import pytest

from elementwise_optimizer_b200 import synth

LO, HI = 2.0 ** -40, 2.0 ** 96


def _moments(w):
    hy = w.hyper
    b1 = np.float32(1.0 - hy["beta1"])
    b2 = np.float32(1.0 - hy["beta2"])
    gs = w.grads(1)
    out = []
    for g in gs:
        g = g.astype(np.float32)
        m = (b1 * g).astype(np.float32)
        v = ((b2 * g).astype(np.float32) * g).astype(np.float32)
        out.append((m, v))
    return out


def _route_counts(moments, group):
    fast = slow = 0
    for m, v in moments:
        n = len(m) // group * group
        if n == 0:
            continue
        ok = lambda x: (np.abs(x[:n]) >= LO) & (np.abs(x[:n]) < HI)
        in_range = (ok(m) & ok(v)).reshape(-1, group).all(axis=1)
        fast += int(in_range.sum())
        slow += int((~in_range).sum())
    return fast, slow


def _eightbit_workload(algo):
    sizes = [1, 64, 100, 333, 512, 1000, 1024, 4095, 4096, 4097, 6144, 8191, 70_001, 1 << 20]
    dtypes = [("f32", "bf16", "f16")[i % 3] for i in range(len(sizes))]
    hy = dict(synth.ADEMAMIX_HYPER if algo == "ademamix" else synth.ADAM_HYPER, weight_decay=0.01)
    return synth.Workload("eightbit", sizes, dtypes, algo, hy, 3, synth.SEED_BASE + 51, "mixed_magnitude")


def _unorm_workload(algo):
    sizes = [1, 2, 31, 33, 255, 257, 1000, 2047, 2048, 2049, 4097, 70_001, 1 << 20]
    dtypes = ("f32", "f16", "bf16")
    hy = dict(synth.ADEMAMIX_HYPER if algo == "ademamix" else synth.ADAM_HYPER, weight_decay=0.01)
    return synth.Workload("unorm", sizes, [dtypes[i % 3] for i in range(len(sizes))], algo, hy, 3,
                          synth.SEED_BASE + 21, "mixed_magnitude")


@pytest.mark.parametrize("make", [_eightbit_workload, _unorm_workload])
@pytest.mark.parametrize("algo", ["adam", "ademamix"])
@pytest.mark.parametrize("group", [4, 8])
def test_both_routes_are_taken(make, algo, group):
    fast, slow = _route_counts(_moments(make(algo)), group)
    # thousands of groups each way, not a handful
    assert fast > 1000 and slow > 1000, (fast, slow)


def test_normal_gradients_take_the_fp32_route():
    """The N(0, 1e-2) gradients of the long 8-bit runs keep about 99 % of
    the groups in range (a |g| below about 3e-5 puts v below 2^-40): those
    runs check mostly the fp32 route."""
    w = synth.Workload("eightbit", [300, 4096, 10_000, 65_541], ["f32", "bf16", "f16", "f32"], "adam",
                       dict(synth.ADAM_HYPER, weight_decay=0.01), 10, synth.SEED_BASE + 52, "normal")
    fast, slow = _route_counts(_moments(w), 4)
    assert fast > 10_000 and slow < fast // 100, (fast, slow)
