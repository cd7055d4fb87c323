"""Argument checks of the torch.optim-style classes that need no GPU (they
run before any tensor is touched)."""
import pytest
import torch

from elementwise_optimizer_b200 import optim


def _p():
    return [torch.nn.Parameter(torch.zeros(4))]


@pytest.mark.parametrize("bad", [-1.0, float("inf"), float("nan")])
def test_max_unorm_must_be_finite_and_non_negative(bad):
    with pytest.raises(ValueError):
        optim.AdamW32bit(_p(), max_unorm=bad)


def test_max_unorm_is_not_combined_with_capturable():
    with pytest.raises(ValueError):
        optim.AdEMAMix32bit(_p(), max_unorm=0.5, capturable=True)
    optim.AdEMAMix32bit(_p(), max_unorm=0.0, capturable=True)   # 0 disables the bound


def test_flatten_is_not_combined_with_capturable():
    with pytest.raises(ValueError):
        optim.Adam32bit(_p(), flatten=True, capturable=True)


def test_unknown_algorithm_is_rejected():
    with pytest.raises(ValueError):
        optim.TwoStateOptimizer(_p(), algo="lamb")


def test_classes_carry_the_options():
    o = optim.AdEMAMix32bit(_p(), lr=2e-3, betas=(0.8, 0.99, 0.999), alpha=4.0, max_unorm=0.25)
    g = o.param_groups[0]
    assert o.algo == "ademamix" and o.max_unorm == 0.25
    assert g["betas"] == (0.8, 0.99) and g["beta3"] == 0.999 and g["alpha"] == 4.0
    assert optim.AdamW32bit(_p()).param_groups[0]["weight_decay"] == 1e-2
    assert optim.Adam32bit(_p()).param_groups[0]["weight_decay"] == 0.0


@pytest.mark.parametrize("bad", [0, -4])
def test_min_8bit_size_must_be_positive(bad):
    with pytest.raises(ValueError):
        optim.AdamW8bit(_p(), min_8bit_size=bad)


def test_8bit_classes_carry_the_options():
    o = optim.AdEMAMix8bit(_p(), lr=2e-3, betas=(0.8, 0.99, 0.999), alpha=4.0, min_8bit_size=1024)
    g = o.param_groups[0]
    assert o.algo == "ademamix" and o.min_8bit_size == 1024
    assert g["betas"] == (0.8, 0.99) and g["beta3"] == 0.999 and g["alpha"] == 4.0
    assert optim.AdamW8bit(_p()).min_8bit_size == 4096
    assert optim.AdamW8bit(_p()).param_groups[0]["weight_decay"] == 1e-2
    assert optim.Adam8bit(_p()).param_groups[0]["weight_decay"] == 0.0
    # the options the 8-bit step does not offer are not accepted
    for kw in (dict(flatten=True), dict(capturable=True), dict(max_unorm=1.0), dict(lamb=True)):
        with pytest.raises(TypeError):
            optim.AdamW8bit(_p(), **kw)
