"""The Python binding's marshalling, checked on the CPU (nothing is launched:
the descriptors are only built and inspected)."""
import pytest
import torch

from elementwise_optimizer_b200 import binding as B


def test_records_carry_pointers_sizes_and_dtype_codes():
    ps = [torch.zeros(5), torch.zeros(7, dtype=torch.float16), torch.zeros(3, dtype=torch.bfloat16)]
    gs = [torch.zeros_like(p) for p in ps]
    s1 = [torch.zeros(p.numel()) for p in ps]
    s2 = [torch.zeros(p.numel()) for p in ps]
    tl = B.TensorList.from_tensors(ps, gs, s1, s2)
    assert tl.count == 3 and tl.desc.count == 3
    for i, p in enumerate(ps):
        r = tl.desc.tensors[i]
        assert r.param == p.data_ptr() and r.grad == gs[i].data_ptr()
        assert r.state1 == s1[i].data_ptr() and r.state2 == s2[i].data_ptr()
        assert r.numel == p.numel() and r.reserved == 0
    assert [tl.desc.tensors[i].dtype for i in range(3)] == [B.DTYPES["f32"], B.DTYPES["f16"],
                                                          B.DTYPES["bf16"]]


def test_marshalling_rejects_what_the_abi_cannot_take():
    p = torch.zeros(4, 4)
    with pytest.raises(ValueError):                      # non-contiguous view
        B.TensorList.from_tensors([p.t()], [p.t()], [torch.zeros(16)], [torch.zeros(16)])
    with pytest.raises(ValueError):                      # grad dtype differs
        B.TensorList.from_tensors([torch.zeros(4)], [torch.zeros(4, dtype=torch.float16)],
                                  [torch.zeros(4)], [torch.zeros(4)])
    with pytest.raises(ValueError):                      # grad size differs
        B.TensorList.from_tensors([torch.zeros(4)], [torch.zeros(5)], [torch.zeros(4)],
                                  [torch.zeros(4)])
    with pytest.raises(TypeError):                       # no storage code for float64
        B.TensorList.from_tensors([torch.zeros(4, dtype=torch.float64)],
                                  [torch.zeros(4, dtype=torch.float64)], [torch.zeros(4)],
                                  [torch.zeros(4)])


def test_empty_list_and_hyper_fields():
    tl = B.TensorList([])
    assert tl.count == 0 and tl.desc.count == 0
    h = B.make_hyper("ademamix", lr=2e-3, beta1=0.8, beta2=0.99, eps=1e-6, weight_decay=0.1,
                     beta3=0.999, alpha=4.0, skip_zeros=True)
    got = (h.lr, h.beta1, h.beta2, h.beta3, h.alpha, h.eps, h.weight_decay)
    want = tuple(float(torch.tensor(x, dtype=torch.float32)) for x in
                 (2e-3, 0.8, 0.99, 0.999, 4.0, 1e-6, 0.1))
    assert got == want
    assert h.algo == B.ALGOS["ademamix"] and h.skip_zeros == 1
    with pytest.raises(KeyError):
        B.make_hyper("lamb")


def test_errors_carry_status_text_and_cuda_code():
    B.lib()
    e = B.Opt2sError(-2, "somewhere", 0)
    assert e.status == -2 and "somewhere" in str(e)
    with pytest.raises(B.Opt2sError) as ex:
        B.check(-1, "here")
    assert ex.value.status == -1
    B.check(0, "fine")
