// opt2s_marshal.cpp -- argument marshalling for the torch.optim front end
// (elementwise_optimizer_b200/optim.py), as a small PyTorch C++ extension.
//
// An eager optimizer.step() must hand the library the current addresses of
// every parameter and gradient of a group.  Reading them from Python costs
// about 100 ns a tensor (attribute lookups and method calls); here one call
// walks the parameter list in C++ and refreshes the library's tensor records
// in place.  Nothing of the optimizer's arithmetic is here: it only reads
// tensor metadata and writes addresses into the records of include/opt2s.h.

#include <torch/extension.h>

#include <cstdint>

#include "opt2s.h"

namespace {

int32_t dtype_code(c10::ScalarType t)
{
    switch (t) {
    case c10::ScalarType::Float: return OPT2S_F32;
    case c10::ScalarType::Half: return OPT2S_F16;
    case c10::ScalarType::BFloat16: return OPT2S_BF16;
    default: return -1;
    }
}

// Refreshes the param and grad addresses of the `n` opt2s_tensor records at
// address `records` from the tensors of `params` (record i <-> params[i]).
// Returns 0 when no address changed, 1 when some did (the records now hold
// the new ones), and -1 when a parameter has no gradient or no longer fits its
// record (element count, storage dtype, contiguity, CUDA placement): the
// caller then rebuilds its records.  The records are untouched on -1.
int64_t refresh_records(py::list params, uintptr_t records, int64_t n)
{
    if (static_cast<int64_t>(py::len(params)) != n) return -1;
    auto* rec = reinterpret_cast<opt2s_tensor*>(records);
    // first pass: check everything, so that -1 leaves the records as they were
    for (int64_t i = 0; i < n; ++i) {
        PyObject* o = PyList_GET_ITEM(params.ptr(), i);
        if (!THPVariable_Check(o)) return -1;
        const at::Tensor& p = THPVariable_Unpack(o);
        const at::Tensor& g = p.grad();
        if (!g.defined() || !p.is_cuda() || !g.is_cuda() || !p.is_contiguous() || !g.is_contiguous())
            return -1;
        if (p.numel() != rec[i].numel || g.numel() != rec[i].numel) return -1;
        if (dtype_code(p.scalar_type()) != rec[i].dtype || g.scalar_type() != p.scalar_type()) return -1;
    }
    int64_t changed = 0;
    for (int64_t i = 0; i < n; ++i) {
        const at::Tensor& p = THPVariable_Unpack(PyList_GET_ITEM(params.ptr(), i));
        void* pa = p.data_ptr();
        const void* ga = p.grad().data_ptr();
        if (rec[i].param != pa || rec[i].grad != ga) {
            rec[i].param = pa;
            rec[i].grad = ga;
            changed = 1;
        }
    }
    return changed;
}

}  // namespace

PYBIND11_MODULE(TORCH_EXTENSION_NAME, m)
{
    m.def("refresh_records", &refresh_records,
          "Refresh the param/grad addresses of opt2s_tensor records from a parameter list");
}
