// opt2s_marshal.cpp -- argument marshalling for the torch.optim front end
// (elementwise_optimizer_b200/optim.py), as a small PyTorch C++ extension.
//
// An eager optimizer.step() must hand the library the current addresses of
// every parameter and gradient of a group.  Reading them from Python costs
// about 100 ns a tensor (attribute lookups and method calls); here one call
// walks the parameter list in C++ and refreshes the library's tensor records
// in place.  Nothing of the optimizer's arithmetic is here: it only reads
// tensor metadata and writes addresses into the records of include/opt2s.h.

#include <torch/csrc/autograd/variable.h>
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

// The start of a tensor's data (its storage's base plus its offset), read
// from the TensorImpl without the checks data_ptr() adds for tensors that
// can have no storage: every tensor here is a dense CUDA tensor, which is
// checked first.
inline void* start_of(const c10::TensorImpl* t)
{
    return static_cast<char*>(t->storage().data_ptr().get()) + t->storage_offset() * t->itemsize();
}

// Whether a parameter and its gradient still fit record r (opt2s_tensor or
// opt2s_tensor8): both defined, dense, contiguous CUDA tensors of the
// record's element count and dtype.
template <typename Rec>
inline bool fits(const c10::TensorImpl* p, const c10::TensorImpl* g, const Rec& r)
{
    return p->layout() == c10::kStrided && g->layout() == c10::kStrided &&
           p->is_cuda() && g->is_cuda() && p->is_contiguous() && g->is_contiguous() &&
           p->numel() == r.numel && g->numel() == r.numel &&
           dtype_code(p->dtype().toScalarType()) == r.dtype && g->dtype() == p->dtype();
}

// The gradient of a parameter (the autograd metadata's grad field: the
// tensor p.grad returns, without its non-leaf warning path), or nullptr.
inline const c10::TensorImpl* grad_of(const at::Tensor& p)
{
    const auto* meta = torch::autograd::impl::get_autograd_meta(p);
    if (!meta || !meta->grad_.defined()) return nullptr;
    return meta->grad_.unsafeGetTensorImpl();
}

// Refreshes the param and grad addresses of the `n` records (Rec:
// opt2s_tensor or opt2s_tensor8) at address `records` from the tensors of
// `params` (record i <-> params[i]).  Returns 0 when no address changed, 1
// when some did (the records now hold the new ones), and -1 when a parameter
// has no gradient or no longer fits its record (element count, storage
// dtype, contiguity, CUDA placement): the caller then rebuilds its records.
// The records are untouched on -1.  One pass checks every tensor and
// compares its addresses; only when an address changed does a second pass,
// from the first change, write them.
template <typename Rec>
int64_t refresh(py::list params, uintptr_t records, int64_t n)
{
    if (static_cast<int64_t>(py::len(params)) != n) return -1;
    auto* rec = reinterpret_cast<Rec*>(records);
    PyObject* const* items = PySequence_Fast_ITEMS(params.ptr());
    int64_t first_change = -1;
    for (int64_t i = 0; i < n; ++i) {
        if (!THPVariable_Check(items[i])) return -1;
        const at::Tensor& p = THPVariable_Unpack(items[i]);
        const c10::TensorImpl* g = grad_of(p);
        const c10::TensorImpl* pi = p.unsafeGetTensorImpl();
        if (!g || !fits(pi, g, rec[i])) return -1;
        if (first_change < 0 && (rec[i].param != start_of(pi) || rec[i].grad != start_of(g)))
            first_change = i;
    }
    if (first_change < 0) return 0;
    for (int64_t i = first_change; i < n; ++i) {
        const at::Tensor& p = THPVariable_Unpack(items[i]);
        rec[i].param = start_of(p.unsafeGetTensorImpl());
        rec[i].grad = start_of(grad_of(p));
    }
    return 1;
}

int64_t refresh_records(py::list params, uintptr_t records, int64_t n)
{
    return refresh<opt2s_tensor>(params, records, n);
}

int64_t refresh_records8(py::list params, uintptr_t records, int64_t n)
{
    return refresh<opt2s_tensor8>(params, records, n);
}

}  // namespace

PYBIND11_MODULE(TORCH_EXTENSION_NAME, m)
{
    m.def("refresh_records", &refresh_records,
          "Refresh the param/grad addresses of opt2s_tensor records from a parameter list");
    m.def("refresh_records8", &refresh_records8,
          "Refresh the param/grad addresses of opt2s_tensor8 records from a parameter list");
}
