// opt2s_noalloc.cu -- opt2s_step_noalloc: the optimizer step without any
// memory allocation by the library.
//
// Why it exists: opt2s_step keeps its chunk table in device memory it gets
// from cudaMalloc (once per collection, cached).  Some callers cannot let a
// library allocate: a runtime that owns every byte of device memory through
// its own pool and forbids other allocators, an embedded or safety-critical
// deployment that fixes its memory footprint at start-up, or code that must
// not trigger the implicit device synchronization cudaMalloc/cudaFree can
// cause.  For them this entry point builds the chunk table in a fixed host
// array and uploads it into a fixed device array declared below, so it calls
// no cudaMalloc, no cudaFree and no allocating library routine, and keeps no
// plan.  The method it computes is the same kernel and the same arithmetic as
// opt2s_step; nothing in the optimizer's definition corresponds to this
// entry point.
//
// Limits and sharing:
//   * at most kNoAllocMaxChunks chunk records per call (65,536 records,
//     3 MiB of device memory per GPU, held from the time the library's device
//     code is loaded on that GPU until the process exits); a collection that
//     needs more is rejected with OPT2S_ERR_TOO_LARGE before any work;
//   * every call on a device shares that one table and leaves it holding the
//     last call's contents; each call rewrites every record it reads, so
//     nothing has to start at zero.  Two calls whose work overlaps on the GPU
//     (different streams, no ordering between them) race on the table;
//   * the first call on each device looks up the table's device address
//     (cudaGetSymbolAddress, with that device current) and caches it; make
//     that first call before any stream capture begins.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda_runtime.h>

#include "opt2s.h"
#include "opt2s_internal.h"

#define OPT2S_API extern "C" __attribute__((visibility("default")))

namespace {

using opt2s::ChunkRec;
using opt2s::StepScalars;

constexpr int64_t kNoAllocMaxChunks = 65536;   // 48 B each: 3 MiB per device
constexpr int64_t kNoAllocChunkElems = 8192;   // elements per chunk record
constexpr int kMaxDevices = 64;

// The device-side scratch: one fixed chunk table per GPU.  In host code this
// name is only a handle for cudaGetSymbolAddress, never a device address.
static __device__ __align__(256) ChunkRec g_noalloc_table[kNoAllocMaxChunks];

// Host-side staging of the table and of the ranges used by the overlap check,
// also fixed-size; a mutex serializes calls from different host threads.
ChunkRec g_host_table[kNoAllocMaxChunks];
struct Range { uintptr_t lo, hi; bool written; };
Range g_ranges[4 * kNoAllocMaxChunks];

std::mutex g_mu;
void* g_table_ptr[kMaxDevices];   // device address of g_noalloc_table, per device

int elem_bytes(int32_t dtype) { return dtype == OPT2S_F32 ? 4 : 2; }

// Same rules as opt2s_step's validation, written without heap use.
int check_hyper(const Hyper* h, int step)
{
    if (!h) return OPT2S_ERR_INVALID_ARG;
    if (h->algo != OPT2S_ADAM && h->algo != OPT2S_ADEMAMIX) return OPT2S_ERR_INVALID_ARG;
    if (h->skip_zeros != 0 && h->skip_zeros != 1) return OPT2S_ERR_INVALID_ARG;
    if (step < 1) return OPT2S_ERR_INVALID_ARG;
    auto unit = [](float b) { return std::isfinite(b) && b >= 0.0f && b < 1.0f; };
    if (!std::isfinite(h->lr) || !unit(h->beta1) || !unit(h->beta2)) return OPT2S_ERR_INVALID_ARG;
    if (!std::isfinite(h->eps) || h->eps < 0.0f) return OPT2S_ERR_INVALID_ARG;
    if (!std::isfinite(h->weight_decay)) return OPT2S_ERR_INVALID_ARG;
    if (h->algo == OPT2S_ADEMAMIX && (!unit(h->beta3) || !std::isfinite(h->alpha)))
        return OPT2S_ERR_INVALID_ARG;
    return OPT2S_OK;
}

// Validates every record and counts the chunks, filling g_ranges; returns a
// status.  *nchunks receives the chunk count (only meaningful on success).
int check_desc(const TensorListDesc* d, int32_t algo, int64_t chunk_elems, int64_t* nchunks)
{
    if (!d || d->count < 0 || (d->count > 0 && !d->tensors)) return OPT2S_ERR_INVALID_ARG;
    int64_t chunks = 0, nr = 0;
    for (int32_t i = 0; i < d->count; ++i) {
        const opt2s_tensor& t = d->tensors[i];
        if (t.numel < 0 || t.reserved != 0) return OPT2S_ERR_INVALID_ARG;
        if (t.dtype != OPT2S_F32 && t.dtype != OPT2S_F16 && t.dtype != OPT2S_BF16)
            return OPT2S_ERR_INVALID_ARG;
        if (t.numel == 0) continue;
        if (t.numel > (int64_t(1) << 40)) return OPT2S_ERR_INVALID_ARG;
        if (!t.param || !t.grad || !t.state1 || !t.state2) return OPT2S_ERR_INVALID_ARG;
        chunks += (t.numel + chunk_elems - 1) / chunk_elems;
        if (chunks > kNoAllocMaxChunks) return OPT2S_ERR_TOO_LARGE;
        const int es = elem_bytes(t.dtype);
        const auto p = reinterpret_cast<uintptr_t>(t.param);
        const auto g = reinterpret_cast<uintptr_t>(t.grad);
        const auto s1 = reinterpret_cast<uintptr_t>(t.state1);
        const auto s2 = reinterpret_cast<uintptr_t>(t.state2);
        if (p % es || g % es || s1 % 4 || s2 % 4) return OPT2S_ERR_INVALID_ARG;
        const uintptr_t n = static_cast<uintptr_t>(t.numel);
        g_ranges[nr++] = {p, p + n * es, true};
        g_ranges[nr++] = {g, g + n * es, false};
        g_ranges[nr++] = {s1, s1 + (algo == OPT2S_ADEMAMIX ? 2 * n : n) * 4, true};
        g_ranges[nr++] = {s2, s2 + n * 4, true};
    }
    std::sort(g_ranges, g_ranges + nr, [](const Range& a, const Range& b) { return a.lo < b.lo; });
    uintptr_t reach_w = 0, reach_any = 0;
    bool have_w = false, have_any = false;
    for (int64_t k = 0; k < nr; ++k) {
        const Range& r = g_ranges[k];
        if (have_w && r.lo < reach_w) return OPT2S_ERR_ALIAS;
        if (r.written && have_any && r.lo < reach_any) return OPT2S_ERR_ALIAS;
        if (r.written) { reach_w = have_w ? std::max(reach_w, r.hi) : r.hi; have_w = true; }
        reach_any = have_any ? std::max(reach_any, r.hi) : r.hi;
        have_any = true;
    }
    *nchunks = chunks;
    return OPT2S_OK;
}

StepScalars scalars(const Hyper* h, int step)
{
    StepScalars s;
    s.lr = h->lr;
    s.beta1 = h->beta1;
    s.beta2 = h->beta2;
    s.beta3 = h->beta3;
    s.one_minus_beta1 = 1.0f - h->beta1;
    s.one_minus_beta2 = 1.0f - h->beta2;
    s.one_minus_beta3 = 1.0f - h->beta3;
    s.alpha = h->alpha;
    s.eps = h->eps;
    s.bc1 = static_cast<float>(1.0 - std::pow(static_cast<double>(h->beta1), static_cast<double>(step)));
    s.bc2 = static_cast<float>(1.0 - std::pow(static_cast<double>(h->beta2), static_cast<double>(step)));
    s.decay = static_cast<float>(1.0 - static_cast<double>(h->lr) * static_cast<double>(h->weight_decay));
    return s;
}

}  // namespace

OPT2S_API int opt2s_step_noalloc(const TensorListDesc* desc, const Hyper* hyper, int step,
                                 cudaStream_t stream)
{
    int st = check_hyper(hyper, step);
    if (st != OPT2S_OK) return st;
    std::lock_guard<std::mutex> lock(g_mu);
    const int64_t ce = kNoAllocChunkElems;
    int64_t nchunks = 0;
    if ((st = check_desc(desc, hyper->algo, ce, &nchunks)) != OPT2S_OK) return st;
    if (nchunks == 0) return OPT2S_OK;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return OPT2S_ERR_CUDA;
    if (!g_table_ptr[dev]) {
        // once per device, with that device current
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_noalloc_table) != cudaSuccess || !ptr) return OPT2S_ERR_CUDA;
        g_table_ptr[dev] = ptr;
    }

    int64_t k = 0;
    for (int32_t i = 0; i < desc->count; ++i) {
        const opt2s_tensor& t = desc->tensors[i];
        const int es = elem_bytes(t.dtype);
        for (int64_t s = 0; s < t.numel; s += ce) {
            ChunkRec& r = g_host_table[k++];
            r.p = static_cast<char*>(t.param) + s * es;
            r.g = static_cast<const char*>(t.grad) + s * es;
            r.m = t.state1 + s;
            r.v = t.state2 + s;
            r.m2 = t.state1 + t.numel + s;
            r.len = static_cast<uint32_t>(std::min(ce, t.numel - s));
            r.dtype = t.dtype;
        }
    }
    auto* table = static_cast<ChunkRec*>(g_table_ptr[dev]);
    if (cudaMemcpyAsync(table, g_host_table, sizeof(ChunkRec) * nchunks, cudaMemcpyHostToDevice,
                        stream) != cudaSuccess)
        return OPT2S_ERR_CUDA;
    if (opt2s::launch_step(table, nchunks, hyper->algo, hyper->skip_zeros, -1, scalars(hyper, step),
                           opt2s::kDefaultBlockThreads, 0, stream) != cudaSuccess)
        return OPT2S_ERR_CUDA;
    return OPT2S_OK;
}

OPT2S_API int64_t opt2s_noalloc_max_chunks(void) { return kNoAllocMaxChunks; }
