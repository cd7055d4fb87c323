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
//     (cudaGetSymbolAddress, with that device current) and caches it.

#include <algorithm>
#include <cstdint>
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
opt2s::Range g_ranges[4 * kNoAllocMaxChunks];

std::mutex g_mu;
void* g_table_ptr[kMaxDevices];   // device address of g_noalloc_table, per device

// Validates every record with the same rules as opt2s_step (shared from
// opt2s_internal.h), checks buffer overlaps through the fixed g_ranges and
// counts the chunks; *nchunks receives the count on success.
int check_desc(const TensorListDesc* d, int32_t algo, int64_t chunk_elems, int64_t* nchunks)
{
    if (!d || d->count < 0 || (d->count > 0 && !d->tensors)) return OPT2S_ERR_INVALID_ARG;
    int64_t chunks = 0;
    size_t nr = 0;
    for (int32_t i = 0; i < d->count; ++i) {
        opt2s::Range r[4];
        int n = 0;
        const int st = opt2s::record_ranges(d->tensors[i], algo, r, &n);
        if (st != OPT2S_OK) return st;
        if (n == 0) continue;
        // every non-empty record takes at least one chunk, so while the count
        // stays within the table, its ranges fit in g_ranges
        chunks += (d->tensors[i].numel + chunk_elems - 1) / chunk_elems;
        if (chunks > kNoAllocMaxChunks) return OPT2S_ERR_TOO_LARGE;
        for (int k = 0; k < n; ++k) g_ranges[nr++] = r[k];
    }
    const int st = opt2s::overlap_status(g_ranges, nr);
    if (st != OPT2S_OK) return st;
    *nchunks = chunks;
    return OPT2S_OK;
}

}  // namespace

OPT2S_API int opt2s_step_noalloc(const TensorListDesc* desc, const Hyper* hyper, int step,
                                 cudaStream_t stream)
{
    OPT2S_RANGE("opt2s_step_noalloc");
    int st = opt2s::validate_hyper(hyper, step);
    if (st != OPT2S_OK) return st;
    std::lock_guard<std::mutex> lock(g_mu);
    const int64_t ce = kNoAllocChunkElems;
    int64_t nchunks = 0;
    if ((st = check_desc(desc, hyper->algo, ce, &nchunks)) != OPT2S_OK) return st;
    if (nchunks == 0) return OPT2S_OK;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return opt2s::record_cuda_error(e);
    if (dev < 0 || dev >= kMaxDevices) return opt2s::record_cuda_error(cudaErrorInvalidDevice);
    if (!g_table_ptr[dev]) {
        // once per device, with that device current
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_table);
        if (e != cudaSuccess) return opt2s::record_cuda_error(e);
        if (!ptr) return opt2s::record_cuda_error(cudaErrorInvalidSymbol);
        g_table_ptr[dev] = ptr;
    }

    int64_t k = 0;
    for (int32_t i = 0; i < desc->count; ++i) {
        const opt2s_tensor& t = desc->tensors[i];
        const int es = opt2s::elem_bytes(t.dtype);
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
    e = cudaMemcpyAsync(table, g_host_table, sizeof(ChunkRec) * nchunks, cudaMemcpyHostToDevice, stream);
    if (e != cudaSuccess) return opt2s::record_cuda_error(e);
    e = opt2s::launch_step(table, nchunks, hyper->algo, hyper->skip_zeros, -1,
                           opt2s::make_scalars(hyper, step), opt2s::kDefaultBlockThreads, 0, stream);
    if (e != cudaSuccess) return opt2s::record_cuda_error(e);
    opt2s::count_launches(1);
    return OPT2S_OK;
}

OPT2S_API int64_t opt2s_noalloc_max_chunks(void) { return kNoAllocMaxChunks; }
