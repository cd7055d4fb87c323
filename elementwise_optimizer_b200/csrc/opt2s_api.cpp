// opt2s_api.cpp -- the C ABI of include/opt2s.h: argument validation, the
// chunk-table builder, plans, and the per-device plan cache.
//
// The issue this library follows (bitsandbytes "Investigate a 256-thread
// SM103 path for small 32-bit optimizer tensors") launches one kernel per
// tensor (section "Problem"), so a model with thousands of bias / norm /
// adapter tensors pays one launch each.  Here the host turns the whole
// collection into a table of chunk records once, uploads it, and every later
// step is a single launch that reads it.  The issue's section "Scope" asks
// that per-device facts be cached per current device and that host dispatch
// overhead stay small; both hold: plans are per device, and a repeated step
// costs one descriptor comparison and one launch.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstddef>
#include <cstring>
#include <list>
#include <mutex>
#include <vector>

#include <cuda_runtime.h>

#include "opt2s.h"
#include "opt2s_internal.h"
#include "opt2s_testing.h"

#define OPT2S_API extern "C" __attribute__((visibility("default")))

using opt2s::ChunkRec;
using opt2s::StepScalars;

struct opt2s_plan {
    int device;
    int32_t algo;
    int32_t only;         // dtype all chunks share (specialised kernel), or -1
    int64_t nchunks;
    ChunkRec* d_chunks;   // device copy of the chunk table
    // Bounded-update-norm workspace (plans made for opt2s_step_max_unorm
    // only): one device allocation holding the norm table, the per-block
    // sums, the tensors' first blocks, the per-tensor scales and the
    // chunk-to-tensor map.
    void* d_unorm;
    opt2s::UnormArgs unorm;
};

namespace {

thread_local int t_last_cuda_error = 0;

std::atomic<int64_t> g_launches{0};   // kernels launched by this library

// Forcing knobs exist only in the test build of the library
// (libopt2s_testing.so, compiled with OPT2S_TESTING); the product build has
// the defaults as constants, so no caller can change its launch geometry.
#ifdef OPT2S_TESTING
int64_t g_chunk_elems = 0;     // forced chunk length (0 = chosen per plan)
int g_block_threads = 0;       // forced threads per block (0 = default)
int g_max_blocks = 0;          // forced cap on blocks (0 = occupancy cap)
std::atomic<int> g_fail_allocs{0};    // plan allocations to fail

bool injected_alloc_failure()
{
    return g_fail_allocs.load() > 0 && g_fail_allocs.fetch_sub(1) > 0;
}
#else
constexpr int64_t g_chunk_elems = 0;
constexpr int g_block_threads = 0;
constexpr int g_max_blocks = 0;

constexpr bool injected_alloc_failure() { return false; }
#endif

int cuda_fail(cudaError_t e)
{
    t_last_cuda_error = static_cast<int>(e);
    return OPT2S_ERR_CUDA;
}

using opt2s::elem_bytes;
using opt2s::make_scalars;
using opt2s::Range;
using opt2s::validate_hyper;

int block_threads_now(int algo, int only)
{
    return g_block_threads > 0 ? g_block_threads : opt2s::default_block_threads(algo, only);
}

// The storage dtype every non-empty tensor of `d` shares, or -1.
int uniform_dtype(const TensorListDesc* d)
{
    int u = -2;
    for (int32_t i = 0; i < d->count; ++i) {
        if (d->tensors[i].numel == 0) continue;
        if (u == -2) u = d->tensors[i].dtype;
        else if (u != d->tensors[i].dtype) return -1;
    }
    return u == -2 ? -1 : u;
}

// Chunk length for a collection: the power of two c in [kMinChunkElems,
// kDefaultChunkElems] that minimizes the modelled time of the slowest warp,
// ceil(chunks / resident_warps) x (c / 32 + 8).  A warp handles its chunks one
// after the other; in a chunk of c elements each lane makes c / 32 element
// updates one after the other, plus about 8 more for fetching the chunk's
// record.  Large collections get long chunks (small table, few record
// fetches); small ones get short chunks so that every resident warp has work
// and each lane's serial part is short.  A 128-element chunk gives each lane
// 4 elements: one 16-byte vector of fp32, or the short-chunk path for 16-bit
// storage, which pays only when the whole plan fits in one wave of warps; so
// a plan with 16-bit tensors takes 128 only then.  Ties go to the longer chunk.
int64_t choose_chunk_elems(const TensorListDesc* d, int64_t resident_warps)
{
    if (resident_warps < 1) return opt2s::kDefaultChunkElems;
    bool all_f32 = true;
    for (int32_t i = 0; i < d->count; ++i)
        if (d->tensors[i].numel > 0 && d->tensors[i].dtype != OPT2S_F32) all_f32 = false;
    int64_t best = opt2s::kDefaultChunkElems;
    int64_t best_cost = -1;
    for (int64_t c = opt2s::kDefaultChunkElems; c >= opt2s::kMinChunkElems; c /= 2) {
        int64_t chunks = 0;
        for (int32_t i = 0; i < d->count; ++i) chunks += (d->tensors[i].numel + c - 1) / c;
        const int64_t waves = (chunks + resident_warps - 1) / resident_warps;
        if (c <= static_cast<int64_t>(opt2s::kShortChunkElems) && !all_f32 && waves > 1) continue;
        const int64_t cost = waves * (c / 32 + 8);
        if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = c; }
    }
    return best;
}

int64_t chunk_elems_for(const TensorListDesc* d, int32_t algo, int only)
{
    if (g_chunk_elems > 0) return g_chunk_elems;
    int64_t warps = 0;
    if (opt2s::resident_warps(algo, 0, only, block_threads_now(algo, only), &warps) != cudaSuccess)
        return opt2s::kDefaultChunkElems;
    return choose_chunk_elems(d, warps);
}

// ---------------------------------------------------------------------------
// Validation (host only, no CUDA call)
// ---------------------------------------------------------------------------

// Every record well formed, and no buffer that is written overlaps any other
// buffer (two gradients may share memory: both are only read).
int validate_desc(const TensorListDesc* d, int32_t algo)
{
    if (!d) return OPT2S_ERR_INVALID_ARG;
    if (algo != OPT2S_ADAM && algo != OPT2S_ADEMAMIX) return OPT2S_ERR_INVALID_ARG;
    if (d->count < 0) return OPT2S_ERR_INVALID_ARG;
    if (d->count > 0 && !d->tensors) return OPT2S_ERR_INVALID_ARG;
    std::vector<Range> ranges;
    for (int32_t i = 0; i < d->count; ++i) {
        Range r[4];
        int n = 0;
        const int st = opt2s::record_ranges(d->tensors[i], algo, r, &n);
        if (st != OPT2S_OK) return st;
        ranges.insert(ranges.end(), r, r + n);
    }
    return opt2s::overlap_status(ranges.data(), ranges.size());
}

// ---------------------------------------------------------------------------
// Chunk-table builder
// ---------------------------------------------------------------------------

// Splits every tensor into chunks of at most `chunk_elems` elements, in
// descriptor order.  Chunk starts are multiples of chunk_elems (a multiple of
// 8), so a tensor whose arrays are 16-byte aligned keeps every chunk on the
// 128-bit vector path.
template <typename Emit>
void for_each_chunk(const TensorListDesc* d, int64_t chunk_elems, Emit emit)
{
    for (int32_t i = 0; i < d->count; ++i) {
        const opt2s_tensor& t = d->tensors[i];
        for (int64_t s = 0; s < t.numel; s += chunk_elems)
            emit(i, t, s, std::min(chunk_elems, t.numel - s));
    }
}

int64_t count_chunks(const TensorListDesc* d, int64_t chunk_elems)
{
    int64_t n = 0;
    for (int32_t i = 0; i < d->count; ++i)
        n += (d->tensors[i].numel + chunk_elems - 1) / chunk_elems;
    return n;
}

// With `short16`, 16-bit chunks of at most kShortChunkElems elements are
// marked for the kernel's short-chunk path.
std::vector<ChunkRec> build_chunk_table(const TensorListDesc* d, int64_t chunk_elems, bool short16)
{
    std::vector<ChunkRec> out;
    out.reserve(static_cast<size_t>(count_chunks(d, chunk_elems)));
    for_each_chunk(d, chunk_elems, [&](int32_t, const opt2s_tensor& t, int64_t s, int64_t len) {
        const int es = elem_bytes(t.dtype);
        ChunkRec r;
        r.p = static_cast<char*>(t.param) + s * es;
        r.g = static_cast<const char*>(t.grad) + s * es;
        r.m = t.state1 + s;
        r.v = t.state2 + s;
        r.m2 = t.state1 + t.numel + s;
        r.len = static_cast<uint32_t>(len);
        r.dtype = t.dtype;
        if (short16 && t.dtype != OPT2S_F32 && len <= static_cast<int64_t>(opt2s::kShortChunkElems))
            r.dtype |= opt2s::kShortFlag;
        out.push_back(r);
    });
    return out;
}

// Host tables of the bounded-update-norm step for `desc` (the plan's chunks
// have `chunk_elems` elements): the norm blocks, the group ranges (first and
// end block of each group of kNormGroupBlocks consecutive blocks of one
// tensor), each tensor's first group (count + 1 entries) and each chunk's
// tensor.  The caller has checked that the block count fits in 32 bits.
struct UnormTables {
    std::vector<ChunkRec> blocks;
    std::vector<uint32_t> ranges;
    std::vector<uint32_t> first_group;
    std::vector<uint32_t> chunk_tensor;
};

UnormTables unorm_tables(const TensorListDesc* desc, int64_t chunk_elems)
{
    using opt2s::kNormBlockElems;
    using opt2s::kNormGroupBlocks;
    UnormTables t;
    t.blocks = build_chunk_table(desc, kNormBlockElems, false);
    t.first_group.assign(static_cast<size_t>(desc->count) + 1, 0);
    uint32_t block0 = 0;
    for (int32_t i = 0; i < desc->count; ++i) {
        const uint32_t nb = static_cast<uint32_t>(
            (desc->tensors[i].numel + kNormBlockElems - 1) / kNormBlockElems);
        for (uint32_t b = 0; b < nb; b += kNormGroupBlocks) {
            t.ranges.push_back(block0 + b);
            t.ranges.push_back(block0 + std::min<uint32_t>(b + kNormGroupBlocks, nb));
        }
        block0 += nb;
        t.first_group[i + 1] = static_cast<uint32_t>(t.ranges.size() / 2);
    }
    for_each_chunk(desc, chunk_elems, [&](int32_t i, const opt2s_tensor&, int64_t, int64_t) {
        t.chunk_tensor.push_back(static_cast<uint32_t>(i));
    });
    return t;
}

// Builds the bounded-update-norm workspace of `plan` for `desc` (host tables,
// then one device allocation and four uploads).
int unorm_workspace(const TensorListDesc* desc, int64_t chunk_elems, opt2s_plan* plan)
{
    if (count_chunks(desc, opt2s::kNormBlockElems) > INT32_MAX) return OPT2S_ERR_TOO_LARGE;
    UnormTables tab = unorm_tables(desc, chunk_elems);
    const std::vector<ChunkRec>& blocks = tab.blocks;
    const std::vector<uint32_t>& ranges = tab.ranges;
    const std::vector<uint32_t>& first_group = tab.first_group;
    const std::vector<uint32_t>& chunk_tensor = tab.chunk_tensor;
    const size_t ngroups = ranges.size() / 2;
    // layout: blocks | partial | group ranges | group sums | first_group | scale | chunk_tensor
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t sizes[] = {up(blocks.size() * sizeof(ChunkRec)), up(blocks.size() * 2 * sizeof(double)),
                            up(ranges.size() * sizeof(uint32_t)), up(ngroups * 2 * sizeof(double)),
                            up(first_group.size() * sizeof(uint32_t)),
                            up(static_cast<size_t>(desc->count) * sizeof(float)),
                            up(chunk_tensor.size() * sizeof(uint32_t))};
    size_t total = 0;
    for (size_t x : sizes) total += x;
    cudaError_t e;
    if (injected_alloc_failure())
        e = cudaErrorMemoryAllocation;                // injected by the test build
    else
        e = cudaMalloc(&plan->d_unorm, total);
    if (e != cudaSuccess) {
        plan->d_unorm = nullptr;
        if (e == cudaErrorMemoryAllocation) { t_last_cuda_error = e; return OPT2S_ERR_NO_MEMORY; }
        return cuda_fail(e);
    }
    char* at[7];
    at[0] = static_cast<char*>(plan->d_unorm);
    for (int k = 1; k < 7; ++k) at[k] = at[k - 1] + sizes[k - 1];
    opt2s::UnormArgs& u = plan->unorm;
    u.blocks = reinterpret_cast<ChunkRec*>(at[0]);
    u.nblocks = static_cast<int64_t>(blocks.size());
    u.partial = reinterpret_cast<double*>(at[1]);
    u.group_range = reinterpret_cast<uint32_t*>(at[2]);
    u.ngroups = static_cast<int64_t>(ngroups);
    u.group_sum = reinterpret_cast<double*>(at[3]);
    u.first_group = reinterpret_cast<uint32_t*>(at[4]);
    u.ntensors = desc->count;
    u.scale = reinterpret_cast<float*>(at[5]);
    u.chunk_tensor = reinterpret_cast<uint32_t*>(at[6]);
    auto put = [&](const void* dst, const void* src, size_t bytes) {
        if (e == cudaSuccess && bytes > 0)
            e = cudaMemcpy(const_cast<void*>(dst), src, bytes, cudaMemcpyHostToDevice);
    };
    put(u.blocks, blocks.data(), blocks.size() * sizeof(ChunkRec));
    put(u.group_range, ranges.data(), ranges.size() * sizeof(uint32_t));
    put(u.first_group, first_group.data(), first_group.size() * sizeof(uint32_t));
    put(u.chunk_tensor, chunk_tensor.data(), chunk_tensor.size() * sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_fail(e);
    return OPT2S_OK;
}

int plan_destroy(opt2s_plan* plan);

int plan_create(const TensorListDesc* desc, int32_t algo, opt2s_plan** out, bool unorm = false)
{
    int st = validate_desc(desc, algo);
    if (st != OPT2S_OK) return st;
    const int only = opt2s::kernel_only(algo, uniform_dtype(desc));
    const int64_t ce = chunk_elems_for(desc, algo, only);
    if (count_chunks(desc, ce) > INT32_MAX) return OPT2S_ERR_TOO_LARGE;
    std::vector<ChunkRec> table =
        build_chunk_table(desc, ce, ce <= static_cast<int64_t>(opt2s::kShortChunkElems));
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    auto* plan = new (std::nothrow) opt2s_plan{dev, algo, only, static_cast<int64_t>(table.size()), nullptr,
                                               nullptr, opt2s::UnormArgs{}};
    if (!plan) return OPT2S_ERR_NO_MEMORY;
    if (!table.empty()) {
        const size_t bytes = table.size() * sizeof(ChunkRec);
        if (injected_alloc_failure())
            e = cudaErrorMemoryAllocation;            // injected by the test build
        else
            e = cudaMalloc(&plan->d_chunks, bytes);
        if (e != cudaSuccess) {
            delete plan;
            if (e == cudaErrorMemoryAllocation) { t_last_cuda_error = e; return OPT2S_ERR_NO_MEMORY; }
            return cuda_fail(e);
        }
        e = cudaMemcpy(plan->d_chunks, table.data(), bytes, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) {
            cudaFree(plan->d_chunks);
            delete plan;
            return cuda_fail(e);
        }
    }
    if (unorm) {
        st = unorm_workspace(desc, ce, plan);
        if (st != OPT2S_OK) {
            const int keep = t_last_cuda_error;
            plan_destroy(plan);
            t_last_cuda_error = keep;
            return st;
        }
    }
    *out = plan;
    return OPT2S_OK;
}

int plan_destroy(opt2s_plan* plan)
{
    if (!plan) return OPT2S_OK;
    int st = OPT2S_OK;
    if (plan->d_chunks || plan->d_unorm) {
        int cur = -1;
        cudaError_t e = cudaGetDevice(&cur);
        const bool switched = e == cudaSuccess && cur != plan->device;
        if (switched) e = cudaSetDevice(plan->device);
        if (e == cudaSuccess && plan->d_chunks) e = cudaFree(plan->d_chunks);   // waits for the device
        if (e == cudaSuccess && plan->d_unorm) e = cudaFree(plan->d_unorm);
        if (e != cudaSuccess) st = cuda_fail(e);
        if (switched) cudaSetDevice(cur);
    }
    delete plan;
    return st;
}

int plan_step(const opt2s_plan* plan, const Hyper* h, int step, cudaStream_t stream)
{
    if (!plan) return OPT2S_ERR_INVALID_ARG;
    int st = validate_hyper(h, step);
    if (st != OPT2S_OK) return st;
    if (h->algo != plan->algo) return OPT2S_ERR_INVALID_ARG;
    if (plan->nchunks == 0) return OPT2S_OK;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev != plan->device) return OPT2S_ERR_DEVICE;
    const int bt = block_threads_now(h->algo, plan->only);
    if (g_block_threads > 0) {   // forced geometry: must fit the kernel
        int widest = 0;
        e = opt2s::max_block_threads(h->algo, h->skip_zeros, plan->only, &widest);
        if (e != cudaSuccess) return cuda_fail(e);
        if (bt > widest) return OPT2S_ERR_INVALID_ARG;
    }
    e = opt2s::launch_step(plan->d_chunks, plan->nchunks, h->algo, h->skip_zeros, plan->only,
                           make_scalars(h, step), bt, g_max_blocks, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return OPT2S_OK;
}

// ---------------------------------------------------------------------------
// Per-device plan cache for opt2s_step, keyed by the descriptor's contents.
// ---------------------------------------------------------------------------

struct CacheEntry {
    int device;
    int32_t algo;
    int64_t chunk_elems;
    bool unorm;                  // plan carries the bounded-update-norm workspace
    std::vector<opt2s_tensor> records;
    opt2s_plan* plan;
};

constexpr size_t kCacheCapacity = 16;
std::mutex g_cache_mu;
std::list<CacheEntry> g_cache;   // most recently used first

bool same_records(const CacheEntry& c, const TensorListDesc* d)
{
    return c.records.size() == static_cast<size_t>(d->count) &&
           (d->count == 0 ||
            std::memcmp(c.records.data(), d->tensors, sizeof(opt2s_tensor) * d->count) == 0);
}

bool all_empty(const TensorListDesc* d)
{
    for (int32_t i = 0; i < d->count; ++i)
        if (d->tensors[i].numel != 0) return false;
    return true;
}

}  // namespace

// ---------------------------------------------------------------------------
// Public entry points
// ---------------------------------------------------------------------------

namespace {

// The cached plan for `desc` on the current device (made on a miss); the
// caller holds g_cache_mu.  Argument errors are reported before device errors.
int cached_plan(const TensorListDesc* desc, int32_t algo, bool unorm, const opt2s_plan** out)
{
    int dev = 0;
    const int64_t ce = g_chunk_elems;   // part of the cache key: 0 = chosen per plan
    // a cache hit needs no device query: compare on the device of the most
    // recent entries first, then confirm the current device
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        // no usable device: still report argument errors first
        int vs = validate_desc(desc, algo);
        if (vs != OPT2S_OK) return vs;
        if (all_empty(desc)) { *out = nullptr; return OPT2S_OK; }
        return cuda_fail(e);
    }
    for (auto it = g_cache.begin(); it != g_cache.end(); ++it) {
        if (it->device == dev && it->algo == algo && it->chunk_elems == ce && it->unorm == unorm &&
            same_records(*it, desc)) {
            if (it != g_cache.begin()) g_cache.splice(g_cache.begin(), g_cache, it);
            *out = g_cache.front().plan;
            return OPT2S_OK;
        }
    }
    opt2s_plan* fresh = nullptr;
    int st = plan_create(desc, algo, &fresh, unorm);
    if (st != OPT2S_OK) return st;
    CacheEntry entry{dev, algo, ce, unorm,
                     std::vector<opt2s_tensor>(desc->tensors, desc->tensors + desc->count), fresh};
    g_cache.push_front(std::move(entry));
    while (g_cache.size() > kCacheCapacity) {
        plan_destroy(g_cache.back().plan);
        g_cache.pop_back();
    }
    *out = fresh;
    return OPT2S_OK;
}

// One step of a plan with per-tensor norms: the bounded update norm
// (lamb == false, max_unorm > 0) or LAMB (lamb == true, Adam moments, the
// weight decay inside the trust-ratio scaled update).
int plan_step_normed(const opt2s_plan* plan, const Hyper* h, bool lamb, float max_unorm, int step,
                     cudaStream_t stream)
{
    if (!plan) return OPT2S_ERR_INVALID_ARG;
    int st = validate_hyper(h, step);
    if (st != OPT2S_OK) return st;
    if (lamb ? h->algo != OPT2S_ADAM : (!std::isfinite(max_unorm) || !(max_unorm > 0.0f)))
        return OPT2S_ERR_INVALID_ARG;
    if (h->algo != plan->algo) return OPT2S_ERR_INVALID_ARG;
    if (plan->nchunks == 0) return OPT2S_OK;
    if (!plan->d_unorm) return OPT2S_ERR_INVALID_ARG;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev != plan->device) return OPT2S_ERR_DEVICE;
    const int bt = block_threads_now(h->algo, -1);
    if (g_block_threads > 0) {   // forced geometry: must fit the kernel
        int widest = 0;
        e = opt2s::max_block_threads_scaled(h->algo, h->skip_zeros, lamb ? 1 : 0, &widest);
        if (e != cudaSuccess) return cuda_fail(e);
        if (bt > widest) return OPT2S_ERR_INVALID_ARG;
    }
    if (lamb)
        e = opt2s::launch_step_lamb(plan->d_chunks, plan->nchunks, h->skip_zeros, make_scalars(h, step),
                                    h->weight_decay, plan->unorm, bt, g_max_blocks, stream);
    else
        e = opt2s::launch_step_max_unorm(plan->d_chunks, plan->nchunks, h->algo, h->skip_zeros,
                                         make_scalars(h, step), plan->unorm, max_unorm, bt,
                                         g_max_blocks, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    const int launched = (plan->unorm.nblocks > 0) + (plan->unorm.ngroups > 0) +
                         (plan->unorm.ntensors > 0) + 1;
    g_launches.fetch_add(launched, std::memory_order_relaxed);
    return OPT2S_OK;
}

}  // namespace

OPT2S_API int opt2s_step(const TensorListDesc* desc, const Hyper* hyper, int step,
                         cudaStream_t stream)
{
    OPT2S_RANGE("opt2s_step");
    int st = validate_hyper(hyper, step);
    if (st != OPT2S_OK) return st;
    if (!desc || desc->count < 0 || (desc->count > 0 && !desc->tensors))
        return OPT2S_ERR_INVALID_ARG;
    if (desc->count == 0) return OPT2S_OK;
    std::unique_lock<std::mutex> lock(g_cache_mu);
    const opt2s_plan* plan = nullptr;
    st = cached_plan(desc, hyper->algo, false, &plan);
    if (st != OPT2S_OK || !plan) return st;
    return plan_step(plan, hyper, step, stream);
}

OPT2S_API int opt2s_step_max_unorm(const TensorListDesc* desc, const Hyper* hyper, float max_unorm,
                                   int step, cudaStream_t stream)
{
    OPT2S_RANGE("opt2s_step_max_unorm");
    int st = validate_hyper(hyper, step);
    if (st != OPT2S_OK) return st;
    if (!std::isfinite(max_unorm) || !(max_unorm > 0.0f)) return OPT2S_ERR_INVALID_ARG;
    if (!desc || desc->count < 0 || (desc->count > 0 && !desc->tensors))
        return OPT2S_ERR_INVALID_ARG;
    if (desc->count == 0) return OPT2S_OK;
    std::unique_lock<std::mutex> lock(g_cache_mu);
    const opt2s_plan* plan = nullptr;
    st = cached_plan(desc, hyper->algo, true, &plan);
    if (st != OPT2S_OK || !plan) return st;
    return plan_step_normed(plan, hyper, false, max_unorm, step, stream);
}

OPT2S_API int opt2s_step_lamb(const TensorListDesc* desc, const Hyper* hyper, int step,
                              cudaStream_t stream)
{
    OPT2S_RANGE("opt2s_step_lamb");
    int st = validate_hyper(hyper, step);
    if (st != OPT2S_OK) return st;
    if (hyper->algo != OPT2S_ADAM) return OPT2S_ERR_INVALID_ARG;
    if (!desc || desc->count < 0 || (desc->count > 0 && !desc->tensors))
        return OPT2S_ERR_INVALID_ARG;
    if (desc->count == 0) return OPT2S_OK;
    std::unique_lock<std::mutex> lock(g_cache_mu);
    const opt2s_plan* plan = nullptr;
    st = cached_plan(desc, hyper->algo, true, &plan);   // the max_unorm step's tables
    if (st != OPT2S_OK || !plan) return st;
    return plan_step_normed(plan, hyper, true, 0.0f, step, stream);
}

OPT2S_API int opt2s_plan_create(const TensorListDesc* desc, int32_t algo, opt2s_plan** out_plan)
{
    if (!out_plan) return OPT2S_ERR_INVALID_ARG;
    *out_plan = nullptr;
    return plan_create(desc, algo, out_plan);
}

OPT2S_API int opt2s_plan_step(const opt2s_plan* plan, const Hyper* hyper, int step,
                              cudaStream_t stream)
{
    OPT2S_RANGE("opt2s_plan_step");
    return plan_step(plan, hyper, step, stream);
}

OPT2S_API int opt2s_plan_destroy(opt2s_plan* plan) { return plan_destroy(plan); }

OPT2S_API int64_t opt2s_plan_num_chunks(const opt2s_plan* plan) { return plan ? plan->nchunks : -1; }

static_assert(sizeof(opt2s_step_scalars) == sizeof(StepScalars), "scalar table layout");
static_assert(offsetof(opt2s_step_scalars, decay) == offsetof(StepScalars, decay), "scalar table layout");
static_assert(offsetof(opt2s_step_scalars, inv_bc1) == offsetof(StepScalars, inv_bc1), "scalar table layout");
static_assert(offsetof(opt2s_step_scalars, inv_bc2) == offsetof(StepScalars, inv_bc2), "scalar table layout");
static_assert(offsetof(opt2s_step_scalars, rcp_bc1_hi) == offsetof(StepScalars, rcp_bc1_hi), "scalar table layout");
static_assert(offsetof(opt2s_step_scalars, rcp_bc2_lo) == offsetof(StepScalars, rcp_bc2_lo), "scalar table layout");

OPT2S_API int opt2s_fill_step_scalars(const Hyper* hyper, int first_step, int count,
                                      opt2s_step_scalars* out)
{
    if (!out || count < 0) return OPT2S_ERR_INVALID_ARG;
    if (count > 0 && first_step > INT32_MAX - (count - 1)) return OPT2S_ERR_INVALID_ARG;
    int st = validate_hyper(hyper, first_step);
    if (st != OPT2S_OK) return st;
    for (int k = 0; k < count; ++k) {
        StepScalars s = make_scalars(hyper, first_step + k);
        opt2s::fill_reciprocals(&s);
        std::memcpy(&out[k], &s, sizeof(s));
    }
    return OPT2S_OK;
}

OPT2S_API int opt2s_plan_step_table(const opt2s_plan* plan, int32_t skip_zeros,
                                    const opt2s_step_scalars* d_table, int32_t table_len,
                                    int32_t* d_index, cudaStream_t stream)
{
    if (!plan || !d_table || !d_index || table_len < 1) return OPT2S_ERR_INVALID_ARG;
    if (skip_zeros != 0 && skip_zeros != 1) return OPT2S_ERR_INVALID_ARG;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev != plan->device) return OPT2S_ERR_DEVICE;
    const int bt = block_threads_now(plan->algo, plan->only);
    if (g_block_threads > 0) {
        int widest = 0;
        e = opt2s::max_block_threads(plan->algo, skip_zeros, plan->only, &widest);
        if (e != cudaSuccess) return cuda_fail(e);
        if (bt > widest) return OPT2S_ERR_INVALID_ARG;
    }
    e = opt2s::launch_step_table(plan->d_chunks, plan->nchunks, plan->algo, skip_zeros, plan->only,
                                 reinterpret_cast<const StepScalars*>(d_table), d_index, table_len,
                                 bt, g_max_blocks, stream);
    if (e != cudaSuccess) return cuda_fail(e);
    g_launches.fetch_add(plan->nchunks > 0 ? 2 : 1, std::memory_order_relaxed);
    return OPT2S_OK;
}

static_assert(OPT2S_MAX_WORLD == opt2s::kMaxWorld, "world limit");

OPT2S_API int opt2s_shard_range(int64_t numel, int32_t world, int32_t rank, int64_t* start,
                                int64_t* len)
{
    if (!start || !len || numel < 0 || world < 1 || world > OPT2S_MAX_WORLD || rank < 0 ||
        rank >= world)
        return OPT2S_ERR_INVALID_ARG;
    const int64_t units = (numel + 7) / 8;                 // 8-element units
    const int64_t u0 = units * rank / world, u1 = units * (rank + 1) / world;
    const int64_t a = std::min(u0 * 8, numel), b = std::min(u1 * 8, numel);
    *start = a;
    *len = b - a;
    return OPT2S_OK;
}

OPT2S_API int opt2s_shard_step(const opt2s_shard_desc* d, const Hyper* hyper, int step,
                               cudaStream_t stream)
{
    OPT2S_RANGE("opt2s_shard_step");
    int st = validate_hyper(hyper, step);
    if (st != OPT2S_OK) return st;
    if (!d || d->reserved != 0) return OPT2S_ERR_INVALID_ARG;
    int64_t start = 0, len = 0;
    if ((st = opt2s_shard_range(d->numel, d->world, d->rank, &start, &len)) != OPT2S_OK) return st;
    if (d->dtype != OPT2S_F32 && d->dtype != OPT2S_F16 && d->dtype != OPT2S_BF16)
        return OPT2S_ERR_INVALID_ARG;
    if (d->numel == 0) return OPT2S_OK;
    const int es = elem_bytes(d->dtype);
    std::vector<Range> ranges;
    const uintptr_t n = static_cast<uintptr_t>(d->numel);
    for (int q = 0; q < d->world; ++q) {
        const auto p = reinterpret_cast<uintptr_t>(d->params[q]);
        const auto g = reinterpret_cast<uintptr_t>(d->grads[q]);
        if (!p || !g || p % es || g % es) return OPT2S_ERR_INVALID_ARG;
        ranges.push_back({p, p + n * es, true});
        ranges.push_back({g, g + n * es, false});
    }
    if (len > 0) {
        const auto s1 = reinterpret_cast<uintptr_t>(d->state1);
        const auto s2 = reinterpret_cast<uintptr_t>(d->state2);
        if (!s1 || !s2 || s1 % 4 || s2 % 4) return OPT2S_ERR_INVALID_ARG;
        const uintptr_t k = static_cast<uintptr_t>(len);
        ranges.push_back({s1, s1 + (hyper->algo == OPT2S_ADEMAMIX ? 2 * k : k) * 4, true});
        ranges.push_back({s2, s2 + k * 4, true});
    }
    if ((st = opt2s::overlap_status(ranges.data(), ranges.size())) != OPT2S_OK) return st;
    if (len == 0) return OPT2S_OK;
    opt2s::ShardArgs a{};
    for (int q = 0; q < d->world; ++q) {
        a.params[q] = d->params[q];
        a.grads[q] = d->grads[q];
    }
    a.m = d->state1;
    a.v = d->state2;
    a.m2 = d->state1 + len;
    a.shard_start = start;
    a.shard_len = len;
    a.world = d->world;
    a.rank = d->rank;
    a.dtype = d->dtype;
    a.chunk_elems = static_cast<int32_t>(g_chunk_elems > 0 ? g_chunk_elems : opt2s::kDefaultChunkElems);
    cudaError_t e = opt2s::launch_shard_step(a, hyper->algo, hyper->skip_zeros, make_scalars(hyper, step),
                                             g_block_threads > 0 ? g_block_threads : opt2s::kAdamBlockThreads,
                                             stream);
    if (e != cudaSuccess) return cuda_fail(e);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return OPT2S_OK;
}

OPT2S_API int opt2s_release_cache(void)
{
    std::lock_guard<std::mutex> lock(g_cache_mu);
    int st = OPT2S_OK;
    for (CacheEntry& c : g_cache) {
        int s = plan_destroy(c.plan);
        if (s != OPT2S_OK) st = s;
    }
    g_cache.clear();
    opt2s::release_cache8();
    return st;
}

OPT2S_API const char* opt2s_error_string(int status)
{
    switch (status) {
    case OPT2S_OK: return "success";
    case OPT2S_ERR_INVALID_ARG: return "invalid argument";
    case OPT2S_ERR_ALIAS: return "a written buffer overlaps another buffer";
    case OPT2S_ERR_NO_MEMORY: return "out of memory for the launch tables";
    case OPT2S_ERR_CUDA: return "a CUDA call failed";
    case OPT2S_ERR_DEVICE: return "plan used on another device than it was created on";
    case OPT2S_ERR_TOO_LARGE: return "collection needs more chunks than a launch can index";
    default: return "unknown status";
    }
}

OPT2S_API int opt2s_last_cuda_error(void) { return t_last_cuda_error; }

OPT2S_API int opt2s_abi_version(void) { return OPT2S_ABI_VERSION; }

// ---------------------------------------------------------------------------
// Validation scaffolding (include/opt2s_testing.h)
// ---------------------------------------------------------------------------

OPT2S_API int opt2s_testing_build_chunks(const TensorListDesc* desc, int32_t algo,
                                         int64_t chunk_elems, opt2s_testing_chunk* out,
                                         int64_t cap, int64_t* out_count)
{
    if (!out_count) return OPT2S_ERR_INVALID_ARG;
    int st = validate_desc(desc, algo);
    if (st != OPT2S_OK) return st;
    const int64_t ce = chunk_elems > 0 ? chunk_elems : opt2s::kDefaultChunkElems;
    const int64_t n = count_chunks(desc, ce);
    *out_count = n;
    if (!out) return OPT2S_OK;
    if (cap < n) return OPT2S_ERR_INVALID_ARG;
    int64_t k = 0;
    for_each_chunk(desc, ce, [&](int32_t i, const opt2s_tensor& t, int64_t s, int64_t len) {
        out[k++] = opt2s_testing_chunk{i, s, len, t.dtype, 0};
    });
    return OPT2S_OK;
}

OPT2S_API int opt2s_testing_unorm_tables(const TensorListDesc* desc, int32_t algo, int64_t chunk_elems,
                                         uint32_t* group_ranges, uint32_t* first_group,
                                         uint32_t* chunk_tensor, int64_t* counts)
{
    if (!counts) return OPT2S_ERR_INVALID_ARG;
    int st = validate_desc(desc, algo);
    if (st != OPT2S_OK) return st;
    if (count_chunks(desc, opt2s::kNormBlockElems) > INT32_MAX) return OPT2S_ERR_TOO_LARGE;
    const int64_t ce = chunk_elems > 0 ? chunk_elems : opt2s::kDefaultChunkElems;
    const UnormTables t = unorm_tables(desc, ce);
    counts[0] = static_cast<int64_t>(t.blocks.size());
    counts[1] = static_cast<int64_t>(t.ranges.size() / 2);
    counts[2] = static_cast<int64_t>(t.chunk_tensor.size());
    if (group_ranges) std::copy(t.ranges.begin(), t.ranges.end(), group_ranges);
    if (first_group) std::copy(t.first_group.begin(), t.first_group.end(), first_group);
    if (chunk_tensor) std::copy(t.chunk_tensor.begin(), t.chunk_tensor.end(), chunk_tensor);
    return OPT2S_OK;
}

OPT2S_API int opt2s_testing_validate(const TensorListDesc* desc, const Hyper* hyper, int step)
{
    int st = validate_hyper(hyper, step);
    if (st != OPT2S_OK) return st;
    return validate_desc(desc, hyper->algo);
}

OPT2S_API int64_t opt2s_testing_default_chunk_elems(void) { return opt2s::kDefaultChunkElems; }

OPT2S_API int opt2s_testing_max_block_threads(int32_t algo, int32_t skip_zeros)
{
    if ((algo != OPT2S_ADAM && algo != OPT2S_ADEMAMIX) || (skip_zeros != 0 && skip_zeros != 1))
        return OPT2S_ERR_INVALID_ARG;
    int widest = 0;
    cudaError_t e = opt2s::max_block_threads(algo, skip_zeros, -1, &widest);
    if (e != cudaSuccess) return cuda_fail(e);
    return widest;
}

OPT2S_API int64_t opt2s_testing_choose_chunk_elems(const TensorListDesc* desc, int64_t resident_warps)
{
    if (!desc || desc->count < 0 || (desc->count > 0 && !desc->tensors)) return OPT2S_ERR_INVALID_ARG;
    return choose_chunk_elems(desc, resident_warps);
}

OPT2S_API int64_t opt2s_testing_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

// ---------------------------------------------------------------------------
// Shared with the other translation units (opt2s_internal.h)
// ---------------------------------------------------------------------------

int opt2s::record_cuda_error(cudaError_t e) { return cuda_fail(e); }

void opt2s::count_launches(int64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

#ifdef OPT2S_TESTING
// ---------------------------------------------------------------------------
// Forcing knobs, fault injection and the division check: test build only
// ---------------------------------------------------------------------------

OPT2S_API int64_t opt2s_testing_set_chunk_elems(int64_t chunk_elems)
{
    const int64_t prev = g_chunk_elems;
    if (chunk_elems >= 0 && chunk_elems % 8 == 0 && chunk_elems <= (int64_t(1) << 31))
        g_chunk_elems = chunk_elems;
    return prev;
}

OPT2S_API int opt2s_testing_set_launch(int block_threads, int max_blocks)
{
    if (block_threads != 0 && (block_threads < 32 || block_threads > 1024 || block_threads % 32))
        return OPT2S_ERR_INVALID_ARG;
    if (max_blocks < 0) return OPT2S_ERR_INVALID_ARG;
    g_block_threads = block_threads;
    g_max_blocks = max_blocks;
    return OPT2S_OK;
}

OPT2S_API int opt2s_testing_fail_allocs(int count)
{
    if (count < 0) return OPT2S_ERR_INVALID_ARG;
    g_fail_allocs.store(count);
    return OPT2S_OK;
}

OPT2S_API int opt2s_testing_check_division(uint64_t seed, int64_t n, int32_t mode,
                                           int64_t* mismatches)
{
    if (!mismatches || n < 0 || mode < 0 || mode > 2) return OPT2S_ERR_INVALID_ARG;
    if (mode == 2 && n > (int64_t{1} << 20)) return OPT2S_ERR_INVALID_ARG;   // n * 2^32 operands
    unsigned long long* d_count = nullptr;
    cudaError_t e = cudaMalloc(&d_count, sizeof(*d_count));
    if (e != cudaSuccess) return cuda_fail(e);
    unsigned long long h = 0;
    e = cudaMemset(d_count, 0, sizeof(*d_count));
    if (e == cudaSuccess) e = opt2s::check_division(seed, n, mode, d_count, 0);
    if (e == cudaSuccess) e = cudaMemcpy(&h, d_count, sizeof(h), cudaMemcpyDeviceToHost);
    cudaFree(d_count);
    if (e != cudaSuccess) return cuda_fail(e);
    *mismatches = static_cast<int64_t>(h);
    return OPT2S_OK;
}
#endif  // OPT2S_TESTING
