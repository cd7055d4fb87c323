// opt2s_api8.cpp -- the C ABI of the 8-bit-state step (include/opt2s.h,
// opt2s_step_8bit): validation, the block and chunk tables, and their
// per-device cache.
//
// The collection mixes tensors whose state is stored in 8 bits (Dettmers et
// al., "8-bit Optimizers via Block-wise Quantization", ICLR 2022: blocks of
// 2,048 elements with one absmax each) and small tensors whose state stays
// fp32 (the min_8bit_size routing of the bitsandbytes issue "Investigate a
// 256-thread SM103 path for small 32-bit optimizer tensors", section
// "Problem").  The host turns it into two tables once -- one record per 8-bit
// block, one per 32-bit chunk -- and every later step is one launch that
// reads them.

#include <cstring>
#include <list>
#include <mutex>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "opt2s.h"
#include "opt2s_internal.h"

#define OPT2S_API extern "C" __attribute__((visibility("default")))

namespace {

using opt2s::Block8Rec;
using opt2s::ChunkRec;
using opt2s::Range;

// 32-bit chunks of the small tensors: 256 elements, so that eight of them
// (one work unit, a warp each) are about one 8-bit block's work.
constexpr int64_t kChunk32 = 256;

int64_t nblocks8(int64_t n) { return (n + opt2s::kBlock8Elems - 1) / opt2s::kBlock8Elems; }

// One record: well formed, and its buffers' address ranges (up to 6).
int record8_ranges(const opt2s_tensor8& t, int32_t algo, Range* out, int* n)
{
    *n = 0;
    if (t.numel < 0) return OPT2S_ERR_INVALID_ARG;
    if (t.dtype != OPT2S_F32 && t.dtype != OPT2S_F16 && t.dtype != OPT2S_BF16)
        return OPT2S_ERR_INVALID_ARG;
    if (t.state_bits != 8 && t.state_bits != 32) return OPT2S_ERR_INVALID_ARG;
    const bool eight = t.state_bits == 8;
    if (!eight && (t.absmax1 || t.absmax2)) return OPT2S_ERR_INVALID_ARG;
    if (t.numel == 0) return OPT2S_OK;
    if (t.numel > (int64_t(1) << 40)) return OPT2S_ERR_INVALID_ARG;
    if (!t.param || !t.grad || !t.state1 || !t.state2) return OPT2S_ERR_INVALID_ARG;
    if (eight && (!t.absmax1 || !t.absmax2)) return OPT2S_ERR_INVALID_ARG;
    const int es = opt2s::elem_bytes(t.dtype);
    const auto p = reinterpret_cast<uintptr_t>(t.param);
    const auto g = reinterpret_cast<uintptr_t>(t.grad);
    const auto s1 = reinterpret_cast<uintptr_t>(t.state1);
    const auto s2 = reinterpret_cast<uintptr_t>(t.state2);
    if (p % es || g % es) return OPT2S_ERR_INVALID_ARG;
    const uintptr_t k = static_cast<uintptr_t>(t.numel);
    const uintptr_t copies = algo == OPT2S_ADEMAMIX ? 2 : 1;   // [m1 | m2] in state1
    const uintptr_t sb = eight ? 1 : 4;                          // bytes a state element
    if (!eight && (s1 % 4 || s2 % 4)) return OPT2S_ERR_INVALID_ARG;
    out[(*n)++] = {p, p + k * es, true};
    out[(*n)++] = {g, g + k * es, false};
    out[(*n)++] = {s1, s1 + copies * k * sb, true};
    out[(*n)++] = {s2, s2 + k * sb, true};
    if (eight) {
        const auto a1 = reinterpret_cast<uintptr_t>(t.absmax1);
        const auto a2 = reinterpret_cast<uintptr_t>(t.absmax2);
        if (a1 % 4 || a2 % 4) return OPT2S_ERR_INVALID_ARG;
        const uintptr_t nb = static_cast<uintptr_t>(nblocks8(t.numel));
        out[(*n)++] = {a1, a1 + copies * nb * 4, true};
        out[(*n)++] = {a2, a2 + nb * 4, true};
    }
    return OPT2S_OK;
}

int validate8(const TensorListDesc8* d, int32_t algo)
{
    if (!d || d->count < 0 || (d->count > 0 && !d->tensors)) return OPT2S_ERR_INVALID_ARG;
    if (algo != OPT2S_ADAM && algo != OPT2S_ADEMAMIX) return OPT2S_ERR_INVALID_ARG;
    std::vector<Range> ranges;
    for (int32_t i = 0; i < d->count; ++i) {
        Range r[6];
        int n = 0;
        const int st = record8_ranges(d->tensors[i], algo, r, &n);
        if (st != OPT2S_OK) return st;
        ranges.insert(ranges.end(), r, r + n);
    }
    return opt2s::overlap_status(ranges.data(), ranges.size());
}

struct Plan8 {
    int device;
    int32_t algo;
    int64_t nblocks, nchunks;
    void* d_mem;                 // Block8Rec[nblocks] then ChunkRec[nchunks]
    std::vector<opt2s_tensor8> records;
};

// Tables of `d` (validated): one Block8Rec per 2,048-element block of every
// 8-bit tensor, one ChunkRec per kChunk32 elements of every 32-bit tensor, in
// descriptor order.
void build_tables(const TensorListDesc8* d, std::vector<Block8Rec>* blocks, std::vector<ChunkRec>* chunks)
{
    for (int32_t i = 0; i < d->count; ++i) {
        const opt2s_tensor8& t = d->tensors[i];
        const int es = opt2s::elem_bytes(t.dtype);
        if (t.state_bits == 8) {
            auto* q1 = static_cast<uint8_t*>(t.state1);
            auto* q2 = static_cast<uint8_t*>(t.state2);
            const int64_t nb = nblocks8(t.numel);
            for (int64_t b = 0; b < nb; ++b) {
                const int64_t s = b * opt2s::kBlock8Elems;
                Block8Rec r;
                r.p = static_cast<char*>(t.param) + s * es;
                r.g = static_cast<const char*>(t.grad) + s * es;
                r.q1 = q1 + s;
                r.q2 = q2 + s;
                r.q3 = q1 + t.numel + s;
                r.a1 = t.absmax1 + b;
                r.a2 = t.absmax2 + b;
                r.a3 = t.absmax1 + nb + b;
                r.len = static_cast<uint32_t>(std::min<int64_t>(opt2s::kBlock8Elems, t.numel - s));
                r.dtype = t.dtype;
                blocks->push_back(r);
            }
        } else {
            auto* s1 = static_cast<float*>(t.state1);
            auto* s2 = static_cast<float*>(t.state2);
            for (int64_t s = 0; s < t.numel; s += kChunk32) {
                ChunkRec r;
                r.p = static_cast<char*>(t.param) + s * es;
                r.g = static_cast<const char*>(t.grad) + s * es;
                r.m = s1 + s;
                r.v = s2 + s;
                r.m2 = s1 + t.numel + s;
                r.len = static_cast<uint32_t>(std::min<int64_t>(kChunk32, t.numel - s));
                r.dtype = t.dtype;
                chunks->push_back(r);
            }
        }
    }
}

int plan8_create(const TensorListDesc8* d, int32_t algo, int dev, Plan8** out)
{
    std::vector<Block8Rec> blocks;
    std::vector<ChunkRec> chunks;
    build_tables(d, &blocks, &chunks);
    if (blocks.size() + (chunks.size() + 7) / 8 > static_cast<size_t>(INT32_MAX)) return OPT2S_ERR_TOO_LARGE;
    auto* plan = new (std::nothrow) Plan8{dev, algo, static_cast<int64_t>(blocks.size()),
                                          static_cast<int64_t>(chunks.size()), nullptr,
                                          std::vector<opt2s_tensor8>(d->tensors, d->tensors + d->count)};
    if (!plan) return OPT2S_ERR_NO_MEMORY;
    const size_t bb = blocks.size() * sizeof(Block8Rec), cb = chunks.size() * sizeof(ChunkRec);
    if (bb + cb > 0) {
        cudaError_t e = cudaMalloc(&plan->d_mem, bb + cb);
        if (e != cudaSuccess) {
            delete plan;
            if (e == cudaErrorMemoryAllocation) { opt2s::record_cuda_error(e); return OPT2S_ERR_NO_MEMORY; }
            return opt2s::record_cuda_error(e);
        }
        if (bb) e = cudaMemcpy(plan->d_mem, blocks.data(), bb, cudaMemcpyHostToDevice);
        if (e == cudaSuccess && cb)
            e = cudaMemcpy(static_cast<char*>(plan->d_mem) + bb, chunks.data(), cb, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) {
            cudaFree(plan->d_mem);
            delete plan;
            return opt2s::record_cuda_error(e);
        }
    }
    *out = plan;
    return OPT2S_OK;
}

void plan8_destroy(Plan8* plan)
{
    if (!plan) return;
    if (plan->d_mem) {
        int cur = -1;
        const bool switched = cudaGetDevice(&cur) == cudaSuccess && cur != plan->device;
        if (switched) cudaSetDevice(plan->device);
        cudaFree(plan->d_mem);                       // waits for the device
        if (switched) cudaSetDevice(cur);
    }
    delete plan;
}

constexpr size_t kCache8Capacity = 16;
std::mutex g_cache8_mu;
std::list<Plan8*> g_cache8;   // most recently used first

bool same8(const Plan8& p, const TensorListDesc8* d)
{
    return p.records.size() == static_cast<size_t>(d->count) &&
           (d->count == 0 ||
            std::memcmp(p.records.data(), d->tensors, sizeof(opt2s_tensor8) * d->count) == 0);
}

}  // namespace

OPT2S_API int opt2s_step_8bit(const TensorListDesc8* desc, const Hyper* hyper, int step,
                              cudaStream_t stream)
{
    OPT2S_RANGE("opt2s_step_8bit");
    int st = opt2s::validate_hyper(hyper, step);
    if (st != OPT2S_OK) return st;
    if (!desc || desc->count < 0 || (desc->count > 0 && !desc->tensors)) return OPT2S_ERR_INVALID_ARG;
    if (desc->count == 0) return OPT2S_OK;
    std::lock_guard<std::mutex> lock(g_cache8_mu);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    Plan8* plan = nullptr;
    if (e == cudaSuccess) {
        for (auto it = g_cache8.begin(); it != g_cache8.end(); ++it) {
            if ((*it)->device == dev && (*it)->algo == hyper->algo && same8(**it, desc)) {
                plan = *it;
                if (it != g_cache8.begin()) g_cache8.splice(g_cache8.begin(), g_cache8, it);
                break;
            }
        }
    }
    if (!plan) {
        if ((st = validate8(desc, hyper->algo)) != OPT2S_OK) return st;   // argument errors first
        if (e != cudaSuccess) return opt2s::record_cuda_error(e);
        if ((st = plan8_create(desc, hyper->algo, dev, &plan)) != OPT2S_OK) return st;
        g_cache8.push_front(plan);
        while (g_cache8.size() > kCache8Capacity) {
            plan8_destroy(g_cache8.back());
            g_cache8.pop_back();
        }
    }
    if (plan->nblocks + plan->nchunks == 0) return OPT2S_OK;
    const auto* d_blocks = static_cast<const Block8Rec*>(plan->d_mem);
    const auto* d_chunks = reinterpret_cast<const ChunkRec*>(static_cast<const char*>(plan->d_mem) +
                                                             plan->nblocks * sizeof(Block8Rec));
    e = opt2s::launch_step8(d_blocks, plan->nblocks, d_chunks, plan->nchunks, hyper->algo,
                            hyper->skip_zeros, opt2s::make_scalars(hyper, step), 0, stream);
    if (e != cudaSuccess) return opt2s::record_cuda_error(e);
    opt2s::count_launches(1);
    return OPT2S_OK;
}

OPT2S_API int opt2s_8bit_state_bits(int64_t numel, int64_t min_8bit_size)
{
    if (min_8bit_size <= 0) min_8bit_size = OPT2S_MIN_8BIT_SIZE;
    return numel >= min_8bit_size ? 8 : 32;
}

void opt2s::release_cache8()
{
    std::lock_guard<std::mutex> lock(g_cache8_mu);
    for (Plan8* p : g_cache8) plan8_destroy(p);
    g_cache8.clear();
}
