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

#include <algorithm>
#include <cmath>
#include <cstring>
#include <list>
#include <mutex>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "opt2s.h"
#include "opt2s_internal.h"
#include "opt2s_testing.h"

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

// ---------------------------------------------------------------------------
// Quantization tables (the layout is described in opt2s_internal.h)
// ---------------------------------------------------------------------------

// The 256 values of a map, ascending: for E = 0..6 and F = 6 - E (signed) or
// 7 - E (unsigned) fraction bits, 10^-E * (0.1 + 0.9*(2f+1)/2^(F+1)) for
// f = 0 .. 2^F - 1 (both signs when signed), plus 0 and 1.0 -- Dettmers et
// al. 2022, sections 2.2 (dynamic tree quantization) and 2.3 (dynamic
// quantization).  Each value is N/D with N = 2^(F+1) + 9*(2f+1) and
// D = 10^(E+1)*2^(F+1), exact binary32 integers: one IEEE division.
void quant_map(bool is_signed, float* out)
{
    int k = 0;
    const int f0 = is_signed ? 6 : 7;
    for (int E = 0; E <= 6; ++E) {
        const int F = f0 - E;
        float D = static_cast<float>(1 << (F + 1));
        for (int e = 0; e <= E; ++e) D *= 10.0f;
        for (int f = 0; f < (1 << F); ++f) {
            const float v = static_cast<float>((1 << (F + 1)) + 9 * (2 * f + 1)) / D;
            out[k++] = v;
            if (is_signed) out[k++] = -v;
        }
    }
    out[k++] = 0.0f;
    out[k++] = 1.0f;
    std::sort(out, out + k);
}

// The binary32 number at or below the exact midpoint of map[j] and map[j+1]
// (binary64 holds the midpoint exactly).
float threshold(const float* map, int j)
{
    const double mid = (static_cast<double>(map[j]) + static_cast<double>(map[j + 1])) * 0.5;
    float t = static_cast<float>(mid);
    if (static_cast<double>(t) > mid) t = std::nextafter(t, -INFINITY);
    return t;
}

// Number of thresholds below x (or at or below it, with `or_equal`).
int thresholds_below(const float* thr, float x, bool or_equal)
{
    return static_cast<int>(or_equal ? std::upper_bound(thr, thr + 255, x) - thr
                                     : std::lower_bound(thr, thr + 255, x) - thr);
}

uint32_t bits_of(float x)
{
    uint32_t u;
    std::memcpy(&u, &x, sizeof u);
    return u;
}

float float_of(uint32_t u)
{
    float x;
    std::memcpy(&x, &u, sizeof x);
    return x;
}

// Slice i of the map with thresholds `thr`, for x of sign `neg`: the code at
// the slice's low end (in value order) in the high 16 bits, and in the low 16
// a value c such that code(x) = (entry + l) >> 16 for l = the low 16 bits of
// x's magnitude, complemented when x < 0.  With t the low 16 bits of the
// slice's threshold magnitude: for x >= 0 the code is base + (l > t), and
// c = 0xFFFF - t makes the carry out of the low half exactly (l > t); for
// x < 0 it is base + (low16 < t) = base + (l > 0xFFFF - t), and c = t.  A
// slice without a threshold has c = 0 (never a carry).
uint32_t slice_entry(const float* thr, uint32_t zero_code, int i, bool neg)
{
    const int r = i >> 7, k = i & 127;
    if (r == 0) return zero_code << 16;                              // |x| < 2^-23
    if (r == opt2s::kQuantRows - 1) return 0;                        // NaN: code 0
    const uint32_t lo_bits = static_cast<uint32_t>(r - 1 + 127 - 23) << 23 | static_cast<uint32_t>(k) << 16;
    const float lo = float_of(lo_bits), hi = float_of(lo_bits + (1u << 16));
    uint32_t c = 0;
    int base;
    if (!neg) {
        // x in [lo, hi): thresholds below lo count; at most one lies in [lo, hi)
        base = thresholds_below(thr, lo, false);
        if (base < 255 && thr[base] < hi) c = 0xFFFFu - (bits_of(thr[base]) & 0xFFFFu);
    } else {
        // x in (-hi, -lo]: thresholds at or below -hi count; at most one lies
        // in (-hi, -lo) and counts when |x| is below its magnitude
        base = thresholds_below(thr, -hi, true);
        if (base < 255 && thr[base] < -lo) c = bits_of(-thr[base]) & 0xFFFFu;
    }
    return static_cast<uint32_t>(base) << 16 | c;
}

}  // namespace

void opt2s::build_quant_tables(uint32_t* out)
{
    float smap[256], umap[256], sthr[255], uthr[255];
    quant_map(true, smap);
    quant_map(false, umap);
    for (int j = 0; j < 255; ++j) {
        sthr[j] = threshold(smap, j);
        uthr[j] = threshold(umap, j);
    }
    constexpr int kSlices = opt2s::kQuantRows * 128;
    std::memcpy(out, smap, sizeof smap);
    std::memcpy(out + 256, umap, sizeof umap);
    for (int i = 0; i < kSlices; ++i) {
        out[512 + i] = slice_entry(sthr, 127, i, false);
        out[512 + kSlices + i] = slice_entry(sthr, 127, i, true);
        out[512 + 2 * kSlices + i] = slice_entry(uthr, 0, i, false);
    }
}

namespace {

struct Plan8 {
    int device;
    int32_t algo;
    int64_t nblocks, nchunks;
    void* d_mem;                 // quantization tables, Block8Rec[nblocks], ChunkRec[nchunks]
    std::vector<opt2s_tensor8> records;
};

constexpr size_t kTableBytes = opt2s::kQuantTableWords * sizeof(uint32_t);   // a multiple of 16

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
    std::vector<uint32_t> tables(opt2s::kQuantTableWords);
    opt2s::build_quant_tables(tables.data());
    cudaError_t e = cudaMalloc(&plan->d_mem, kTableBytes + bb + cb);
    if (e != cudaSuccess) {
        delete plan;
        if (e == cudaErrorMemoryAllocation) { opt2s::record_cuda_error(e); return OPT2S_ERR_NO_MEMORY; }
        return opt2s::record_cuda_error(e);
    }
    char* at = static_cast<char*>(plan->d_mem);
    e = cudaMemcpy(at, tables.data(), kTableBytes, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && bb) e = cudaMemcpy(at + kTableBytes, blocks.data(), bb, cudaMemcpyHostToDevice);
    if (e == cudaSuccess && cb) e = cudaMemcpy(at + kTableBytes + bb, chunks.data(), cb, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        cudaFree(plan->d_mem);
        delete plan;
        return opt2s::record_cuda_error(e);
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
    const char* at = static_cast<const char*>(plan->d_mem);
    const auto* d_tables = reinterpret_cast<const uint32_t*>(at);
    const auto* d_blocks = reinterpret_cast<const Block8Rec*>(at + kTableBytes);
    const auto* d_chunks = reinterpret_cast<const ChunkRec*>(at + kTableBytes + plan->nblocks * sizeof(Block8Rec));
    e = opt2s::launch_step8(d_blocks, plan->nblocks, d_chunks, plan->nchunks, d_tables, hyper->algo,
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

OPT2S_API int opt2s_testing_quant_tables(uint32_t* out, int64_t cap)
{
    if (!out || cap < opt2s::kQuantTableWords) return OPT2S_ERR_INVALID_ARG;
    opt2s::build_quant_tables(out);
    return OPT2S_OK;
}
