// Internal declarations shared by the host API (opt2s_api.cpp), the kernel
// translation unit (opt2s_kernel.cu) and the no-allocation entry point
// (opt2s_noalloc.cu).  Not installed, not public.
#pragma once

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cuda_runtime.h>

#include "opt2s.h"

// Optional NVTX ranges around the host side of each step entry point, for
// timeline tools (build with -DOPT2S_NVTX; NVTX v3 is header-only and costs
// nothing when no tool is attached).  Without the flag they compile away.
#ifdef OPT2S_NVTX
#include <nvtx3/nvToolsExt.h>
namespace opt2s {
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace opt2s
#define OPT2S_RANGE(name) ::opt2s::NvtxRange opt2s_nvtx_range_(name)
#else
#define OPT2S_RANGE(name) ((void)0)
#endif

namespace opt2s {

enum : int { kF32 = 0, kF16 = 1, kBF16 = 2 };
enum : int { kAdam = 0, kAdEMAMix = 1 };

// One work unit of a launch: a contiguous element range [0, len) of one
// tensor, with every pointer already offset to the first element of the
// range.  A warp processes one chunk at a time.
struct alignas(16) ChunkRec {
    void* p;          // param (storage dtype)
    const void* g;    // grad  (storage dtype), read only
    float* m;         // state1 (Adam m, AdEMAMix m1)
    float* v;         // state2
    float* m2;        // state1 + numel (AdEMAMix m2); not read by Adam
    uint32_t len;     // elements in the chunk, >= 1
    int32_t dtype;    // kF32 / kF16 / kBF16, 16-bit ones possibly | kShortFlag
};
static_assert(sizeof(ChunkRec) == 48, "ChunkRec layout");

// Per-step scalars, all fp32 (the bias corrections and decay are evaluated in
// double on the host and rounded once).
struct StepScalars {
    float lr;
    float beta1, beta2, beta3;
    float one_minus_beta1, one_minus_beta2, one_minus_beta3;
    float alpha;
    float eps;
    float bc1, bc2;
    float decay;
    // RN64(1/bc1), RN64(1/bc2), and each split into an fp32 pair
    // (RN32(r), RN32(r - RN32(r))): filled in at launch from bc1/bc2 (both in
    // [2^-25, 1]); the kernels divide by bc1, bc2 exactly through them (see
    // div_by_constant in opt2s_device.cuh)
    double inv_bc1, inv_bc2;
    float rcp_bc1_hi, rcp_bc1_lo, rcp_bc2_hi, rcp_bc2_lo;
};

// Threads per block.  Adam's generic kernel (96 registers) fits 20 resident
// warps per SM as 128-thread blocks (16 as 256-thread blocks); AdEMAMix's (120
// registers) fits 16 warps either way and measured faster as 256-thread blocks;
// Adam specialised to one 16-bit dtype moves two 16-byte param vectors a lane
// per iteration (about 104 registers) and measured fastest as 256-thread
// blocks.  `only` is the dtype every chunk of a plan shares, or -1.
constexpr int kAdamBlockThreads = 128;
constexpr int kAdEMAMixBlockThreads = 256;
constexpr int kSpecialisedBlockThreads = 256;
constexpr int kDefaultBlockThreads = 128;      // the no-alloc entry point's width
// Only Adam over one 16-bit dtype has a specialised kernel.  Kernels
// specialised to fp32 storage (Adam, 78 registers) and to one dtype for
// AdEMAMix (80-90 registers) were built and measured slower on 268 M-element
// steps (4 % and 13 %): they fill more warp slots per SM, and these streaming
// steps ran faster with fewer.
inline int kernel_only(int algo, int uniform_dtype)
{
    return (algo == kAdam && (uniform_dtype == kF16 || uniform_dtype == kBF16)) ? uniform_dtype : -1;
}
inline int default_block_threads(int algo, int only)
{
    if (only >= 0) return kSpecialisedBlockThreads;
    return algo == kAdEMAMix ? kAdEMAMixBlockThreads : kAdamBlockThreads;
}
constexpr int64_t kDefaultChunkElems = 2048;   // largest chunk the plan builder picks
constexpr int64_t kMinChunkElems = 128;        // one 16-byte fp32 vector per lane

// A plan whose chunk length is at most kShortChunkElems marks its 16-bit
// chunks (dtype | kShortFlag) for the short-chunk path: 4 elements per lane
// with element-wise accesses instead of one 16-byte vector of 8.  The chunk
// length chooser picks such a length for a plan with 16-bit tensors only when
// the plan fits in one wave of warps, where each lane's serial work decides.
constexpr uint32_t kShortChunkElems = 128;
enum : int { kShortFlag = 8 };

// The sharded (ZeRO-style) step of one rank.  Every rank holds the whole flat
// param and grad buffers (same layout); this rank updates the elements
// [shard_start, shard_start + shard_len) with the rank-order mean of all
// ranks' gradients and writes the new values into every rank's param buffer.
constexpr int kMaxWorld = 8;
struct ShardArgs {
    void* params[kMaxWorld];        // rank q's flat param buffer, addressable here
    const void* grads[kMaxWorld];   // rank q's flat grad buffer, addressable here
    float* m;                       // this rank's shard state (shard-relative)
    float* v;
    float* m2;                      // AdEMAMix: m + shard_len
    int64_t shard_start;
    int64_t shard_len;
    int32_t world;
    int32_t rank;
    int32_t dtype;
    int32_t chunk_elems;
};

cudaError_t launch_shard_step(const ShardArgs& a, int algo, int skip_zeros, const StepScalars& s,
                              int block_threads, cudaStream_t stream);

// Launches one step over `nchunks` records at `d_chunks` (device memory) on
// `stream`.  block_threads: multiple of 32; max_blocks <= 0: occupancy-based
// cap (resident blocks per SM x SM count).  Returns the launch status.
cudaError_t launch_step(const ChunkRec* d_chunks, int64_t nchunks, int algo,
                        int skip_zeros, int only, const StepScalars& s,
                        int block_threads, int max_blocks,
                        cudaStream_t stream);

// The bounded-update-norm step (max_unorm > 0).  Device arrays, all owned
// by the plan: `blocks` is the norm table (each tensor cut into blocks of
// kNormBlockElems elements, in descriptor order) with two doubles of
// `partial` per block; a tensor's blocks form groups of kNormGroupBlocks
// consecutive blocks, group q spanning blocks [group_range[2q],
// group_range[2q + 1]) with two doubles of `group_sum`; tensor t owns groups
// [first_group[t], first_group[t + 1]); `scale` holds one float per tensor,
// and chunk_tensor[c] is the tensor of the plan's chunk c.
constexpr int64_t kNormBlockElems = 2048;
constexpr int64_t kNormGroupBlocks = 64;
struct UnormArgs {
    const ChunkRec* blocks;
    int64_t nblocks;
    double* partial;               // 2 * nblocks
    const uint32_t* group_range;   // 2 * ngroups
    int64_t ngroups;
    double* group_sum;             // 2 * ngroups
    const uint32_t* first_group;   // ntensors + 1 entries
    int32_t ntensors;
    float* scale;                  // ntensors
    const uint32_t* chunk_tensor;  // one per chunk of the plan
};

// Launches the four kernels of the bounded-update-norm step on `stream`
// (block sums, group sums, per-tensor scales, the scaled step over the plan's
// chunks).
cudaError_t launch_step_max_unorm(const ChunkRec* d_chunks, int64_t nchunks, int algo,
                                  int skip_zeros, const StepScalars& s, const UnormArgs& u,
                                  float max_unorm, int block_threads, int max_blocks,
                                  cudaStream_t stream);

// Launches the four kernels of the LAMB step (Adam moments) on `stream`: the
// same tables and launches, with the sums of (u + weight_decay*p)^2, the
// trust ratio ||p|| / ||u + weight_decay*p|| per tensor, and
// p = p - lr*(ratio*(u + weight_decay*p)).
cudaError_t launch_step_lamb(const ChunkRec* d_chunks, int64_t nchunks, int skip_zeros,
                             const StepScalars& s, float weight_decay, const UnormArgs& u,
                             int block_threads, int max_blocks, cudaStream_t stream);

// Widest block the scaled step kernel (bounded norm, or LAMB when `lamb`)
// can launch with.
cudaError_t max_block_threads_scaled(int algo, int skip_zeros, int lamb, int* out);

// The step with 8-bit blockwise state.  A tensor with 8-bit state is cut
// into blocks of kBlock8Elems elements; each block is one record, stepped by
// one CTA: its param and grad (storage dtype), its codes of m (q1), v (q2)
// and, for AdEMAMix, m2 (q3), and the block's absmax of each (a1, a2, a3: one
// float each), all offset to the block's first element.  Small tensors with
// fp32 state are ChunkRec chunks of the same launch.
constexpr int64_t kBlock8Elems = 2048;
struct alignas(16) Block8Rec {
    void* p;
    const void* g;
    uint8_t* q1;
    uint8_t* q2;
    uint8_t* q3;      // AdEMAMix: codes of m2; not read by Adam
    float* a1;
    float* a2;
    float* a3;        // AdEMAMix: absmax of m2
    uint32_t len;     // elements in the block, 1..kBlock8Elems
    int32_t dtype;
};
static_assert(sizeof(Block8Rec) == 80, "Block8Rec layout");

// The quantization tables of the 8-bit step, as 32-bit words: the signed
// and the unsigned map (256 binary32 values each, ascending), then the slice
// entries (kQuantRows x 128 each) of the signed map for x >= 0 and for x < 0
// and of the unsigned map.  A slice entry is (code at the slice's low end in
// value order) << 16 | (low 16 bits of the magnitude of the one threshold
// inside the slice, or a value whose compare never holds).  Built on the host
// by build_quant_tables (opt2s_api8.cpp) and copied into every CTA's shared
// memory.
constexpr int kQuantRows = 26;
constexpr int kQuantTableWords = 512 + 3 * kQuantRows * 128;

// Fills `out` (kQuantTableWords words) with the tables above.
void build_quant_tables(uint32_t* out);

// Launches one 8-bit-state step on `stream`: `nblocks` block records,
// `nchunks` 32-bit chunk records and the quantization tables (device memory,
// 16-byte aligned).  max_blocks <= 0: the occupancy cap (resident CTAs per SM
// x SMs).
cudaError_t launch_step8(const Block8Rec* d_blocks, int64_t nblocks, const ChunkRec* d_chunks,
                         int64_t nchunks, const uint32_t* d_tables, int algo, int skip_zeros,
                         const StepScalars& s, int max_blocks, cudaStream_t stream);

// Frees the cached plans of the 8-bit-state step (opt2s_api8.cpp); called by
// opt2s_release_cache.
void release_cache8();

// Sets s->inv_bc1, s->inv_bc2 = RN64(1/bc1), RN64(1/bc2) and their fp32
// splits rcp_bc*_hi = RN32(inv), rcp_bc*_lo = RN32(inv - hi) (host).
void fill_reciprocals(StepScalars* s);

// Launches one step whose scalars are d_table[*d_index] (device memory),
// followed by a one-thread launch that advances *d_index (to -1 after the
// last entry).  Both launches may be captured in a CUDA graph.
cudaError_t launch_step_table(const ChunkRec* d_chunks, int64_t nchunks, int algo,
                              int skip_zeros, int only, const StepScalars* d_table, int* d_index,
                              int table_len, int block_threads, int max_blocks,
                              cudaStream_t stream);

// Resident warps of the step kernel for (algo, skip_zeros) on the current
// device at `block_threads` threads per block (blocks per SM x SMs x warps).
cudaError_t resident_warps(int algo, int skip_zeros, int only, int block_threads, int64_t* out);

// Widest block (threads, a multiple of 32) the step kernel for (algo,
// skip_zeros) can be launched with: its registers per thread limit it.
cudaError_t max_block_threads(int algo, int skip_zeros, int only, int* out);

// Validation scaffolding: counts into *d_count (device memory) the operands
// among n seeded random ones for which the kernel's constant division differs
// from __fdiv_rn (mode 0: any x; mode 1: x/d near a rounding boundary).
cudaError_t check_division(uint64_t seed, int64_t n, int mode, unsigned long long* d_count,
                           cudaStream_t stream);

// Number of blocks a launch of `nchunks` chunks uses on the current device.
cudaError_t grid_for(int64_t nchunks, int algo, int skip_zeros, int only,
                     int block_threads, int max_blocks, int* grid);

// ---------------------------------------------------------------------------
// Host-side rules every entry point applies, in one place.  None of them
// touches the heap, so the no-allocation entry point uses them too.
// ---------------------------------------------------------------------------

inline int elem_bytes(int32_t dtype) { return dtype == OPT2S_F32 ? 4 : 2; }

// Hyper-parameters and step number of one call.
inline int validate_hyper(const Hyper* h, int step)
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

// The per-step scalars: bias corrections and decay evaluated in double and
// rounded to fp32 once, 1 - beta as fp32 subtractions.  The reciprocals of
// the bias corrections are filled in at launch (fill_reciprocals).
inline StepScalars make_scalars(const Hyper* h, int step)
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
    s.inv_bc1 = s.inv_bc2 = 0.0;
    s.rcp_bc1_hi = s.rcp_bc1_lo = s.rcp_bc2_hi = s.rcp_bc2_lo = 0.0f;
    return s;
}

// An address range [lo, hi) of one buffer, and whether the step writes it.
struct Range {
    uintptr_t lo, hi;
    bool written;
};

// Checks one record of a collection stepped with `algo` and writes the
// ranges of its four buffers to out[0..3] (*n = 4), or *n = 0 for an empty
// record.  Pointers need element alignment; AdEMAMix's state1 spans 2*numel
// floats.
inline int record_ranges(const opt2s_tensor& t, int32_t algo, Range* out, int* n)
{
    *n = 0;
    if (t.numel < 0 || t.reserved != 0) return OPT2S_ERR_INVALID_ARG;
    if (t.dtype != OPT2S_F32 && t.dtype != OPT2S_F16 && t.dtype != OPT2S_BF16)
        return OPT2S_ERR_INVALID_ARG;
    if (t.numel == 0) return OPT2S_OK;
    if (t.numel > (int64_t(1) << 40)) return OPT2S_ERR_INVALID_ARG;
    if (!t.param || !t.grad || !t.state1 || !t.state2) return OPT2S_ERR_INVALID_ARG;
    const int es = elem_bytes(t.dtype);
    const auto p = reinterpret_cast<uintptr_t>(t.param);
    const auto g = reinterpret_cast<uintptr_t>(t.grad);
    const auto s1 = reinterpret_cast<uintptr_t>(t.state1);
    const auto s2 = reinterpret_cast<uintptr_t>(t.state2);
    if (p % es || g % es || s1 % 4 || s2 % 4) return OPT2S_ERR_INVALID_ARG;
    const uintptr_t k = static_cast<uintptr_t>(t.numel);
    out[0] = {p, p + k * es, true};
    out[1] = {g, g + k * es, false};
    out[2] = {s1, s1 + (algo == OPT2S_ADEMAMIX ? 2 * k : k) * 4, true};
    out[3] = {s2, s2 + k * 4, true};
    *n = 4;
    return OPT2S_OK;
}

// Sorts r[0..n) in place by start and reports OPT2S_ERR_ALIAS if a written
// range overlaps any other range (two read-only ranges may overlap: several
// tensors may share one gradient buffer).  Each range is compared with the
// furthest-reaching earlier range of each kind.
inline int overlap_status(Range* r, size_t n)
{
    std::sort(r, r + n, [](const Range& a, const Range& b) { return a.lo < b.lo; });
    uintptr_t reach_w = 0, reach_any = 0;
    bool have_w = false, have_any = false;
    for (size_t i = 0; i < n; ++i) {
        if (have_w && r[i].lo < reach_w) return OPT2S_ERR_ALIAS;
        if (r[i].written && have_any && r[i].lo < reach_any) return OPT2S_ERR_ALIAS;
        if (r[i].written) { reach_w = have_w ? std::max(reach_w, r[i].hi) : r[i].hi; have_w = true; }
        reach_any = have_any ? std::max(reach_any, r[i].hi) : r[i].hi;
        have_any = true;
    }
    return OPT2S_OK;
}

// Keeps `e` as this thread's last CUDA error (opt2s_last_cuda_error) and
// returns OPT2S_ERR_CUDA.  Defined in opt2s_api.cpp.
int record_cuda_error(cudaError_t e);

// Adds n to the count of kernels this library has launched.  Defined in
// opt2s_api.cpp.
void count_launches(int64_t n);

}  // namespace opt2s
