// opt2s_kernel.cu -- the persistent multi-tensor optimizer-step kernel for
// B200 (sm_100a).
//
// One launch steps a whole tensor collection.  The host splits every tensor
// into chunks of at most a few thousand elements (opt2s_api.cpp); each warp
// takes chunks c = warp, warp + total_warps, ... and streams through them with
// 128-bit loads and stores, so 2,000 tiny bias/norm tensors cost one launch
// and a multi-GB tensor is spread over every SM.  The path has no cross-
// element reduction and no data reuse, so there is no shared-memory staging
// and no tensor-core work: it is bound by HBM bandwidth (28 bytes per element
// for fp32 Adam, 36 for fp32 AdEMAMix).
//
// The element arithmetic and the chunk walkers live in opt2s_device.cuh.
// Every element's result is the plain IEEE evaluation of the documented fp32
// order whatever code path, chunk, warp or block computed it: the issue's
// "Correctness oracle" section requires that launch geometry must not change
// optimizer arithmetic.

#include <mutex>

#include "opt2s_device.cuh"

namespace opt2s {
namespace {

// ---------------------------------------------------------------------------
// The sharded step (reduce-scatter + update + all-gather in one kernel).
//
// Element e of this rank's shard gets g = (g_0[e] + g_1[e] + ... + g_{W-1}[e])
// / W, widened exactly, summed in rank order and divided with IEEE fp32
// operations, then the same update as the plain step; the new param is stored
// into the param buffer of every rank.  Ranks touch disjoint shards, grads are
// only read and state is local, so ranks never wait on one another inside the
// kernel; the caller orders the step between two cross-rank barriers (grads
// final before, params read after).  Peer buffers are reached with ordinary
// loads and stores (NVLink on a multi-GPU node; no TMA, no multicast).
// ---------------------------------------------------------------------------
template <int DT, int ALGO, bool SKIP, int W>
__device__ __forceinline__ void shard_scalar(const ShardArgs& a, int64_t k, const StepScalars& s)
{
    using P = Param<DT>;
    const int64_t e = a.shard_start + k;
    constexpr int B = P::kBytes;
    float g = P::load1(static_cast<const char*>(a.grads[0]) + e * B, 0);
#pragma unroll
    for (int q = 1; q < W; ++q)
        g = __fadd_rn(g, P::load1(static_cast<const char*>(a.grads[q]) + e * B, 0));
    g = __fdiv_rn(g, static_cast<float>(W));
    if (SKIP && g == 0.0f) return;
    float p = P::load1(static_cast<const char*>(a.params[a.rank]) + e * B, 0);
    float m = ld_global(a.m + k);
    float v = ld_global(a.v + k);
    float m2 = 0.0f;
    if (ALGO == kAdEMAMix) m2 = ld_global(a.m2 + k);
    update<ALGO, false>(g, p, m, v, m2, s);
#pragma unroll
    for (int q = 0; q < W; ++q) P::store1(static_cast<char*>(a.params[q]) + e * B, 0, p);
    st_global(a.m + k, m);
    st_global(a.v + k, v);
    if (ALGO == kAdEMAMix) st_global(a.m2 + k, m2);
}

// Elements [k0, k0 + len) of the shard (shard-relative), one warp; W ranks.
// Like the plain step's vector body, each lane moves 8 elements per iteration.
template <int DT, int ALGO, bool SKIP, int W>
__device__ __forceinline__ void shard_chunk(const ShardArgs& a, int64_t k0, uint32_t len,
                                            const StepScalars& s, int lane)
{
    using P = Param<DT>;
    constexpr int V = P::kVec;
    constexpr int U = 8 / V;
    constexpr int B = P::kBytes;
    const int64_t e0 = a.shard_start + k0;
    const char* own = static_cast<const char*>(a.params[a.rank]) + e0 * B;
    uint32_t head = static_cast<uint32_t>(((16u - (reinterpret_cast<uintptr_t>(own) & 15u)) & 15u) / B);
    bool vec_ok = aligned16(a.m + k0, head, 4) && aligned16(a.v + k0, head, 4) &&
                  (ALGO != kAdEMAMix || aligned16(a.m2 + k0, head, 4));
#pragma unroll
    for (int q = 0; q < W; ++q)
        vec_ok = vec_ok && aligned16(static_cast<const char*>(a.params[q]) + e0 * B, head, B) &&
                 aligned16(static_cast<const char*>(a.grads[q]) + e0 * B, head, B);
    if (!vec_ok || head > len) head = len;
    const uint32_t nvec = (len - head) / V;
    const uint32_t body_end = head + nvec * V;
    for (uint32_t i = lane; i < head; i += 32) shard_scalar<DT, ALGO, SKIP, W>(a, k0 + i, s);
    for (uint32_t i = body_end + lane; i < len; i += 32) shard_scalar<DT, ALGO, SKIP, W>(a, k0 + i, s);

    for (uint32_t v0 = 0; v0 < nvec; v0 += 32 * U) {
        typename P::Raw graw[U][W], praw[U];
        float m[U][V], v[U][V], m2[U][V];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t vi = v0 + u * 32 + lane;
            if (vi < nvec) {
                const uint32_t i = head + vi * V;      // chunk-relative element
                const int64_t k = k0 + i;              // shard-relative element
                const int64_t e = e0 + i;              // flat element
#pragma unroll
                for (int q = 0; q < W; ++q)
                    graw[u][q] = P::load(static_cast<const char*>(a.grads[q]) + e * B, 0);
                praw[u] = P::load(static_cast<const char*>(a.params[a.rank]) + e * B, 0);
                load_state<V>(a.m + k, 0, m[u]);
                load_state<V>(a.v + k, 0, v[u]);
                if (ALGO == kAdEMAMix) load_state<V>(a.m2 + k, 0, m2[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t vi = v0 + u * 32 + lane;
            if (vi < nvec) {
                const uint32_t i = head + vi * V;
                const int64_t k = k0 + i;
                const int64_t e = e0 + i;
                float g[V], p[V];
                P::widen(graw[u][0], g);
                P::widen(praw[u], p);
#pragma unroll
                for (int q = 1; q < W; ++q) {
                    float x[V];
                    P::widen(graw[u][q], x);
#pragma unroll
                    for (int j = 0; j < V; ++j) g[j] = __fadd_rn(g[j], x[j]);
                }
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    g[j] = __fdiv_rn(g[j], static_cast<float>(W));
                    update<ALGO, SKIP>(g[j], p[j], m[u][j], v[u][j], m2[u][j], s);
                }
                const typename P::Raw out = P::narrow(p, praw[u], g, SKIP);
#pragma unroll
                for (int q = 0; q < W; ++q)
                    P::store(static_cast<char*>(a.params[q]) + e * B, 0, out);
                store_state<V>(a.m + k, 0, m[u]);
                store_state<V>(a.v + k, 0, v[u]);
                if (ALGO == kAdEMAMix) store_state<V>(a.m2 + k, 0, m2[u]);
            }
        }
    }
}

template <int ALGO, bool SKIP, int W>
__global__ void shard_step_kernel(ShardArgs a, StepScalars s)
{
    const int lane = threadIdx.x & 31;
    const int warps_per_block = blockDim.x >> 5;
    const int64_t warp = static_cast<int64_t>(blockIdx.x) * warps_per_block + (threadIdx.x >> 5);
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * warps_per_block;
    const int64_t ce = a.chunk_elems;
    const int64_t nchunks = (a.shard_len + ce - 1) / ce;
    for (int64_t c = warp; c < nchunks; c += nwarps) {
        const int64_t k0 = c * ce;
        const uint32_t len = static_cast<uint32_t>(min(ce, a.shard_len - k0));
        switch (a.dtype) {
        case kF32: shard_chunk<kF32, ALGO, SKIP, W>(a, k0, len, s, lane); break;
        case kF16: shard_chunk<kF16, ALGO, SKIP, W>(a, k0, len, s, lane); break;
        default: shard_chunk<kBF16, ALGO, SKIP, W>(a, k0, len, s, lane); break;
        }
    }
}

using ShardFn = void (*)(ShardArgs, StepScalars);

template <int ALGO, bool SKIP>
ShardFn pick_shard_w(int world)
{
    switch (world) {
    case 1: return shard_step_kernel<ALGO, SKIP, 1>;
    case 2: return shard_step_kernel<ALGO, SKIP, 2>;
    case 3: return shard_step_kernel<ALGO, SKIP, 3>;
    case 4: return shard_step_kernel<ALGO, SKIP, 4>;
    case 5: return shard_step_kernel<ALGO, SKIP, 5>;
    case 6: return shard_step_kernel<ALGO, SKIP, 6>;
    case 7: return shard_step_kernel<ALGO, SKIP, 7>;
    default: return shard_step_kernel<ALGO, SKIP, 8>;
    }
}

ShardFn pick_shard(int algo, int skip, int world)
{
    if (algo == kAdEMAMix)
        return skip ? pick_shard_w<kAdEMAMix, true>(world) : pick_shard_w<kAdEMAMix, false>(world);
    return skip ? pick_shard_w<kAdam, true>(world) : pick_shard_w<kAdam, false>(world);
}

// The whole step: warp w takes chunks w, w + W, w + 2W, ... of the table.
// ONLY < 0: every chunk dispatches on its own dtype; ONLY >= 0: every chunk
// of the plan has that dtype (the host guarantees it), so the kernel carries
// only that body and fewer registers.  SHORT: chunks marked with kShortFlag
// take the short-chunk path; otherwise they take the vector path, with the
// same result (the table-driven kernel does so, which keeps its register
// count at the plain kernel's).
template <int ALGO, bool SKIP, int ONLY, bool SHORT>
__device__ __forceinline__ void step_body(const ChunkRec* __restrict__ chunks, int nchunks,
                                          const StepScalars& s)
{
    const int lane = threadIdx.x & 31;
    const int warps_per_block = blockDim.x >> 5;
    const int warp = blockIdx.x * warps_per_block + (threadIdx.x >> 5);
    const int nwarps = gridDim.x * warps_per_block;
    for (int c = warp; c < nchunks; c += nwarps) {
        const ChunkRec rec = chunks[c];
        const bool short16 = SHORT && (rec.dtype & kShortFlag) != 0;
        if (ONLY >= 0) {
            // one 16-bit dtype: two 16-byte param vectors a lane per iteration
            // (16 elements), the bytes in flight of the fp32 path
            constexpr int D = ONLY >= 0 ? ONLY : kF16;
            if (short16) short_chunk<D, ALGO, SKIP>(rec, s, lane);
            else run_chunk<D, ALGO, SKIP, kPlain, 2>(rec, s, lane);
        } else {
            switch (rec.dtype & ~kShortFlag) {
            case kF32: run_chunk<kF32, ALGO, SKIP>(rec, s, lane); break;
            case kF16:
                if (short16) short_chunk<kF16, ALGO, SKIP>(rec, s, lane);
                else run_chunk<kF16, ALGO, SKIP>(rec, s, lane);
                break;
            default:
                if (short16) short_chunk<kBF16, ALGO, SKIP>(rec, s, lane);
                else run_chunk<kBF16, ALGO, SKIP>(rec, s, lane);
                break;
            }
        }
    }
}

// Per-step scalars passed by value (the host computes them for each call).
template <int ALGO, bool SKIP, int ONLY>
__global__ void step_kernel(const ChunkRec* __restrict__ chunks, int nchunks, StepScalars s)
{
    step_body<ALGO, SKIP, ONLY, true>(chunks, nchunks, s);
}

// Per-step scalars read from a device table at a device-resident index, so a
// captured CUDA graph performs the next step at every replay.  An index
// outside [0, table_len) performs no update.
template <int ALGO, bool SKIP, int ONLY>
__global__ void step_kernel_table(const ChunkRec* __restrict__ chunks, int nchunks,
                                  const StepScalars* __restrict__ table, const int* index,
                                  int table_len)
{
    const int idx = *index;
    if (idx < 0 || idx >= table_len) return;
    const StepScalars s = table[idx];
    step_body<ALGO, SKIP, ONLY, false>(chunks, nchunks, s);
}

// Moves the index to the next table entry; -1 once the table is used up.
__global__ void advance_index_kernel(int* index, int table_len)
{
    const int idx = *index;
    *index = (idx >= 0 && idx + 1 < table_len) ? idx + 1 : -1;
}

// ---------------------------------------------------------------------------
// The steps with per-tensor norms, four launches each:
//   * bounded update norm (max_unorm > 0): the norm of the update direction
//     u is bounded by max_unorm times the weight norm;
//   * LAMB (You et al. 2020, Algorithm 2): the decayed direction w = u + wd*p
//     is scaled by the trust ratio ||p|| / ||w||.
// The launches:
//   1. unorm_partials_kernel: for every block of kNormBlockElems elements of
//      a tensor (the host's norm table, fixed blocks whatever the plan's
//      chunk length), the sums of d^2 (d = u, or w for LAMB; 0 for an element
//      skip_zeros leaves alone) and of p^2 (p the param before the step).
//      Nothing is written but the two sums;
//   2. unorm_group_kernel: the sums of each group of kNormGroupBlocks
//      consecutive blocks of a tensor (one warp per group);
//   3. unorm_scale_kernel: per tensor, the sums of its groups, D = sqrt(sd),
//      P = sqrt(sp), and the scale (binary64, rounded to fp32 once):
//      max_unorm*P/D if D > max_unorm*P, else 1; or for LAMB P/D if P > 0
//      and D > 0, else 1;
//   4. step_kernel_scaled: the step over the plan's chunks with
//      p = p*decay - lr*(scale*u), or p = p - lr*(scale*w) for LAMB, the
//      scale read through the chunk's tensor.
// The element arithmetic is the plain step's (moments, the exact divisions by
// bc1 and bc2, direction_of); the norm pass and the scaled step take the
// divisions of a lane's elements with one range test (the fp32 route, or the
// binary64 route for all when a value is out of its range; both exact), which
// measured 3 % faster on the bounded-norm and LAMB steps than a test, or the
// binary64 route, element by element.  Every sum
// has a fixed order: lane l of the warp that owns a block adds the elements
// of its runs (V consecutive elements at V*l + 32*V*r, V = 4 for fp32 and 8
// for 16-bit storage) in index order, the 32 lanes then combine in a fixed
// shuffle tree, a group's blocks and a tensor's groups are combined in fixed
// orders too; so the scale does not depend on the plan's chunk length, the
// block width or the storage alignment.  Aligned blocks move each run with
// one 16-byte access per array.
//
// Each lane adds its squares in binary64: the square of a binary32 x is exact
// in binary64, so one fused multiply-add gives the same sum as a multiply and
// an add.  (A double-float lane sum -- two binary32 numbers, TwoProduct and
// TwoSum on the fp32 pipe -- avoids the float-to-double conversions but
// measured slower on B200: more instructions per element.)  The partials
// kernel is limited to 64 registers per thread for Adam, 4 CTAs of 256
// threads per SM: the extra resident warps hide more of the load latency,
// and measured faster than 3 CTAs at 80 registers.  AdEMAMix, with a third
// state array, spills at 64 and measured 0.6 % faster at 3 CTAs.
// ---------------------------------------------------------------------------
struct SquareSum {
    double s = 0.0;
    __device__ __forceinline__ void add(float x)
    {
        const double xd = static_cast<double>(x);
        s = __fma_rn(xd, xd, s);
    }
    __device__ __forceinline__ double total() const { return s; }
};

// One norm block by one warp.  Lane l owns the V-element runs starting at
// V*l + 32*V*r (r = 0, 1, ...; V = the storage vector's elements: 4 for fp32,
// 8 for 16-bit storage) and adds their elements in index order, run after
// run.  When the block's arrays are 16-byte aligned a run is one vector
// access per array; otherwise its elements are read one by one, in the same
// lane assignment, so the sums do not depend on the alignment.
template <int DT, int ALGO, bool SKIP, int MODE>
__device__ __forceinline__ void norm_block(const ChunkRec& c, const StepScalars& s, int lane,
                                           float wd, double& sd, double& sp)
{
    using P = Param<DT>;
    constexpr int V = P::kVec;
    constexpr int R = 8 / V;              // runs a lane loads per iteration: 8 elements
    constexpr int K = R * V;
    const uint32_t len = c.len;
    const bool vec = aligned16(c.p, 0, P::kBytes) && aligned16(c.g, 0, P::kBytes) &&
                     aligned16(c.m, 0, 4) && aligned16(c.v, 0, 4) &&
                     (ALGO != kAdEMAMix || aligned16(c.m2, 0, 4));
    SquareSum ad, ap;
    for (uint32_t base = 0; base < len; base += 32 * K) {
        float g[K], p[K], m[K], v[K], m2[K];
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const uint32_t e0 = base + (r * 32 + lane) * V;
            if (vec && e0 + V <= len) {
                float x[V], y[V], a[V], b[V], d[V];
                P::widen(P::load(c.g, e0), x);
                P::widen(P::load(c.p, e0), y);
                load_state<V>(c.m, e0, a);
                load_state<V>(c.v, e0, b);
                if (ALGO == kAdEMAMix) load_state<V>(c.m2, e0, d);
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    g[r * V + j] = x[j];
                    p[r * V + j] = y[j];
                    m[r * V + j] = a[j];
                    v[r * V + j] = b[j];
                    m2[r * V + j] = ALGO == kAdEMAMix ? d[j] : 0.0f;
                }
            } else {
#pragma unroll
                for (int j = 0; j < V; ++j) {
                    const uint32_t i = e0 + j;
                    const int k = r * V + j;
                    g[k] = p[k] = m[k] = v[k] = m2[k] = 0.0f;
                    if (i < len) {
                        g[k] = P::load1(c.g, i);
                        p[k] = P::load1(c.p, i);
                        m[k] = ld_global(c.m + i);
                        v[k] = ld_global(c.v + i);
                        if (ALGO == kAdEMAMix) m2[k] = ld_global(c.m2 + i);
                    }
                }
            }
        }
        // the moments of all K elements, then their bias-correction
        // divisions with one range test (the fp32 route when every value is
        // in its range, else the binary64 route for all: both are exact)
        // and the directions
        uint32_t key = 0;
#pragma unroll
        for (int k = 0; k < K; ++k) {
            moments<ALGO>(g[k], m[k], v[k], m2[k], s);
            key = max(key, max(fma_range_key(m[k]), fma_range_key(v[k])));
        }
        if (__builtin_expect(key >= kFmaRangeEnd, 0)) {
#pragma unroll
            for (int k = 0; k < K; ++k) {
                m[k] = div_by_constant(m[k], s.inv_bc1);
                v[k] = div_by_constant(v[k], s.inv_bc2);
            }
        } else {
#pragma unroll
            for (int k = 0; k < K; ++k) {
                m[k] = div_by_constant_in_range(m[k], s.bc1, s.rcp_bc1_hi, s.rcp_bc1_lo);
                v[k] = div_by_constant_in_range(v[k], s.bc2, s.rcp_bc2_hi, s.rcp_bc2_lo);
            }
        }
#pragma unroll
        for (int k = 0; k < K; ++k) {
            if (base + ((k / V) * 32 + lane) * V + (k % V) < len) {
                ap.add(p[k]);
                if (!(SKIP && g[k] == 0.0f)) {
                    const float u = direction_of<ALGO>(m[k], v[k], m2[k], s);
                    ad.add(MODE == kLamb ? lamb_direction(u, p[k], wd) : u);
                }
            }
        }
    }
    sd = ad.total();
    sp = ap.total();
}

__device__ __forceinline__ void warp_tree_sum(double& a, double& b)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        a = __dadd_rn(a, __shfl_down_sync(0xffffffffu, a, off));
        b = __dadd_rn(b, __shfl_down_sync(0xffffffffu, b, off));
    }
}

constexpr int kNormThreads = 256;

template <int ALGO, bool SKIP, int MODE>
__global__ void __launch_bounds__(kNormThreads, ALGO == kAdEMAMix ? 3 : 4) unorm_partials_kernel(const ChunkRec* __restrict__ blocks, int nblocks,
                                      StepScalars s, float wd, double2* __restrict__ partial)
{
    const int lane = threadIdx.x & 31;
    const int warps_per_block = blockDim.x >> 5;
    const int warp = blockIdx.x * warps_per_block + (threadIdx.x >> 5);
    const int nwarps = gridDim.x * warps_per_block;
    for (int b = warp; b < nblocks; b += nwarps) {
        const ChunkRec rec = blocks[b];
        double sd = 0.0, sp = 0.0;
        switch (rec.dtype & ~kShortFlag) {
        case kF32: norm_block<kF32, ALGO, SKIP, MODE>(rec, s, lane, wd, sd, sp); break;
        case kF16: norm_block<kF16, ALGO, SKIP, MODE>(rec, s, lane, wd, sd, sp); break;
        default: norm_block<kBF16, ALGO, SKIP, MODE>(rec, s, lane, wd, sd, sp); break;
        }
        warp_tree_sum(sd, sp);
        if (lane == 0) partial[b] = make_double2(sd, sp);
    }
}

// One warp per group: group q holds blocks [range[q].x, range[q].y) of one
// tensor (at most kNormGroupBlocks); lane l adds blocks x + l, x + l + 32 in
// turn, then a fixed tree over lanes.
__global__ void unorm_group_kernel(const double2* __restrict__ partial,
                                   const uint2* __restrict__ range, int ngroups,
                                   double2* __restrict__ group_sum)
{
    static_assert(kNormGroupBlocks <= 64, "two blocks per lane");
    const int lane = threadIdx.x & 31;
    const int warps_per_block = blockDim.x >> 5;
    const int nwarps = gridDim.x * warps_per_block;
    for (int q = blockIdx.x * warps_per_block + (threadIdx.x >> 5); q < ngroups; q += nwarps) {
        const uint2 r = range[q];
        double sd = 0.0, sp = 0.0;
        for (uint32_t b = r.x + lane; b < r.y; b += 32) {
            const double2 x = partial[b];
            sd = __dadd_rn(sd, x.x);
            sp = __dadd_rn(sp, x.y);
        }
        warp_tree_sum(sd, sp);
        if (lane == 0) group_sum[q] = make_double2(sd, sp);
    }
}

// One CTA of kScaleThreads threads per tensor (tensor t owns groups
// [first[t], first[t + 1])): thread j keeps four running sums, sum k taking
// groups j + (4i + k)*kScaleThreads for i = 0, 1, ... in turn, then
// (s0 + s1) + (s2 + s3), then a fixed tree over lanes and over the CTA's
// warps.  The order depends only on the tensor, not on the grid.
constexpr int kScaleThreads = 1024;

template <int MODE>
__global__ void __launch_bounds__(kScaleThreads)
unorm_scale_kernel(const double2* __restrict__ sums, const uint32_t* __restrict__ first,
                   int ntensors, float max_unorm, float* __restrict__ scale)
{
    constexpr int kWarps = kScaleThreads / 32;
    __shared__ double sd_w[kWarps], sp_w[kWarps];
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    for (int t = blockIdx.x; t < ntensors; t += gridDim.x) {   // the same t for the whole CTA
        double ad[4] = {0.0, 0.0, 0.0, 0.0}, ap[4] = {0.0, 0.0, 0.0, 0.0};
        const uint32_t end = first[t + 1];
        for (uint32_t b = first[t] + threadIdx.x; b < end; b += 4 * kScaleThreads) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t i = b + k * kScaleThreads;
                if (i < end) {
                    const double2 x = sums[i];
                    ad[k] = __dadd_rn(ad[k], x.x);
                    ap[k] = __dadd_rn(ap[k], x.y);
                }
            }
        }
        double sd = __dadd_rn(__dadd_rn(ad[0], ad[1]), __dadd_rn(ad[2], ad[3]));
        double sp = __dadd_rn(__dadd_rn(ap[0], ap[1]), __dadd_rn(ap[2], ap[3]));
        warp_tree_sum(sd, sp);
        if (lane == 0) { sd_w[w] = sd; sp_w[w] = sp; }
        __syncthreads();
        if (w == 0) {
            sd = lane < kWarps ? sd_w[lane] : 0.0;
            sp = lane < kWarps ? sp_w[lane] : 0.0;
            warp_tree_sum(sd, sp);
            if (lane == 0) {
                const double D = __dsqrt_rn(sd), P = __dsqrt_rn(sp);
                if (MODE == kLamb) {
                    scale[t] = (P > 0.0 && D > 0.0) ? __double2float_rn(__ddiv_rn(P, D)) : 1.0f;
                } else {
                    const double limit = __dmul_rn(static_cast<double>(max_unorm), P);
                    scale[t] = D > limit ? __double2float_rn(__ddiv_rn(limit, D)) : 1.0f;
                }
            }
        }
        __syncthreads();   // the shared sums are reused by the next tensor
    }
}

// The scaled step's division route: a group at a time, except with
// skip_zeros, whose per-element selects would take the kernel from 128 to 156
// registers (AdEMAMix).
template <bool SKIP>
constexpr int kScaledRoute = SKIP ? kDivWide : kDivGroup;

template <int ALGO, bool SKIP, int MODE>
__global__ void step_kernel_scaled(const ChunkRec* __restrict__ chunks, int nchunks,
                                   StepScalars s, const uint32_t* __restrict__ chunk_tensor,
                                   const float* __restrict__ scale, float wd)
{
    const int lane = threadIdx.x & 31;
    const int warps_per_block = blockDim.x >> 5;
    const int warp = blockIdx.x * warps_per_block + (threadIdx.x >> 5);
    const int nwarps = gridDim.x * warps_per_block;
    for (int c = warp; c < nchunks; c += nwarps) {
        const ChunkRec rec = chunks[c];
        const float sc = scale[chunk_tensor[c]];
        switch (rec.dtype & ~kShortFlag) {
        case kF32: run_chunk<kF32, ALGO, SKIP, MODE, 1, kScaledRoute<SKIP>>(rec, s, lane, sc, wd); break;
        case kF16: run_chunk<kF16, ALGO, SKIP, MODE, 1, kScaledRoute<SKIP>>(rec, s, lane, sc, wd); break;
        default: run_chunk<kBF16, ALGO, SKIP, MODE, 1, kScaledRoute<SKIP>>(rec, s, lane, sc, wd); break;
        }
    }
}

using KernelFn = void (*)(const ChunkRec*, int, StepScalars);
using TableKernelFn = void (*)(const ChunkRec*, int, const StepScalars*, const int*, int);

template <int ALGO, bool SKIP>
KernelFn pick_only(int only)
{
    if (only == kF16) return step_kernel<ALGO, SKIP, kF16>;
    if (only == kBF16) return step_kernel<ALGO, SKIP, kBF16>;
    return step_kernel<ALGO, SKIP, -1>;
}

// Specialised bodies exist for Adam over one 16-bit dtype (measured faster
// there); every other combination uses the per-chunk dispatch.
KernelFn pick(int algo, int skip, int only)
{
    if (algo == kAdEMAMix) return skip ? step_kernel<kAdEMAMix, true, -1> : step_kernel<kAdEMAMix, false, -1>;
    return skip ? pick_only<kAdam, true>(only) : pick_only<kAdam, false>(only);
}

template <int ALGO, bool SKIP>
TableKernelFn pick_table_only(int only)
{
    if (only == kF16) return step_kernel_table<ALGO, SKIP, kF16>;
    if (only == kBF16) return step_kernel_table<ALGO, SKIP, kBF16>;
    return step_kernel_table<ALGO, SKIP, -1>;
}

TableKernelFn pick_table(int algo, int skip, int only)
{
    if (algo == kAdEMAMix)
        return skip ? step_kernel_table<kAdEMAMix, true, -1> : step_kernel_table<kAdEMAMix, false, -1>;
    return skip ? pick_table_only<kAdam, true>(only) : pick_table_only<kAdam, false>(only);
}

constexpr int kOnlyClasses = 3;   // generic, f16, bf16
int only_class(int algo, int only)
{
    if (algo == kAdEMAMix) return 0;
    return only == kF16 ? 1 : (only == kBF16 ? 2 : 0);
}

// Resident blocks per SM and SM count, cached per device (and kernel / block
// size): device attributes are per device, not per process.
constexpr int kMaxDevices = 64;
struct OccEntry { int block_threads; int blocks_per_sm; };
struct DeviceInfo { int sms; OccEntry occ[4 * kOnlyClasses][6]; };
DeviceInfo g_info[kMaxDevices];
bool g_info_ok[kMaxDevices];
std::mutex g_info_mu;   // guards g_info / g_info_ok (host threads may launch concurrently)

cudaError_t device_info(int dev, DeviceInfo** out)
{
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (!g_info_ok[dev]) {
        int sms = 0;
        cudaError_t e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        g_info[dev].sms = sms;
        for (auto& row : g_info[dev].occ)
            for (auto& x : row) x = OccEntry{0, 0};
        g_info_ok[dev] = true;
    }
    *out = &g_info[dev];
    return cudaSuccess;
}

}  // namespace

cudaError_t grid_for(int64_t nchunks, int algo, int skip_zeros, int only, int block_threads,
                     int max_blocks, int* grid)
{
    const int warps_per_block = block_threads / 32;
    const int64_t need = (nchunks + warps_per_block - 1) / warps_per_block;
    int cap = max_blocks;
    if (cap <= 0) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        std::lock_guard<std::mutex> lock(g_info_mu);
        DeviceInfo* info = nullptr;
        if ((e = device_info(dev, &info)) != cudaSuccess) return e;
        const int k = ((algo == kAdEMAMix ? 2 : 0) + (skip_zeros ? 1 : 0)) * kOnlyClasses + only_class(algo, only);
        int per_sm = 0;
        for (auto& x : info->occ[k])
            if (x.block_threads == block_threads) per_sm = x.blocks_per_sm;
        if (per_sm == 0) {
            e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                &per_sm, pick(algo, skip_zeros, only), block_threads, 0);
            if (e != cudaSuccess) return e;
            if (per_sm < 1) per_sm = 1;
            for (auto& x : info->occ[k])
                if (x.block_threads == 0) { x = OccEntry{block_threads, per_sm}; break; }
        }
        cap = per_sm * info->sms;
    }
    *grid = static_cast<int>(need < cap ? need : cap);
    return cudaSuccess;
}

cudaError_t resident_warps(int algo, int skip_zeros, int only, int block_threads, int64_t* out)
{
    int grid = 0;
    // the occupancy cap is what grid_for returns for an unbounded chunk count
    cudaError_t e = grid_for(INT64_MAX / 2, algo, skip_zeros, only, block_threads, 0, &grid);
    if (e != cudaSuccess) return e;
    *out = static_cast<int64_t>(grid) * (block_threads / 32);
    return cudaSuccess;
}

cudaError_t max_block_threads(int algo, int skip_zeros, int only, int* out)
{
    cudaFuncAttributes attr;
    cudaError_t e = cudaFuncGetAttributes(&attr, pick(algo, skip_zeros, only));
    if (e != cudaSuccess) return e;
    *out = attr.maxThreadsPerBlock / 32 * 32;
    return cudaSuccess;
}

cudaError_t launch_step(const ChunkRec* d_chunks, int64_t nchunks, int algo, int skip_zeros,
                        int only, const StepScalars& s, int block_threads, int max_blocks,
                        cudaStream_t stream)
{
    if (nchunks <= 0) return cudaSuccess;
    int grid = 0;
    cudaError_t e = grid_for(nchunks, algo, skip_zeros, only, block_threads, max_blocks, &grid);
    if (e != cudaSuccess) return e;
    int n = static_cast<int>(nchunks);
    StepScalars sc = s;
    fill_reciprocals(&sc);   // correctly rounded binary64 reciprocals (IEEE)
    void* args[] = {const_cast<ChunkRec**>(&d_chunks), &n, &sc};
    return cudaLaunchKernel(reinterpret_cast<const void*>(pick(algo, skip_zeros, only)),
                            dim3(grid), dim3(block_threads), args, 0, stream);
}

cudaError_t launch_shard_step(const ShardArgs& a, int algo, int skip_zeros, const StepScalars& s,
                              int block_threads, cudaStream_t stream)
{
    if (a.shard_len <= 0) return cudaSuccess;
    ShardFn fn = pick_shard(algo, skip_zeros, a.world);
    int dev = 0, sms = 0, per_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, block_threads, 0);
    if (e != cudaSuccess) return e;
    const int64_t nchunks = (a.shard_len + a.chunk_elems - 1) / a.chunk_elems;
    const int64_t need = (nchunks + block_threads / 32 - 1) / (block_threads / 32);
    const int64_t cap = static_cast<int64_t>(per_sm < 1 ? 1 : per_sm) * sms;
    const int grid = static_cast<int>(need < cap ? need : cap);
    ShardArgs aa = a;
    StepScalars sc = s;
    fill_reciprocals(&sc);
    void* args[] = {&aa, &sc};
    return cudaLaunchKernel(reinterpret_cast<const void*>(fn), dim3(grid), dim3(block_threads), args, 0,
                            stream);
}

void fill_reciprocals(StepScalars* s)
{
    s->inv_bc1 = 1.0 / static_cast<double>(s->bc1);
    s->inv_bc2 = 1.0 / static_cast<double>(s->bc2);
    // inv - hi is exact in binary64 (the two agree to 24 bits)
    s->rcp_bc1_hi = static_cast<float>(s->inv_bc1);
    s->rcp_bc1_lo = static_cast<float>(s->inv_bc1 - static_cast<double>(s->rcp_bc1_hi));
    s->rcp_bc2_hi = static_cast<float>(s->inv_bc2);
    s->rcp_bc2_lo = static_cast<float>(s->inv_bc2 - static_cast<double>(s->rcp_bc2_hi));
}

cudaError_t launch_step_table(const ChunkRec* d_chunks, int64_t nchunks, int algo, int skip_zeros,
                              int only, const StepScalars* d_table, int* d_index, int table_len,
                              int block_threads, int max_blocks, cudaStream_t stream)
{
    if (nchunks > 0) {
        int grid = 0;
        cudaError_t e = grid_for(nchunks, algo, skip_zeros, only, block_threads, max_blocks, &grid);
        if (e != cudaSuccess) return e;
        int n = static_cast<int>(nchunks);
        const int* idx = d_index;
        int len = table_len;
        void* args[] = {const_cast<ChunkRec**>(&d_chunks), &n, const_cast<StepScalars**>(&d_table),
                        const_cast<int**>(&idx), &len};
        e = cudaLaunchKernel(reinterpret_cast<const void*>(pick_table(algo, skip_zeros, only)),
                             dim3(grid), dim3(block_threads), args, 0, stream);
        if (e != cudaSuccess) return e;
    }
    void* args2[] = {&d_index, &table_len};
    return cudaLaunchKernel(reinterpret_cast<const void*>(advance_index_kernel), dim3(1), dim3(1),
                            args2, 0, stream);
}

namespace {

// Resident blocks per SM of one of the max_unorm kernels at block_threads,
// cached per device.
struct UnormOcc { const void* fn; int block_threads; int per_sm; };
UnormOcc g_unorm_occ[kMaxDevices][24];

cudaError_t unorm_grid(const void* fn, int64_t warps_needed, int block_threads, int* grid)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_info_mu);
    DeviceInfo* info = nullptr;
    if ((e = device_info(dev, &info)) != cudaSuccess) return e;
    int per_sm = 0;
    for (auto& x : g_unorm_occ[dev])
        if (x.fn == fn && x.block_threads == block_threads) per_sm = x.per_sm;
    if (per_sm == 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, block_threads, 0);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) per_sm = 1;
        for (auto& x : g_unorm_occ[dev])
            if (x.fn == nullptr) { x = UnormOcc{fn, block_threads, per_sm}; break; }
    }
    const int64_t warps_per_block = block_threads / 32;
    const int64_t need = (warps_needed + warps_per_block - 1) / warps_per_block;
    const int64_t cap = static_cast<int64_t>(per_sm) * info->sms;
    *grid = static_cast<int>(need < cap ? need : cap);
    return cudaSuccess;
}

template <int ALGO, bool SKIP, int MODE>
cudaError_t launch_unorm_typed(const ChunkRec* d_chunks, int64_t nchunks, const StepScalars& sc,
                               const UnormArgs& u, float max_unorm, float wd, int block_threads,
                               int max_blocks, cudaStream_t stream)
{
    int grid = 0;
    cudaError_t e = cudaSuccess;
    if (u.nblocks > 0) {
        const void* k1 = reinterpret_cast<const void*>(unorm_partials_kernel<ALGO, SKIP, MODE>);
        if ((e = unorm_grid(k1, u.nblocks, kNormThreads, &grid)) != cudaSuccess) return e;
        unorm_partials_kernel<ALGO, SKIP, MODE><<<grid, kNormThreads, 0, stream>>>(
            u.blocks, static_cast<int>(u.nblocks), sc, wd, reinterpret_cast<double2*>(u.partial));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (u.ngroups > 0) {
        const void* kg = reinterpret_cast<const void*>(unorm_group_kernel);
        if ((e = unorm_grid(kg, u.ngroups, kNormThreads, &grid)) != cudaSuccess) return e;
        unorm_group_kernel<<<grid, kNormThreads, 0, stream>>>(
            reinterpret_cast<const double2*>(u.partial), reinterpret_cast<const uint2*>(u.group_range),
            static_cast<int>(u.ngroups), reinterpret_cast<double2*>(u.group_sum));
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (u.ntensors > 0) {
        const void* k2 = reinterpret_cast<const void*>(unorm_scale_kernel<MODE>);
        // one CTA per tensor, up to the resident CTAs of the device
        if ((e = unorm_grid(k2, static_cast<int64_t>(u.ntensors) * (kScaleThreads / 32), kScaleThreads,
                            &grid)) != cudaSuccess)
            return e;
        unorm_scale_kernel<MODE><<<grid, kScaleThreads, 0, stream>>>(
            reinterpret_cast<const double2*>(u.group_sum), u.first_group, u.ntensors, max_unorm,
            u.scale);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (nchunks > 0) {
        const void* k3 = reinterpret_cast<const void*>(step_kernel_scaled<ALGO, SKIP, MODE>);
        if (max_blocks > 0) {
            const int64_t need = (nchunks + block_threads / 32 - 1) / (block_threads / 32);
            grid = static_cast<int>(need < max_blocks ? need : max_blocks);
        } else if ((e = unorm_grid(k3, nchunks, block_threads, &grid)) != cudaSuccess) {
            return e;
        }
        step_kernel_scaled<ALGO, SKIP, MODE><<<grid, block_threads, 0, stream>>>(
            d_chunks, static_cast<int>(nchunks), sc, u.chunk_tensor, u.scale, wd);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_step_max_unorm(const ChunkRec* d_chunks, int64_t nchunks, int algo,
                                  int skip_zeros, const StepScalars& s, const UnormArgs& u,
                                  float max_unorm, int block_threads, int max_blocks,
                                  cudaStream_t stream)
{
    StepScalars sc = s;
    fill_reciprocals(&sc);
    if (algo == kAdEMAMix)
        return skip_zeros ? launch_unorm_typed<kAdEMAMix, true, kScaled>(
                                d_chunks, nchunks, sc, u, max_unorm, 0.0f, block_threads, max_blocks, stream)
                          : launch_unorm_typed<kAdEMAMix, false, kScaled>(
                                d_chunks, nchunks, sc, u, max_unorm, 0.0f, block_threads, max_blocks, stream);
    return skip_zeros ? launch_unorm_typed<kAdam, true, kScaled>(
                            d_chunks, nchunks, sc, u, max_unorm, 0.0f, block_threads, max_blocks, stream)
                      : launch_unorm_typed<kAdam, false, kScaled>(
                            d_chunks, nchunks, sc, u, max_unorm, 0.0f, block_threads, max_blocks, stream);
}

cudaError_t launch_step_lamb(const ChunkRec* d_chunks, int64_t nchunks, int skip_zeros,
                             const StepScalars& s, float weight_decay, const UnormArgs& u,
                             int block_threads, int max_blocks, cudaStream_t stream)
{
    StepScalars sc = s;
    fill_reciprocals(&sc);
    return skip_zeros ? launch_unorm_typed<kAdam, true, kLamb>(d_chunks, nchunks, sc, u, 0.0f, weight_decay,
                                                               block_threads, max_blocks, stream)
                      : launch_unorm_typed<kAdam, false, kLamb>(d_chunks, nchunks, sc, u, 0.0f, weight_decay,
                                                                block_threads, max_blocks, stream);
}

cudaError_t max_block_threads_scaled(int algo, int skip_zeros, int lamb, int* out)
{
    cudaFuncAttributes attr{};
    const void* fn =
        lamb ? (skip_zeros ? reinterpret_cast<const void*>(step_kernel_scaled<kAdam, true, kLamb>)
                           : reinterpret_cast<const void*>(step_kernel_scaled<kAdam, false, kLamb>))
        : algo == kAdEMAMix
            ? (skip_zeros ? reinterpret_cast<const void*>(step_kernel_scaled<kAdEMAMix, true, kScaled>)
                          : reinterpret_cast<const void*>(step_kernel_scaled<kAdEMAMix, false, kScaled>))
            : (skip_zeros ? reinterpret_cast<const void*>(step_kernel_scaled<kAdam, true, kScaled>)
                          : reinterpret_cast<const void*>(step_kernel_scaled<kAdam, false, kScaled>));
    cudaError_t e = cudaFuncGetAttributes(&attr, fn);
    if (e != cudaSuccess) return e;
    *out = attr.maxThreadsPerBlock / 32 * 32;
    return cudaSuccess;
}

}  // namespace opt2s
