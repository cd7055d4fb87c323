// opt2s_kernel8.cu -- the optimizer step with 8-bit blockwise state, in one
// persistent launch for a collection that mixes 8-bit-state tensors with
// small 32-bit-state ones.
//
// State format: Dettmers, Lewis, Shleifer & Zettlemoyer, "8-bit Optimizers
// via Block-wise Quantization", ICLR 2022.  A tensor's state is cut into
// blocks of 2,048 elements (section 2.1); each block stores one fp32 absmax
// per state quantity and one byte per element, the index of a value of a
// 256-entry quantization map: dynamic tree quantization for the signed first
// moments (section 2.2), dynamic quantization for the non-negative second
// moment (section 2.3).  The bitsandbytes issue "Investigate a 256-thread
// SM103 path for small 32-bit optimizer tensors", section "Problem", gives
// the routing: tensors below min_8bit_size = 4,096 elements keep fp32 state
// and the 32-bit kernel.  Here both kinds run in the same launch.
//
// The maps (ascending; code c is the c-th smallest value): for E = 0..6 and
// F = 6 - E (signed) or 7 - E (unsigned) fraction bits, the values
//     10^-E * (0.1 + 0.9*(2f + 1)/2^(F+1)),  f = 0 .. 2^F - 1
// (with both signs for the signed map), plus 0 and 1.0.  Each value is
// N/D with N = 2^(F+1) + 9*(2f+1) and D = 10^(E+1)*2^(F+1), exact binary32
// integers, so one IEEE division gives it rounded once.  Every CTA builds the
// two maps in shared memory at start, and the thresholds between neighbours:
// T_j = the binary32 number at or below the exact midpoint of map[j] and
// map[j+1] (binary64 holds the midpoint exactly).  For a binary32 x,
// x > T_j exactly when x lies above that midpoint, so the number of
// thresholds below x is the code of the nearest map value, an exact tie going
// to the lower code.  A binary search over the 255 thresholds finds it.
//
// Per 8-bit block (one CTA of 256 threads, 8 consecutive elements a thread):
//   1. dequantize: m = map_s[code]*absmax (fp32 product), v with map_u;
//   2. the plain step's element update (opt2s_device.cuh), param stored;
//   3. the block's new absmax of |m|, v (, |m2|): fmaxf over the thread's
//      elements, the warp and the CTA's 8 warps (max is exact, so the order
//      does not matter; NaNs are ignored);
//   4. quantize: code of m/absmax (IEEE fp32 division), or the code of 0
//      when the absmax is 0; thread 0 stores the new absmaxes.
// With skip_zeros an element whose gradient is zero keeps its param and its
// dequantized state, which is requantized with the block's new absmax.
// Warps of a CTA walk the 32-bit chunks of small tensors exactly as the plain
// step kernel does (the same device functions), eight chunks per work unit.

#include <mutex>

#include "opt2s_device.cuh"

namespace opt2s {
namespace {

constexpr int kB8Threads = 256;                  // one CTA per 8-bit block
constexpr int kB8PerThread = kBlock8Elems / kB8Threads;
static_assert(kB8PerThread == 8, "eight elements a thread");

struct Maps {
    float smap[256], umap[256];   // signed (m, m2) and unsigned (v) maps
    float sthr[256], uthr[256];   // thresholds between neighbours (255 used)
    float red[2][3][kB8Threads / 32];   // per-warp maxima, double-buffered
};

// Value of map entry k before sorting: the k-th (value, sign) of the
// construction above, in the order of E, f (and sign); k = 254 is 0 and
// k = 255 is 1.0.
__device__ float map_value(bool is_signed, int k)
{
    const int f0 = is_signed ? 6 : 7;
    int at = 0;
    for (int E = 0; E <= 6; ++E) {
        const int F = f0 - E;
        const int per = (1 << F) * (is_signed ? 2 : 1);
        if (k < at + per) {
            const int r = k - at;
            const int f = is_signed ? r >> 1 : r;
            float D = static_cast<float>(1 << (F + 1));
            for (int e = 0; e <= E; ++e) D = __fmul_rn(D, 10.0f);
            const float N = static_cast<float>((1 << (F + 1)) + 9 * (2 * f + 1));
            const float v = __fdiv_rn(N, D);
            return (is_signed && (r & 1)) ? -v : v;
        }
        at += per;
    }
    return k == at ? 0.0f : 1.0f;
}

// Builds both maps and their thresholds in shared memory (all threads of the
// CTA take part; ends with a barrier).  Sorting: the rank of a value is the
// number of values below it (all 256 are distinct).
__device__ void build_maps(Maps& mp)
{
    const int t = threadIdx.x;
    const float sv = map_value(true, t);
    const float uv = map_value(false, t);
    mp.sthr[t] = sv;             // unsorted values, for the ranking
    mp.uthr[t] = uv;
    __syncthreads();
    int rs = 0, ru = 0;
    for (int j = 0; j < 256; ++j) {
        rs += mp.sthr[j] < sv;
        ru += mp.uthr[j] < uv;
    }
    mp.smap[rs] = sv;
    mp.umap[ru] = uv;
    __syncthreads();
    if (t < 255) {
        mp.sthr[t] = __double2float_rd(__dmul_rn(__dadd_rn(static_cast<double>(mp.smap[t]),
                                                           static_cast<double>(mp.smap[t + 1])), 0.5));
        mp.uthr[t] = __double2float_rd(__dmul_rn(__dadd_rn(static_cast<double>(mp.umap[t]),
                                                           static_cast<double>(mp.umap[t + 1])), 0.5));
    }
    __syncthreads();
}

// Code of the nearest map value: the number of thresholds below x.
__device__ __forceinline__ uint32_t code_of(const float* thr, float x)
{
    uint32_t c = 0;
#pragma unroll
    for (uint32_t step = 128; step >= 1; step >>= 1)
        if (x > thr[c + step - 1]) c += step;
    return c;
}

__device__ __forceinline__ uint32_t quantize(const float* thr, float x, float amax, uint32_t zero)
{
    return amax > 0.0f ? code_of(thr, __fdiv_rn(x, amax)) : zero;
}

__device__ __forceinline__ float warp_max(float x)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, off));
    return x;
}

// Eight codes of a thread: one 8-byte access when `vec`, else byte by byte.
__device__ __forceinline__ void load_codes(const uint8_t* q, uint32_t i, uint32_t len, bool vec,
                                           uint32_t (&c)[kB8PerThread])
{
    if (vec) {
        const uint2 w = *reinterpret_cast<const uint2*>(q + i);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            c[k] = (w.x >> (8 * k)) & 0xFFu;
            c[4 + k] = (w.y >> (8 * k)) & 0xFFu;
        }
    } else {
#pragma unroll
        for (int k = 0; k < kB8PerThread; ++k) c[k] = i + k < len ? q[i + k] : 0u;
    }
}

__device__ __forceinline__ void store_codes(uint8_t* q, uint32_t i, uint32_t len, bool vec,
                                            const uint32_t (&c)[kB8PerThread])
{
    if (vec) {
        uint2 w;
        w.x = c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24);
        w.y = c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24);
        *reinterpret_cast<uint2*>(q + i) = w;
    } else {
#pragma unroll
        for (int k = 0; k < kB8PerThread; ++k)
            if (i + k < len) q[i + k] = static_cast<uint8_t>(c[k]);
    }
}

__device__ __forceinline__ bool al(const void* q, uint32_t bytes)
{
    return (reinterpret_cast<uintptr_t>(q) & (bytes - 1)) == 0;
}

// One 8-bit block by the whole CTA.  `buf` selects the half of the reduction
// scratch this block uses (alternating between a CTA's blocks, so that no
// second barrier is needed before the next block writes it).
template <int DT, int ALGO, bool SKIP>
__device__ void block8(const Block8Rec& b, const StepScalars& s, Maps& mp, int buf)
{
    using P = Param<DT>;
    constexpr int V = P::kVec;
    const uint32_t len = b.len;
    const uint32_t i0 = threadIdx.x * kB8PerThread;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // full, aligned blocks move 8 elements a thread in 16-byte (param, grad)
    // and 8-byte (codes) accesses; others go element by element
    const bool vec = len == static_cast<uint32_t>(kBlock8Elems) && al(b.p, 16) && al(b.g, 16) &&
                     al(b.q1, 8) && al(b.q2, 8) && (ALGO != kAdEMAMix || al(b.q3, 8));

    const float a1 = b.a1[0], a2 = b.a2[0];
    const float a3 = ALGO == kAdEMAMix ? b.a3[0] : 0.0f;
    uint32_t c1[kB8PerThread], c2[kB8PerThread], c3[kB8PerThread];
    load_codes(b.q1, i0, len, vec, c1);
    load_codes(b.q2, i0, len, vec, c2);
    if (ALGO == kAdEMAMix) load_codes(b.q3, i0, len, vec, c3);
    float g[kB8PerThread], p[kB8PerThread];
    typename P::Raw praw[8 / V], graw[8 / V];
    if (vec) {
#pragma unroll
        for (int u = 0; u < 8 / V; ++u) {
            graw[u] = P::load(b.g, i0 + u * V);
            praw[u] = P::load(b.p, i0 + u * V);
        }
#pragma unroll
        for (int u = 0; u < 8 / V; ++u) {
            float x[V], y[V];
            P::widen(graw[u], x);
            P::widen(praw[u], y);
#pragma unroll
            for (int j = 0; j < V; ++j) { g[u * V + j] = x[j]; p[u * V + j] = y[j]; }
        }
    } else {
#pragma unroll
        for (int k = 0; k < kB8PerThread; ++k) {
            const bool in = i0 + k < len;
            g[k] = in ? P::load1(b.g, i0 + k) : 0.0f;
            p[k] = in ? P::load1(b.p, i0 + k) : 0.0f;
        }
    }

    float m[kB8PerThread], v[kB8PerThread], m2[kB8PerThread];
    float x1 = 0.0f, x2 = 0.0f, x3 = 0.0f;
#pragma unroll
    for (int k = 0; k < kB8PerThread; ++k) {
        m[k] = __fmul_rn(mp.smap[c1[k]], a1);
        v[k] = __fmul_rn(mp.umap[c2[k]], a2);
        m2[k] = ALGO == kAdEMAMix ? __fmul_rn(mp.smap[c3[k]], a3) : 0.0f;
        if (i0 + k < len) {
            update<ALGO, SKIP>(g[k], p[k], m[k], v[k], m2[k], s);
            x1 = fmaxf(x1, fabsf(m[k]));
            x2 = fmaxf(x2, fabsf(v[k]));
            if (ALGO == kAdEMAMix) x3 = fmaxf(x3, fabsf(m2[k]));
        }
    }
    if (vec) {
#pragma unroll
        for (int u = 0; u < 8 / V; ++u) {
            float y[V], gg[V];
#pragma unroll
            for (int j = 0; j < V; ++j) { y[j] = p[u * V + j]; gg[j] = g[u * V + j]; }
            P::store(b.p, i0 + u * V, P::narrow(y, praw[u], gg, SKIP));
        }
    } else {
#pragma unroll
        for (int k = 0; k < kB8PerThread; ++k)
            if (i0 + k < len && !(SKIP && g[k] == 0.0f)) P::store1(b.p, i0 + k, p[k]);
    }

    // the block's new absmaxes
    x1 = warp_max(x1);
    x2 = warp_max(x2);
    if (ALGO == kAdEMAMix) x3 = warp_max(x3);
    if (lane == 0) {
        mp.red[buf][0][warp] = x1;
        mp.red[buf][1][warp] = x2;
        mp.red[buf][2][warp] = x3;
    }
    __syncthreads();
    float n1 = 0.0f, n2 = 0.0f, n3 = 0.0f;
#pragma unroll
    for (int w = 0; w < kB8Threads / 32; ++w) {
        n1 = fmaxf(n1, mp.red[buf][0][w]);
        n2 = fmaxf(n2, mp.red[buf][1][w]);
        n3 = fmaxf(n3, mp.red[buf][2][w]);
    }
    // every thread has read the old absmaxes (before the barrier)
    if (threadIdx.x == 0) {
        b.a1[0] = n1;
        b.a2[0] = n2;
        if (ALGO == kAdEMAMix) b.a3[0] = n3;
    }
#pragma unroll
    for (int k = 0; k < kB8PerThread; ++k) {
        c1[k] = quantize(mp.sthr, m[k], n1, 127u);
        c2[k] = quantize(mp.uthr, v[k], n2, 0u);
        if (ALGO == kAdEMAMix) c3[k] = quantize(mp.sthr, m2[k], n3, 127u);
    }
    store_codes(b.q1, i0, len, vec, c1);
    store_codes(b.q2, i0, len, vec, c2);
    if (ALGO == kAdEMAMix) store_codes(b.q3, i0, len, vec, c3);
}

// Work unit u < nblocks: 8-bit block u, by the whole CTA.  Otherwise unit u
// holds the 32-bit chunks 8(u - nblocks) .. 8(u - nblocks) + 7, one a warp.
template <int ALGO, bool SKIP>
__global__ void __launch_bounds__(kB8Threads)
step8_kernel(const Block8Rec* __restrict__ blocks, int nblocks, const ChunkRec* __restrict__ chunks,
             int nchunks, StepScalars s)
{
    __shared__ Maps mp;
    build_maps(mp);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int units = nblocks + (nchunks + kB8Threads / 32 - 1) / (kB8Threads / 32);
    int buf = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {   // the same u for the whole CTA
        if (u < nblocks) {
            const Block8Rec b = blocks[u];
            switch (b.dtype) {
            case kF32: block8<kF32, ALGO, SKIP>(b, s, mp, buf); break;
            case kF16: block8<kF16, ALGO, SKIP>(b, s, mp, buf); break;
            default: block8<kBF16, ALGO, SKIP>(b, s, mp, buf); break;
            }
            buf ^= 1;
        } else {
            const int c = (u - nblocks) * (kB8Threads / 32) + warp;
            if (c < nchunks) {
                const ChunkRec rec = chunks[c];
                switch (rec.dtype & ~kShortFlag) {
                case kF32: run_chunk<kF32, ALGO, SKIP>(rec, s, lane); break;
                case kF16: run_chunk<kF16, ALGO, SKIP>(rec, s, lane); break;
                default: run_chunk<kBF16, ALGO, SKIP>(rec, s, lane); break;
                }
            }
        }
    }
}

using Kernel8Fn = void (*)(const Block8Rec*, int, const ChunkRec*, int, StepScalars);

Kernel8Fn pick8(int algo, int skip)
{
    if (algo == kAdEMAMix) return skip ? step8_kernel<kAdEMAMix, true> : step8_kernel<kAdEMAMix, false>;
    return skip ? step8_kernel<kAdam, true> : step8_kernel<kAdam, false>;
}

constexpr int kMaxDevices8 = 64;
int g_occ8[kMaxDevices8][4];   // resident CTAs per SM, per device and kernel
int g_sms8[kMaxDevices8];
std::mutex g_occ8_mu;

}  // namespace

cudaError_t launch_step8(const Block8Rec* d_blocks, int64_t nblocks, const ChunkRec* d_chunks,
                         int64_t nchunks, int algo, int skip_zeros, const StepScalars& s,
                         int max_blocks, cudaStream_t stream)
{
    const int64_t units = nblocks + (nchunks + kB8Threads / 32 - 1) / (kB8Threads / 32);
    if (units <= 0) return cudaSuccess;
    Kernel8Fn fn = pick8(algo, skip_zeros);
    int cap = max_blocks;
    if (cap <= 0) {
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= kMaxDevices8) return cudaErrorInvalidDevice;
        std::lock_guard<std::mutex> lock(g_occ8_mu);
        const int k = (algo == kAdEMAMix ? 2 : 0) + (skip_zeros ? 1 : 0);
        if (g_occ8[dev][k] == 0) {
            int per_sm = 0, sms = 0;
            e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e == cudaSuccess)
                e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kB8Threads, 0);
            if (e != cudaSuccess) return e;
            g_sms8[dev] = sms;
            g_occ8[dev][k] = per_sm < 1 ? 1 : per_sm;
        }
        cap = g_occ8[dev][k] * g_sms8[dev];
    }
    const int grid = static_cast<int>(units < cap ? units : cap);
    StepScalars sc = s;
    fill_reciprocals(&sc);
    int nb = static_cast<int>(nblocks), nc = static_cast<int>(nchunks);
    void* args[] = {const_cast<Block8Rec**>(&d_blocks), &nb, const_cast<ChunkRec**>(&d_chunks), &nc, &sc};
    return cudaLaunchKernel(reinterpret_cast<const void*>(fn), dim3(grid), dim3(kB8Threads), args, 0,
                            stream);
}

}  // namespace opt2s
