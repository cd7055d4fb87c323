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
// integers, so one IEEE division gives it rounded once.  The host builds the
// two maps and the slice tables below once per plan (opt2s_api8.cpp,
// build_quant_tables) and uploads them with it; every CTA copies them into
// shared memory at start.
//
// Quantization: the code of x = RN32(m / absmax) is the map value nearest to
// x, an exact tie going to the lower code.  With T_j the binary32 number at
// or below the exact midpoint of map[j] and map[j+1] (binary64 holds the
// midpoint exactly), x > T_j exactly when x lies above that midpoint, so the
// code is the number of thresholds below x.  Rather than search the 255
// thresholds, each CTA tabulates them over the bits of x: the exponent picks
// a row (|x| below 2^-23, where the nearest value is 0 in both maps; one row
// per binade up to 2^0; NaN), the top 7 fraction bits a slice of the row.
// Every slice is narrower than the gap between two thresholds (the finest,
// 0.9/128 at the top of the unsigned map, is above the widest slice, 2^-8),
// so a slice holds at most one threshold; with t the low 16 bits of its
// magnitude (the rest of its bits are the slice's own), the code is
// base + (low16(x) > t) for x >= 0 and base + (low16(x) < t) for x < 0, base
// the code at the slice's low end in value order.  The slice's 4-byte entry
// holds base in its high half and, in its low half, 0xFFFF - t for x >= 0 or
// t for x < 0 (0 without a threshold), so that with key = low16(x), or its
// complement for x < 0, the code is (entry + key) >> 16: one addition whose
// carry does the comparison.  The signed map has a table per sign.
// x itself is first taken as RN32(m * RN32(1/absmax)), within 3 ulp of
// RN32(m/absmax); only when that lies within 4 ulp of the slice's threshold, or
// of an edge of a slice without one (about 9 cases in 65,536), is x
// recomputed exactly as RN32(RN64(m * RN64(1/absmax))): for every quotient in
// the binary32 normal range that is RN32(m/absmax) (the binary64 product errs
// by less than 2^-52, while a quotient that is not representable never lies
// within 2^-49 of a binary32 rounding boundary; see div_by_constant in
// opt2s_device.cuh), and below it both give the code of 0.
//
// Per 8-bit block (one CTA of 256 threads, 8 elements a thread; fp32 storage
// takes elements 4t..4t+3 and 1024+4t..1024+4t+3, 16-bit storage 8t..8t+7, so
// that every warp access is contiguous):
//   1. dequantize: m = map_s[code]*absmax (fp32 product), v with map_u;
//   2. the plain step's element update (opt2s_device.cuh; its fp32 route for
//      the bias-correction divisions), a few elements at a time with one
//      range test for their divisions (update_group), param stored;
//   3. the block's new absmax of |m|, v (, |m2|): fmaxf over the thread's
//      elements (NaNs are ignored), then an unsigned maximum of the bit
//      patterns over the warp (one warp reduction) and the CTA's 8 warps
//      (max is exact, so the order does not matter);
//   4. quantize each value with the block's new absmax, or store the code of
//      0 when it is 0 (a thread's eight values of a state take one test for
//      the rare exact quotients); thread 0 stores the new absmaxes.
// With skip_zeros an element whose gradient is zero keeps its param and its
// dequantized state, which is requantized with the block's new absmax.
// Warps of a CTA walk the 32-bit chunks of small tensors element-wise with the
// plain step's element update (opt2s_device.cuh), eight chunks per work unit.

#include <cstddef>
#include <mutex>

#include "opt2s_device.cuh"

namespace opt2s {
namespace {

constexpr int kB8Threads = 256;                  // one CTA per 8-bit block
// Resident CTAs per SM the registers must allow: the kernel waits on loads
// and on its barrier, so more resident CTAs measured faster (Adam: 4 CTAs at
// 64 registers beat 3 at 80, 2 at 128 and 5 at 48, which spills; with the
// grouped update, 4 CTAs with a few spilled bytes still beat 3 without: Adam
// 1.109 against 1.149 ms, AdEMAMix 1.403 against 1.439 at 268 M elements).
// Each CTA also prefetches its next block into L2.
template <int ALGO>
constexpr int kB8MinCtas = 4;
constexpr int kB8PerThread = kBlock8Elems / kB8Threads;
static_assert(kB8PerThread == 8, "eight elements a thread");
// Elements a thread updates together (update_group): measured at 268 M
// elements against the element-by-element loop (1.280 / 1.656 ms for fp32
// Adam / bf16 AdEMAMix): groups of 4 for Adam (1.109 ms; 8: 1.184; 2: 1.134),
// 8 for AdEMAMix (1.403 ms; 4: 1.432), and 2 with skip_zeros, whose selects
// cost registers (Adam 1.146 ms, 4: 1.175, 8: 1.200; AdEMAMix 1.588 ms, 8
// spills and takes 1.98, against 1.80 before).
template <int ALGO, bool SKIP>
constexpr int kGroup = SKIP ? 2 : (ALGO == kAdEMAMix ? 8 : 4);

constexpr int kRows = kQuantRows;         // |x| < 2^-23; 24 binades 2^-23 .. 2^0; NaN
constexpr int kSlices = kRows * 128;      // 128 slices a row
constexpr uint32_t kZeroSigned = 127;     // code of 0 in the signed map
constexpr uint32_t kZeroUnsigned = 0;     // and in the unsigned one

struct Maps {
    float smap[256], umap[256];          // signed (m, m2) and unsigned (v) maps
    uint32_t stab[2][kSlices];           // slices of the signed map, x >= 0 and x < 0
    uint32_t utab[kSlices];              // slices of the unsigned map
    alignas(16) uint32_t red[2][3][kB8Threads / 32];   // per-warp maxima (bits), double-buffered
};
constexpr size_t kMapsBytes = sizeof(Maps);

// The tables as the host lays them out (QuantTables, opt2s_internal.h) are
// the leading words of Maps; each CTA copies them in at start.
static_assert(offsetof(Maps, smap) == 0 && offsetof(Maps, umap) == 256 * 4 &&
                  offsetof(Maps, stab) == 512 * 4 && offsetof(Maps, utab) == (512 + 2 * kSlices) * 4,
              "table layout");
static_assert(kQuantTableWords == 512 + 3 * kSlices, "table size");

__device__ void load_maps(Maps& mp, const uint4* __restrict__ tables)
{
    uint4* dst = reinterpret_cast<uint4*>(&mp);
    for (int i = threadIdx.x; i < kQuantTableWords / 4; i += kB8Threads) dst[i] = tables[i];
    __syncthreads();
}

// The slice entry of x's bits b: (code at the slice's low end) << 16 | c
// (opt2s_api8.cpp, slice_entry).  The exponent and the top 7 fraction bits,
// bits 16..30 of b, number the slices of all binades in order; clamping puts
// every |x| below 2^-23 in slice 0 of the first row and every NaN in the last
// slice of the NaN row.  The signed map's table follows the sign (the second
// table for x < 0).  The unsigned map is indexed with the sign bit left in:
// any x with it set (-0, -NaN; v is never negative otherwise) clamps to the
// NaN row, whose code 0 is also the nearest code of every x <= 0 there.
template <bool SIGNED>
__device__ __forceinline__ uint32_t slice_of(const Maps& mp, uint32_t b)
{
    constexpr int kLow = (127 - 24) * 128;    // slice number of 2^-23
    if (SIGNED) {
        const int i = __vimin_s32_relu(static_cast<int>((b >> 16) & 0x7FFFu) - kLow, kSlices - 1);
        const uint32_t other = static_cast<uint32_t>(static_cast<int32_t>(b) >> 31) & kSlices;
        return (&mp.stab[0][0])[i + other];       // the two tables are contiguous
    }
    return mp.utab[__vimin_s32_relu(static_cast<int>(b >> 16) - kLow, kSlices - 1)];
}

// The low 16 bits of x's magnitude as the slice entries expect them: as they
// are for x >= 0, complemented for x < 0 (signed map only).  The code is then
// (entry + key) >> 16: the carry out of the low half adds the threshold.
template <bool SIGNED>
__device__ __forceinline__ uint32_t low_key(uint32_t b)
{
    return SIGNED ? (b ^ static_cast<uint32_t>(static_cast<int32_t>(b) >> 31)) & 0xFFFFu : b & 0xFFFFu;
}

// Quantization of one value m with absmax > 0, in two parts.  fast_sum
// takes the fast quotient RN32(m*r32), r32 = RN32(1/absmax), within 3 ulp of
// RN32(m/absmax), and returns sum = entry + key for it, whose high half is
// then the code.  The code is certain unless the key lies within 4 of the
// slice's threshold; with sum as above, (sum + 5) mod 2^16 <= 8 exactly then
// (near_key).  That one test also covers a quotient near a slice boundary: in
// a slice without a threshold (low half 0) it holds within 4 of either edge,
// and no slice that holds a threshold has another one within 8 ulp beyond its
// edges (a property of the two maps, checked on the host by the tests), so a
// fast quotient that crosses an edge from such a slice crosses no threshold.
// exact_sum gives the sum for the exact quotient RN32(RN64(m * RN64(1/absmax)))
// (r64 = RN64(1/absmax)), for the values that near_key flags.
template <bool SIGNED>
__device__ __forceinline__ uint32_t sum_of_bits(const Maps& mp, uint32_t b)
{
    return slice_of<SIGNED>(mp, b) + low_key<SIGNED>(b);
}
template <bool SIGNED>
__device__ __forceinline__ uint32_t fast_sum(const Maps& mp, float m, float r32)
{
    return sum_of_bits<SIGNED>(mp, __float_as_uint(__fmul_rn(m, r32)));
}
template <bool SIGNED>
__device__ __forceinline__ uint32_t exact_sum(const Maps& mp, float m, double r64)
{
    return sum_of_bits<SIGNED>(mp, __float_as_uint(__double2float_rn(__dmul_rn(static_cast<double>(m), r64))));
}
__device__ __forceinline__ uint32_t near_key(uint32_t sum)
{
    return (sum + 5u) & 0xFFFFu;    // <= 8: the fast quotient does not decide
}

// The maximum over the warp of a value that is >= +0 and not NaN: such
// binary32 values order like their bit patterns as unsigned integers, so one
// warp reduction on the bits gives it (the result as bits).
__device__ __forceinline__ uint32_t warp_max_bits(float x)
{
    return __reduce_max_sync(0xffffffffu, __float_as_uint(x));
}

// The maximum of the eight per-warp maxima (bits, as above) of one quantity.
__device__ __forceinline__ float block_max(const uint32_t (&r)[kB8Threads / 32])
{
    const uint4 a = *reinterpret_cast<const uint4*>(&r[0]);
    const uint4 b = *reinterpret_cast<const uint4*>(&r[4]);
    return __uint_as_float(max(__vimax3_u32(a.x, a.y, a.z), __vimax3_u32(a.w, b.x, __vimax3_u32(b.y, b.z, b.w))));
}

// Element j of run u of this thread (runs of V elements, one storage vector
// each): fp32 (V = 4) takes 4t..4t+3 and 1024+4t..1024+4t+3, 16-bit (V = 8)
// 8t..8t+7, so that each warp access is contiguous.
template <int V>
__device__ __forceinline__ uint32_t elem(int u, int j)
{
    return static_cast<uint32_t>(u * (kBlock8Elems * V / 8) + threadIdx.x * V + j);
}

// A thread's eight codes, packed four to a 32-bit word (word w holds the codes
// of elements 4w .. 4w+3 of the thread, lowest byte first): one V-byte
// access per run when `vec`, else byte by byte (0 past the end of the block).
template <int V>
__device__ __forceinline__ void load_codes(const uint8_t* q, uint32_t len, bool vec, uint32_t (&w)[2])
{
#pragma unroll
    for (int u = 0; u < 8 / V; ++u) {
        const uint32_t e = elem<V>(u, 0);
        if (vec) {
            if (V == 8) {
                const uint2 x = *reinterpret_cast<const uint2*>(q + e);
                w[0] = x.x;
                w[1] = x.y;
            } else {
                w[u] = *reinterpret_cast<const uint32_t*>(q + e);
            }
        } else {
#pragma unroll
            for (int h = 0; h < V / 4; ++h) {
                uint32_t x = 0;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    if (e + 4 * h + k < len) x |= static_cast<uint32_t>(q[e + 4 * h + k]) << (8 * k);
                w[u * (V / 4) + h] = x;
            }
        }
    }
}

// Byte k & 3 of word k >> 2, zero-extended (one byte permute).
__device__ __forceinline__ uint32_t code_at(const uint32_t (&w)[2], int k)
{
    return __byte_perm(w[k >> 2], 0u, 0x4440u | static_cast<uint32_t>(k & 3));
}

// Four codes (each < 256) packed into one word, c0 in the lowest byte.
__device__ __forceinline__ uint32_t pack4(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3)
{
    return __byte_perm(__byte_perm(c0, c1, 0x0040u), __byte_perm(c2, c3, 0x0040u), 0x5410u);
}

// The codes of a thread's eight values x[] of one state, packed as the code
// arrays store them (zero_code for all when the block's absmax is 0).
// All eight fast quotients and table lookups come first, with one test for
// the lot; the rare exact quotients (about 9 values in 65,536) follow in a
// branch of their own, so that no per-value branch separates the lookups.
template <bool SIGNED>
__device__ __forceinline__ void quantize8(const Maps& mp, const float (&x)[kB8PerThread], float absmax,
                                          uint32_t zero_code, uint32_t (&w)[2])
{
    if (absmax > 0.0f) {
        const float r32 = __frcp_rn(absmax);     // for the fast quotient
        uint32_t sum[kB8PerThread];
        uint32_t near = 0xFFFFu;
#pragma unroll
        for (int k = 0; k < kB8PerThread; ++k) {
            sum[k] = fast_sum<SIGNED>(mp, x[k], r32);
            near = min(near, near_key(sum[k]));
        }
        if (__builtin_expect(near <= 8u, 0)) {
            const double r64 = __drcp_rn(static_cast<double>(absmax));
#pragma unroll
            for (int k = 0; k < kB8PerThread; ++k)
                if (near_key(sum[k]) <= 8u) sum[k] = exact_sum<SIGNED>(mp, x[k], r64);
        }
        w[0] = pack4(sum[0] >> 16, sum[1] >> 16, sum[2] >> 16, sum[3] >> 16);
        w[1] = pack4(sum[4] >> 16, sum[5] >> 16, sum[6] >> 16, sum[7] >> 16);
    } else {
        w[0] = w[1] = zero_code * 0x01010101u;
    }
}

template <int V>
__device__ __forceinline__ void store_codes(uint8_t* q, uint32_t len, bool vec, const uint32_t (&w)[2])
{
#pragma unroll
    for (int u = 0; u < 8 / V; ++u) {
        const uint32_t e = elem<V>(u, 0);
        if (vec) {
            if (V == 8)
                *reinterpret_cast<uint2*>(q + e) = make_uint2(w[0], w[1]);
            else
                *reinterpret_cast<uint32_t*>(q + e) = w[u];
        } else {
#pragma unroll
            for (int k = 0; k < V; ++k)
                if (e + k < len) q[e + k] = static_cast<uint8_t>(code_at(w, u * V + k));
        }
    }
}

// Asks L2 for the lines of the next block this CTA will step (param, grad and
// codes), so that its loads after this block's barrier find them there.
template <int ALGO>
__device__ __forceinline__ void prefetch_block(const Block8Rec& b, int es)
{
    const uint32_t t = threadIdx.x;
    const uint32_t pg_lines = (b.len * es + 127) / 128, q_lines = (b.len + 127) / 128;
    auto pf = [](const void* a) { asm volatile("prefetch.global.L2 [%0];" :: "l"(a)); };
    for (uint32_t l = t; l < pg_lines; l += kB8Threads) {
        pf(static_cast<const char*>(b.p) + 128 * l);
        pf(static_cast<const char*>(b.g) + 128 * l);
    }
    if (t < q_lines) {
        pf(b.q1 + 128 * t);
        pf(b.q2 + 128 * t);
        if (ALGO == kAdEMAMix) pf(b.q3 + 128 * t);
    }
}

__device__ __forceinline__ bool al(const void* q, uint32_t bytes)
{
    return (reinterpret_cast<uintptr_t>(q) & (bytes - 1)) == 0;
}

// All eight elements, G at a time.
template <int ALGO, bool SKIP, int G, int O = 0>
__device__ __forceinline__ void update_all(const float (&g)[kB8PerThread], float (&p)[kB8PerThread],
                                           float (&m)[kB8PerThread], float (&v)[kB8PerThread],
                                           float (&m2)[kB8PerThread], const StepScalars& s)
{
    static_assert(kB8PerThread % G == 0, "groups tile the thread's elements");
    update_group<ALGO, SKIP, kPlain, O, G>(g, p, m, v, m2, s);
    if constexpr (O + G < kB8PerThread) update_all<ALGO, SKIP, G, O + G>(g, p, m, v, m2, s);
}

// One 8-bit block by the whole CTA.  `buf` selects the half of the reduction
// scratch this block uses (alternating between a CTA's blocks, so that no
// second barrier is needed before the next block writes it).
// FULL: a whole block of kBlock8Elems elements whose arrays are aligned for
// the vector accesses (the common case, with no per-element bounds checks);
// otherwise elements are accessed one by one and those past `len` skipped.
template <int DT, int ALGO, bool SKIP, bool FULL>
__device__ __forceinline__ void block8(const Block8Rec& b, const StepScalars& s, Maps& mp, int buf)
{
    using P = Param<DT>;
    constexpr int V = P::kVec;
    constexpr int R = 8 / V;   // runs a thread
    const uint32_t len = FULL ? static_cast<uint32_t>(kBlock8Elems) : b.len;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr bool vec = FULL;

    const float a1 = b.a1[0], a2 = b.a2[0];
    const float a3 = ALGO == kAdEMAMix ? b.a3[0] : 0.0f;
    uint32_t c1[2], c2[2], c3[2];
    load_codes<V>(b.q1, len, vec, c1);
    load_codes<V>(b.q2, len, vec, c2);
    if (ALGO == kAdEMAMix) load_codes<V>(b.q3, len, vec, c3);
    float g[kB8PerThread], p[kB8PerThread];
    typename P::Raw praw[R], graw[R];
    if (vec) {
#pragma unroll
        for (int u = 0; u < R; ++u) {
            graw[u] = P::load(b.g, elem<V>(u, 0));
            praw[u] = P::load(b.p, elem<V>(u, 0));
        }
#pragma unroll
        for (int u = 0; u < R; ++u) {
            float x[V], y[V];
            P::widen(graw[u], x);
            P::widen(praw[u], y);
#pragma unroll
            for (int j = 0; j < V; ++j) { g[u * V + j] = x[j]; p[u * V + j] = y[j]; }
        }
    } else {
#pragma unroll
        for (int u = 0; u < R; ++u)
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const uint32_t e = elem<V>(u, j);
                g[u * V + j] = e < len ? P::load1(b.g, e) : 0.0f;
                p[u * V + j] = e < len ? P::load1(b.p, e) : 0.0f;
            }
    }

    float m[kB8PerThread], v[kB8PerThread], m2[kB8PerThread];
#pragma unroll
    for (int k = 0; k < kB8PerThread; ++k) {
        m[k] = __fmul_rn(mp.smap[code_at(c1, k)], a1);
        v[k] = __fmul_rn(mp.umap[code_at(c2, k)], a2);
        m2[k] = ALGO == kAdEMAMix ? __fmul_rn(mp.smap[code_at(c3, k)], a3) : 0.0f;
    }
    // (elements past the end of a partial block are stepped too, from zero
    // inputs, and then left out of the absmaxes and the stores)
    update_all<ALGO, SKIP, kGroup<ALGO, SKIP>>(g, p, m, v, m2, s);
    float x1 = 0.0f, x2 = 0.0f, x3 = 0.0f;
#pragma unroll
    for (int k = 0; k < kB8PerThread; ++k)
        if (FULL || elem<V>(k / V, k % V) < len) {
            x1 = fmaxf(x1, fabsf(m[k]));
            x2 = fmaxf(x2, fabsf(v[k]));
            if (ALGO == kAdEMAMix) x3 = fmaxf(x3, fabsf(m2[k]));
        }
    if (vec) {
#pragma unroll
        for (int u = 0; u < R; ++u) {
            float y[V], gg[V];
#pragma unroll
            for (int j = 0; j < V; ++j) { y[j] = p[u * V + j]; gg[j] = g[u * V + j]; }
            P::store(b.p, elem<V>(u, 0), P::narrow(y, praw[u], gg, SKIP));
        }
    } else {
#pragma unroll
        for (int u = 0; u < R; ++u)
#pragma unroll
            for (int j = 0; j < V; ++j) {
                const uint32_t e = elem<V>(u, j);
                if (e < len && !(SKIP && g[u * V + j] == 0.0f)) P::store1(b.p, e, p[u * V + j]);
            }
    }

    // the block's new absmaxes
    // (x1, x2, x3 are >= +0 and never NaN: fmaxf from +0 skips NaN)
    const uint32_t w1 = warp_max_bits(x1), w2 = warp_max_bits(x2);
    const uint32_t w3 = ALGO == kAdEMAMix ? warp_max_bits(x3) : 0u;
    if (lane == 0) {
        mp.red[buf][0][warp] = w1;
        mp.red[buf][1][warp] = w2;
        mp.red[buf][2][warp] = w3;
    }
    __syncthreads();
    const float n1 = block_max(mp.red[buf][0]), n2 = block_max(mp.red[buf][1]);
    const float n3 = ALGO == kAdEMAMix ? block_max(mp.red[buf][2]) : 0.0f;
    // every thread has read the old absmaxes (before the barrier)
    if (threadIdx.x == 0) {
        b.a1[0] = n1;
        b.a2[0] = n2;
        if (ALGO == kAdEMAMix) b.a3[0] = n3;
    }
    quantize8<true>(mp, m, n1, kZeroSigned, c1);
    quantize8<false>(mp, v, n2, kZeroUnsigned, c2);
    if (ALGO == kAdEMAMix) quantize8<true>(mp, m2, n3, kZeroSigned, c3);
    store_codes<V>(b.q1, len, vec, c1);
    store_codes<V>(b.q2, len, vec, c2);
    if (ALGO == kAdEMAMix) store_codes<V>(b.q3, len, vec, c3);
}

// A ragged or unaligned block, out of line so that it does not add to the
// full-block path's registers.
template <int DT, int ALGO, bool SKIP>
__device__ __noinline__ void block8_part(const Block8Rec b, const StepScalars s, Maps& mp, int buf)
{
    block8<DT, ALGO, SKIP, false>(b, s, mp, buf);
}

template <int DT, int ALGO, bool SKIP>
__device__ __forceinline__ void block8_any(const Block8Rec& b, const StepScalars& s, Maps& mp, int buf)
{
    constexpr int V = Param<DT>::kVec;
    const bool full = b.len == static_cast<uint32_t>(kBlock8Elems) && al(b.p, 16) && al(b.g, 16) &&
                      al(b.q1, V) && al(b.q2, V) && (ALGO != kAdEMAMix || al(b.q3, V));
    if (full) block8<DT, ALGO, SKIP, true>(b, s, mp, buf);
    else block8_part<DT, ALGO, SKIP>(b, s, mp, buf);
}

// A 32-bit chunk (at most 256 elements of a small tensor) by one warp: lane l
// takes elements l, l + 32, ..., a few at a time, all their loads first
// (so they are in flight together rather than one dependent round trip an
// element), then the plain step's element update and the stores.  A skipped
// element is not written back.  Element-wise accesses keep every array's
// alignment free; the few registers leave the 8-bit block path the kernel's
// register budget.
// Adam batches 4 elements a lane (the issue's mixed AdamW collection: 28.7 to
// 24.7 us); AdEMAMix, whose third state array makes wider batches cost the
// 8-bit block path registers, 1 (2 measured 1.3 % slower on the 268 M step).
template <int ALGO>
constexpr int kSmallBatch = ALGO == kAdEMAMix ? 1 : 4;

template <int DT, int ALGO, bool SKIP>
__device__ __forceinline__ void small_chunk(const ChunkRec& c, const StepScalars& s, int lane)
{
    using P = Param<DT>;
    constexpr int K = kSmallBatch<ALGO>;
    for (uint32_t base = 0; base < c.len; base += 32 * K) {
        float g[K], p[K], m[K], v[K], m2[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const uint32_t i = base + lane + 32 * k;
            g[k] = p[k] = m[k] = v[k] = m2[k] = 0.0f;
            if (i < c.len) {
                g[k] = P::load1(c.g, i);
                p[k] = P::load1(c.p, i);
                m[k] = ld_global(c.m + i);
                v[k] = ld_global(c.v + i);
                if (ALGO == kAdEMAMix) m2[k] = ld_global(c.m2 + i);
            }
        }
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const uint32_t i = base + lane + 32 * k;
            if (i < c.len && !(SKIP && g[k] == 0.0f)) {
                update<ALGO, false>(g[k], p[k], m[k], v[k], m2[k], s);
                P::store1(c.p, i, p[k]);
                st_global(c.m + i, m[k]);
                st_global(c.v + i, v[k]);
                if (ALGO == kAdEMAMix) st_global(c.m2 + i, m2[k]);
            }
        }
    }
}

// Work unit u < nblocks: 8-bit block u, by the whole CTA.  Otherwise unit u
// holds the 32-bit chunks 8(u - nblocks) .. 8(u - nblocks) + 7, one a warp.
// The maps and slice tables live in dynamic shared memory (kMapsBytes).
template <int ALGO, bool SKIP>
__global__ void __launch_bounds__(kB8Threads, kB8MinCtas<ALGO>)
step8_kernel(const Block8Rec* __restrict__ blocks, int nblocks, const ChunkRec* __restrict__ chunks,
             int nchunks, const uint4* __restrict__ tables, StepScalars s)
{
    extern __shared__ __align__(16) unsigned char smem8[];
    Maps& mp = *reinterpret_cast<Maps*>(smem8);
    load_maps(mp, tables);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int units = nblocks + (nchunks + kB8Threads / 32 - 1) / (kB8Threads / 32);
    int buf = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {   // the same u for the whole CTA
        if (u < nblocks) {
            const Block8Rec b = blocks[u];
            if (u + static_cast<int>(gridDim.x) < nblocks) {
                const Block8Rec nb = blocks[u + gridDim.x];
                prefetch_block<ALGO>(nb, nb.dtype == kF32 ? 4 : 2);
            }
            switch (b.dtype) {
            case kF32: block8_any<kF32, ALGO, SKIP>(b, s, mp, buf); break;
            case kF16: block8_any<kF16, ALGO, SKIP>(b, s, mp, buf); break;
            default: block8_any<kBF16, ALGO, SKIP>(b, s, mp, buf); break;
            }
            buf ^= 1;
        } else {
            const int c = (u - nblocks) * (kB8Threads / 32) + warp;
            if (c < nchunks) {
                const ChunkRec rec = chunks[c];
                switch (rec.dtype & ~kShortFlag) {
                case kF32: small_chunk<kF32, ALGO, SKIP>(rec, s, lane); break;
                case kF16: small_chunk<kF16, ALGO, SKIP>(rec, s, lane); break;
                default: small_chunk<kBF16, ALGO, SKIP>(rec, s, lane); break;
                }
            }
        }
    }
}

using Kernel8Fn = void (*)(const Block8Rec*, int, const ChunkRec*, int, const uint4*, StepScalars);

Kernel8Fn pick8(int algo, int skip)
{
    if (algo == kAdEMAMix) return skip ? step8_kernel<kAdEMAMix, true> : step8_kernel<kAdEMAMix, false>;
    return skip ? step8_kernel<kAdam, true> : step8_kernel<kAdam, false>;
}

constexpr int kMaxDevices8 = 64;
int g_occ8[kMaxDevices8][4];   // resident CTAs per SM, per device and kernel (0: not set up)
int g_sms8[kMaxDevices8];
std::mutex g_occ8_mu;

}  // namespace

cudaError_t launch_step8(const Block8Rec* d_blocks, int64_t nblocks, const ChunkRec* d_chunks,
                         int64_t nchunks, const uint32_t* d_tables, int algo, int skip_zeros,
                         const StepScalars& s, int max_blocks, cudaStream_t stream)
{
    const int64_t units = nblocks + (nchunks + kB8Threads / 32 - 1) / (kB8Threads / 32);
    if (units <= 0) return cudaSuccess;
    Kernel8Fn fn = pick8(algo, skip_zeros);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices8) return cudaErrorInvalidDevice;
    int cap = 0;
    {
        std::lock_guard<std::mutex> lock(g_occ8_mu);
        const int k = (algo == kAdEMAMix ? 2 : 0) + (skip_zeros ? 1 : 0);
        if (g_occ8[dev][k] == 0) {
            // the tables take more than the default 48 KB of shared memory
            int per_sm = 0, sms = 0;
            e = cudaFuncSetAttribute(reinterpret_cast<const void*>(fn),
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(kMapsBytes));
            if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
            if (e == cudaSuccess)
                e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kB8Threads, kMapsBytes);
            if (e != cudaSuccess) return e;
            g_sms8[dev] = sms;
            g_occ8[dev][k] = per_sm < 1 ? 1 : per_sm;
        }
        cap = g_occ8[dev][k] * g_sms8[dev];
    }
    if (max_blocks > 0) cap = max_blocks;
    const int grid = static_cast<int>(units < cap ? units : cap);
    StepScalars sc = s;
    fill_reciprocals(&sc);
    int nb = static_cast<int>(nblocks), nc = static_cast<int>(nchunks);
    const uint4* tab = reinterpret_cast<const uint4*>(d_tables);
    void* args[] = {const_cast<Block8Rec**>(&d_blocks), &nb, const_cast<ChunkRec**>(&d_chunks), &nc,
                    const_cast<uint4**>(&tab), &sc};
    return cudaLaunchKernel(reinterpret_cast<const void*>(fn), dim3(grid), dim3(kB8Threads), args,
                            kMapsBytes, stream);
}

}  // namespace opt2s
