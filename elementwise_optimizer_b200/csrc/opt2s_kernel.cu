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
// Arithmetic: the 32-bit two-state update of bitsandbytes issue "Investigate
// a 256-thread SM103 path for small 32-bit optimizer tensors" (sections
// "Problem", "Scope", "Correctness oracle"), with the standard Adam (Kingma &
// Ba 2015, Algorithm 1), decoupled weight decay (Loshchilov & Hutter 2019,
// Algorithm 2) and AdEMAMix (Pagliardini et al. 2024, Algorithm 1)
// definitions.  Every operation is an explicit round-to-nearest intrinsic
// (__fmul_rn / __fadd_rn / __fdiv_rn / __fsqrt_rn) or the exact constant
// division below, none of which the compiler may contract into FMA, so the
// result of an element equals the plain IEEE evaluation of the documented
// order and never depends on which code
// path (vector body, scalar head/tail), chunk, warp or block computed it: the
// issue's "Correctness oracle" section requires that launch geometry must not
// change optimizer arithmetic.

#include <mutex>

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "opt2s_internal.h"

namespace opt2s {
namespace {

// Global loads and stores with the default cache policy.  Every byte of a
// step is touched once, but measured on B200 the default (evict-normal)
// policy streams this read-modify-write pattern about 1% faster than the
// evict-first hints of ld/st.global.cs.
template <typename T>
__device__ __forceinline__ T ld_global(const T* p) { return *p; }
template <typename T>
__device__ __forceinline__ void st_global(T* p, const T& v) { *p = v; }

// ---------------------------------------------------------------------------
// Exact division by a per-launch constant.
//
// For every binary32 x and every binary32 d with 0 < |d| <= 1 (the bias
// corrections bc1, bc2 lie in (0, 1]), with r = RN64(1/d) the correctly
// rounded binary64 reciprocal computed once per launch on the host:
//            RN32( RN64(x * r) ) == RN32(x / d).
// Why: RN64(x*r) = (x/d)(1+e) with |e| <= 2^-52 + 2^-106, so it suffices that
// x/d is never within 2^-49 (relative) of a binary32 rounding boundary
// unless it is a binary32 number itself (then |e| < half an ulp keeps it).
// A boundary is M = Mi*2^k with Mi odd; x - d*M is a multiple of the smaller
// of the units of x's last bit and of d*M's last bit, and d*M spans fewer
// than 2^49 of the latter, so if x != d*M then |x/d - M| >= 2^-49 |M|.
// x == d*M cannot happen: for normal-range boundaries Mi has 25 significant
// bits while x has 24, and a subnormal-range boundary (an odd multiple of
// 2^-150) times |d| <= 1 is never a multiple of 2^-149 as every binary32 x
// is.  binary64 neither overflows nor underflows here, and 0, +-Inf and NaN
// pass through the product unchanged.  (The exclusion argument used in the
// analysis of double rounding; see Muller et al., Handbook of Floating-Point
// Arithmetic, 2nd ed., ch. 4.)  A GPU test checks it against __fdiv_rn on
// random operands of every class.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float div_by_constant(float x, double r)
{
    return __double2float_rn(__dmul_rn(static_cast<double>(x), r));
}

// ---------------------------------------------------------------------------
// The per-element update.  direction() moves the moments of one element (in
// place) and returns its update direction u = num/den; m/bc1 and v/bc2 use
// the exact constant division above, num/den is an IEEE division.  update()
// then applies the step to p.  With SKIP, an element whose gradient compares
// equal to zero (+0 or -0) is left untouched (no decay either).  MODE:
//   kPlain   p = p*decay - lr*u
//   kScaled  p = p*decay - lr*(scale*u)   (bounded update norm; scale = 1
//                                          gives the plain value)
//   kLamb    p = p - lr*(scale*w), w = u + wd*p   (LAMB: the weight decay
//                                          inside the trust-ratio scaled step)
// ---------------------------------------------------------------------------
enum : int { kPlain = 0, kScaled = 1, kLamb = 2 };

template <int ALGO>
__device__ __forceinline__ float direction(float g, float& m, float& v, float& m2,
                                           const StepScalars& s)
{
    m = __fadd_rn(__fmul_rn(s.beta1, m), __fmul_rn(s.one_minus_beta1, g));
    v = __fadd_rn(__fmul_rn(s.beta2, v),
                  __fmul_rn(__fmul_rn(s.one_minus_beta2, g), g));
    float num = div_by_constant(m, s.inv_bc1);
    if (ALGO == kAdEMAMix) {
        m2 = __fadd_rn(__fmul_rn(s.beta3, m2), __fmul_rn(s.one_minus_beta3, g));
        num = __fadd_rn(num, __fmul_rn(s.alpha, m2));
    }
    const float den = __fadd_rn(__fsqrt_rn(div_by_constant(v, s.inv_bc2)), s.eps);
    return __fdiv_rn(num, den);
}

// LAMB's decayed direction w = u + wd*p of an element.
__device__ __forceinline__ float lamb_direction(float u, float p, float wd)
{
    return __fadd_rn(u, __fmul_rn(wd, p));
}

template <int ALGO, bool SKIP, int MODE = kPlain>
__device__ __forceinline__ void update(float g, float& p, float& m, float& v,
                                       float& m2, const StepScalars& s, float scale = 1.0f,
                                       float wd = 0.0f)
{
    if (SKIP && g == 0.0f) return;
    const float u = direction<ALGO>(g, m, v, m2, s);
    if (MODE == kLamb)
        p = __fsub_rn(p, __fmul_rn(s.lr, __fmul_rn(scale, lamb_direction(u, p, wd))));
    else
        p = __fsub_rn(__fmul_rn(p, s.decay), __fmul_rn(s.lr, MODE == kScaled ? __fmul_rn(scale, u) : u));
}

// ---------------------------------------------------------------------------
// Storage traits of param / grad.  kVec elements make one 16-byte access.
// ---------------------------------------------------------------------------
template <int DT> struct Param;

template <> struct Param<kF32> {
    static constexpr int kVec = 4;
    static constexpr int kBytes = 4;
    using Raw = float4;
    __device__ static Raw load(const void* b, uint32_t i) {
        return ld_global(reinterpret_cast<const float4*>(static_cast<const float*>(b) + i));
    }
    __device__ static void store(void* b, uint32_t i, const Raw& r) {
        st_global(reinterpret_cast<float4*>(static_cast<float*>(b) + i), r);
    }
    __device__ static void widen(const Raw& r, float (&x)[4]) {
        x[0] = r.x; x[1] = r.y; x[2] = r.z; x[3] = r.w;
    }
    __device__ static Raw narrow(const float (&x)[4], const Raw&, const float (&)[4], bool) {
        // fp32: an untouched element already holds its loaded bits
        return make_float4(x[0], x[1], x[2], x[3]);
    }
    __device__ static float load1(const void* b, uint32_t i) {
        return ld_global(static_cast<const float*>(b) + i);
    }
    __device__ static void store1(void* b, uint32_t i, float x) {
        st_global(static_cast<float*>(b) + i, x);
    }
    // kVec elements from an address that need not be 16-byte aligned
    __device__ static Raw load_elems(const void* b, uint32_t i) {
        const float* f = static_cast<const float*>(b) + i;
        return make_float4(ld_global(f), ld_global(f + 1), ld_global(f + 2), ld_global(f + 3));
    }
};

// Shared by the two 16-bit formats: only the conversions differ.
template <typename H2, typename Cvt> struct Param16 {
    static constexpr int kVec = 8;
    static constexpr int kBytes = 2;
    using Raw = uint4;
    __device__ static Raw load(const void* b, uint32_t i) {
        return ld_global(reinterpret_cast<const uint4*>(static_cast<const unsigned short*>(b) + i));
    }
    __device__ static void store(void* b, uint32_t i, const Raw& r) {
        st_global(reinterpret_cast<uint4*>(static_cast<unsigned short*>(b) + i), r);
    }
    __device__ static void widen(const Raw& r, float (&x)[8]) {
        const H2* h = reinterpret_cast<const H2*>(&r);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float2 f = Cvt::to_float2(h[k]);
            x[2 * k] = f.x;
            x[2 * k + 1] = f.y;
        }
    }
    // Round to nearest even; with `skip`, elements whose gradient is zero keep
    // their original storage bits exactly (NaN payloads included).
    __device__ static Raw narrow(const float (&x)[8], const Raw& orig,
                                 const float (&g)[8], bool skip) {
        Raw r;
        H2* h = reinterpret_cast<H2*>(&r);
#pragma unroll
        for (int k = 0; k < 4; ++k) h[k] = Cvt::from_float2(x[2 * k], x[2 * k + 1]);
        if (skip) {
            uint32_t* w = reinterpret_cast<uint32_t*>(&r);
            const uint32_t* o = reinterpret_cast<const uint32_t*>(&orig);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint32_t mask = 0xFFFFu << (16 * (j & 1));
                if (g[j] == 0.0f) w[j >> 1] = (w[j >> 1] & ~mask) | (o[j >> 1] & mask);
            }
        }
        return r;
    }
    __device__ static float load1(const void* b, uint32_t i) {
        return Cvt::to_float(ld_global(static_cast<const unsigned short*>(b) + i));
    }
    // kVec elements from an address that need not be 16-byte aligned
    __device__ static Raw load_elems(const void* b, uint32_t i) {
        const unsigned short* h = static_cast<const unsigned short*>(b) + i;
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            w[k] = static_cast<uint32_t>(ld_global(h + 2 * k)) |
                   (static_cast<uint32_t>(ld_global(h + 2 * k + 1)) << 16);
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
    __device__ static void store1(void* b, uint32_t i, float x) {
        st_global(static_cast<unsigned short*>(b) + i, Cvt::from_float(x));
    }
};

struct CvtF16 {
    __device__ static float2 to_float2(__half2 h) { return __half22float2(h); }
    __device__ static __half2 from_float2(float a, float b) { return __floats2half2_rn(a, b); }
    __device__ static float to_float(unsigned short u) { return __half2float(__ushort_as_half(u)); }
    __device__ static unsigned short from_float(float x) { return __half_as_ushort(__float2half_rn(x)); }
};

struct CvtBF16 {
    __device__ static float2 to_float2(__nv_bfloat162 h) { return __bfloat1622float2(h); }
    __device__ static __nv_bfloat162 from_float2(float a, float b) { return __floats2bfloat162_rn(a, b); }
    __device__ static float to_float(unsigned short u) { return __bfloat162float(__ushort_as_bfloat16(u)); }
    __device__ static unsigned short from_float(float x) { return __bfloat16_as_ushort(__float2bfloat16_rn(x)); }
};

template <> struct Param<kF16> : Param16<__half2, CvtF16> {};
template <> struct Param<kBF16> : Param16<__nv_bfloat162, CvtBF16> {};

// fp32 state: N elements as N/4 16-byte accesses.
template <int N>
__device__ __forceinline__ void load_state(const float* b, uint32_t i, float (&x)[N]) {
#pragma unroll
    for (int k = 0; k < N / 4; ++k) {
        const float4 t = ld_global(reinterpret_cast<const float4*>(b + i) + k);
        x[4 * k] = t.x; x[4 * k + 1] = t.y; x[4 * k + 2] = t.z; x[4 * k + 3] = t.w;
    }
}

// fp32 state through 16-byte accesses when `vec`, else element by element.
template <int N>
__device__ __forceinline__ void load_state_any(const float* b, uint32_t i, bool vec, float (&x)[N]) {
    if (vec) {
        load_state<N>(b, i, x);
    } else {
#pragma unroll
        for (int k = 0; k < N; ++k) x[k] = ld_global(b + i + k);
    }
}

template <int N>
__device__ __forceinline__ void store_state(float* b, uint32_t i, const float (&x)[N]);

template <int N>
__device__ __forceinline__ void store_state_any(float* b, uint32_t i, bool vec, const float (&x)[N]) {
    if (vec) {
        store_state<N>(b, i, x);
    } else {
#pragma unroll
        for (int k = 0; k < N; ++k) st_global(b + i + k, x[k]);
    }
}

template <int N>
__device__ __forceinline__ void store_state(float* b, uint32_t i, const float (&x)[N]) {
#pragma unroll
    for (int k = 0; k < N / 4; ++k)
        st_global(reinterpret_cast<float4*>(b + i) + k,
               make_float4(x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3]));
}

// One element through the scalar path (chunk head, tail, or a chunk whose
// arrays are not mutually 16-byte aligned).  A skipped element is not even
// written back.
template <int DT, int ALGO, bool SKIP, int MODE = kPlain>
__device__ __forceinline__ void scalar_element(const ChunkRec& c, uint32_t i,
                                               const StepScalars& s, float scale = 1.0f,
                                               float wd = 0.0f)
{
    using P = Param<DT>;
    const float g = P::load1(c.g, i);
    if (SKIP && g == 0.0f) return;
    float p = P::load1(c.p, i);
    float m = ld_global(c.m + i);
    float v = ld_global(c.v + i);
    float m2 = 0.0f;
    if (ALGO == kAdEMAMix) m2 = ld_global(c.m2 + i);
    update<ALGO, false, MODE>(g, p, m, v, m2, s, scale, wd);
    P::store1(c.p, i, p);
    st_global(c.m + i, m);
    st_global(c.v + i, v);
    if (ALGO == kAdEMAMix) st_global(c.m2 + i, m2);
}

__device__ __forceinline__ bool aligned16(const void* q, uint32_t head, int bytes) {
    return ((reinterpret_cast<uintptr_t>(q) + static_cast<uintptr_t>(head) * bytes) & 15u) == 0;
}

// Alignment of the arrays other than param at the vector body's start.
struct Aligned {
    bool g, m, v, m2;
    __device__ bool all() const { return g && m && v && m2; }
};

// The vector body of a chunk: vectors [0, nvec) starting at element `head`,
// at which param is 16-byte aligned.  ALL: every other array is aligned too
// (the common case); otherwise each array uses 16-byte or element-wise
// accesses according to its own flag.  In the aligned case every lane moves 8
// elements per iteration (two 16-byte vectors of fp32, or one of fp16/bf16),
// so a warp iteration covers 256 contiguous elements of each array; the mixed
// case moves one vector per lane per iteration.
template <int DT, int ALGO, bool SKIP, bool ALL, int MODE = kPlain>
__device__ __forceinline__ void vector_body(const ChunkRec& c, const StepScalars& s, int lane,
                                            uint32_t head, uint32_t nvec, Aligned al,
                                            float scale = 1.0f, float wd = 0.0f)
{
    using P = Param<DT>;
    constexpr int V = P::kVec;
    constexpr int U = ALL ? 8 / V : 1;   // the mixed path keeps fewer values live
    for (uint32_t v0 = 0; v0 < nvec; v0 += 32 * U) {
        typename P::Raw graw[U], praw[U];
        float m[U][V], v[U][V], m2[U][V];
        // all loads of the iteration first, so they are in flight together
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t vi = v0 + u * 32 + lane;
            if (vi < nvec) {
                const uint32_t e = head + vi * V;
                graw[u] = (ALL || al.g) ? P::load(c.g, e) : P::load_elems(c.g, e);
                praw[u] = P::load(c.p, e);
                load_state_any<V>(c.m, e, ALL || al.m, m[u]);
                load_state_any<V>(c.v, e, ALL || al.v, v[u]);
                if (ALGO == kAdEMAMix) load_state_any<V>(c.m2, e, ALL || al.m2, m2[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t vi = v0 + u * 32 + lane;
            if (vi < nvec) {
                const uint32_t e = head + vi * V;
                float g[V], p[V];
                P::widen(graw[u], g);
                P::widen(praw[u], p);
#pragma unroll
                for (int j = 0; j < V; ++j)
                    update<ALGO, SKIP, MODE>(g[j], p[j], m[u][j], v[u][j], m2[u][j], s, scale, wd);
                P::store(c.p, e, P::narrow(p, praw[u], g, SKIP));
                store_state_any<V>(c.m, e, ALL || al.m, m[u]);
                store_state_any<V>(c.v, e, ALL || al.v, v[u]);
                if (ALGO == kAdEMAMix) store_state_any<V>(c.m2, e, ALL || al.m2, m2[u]);
            }
        }
    }
}

// One chunk, processed by one warp: a scalar head up to the element at which
// param is 16-byte aligned, the vector body, and a scalar tail.
template <int DT, int ALGO, bool SKIP, int MODE = kPlain>
__device__ __forceinline__ void run_chunk(const ChunkRec& c, const StepScalars& s, int lane,
                                          float scale = 1.0f, float wd = 0.0f)
{
    using P = Param<DT>;
    constexpr int V = P::kVec;
    const uint32_t len = c.len;
    uint32_t head = static_cast<uint32_t>(
        ((16u - (reinterpret_cast<uintptr_t>(c.p) & 15u)) & 15u) / P::kBytes);
    if (head > len) head = len;
    const uint32_t nvec = (len - head) / V;
    const uint32_t body_end = head + nvec * V;

    for (uint32_t i = lane; i < head; i += 32)
        scalar_element<DT, ALGO, SKIP, MODE>(c, i, s, scale, wd);
    for (uint32_t i = body_end + lane; i < len; i += 32)
        scalar_element<DT, ALGO, SKIP, MODE>(c, i, s, scale, wd);

    const Aligned al{aligned16(c.g, head, P::kBytes), aligned16(c.m, head, 4),
                     aligned16(c.v, head, 4), ALGO != kAdEMAMix || aligned16(c.m2, head, 4)};
    if (al.all())
        vector_body<DT, ALGO, SKIP, true, MODE>(c, s, lane, head, nvec, al, scale, wd);
    else
        vector_body<DT, ALGO, SKIP, false, MODE>(c, s, lane, head, nvec, al, scale, wd);
}

// A short 16-bit chunk (its record's dtype carries kShortFlag), processed by
// one warp with element-wise accesses: lane l takes elements l, l + 32, l + 64
// and l + 96, so each access instruction is still contiguous across the warp,
// and a lane updates at most 4 elements where one 16-byte vector would give it
// 8.  All loads come first, then the updates and stores.  Same arithmetic as
// the vector body; a skipped element is not written back.  Kept out of line,
// with its arguments by value (no stack frame), so that the step kernel's
// register count stays that of its vector path.
template <int DT, int ALGO, bool SKIP>
__device__ __noinline__ void short_chunk(const ChunkRec c, const StepScalars s, int lane)
{
    using P = Param<DT>;
    constexpr int K = kShortChunkElems / 32;
    const uint32_t len = c.len;
    float g[K], p[K], m[K], v[K], m2[K];
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const uint32_t i = lane + 32 * k;
        g[k] = p[k] = m[k] = v[k] = m2[k] = 0.0f;
        if (i < len) {
            g[k] = P::load1(c.g, i);
            p[k] = P::load1(c.p, i);
            m[k] = ld_global(c.m + i);
            v[k] = ld_global(c.v + i);
            if (ALGO == kAdEMAMix) m2[k] = ld_global(c.m2 + i);
        }
    }
#pragma unroll
    for (int k = 0; k < K; ++k) {
        const uint32_t i = lane + 32 * k;
        if (i < len && !(SKIP && g[k] == 0.0f)) {
            update<ALGO, false>(g[k], p[k], m[k], v[k], m2[k], s);
            P::store1(c.p, i, p[k]);
            st_global(c.m + i, m[k]);
            st_global(c.v + i, v[k]);
            if (ALGO == kAdEMAMix) st_global(c.m2 + i, m2[k]);
        }
    }
}

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
            constexpr int D = ONLY >= 0 ? ONLY : kF16;
            if (short16) short_chunk<D, ALGO, SKIP>(rec, s, lane);
            else run_chunk<D, ALGO, SKIP>(rec, s, lane);
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
// The element arithmetic is direction(), as in the plain step.  Every sum
// has a fixed order: lane l of the warp that owns a block adds the block's
// elements l, l + 32, l + 64, ... one after the other, the 32 lanes then
// combine in a fixed shuffle tree, a group's blocks and a tensor's groups are
// combined in fixed orders too; so the scale does not depend on the plan's
// chunk length, the block width or the storage alignment.  Accesses are
// element-wise and contiguous across the warp.
//
// Each lane accumulates its 64 squares of a block as a double-float: an
// unevaluated sum hi + lo of two binary32 numbers.  The square of a binary32
// x is exactly sq + err with sq = RN(x*x) and err = fma(x, x, -sq) (exact for
// 2^-50 <= |x| <= 2^56: no underflow of err, and 64 squares stay below
// 2^128), and hi + sq is split exactly into s + e by Knuth's TwoSum (Knuth,
// TAOCP vol. 2, 4.2.2, Theorem B); only lo + (e + err) is rounded, which
// errs by at most 2^-48 of the running sum.  Elements outside that range
// are added to a binary64 sum instead.  The lane's total is hi + lo + that
// sum in binary64, so the block's sum errs by at most about 2^-42 of itself,
// far below the fp32 rounding of the scale.  All of it stays on the fp32
// pipe: no float-to-double conversion per element.
// ---------------------------------------------------------------------------
constexpr float kSquareLo = 0x1p-50f;   // |x| range whose square splits exactly
constexpr float kSquareHi = 0x1p56f;

struct SquareSum {
    float hi = 0.0f, lo = 0.0f;
    double wide = 0.0;   // squares of out-of-range values

    __device__ __forceinline__ void add(float x)
    {
        const float ax = fabsf(x);
        if (ax >= kSquareLo && ax <= kSquareHi) {
            const float sq = __fmul_rn(x, x);
            const float err = __fmaf_rn(x, x, -sq);
            const float s = __fadd_rn(hi, sq);
            const float bp = __fsub_rn(s, hi);
            const float e = __fadd_rn(__fsub_rn(hi, __fsub_rn(s, bp)), __fsub_rn(sq, bp));
            hi = s;
            lo = __fadd_rn(lo, __fadd_rn(e, err));
        } else if (x != 0.0f) {
            const double xd = static_cast<double>(x);
            wide = __fma_rn(xd, xd, wide);
        }
    }

    __device__ __forceinline__ double total() const
    {
        return __dadd_rn(__dadd_rn(static_cast<double>(hi), static_cast<double>(lo)), wide);
    }
};

template <int DT, int ALGO, bool SKIP, int MODE>
__device__ __forceinline__ void norm_block(const ChunkRec& c, const StepScalars& s, int lane,
                                           float wd, double& sd, double& sp)
{
    using P = Param<DT>;
    constexpr int K = 8;
    const uint32_t len = c.len;
    SquareSum ad, ap;
    for (uint32_t base = 0; base < len; base += 32 * K) {
        float g[K], p[K], m[K], v[K], m2[K];
#pragma unroll
        for (int k = 0; k < K; ++k) {
            const uint32_t i = base + lane + 32 * k;
            g[k] = p[k] = m[k] = v[k] = m2[k] = 0.0f;
            if (i < len) {
                g[k] = P::load1(c.g, i);
                p[k] = P::load1(c.p, i);
                m[k] = ld_global(c.m + i);
                v[k] = ld_global(c.v + i);
                if (ALGO == kAdEMAMix) m2[k] = ld_global(c.m2 + i);
            }
        }
#pragma unroll
        for (int k = 0; k < K; ++k) {
            if (base + lane + 32 * k < len) {
                ap.add(p[k]);
                if (!(SKIP && g[k] == 0.0f)) {
                    const float u = direction<ALGO>(g[k], m[k], v[k], m2[k], s);
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

template <int ALGO, bool SKIP, int MODE>
__global__ void unorm_partials_kernel(const ChunkRec* __restrict__ blocks, int nblocks,
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
        case kF32: run_chunk<kF32, ALGO, SKIP, MODE>(rec, s, lane, sc, wd); break;
        case kF16: run_chunk<kF16, ALGO, SKIP, MODE>(rec, s, lane, sc, wd); break;
        default: run_chunk<kBF16, ALGO, SKIP, MODE>(rec, s, lane, sc, wd); break;
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

int only_class(int algo, int only)
{
    if (algo == kAdEMAMix) return 0;
    return only == kF16 ? 1 : (only == kBF16 ? 2 : 0);
}

// Resident blocks per SM and SM count, cached per device (and kernel / block
// size): device attributes are per device, not per process.
constexpr int kMaxDevices = 64;
struct OccEntry { int block_threads; int blocks_per_sm; };
struct DeviceInfo { int sms; OccEntry occ[12][6]; };
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

// ---------------------------------------------------------------------------
// Validation scaffolding: div_by_constant against __fdiv_rn on random operands.
// Operands come from the SplitMix64 output function (Steele, Lea & Flood,
// "Fast splittable pseudorandom number generators", OOPSLA 2014) applied to a
// counter.  mode 0: x is a random bit pattern (every class: zeros, subnormals,
// normals, infinities, NaNs).  mode 1: x = RN32(d * B) for B a random rounding
// boundary, so x/d lies close to a boundary (the hard cases).  d is a random
// binary32 in (0, 1] (subnormals included; d = 1 about once in 1,024 draws).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t splitmix64(uint64_t z)
{
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__global__ void check_division_kernel(uint64_t seed, int64_t n, int mode,
                                      unsigned long long* mismatches)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
        const uint64_t h1 = splitmix64(seed + 3 * static_cast<uint64_t>(i));
        const uint64_t h2 = splitmix64(seed + 3 * static_cast<uint64_t>(i) + 1);
        uint32_t dbits = (static_cast<uint32_t>(h2 >> 32) % 127u) << 23 |
                         static_cast<uint32_t>(h2 & 0x7FFFFFu);
        if (dbits == 0) dbits = 1;
        if ((h2 >> 54) == 0) dbits = 0x3F800000u;          // d = 1
        const float d = __uint_as_float(dbits);
        float x;
        if (mode == 0) {
            x = __uint_as_float(static_cast<uint32_t>(h1));
        } else {
            // a rounding boundary: the midpoint just above a random finite float
            const uint64_t h3 = splitmix64(seed + 3 * static_cast<uint64_t>(i) + 2);
            const float f = __uint_as_float(static_cast<uint32_t>(h3) & 0x7F7FFFFFu);
            const double mid = 0.5 * (static_cast<double>(f) +
                                      static_cast<double>(__uint_as_float(__float_as_uint(f) + 1)));
            x = __double2float_rn(__dmul_rn(mid, static_cast<double>(d)));
            if (h1 & 1) x = -x;
        }
        const float a = div_by_constant(x, __drcp_rn(static_cast<double>(d)));
        const float b = __fdiv_rn(x, d);
        const bool same = __float_as_uint(a) == __float_as_uint(b) || (isnan(a) && isnan(b));
        if (!same) atomicAdd(mismatches, 1ull);
    }
}

}  // namespace

cudaError_t check_division(uint64_t seed, int64_t n, int mode, unsigned long long* d_count,
                           cudaStream_t stream)
{
    check_division_kernel<<<148 * 8, 256, 0, stream>>>(seed, n, mode, d_count);
    return cudaGetLastError();
}

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
        const int k = ((algo == kAdEMAMix ? 2 : 0) + (skip_zeros ? 1 : 0)) * 3 + only_class(algo, only);
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
    constexpr int kNormThreads = 256;
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
