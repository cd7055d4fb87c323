// opt2s_device.cuh -- the element arithmetic and the chunk walkers shared by
// the step kernels (opt2s_kernel.cu) and the 8-bit-state kernel
// (opt2s_kernel8.cu).  Device code only; every name is local to the
// translation unit that includes it.
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
// order and never depends on which code path (vector body, scalar head/tail),
// chunk, warp or block computed it.
#pragma once

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
// Exact division by a per-launch constant d, 2^-25 <= d <= 1 (the bias
// corrections bc1, bc2), with r = RN64(1/d) and its fp32 split hi = RN32(r),
// lo = RN32(r - hi) computed once per launch on the host.
//
// Wide route, for every binary32 x:  RN32( RN64(x * r) ) == RN32(x / d).
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
// Arithmetic, 2nd ed., ch. 4.)
//
// fp32 route, for 2^-40 <= |x| < 2^96 (everything else takes the wide route):
//     q0 = RN32(x*hi + RN32(x*lo)),  rem = x - q0*d,  q = RN32(q0 + rem*hi).
// hi + lo is 1/d to within 2^-47 (relative), so q0 is x/d to within half an
// ulp plus 2^-46 relative: a faithful quotient.  The remainder of a faithful
// quotient is a binary32 number, so one FMA computes it exactly (it is a
// multiple of 2^-111 here: no underflow), and with hi the correctly rounded
// reciprocal, RN32(q0 + rem*hi) is the correctly rounded quotient
// (Markstein's theorem: P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990; also
// Muller et al., ch. 4).  No step overflows or underflows in that range
// (|x/d| < 2^121).
// Which route a kernel uses is a measured choice (both are exact): the
// binary64 route element by element in the plain step kernels (kDivWide);
// the fp32 route with one range test for a group of elements, and the
// binary64 route for the whole group when any value is out of range
// (update_group, kDivGroup), in the 8-bit-state kernel, the norm pass and
// the scaled step.  A per-element range test cost those kernels more than the
// route saved: its branch keeps the elements' dependent chains from
// interleaving.
// GPU tests check both routes against __fdiv_rn: every binary32 x for a
// sample of divisors, and random operands near rounding boundaries.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float div_by_constant(float x, double r)
{
    return __double2float_rn(__dmul_rn(static_cast<double>(x), r));
}

// The fp32 route's range as one unsigned comparison: x is in range exactly
// when fma_range_key(x) < kFmaRangeEnd (the biased exponent of |x| in
// [87, 223), i.e. 2^-40 <= |x| < 2^96).  The maximum of several keys tests
// several values at once.
constexpr uint32_t kFmaRangeEnd = 136u << 23;
__device__ __forceinline__ uint32_t fma_range_key(float x)
{
    return (__float_as_uint(x) & 0x7F800000u) - (87u << 23);
}

// The fp32 route's arithmetic, for x in its range.
__device__ __forceinline__ float div_by_constant_in_range(float x, float d, float hi, float lo)
{
    const float q0 = __fmaf_rn(x, hi, __fmul_rn(x, lo));
    const float rem = __fmaf_rn(-q0, d, x);
    return __fmaf_rn(rem, hi, q0);
}

// Routes of m/bc1 and v/bc2 in the vector walkers: the binary64 product
// element by element, or the fp32 route a group at a time (update_group).
enum : int { kDivWide = 0, kDivGroup = 1 };

// ---------------------------------------------------------------------------
// The per-element update.  direction() moves the moments of one element (in
// place) and returns its update direction u = num/den; m/bc1 and v/bc2 use
// the exact constant division above (the binary64 route), num/den is an
// IEEE division.  update()
// then applies the step to p.  With SKIP, an element whose gradient compares
// equal to zero (+0 or -0) is left untouched (no decay either).  MODE:
//   kPlain   p = p*decay - lr*u
//   kScaled  p = p*decay - lr*(scale*u)   (bounded update norm; scale = 1
//                                          gives the plain value)
//   kLamb    p = p - lr*(scale*w), w = u + wd*p   (LAMB: the weight decay
//                                          inside the trust-ratio scaled step)
// ---------------------------------------------------------------------------
enum : int { kPlain = 0, kScaled = 1, kLamb = 2 };

// The moments of one element, in place: m, v (and AdEMAMix's m2).
template <int ALGO>
__device__ __forceinline__ void moments(float g, float& m, float& v, float& m2, const StepScalars& s)
{
    m = __fadd_rn(__fmul_rn(s.beta1, m), __fmul_rn(s.one_minus_beta1, g));
    v = __fadd_rn(__fmul_rn(s.beta2, v),
                  __fmul_rn(__fmul_rn(s.one_minus_beta2, g), g));
    if (ALGO == kAdEMAMix) m2 = __fadd_rn(__fmul_rn(s.beta3, m2), __fmul_rn(s.one_minus_beta3, g));
}

// u = num/den from the bias-corrected moments mh = m/bc1 and vh = v/bc2.
template <int ALGO>
__device__ __forceinline__ float direction_of(float mh, float vh, float m2, const StepScalars& s)
{
    const float num = ALGO == kAdEMAMix ? __fadd_rn(mh, __fmul_rn(s.alpha, m2)) : mh;
    const float den = __fadd_rn(__fsqrt_rn(vh), s.eps);
    return __fdiv_rn(num, den);
}

// The plain step's param update: p*decay - lr*u.
__device__ __forceinline__ float plain_param(float p, float u, const StepScalars& s)
{
    return __fsub_rn(__fmul_rn(p, s.decay), __fmul_rn(s.lr, u));
}

template <int ALGO>
__device__ __forceinline__ float direction(float g, float& m, float& v, float& m2,
                                           const StepScalars& s)
{
    moments<ALGO>(g, m, v, m2, s);
    return direction_of<ALGO>(div_by_constant(m, s.inv_bc1), div_by_constant(v, s.inv_bc2), m2, s);
}

// LAMB's decayed direction w = u + wd*p of an element.
__device__ __forceinline__ float lamb_direction(float u, float p, float wd)
{
    return __fadd_rn(u, __fmul_rn(wd, p));
}

// The param after the step, from its direction u (MODE as above).
template <int MODE>
__device__ __forceinline__ float param_after(float p, float u, const StepScalars& s, float scale,
                                             float wd)
{
    if (MODE == kLamb) return __fsub_rn(p, __fmul_rn(s.lr, __fmul_rn(scale, lamb_direction(u, p, wd))));
    return plain_param(p, MODE == kScaled ? __fmul_rn(scale, u) : u, s);
}

template <int ALGO, bool SKIP, int MODE = kPlain>
__device__ __forceinline__ void update(float g, float& p, float& m, float& v,
                                       float& m2, const StepScalars& s, float scale = 1.0f,
                                       float wd = 0.0f)
{
    if (SKIP && g == 0.0f) return;
    const float u = direction<ALGO>(g, m, v, m2, s);
    p = param_after<MODE>(p, u, s, scale, wd);
}

// update() on G of a thread's elements, O .. O+G-1 of its arrays, phase by
// phase: the moments of all G, one range test for all their bias-correction
// divisions (the fp32 route when every value is in its range, else the
// binary64 route for all G: both are exact, so either gives the same
// quotients), then the directions and the params.  No per-element branch
// separates the elements' dependent chains, so they interleave.  With SKIP an
// element whose gradient compares equal to zero keeps p, m, v and m2.
template <int ALGO, bool SKIP, int MODE, int O, int G, int N>
__device__ __forceinline__ void update_group(const float (&g)[N], float (&p)[N], float (&m)[N],
                                             float (&v)[N], float (&m2)[N], const StepScalars& s,
                                             float scale = 1.0f, float wd = 0.0f)
{
    static_assert(O + G <= N, "group inside the arrays");
    float mn[G], vn[G], m2n[G], mh[G], vh[G];
    uint32_t key = 0;
#pragma unroll
    for (int j = 0; j < G; ++j) {
        mn[j] = m[O + j];
        vn[j] = v[O + j];
        m2n[j] = m2[O + j];
        moments<ALGO>(g[O + j], mn[j], vn[j], m2n[j], s);
        key = max(key, max(fma_range_key(mn[j]), fma_range_key(vn[j])));
    }
    if (__builtin_expect(key >= kFmaRangeEnd, 0)) {
#pragma unroll
        for (int j = 0; j < G; ++j) {
            mh[j] = div_by_constant(mn[j], s.inv_bc1);
            vh[j] = div_by_constant(vn[j], s.inv_bc2);
        }
    } else {
#pragma unroll
        for (int j = 0; j < G; ++j) {
            mh[j] = div_by_constant_in_range(mn[j], s.bc1, s.rcp_bc1_hi, s.rcp_bc1_lo);
            vh[j] = div_by_constant_in_range(vn[j], s.bc2, s.rcp_bc2_hi, s.rcp_bc2_lo);
        }
    }
#pragma unroll
    for (int j = 0; j < G; ++j) {
        const float pn = param_after<MODE>(p[O + j], direction_of<ALGO>(mh[j], vh[j], m2n[j], s), s, scale, wd);
        if (!SKIP || g[O + j] != 0.0f) {
            p[O + j] = pn;
            m[O + j] = mn[j];
            v[O + j] = vn[j];
            m2[O + j] = m2n[j];
        }
    }
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
template <int DT, int ALGO, bool SKIP, bool ALL, int MODE = kPlain, int U16 = 1, int ROUTE = kDivWide>
__device__ __forceinline__ void vector_body(const ChunkRec& c, const StepScalars& s, int lane,
                                            uint32_t head, uint32_t nvec, Aligned al,
                                            float scale = 1.0f, float wd = 0.0f)
{
    using P = Param<DT>;
    constexpr int V = P::kVec;
    // vectors a lane moves per iteration: 8 elements (U16 x 8 for 16-bit
    // storage in the kernels specialised to one dtype); the mixed path keeps
    // fewer values live
    constexpr int U = ALL ? (V == 8 ? U16 : 8 / V) : 1;
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
                if (ROUTE == kDivGroup) {
                    update_group<ALGO, SKIP, MODE, 0, V, V>(g, p, m[u], v[u], m2[u], s, scale, wd);
                } else {
#pragma unroll
                    for (int j = 0; j < V; ++j)
                        update<ALGO, SKIP, MODE>(g[j], p[j], m[u][j], v[u][j], m2[u][j], s, scale, wd);
                }
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
template <int DT, int ALGO, bool SKIP, int MODE = kPlain, int U16 = 1, int ROUTE = kDivWide>
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
        vector_body<DT, ALGO, SKIP, true, MODE, U16, ROUTE>(c, s, lane, head, nvec, al, scale, wd);
    else
        vector_body<DT, ALGO, SKIP, false, MODE, 1, ROUTE>(c, s, lane, head, nvec, al, scale, wd);
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

}  // namespace
}  // namespace opt2s
