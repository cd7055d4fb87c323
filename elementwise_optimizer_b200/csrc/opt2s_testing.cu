// opt2s_testing.cu -- validation scaffolding built only into the test
// variant of the library (libopt2s_testing.so): a kernel that checks the
// step kernel's exact division by a per-launch constant against IEEE
// division on random operands.  The bitsandbytes issue "Investigate a
// 256-thread SM103 path for small 32-bit optimizer tensors", section "Scope",
// keeps experimental forcing and checks in validation scaffolding, out of the
// public API.

#include "opt2s_device.cuh"

namespace opt2s {
namespace {

// ---------------------------------------------------------------------------
// Validation scaffolding: both routes of the constant division against
// __fdiv_rn (the fp32 route on the operands in its range).  Operands come from the SplitMix64 output function (Steele, Lea
// & Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014)
// applied to a counter.
// Divisors lie in [2^-25, 1], the bias corrections' range: a random binade
// and significand, with d = 1, powers of two and all-ones significands drawn
// often.  The reciprocal and its fp32 split are formed as the host forms them.
//   mode 0: n operands, x a random bit pattern (every class: zeros,
//           subnormals, normals, infinities, NaNs);
//   mode 1: n operands, x = RN32(d * B) for B a random rounding boundary, so
//           that x/d lies close to a boundary (the hard cases);
//   mode 2: n divisors, each with every one of the 2^32 binary32 x.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t splitmix64(uint64_t z)
{
    z += 0x9E3779B97F4A7C15ull;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

__device__ __forceinline__ float draw_divisor(uint64_t h)
{
    uint32_t bits = (102u + static_cast<uint32_t>((h >> 32) % 25u)) << 23 |
                    static_cast<uint32_t>(h & 0x7FFFFFu);          // [2^-25, 1)
    if (((h >> 44) & 15u) == 0) bits &= 0xFF800000u;               // a power of two
    if (((h >> 48) & 15u) == 0) bits |= 0x007FFFFFu;               // all-ones significand
    if (((h >> 52) & 63u) == 0) bits = 0x3F800000u;                // d = 1
    return __uint_as_float(bits);
}

__device__ __forceinline__ bool same_quotient(float x, float d)
{
    const double r = __drcp_rn(static_cast<double>(d));
    const float hi = __double2float_rn(r);
    const float lo = __double2float_rn(__dsub_rn(r, static_cast<double>(hi)));
    const float a = div_by_constant(x, r);                   // binary64 route
    const float b = __fdiv_rn(x, d);
    auto same = [](float u, float w) { return __float_as_uint(u) == __float_as_uint(w) || (isnan(u) && isnan(w)); };
    // the fp32 route, for x in its range (a group with a value outside it
    // takes the binary64 route)
    const bool in_range = fma_range_key(x) < kFmaRangeEnd;
    return same(a, b) && (!in_range || same(div_by_constant_in_range(x, d, hi, lo), b));
}

__global__ void check_division_kernel(uint64_t seed, int64_t n, int mode,
                                      unsigned long long* mismatches)
{
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t total = mode == 2 ? (n << 32) : n;
    unsigned long long bad = 0;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        float x, d;
        if (mode == 2) {
            d = draw_divisor(splitmix64(seed + static_cast<uint64_t>(i >> 32)));
            x = __uint_as_float(static_cast<uint32_t>(i));
        } else {
            const uint64_t h1 = splitmix64(seed + 3 * static_cast<uint64_t>(i));
            d = draw_divisor(splitmix64(seed + 3 * static_cast<uint64_t>(i) + 1));
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
        }
        if (!same_quotient(x, d)) ++bad;
    }
    if (bad) atomicAdd(mismatches, bad);
}

}  // namespace

cudaError_t check_division(uint64_t seed, int64_t n, int mode, unsigned long long* d_count,
                           cudaStream_t stream)
{
    check_division_kernel<<<148 * 8, 256, 0, stream>>>(seed, n, mode, d_count);
    return cudaGetLastError();
}

}  // namespace opt2s
