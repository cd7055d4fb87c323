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

}  // namespace opt2s
