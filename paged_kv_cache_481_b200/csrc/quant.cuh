// Affine 8-bit quantization of one (token, head) row, shared by the int8
// cache write and the decode's fused append so both take identical
// decisions (brentwoodlivery.com 5.3.18, low-bit KV cache: with b = 8,
// s = (r_max - r_min) / 255, z = round(-r_min / s), q = round(r / s) + z).
// Decisions in fp32 with IEEE division and round-half-to-even; codes are
// clamped to [0, 255]; a row with no spread (all values c) uses s = |c|
// (1 when c = 0) so that it reconstructs exactly.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace pa {

// One row of E * 32 values, E per lane of a full warp (lane l holds values
// [E l, E (l + 1))).  Returns this lane's E codes packed little-endian into
// the low 8 E bits; every lane gets the row's (s, z).
template <int E>
__device__ __forceinline__ uint32_t quantize_row_warp(const float (&x)[E], float &sc, float &z)
{
    float rmin = x[0], rmax = x[0];
#pragma unroll
    for (int e = 1; e < E; ++e) {
        rmin = fminf(rmin, x[e]);
        rmax = fmaxf(rmax, x[e]);
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
        rmin = fminf(rmin, __shfl_xor_sync(kFullMask, rmin, off));
        rmax = fmaxf(rmax, __shfl_xor_sync(kFullMask, rmax, off));
    }
    sc = (rmax - rmin) / 255.0f;
    if (sc == 0.0f)
        sc = rmax != 0.0f ? fabsf(rmax) : 1.0f;
    z = rintf(-rmin / sc);
    uint32_t packed = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const float q = fminf(fmaxf(rintf(x[e] / sc) + z, 0.0f), 255.0f);
        packed |= uint32_t(q) << (8 * e);
    }
    return packed;
}

} // namespace pa
