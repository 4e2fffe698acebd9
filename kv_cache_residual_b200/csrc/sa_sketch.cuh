// One row of the block-mean scan sketch, computed by one warp (lane l holds
// elements [l E, l E + E) of the row, E = D / 32): relative to the unit's
// centre m (its typical key mu_k), t = kbar - m, s = fl32(max|t| / 127),
// code = clamp(rint(t / s), +-127) and the f32 upper bounds rn >= ||t - s
// code||_2, kn >= ||s code||_2.  Centring shifts every block's score by the
// same qbar . m, which leaves the ranking unchanged, and lets the 8-bit codes
// resolve the blocks' differences rather than the key mean they share.  In
// fp64, t and t - s code are each rounded once (|error| <= 2^-53 of the
// value) and the sums of squares carry at most (D + 5) 2^-53 relative error:
// rn adds 2^-52 (||t|| + ||r||) and both bounds a 2^-40 relative margin
// before rounding up.  Used by the prefill / block-summary sketch kernel and
// by the cache append.
#pragma once

#include "sa_common.cuh"

namespace sa {

template <int D>
__device__ __forceinline__ void sketch_row(const float (&kbar)[D / 32], const double (&m)[D / 32],
                                           int8_t* __restrict__ code_row, float4* __restrict__ meta_row) {
    constexpr int E = D / 32;
    const int lane = threadIdx.x & 31;
    double t[E];
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        t[e] = (double)kbar[e] - m[e];
        amax = fmaxf(amax, (float)fabs(t[e]));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    // amax may round below max|t|: the clamp keeps the codes in range
    const float sc = amax / 127.0f;
    int c[E];
    double r2 = 0.0, k2 = 0.0, t2 = 0.0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        int ci = 0;
        if (sc > 0.f) ci = max(-127, min(127, (int)rint(t[e] / (double)sc)));
        c[e] = ci;
        const double q = (double)sc * (double)ci;         // exact
        const double r = t[e] - q;
        r2 = fma(r, r, r2);
        k2 = fma(q, q, k2);
        t2 = fma(t[e], t[e], t2);
    }
    r2 = group_sum_f64<32>(r2);
    k2 = group_sum_f64<32>(k2);
    t2 = group_sum_f64<32>(t2);
    uint32_t packed = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) packed |= (uint32_t)(c[e] & 0xff) << (8 * e);
    if constexpr (E == 4) *reinterpret_cast<uint32_t*>(code_row + lane * E) = packed;
    else *reinterpret_cast<uint16_t*>(code_row + lane * E) = (uint16_t)packed;
    if (lane == 0) {
        const double mg = 1.0 + 0x1p-40;
        const double rn = sqrt(r2) * mg + 0x1p-52 * (sqrt(t2) + sqrt(r2)) * mg;
        *meta_row = make_float4(sc, __double2float_ru(rn), __double2float_ru(sqrt(k2) * mg), 0.f);
    }
}

}  // namespace sa
