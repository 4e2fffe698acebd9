// CTA-level merges of per-lane online-softmax states, and the fixed-order
// combine of split partials.  Shared by prefill, decode and dense kernels.
#pragma once

#include "sa_common.cuh"

namespace sa {

// Record of one split: m[G], l[G], acc[G][D] (floats, contiguous).
template <int G, int D>
struct Rec {
    static constexpr int kFloats = G * (2 + D);
};

// Merge the lane-group states of a warp (groups hold different rows of the
// same dims) so that every group ends with the warp's state.
template <int G, int EPC, int CPR>
__device__ __forceinline__ void warp_merge(Online<G, EPC>& st) {
#pragma unroll
    for (int off = CPR; off < 32; off <<= 1) st.merge_xor(off);
}

// Cross-warp merge into one record.  `sm` holds kWarps * G * (D + 2) floats.
// Deterministic: warps are combined in index order.
template <int G, int EPC, int CPR, int D>
__device__ void cta_merge_store(const Online<G, EPC>& st, float* sm, float* rec) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int W = D + 2;
    if (lane < CPR) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float* row = sm + (warp * G + h) * W;
#pragma unroll
            for (int e = 0; e < EPC; ++e) row[2 + lane * EPC + e] = st.acc[h][e];
            if (lane == 0) { row[0] = st.m[h]; row[1] = st.l[h]; }
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
        const int h = idx / D, e = idx - h * D;
        float M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sm[(w * G + h) * W]);
        float A = 0.f, Ls = 0.f;
        for (int w = 0; w < kWarps; ++w) {
            const float* row = sm + (w * G + h) * W;
            const float f = (row[0] == -INFINITY) ? 0.f : ex2(row[0] - M);
            A = fmaf(row[2 + e], f, A);
            Ls = fmaf(row[1], f, Ls);
        }
        rec[2 * G + h * D + e] = A;
        if (e == 0) { rec[h] = M; rec[G + h] = Ls; }
    }
    __syncthreads();
}

// Combine `ns` split records (stride `stride` floats, written by other CTAs)
// for head h, dim e, in split order.  Returns acc; M and L through refs.
template <int G, int D>
__device__ __forceinline__ float combine_splits(const float* recs, int ns, int stride, int h, int e,
                                                float& M, float& Ls) {
    M = -INFINITY;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, ldcg(recs + (size_t)s * stride + h));
    float A = 0.f;
    Ls = 0.f;
    for (int s = 0; s < ns; ++s) {
        const float* r = recs + (size_t)s * stride;
        const float m = ldcg(r + h);
        const float f = (m == -INFINITY) ? 0.f : ex2(m - M);
        A = fmaf(ldcg(r + 2 * G + h * D + e), f, A);
        Ls = fmaf(ldcg(r + G + h), f, Ls);
    }
    return A;
}

}  // namespace sa
