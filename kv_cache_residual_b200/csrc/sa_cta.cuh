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

// Split combine in two phases, for the last CTA of a unit:
//  1. per head (one warp per head, lanes over splits): M = max_s m_s and
//     L = sum_s l_s 2^(m_s - M), into s_M[h], s_L[h];
//  2. per (head, dim): acc = sum_s acc_s 2^(m_s - M), in split order, four
//     splits' loads in flight at a time.
// `off` selects the record (0: exact, G*(2+D): prior).  Deterministic.
// Record loads: other CTAs' records through L2 (.cg), or this CTA's own
// records in shared memory (plain generic loads).
template <bool SH>
__device__ __forceinline__ float ld_rec(const float* p) {
    if constexpr (SH) return *p;
    else return __ldcg(p);
}

template <int G, int D, bool SH = false>
__device__ void combine_heads(const float* recs, int ns, int stride, int off, float* s_M, float* s_L) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    for (int h = warp; h < G; h += nw) {
        float M = -INFINITY;
        for (int s = lane; s < ns; s += 32) M = fmaxf(M, ld_rec<SH>(recs + (size_t)s * stride + off + h));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        float Ls = 0.f;
        for (int s = lane; s < ns; s += 32) {
            const float m = ld_rec<SH>(recs + (size_t)s * stride + off + h);
            const float l = ld_rec<SH>(recs + (size_t)s * stride + off + G + h);
            Ls += (m == -INFINITY) ? 0.f : l * ex2(m - M);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, o);
        if (lane == 0) { s_M[h] = M; s_L[h] = Ls; }
    }
}

template <int G, int D, bool SH = false>
__device__ __forceinline__ float combine_acc(const float* recs, int ns, int stride, int off, int h, int e, float M) {
    float A = 0.f;
    int s = 0;
    for (; s + 4 <= ns; s += 4) {
        float m[4], a[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float* r = recs + (size_t)(s + j) * stride + off;
            m[j] = ld_rec<SH>(r + h);
            a[j] = ld_rec<SH>(r + 2 * G + h * D + e);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) A = fmaf(a[j], (m[j] == -INFINITY) ? 0.f : ex2(m[j] - M), A);
    }
    for (; s < ns; ++s) {
        const float* r = recs + (size_t)s * stride + off;
        const float m = ld_rec<SH>(r + h);
        A = fmaf(ld_rec<SH>(r + 2 * G + h * D + e), (m == -INFINITY) ? 0.f : ex2(m - M), A);
    }
    return A;
}

}  // namespace sa
