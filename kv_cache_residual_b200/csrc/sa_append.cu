// Cache append during decode: one token per unit written at position L and
// the statistics refreshed to cover L + 1 tokens (sa_append in sa_decode.h).
//
// k_append: grid (B*Hkv), 128 threads; thread e owns column e of the unit's
// new key and value row (e < d).  It copies the row into the cache, adds it
// to the key and value totals, and for each query head h of the unit takes
// the logit p = s mu_q,h . k_new (a block sum in warp order) to fold the new
// token into the typical query's attention: log_z0 grows by ln(1 + e^(p -
// log_z0)) and O_Est becomes the mass-weighted mix of the old O_Est and v_new
// (RESA, key design 1: O_Est and Z are that query's softmax over the cache).
// When the token completes 16-token block `blk`, warp 0 then forms that
// block's mean (fp64 sum of its 16 rows, rounded once to the cache dtype, as
// the prefill does), raises kbar_absmax and writes the block's sketch row
// (sketch_row, shared with the prefill's sketch kernel).  When the statistics
// carry per-block key bounds, a second launch forms the completed block's
// elementwise minimum and maximum.
#include "sa_common.cuh"
#include "sa_internal.h"
#include "sa_sketch.cuh"

namespace sa {

constexpr int kAppendThreads = 128;

template <typename T, int D, int G>
__global__ void __launch_bounds__(kAppendThreads)
k_append(const T* __restrict__ k_new, const T* __restrict__ v_new, T* __restrict__ k, T* __restrict__ v,
         sa_stats st, int Hq, int Hkv, int L, int ld, float scale, int blk) {
    static_assert(D <= kAppendThreads, "one thread per column");
    constexpr int NW = kAppendThreads / 32;
    __shared__ float s_part[G][NW];
    const int u = blockIdx.x, b = u / Hkv, g = u - b * Hkv;
    const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
    const bool live = e < D;
    const size_t qh0 = (size_t)b * Hq + (size_t)g * G;
    float kf = 0.f, vf = 0.f;
    if (live) {
        const T kr = k_new[(size_t)u * D + e], vr = v_new[(size_t)u * D + e];
        const size_t row = ((size_t)u * ld + L) * D + e;
        k[row] = kr;
        v[row] = vr;
        kf = to_f32<T>(kr);
        vf = to_f32<T>(vr);
        st.sum_k[(size_t)u * D + e] += kf;
        st.sum_v[(size_t)u * D + e] += vf;
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float x = live ? st.mu_q[(qh0 + h) * D + e] * kf : 0.f;
        x = group_sum<32>(x);
        if (lane == 0) s_part[h][warp] = x;
    }
    __syncthreads();
    float lz_new[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float x = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) x += s_part[h][w];
        const float p = scale * x;
        const float lz = st.log_z0[qh0 + h];
        const float m = fmaxf(lz, p);
        lz_new[h] = m + log1pf(expf(-fabsf(lz - p)));
        if (live) {
            float* o = st.o_est + (qh0 + h) * D + e;
            *o = expf(lz - lz_new[h]) * *o + expf(p - lz_new[h]) * vf;
        }
    }
    __syncthreads();           // every thread has read log_z0; the new row is in the cache
    if (e == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) st.log_z0[qh0 + h] = lz_new[h];
    }
    if (blk < 0 || warp != 0) return;
    // the completed block: lane l owns columns [l E, l E + E)
    constexpr int E = D / 32;
    double sum[E];
#pragma unroll
    for (int c = 0; c < E; ++c) sum[c] = 0.0;
    for (int j = 0; j < 16; ++j) {
        const T* r = k + ((size_t)u * ld + 16 * (size_t)blk + j) * D + lane * E;
#pragma unroll
        for (int c = 0; c < E; ++c) sum[c] += (double)to_f32<T>(r[c]);
    }
    const size_t row = (size_t)u * (ld / 16) + blk;
    T* bm = reinterpret_cast<T*>(st.blk_mean) + row * D + lane * E;
    float kbar[E];
    double m[E];
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < E; ++c) {
        const T mean = round_from_f64<T>(sum[c] * 0.0625);
        bm[c] = mean;
        kbar[c] = to_f32<T>(mean);
        amax = fmaxf(amax, fabsf(kbar[c]));
        m[c] = (double)st.mu_k[(size_t)u * D + lane * E + c];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    // non-negative floats order like their bit patterns as signed ints
    if (lane == 0 && amax > 0.f) atomicMax(reinterpret_cast<int*>(st.kbar_absmax + u), __float_as_int(amax));
    sketch_row<D>(kbar, m, st.blk_code + row * D, reinterpret_cast<float4*>(st.blk_meta) + row);
}

template <typename T, int D, int G>
static cudaError_t append_t(const Dims& d, const void* k_new, const void* v_new, void* k, void* v,
                            const sa_stats& st, float scale, cudaStream_t s) {
    k_append<T, D, G><<<d.U(), kAppendThreads, 0, s>>>(
        reinterpret_cast<const T*>(k_new), reinterpret_cast<const T*>(v_new), reinterpret_cast<T*>(k),
        reinterpret_cast<T*>(v), st, d.Hq, d.Hkv, d.L, d.ld, scale, (d.L + 1) % 16 == 0 ? (d.L + 1) / 16 - 1 : -1);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || st.blk_min == nullptr || (d.L + 1) % 16 != 0) return e;
    // the completed block's key bounds (after the row is written, same stream)
    return launch_block_minmax(d, k, (d.L + 1) / 16 - 1, (d.L + 1) / 16, st.blk_min, st.blk_max, s);
}

template <typename T, int D>
static cudaError_t append_g(const Dims& d, const void* k_new, const void* v_new, void* k, void* v,
                            const sa_stats& st, float scale, cudaStream_t s) {
    switch (d.G) {
        case 1: return append_t<T, D, 1>(d, k_new, v_new, k, v, st, scale, s);
        case 2: return append_t<T, D, 2>(d, k_new, v_new, k, v, st, scale, s);
        case 4: return append_t<T, D, 4>(d, k_new, v_new, k, v, st, scale, s);
        case 8: return append_t<T, D, 8>(d, k_new, v_new, k, v, st, scale, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_append(const Dims& d, const void* k_new, const void* v_new, void* k, void* v,
                          const sa_stats& st, float scale, cudaStream_t s) {
    if (d.bf16)
        return d.d == 128 ? append_g<__nv_bfloat16, 128>(d, k_new, v_new, k, v, st, scale, s)
                          : append_g<__nv_bfloat16, 64>(d, k_new, v_new, k, v, st, scale, s);
    return d.d == 128 ? append_g<float, 128>(d, k_new, v_new, k, v, st, scale, s)
                      : append_g<float, 64>(d, k_new, v_new, k, v, st, scale, s);
}

}  // namespace sa
