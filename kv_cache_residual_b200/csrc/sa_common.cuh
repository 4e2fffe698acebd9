// Device-side building blocks shared by the sparse-decode kernels (sm_100a).
//
// Row geometry: a cache row (one token's key or value, d elements) is read as
// 16-byte chunks; CPR = chunks per row lanes form a "lane group" that owns one
// row at a time, each lane holding EPC = 16 / sizeof(T) consecutive elements.
//   bf16, d=128: 16 lanes x 8 elems (2 groups per warp)
//   bf16, d=64 :  8 lanes x 8 elems (4 groups per warp)
//   f32,  d=128: 32 lanes x 4 elems (1 group per warp)
//   f32,  d=64 : 16 lanes x 4 elems (2 groups per warp)
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {

constexpr int kBlock = 16;          // tokens per selection block
constexpr int kThreads = 256;       // threads per CTA for every kernel here
constexpr int kWarps = kThreads / 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename T, int D>
struct Geom {
    static constexpr int EPC = 16 / (int)sizeof(T);   // elements per 16-B chunk
    static constexpr int CPR = D / EPC;               // chunks (lanes) per row
    static constexpr int GPW = 32 / CPR;              // lane groups per warp
    static constexpr int NG = GPW * kWarps;           // lane groups per CTA
    static_assert(CPR >= 1 && CPR <= 32 && (32 % CPR) == 0, "row geometry");
};

// ---- loads ---------------------------------------------------------------

__device__ __forceinline__ uint4 ld_nc16(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// streaming read that does not allocate in L1
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

template <typename T>
__device__ __forceinline__ void unpack(const uint4& w, float* f);

template <>
__device__ __forceinline__ void unpack<__nv_bfloat16>(const uint4& w, float* f) {
    f[0] = bf16lo(w.x); f[1] = bf16hi(w.x);
    f[2] = bf16lo(w.y); f[3] = bf16hi(w.y);
    f[4] = bf16lo(w.z); f[5] = bf16hi(w.z);
    f[6] = bf16lo(w.w); f[7] = bf16hi(w.w);
}

template <>
__device__ __forceinline__ void unpack<float>(const uint4& w, float* f) {
    f[0] = __uint_as_float(w.x); f[1] = __uint_as_float(w.y);
    f[2] = __uint_as_float(w.z); f[3] = __uint_as_float(w.w);
}

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// one rounding from fp64 to the storage type (nearest, ties to even)
template <typename T>
__device__ __forceinline__ T round_from_f64(double x);
template <>
__device__ __forceinline__ float round_from_f64<float>(double x) { return __double2float_rn(x); }
template <>
__device__ __forceinline__ __nv_bfloat16 round_from_f64<__nv_bfloat16>(double x) {
    unsigned short r;
    asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(r) : "d"(x));
    return __ushort_as_bfloat16(r);
}

// pack EPC values of T into one 16-byte chunk (element 0 in the low bits)
__device__ __forceinline__ uint4 pack16(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
}
__device__ __forceinline__ uint4 pack16(const __nv_bfloat16* f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = (uint32_t)__bfloat16_as_ushort(f[2 * i]) | ((uint32_t)__bfloat16_as_ushort(f[2 * i + 1]) << 16);
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// ---- arithmetic ------------------------------------------------------------

// 2^x via the SFU instruction (relative error ~2^-22; ftz; 2^-inf = 0)
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// d = a * b + d on two fp32 lanes at once (packed FMA, round to nearest)
__device__ __forceinline__ void ffma2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
    asm("{\n\t.reg .b64 A, B, C;\n\tmov.b64 A, {%2, %3};\n\tmov.b64 B, {%4, %5};\n\tmov.b64 C, {%0, %1};\n\t"
        "fma.rn.f32x2 C, A, B, C;\n\tmov.b64 {%0, %1}, C;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__host__ __device__ constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

template <int W>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
    for (int off = W / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

template <int W>
__device__ __forceinline__ double group_sum_f64(double x) {
#pragma unroll
    for (int off = W / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// ---- online softmax over G query heads, per lane chunk -------------------
// Logits are in log2 units (queries pre-scaled by s*log2(e)).  m: running max,
// l: sum of 2^(x - m), acc: sum of 2^(x - m) v over this lane's EPC dims.
template <int G, int EPC>
struct Online {
    float m[G], l[G], acc[G][EPC];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            m[h] = -INFINITY; l[h] = 0.f;
#pragma unroll
            for (int e = 0; e < EPC; ++e) acc[h][e] = 0.f;
        }
    }
    __device__ __forceinline__ void add(int h, float x, const float* v) {
        if (x > m[h]) {                     // uniform within a lane group
            const float sc = ex2(m[h] - x);
            l[h] *= sc;
#pragma unroll
            for (int e = 0; e < EPC; ++e) acc[h][e] *= sc;
            m[h] = x;
        }
        const float p = ex2(x - m[h]);
        l[h] += p;
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc[h][e] = fmaf(p, v[e], acc[h][e]);
    }
    // merge with the state of the lane `off` lanes away (same dims, other rows)
    __device__ __forceinline__ void merge_xor(int off) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const float mo = __shfl_xor_sync(0xffffffffu, m[h], off);
            const float lo = __shfl_xor_sync(0xffffffffu, l[h], off);
            const float mn = fmaxf(m[h], mo);
            const float a = (m[h] == -INFINITY) ? 0.f : ex2(m[h] - mn);
            const float b = (mo == -INFINITY) ? 0.f : ex2(mo - mn);
            l[h] = l[h] * a + lo * b;
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                const float ao = __shfl_xor_sync(0xffffffffu, acc[h][e], off);
                acc[h][e] = acc[h][e] * a + ao * b;
            }
            m[h] = mn;
        }
    }
};

// ---- SplitMix64 (Steele, Lea & Flood 2014), counter form -------------------
constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}
// first output of a SplitMix64 generator whose state is x
__host__ __device__ __forceinline__ uint64_t sm_out(uint64_t x) { return mix64(x + kGamma); }

__host__ __device__ __forceinline__ uint64_t unit_key(uint64_t seed, uint64_t b, uint64_t g, uint64_t step) {
    uint64_t k = sm_out(seed);
    k = sm_out(k ^ b);
    k = sm_out(k ^ g);
    return sm_out(k ^ step);
}
__host__ __device__ __forceinline__ uint32_t draw_rank(uint64_t key, uint32_t i, uint32_t n) {
    const uint64_t x = sm_out(key + (uint64_t)i * kGamma);
    return (uint32_t)(((x >> 32) * (uint64_t)n) >> 32);
}

// ---- "last CTA of the unit" completion counter ------------------------------
// Every CTA of a unit publishes its partial result, then takes a ticket; the
// CTA that takes the last ticket combines all partials and resets the counter
// to zero for the next call.  No CTA ever waits on another.
__device__ __forceinline__ bool last_cta_of_unit(unsigned* counter, unsigned nsplit) {
    __shared__ unsigned s_ticket;
    __threadfence();                      // publish this thread's partial writes
    __syncthreads();
    if (threadIdx.x == 0) s_ticket = atomicAdd(counter, 1u);
    __syncthreads();
    const bool last = (s_ticket == nsplit - 1);
    if (last) __threadfence();            // order the reads of other CTAs' partials
    return last;
}
__device__ __forceinline__ void reset_counter(unsigned* counter) {
    if (threadIdx.x == 0) *counter = 0u;
}

// L2-coherent loads for data written by other CTAs of the same launch
__device__ __forceinline__ float ldcg(const float* p) { return __ldcg(p); }
__device__ __forceinline__ double ldcg(const double* p) { return __ldcg(p); }

}  // namespace sa
