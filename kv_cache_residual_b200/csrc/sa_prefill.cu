// Prefill-end statistics (RESA, Method, key design 1 "Prior Estimator"):
// the typical query mu_Q (mean of the context queries), then ONE streaming
// pass over K and V per unit that computes, for the G query heads of the
// group, the prior attention of mu_Q over all L tokens (O_Est and the
// normaliser, "one extra query appended at prefill end"), the key / value
// totals (OpenAttention stage 04 tail sums) and the 16-token block means
// (summed in fp64, rounded once to the cache dtype).
//
//   k_qmean : grid (nsq, B*Hq)   partial column sums of Q_ctx, last CTA -> mu_q
//   bf16 caches: the tensor-core stream kernel in its prefill mode
//             (k_stream_tc, sa_decode_core.cuh): mu_Q (split into bf16 hi +
//             lo) as the prior columns of the same MMAs as the decode, over
//             every token, with the block means, key / value totals and the
//             largest |block mean| formed from the shared-memory tiles
//   fp32 caches:
//   k_kvpass: grid (nskv, B*Hkv) online softmax of s*mu_q.K_j over a token range
//                                + sums + block means; last CTA -> o_est, log_z0,
//                                mu_k, sum_k, sum_v, kbar_absmax
#include "sa_common.cuh"
#include "sa_cta.cuh"
#include "sa_internal.h"
#include "sa_sketch.cuh"

#include <type_traits>

namespace sa {

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
k_qmean(const T* __restrict__ q_ctx, int L, int rows, int nsq, float* __restrict__ part,
        unsigned* __restrict__ cnt, float* __restrict__ mu_q) {
    using Gm = Geom<T, D>;
    constexpr int EPC = Gm::EPC, CPR = Gm::CPR, NG = Gm::NG;
    __shared__ float red[NG * D];
    const int bh = blockIdx.y, split = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gi = warp * Gm::GPW + lane / CPR, li = lane % CPR;
    const T* base = q_ctx + (size_t)bh * L * D + li * EPC;
    const int r0 = split * rows, r1 = min(L, r0 + rows);
    float acc[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) acc[e] = 0.f;
    int r = r0 + gi;
    for (; r + 3 * NG < r1; r += 4 * NG) {           // 4 rows in flight per lane
        uint4 w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) w[j] = ld_stream16(base + (size_t)(r + j * NG) * D);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float f[EPC];
            unpack<T>(w[j], f);
#pragma unroll
            for (int e = 0; e < EPC; ++e) acc[e] += f[e];
        }
    }
    for (; r < r1; r += NG) {
        float f[EPC];
        unpack<T>(ld_stream16(base + (size_t)r * D), f);
#pragma unroll
        for (int e = 0; e < EPC; ++e) acc[e] += f[e];
    }
#pragma unroll
    for (int e = 0; e < EPC; ++e) red[gi * D + li * EPC + e] = acc[e];
    __syncthreads();
    for (int c = threadIdx.x; c < D; c += kThreads) {
        float s = 0.f;
        for (int g = 0; g < NG; ++g) s += red[g * D + c];
        part[((size_t)bh * nsq + split) * D + c] = s;
    }
    if (!last_cta_of_unit(cnt + bh, nsq)) return;
    for (int c = threadIdx.x; c < D; c += kThreads) {
        float s = 0.f;
        for (int sp = 0; sp < nsq; ++sp) s += ldcg(part + ((size_t)bh * nsq + sp) * D + c);
        mu_q[(size_t)bh * D + c] = s / (float)L;
    }
    reset_counter(cnt + bh);
}

// two CTAs per SM (registers capped at 128): one CTA of 8 warps per SM left
// the pass latency-bound at ~0.2 of the HBM peak
template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, 2)
k_kvpass(const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ mu_q,
         int Hq, int Hkv, int L, int ld, int tok, int nskv, float qscale, int stride,
         float* __restrict__ part, unsigned* __restrict__ cnt, sa_stats st) {
    using Gm = Geom<T, D>;
    constexpr int EPC = Gm::EPC, CPR = Gm::CPR, NG = Gm::NG;
    __shared__ float sm[kWarps * G * (D + 2)];
    __shared__ double smd[kWarps * D];
    __shared__ float smv[kWarps * D];
    __shared__ float sma[kWarps];
    const int u = blockIdx.y, split = blockIdx.x;
    const int b = u / Hkv, g = u - b * Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gi = warp * Gm::GPW + lane / CPR, li = lane % CPR;
    const int nb = L / 16;
    const size_t ubase = (size_t)u * ld * D;
    const T* K = k + ubase + li * EPC;
    const T* V = v + ubase + li * EPC;
    T* BM = reinterpret_cast<T*>(st.blk_mean) + (size_t)u * (ld / 16) * D + li * EPC;

    float q0[G][EPC];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < EPC; ++e)
            q0[h][e] = mu_q[((size_t)b * Hq + g * G + h) * D + li * EPC + e] * qscale;

    Online<G, EPC> os;
    os.init();
    double ks[EPC];
    float vs[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) { ks[e] = 0.0; vs[e] = 0.f; }
    float amax = 0.f;

    // warp-uniform loop: each warp step covers GPW consecutive blocks, one per
    // lane group; groups past the end compute on zeros and skip the updates
    const int blk0 = split * (tok / 16), blk1 = min(nb, blk0 + tok / 16);
    const int gsub = lane / CPR;
    for (int wb = blk0 + warp * Gm::GPW; wb < blk1; wb += NG) {
        const int blk = wb + gsub;
        const bool valid = blk < blk1;
        double bs[EPC];
#pragma unroll
        for (int e = 0; e < EPC; ++e) bs[e] = 0.0;
#pragma unroll 1
        for (int j0 = 0; j0 < 16; j0 += 4) {
            uint4 wk[4], wv[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const size_t off = (size_t)(blk * 16 + j0 + j) * D;
                wk[j] = valid ? ld_stream16(K + off) : make_uint4(0, 0, 0, 0);
                wv[j] = valid ? ld_stream16(V + off) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float kf[EPC], vf[EPC];
                unpack<T>(wk[j], kf);
                unpack<T>(wv[j], vf);
#pragma unroll
                for (int e = 0; e < EPC; ++e) { bs[e] += (double)kf[e]; vs[e] += vf[e]; }
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float x = 0.f;
#pragma unroll
                    for (int e = 0; e < EPC; ++e) x = fmaf(q0[h][e], kf[e], x);
                    x = group_sum<CPR>(x);           // all lanes of the warp take part
                    if (valid) os.add(h, x, vf);
                }
            }
        }
        if (valid) {
            // block mean: fp64 sum of 16 rows, times 1/16 (exact), one rounding
            T mean[EPC];
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                ks[e] += bs[e];
                mean[e] = round_from_f64<T>(bs[e] * 0.0625);
                amax = fmaxf(amax, fabsf(to_f32<T>(mean[e])));
            }
            *reinterpret_cast<uint4*>(BM + (size_t)blk * D) = pack16(mean);
        }
    }

    // merge: groups of a warp, then warps (fixed order)
    warp_merge<G, EPC, CPR>(os);
#pragma unroll
    for (int off = CPR; off < 32; off <<= 1) {
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
            ks[e] += __shfl_xor_sync(0xffffffffu, ks[e], off);
            vs[e] += __shfl_xor_sync(0xffffffffu, vs[e], off);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    if (lane < CPR) {
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
            smd[warp * D + li * EPC + e] = ks[e];
            smv[warp * D + li * EPC + e] = vs[e];
        }
        if (lane == 0) sma[warp] = amax;
    }
    float* rec = part + ((size_t)u * nskv + split) * stride;
    cta_merge_store<G, EPC, CPR, D>(os, sm, rec);       // syncs inside
    constexpr int F = (2 * G + G * D + D + 1 + 1) & ~1;
    double* recd = reinterpret_cast<double*>(rec + F);
    for (int c = threadIdx.x; c < D; c += kThreads) {
        double s = 0.0;
        float sv = 0.f;
        for (int w = 0; w < kWarps; ++w) { s += smd[w * D + c]; sv += smv[w * D + c]; }
        recd[c] = s;
        rec[2 * G + G * D + c] = sv;
    }
    if (threadIdx.x == 0) {
        float a = 0.f;
        for (int w = 0; w < kWarps; ++w) a = fmaxf(a, sma[w]);
        rec[2 * G + G * D + D] = a;
    }

    if (!last_cta_of_unit(cnt + u, nskv)) return;
    const float* recs = part + (size_t)u * nskv * stride;
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
        const int h = idx / D, e = idx - h * D;
        float M, Ls;
        const float A = combine_splits<G, D>(recs, nskv, stride, h, e, M, Ls);
        const size_t qh = (size_t)b * Hq + g * G + h;
        st.o_est[qh * D + e] = A / Ls;
        if (e == 0) st.log_z0[qh] = (M + log2f(Ls)) * kLn2;
    }
    for (int c = threadIdx.x; c < D; c += kThreads) {
        double s = 0.0;
        float sv = 0.f;
        for (int sp = 0; sp < nskv; ++sp) {
            const float* r = recs + (size_t)sp * stride;
            s += ldcg(reinterpret_cast<const double*>(r + F) + c);
            sv += ldcg(r + 2 * G + G * D + c);
        }
        st.sum_k[(size_t)u * D + c] = (float)s;
        st.mu_k[(size_t)u * D + c] = (float)(s / (double)L);
        st.sum_v[(size_t)u * D + c] = sv;
    }
    if (threadIdx.x == 0) {
        float a = 0.f;
        for (int sp = 0; sp < nskv; ++sp) a = fmaxf(a, ldcg(recs + (size_t)sp * stride + 2 * G + G * D + D));
        st.kbar_absmax[u] = a;
    }
    reset_counter(cnt + u);
}

// Block means of blocks [blk_begin, blk_end) of every unit; raises kbar_absmax.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
k_blockmeans(const T* __restrict__ k, int ld, int blk_begin, int blk_end, T* __restrict__ blk_mean,
             float* __restrict__ kbar_absmax) {
    using Gm = Geom<T, D>;
    constexpr int EPC = Gm::EPC, CPR = Gm::CPR, NG = Gm::NG;
    const int u = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gi = warp * Gm::GPW + lane / CPR, li = lane % CPR;
    const int nb = ld / 16;
    const T* K = k + (size_t)u * ld * D + li * EPC;
    float amax = 0.f;
    for (int blk = blk_begin + blockIdx.x * NG + gi; blk < blk_end; blk += gridDim.x * NG) {
        double bs[EPC];
#pragma unroll
        for (int e = 0; e < EPC; ++e) bs[e] = 0.0;
        for (int j = 0; j < 16; ++j) {
            float kf[EPC];
            unpack<T>(ld_nc16(K + (size_t)(blk * 16 + j) * D), kf);
#pragma unroll
            for (int e = 0; e < EPC; ++e) bs[e] += (double)kf[e];
        }
        T mean[EPC];
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
            mean[e] = round_from_f64<T>(bs[e] * 0.0625);
            amax = fmaxf(amax, fabsf(to_f32<T>(mean[e])));
        }
        *reinterpret_cast<uint4*>(blk_mean + ((size_t)u * nb + blk) * D + li * EPC) = pack16(mean);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
    // non-negative floats order like their bit patterns as signed ints
    if (lane == 0 && amax > 0.f) atomicMax(reinterpret_cast<int*>(kbar_absmax + u), __float_as_int(amax));
}

// Scan sketch of block rows [blk_begin, blk_end) of every unit, one warp per
// row (sketch_row in sa_sketch.cuh), relative to the unit's centre m (its
// typical key mu_k).
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
k_sketch(const T* __restrict__ bm, const float* __restrict__ centre, int nb, int blk_begin, int blk_end,
         int8_t* __restrict__ code, float4* __restrict__ meta) {
    constexpr int E = D / 32;                 // elements per lane
    const int u = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    double m[E];
#pragma unroll
    for (int e = 0; e < E; ++e) m[e] = (double)centre[(size_t)u * D + lane * E + e];
    for (int blk = blk_begin + blockIdx.x * kWarps + warp; blk < blk_end; blk += gridDim.x * kWarps) {
        const size_t row = (size_t)u * nb + blk;
        const T* src = bm + row * D + lane * E;
        float kbar[E];
#pragma unroll
        for (int e = 0; e < E; ++e) kbar[e] = to_f32<T>(src[e]);
        sketch_row<D>(kbar, m, code + row * D, meta + row);
    }
}

template <typename T, int D>
static cudaError_t sketch_t(const Dims& d, const void* bm, const float* centre, int b0, int b1, int8_t* code,
                            float* meta, cudaStream_t s) {
    const int nblk = b1 - b0;
    const int gx = max(1, min(cdiv(nblk, kWarps), cdiv(4 * kSmTarget, d.U())));
    k_sketch<T, D><<<dim3(gx, d.U()), kThreads, 0, s>>>(reinterpret_cast<const T*>(bm), centre, d.nbl(), b0, b1,
                                                        code, reinterpret_cast<float4*>(meta));
    return cudaGetLastError();
}

cudaError_t launch_block_sketch(const Dims& d, const void* bm, const float* centre, int b0, int b1, int8_t* code,
                                float* meta, cudaStream_t s) {
    if (d.bf16) return d.d == 128 ? sketch_t<__nv_bfloat16, 128>(d, bm, centre, b0, b1, code, meta, s)
                                  : sketch_t<__nv_bfloat16, 64>(d, bm, centre, b0, b1, code, meta, s);
    return d.d == 128 ? sketch_t<float, 128>(d, bm, centre, b0, b1, code, meta, s)
                      : sketch_t<float, 64>(d, bm, centre, b0, b1, code, meta, s);
}

// Elementwise key minimum and maximum of blocks [blk_begin, blk_end) of every
// unit (Quest's per-block key bounds, the summaries of SA_SCORE_QUEST): one
// thread per (block, 16-byte chunk of the row), its 16 rows read with 16-byte
// loads.  Values of the cache, so nothing is rounded.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
k_block_minmax(const T* __restrict__ k, int ld, int blk_begin, int blk_end, T* __restrict__ bmin,
               T* __restrict__ bmax) {
    using Gm = Geom<T, D>;
    constexpr int EPC = Gm::EPC, CPR = Gm::CPR;
    const int u = blockIdx.y, nb = ld / 16;
    const int items = (blk_end - blk_begin) * CPR;
    for (int it = blockIdx.x * kThreads + threadIdx.x; it < items; it += gridDim.x * kThreads) {
        const int blk = blk_begin + it / CPR, ch = it - (it / CPR) * CPR;
        const T* src = k + ((size_t)u * ld + (size_t)blk * 16) * D + ch * EPC;
        float mn[EPC], mx[EPC], f[EPC];
        unpack<T>(ld_nc16(src), mn);
#pragma unroll
        for (int e = 0; e < EPC; ++e) mx[e] = mn[e];
#pragma unroll 4
        for (int j = 1; j < 16; ++j) {
            unpack<T>(ld_nc16(src + (size_t)j * D), f);
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                mn[e] = fminf(mn[e], f[e]);
                mx[e] = fmaxf(mx[e], f[e]);
            }
        }
        T omn[EPC], omx[EPC];
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
            omn[e] = round_from_f64<T>((double)mn[e]);       // exact: a value of the cache
            omx[e] = round_from_f64<T>((double)mx[e]);
        }
        const size_t o = ((size_t)u * nb + blk) * D + ch * EPC;
        *reinterpret_cast<uint4*>(bmin + o) = pack16(omn);
        *reinterpret_cast<uint4*>(bmax + o) = pack16(omx);
    }
}

template <typename T, int D>
static cudaError_t minmax_t(const Dims& d, const void* k, int b0, int b1, void* bmin, void* bmax, cudaStream_t s) {
    using Gm = Geom<T, D>;
    const int items = (b1 - b0) * Gm::CPR;
    const int gx = max(1, min(cdiv(items, kThreads), cdiv(4 * kSmTarget, d.U())));
    k_block_minmax<T, D><<<dim3(gx, d.U()), kThreads, 0, s>>>(reinterpret_cast<const T*>(k), d.ld, b0, b1,
                                                              reinterpret_cast<T*>(bmin), reinterpret_cast<T*>(bmax));
    return cudaGetLastError();
}

cudaError_t launch_block_minmax(const Dims& d, const void* k, int b0, int b1, void* bmin, void* bmax,
                                cudaStream_t s) {
    if (d.bf16) return d.d == 128 ? minmax_t<__nv_bfloat16, 128>(d, k, b0, b1, bmin, bmax, s)
                                  : minmax_t<__nv_bfloat16, 64>(d, k, b0, b1, bmin, bmax, s);
    return d.d == 128 ? minmax_t<float, 128>(d, k, b0, b1, bmin, bmax, s)
                      : minmax_t<float, 64>(d, k, b0, b1, bmin, bmax, s);
}

// ---- dispatch ------------------------------------------------------------

template <typename T, int D, int G>
static cudaError_t prefill_t(const Dims& d, const PrefillPlan& p, const PrefillArgs& a, cudaStream_t s) {
    char* ws = a.ws;
    k_qmean<T, D><<<dim3(p.nsq, d.B * d.Hq), kThreads, 0, s>>>(
        reinterpret_cast<const T*>(a.q_ctx), d.L, p.rows_q, p.nsq,
        reinterpret_cast<float*>(ws + p.off_qpart), reinterpret_cast<unsigned*>(ws + p.off_qcnt),
        a.st.mu_q);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        // the tensor-core stream kernel: mu_Q as the prior columns of its MMAs
        e = launch_prefill_stream(d, p, a.k, a.v, a.st, a.scale, ws + p.off_kvpart, ws + p.off_kvcnt, s);
    } else {
        k_kvpass<T, D, G><<<dim3(p.nskv, d.U()), kThreads, 0, s>>>(
            reinterpret_cast<const T*>(a.k), reinterpret_cast<const T*>(a.v), a.st.mu_q, d.Hq, d.Hkv, d.L, d.ld,
            p.tok_kv, p.nskv, a.scale * kLog2e, p.kv_stride, reinterpret_cast<float*>(ws + p.off_kvpart),
            reinterpret_cast<unsigned*>(ws + p.off_kvcnt), a.st);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    e = launch_block_sketch(d, a.st.blk_mean, a.st.mu_k, 0, d.L / 16, a.st.blk_code, a.st.blk_meta, s);
    if (e != cudaSuccess || a.st.blk_min == nullptr) return e;
    return launch_block_minmax(d, a.k, 0, d.L / 16, a.st.blk_min, a.st.blk_max, s);
}

template <typename T, int D>
static cudaError_t prefill_g(const Dims& d, const PrefillPlan& p, const PrefillArgs& a, cudaStream_t s) {
    switch (d.G) {
        case 1: return prefill_t<T, D, 1>(d, p, a, s);
        case 2: return prefill_t<T, D, 2>(d, p, a, s);
        case 4: return prefill_t<T, D, 4>(d, p, a, s);
        case 8: return prefill_t<T, D, 8>(d, p, a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_prefill(const Dims& d, const PrefillPlan& p, const PrefillArgs& a, cudaStream_t s) {
    if (d.bf16) return d.d == 128 ? prefill_g<__nv_bfloat16, 128>(d, p, a, s) : prefill_g<__nv_bfloat16, 64>(d, p, a, s);
    return d.d == 128 ? prefill_g<float, 128>(d, p, a, s) : prefill_g<float, 64>(d, p, a, s);
}

template <typename T, int D>
static cudaError_t blockmeans_t(const Dims& d, const void* k, int b0, int b1, void* bm, float* amax,
                                const float* centre, int8_t* code, float* meta, cudaStream_t s) {
    using Gm = Geom<T, D>;
    const int nblk = b1 - b0;
    const int gx = max(1, min(cdiv(nblk, Gm::NG), cdiv(kSmTarget, d.U())));
    k_blockmeans<T, D><<<dim3(gx, d.U()), kThreads, 0, s>>>(
        reinterpret_cast<const T*>(k), d.ld, b0, b1, reinterpret_cast<T*>(bm), amax);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return sketch_t<T, D>(d, bm, centre, b0, b1, code, meta, s);
}

cudaError_t launch_block_summaries(const Dims& d, const void* k, int b0, int b1, void* bm, float* amax,
                                   const float* centre, int8_t* code, float* meta, cudaStream_t s) {
    if (d.bf16) return d.d == 128 ? blockmeans_t<__nv_bfloat16, 128>(d, k, b0, b1, bm, amax, centre, code, meta, s)
                                  : blockmeans_t<__nv_bfloat16, 64>(d, k, b0, b1, bm, amax, centre, code, meta, s);
    return d.d == 128 ? blockmeans_t<float, 128>(d, k, b0, b1, bm, amax, centre, code, meta, s)
                      : blockmeans_t<float, 64>(d, k, b0, b1, bm, amax, centre, code, meta, s);
}

}  // namespace sa
