// Sparse decode with the residual folded into the same pass, and the dense
// flash-decode reference.
//
// k_decode<MODE>: grid (nsd, B*Hkv).  The unit's token list is
//   [sink 0..s_eff) [chosen blocks, ascending] [window L-w_eff..L) [draws]
// split evenly over the CTAs of the unit.  Each lane group gathers one token
// row at a time (16-byte loads), computes the G logits of the group's query
// heads, and keeps an fp32 online softmax (OpenAttention page: exact tokens and
// the tail handled in one online softmax).  Mode extras in the same pass:
//   RESA  : a second online softmax of the prior logits s mu_Q . K_j over I
//           (the prior terms the RESA delta merge removes at I);
//   PROXY : the sums of K and V over I (tail sums = totals minus these);
//   SAMPLE: draws enter the softmax with logit + ln(n_T / b) (vAttention
//           eq. 3 reweighting).
// The CTA that finishes the unit last combines the splits in split order and
// applies the residual (RESA Online Aggregator; proxy token) -> out[b, h, :].
//
// k_dense: grid (nsdn, B*Hkv), the same engine over all L tokens.
#include "sa_common.cuh"
#include "sa_cta.cuh"
#include "sa_internal.h"
#include "sa_tc.cuh"

#include <type_traits>

namespace sa {

// Position and log2-weight of token t of a unit's list, ordered
//   [sink 0..s_eff) [window L-w_eff..L) [chosen blocks, ascending] [draws]
// so that the rows that do not depend on the step's selection come first.
struct TokenMap {
    int s_eff, w_eff, kk, n_i, win0;   // win0 = L - w_eff
    const int32_t* blk;                // chosen blocks of the unit (ascending)
    const int32_t* samp;               // draws of the unit
    float lw_samp;                     // log2(n_T / b)
    __device__ __forceinline__ int pos(int t, float& lw) const {
        lw = 0.f;
        if (t < s_eff) return t;
        if (t < s_eff + w_eff) return win0 + (t - s_eff);
        if (t < n_i) {
            const int j = t - s_eff - w_eff;
            return 16 * __ldcg(blk + (j >> 4)) + (j & 15);
        }
        lw = lw_samp;
        return __ldcg(samp + (t - n_i));
    }
};

// Last CTA of a unit: combine the split records in split order and fold in
// the mode's residual (RESA Online Aggregator, proxy token), then write
// out[b, h, :] for the G heads of the unit.  Record layout per split:
// exact m[G], l[G], acc[G][D]; prior m0, l0, acc0 (same shape); ksum[D], vsum[D].
// Shared scratch: s_acc, s_acc0 [G*D], s_ml [4G], s_t [2D], s_hs [G].
template <typename T, int D, int G, int MODE, bool SH = false>
__device__ void decode_epilogue(const float* recs, int nsd, int rec, const T* qg, const sa_stats& st, int u,
                                int b, int g, int Hq, int nt, float scale, float lambda, float* out,
                                float* s_acc, float* s_acc0, float* s_ml, float* s_t, float* s_hs) {
    constexpr bool PRIOR = (MODE == SA_RESA);
    constexpr bool SUMS = (MODE == SA_PROXY);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    combine_heads<G, D, SH>(recs, nsd, rec, 0, s_ml, s_ml + G);
    if constexpr (PRIOR) combine_heads<G, D, SH>(recs, nsd, rec, G * (2 + D), s_ml + 2 * G, s_ml + 3 * G);
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int h = idx / D, e = idx - h * D;
        s_acc[idx] = combine_acc<G, D, SH>(recs, nsd, rec, 0, h, e, s_ml[h]);
        if constexpr (PRIOR)
            s_acc0[idx] = combine_acc<G, D, SH>(recs, nsd, rec, G * (2 + D), h, e, s_ml[2 * G + h]);
    }
    if constexpr (SUMS) {
        if (nt > 0) {
            for (int c = threadIdx.x; c < D; c += blockDim.x) {
                float sk = 0.f, sv = 0.f;
                for (int sp = 0; sp < nsd; ++sp) {
                    sk += ld_rec<SH>(recs + (size_t)sp * rec + 2 * G * (2 + D) + c);
                    sv += ld_rec<SH>(recs + (size_t)sp * rec + 2 * G * (2 + D) + D + c);
                }
                s_t[c] = (st.sum_k[(size_t)u * D + c] - sk) / (float)nt;       // tail-mean key
                s_t[D + c] = (st.sum_v[(size_t)u * D + c] - sv) / (float)nt;   // tail-mean value
            }
        }
    }
    __syncthreads();
    // per-head scalar, one warp per head: RESA bias c_h = s (q_h - mu_Q,h) . mu_K,
    // PROXY logit z_h = s q_h . kbar_T + ln n_T   (both in log2 units)
    if ((PRIOR || SUMS) && nt > 0) {
        for (int h = warp; h < G; h += nwarps) {
            const size_t qh = (size_t)b * Hq + g * G + h;
            float x = 0.f;
#pragma unroll
            for (int e = lane; e < D; e += 32) {
                const float qe = to_f32<T>(qg[(size_t)h * D + e]);
                if constexpr (PRIOR) x = fmaf(qe - st.mu_q[qh * D + e], st.mu_k[(size_t)u * D + e], x);
                else x = fmaf(qe, s_t[e], x);
            }
            x = group_sum<32>(x);
            if (lane == 0) s_hs[h] = PRIOR ? x * scale * kLog2e : x * scale * kLog2e + log2f((float)nt);
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int h = idx / D, e = idx - h * D;
        const size_t qh = (size_t)b * Hq + g * G + h;
        const float M = s_ml[h], Ls = s_ml[G + h], A = s_acc[idx];
        float o;
        if (nt == 0 || MODE == SA_DROP || MODE == SA_SAMPLE) {
            o = Ls > 0.f ? A / Ls : 0.f;          // an empty set carries no mass
        } else if constexpr (PRIOR) {
            // RESA Online Aggregator with all masses relative to one max:
            //   Z (log2) = log2 A_h + c_h; prior mass at I = l0 2^(m0 + c);
            //   tail D_T = Z (1 - l0 2^(m0 - log2 A)) clamped at 0,
            //   tail N_T = Z (O_Est - acc0 2^(m0 - log2 A))
            const float lz = st.log_z0[qh] * kLog2e;
            const float zl = lz + s_hs[h];
            const float M0 = s_ml[2 * G + h], L0 = s_ml[3 * G + h];
            const float rI = (M0 == -INFINITY) ? 0.f : ex2(M0 - lz);
            const float Mx = fmaxf(M, zl);
            const float wI = (M == -INFINITY) ? 0.f : ex2(M - Mx);
            const float wT = lambda * ex2(zl - Mx);
            const float num = A * wI + wT * (st.o_est[qh * D + e] - s_acc0[idx] * rI);
            const float den = Ls * wI + wT * fmaxf(0.f, 1.f - L0 * rI);
            o = den > 0.f ? num / den : 0.f;
        } else {
            const float z = s_hs[h];
            const float Mx = fmaxf(M, z);
            const float wI = (M == -INFINITY) ? 0.f : ex2(M - Mx);
            const float wP = ex2(z - Mx);
            o = (A * wI + wP * s_t[D + e]) / (Ls * wI + wP);
        }
        out[qh * D + e] = o;
    }
}

template <typename T, int D, int G, int MODE>
__global__ void __launch_bounds__(kThreads)
k_decode(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, sa_stats st,
         const int32_t* __restrict__ blk_idx, int kb_stride, const int32_t* __restrict__ samp_idx,
         const int32_t* __restrict__ samp_count, int sample_cap, int Hq, int Hkv, int L, SetGeom sg,
         int tok, int nsd, int rec, float qscale, float scale, float lambda,
         float* __restrict__ part, unsigned* __restrict__ cnt, float* __restrict__ out) {
    constexpr bool PRIOR = (MODE == SA_RESA);
    constexpr bool SUMS = (MODE == SA_PROXY);
    constexpr bool SAMP = (MODE == SA_SAMPLE);
    using Gm = Geom<T, D>;
    constexpr int EPC = Gm::EPC, CPR = Gm::CPR, GPW = Gm::GPW, NG = Gm::NG;
    constexpr int kSmW = (G * (D + 2) > 2 * D) ? G * (D + 2) : 2 * D;   // per warp
    __shared__ float sm[kWarps * kSmW];
    __shared__ float s_acc[G * D];
    __shared__ float s_acc0[PRIOR ? G * D : 1];
    __shared__ float s_ml[4 * G];
    __shared__ float s_t[2 * D];
    __shared__ float s_hs[G];

    const int u = blockIdx.y, split = blockIdx.x;
    const int b = u / Hkv, g = u - b * Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int li = lane % CPR, gsub = lane / CPR;
    const size_t ubase = (size_t)u * L * D;
    const T* K = k + ubase + li * EPC;
    const T* V = v + ubase + li * EPC;
    const T* qg = q + ((size_t)b * Hq + (size_t)g * G) * D;

    const int nt = sg.n_t;
    const int bu = (SAMP && nt > 0) ? min(__ldg(samp_count + u), sample_cap) : 0;
    TokenMap tm;
    tm.s_eff = sg.s_eff; tm.w_eff = sg.w_eff; tm.kk = sg.kk; tm.n_i = sg.n_i; tm.win0 = L - sg.w_eff;
    tm.blk = blk_idx + (size_t)u * kb_stride;
    tm.samp = samp_idx + (size_t)u * (sample_cap > 0 ? sample_cap : 0);
    tm.lw_samp = bu > 0 ? log2f((float)nt / (float)bu) : 0.f;
    const int n_tok = sg.n_i + bu;

    float qv[G][EPC];
    float q0[PRIOR ? G : 1][EPC];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float f[EPC];
        unpack<T>(ld_nc16(qg + (size_t)h * D + li * EPC), f);
#pragma unroll
        for (int e = 0; e < EPC; ++e) qv[h][e] = f[e] * qscale;
        if constexpr (PRIOR) {
#pragma unroll
            for (int e = 0; e < EPC; ++e)
                q0[h][e] = st.mu_q[((size_t)b * Hq + g * G + h) * D + li * EPC + e] * qscale;
        }
    }
    Online<G, EPC> os;
    os.init();
    Online<PRIOR ? G : 1, EPC> os0;
    os0.init();
    float ks[EPC], vs[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) { ks[e] = 0.f; vs[e] = 0.f; }

    const int t0 = split * tok, t1 = min(n_tok, t0 + tok);
    // warp-uniform: a warp step covers 2 x GPW tokens (2 per lane group)
    for (int wt = t0 + warp * 2 * GPW; wt < t1; wt += 2 * NG) {
        uint4 wk[2], wv[2];
        float lw[2];
        bool ok[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int t = wt + j * GPW + gsub;
            ok[j] = t < t1;
            lw[j] = 0.f;
            const int p = ok[j] ? tm.pos(t, lw[j]) : 0;
            ok[j] = ok[j] && (unsigned)p < (unsigned)L;   // a position outside the cache is skipped
            if (ok[j]) {
                const size_t off = (size_t)p * D;
                wk[j] = ld_nc16(K + off);
                wv[j] = ld_nc16(V + off);
            } else {
                wk[j] = make_uint4(0, 0, 0, 0);
                wv[j] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int t = wt + j * GPW + gsub;
            float kf[EPC], vf[EPC];
            unpack<T>(wk[j], kf);
            unpack<T>(wv[j], vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float x = 0.f;
#pragma unroll
                for (int e = 0; e < EPC; ++e) x = fmaf(qv[h][e], kf[e], x);
                x = group_sum<CPR>(x) + lw[j];
                if (ok[j]) os.add(h, x, vf);
            }
            if constexpr (PRIOR) {
                const bool exact = ok[j] && t < sg.n_i;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float x = 0.f;
#pragma unroll
                    for (int e = 0; e < EPC; ++e) x = fmaf(q0[h][e], kf[e], x);
                    x = group_sum<CPR>(x);
                    if (exact) os0.add(h, x, vf);
                }
            }
            if constexpr (SUMS) {
                if (ok[j] && t < sg.n_i) {
#pragma unroll
                    for (int e = 0; e < EPC; ++e) { ks[e] += kf[e]; vs[e] += vf[e]; }
                }
            }
        }
    }

    // ---- publish this split ------------------------------------------------------
    float* r = part + ((size_t)u * nsd + split) * rec;
    warp_merge<G, EPC, CPR>(os);
    cta_merge_store<G, EPC, CPR, D>(os, sm, r);
    if constexpr (PRIOR) {
        warp_merge<G, EPC, CPR>(os0);
        cta_merge_store<G, EPC, CPR, D>(os0, sm, r + G * (2 + D));
    }
    if constexpr (SUMS) {
#pragma unroll
        for (int off = CPR; off < 32; off <<= 1)
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                ks[e] += __shfl_xor_sync(0xffffffffu, ks[e], off);
                vs[e] += __shfl_xor_sync(0xffffffffu, vs[e], off);
            }
        if (lane < CPR) {
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                sm[warp * 2 * D + li * EPC + e] = ks[e];
                sm[warp * 2 * D + D + li * EPC + e] = vs[e];
            }
        }
        __syncthreads();
        for (int c = threadIdx.x; c < 2 * D; c += kThreads) {
            float s = 0.f;
            for (int w = 0; w < kWarps; ++w) s += sm[w * 2 * D + c];
            r[2 * G * (2 + D) + c] = s;
        }
    }

    if (!last_cta_of_unit(cnt + u, nsd)) return;
    decode_epilogue<T, D, G, MODE>(part + (size_t)u * nsd * rec, nsd, rec, qg, st, u, b, g, Hq, sg.n_t, scale,
                                   lambda, out, s_acc, s_acc0, s_ml, s_t, s_hs);
    reset_counter(cnt + u);
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads)
k_dense(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, int Hq, int Hkv,
        int L, int tok, int nsdn, int rec, float qscale, float* __restrict__ part,
        unsigned* __restrict__ cnt, float* __restrict__ out) {
    using Gm = Geom<T, D>;
    constexpr int EPC = Gm::EPC, CPR = Gm::CPR, GPW = Gm::GPW, NG = Gm::NG;
    __shared__ float sm[kWarps * G * (D + 2)];
    const int u = blockIdx.y, split = blockIdx.x;
    const int b = u / Hkv, g = u - b * Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int li = lane % CPR, gsub = lane / CPR;
    const size_t ubase = (size_t)u * L * D;
    const T* K = k + ubase + li * EPC;
    const T* V = v + ubase + li * EPC;
    const T* qg = q + ((size_t)b * Hq + (size_t)g * G) * D;
    float qv[G][EPC];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float f[EPC];
        unpack<T>(ld_nc16(qg + (size_t)h * D + li * EPC), f);
#pragma unroll
        for (int e = 0; e < EPC; ++e) qv[h][e] = f[e] * qscale;
    }
    Online<G, EPC> os;
    os.init();
    const int t0 = split * tok, t1 = min(L, t0 + tok);
    for (int wt = t0 + warp * 4 * GPW; wt < t1; wt += 4 * NG) {
        uint4 wk[4], wv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = wt + j * GPW + gsub;
            const bool ok = t < t1;
            wk[j] = ok ? ld_stream16(K + (size_t)t * D) : make_uint4(0, 0, 0, 0);
            wv[j] = ok ? ld_stream16(V + (size_t)t * D) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const bool ok = wt + j * GPW + gsub < t1;
            float kf[EPC], vf[EPC];
            unpack<T>(wk[j], kf);
            unpack<T>(wv[j], vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float x = 0.f;
#pragma unroll
                for (int e = 0; e < EPC; ++e) x = fmaf(qv[h][e], kf[e], x);
                x = group_sum<CPR>(x);
                if (ok) os.add(h, x, vf);
            }
        }
    }
    float* r = part + ((size_t)u * nsdn + split) * rec;
    warp_merge<G, EPC, CPR>(os);
    cta_merge_store<G, EPC, CPR, D>(os, sm, r);
    if (!last_cta_of_unit(cnt + u, nsdn)) return;
    const float* recs = part + (size_t)u * nsdn * rec;
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
        const int h = idx / D, e = idx - h * D;
        float M, Ls;
        const float A = combine_splits<G, D>(recs, nsdn, rec, h, e, M, Ls);
        out[((size_t)b * Hq + g * G + h) * D + e] = A / Ls;
    }
    reset_counter(cnt + u);
}


// ============================================================================
// bf16 caches: one stream kernel for the sparse gather and the dense pass
// ============================================================================
// A CTA owns a chunk of consecutive 64-token tiles of one unit and streams
// them through a 3-stage cp.async ring of padded shared tiles; its 4 warps
// take 16 rows each per tile (tensor-core engine, sa_tc.cuh).  A unit that
// fits one chunk (the usual case at batch 32: one CTA per unit, one wave)
// finishes in the same CTA; otherwise the chunks' records are combined by
// the unit's last CTA.

constexpr int kTcTile = 64;        // tokens per shared-memory tile
constexpr int kTcWarps = 4;        // 16 tokens per warp per tile
constexpr int kTcThreads = 32 * kTcWarps;
constexpr int kStages = 3;
constexpr int kDenseMode = 4;      // MODE value of the dense pass

template <int D>
struct StageLayout {
    static constexpr int kTileBytes = kTcTile * tc::Pitch<D>::kBytes;   // one of K or V
    static constexpr int kBytes = 2 * kTileBytes + kTcTile * 4;         // K, V, row positions
};

// The unit's chosen blocks and draws are cached in shared memory (after the
// ring) when they fit; longer lists are read from global memory.
constexpr int kBlkCache = 1024;
constexpr int kSampCache = 256;

template <int D, int G, int MODE>
constexpr size_t stream_smem() {
    constexpr bool PRIOR = (MODE == SA_RESA);
    constexpr size_t ring = (size_t)kStages * StageLayout<D>::kBytes + (kBlkCache + kSampCache) * 4;
    constexpr size_t merge = (size_t)(kTcWarps * G * 4 + (PRIOR ? 2 : 1) * kTcWarps * G * D) * 4;
    constexpr size_t tail = (size_t)(2 * G * (2 + D) + 2 * D) * 4        // own record
                            + (size_t)(2 * G * D + 4 * G + 2 * D + G) * 4;  // epilogue scratch
    constexpr size_t m = merge + tail;
    return ring > m ? ring : m;
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p));
}

template <int D, int G, int MODE>
__global__ void __launch_bounds__(kTcThreads)
k_stream_tc(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
            const __nv_bfloat16* __restrict__ v, sa_stats st, const int32_t* __restrict__ blk_idx, int kb_stride,
            const int32_t* __restrict__ samp_idx, const int32_t* __restrict__ samp_count, int sample_cap, int Hq,
            int Hkv, int L, SetGeom sg, int tpc, int nchunk, int rec, float qscale, float scale, float lambda,
            float* __restrict__ part, unsigned* __restrict__ cnt, float* __restrict__ out) {
    constexpr bool DENSE = (MODE == kDenseMode);
    constexpr bool PRIOR = (MODE == SA_RESA);
    constexpr bool SUMS = (MODE == SA_PROXY);
    constexpr bool SAMP = (MODE == SA_SAMPLE);
    constexpr int P = tc::Pitch<D>::kBytes;
    constexpr int TB = StageLayout<D>::kTileBytes;
    constexpr int SB = StageLayout<D>::kBytes;
    extern __shared__ __align__(16) unsigned char smem[];
    int* s_blk = reinterpret_cast<int*>(smem + (size_t)kStages * SB);
    int* s_samp = s_blk + kBlkCache;

    const int u = blockIdx.y, chunk = blockIdx.x;
    const int b = u / Hkv, g = u - b * Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const size_t ubase = (size_t)u * L * D;
    const __nv_bfloat16* K = k + ubase;
    const __nv_bfloat16* V = v + ubase;
    const __nv_bfloat16* qg = q + ((size_t)b * Hq + (size_t)g * G) * D;
    const size_t qh0 = (size_t)b * Hq + (size_t)g * G;

    // the epilogue's inputs (query, prefill statistics) into L2 while streaming
    if constexpr (!DENSE) {
        const int t = threadIdx.x;
        if (t * 64 < G * D * 2) prefetch_l2(reinterpret_cast<const char*>(qg) + t * 64);
        if constexpr (PRIOR) {
            if (t * 128 < G * D * 4) {
                prefetch_l2(reinterpret_cast<const char*>(st.mu_q + qh0 * D) + t * 128);
                prefetch_l2(reinterpret_cast<const char*>(st.o_est + qh0 * D) + t * 128);
            }
            if (t * 128 < D * 4) prefetch_l2(reinterpret_cast<const char*>(st.mu_k + (size_t)u * D) + t * 128);
            if (t == 0) prefetch_l2(st.log_z0 + qh0);
        }
        if constexpr (SUMS) {
            if (t * 128 < D * 4) {
                prefetch_l2(reinterpret_cast<const char*>(st.sum_k + (size_t)u * D) + t * 128);
                prefetch_l2(reinterpret_cast<const char*>(st.sum_v + (size_t)u * D) + t * 128);
            }
        }
    }

    const int nt = DENSE ? 0 : sg.n_t;
    const int n_i = DENSE ? L : sg.n_i;
    const int win0 = L - sg.w_eff;
    const int32_t* gblk = blk_idx + (size_t)u * kb_stride;
    const int32_t* gsamp = samp_idx + (size_t)u * (sample_cap > 0 ? sample_cap : 0);
    // rows [0, n_indep) do not depend on the selection; the tile range uses an
    // upper bound on the list length (draw capacity); the exact count and the
    // lists are read once the selection is visible
    const int n_indep = DENSE ? L : sg.s_eff + sg.w_eff;
    const int n_hi = DENSE ? L : sg.n_i + ((SAMP && nt > 0) ? sample_cap : 0);
    int n_tok = n_hi;
    float lw_samp = 0.f;
    const bool blk_sm = sg.kk <= kBlkCache;
    bool samp_sm = true;
    bool sel_ready = DENSE || n_indep >= n_hi;
    // Under programmatic dependent launch the preceding selection kernel may
    // still be running: wait for it before the first selection-dependent read
    // (a no-op when the kernel was launched normally).  Called at the same
    // point by every thread.
    auto wait_selection = [&]() {
        if (!sel_ready) {
            asm volatile("griddepcontrol.wait;\n" ::: "memory");
            int bu = 0;
            if (SAMP && nt > 0) {
                bu = min(__ldcg(samp_count + u), sample_cap);
                lw_samp = bu > 0 ? log2f((float)nt / (float)bu) : 0.f;
                n_tok = sg.n_i + bu;
            }
            samp_sm = bu <= kSampCache;
            if (blk_sm)
                for (int x = threadIdx.x; x < sg.kk; x += kTcThreads) s_blk[x] = __ldcg(gblk + x);
            if (samp_sm)
                for (int x = threadIdx.x; x < bu; x += kTcThreads) s_samp[x] = __ldcg(gsamp + x);
            __syncthreads();
            sel_ready = true;
        }
    };
    // token t of the unit's list -> cache row, or -1 (masked)
    //   [sink 0..s_eff) [window L-w_eff..L) [chosen blocks] [draws]
    auto pos_of = [&](int t) -> int {
        int p;
        if (DENSE) p = t < L ? t : -1;
        else if (t >= n_tok) p = -1;
        else if (t < sg.s_eff) p = t;
        else if (t < n_indep) p = win0 + (t - sg.s_eff);
        else if (t < n_i) {
            const int j = t - n_indep;
            p = 16 * (blk_sm ? s_blk[j >> 4] : __ldcg(gblk + (j >> 4))) + (j & 15);
        } else {
            const int j = t - n_i;
            p = samp_sm ? s_samp[j] : __ldcg(gsamp + j);
        }
        return (unsigned)p < (unsigned)L ? p : -1;         // outside the cache: masked
    };
    const int ntiles = (n_hi + kTcTile - 1) / kTcTile;
    const int tile0 = chunk * tpc, tile1 = min(ntiles, tile0 + tpc);

    // K/V rows of tile i into its stage (cp.async; masked rows zero-filled).
    // The tile's row positions go to the stage first (one barrier), so the
    // copy loop reads one shared word per 16-byte chunk.
    auto issue = [&](int i) {
        if (i < tile1) {
            if ((i + 1) * kTcTile > n_indep) wait_selection();
            unsigned char* sb = smem + (size_t)(i % kStages) * SB;
            int* pos = reinterpret_cast<int*>(sb + 2 * TB);
            if (threadIdx.x < kTcTile) pos[threadIdx.x] = pos_of(i * kTcTile + threadIdx.x);
            __syncthreads();
            constexpr int CPR = D / 8;
            const uint32_t sk = tc::smem_u32(sb), sv = sk + TB;
#pragma unroll 4
            for (int idx = threadIdx.x; idx < kTcTile * CPR; idx += kTcThreads) {
                const int row = idx / CPR, ch = idx - row * CPR;
                const int p = pos[row];
                const uint32_t o = row * P + ch * 16;
                if (p >= 0) {
                    tc::cp16(sk + o, K + (size_t)p * D + ch * 8);
                    tc::cp16(sv + o, V + (size_t)p * D + ch * 8);
                } else {
                    tc::st_zero16(sk + o);
                    tc::st_zero16(sv + o);
                }
            }
        }
        tc::cp_commit();
    };

    // first tiles in flight before the query / prior fragments are loaded
#pragma unroll
    for (int i = 0; i < kStages - 1; ++i) issue(tile0 + i);
    tc::WarpAttn<D, G, PRIOR> wa;
    {
        const int gh = min(lane >> 2, G - 1);
        wa.init(qg + (size_t)gh * D, PRIOR ? st.mu_q + (qh0 + gh) * D : nullptr);
    }
    float ks[2] = {0.f, 0.f};      // SUMS: this thread's column pair of K (c < D/2) or V (c >= D/2)
    for (int i = tile0; i < tile1; ++i) {
        issue(i + kStages - 1);
        tc::cp_wait<kStages - 1>();
        __syncthreads();
        unsigned char* sb = smem + (size_t)(i % kStages) * SB;
        const int base = i * kTcTile;
        if constexpr (SUMS) {
            // column pair (2c, 2c+1) of K (c < D/2) or of V (c >= D/2) over the
            // exact rows of the tile, which form the prefix [0, nr)
            const int c = threadIdx.x;
            const int nr = max(0, min(kTcTile, n_i - base));
            if (c < D) {
                const unsigned char* src = sb + (c < D / 2 ? 0 : TB) + (c % (D / 2)) * 4;
#pragma unroll 8
                for (int r = 0; r < nr; ++r) {
                    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src + r * P));
                    ks[0] += f.x;
                    ks[1] += f.y;
                }
            }
        }
        const int r0 = warp * 16;
        if (base + r0 < n_tok) {
            const int tq = lane & 3;
            const int rows[4] = {r0 + 2 * tq, r0 + 2 * tq + 1, r0 + 8 + 2 * tq, r0 + 9 + 2 * tq};
            float xadd[4];
            bool in_i[4];
            const int* pos = reinterpret_cast<const int*>(sb + 2 * TB);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int t = base + rows[j];
                const bool ok = pos[rows[j]] >= 0;
                xadd[j] = !ok ? -INFINITY : (t >= n_i ? lw_samp : 0.f);
                in_i[j] = PRIOR && ok && t < n_i;
            }
            const uint32_t sk = tc::smem_u32(sb);
            wa.step16(sk, sk + TB, r0, xadd, in_i, qscale);
        }
        __syncthreads();              // this stage is refilled by a later issue()
    }
    tc::cp_wait<0>();
    __syncthreads();

    // ---- this chunk's record --------------------------------------------------------
    float* fb = reinterpret_cast<float*>(smem);
    float* ml = fb;                                     // [W][G][4]
    float* acc = ml + kTcWarps * G * 4;                 // [W][G][D]
    float* acc0 = acc + kTcWarps * G * D;               // [W][G][D] (PRIOR)
    float* own = acc + (PRIOR ? 2 : 1) * kTcWarps * G * D;   // own record when the unit is one chunk
    float* scratch = own + 2 * G * (2 + D) + 2 * D;
    wa.store(ml, acc, acc0);
    __syncthreads();
    const bool single = (nchunk == 1);
    float* r = single ? own : part + ((size_t)u * nchunk + chunk) * rec;
    tc::merge_warps<D, G, PRIOR>(ml, acc, acc0, kTcWarps, r);
    if constexpr (SUMS) {
        if (threadIdx.x < D) {
            const int c = threadIdx.x;
            const int col = 2 * (c % (D / 2)) + (c < D / 2 ? 0 : D);
            r[2 * G * (2 + D) + col] = ks[0];
            r[2 * G * (2 + D) + col + 1] = ks[1];
        }
    }
    if (single) {
        __syncthreads();
    } else if (!last_cta_of_unit(cnt + u, nchunk)) {
        return;
    }

    // ---- the unit's output --------------------------------------------------------------
    float* s_acc = scratch;
    float* s_acc0 = s_acc + G * D;
    float* s_ml = s_acc0 + G * D;
    float* s_t = s_ml + 4 * G;
    float* s_hs = s_t + 2 * D;
    const float* recs = single ? own : part + (size_t)u * nchunk * rec;
    if constexpr (DENSE) {
        if (single) combine_heads<G, D, true>(recs, 1, rec, 0, s_ml, s_ml + G);
        else combine_heads<G, D, false>(recs, nchunk, rec, 0, s_ml, s_ml + G);
        __syncthreads();
        for (int idx = threadIdx.x; idx < G * D; idx += kTcThreads) {
            const int h = idx / D, e = idx - h * D;
            const float A = single ? combine_acc<G, D, true>(recs, 1, rec, 0, h, e, s_ml[h])
                                   : combine_acc<G, D, false>(recs, nchunk, rec, 0, h, e, s_ml[h]);
            out[((size_t)b * Hq + g * G + h) * D + e] = A / s_ml[G + h];
        }
    } else {
        constexpr int EM = DENSE ? SA_DROP : MODE;
        if (single)
            decode_epilogue<__nv_bfloat16, D, G, EM, true>(recs, 1, rec, qg, st, u, b, g, Hq, nt, scale, lambda,
                                                           out, s_acc, s_acc0, s_ml, s_t, s_hs);
        else
            decode_epilogue<__nv_bfloat16, D, G, EM, false>(recs, nchunk, rec, qg, st, u, b, g, Hq, nt, scale,
                                                            lambda, out, s_acc, s_acc0, s_ml, s_t, s_hs);
    }
    if (!single) reset_counter(cnt + u);
}

// ---- dispatch ----------------------------------------------------------------

template <int D, int G, int MODE>
static cudaError_t stream_launch(const Dims& d, dim3 grid, const void* q, const void* k, const void* v,
                                 const sa_stats& st, const sa_selection& sel, const sa_select_params& sp,
                                 const SetGeom& sg, int tpc, int nchunk, int rec, float scale, float lambda,
                                 char* part, char* cnt, float* out, bool pdl, cudaStream_t s) {
    constexpr size_t sm = stream_smem<D, G, MODE>();
    static std::atomic<unsigned long long> opted{0};
    cudaError_t e = opt_in_smem(k_stream_tc<D, G, MODE>, sm, opted);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = sm;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_stream_tc<D, G, MODE>, reinterpret_cast<const __nv_bfloat16*>(q),
                              reinterpret_cast<const __nv_bfloat16*>(k), reinterpret_cast<const __nv_bfloat16*>(v),
                              st, (const int32_t*)sel.blk_idx, (int)sp.k_blocks, (const int32_t*)sel.samp_idx,
                              (const int32_t*)sel.samp_count, (int)sp.sample_cap, d.Hq, d.Hkv, d.L, sg, tpc, nchunk,
                              rec, scale * kLog2e, scale, lambda, reinterpret_cast<float*>(part),
                              reinterpret_cast<unsigned*>(cnt), out);
}

template <typename T, int D, int G, int MODE>
static cudaError_t decode_m(const Dims& d, const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        return stream_launch<D, G, MODE>(d, dim3(p.nsd, d.U()), a.q, a.k, a.v, a.st, a.sel, a.sp, p.g, p.tok_d,
                                         p.nsd, p.rec, a.scale, a.dp.lambda, a.ws + p.off_part, a.ws + p.off_cnt,
                                         a.out, a.pdl, s);
    } else {
        k_decode<T, D, G, MODE><<<dim3(p.nsd, d.U()), kThreads, 0, s>>>(
            reinterpret_cast<const T*>(a.q), reinterpret_cast<const T*>(a.k), reinterpret_cast<const T*>(a.v),
            a.st, a.sel.blk_idx, a.sp.k_blocks, a.sel.samp_idx, a.sel.samp_count, a.sp.sample_cap,
            d.Hq, d.Hkv, d.L, p.g, p.tok_d, p.nsd, p.rec, a.scale * kLog2e, a.scale, a.dp.lambda,
            reinterpret_cast<float*>(a.ws + p.off_part), reinterpret_cast<unsigned*>(a.ws + p.off_cnt), a.out);
        return cudaGetLastError();
    }
}

template <typename T, int D, int G>
static cudaError_t decode_t(const Dims& d, const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
    switch (a.dp.mode) {
        case SA_DROP: return decode_m<T, D, G, SA_DROP>(d, p, a, s);
        case SA_RESA: return decode_m<T, D, G, SA_RESA>(d, p, a, s);
        case SA_PROXY: return decode_m<T, D, G, SA_PROXY>(d, p, a, s);
        case SA_SAMPLE: return decode_m<T, D, G, SA_SAMPLE>(d, p, a, s);
    }
    return cudaErrorInvalidValue;
}

template <typename T, int D>
static cudaError_t decode_g(const Dims& d, const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
    switch (d.G) {
        case 1: return decode_t<T, D, 1>(d, p, a, s);
        case 2: return decode_t<T, D, 2>(d, p, a, s);
        case 4: return decode_t<T, D, 4>(d, p, a, s);
        case 8: return decode_t<T, D, 8>(d, p, a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const Dims& d, const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
    if (d.bf16) return d.d == 128 ? decode_g<__nv_bfloat16, 128>(d, p, a, s) : decode_g<__nv_bfloat16, 64>(d, p, a, s);
    return d.d == 128 ? decode_g<float, 128>(d, p, a, s) : decode_g<float, 64>(d, p, a, s);
}

template <typename T, int D, int G>
static cudaError_t dense_t(const Dims& d, const DensePlan& p, const DenseArgs& a, cudaStream_t s) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        SetGeom sg{};
        sa_stats st{};
        sa_selection sel{};
        sa_select_params sp{};
        return stream_launch<D, G, kDenseMode>(d, dim3(p.nsdn, d.U()), a.q, a.k, a.v, st, sel, sp, sg,
                                               p.tok / kTcTile, p.nsdn, p.rec, a.scale, 1.f, a.ws + p.off_part,
                                               a.ws + p.off_cnt, a.out, false, s);
    } else {
        k_dense<T, D, G><<<dim3(p.nsdn, d.U()), kThreads, 0, s>>>(
            reinterpret_cast<const T*>(a.q), reinterpret_cast<const T*>(a.k), reinterpret_cast<const T*>(a.v),
            d.Hq, d.Hkv, d.L, p.tok, p.nsdn, p.rec, a.scale * kLog2e,
            reinterpret_cast<float*>(a.ws + p.off_part), reinterpret_cast<unsigned*>(a.ws + p.off_cnt), a.out);
        return cudaGetLastError();
    }
}

template <typename T, int D>
static cudaError_t dense_g(const Dims& d, const DensePlan& p, const DenseArgs& a, cudaStream_t s) {
    switch (d.G) {
        case 1: return dense_t<T, D, 1>(d, p, a, s);
        case 2: return dense_t<T, D, 2>(d, p, a, s);
        case 4: return dense_t<T, D, 4>(d, p, a, s);
        case 8: return dense_t<T, D, 8>(d, p, a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_dense(const Dims& d, const DensePlan& p, const DenseArgs& a, cudaStream_t s) {
    if (d.bf16) return d.d == 128 ? dense_g<__nv_bfloat16, 128>(d, p, a, s) : dense_g<__nv_bfloat16, 64>(d, p, a, s);
    return d.d == 128 ? dense_g<float, 128>(d, p, a, s) : dense_g<float, 64>(d, p, a, s);
}

}  // namespace sa
