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

// Position and log2-weight of token t of a unit's list.
struct TokenMap {
    int s_eff, kk, n_i, win0;      // win0 = L - w_eff
    const int32_t* blk;            // chosen blocks of the unit (ascending)
    const int32_t* samp;           // draws of the unit
    float lw_samp;                 // log2(n_T / b)
    __device__ __forceinline__ int pos(int t, float& lw) const {
        lw = 0.f;
        if (t < s_eff) return t;
        const int tb = t - s_eff;
        if (tb < 16 * kk) return 16 * __ldg(blk + (tb >> 4)) + (tb & 15);
        if (t < n_i) return win0 + (tb - 16 * kk);
        lw = lw_samp;
        return __ldg(samp + (t - n_i));
    }
};

// Last CTA of a unit: combine the split records in split order and fold in
// the mode's residual (RESA Online Aggregator, proxy token), then write
// out[b, h, :] for the G heads of the unit.  Record layout per split:
// exact m[G], l[G], acc[G][D]; prior m0, l0, acc0 (same shape); ksum[D], vsum[D].
// Shared scratch: s_acc, s_acc0 [G*D], s_ml [4G], s_t [2D], s_hs [G].
template <typename T, int D, int G, int MODE>
__device__ void decode_epilogue(const float* recs, int nsd, int rec, const T* qg, const sa_stats& st, int u,
                                int b, int g, int Hq, int nt, float scale, float lambda, float* out,
                                float* s_acc, float* s_acc0, float* s_ml, float* s_t, float* s_hs) {
    constexpr bool PRIOR = (MODE == SA_RESA);
    constexpr bool SUMS = (MODE == SA_PROXY);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    combine_heads<G, D>(recs, nsd, rec, 0, s_ml, s_ml + G);
    if constexpr (PRIOR) combine_heads<G, D>(recs, nsd, rec, G * (2 + D), s_ml + 2 * G, s_ml + 3 * G);
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int h = idx / D, e = idx - h * D;
        s_acc[idx] = combine_acc<G, D>(recs, nsd, rec, 0, h, e, s_ml[h]);
        if constexpr (PRIOR) s_acc0[idx] = combine_acc<G, D>(recs, nsd, rec, G * (2 + D), h, e, s_ml[2 * G + h]);
    }
    if constexpr (SUMS) {
        if (nt > 0) {
            for (int c = threadIdx.x; c < D; c += blockDim.x) {
                float sk = 0.f, sv = 0.f;
                for (int sp = 0; sp < nsd; ++sp) {
                    sk += ldcg(recs + (size_t)sp * rec + 2 * G * (2 + D) + c);
                    sv += ldcg(recs + (size_t)sp * rec + 2 * G * (2 + D) + D + c);
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
    tm.s_eff = sg.s_eff; tm.kk = sg.kk; tm.n_i = sg.n_i; tm.win0 = L - sg.w_eff;
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
// bf16 caches: tensor-core tiles (see sa_tc.cuh)
// ============================================================================

constexpr int kTcTile = 64;        // tokens per shared-memory tile
constexpr int kTcWarps = 4;        // 16 tokens per warp
constexpr int kTcThreads = 32 * kTcWarps;

// Copies rows pos[0..kTcTile) of K and V (16-byte cp.async; pos < 0 zero-fills)
// into padded shared tiles.
template <int D>
__device__ __forceinline__ void tc_fetch_tile(const __nv_bfloat16* K, const __nv_bfloat16* V, const int* pos,
                                              uint32_t sk, uint32_t sv) {
    constexpr int CPR = D / 8;
    constexpr int P = tc::Pitch<D>::kBytes;
#pragma unroll 4
    for (int idx = threadIdx.x; idx < 2 * kTcTile * CPR; idx += kTcThreads) {
        const int kv = idx / (kTcTile * CPR);
        const int rem = idx - kv * kTcTile * CPR;
        const int row = rem / CPR, ch = rem - row * CPR;
        const uint32_t dst = (kv ? sv : sk) + row * P + ch * 16;
        const int p = pos[row];
        if (p >= 0) tc::cp16(dst, (kv ? V : K) + (size_t)p * D + ch * 8);
        else tc::st_zero16(dst);
    }
}

template <int D, int G, int MODE>
__global__ void __launch_bounds__(kTcThreads)
k_decode_tc(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
            const __nv_bfloat16* __restrict__ v, sa_stats st, const int32_t* __restrict__ blk_idx, int kb_stride,
            const int32_t* __restrict__ samp_idx, const int32_t* __restrict__ samp_count, int sample_cap, int Hq,
            int Hkv, int L, SetGeom sg, int nsd, int rec, float qscale, float scale, float lambda,
            float* __restrict__ part, unsigned* __restrict__ cnt, float* __restrict__ out) {
    constexpr bool PRIOR = (MODE == SA_RESA);
    constexpr bool SUMS = (MODE == SA_PROXY);
    constexpr bool SAMP = (MODE == SA_SAMPLE);
    constexpr int PE = tc::Pitch<D>::kElems;
    extern __shared__ __align__(16) unsigned char smem[];
    __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem);
    __nv_bfloat16* sV = sK + kTcTile * PE;
    int* s_pos = reinterpret_cast<int*>(sV + kTcTile * PE);
    float* s_lw = reinterpret_cast<float*>(s_pos + kTcTile);
    float* s_sum = s_lw + kTcTile;                       // [2D] proxy sums of this tile
    float* fbuf = reinterpret_cast<float*>(smem);         // reused after the tiles are consumed

    const int u = blockIdx.y, split = blockIdx.x;
    const int b = u / Hkv, g = u - b * Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const size_t ubase = (size_t)u * L * D;
    const __nv_bfloat16* qg = q + ((size_t)b * Hq + (size_t)g * G) * D;

    const int nt = sg.n_t;
    const int bu = (SAMP && nt > 0) ? min(__ldg(samp_count + u), sample_cap) : 0;
    TokenMap tm;
    tm.s_eff = sg.s_eff; tm.kk = sg.kk; tm.n_i = sg.n_i; tm.win0 = L - sg.w_eff;
    tm.blk = blk_idx + (size_t)u * kb_stride;
    tm.samp = samp_idx + (size_t)u * (sample_cap > 0 ? sample_cap : 0);
    tm.lw_samp = bu > 0 ? log2f((float)nt / (float)bu) : 0.f;
    const int n_tok = sg.n_i + bu;
    const int t0 = split * kTcTile, t1 = min(n_tok, t0 + kTcTile);

    if (threadIdx.x < kTcTile) {
        const int t = t0 + threadIdx.x;
        float lw = 0.f;
        int p = (t < t1) ? tm.pos(t, lw) : -1;
        if ((unsigned)p >= (unsigned)L) p = -1;          // outside the cache: masked
        s_pos[threadIdx.x] = p;
        s_lw[threadIdx.x] = p >= 0 ? lw : -INFINITY;
    }
    __syncthreads();
    tc_fetch_tile<D>(k + ubase, v + ubase, s_pos, tc::smem_u32(sK), tc::smem_u32(sV));
    tc::cp_commit();

    tc::WarpAttn<D, G, PRIOR> wa;
    {
        const int gh = min((lane >> 2), G - 1);
        wa.init(qg + (size_t)gh * D, PRIOR ? st.mu_q + ((size_t)b * Hq + g * G + gh) * D : nullptr);
    }
    tc::cp_wait<0>();
    __syncthreads();

    if constexpr (SUMS) {            // sums of K and V over the exact rows of this tile
        for (int c = threadIdx.x; c < 2 * D; c += kTcThreads) {
            const __nv_bfloat16* src = (c < D ? sK : sV) + (c < D ? c : c - D);
            float acc = 0.f;
            for (int r = 0; r < kTcTile; ++r)
                if (t0 + r < sg.n_i && s_pos[r] >= 0) acc += __bfloat162float(src[r * PE]);
            s_sum[c] = acc;
        }
    }
    const int r0 = warp * 16;
    if (t0 + r0 < t1) {
        const int tq = lane & 3;
        const int rows[4] = {r0 + 2 * tq, r0 + 2 * tq + 1, r0 + 8 + 2 * tq, r0 + 9 + 2 * tq};
        float xadd[4];
        bool in_i[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            xadd[j] = s_lw[rows[j]];
            in_i[j] = (t0 + rows[j] < sg.n_i) && s_pos[rows[j]] >= 0;
        }
        wa.step16(tc::smem_u32(sK), tc::smem_u32(sV), r0, xadd, in_i, qscale);
    }
    float sum_keep[2];
    if constexpr (SUMS) {
        sum_keep[0] = threadIdx.x < 2 * D ? s_sum[threadIdx.x] : 0.f;
        sum_keep[1] = threadIdx.x + kTcThreads < 2 * D ? s_sum[threadIdx.x + kTcThreads] : 0.f;
    }
    __syncthreads();                   // tiles consumed: reuse the region
    float* ml = fbuf;                                   // [W][G][4]
    float* acc = ml + kTcWarps * G * 4;                 // [W][G][D]
    float* acc0 = acc + kTcWarps * G * D;               // [W][G][D]
    wa.store(ml, acc, acc0);
    __syncthreads();
    float* r = part + ((size_t)u * nsd + split) * rec;
    tc::merge_warps<D, G, PRIOR>(ml, acc, acc0, kTcWarps, r);
    if constexpr (SUMS) {
        if (threadIdx.x < 2 * D) r[2 * G * (2 + D) + threadIdx.x] = sum_keep[0];
        if (threadIdx.x + kTcThreads < 2 * D) r[2 * G * (2 + D) + threadIdx.x + kTcThreads] = sum_keep[1];
    }
    if (!last_cta_of_unit(cnt + u, nsd)) return;
    float* s_acc = fbuf;
    float* s_acc0 = s_acc + G * D;
    float* s_ml = s_acc0 + G * D;
    float* s_t = s_ml + 4 * G;
    float* s_hs = s_t + 2 * D;
    decode_epilogue<__nv_bfloat16, D, G, MODE>(part + (size_t)u * nsd * rec, nsd, rec, qg, st, u, b, g, Hq, nt,
                                               scale, lambda, out, s_acc, s_acc0, s_ml, s_t, s_hs);
    reset_counter(cnt + u);
}

constexpr int kDenseStages = 3;

template <int D, int G>
__global__ void __launch_bounds__(kTcThreads)
k_dense_tc(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
           const __nv_bfloat16* __restrict__ v, int Hq, int Hkv, int L, int tok, int nsdn, int rec, float qscale,
           float* __restrict__ part, unsigned* __restrict__ cnt, float* __restrict__ out) {
    constexpr int PE = tc::Pitch<D>::kElems;
    constexpr int STAGE = 2 * kTcTile * PE;             // bf16 elements per stage (K and V)
    extern __shared__ __align__(16) unsigned char smem[];
    __nv_bfloat16* tiles = reinterpret_cast<__nv_bfloat16*>(smem);
    int* s_pos = reinterpret_cast<int*>(tiles + kDenseStages * STAGE);   // [stages][tile]
    float* fbuf = reinterpret_cast<float*>(smem);

    const int u = blockIdx.y, split = blockIdx.x;
    const int b = u / Hkv, g = u - b * Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const size_t ubase = (size_t)u * L * D;
    const __nv_bfloat16* qg = q + ((size_t)b * Hq + (size_t)g * G) * D;
    const int t0 = split * tok, t1 = min(L, t0 + tok);
    const int ntiles = (t1 - t0 + kTcTile - 1) / kTcTile;

    auto issue = [&](int i) {
        if (i < ntiles) {
            const int st = i % kDenseStages;
            int* pos = s_pos + st * kTcTile;
            // positions of the tile (the previous tile on this stage is consumed)
            if (threadIdx.x < kTcTile) {
                const int t = t0 + i * kTcTile + threadIdx.x;
                pos[threadIdx.x] = t < t1 ? t : -1;
            }
            __syncthreads();
            const uint32_t base = tc::smem_u32(tiles + st * STAGE);
            tc_fetch_tile<D>(k + ubase, v + ubase, pos, base, base + kTcTile * tc::Pitch<D>::kBytes);
        }
        tc::cp_commit();
    };

    tc::WarpAttn<D, G, false> wa;
    wa.init(qg + (size_t)min(lane >> 2, G - 1) * D, nullptr);
#pragma unroll
    for (int i = 0; i < kDenseStages - 1; ++i) issue(i);
    for (int i = 0; i < ntiles; ++i) {
        issue(i + kDenseStages - 1);
        tc::cp_wait<kDenseStages - 1>();
        __syncthreads();
        const int st = i % kDenseStages;
        const int r0 = warp * 16;
        const int rem = t1 - (t0 + i * kTcTile);
        if (r0 < rem) {
            const int tq = lane & 3;
            const int rows[4] = {r0 + 2 * tq, r0 + 2 * tq + 1, r0 + 8 + 2 * tq, r0 + 9 + 2 * tq};
            float xadd[4];
            bool in_i[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) { xadd[j] = rows[j] < rem ? 0.f : -INFINITY; in_i[j] = false; }
            const uint32_t base = tc::smem_u32(tiles + st * STAGE);
            wa.step16(base, base + kTcTile * tc::Pitch<D>::kBytes, r0, xadd, in_i, qscale);
        }
        __syncthreads();              // stage st is refilled by the next issue()
    }
    tc::cp_wait<0>();
    __syncthreads();
    float* ml = fbuf;
    float* acc = ml + kTcWarps * G * 4;
    wa.store(ml, acc, nullptr);
    __syncthreads();
    float* r = part + ((size_t)u * nsdn + split) * rec;
    tc::merge_warps<D, G, false>(ml, acc, nullptr, kTcWarps, r);
    if (!last_cta_of_unit(cnt + u, nsdn)) return;
    const float* recs = part + (size_t)u * nsdn * rec;
    float* s_M = fbuf;
    float* s_L = fbuf + G;
    __syncthreads();
    combine_heads<G, D>(recs, nsdn, rec, 0, s_M, s_L);
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += kTcThreads) {
        const int h = idx / D, e = idx - h * D;
        out[((size_t)b * Hq + g * G + h) * D + e] = combine_acc<G, D>(recs, nsdn, rec, 0, h, e, s_M[h]) / s_L[h];
    }
    reset_counter(cnt + u);
}

template <int D, int G>
size_t decode_tc_smem() {
    constexpr int PE = tc::Pitch<D>::kElems;
    size_t tiles = 2 * kTcTile * PE * sizeof(__nv_bfloat16) + kTcTile * 8 + 2 * D * 4;
    size_t merge = (kTcWarps * G * 4 + 2 * kTcWarps * G * D) * sizeof(float);
    size_t epi = (2 * G * D + 4 * G + 2 * D + G) * sizeof(float);
    size_t m = merge > epi ? merge : epi;
    return tiles > m ? tiles : m;
}

template <int D, int G>
size_t dense_tc_smem() {
    constexpr int PE = tc::Pitch<D>::kElems;
    size_t tiles = kDenseStages * (2 * kTcTile * PE * sizeof(__nv_bfloat16) + kTcTile * 4);
    size_t merge = (kTcWarps * G * 4 + kTcWarps * G * D) * sizeof(float);
    return tiles > merge ? tiles : merge;
}

// ---- dispatch ----------------------------------------------------------------

template <typename T, int D, int G, int MODE>
static cudaError_t decode_m(const Dims& d, const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        const size_t sm = decode_tc_smem<D, G>();
        if (sm > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(k_decode_tc<D, G, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
            if (e != cudaSuccess) return e;
        }
        k_decode_tc<D, G, MODE><<<dim3(p.nsd, d.U()), kTcThreads, sm, s>>>(
            reinterpret_cast<const T*>(a.q), reinterpret_cast<const T*>(a.k), reinterpret_cast<const T*>(a.v),
            a.st, a.sel.blk_idx, a.sp.k_blocks, a.sel.samp_idx, a.sel.samp_count, a.sp.sample_cap,
            d.Hq, d.Hkv, d.L, p.g, p.nsd, p.rec, a.scale * kLog2e, a.scale, a.dp.lambda,
            reinterpret_cast<float*>(a.ws + p.off_part), reinterpret_cast<unsigned*>(a.ws + p.off_cnt), a.out);
    } else {
        k_decode<T, D, G, MODE><<<dim3(p.nsd, d.U()), kThreads, 0, s>>>(
            reinterpret_cast<const T*>(a.q), reinterpret_cast<const T*>(a.k), reinterpret_cast<const T*>(a.v),
            a.st, a.sel.blk_idx, a.sp.k_blocks, a.sel.samp_idx, a.sel.samp_count, a.sp.sample_cap,
            d.Hq, d.Hkv, d.L, p.g, p.tok_d, p.nsd, p.rec, a.scale * kLog2e, a.scale, a.dp.lambda,
            reinterpret_cast<float*>(a.ws + p.off_part), reinterpret_cast<unsigned*>(a.ws + p.off_cnt), a.out);
    }
    return cudaGetLastError();
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
        const size_t sm = dense_tc_smem<D, G>();
        cudaError_t e = cudaFuncSetAttribute(k_dense_tc<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        k_dense_tc<D, G><<<dim3(p.nsdn, d.U()), kTcThreads, sm, s>>>(
            reinterpret_cast<const T*>(a.q), reinterpret_cast<const T*>(a.k), reinterpret_cast<const T*>(a.v),
            d.Hq, d.Hkv, d.L, p.tok, p.nsdn, p.rec, a.scale * kLog2e,
            reinterpret_cast<float*>(a.ws + p.off_part), reinterpret_cast<unsigned*>(a.ws + p.off_cnt), a.out);
    } else {
        k_dense<T, D, G><<<dim3(p.nsdn, d.U()), kThreads, 0, s>>>(
            reinterpret_cast<const T*>(a.q), reinterpret_cast<const T*>(a.k), reinterpret_cast<const T*>(a.v),
            d.Hq, d.Hkv, d.L, p.tok, p.nsdn, p.rec, a.scale * kLog2e,
            reinterpret_cast<float*>(a.ws + p.off_part), reinterpret_cast<unsigned*>(a.ws + p.off_cnt), a.out);
    }
    return cudaGetLastError();
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
