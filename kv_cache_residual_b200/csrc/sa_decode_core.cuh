// Device code of the decode kernels: the residual epilogue (RESA Online
// Aggregator, proxy token, sampled tail) and the bf16 stream pass over a
// unit's token list (tensor-core engine, sa_tc.cuh).
#pragma once

#include <type_traits>

#include "sa_common.cuh"
#include "sa_cta.cuh"
#include "sa_internal.h"
#include "sa_tc.cuh"

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
// The statistics a RESA epilogue reads, loaded ahead of it: O_Est and ln Z0
// of this thread's outputs (idx = threadIdx.x + k * blockDim.x) and the
// per-head bias c_h = s (q_h - mu_Q,h) . mu_K (log2 units) in shared memory.
template <int D, int G>
struct EpiPre {
    static constexpr int kPer = (G * D + 127) / 128;    // output elements per thread (>= 128 threads)
    float oe[kPer], lz[kPer];
};

// Loads pre (every thread): O_Est and ln Z0 of this thread's outputs.
template <int D, int G>
__device__ __forceinline__ void epi_load(EpiPre<D, G>& pre, const sa_stats& st, int b, int g, int Hq) {
#pragma unroll
    for (int k = 0; k < EpiPre<D, G>::kPer; ++k) {
        const int idx = threadIdx.x + k * blockDim.x;
        const size_t qh = (size_t)b * Hq + g * G + (idx < G * D ? idx / D : 0);
        pre.oe[k] = idx < G * D ? st.o_est[qh * D + idx % D] : 0.f;
        pre.lz[k] = idx < G * D ? st.log_z0[qh] : 0.f;
    }
}

// The operands of the per-head bias c_h of a CTA of NW warps (warp w takes
// heads w, w + NW, ...), loaded into registers by bias_load early and summed
// by bias_sum late, so that their latency hides behind other work.
template <int D, int G, int NW>
struct BiasPre {
    static constexpr int kHpw = (G + NW - 1) / NW;      // heads per warp
    static constexpr int kPl = D / 32;                  // elements per lane
    float q[kHpw][kPl], mq[kHpw][kPl], mk[kPl];
};

template <typename T, int D, int G, int NW>
__device__ __forceinline__ void bias_load(BiasPre<D, G, NW>& bp, const T* qg, const sa_stats& st, int u, int b,
                                          int g, int Hq) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int j = 0; j < BiasPre<D, G, NW>::kPl; ++j) bp.mk[j] = st.mu_k[(size_t)u * D + lane + 32 * j];
#pragma unroll
    for (int x = 0; x < BiasPre<D, G, NW>::kHpw; ++x) {
        const int h = warp + x * NW;
        const size_t qh = (size_t)b * Hq + g * G + (h < G ? h : 0);
#pragma unroll
        for (int j = 0; j < BiasPre<D, G, NW>::kPl; ++j) {
            bp.q[x][j] = h < G ? to_f32<T>(qg[(size_t)h * D + lane + 32 * j]) : 0.f;
            bp.mq[x][j] = h < G ? st.mu_q[qh * D + lane + 32 * j] : 0.f;
        }
    }
}

// hs[h] = s (q_h - mu_Q,h) . mu_K in log2 units; a barrier must follow
// before hs is read.
template <int D, int G, int NW>
__device__ __forceinline__ void bias_sum(const BiasPre<D, G, NW>& bp, float* hs, float scale) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int x = 0; x < BiasPre<D, G, NW>::kHpw; ++x) {
        const int h = warp + x * NW;
        if (h >= G) break;
        float y = 0.f;
#pragma unroll
        for (int j = 0; j < BiasPre<D, G, NW>::kPl; ++j) y = fmaf(bp.q[x][j] - bp.mq[x][j], bp.mk[j], y);
        y = group_sum<32>(y);
        if (lane == 0) hs[h] = y * scale * kLog2e;
    }
}

// Fills pre (every thread) and hs[G] (one warp per head); the caller puts a
// barrier between this and the epilogue.
template <typename T, int D, int G>
__device__ __forceinline__ void epi_preload(EpiPre<D, G>& pre, float* hs, const T* qg, const sa_stats& st, int u,
                                            int b, int g, int Hq, float scale) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    epi_load<D, G>(pre, st, b, g, Hq);
    for (int h = warp; h < G; h += nwarps) {
        const size_t qh = (size_t)b * Hq + g * G + h;
        float x = 0.f;
#pragma unroll
        for (int e = lane; e < D; e += 32)
            x = fmaf(to_f32<T>(qg[(size_t)h * D + e]) - st.mu_q[qh * D + e], st.mu_k[(size_t)u * D + e], x);
        x = group_sum<32>(x);
        if (lane == 0) hs[h] = x * scale * kLog2e;
    }
}

// One output element of head h from the unit's combined exact state over the
// read set (max M, mass Ls, accumulator A, log2 units) and the mode's
// residual.  RESA (Online Aggregator, with all masses relative to one max):
// Z (log2) = log2 A_h + c_h with log2 A_h = lz2 and c_h = hs; prior mass at
// I = L0 2^(M0 + c); tail D_T = Z (1 - L0 2^(M0 - log2 A)) clamped at 0,
// tail N_T = Z (O_Est - A0 2^(M0 - log2 A)), scaled by lambda.  PROXY: one
// token of logit z (log2) and value tv.  DROP / SAMPLE (the draws are already
// in the state), or no tail: the normalised state.
template <int MODE>
__device__ __forceinline__ float resid_value(int nt, float M, float Ls, float A, float M0, float L0, float A0,
                                             float lz2, float hs, float oe, float lambda, float z, float tv) {
    if (nt == 0 || MODE == SA_DROP || MODE == SA_SAMPLE) {
        return Ls > 0.f ? A / Ls : 0.f;           // an empty set carries no mass
    } else if constexpr (MODE == SA_RESA) {
        const float zl = lz2 + hs;
        const float rI = (M0 == -INFINITY) ? 0.f : ex2(M0 - lz2);
        const float Mx = fmaxf(M, zl);
        const float wI = (M == -INFINITY) ? 0.f : ex2(M - Mx);
        const float wT = lambda * ex2(zl - Mx);
        const float num = A * wI + wT * (oe - A0 * rI);
        const float den = Ls * wI + wT * fmaxf(0.f, 1.f - L0 * rI);
        return den > 0.f ? num / den : 0.f;
    } else {
        const float Mx = fmaxf(M, z);
        const float wI = (M == -INFINITY) ? 0.f : ex2(M - Mx);
        const float wP = ex2(z - Mx);
        return (A * wI + wP * tv) / (Ls * wI + wP);
    }
}

// pre / hs_pre: RESA statistics already loaded by epi_preload (null: loaded
// here, first, so that their latency overlaps the combination of the records)
template <typename T, int D, int G, int MODE, bool SH = false>
__device__ __forceinline__ void decode_epilogue(const float* recs, int nsd, int rec, const T* qg, const sa_stats& st,
                                                int u, int b, int g, int Hq, int nt, float scale, float lambda,
                                                float* out, float* s_acc, float* s_acc0, float* s_ml, float* s_t,
                                                float* s_hs, const EpiPre<D, G>* pre = nullptr,
                                                const float* hs_pre = nullptr) {
    constexpr bool PRIOR = (MODE == SA_RESA);
    constexpr bool SUMS = (MODE == SA_PROXY);
    constexpr int kPer = EpiPre<D, G>::kPer;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    EpiPre<D, G> loc;
    const float* hsv = s_hs;
    if constexpr (PRIOR) {
        if (nt > 0) {
            if (pre != nullptr) {
                loc = *pre;
                hsv = hs_pre;
            } else {
                epi_preload<T, D, G>(loc, s_hs, qg, st, u, b, g, Hq, scale);
            }
        }
    }
    const float* oe = loc.oe;
    const float* lz = loc.lz;
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
    // PROXY logit z_h = s q_h . kbar_T + ln n_T (log2 units), one warp per head
    if (SUMS && nt > 0) {
        for (int h = warp; h < G; h += nwarps) {
            float x = 0.f;
#pragma unroll
            for (int e = lane; e < D; e += 32) x = fmaf(to_f32<T>(qg[(size_t)h * D + e]), s_t[e], x);
            x = group_sum<32>(x);
            if (lane == 0) s_hs[h] = x * scale * kLog2e + log2f((float)nt);
        }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < kPer; ++k) {
        const int idx = threadIdx.x + k * blockDim.x;
        if (idx >= G * D) break;
        const int h = idx / D, e = idx - h * D;
        const size_t qh = (size_t)b * Hq + g * G + h;
        const float M = s_ml[h], Ls = s_ml[G + h], A = s_acc[idx];
        float o;
        if constexpr (PRIOR)
            o = resid_value<MODE>(nt, M, Ls, A, s_ml[2 * G + h], s_ml[3 * G + h], s_acc0[idx], lz[k] * kLog2e,
                                  nt > 0 ? hsv[h] : 0.f, oe[k], lambda, 0.f, 0.f);
        else if constexpr (SUMS)
            o = resid_value<MODE>(nt, M, Ls, A, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, lambda, nt > 0 ? s_hs[h] : 0.f,
                                  nt > 0 ? s_t[D + e] : 0.f);
        else
            o = resid_value<MODE>(nt, M, Ls, A, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, lambda, 0.f, 0.f);
        out[qh * D + e] = o;
    }
}

// ============================================================================
// bf16 caches: one stream kernel for the sparse gather, the dense pass and
// the prefill's KV pass
// ============================================================================
// A CTA owns a chunk of consecutive 64-token tiles of one unit and streams
// them through a cp.async ring of padded shared tiles (stream_stages: two
// stages for the decode, three for the all-token passes); its 4 warps take
// 16 rows each per tile (tensor-core engine, sa_tc.cuh).  A unit that fits
// one chunk (the usual case at batch 32 and at one sequence with small
// reads: one CTA per unit) finishes in the same CTA; otherwise the chunks'
// records are combined by the unit's last CTA.

constexpr int kTcTile = 64;        // tokens per shared-memory tile
constexpr int kTcWarps = 4;        // 16 tokens per warp per tile
constexpr int kTcThreads = 32 * kTcWarps;
// ring stages: three for the all-token passes (dense, prefill: bandwidth);
// two for the decode, whose units hold a few tiles (one tile in flight
// while the previous is computed; a shorter prologue at one sequence)
template <int MODE>
__host__ __device__ constexpr int stream_stages() { return MODE >= 4 ? 3 : 2; }
constexpr int kDenseMode = 4;      // MODE value of the dense pass
constexpr int kPrefillMode = 5;    // MODE value of the prefill pass (RESA prior, totals, block means)

// floats of a chunk record: exact (m, l, acc) and prior state per head, then
// the key and value sums (proxy); the prefill pass keeps the key totals in
// fp64 (2 d floats) and the largest |block mean| instead (its value totals
// are the exact columns' accumulator: a zero query weighs every token 1)
template <int D, int G, int MODE>
__host__ __device__ constexpr int stream_rec() {
    return MODE == kPrefillMode ? ((2 * G * (2 + D) + 2 * D + 1 + 3) & ~3) : 2 * G * (2 + D) + 2 * D;
}

template <int D>
struct StageLayout {
    static constexpr int kTileBytes = kTcTile * tc::Pitch<D>::kBytes;   // one of K or V
    static constexpr int kBytes = 2 * kTileBytes + kTcTile * 8;         // K, V, row positions, row heads
};

// The unit's chosen blocks and draws are cached in shared memory (after the
// ring) when they fit; longer lists are read from global memory.  (Sized so
// that a decode CTA fits on an SM beside two selection CTAs.)
constexpr int kBlkCache = 256;
constexpr int kSampCache = 256;

template <int D, int G, int MODE>
__host__ __device__ constexpr size_t stream_area_smem() {     // stages, then the merge / epilogue scratch over them
    constexpr bool PRIOR = (MODE == SA_RESA || MODE == kPrefillMode);
    constexpr size_t ring = (size_t)stream_stages<MODE>() * StageLayout<D>::kBytes;
    constexpr size_t merge = (size_t)(kTcWarps * G * 4 + (PRIOR ? 2 : 1) * kTcWarps * G * D) * 4;
    constexpr size_t tail = (size_t)stream_rec<D, G, MODE>() * 4       // own record
                            + (size_t)(2 * G * D + 4 * G + 2 * D + G) * 4;  // epilogue scratch
    constexpr size_t m = merge + tail;
    return ring > m ? ring : m;
}

template <int D, int G, int MODE>
__host__ __device__ constexpr size_t stream_smem() {          // the stream kernel: area + the two list caches after the stages
    // after the stages: the list caches, or the prefill pass's key-sum scratch
    constexpr size_t caches = (size_t)(kBlkCache + kSampCache) * 4;
    constexpr size_t pf = MODE == kPrefillMode ? (size_t)4 * D * 8 + 64 : 0;
    constexpr size_t lists = (size_t)stream_stages<MODE>() * StageLayout<D>::kBytes + (caches > pf ? caches : pf);
    constexpr size_t a = stream_area_smem<D, G, MODE>();
    return a > lists ? a : lists;
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p));
}

// Inputs and outputs of the bf16 stream pass (layouts of sa_decode /
// sa_dense_decode in sa_decode.h).
struct StreamIo {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    sa_stats st;
    const int32_t* blk_idx;
    int kb_stride;
    const int32_t* samp_idx;
    const int32_t* samp_count;
    int sample_cap;
    int Hq, Hkv, L;
    int ld;                      // tokens per unit in the cache allocation
    SetGeom sg;
    int tpc, nchunk, rec;        // tiles per chunk, chunks per unit, floats per chunk record
    float qscale, scale, lambda;
    float* part;
    unsigned* cnt;
    float* out;
    int per_head;                // draws per query head (rows b Hq + g G + h of samp_idx / samp_count)
};

// Chunk `chunk` of unit u.  smem: the dynamic area (stream_smem<> bytes);
// s_blk / s_samp: shared caches of the chosen blocks / draws (kBlkCache /
// kSampCache entries); the lists are read from global memory once the
// selection kernel (a programmatic dependency, or an earlier launch) is done.
template <int D, int G, int MODE>
__device__ __forceinline__ void stream_unit(const StreamIo& io, unsigned char* smem, int* s_blk, int* s_samp, int u,
                                            int chunk) {
    const __nv_bfloat16* __restrict__ q = io.q;
    const __nv_bfloat16* __restrict__ k = io.k;
    const __nv_bfloat16* __restrict__ v = io.v;
    const sa_stats& st = io.st;
    const int32_t* __restrict__ blk_idx = io.blk_idx;
    const int kb_stride = io.kb_stride;
    const int32_t* __restrict__ samp_idx = io.samp_idx;
    const int32_t* __restrict__ samp_count = io.samp_count;
    const int sample_cap = io.sample_cap, Hq = io.Hq, Hkv = io.Hkv, L = io.L;
    const SetGeom& sg = io.sg;
    const int tpc = io.tpc, nchunk = io.nchunk, rec = io.rec;
    const float qscale = io.qscale, scale = io.scale, lambda = io.lambda;
    float* __restrict__ part = io.part;
    unsigned* __restrict__ cnt = io.cnt;
    float* __restrict__ out = io.out;
    constexpr bool PREFILL = (MODE == kPrefillMode);   // the typical query over every token
    constexpr bool DENSE = (MODE == kDenseMode);
    constexpr bool ALL = DENSE || PREFILL;               // every token of the unit, no selection
    constexpr bool PRIOR = (MODE == SA_RESA) || PREFILL;
    constexpr bool SUMS = (MODE == SA_PROXY);
    constexpr bool SAMP = (MODE == SA_SAMPLE);
    constexpr int P = tc::Pitch<D>::kBytes;
    constexpr int TB = StageLayout<D>::kTileBytes;
    constexpr int SB = StageLayout<D>::kBytes;
    constexpr int kStages = stream_stages<MODE>();

    const int b = u / Hkv, g = u - b * Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const size_t ubase = (size_t)u * io.ld * D;
    const __nv_bfloat16* K = k + ubase;
    const __nv_bfloat16* V = v + ubase;
    const __nv_bfloat16* qg = q + ((size_t)b * Hq + (size_t)g * G) * D;
    const size_t qh0 = (size_t)b * Hq + (size_t)g * G;

    // the epilogue's inputs (query, prefill statistics) into L2 while streaming
    if constexpr (!ALL) {
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

    const int nt = ALL ? 0 : sg.n_t;
    const int n_i = ALL ? L : sg.n_i;
    const int win0 = L - sg.w_eff;
    const int32_t* gblk = blk_idx + (size_t)u * kb_stride;
    const int32_t* gsamp = samp_idx + (size_t)u * (sample_cap > 0 ? sample_cap : 0);
    // rows [0, n_indep) do not depend on the selection; the tile range uses an
    // upper bound on the list length (draw capacity); the exact count and the
    // lists are read once the selection is visible
    const int n_indep = ALL ? L : sg.s_eff + sg.w_eff;
    // per-head draws: head h's list follows head h-1's, each token tagged with
    // its head (it enters that head's softmax alone, weighted n_T / b_h)
    const bool PH = SAMP && io.per_head != 0;
    const int32_t* gsamp_ph = samp_idx + ((size_t)b * Hq + (size_t)g * G) * (sample_cap > 0 ? sample_cap : 0);
    int ph_pre[G + 1];
    float ph_lw[G];
#pragma unroll
    for (int h = 0; h <= G; ++h) ph_pre[h] = 0;
#pragma unroll
    for (int h = 0; h < G; ++h) ph_lw[h] = 0.f;
    const int n_hi = ALL ? L : sg.n_i + ((SAMP && nt > 0) ? (PH ? G : 1) * sample_cap : 0);
    int n_tok = n_hi;
    float lw_samp = 0.f;
    const bool blk_sm = sg.kk <= kBlkCache;
    bool samp_sm = true;
    bool sel_ready = ALL || n_indep >= n_hi;
    // Under programmatic dependent launch the preceding selection kernel may
    // still be running: wait for it before the first selection-dependent read
    // (a no-op when the kernel was launched normally).  Called at the same
    // point by every thread.
    auto wait_selection = [&]() {
        if (!sel_ready) {
            asm volatile("griddepcontrol.wait;\n" ::: "memory");
            int bu = 0;
            if (SAMP && nt > 0) {
                if (PH) {
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const int bh = min(__ldcg(samp_count + (size_t)b * Hq + g * G + h), sample_cap);
                        ph_pre[h + 1] = ph_pre[h] + bh;
                        ph_lw[h] = bh > 0 ? log2f((float)nt / (float)bh) : 0.f;
                    }
                    n_tok = sg.n_i + ph_pre[G];
                } else {
                    bu = min(__ldcg(samp_count + u), sample_cap);
                    lw_samp = bu > 0 ? log2f((float)nt / (float)bu) : 0.f;
                    n_tok = sg.n_i + bu;
                }
            }
            samp_sm = !PH && bu <= kSampCache;
            if (blk_sm)
                for (int x = threadIdx.x; x < sg.kk; x += kTcThreads) s_blk[x] = __ldcg(gblk + x);
            if (samp_sm)
                for (int x = threadIdx.x; x < bu; x += kTcThreads) s_samp[x] = __ldcg(gsamp + x);
            __syncthreads();
            sel_ready = true;
        }
    };
    // token t of the unit's list -> cache row, or -1 (masked), and the head
    // it belongs to (-1: every head)
    //   [sink 0..s_eff) [window L-w_eff..L) [chosen blocks] [draws]
    auto pos_of = [&](int t, int& tag) -> int {
        int p;
        tag = -1;
        if (ALL) p = t < L ? t : -1;
        else if (t >= n_tok) p = -1;
        else if (t < sg.s_eff) p = t;
        else if (t < n_indep) p = win0 + (t - sg.s_eff);
        else if (t < n_i) {
            const int j = t - n_indep;
            p = 16 * (blk_sm ? s_blk[j >> 4] : __ldcg(gblk + (j >> 4))) + (j & 15);
        } else if (PH) {
            const int j = t - n_i;
            int h = 0;
#pragma unroll
            for (int x = 1; x < G; ++x) h += (j >= ph_pre[x]) ? 1 : 0;
            tag = h;
            p = __ldcg(gsamp_ph + (size_t)h * sample_cap + (j - ph_pre[h]));
        } else {
            const int j = t - n_i;
            p = samp_sm ? s_samp[j] : __ldcg(gsamp + j);
        }
        return (unsigned)p < (unsigned)L ? p : -1;         // outside the cache: masked
    };
    const int ntiles = (n_hi + kTcTile - 1) / kTcTile;
    const int tile0 = chunk * tpc, tile1 = min(ntiles, tile0 + tpc);

    // Row positions of tile i go to its stage's pos array (every thread
    // calls this at the same point; a barrier must follow before the copy).
    auto put_pos = [&](int i) {
        if (i < tile1) {
            if ((i + 1) * kTcTile > n_indep) wait_selection();
            int* pos = reinterpret_cast<int*>(smem + (size_t)(i % kStages) * SB + 2 * TB);
            if (threadIdx.x < kTcTile) {
                int tag;
                pos[threadIdx.x] = pos_of(i * kTcTile + threadIdx.x, tag);
                pos[kTcTile + threadIdx.x] = tag;
            }
        }
    };
    // K/V rows of tile i into its stage (cp.async; masked rows zero-filled)
    auto copy_tile = [&](int i) {
        if (i < tile1) {
            unsigned char* sb = smem + (size_t)(i % kStages) * SB;
            const int* pos = reinterpret_cast<const int*>(sb + 2 * TB);
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

    // The query and (RESA) the epilogue's statistics are loaded into
    // registers first and used only later, so that their latency hides
    // behind the first two tiles, which are put in flight next.
    // G <= 4: tokens on the MMA rows (no row spent on absent heads); G = 8:
    // heads on the rows
    constexpr bool kTokRows = (G <= 4);
    using Engine = typename std::conditional<kTokRows, tc::WarpAttnT<D, G, PRIOR>, tc::WarpAttn<D, G, PRIOR>>::type;
    Engine wa;
    if constexpr (kTokRows) wa.load(PREFILL ? nullptr : qg, PRIOR ? st.mu_q + qh0 * D : nullptr);
    __shared__ float s_bias[8];
    EpiPre<D, G> pre;
    BiasPre<D, G, kTcWarps> bpre;
    if constexpr (PRIOR) {
        if (nt > 0) {
            epi_load<D, G>(pre, st, b, g, Hq);
            bias_load<__nv_bfloat16, D, G, kTcWarps>(bpre, qg, st, u, b, g, Hq);
        }
    }
    // kStages - 1 tiles in flight ahead of the one being computed
#pragma unroll
    for (int j = 0; j < kStages - 1; ++j) put_pos(tile0 + j);
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kStages - 1; ++j) copy_tile(tile0 + j);
    if constexpr (kTokRows) {
        wa.finish();
    } else {
        const int gh = min(lane >> 2, G - 1);
        wa.init(PREFILL ? nullptr : qg + (size_t)gh * D, PRIOR ? st.mu_q + (qh0 + gh) * D : nullptr);
    }
    float ks[2] = {0.f, 0.f};      // SUMS: this thread's column pair of K (c < D/2) or V (c >= D/2)
    // PREFILL: thread t takes the four columns 4c .. 4c+3, c = t mod (D/4), of
    // block t / (D/4) of every tile (threads past the tile's four blocks
    // idle at D = 64): fp64 key sums, the largest |block mean|
    constexpr int kQuads = D / 4;
    double pk[4] = {0.0, 0.0, 0.0, 0.0};
    float amax = 0.f;
    for (int i = tile0; i < tile1; ++i) {
        // the tile range was sized by the draw capacity: once the list length
        // is known, the tiles past it hold only masked rows (the copies of
        // the next two are drained after the loop)
        if (sel_ready && i * kTcTile >= n_tok) break;     // uniform
        // stage (i + kStages - 1) % kStages was last read by tile i-1,
        // finished before the trailing barrier of the previous iteration
        put_pos(i + kStages - 1);
        tc::cp_wait<kStages - 2>();   // this thread's copies of tile i have landed
        __syncthreads();              // everyone's, and the positions of the next tile
        copy_tile(i + kStages - 1);
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
        if constexpr (PREFILL) {
            // block means: the fp64 sum of 16 rows times 1/16 (exact), one
            // rounding to bf16 (L is a whole number of blocks)
            const int c = threadIdx.x % kQuads, grp = threadIdx.x / kQuads;
            const int rb = grp * 16;
            if (grp < 4 && base + rb < L) {
                const unsigned char* kp = sb + rb * P + c * 8;
                double s4[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
                for (int r = 0; r < 16; ++r) {
                    const uint2 w = *reinterpret_cast<const uint2*>(kp + r * P);
                    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
                    const float2 b2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
                    s4[0] += (double)a.x;
                    s4[1] += (double)a.y;
                    s4[2] += (double)b2.x;
                    s4[3] += (double)b2.y;
                }
                __nv_bfloat16 mean[4];
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    mean[x] = round_from_f64<__nv_bfloat16>(s4[x] * 0.0625);
                    amax = fmaxf(amax, fabsf(__bfloat162float(mean[x])));
                    pk[x] += s4[x];
                }
                const size_t row = (size_t)u * (io.ld / 16) + (size_t)((base + rb) / 16);
                *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(st.blk_mean) + row * D + 4 * c) =
                    *reinterpret_cast<const uint2*>(mean);
            }
        }
        const int r0 = warp * 16;
        if (base + r0 < n_tok) {
            constexpr int NR = kTokRows ? 2 : 4;            // token rows of this lane
            int rows[NR];
            if constexpr (kTokRows) {
                rows[0] = Engine::row(r0, 0);
                rows[1] = Engine::row(r0, 1);
            } else {
                const int tq = lane & 3;
                rows[0] = r0 + 2 * tq;
                rows[1] = r0 + 2 * tq + 1;
                rows[2] = r0 + 8 + 2 * tq;
                rows[3] = r0 + 9 + 2 * tq;
            }
            bool in_i[NR];
            const int* pos = reinterpret_cast<const int*>(sb + 2 * TB);
            // log2-weight of token j for a head: 0 on I, n_T / b for a draw
            // (per-head draws: only for the head that drew it), -inf if masked
            auto xw = [&](int j, int head) -> float {
                const int t = base + rows[j];
                if (pos[rows[j]] < 0) return -INFINITY;
                if (t < n_i) return 0.f;
                if (!PH) return lw_samp;
                const int tag = pos[kTcTile + rows[j]];
                float lw = 0.f;
#pragma unroll
                for (int h = 0; h < G; ++h) lw = (h == tag) ? ph_lw[h] : lw;
                return tag == head ? lw : -INFINITY;
            };
#pragma unroll
            for (int j = 0; j < NR; ++j) in_i[j] = PRIOR && pos[rows[j]] >= 0 && base + rows[j] < n_i;
            const uint32_t sk = tc::smem_u32(sb);
            if constexpr (kTokRows) {
                float xadd[2][2];
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int e = 0; e < 2; ++e) xadd[j][e] = xw(j, 2 * (lane & 3) + e);
                wa.step16(sk, sk + TB, r0, xadd, in_i, qscale);
            } else {
                float xadd[NR];
#pragma unroll
                for (int j = 0; j < NR; ++j) xadd[j] = xw(j, lane >> 2);
                wa.step16(sk, sk + TB, r0, xadd, in_i, qscale);
            }
        }
        __syncthreads();              // stage i%3 is refilled for tile i+3
    }
    tc::cp_wait<0>();
    __syncthreads();

    // ---- this chunk's record --------------------------------------------------------
    float* fb = reinterpret_cast<float*>(smem);
    float* ml = fb;                                     // [W][G][4]
    float* acc = ml + kTcWarps * G * 4;                 // [W][G][D]
    float* acc0 = acc + kTcWarps * G * D;               // [W][G][D] (PRIOR)
    float* own = acc + (PRIOR ? 2 : 1) * kTcWarps * G * D;   // own record when the unit is one chunk
    float* scratch = own + stream_rec<D, G, MODE>();
    wa.store(ml, acc, acc0);
    if constexpr (PRIOR) {
        if (nt > 0) bias_sum<D, G, kTcWarps>(bpre, s_bias, scale);
    }
    __syncthreads();
    const bool single = (nchunk == 1);
    if constexpr (!DENSE && !SUMS && !PREFILL) {
        if (single) {
            // the unit in one chunk: its output straight from the warps'
            // states (the merge, in warp order, then the mode's residual)
#pragma unroll
            for (int k = 0; k < EpiPre<D, G>::kPer; ++k) {
                const int idx = threadIdx.x + k * kTcThreads;
                if (idx >= G * D) break;
                const int h = idx / D, e = idx - h * D;
                float st4[2][3];                      // (M, Ls, A) of the exact and prior states
#pragma unroll
                for (int pr = 0; pr < (PRIOR ? 2 : 1); ++pr) {
                    float M = -INFINITY;
#pragma unroll
                    for (int w = 0; w < kTcWarps; ++w) M = fmaxf(M, ml[(w * G + h) * 4 + 2 * pr]);
                    float A = 0.f, Ls = 0.f;
#pragma unroll
                    for (int w = 0; w < kTcWarps; ++w) {
                        const float mw = ml[(w * G + h) * 4 + 2 * pr];
                        const float f = (mw == -INFINITY) ? 0.f : ex2(mw - M);
                        A = fmaf((pr ? acc0 : acc)[(w * G + h) * D + e], f, A);
                        Ls = fmaf(ml[(w * G + h) * 4 + 2 * pr + 1], f, Ls);
                    }
                    st4[pr][0] = M;
                    st4[pr][1] = Ls;
                    st4[pr][2] = A;
                }
                float o;
                if constexpr (PRIOR)
                    o = resid_value<MODE>(nt, st4[0][0], st4[0][1], st4[0][2], st4[1][0], st4[1][1], st4[1][2],
                                          pre.lz[k] * kLog2e, nt > 0 ? s_bias[h] : 0.f, pre.oe[k], lambda, 0.f, 0.f);
                else
                    o = resid_value<MODE>(nt, st4[0][0], st4[0][1], st4[0][2], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, lambda,
                                          0.f, 0.f);
                out[(qh0 + h) * D + e] = o;
            }
            return;
        }
    }
    float* r = single ? own : part + ((size_t)u * nchunk + chunk) * rec;
    tc::merge_warps<D, G, PRIOR>(ml, acc, acc0, kTcWarps, r);
    if constexpr (PREFILL) {
        // the chunk's totals (after the prior state): key sums in fp64, value
        // sums, the largest |block mean|; thread partials meet in the
        // list-cache area, which the prefill pass does not use
        double* s_pk = reinterpret_cast<double*>(smem + (size_t)kStages * SB);     // [4][D]
        float* s_am = reinterpret_cast<float*>(s_pk + 4 * D);                     // [warps]
        const int c = threadIdx.x % kQuads, grp = threadIdx.x / kQuads;
        if (grp < 4) {
#pragma unroll
            for (int x = 0; x < 4; ++x) s_pk[grp * D + 4 * c + x] = pk[x];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) s_am[warp] = amax;
        __syncthreads();
        double* rk = reinterpret_cast<double*>(r + 2 * G * (2 + D));
        for (int e = threadIdx.x; e < D; e += kTcThreads) {
            double a = 0.0;
#pragma unroll
            for (int x = 0; x < 4; ++x) a += s_pk[x * D + e];
            rk[e] = a;
        }
        if (threadIdx.x == 0) {
            float a = 0.f;
#pragma unroll
            for (int w = 0; w < kTcWarps; ++w) a = fmaxf(a, s_am[w]);
            r[2 * G * (2 + D) + 2 * D] = a;
        }
    }
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
    // The other chunks' records into shared memory (after the scratch) with
    // every load in flight at once, when they fit: combining them straight
    // from L2 chains one round trip per few records and elements.  Dense
    // needs only the exact state (the first G (2 + D) floats of a record).
    int rs = rec;
    bool sh = single;
    if (!single) {
        const int w = DENSE ? G * (2 + D) : rec;
        const int o = (int)(s_hs + G - fb + 3) & ~3;                 // float index, 16-byte aligned
        if ((w & 3) == 0 && (size_t)(o + nchunk * w) * 4 <= stream_smem<D, G, MODE>()) {
            float4* dst = reinterpret_cast<float4*>(fb + o);
            const int w4 = w / 4, n4 = nchunk * w4;
            constexpr int UN = 8;
            for (int x0 = 0; x0 < n4; x0 += UN * kTcThreads) {
                float4 t[UN];
#pragma unroll
                for (int j = 0; j < UN; ++j) {
                    const int x = x0 + j * kTcThreads + threadIdx.x;
                    if (x < n4) {
                        const int c = x / w4, y = x - c * w4;
                        t[j] = __ldcg(reinterpret_cast<const float4*>(recs + (size_t)c * rec) + y);
                    }
                }
#pragma unroll
                for (int j = 0; j < UN; ++j) {
                    const int x = x0 + j * kTcThreads + threadIdx.x;
                    if (x < n4) dst[x] = t[j];
                }
            }
            __syncthreads();
            recs = fb + o;
            rs = w;
            sh = true;
        }
    }
    if constexpr (PREFILL) {
        // O_Est and log Z of the typical queries (the prior state); the value
        // totals (head 0's exact state: every token weighted 1, so its
        // accumulator is the sum of the value rows); the key totals in chunk
        // order; the largest |block mean|
        constexpr int OP = G * (2 + D), OS = 2 * G * (2 + D);
        if (sh) {
            combine_heads<G, D, true>(recs, nchunk, rs, OP, s_ml, s_ml + G);
            combine_heads<G, D, true>(recs, nchunk, rs, 0, s_ml + 2 * G, s_ml + 3 * G);
        } else {
            combine_heads<G, D, false>(recs, nchunk, rs, OP, s_ml, s_ml + G);
            combine_heads<G, D, false>(recs, nchunk, rs, 0, s_ml + 2 * G, s_ml + 3 * G);
        }
        __syncthreads();
        for (int idx = threadIdx.x; idx < G * D; idx += kTcThreads) {
            const int h = idx / D, e = idx - h * D;
            const float A = sh ? combine_acc<G, D, true>(recs, nchunk, rs, OP, h, e, s_ml[h])
                               : combine_acc<G, D, false>(recs, nchunk, rs, OP, h, e, s_ml[h]);
            st.o_est[(qh0 + h) * D + e] = A / s_ml[G + h];
            if (e == 0) st.log_z0[qh0 + h] = (s_ml[h] + log2f(s_ml[G + h])) * kLn2;
        }
        for (int e = threadIdx.x; e < D; e += kTcThreads) {
            const float sv = sh ? combine_acc<G, D, true>(recs, nchunk, rs, 0, 0, e, s_ml[2 * G])
                                : combine_acc<G, D, false>(recs, nchunk, rs, 0, 0, e, s_ml[2 * G]);
            double a = 0.0;
            for (int c = 0; c < nchunk; ++c) {
                const float* rc = recs + (size_t)c * rs;
                a += sh ? reinterpret_cast<const double*>(rc + OS)[e] : __ldcg(reinterpret_cast<const double*>(rc + OS) + e);
            }
            st.sum_k[(size_t)u * D + e] = (float)a;
            st.mu_k[(size_t)u * D + e] = (float)(a / (double)L);
            st.sum_v[(size_t)u * D + e] = sv;
        }
        if (threadIdx.x == 0) {
            float a = 0.f;
            for (int c = 0; c < nchunk; ++c)
                a = fmaxf(a, sh ? recs[(size_t)c * rs + OS + 2 * D] : __ldcg(recs + (size_t)c * rs + OS + 2 * D));
            st.kbar_absmax[u] = a;
        }
    } else if constexpr (DENSE) {
        if (sh) combine_heads<G, D, true>(recs, nchunk, rs, 0, s_ml, s_ml + G);
        else combine_heads<G, D, false>(recs, nchunk, rs, 0, s_ml, s_ml + G);
        __syncthreads();
        for (int idx = threadIdx.x; idx < G * D; idx += kTcThreads) {
            const int h = idx / D, e = idx - h * D;
            const float A = sh ? combine_acc<G, D, true>(recs, nchunk, rs, 0, h, e, s_ml[h])
                               : combine_acc<G, D, false>(recs, nchunk, rs, 0, h, e, s_ml[h]);
            out[((size_t)b * Hq + g * G + h) * D + e] = A / s_ml[G + h];
        }
    } else {
        constexpr int EM = DENSE ? SA_DROP : MODE;
        if (sh)
            decode_epilogue<__nv_bfloat16, D, G, EM, true>(recs, nchunk, rs, qg, st, u, b, g, Hq, nt, scale,
                                                           lambda, out, s_acc, s_acc0, s_ml, s_t, s_hs, &pre,
                                                           s_bias);
        else
            decode_epilogue<__nv_bfloat16, D, G, EM, false>(recs, nchunk, rs, qg, st, u, b, g, Hq, nt, scale,
                                                            lambda, out, s_acc, s_acc0, s_ml, s_t, s_hs, &pre,
                                                            s_bias);
    }
    if (!single) reset_counter(cnt + u);
}

template <int D, int G, int MODE>
__global__ void __launch_bounds__(kTcThreads, 2)
k_stream_tc(StreamIo io) {
    constexpr int SB = StageLayout<D>::kBytes;
    extern __shared__ __align__(16) unsigned char smem[];
    int* s_blk = reinterpret_cast<int*>(smem + (size_t)stream_stages<MODE>() * SB);
    stream_unit<D, G, MODE>(io, smem, s_blk, s_blk + kBlkCache, blockIdx.y, blockIdx.x);
}


}  // namespace sa
