#pragma once
// Device code of the per-step selection (vAttention, Method, overall
// framework: I_f = sink + local window + top-k; the top-k ranks 16-token
// blocks by their mean key, the block selection of Quest / ArkVale that RESA
// wraps), used by the selection kernels.
//
// select_unit (one unit per CTA, or a slice of one when split):
//   scan  : score intervals of the unit's candidate blocks from the int8
//           sketch of the centred block summaries (0.56x their bytes at
//           d = 128, bf16): y_c = sf s_c (Q . code_c) by integer dot products
//           (Q a 15-bit code of qbar = sum_h q_h), and [y_c - e_c, y_c + e_c]
//           certain to hold z_c = x_c - qbar . m, the exact score
//           x_c = sum_h q_h . kbar_c less a constant common to all blocks.
//           The HBM-bound part: one read of the sketch, streamed by bulk
//           copies.  With one CTA per unit (enough units to fill the GPU) the
//           bounds stay in shared memory; with several CTAs per unit they go
//           to the workspace and the CTA that finishes the unit last
//           (completion ticket, no wait) takes over.
//   top-k : the k best lower bounds (per-warp running lists merged, or a
//           radix select for k > 32); thr = the k-th.  Every candidate whose
//           upper bound reaches thr is in the band; the exact top k by
//           (x desc, block index asc) lies inside it.  A band of exactly k is
//           the answer; otherwise its members are rescored exactly from the
//           bf16 / fp32 summaries (exact products, double-double sum, one
//           rounding) and ranked.  The decision is the exact one.
//   draws : tail positions for the sampling estimator (SplitMix64 counters).
#include "sa_bulk.cuh"
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {


constexpr int kSmemKeys = 4096;     // candidate keys held in shared memory (16 KB)
constexpr int kBandCap = 512;       // band members ranked in shared memory
constexpr int kWarpTopK = 32;       // largest k of the warp-argmax path

// The scan's shared-memory ring over the sketch: kStages stages, each SR = 128
// consecutive block rows as SR x D int8 codes followed by SR x 16 bytes of
// {s, rn, kn, 0}.  A code row is CPR 16-byte chunks (one per lane of a lane
// group, GPW groups per warp); a warp scores R rows per lane group of each
// stage (SR = NW * GPW * R, NW warps per CTA).  Each stage is 18 KB at
// d = 128.
template <int D, int NW, int STAGES>
struct SketchRing {
    static constexpr int kStages = STAGES;
    static constexpr int SR = 128;
    static constexpr int kCodeBytes = SR * D;
    static constexpr int kMetaBytes = SR * 16;
    static constexpr int kStageBytes = kCodeBytes + kMetaBytes;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int CPR = D / 16;
    static constexpr int GPW = 32 / CPR;
    static constexpr int R = SR / (NW * GPW);
    static constexpr size_t kSmem = (size_t)kRingBytes + 8 * kStages;      // ring + its barriers
    static_assert(R >= 1 && (R & (R - 1)) == 0 && CPR >= R, "stage geometry");
};

__device__ __forceinline__ uint32_t fkey(float y) {
    const uint32_t b = __float_as_uint(y + 0.0f);   // -0 -> +0
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float fkey_inv(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}
__device__ __forceinline__ unsigned long long dkey(double x) {
    const unsigned long long b = (unsigned long long)__double_as_longlong(x + 0.0);
    return (b >> 63) ? ~b : (b | 0x8000000000000000ull);
}
// score key and block index in one orderable word: larger = better,
// equal scores ordered by lower index
__device__ __forceinline__ unsigned long long comp_key(uint32_t key, int i) {
    return ((unsigned long long)key << 32) | (unsigned long long)(~(uint32_t)i);
}
__device__ __forceinline__ int comp_index(unsigned long long c) { return (int)(~(uint32_t)c); }

__device__ __forceinline__ unsigned long long shfl_xor_u64(unsigned long long v, int off) {
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, (uint32_t)v, off);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, (uint32_t)(v >> 32), off);
    return ((unsigned long long)hi << 32) | lo;
}
__device__ __forceinline__ unsigned long long shfl_u64(unsigned long long v, int src) {
    const uint32_t lo = __shfl_sync(0xffffffffu, (uint32_t)v, src);
    const uint32_t hi = __shfl_sync(0xffffffffu, (uint32_t)(v >> 32), src);
    return ((unsigned long long)hi << 32) | lo;
}
__device__ __forceinline__ unsigned long long shfl_up_u64(unsigned long long v, int d) {
    const uint32_t lo = __shfl_up_sync(0xffffffffu, (uint32_t)v, d);
    const uint32_t hi = __shfl_up_sync(0xffffffffu, (uint32_t)(v >> 32), d);
    return ((unsigned long long)hi << 32) | lo;
}
__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const unsigned long long o = shfl_xor_u64(v, off);
        v = o > v ? o : v;
    }
    return v;
}

// Block-wide exclusive scan of one int per thread (thread order).  Returns
// this thread's exclusive prefix; *total gets the sum.  Uses sw[NT/32 + 1].
template <int NT>
__device__ __forceinline__ int block_exscan(int v, int* sw, int* total) {
    constexpr int NW = NT / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) sw[warp] = inc;
    __syncthreads();
    if (threadIdx.x == 0) {
        int s = 0;
        for (int w = 0; w < NW; ++w) { const int c = sw[w]; sw[w] = s; s += c; }
        sw[NW] = s;
    }
    __syncthreads();
    const int r = sw[warp] + inc - v;
    *total = sw[NW];
    __syncthreads();
    return r;
}

template <int NT>
__device__ __forceinline__ int block_sum(int v, int* sw) {
    int tot;
    (void)block_exscan<NT>(v, sw, &tot);
    return tot;
}

// Radix select (MSB first, 8 bits per pass) of the kk-th largest key among
// key(0..n-1).  On return *thr is that key and *need is how many of the keys
// equal to it belong to the top kk (the rest of the top kk is strictly above).
template <int NT, typename KT, typename KeyFn>
__device__ void radix_select(KeyFn key, int n, int kk, KT* thr, int* need, unsigned* hist,
                             int* s_digit, int* s_rem) {
    KT prefix = 0, mask = 0;
    int rem = kk;
    const int lane = threadIdx.x & 31;
    for (int shift = (int)sizeof(KT) * 8 - 8; shift >= 0; shift -= 8) {
        for (int x = threadIdx.x; x < 256; x += NT) hist[x] = 0;
        __syncthreads();
        // warp-aggregated: lanes with equal digits add once (scores share their
        // top bits, so per-lane atomics would serialise on a few bins)
        for (int i0 = 0; i0 < n; i0 += NT) {
            const int i = i0 + threadIdx.x;
            int digit = 256;                        // 256 = nothing to count
            if (i < n) {
                const KT kx = key(i);
                if ((kx & mask) == prefix) digit = (int)((kx >> shift) & 0xFF);
            }
            const unsigned peers = __match_any_sync(0xffffffffu, digit);
            if (digit < 256 && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (unsigned)__popc(peers));
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // lane owns bins 255-8*lane .. 248-8*lane (descending digits)
            unsigned c[8], loc = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { c[j] = hist[255 - 8 * lane - j]; loc += c[j]; }
            unsigned inc = loc;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const unsigned o = __shfl_up_sync(0xffffffffu, inc, off);
                if (lane >= off) inc += o;
            }
            unsigned ex = inc - loc;
            if (ex < (unsigned)rem && inc >= (unsigned)rem) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (ex + c[j] >= (unsigned)rem) { *s_digit = 255 - 8 * lane - j; *s_rem = rem - (int)ex; break; }
                    ex += c[j];
                }
            }
        }
        __syncthreads();
        prefix |= (KT)(*s_digit) << shift;
        mask |= (KT)0xFF << shift;
        rem = *s_rem;
        __syncthreads();
    }
    *thr = prefix;
    *need = rem;
}

// Writes, in ascending index order, c_lo + i for the top kk of key(0..n-1):
// every key above thr, and the first `need` keys equal to thr (lowest index
// first).  Each thread owns one contiguous chunk of indices.
template <int NT, typename KT, typename KeyFn>
__device__ void emit_topk(KeyFn key, int n, KT thr, int need, int kk, int c_lo, int32_t* out_idx, int* sw) {
    const int C = (n + NT - 1) / NT;
    const int i0 = min(n, (int)threadIdx.x * C), i1 = min(n, i0 + C);
    int eqc = 0;
    for (int i = i0; i < i1; ++i) eqc += (key(i) == thr) ? 1 : 0;
    int tot;
    const int eq_before = block_exscan<NT>(eqc, sw, &tot);
    int selc = 0, r = eq_before;
    for (int i = i0; i < i1; ++i) {
        const KT kx = key(i);
        if (kx > thr) ++selc;
        else if (kx == thr) { if (r < need) ++selc; ++r; }
    }
    int p = block_exscan<NT>(selc, sw, &tot);
    r = eq_before;
    for (int i = i0; i < i1; ++i) {
        const KT kx = key(i);
        bool take = kx > thr;
        if (kx == thr) { take = r < need; ++r; }
        if (take && p < kk) out_idx[p++] = c_lo + i;
    }
}

// Top kk (kk <= 32, n <= KEYS) of keys[0..n) by argmax rounds: every warp
// holds a contiguous span in registers and extracts its best kk one at a time
// (lane max, then warp max over 64-bit (key, ~index) words); warp 0 then
// merges the per-warp lists the same way.  s_list[0..kk) gets the result in
// rank order.  s_cand holds NT/32 * kk words.
template <int NT, int KEYS = kSmemKeys>
__device__ void warp_topk(const uint32_t* keys, int n, int kk, unsigned long long* s_cand,
                          unsigned long long* s_list) {
    constexpr int NW = NT / 32;
    constexpr int C = KEYS / NT;                       // keys per lane (n <= KEYS)
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int span = (n + NW - 1) / NW;
    const int w0 = warp * span;
    unsigned long long c[C];
#pragma unroll
    for (int j = 0; j < C; ++j) {
        const int i = w0 + j * 32 + lane;
        c[j] = (j * 32 + lane < span && i < n) ? comp_key(keys[i], i) : 0ull;
    }
    for (int r = 0; r < kk; ++r) {
        unsigned long long m = 0ull;
#pragma unroll
        for (int j = 0; j < C; ++j) m = c[j] > m ? c[j] : m;
        const unsigned long long best = warp_max_u64(m);
#pragma unroll
        for (int j = 0; j < C; ++j) if (c[j] == best) c[j] = 0ull;     // keys are unique
        if (lane == 0) s_cand[warp * kk + r] = best;
    }
    __syncthreads();
    if (warp == 0) {
        constexpr int CM = NW * kWarpTopK / 32;        // candidates per lane
        unsigned long long d[CM];
#pragma unroll
        for (int j = 0; j < CM; ++j) {
            const int i = j * 32 + lane;
            d[j] = i < NW * kk ? s_cand[i] : 0ull;
        }
        for (int r = 0; r < kk; ++r) {
            unsigned long long m = 0ull;
#pragma unroll
            for (int j = 0; j < CM; ++j) m = d[j] > m ? d[j] : m;
            const unsigned long long best = warp_max_u64(m);
#pragma unroll
            for (int j = 0; j < CM; ++j) if (d[j] == best) d[j] = 0ull;
            if (lane == 0) s_list[r] = best;
        }
    }
    __syncthreads();
}

constexpr int kCandCap = 256;

// Top kk (kk <= 32, or <= CC with BLOCKB; kk < n) of the n lower-bound keys lk[] in shared memory by
// (key desc, index asc), in rank order into s_list, and the band {upper >=
// thr} (thr = the kk-th lower key) into s_bidx / *s_band.  Thread t owns the
// keys t, t + NT, ... (n <= 32 NT) and takes their maximum; in each warp a
// lower bound B_w on the kk-th largest of its 32 maxima has at least kk keys
// at or above it, and so does B = max_w B_w, so thr >= B.  The candidates
// are the keys whose upper bound reaches B: they contain the top kk by lower
// bound and the whole band, and are usually few; they are compacted (each
// thread's matches at its place in a block scan) into s_c / s_u (up to CC),
// ranked exactly, and the band is read off them (its first kBandCap members
// listed, all counted).  Returns false, having written nothing, when more
// than CC keys reach B.  *s_b must be zero on entry and visible to every
// thread; sw holds NT/32 ints.  BLOCKB: B is instead the kk-th largest of all
// NT maxima to 16 bits (a bitwise search with block-wide counts, 16
// barriers), a tighter bound when kk is large against the 32 maxima of one
// warp; kk may then be up to CC (s_list holds kk entries).
template <int NT, int KEYS = kSmemKeys, int CC = kCandCap, bool BLOCKB = false>
__device__ bool topk_band(const uint32_t* lk, const uint32_t* uk, int n, int kk, unsigned long long* s_list,
                          unsigned long long* s_c, uint32_t* s_u, int* sw, unsigned* s_b, int* s_bidx,
                          int* s_band) {
    constexpr int NW = NT / 32;
    static_assert(KEYS <= 32 * NT, "one mask bit per owned key");
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t gm = 0u;
#pragma unroll 4
    for (int i = threadIdx.x; i < n; i += NT) gm = max(gm, lk[i]);
    uint32_t bnd = 0u;
    if constexpr (BLOCKB) {
        for (int bit = 31; bit >= 16; --bit) {
            const uint32_t cand = bnd | (1u << bit);
            if (__syncthreads_count(gm >= cand) >= kk) bnd = cand;
        }
    } else {
        uint32_t bw = 0u;
#pragma unroll 8
        for (int bit = 31; bit >= 16; --bit) {
            const uint32_t cand = bw | (1u << bit);
            if (__popc(__ballot_sync(0xffffffffu, gm >= cand)) >= kk) bw = cand;
        }
        if (lane == 0) atomicMax(s_b, bw);
        __syncthreads();
        bnd = *s_b;
    }
    // this thread's keys whose upper bound reaches B, as a bit mask
    unsigned mine = 0u;
#pragma unroll 4
    for (int j = 0; j * NT + (int)threadIdx.x < n; ++j) mine |= (uk[j * NT + threadIdx.x] >= bnd ? 1u : 0u) << j;
    const int cnt = __popc(mine);
    int inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += x;
    }
    if (lane == 31) sw[warp] = inc;
    __syncthreads();
    int off = inc - cnt, nc = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        const int x = sw[w];
        off += w < warp ? x : 0;
        nc += x;
    }
    if (nc > CC) return false;                       // (uniform: every thread summed the same counts)
    while (mine != 0u) {
        const int j = __ffs(mine) - 1;
        mine &= mine - 1u;
        const int i = j * NT + threadIdx.x;
        s_c[off] = comp_key(lk[i], i);
        s_u[off] = uk[i];
        ++off;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < nc; j += NT) {
        const unsigned long long c = s_c[j];
        int r = 0;
#pragma unroll 4
        for (int q = 0; q < nc; ++q) r += s_c[q] > c ? 1 : 0;
        if (r < kk) s_list[r] = c;
    }
    __syncthreads();
    if (warp == 0) {
        const uint32_t thr = (uint32_t)(s_list[kk - 1] >> 32);
        int base = 0;
        for (int j0 = 0; j0 < nc; j0 += 32) {
            const int j = j0 + lane;
            const bool in = j < nc && s_u[j] >= thr;
            const unsigned m = __ballot_sync(0xffffffffu, in);
            const int pos = base + __popc(m & ((1u << lane) - 1u));
            if (in && pos < kBandCap) s_bidx[pos] = comp_index(s_c[j]);
            base += __popc(m);
        }
        if (lane == 0) *s_band = base;
    }
    __syncthreads();
    return true;
}

// Ascending sort of one int per lane across the warp (bitonic network).
__device__ __forceinline__ int warp_sort_asc(int v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const int o = __shfl_xor_sync(0xffffffffu, v, stride);
            const bool up = ((lane & size) == 0);
            const bool lower = ((lane & stride) == 0);
            v = (lower == up) ? min(v, o) : max(v, o);
        }
    }
    return v;
}

// Sorts s_list[0..kk) (kk <= 32) by block index and writes c_lo + index in
// ascending order (one warp).
__device__ __forceinline__ void emit_sorted_list(const unsigned long long* s_list, int kk, int c_lo,
                                                 int32_t* out_idx, int* s_sorted) {
    if (threadIdx.x >= 32) return;
    const int lane = threadIdx.x;
    const int v = warp_sort_asc(lane < kk ? comp_index(s_list[lane]) : 0x7fffffff);
    if (lane < kk) {
        out_idx[lane] = c_lo + v;
        s_sorted[lane] = c_lo + v;
    }
}

// s + p with the rounding error of the addition carried into c (error-free
// two-sum; explicit roundings so nothing is contracted or reassociated)
__device__ __forceinline__ void two_sum_acc(double& s, double& c, double p) {
    const double t = __dadd_rn(s, p);
    const double bp = __dsub_rn(t, s);
    const double err = __dadd_rn(__dsub_rn(s, __dsub_rn(t, bp)), __dsub_rn(p, bp));
    s = t;
    c = __dadd_rn(c, err);
}

// Exact block score sum_h sum_e q_he kbar_ce rounded once, for M rows at a
// time (warp-collective; lane 0 holds the results).  Each product of two bf16
// / fp32 values is exact in fp64; the products are added in double-double
// (two-sum, errors summed apart), lanes combined the same way, and the two
// parts rounded together, which is the correctly rounded sum unless the exact
// sum lies within ~n^2 2^-106 sum|terms| of a rounding boundary.  Identical
// rows always get identical scores.
template <typename T, int D, int G, int M>
__device__ __forceinline__ void exact_scores(const T* const (&rows)[M], const bool (&live)[M], const float* s_qh,
                                             double (&x)[M]) {
    const int lane = threadIdx.x & 31;
    float k[M][D / 32];
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
        for (int i = 0; i < D / 32; ++i) k[m][i] = live[m] ? to_f32<T>(rows[m][lane + 32 * i]) : 0.f;
    // the M members' chains advance together (independent, so they overlap)
    double s[M], c[M];
#pragma unroll
    for (int m = 0; m < M; ++m) { s[m] = 0.0; c[m] = 0.0; }
#pragma unroll
    for (int i = 0; i < D / 32; ++i)
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const double qv = (double)s_qh[h * D + lane + 32 * i];
#pragma unroll
            for (int m = 0; m < M; ++m) two_sum_acc(s[m], c[m], __dmul_rn(qv, (double)k[m][i]));
        }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int m = 0; m < M; ++m) {
            const double so = __shfl_xor_sync(0xffffffffu, s[m], off);
            const double co = __shfl_xor_sync(0xffffffffu, c[m], off);
            two_sum_acc(s[m], c[m], so);
            c[m] = __dadd_rn(c[m], co);
        }
#pragma unroll
    for (int m = 0; m < M; ++m) x[m] = __dadd_rn(s[m], c[m]) + 0.0;      // -0 -> +0
}

// exact scores of the band members s_bidx[0..nb) into s_bx (two members
// per warp, their rows in flight together)
template <typename T, int D, int G, int NW>
__device__ void rescore_members(const T* bm, const int* s_bidx, int nb, const float* s_qh, double* s_bx) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // member warp + m * NW, m < 2: a band of up to 2 NW is one round
    for (int jb = 0; jb < nb; jb += 2 * NW) {
        const T* rows[2];
        bool live[2];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int j = jb + warp + m * NW;
            live[m] = j < nb;
            rows[m] = bm + (size_t)(live[m] ? s_bidx[j] : 0) * D;
        }
        if (!live[0]) continue;                       // warp-uniform
        double x[2];
        exact_scores<T, D, G, 2>(rows, live, s_qh, x);
#pragma unroll
        for (int m = 0; m < 2; ++m)
            if (lane == 0 && live[m]) s_bx[jb + warp + m * NW] = x[m];
    }
}

// The unit's tail draws (vAttention, Method, key design 1: uniform draws
// from the residual, with replacement): min(sample_b, sample_cap) positions
// when the tail is not empty, written to samp_idx (and s_copy when they fit
// s_copy_cap), their count to samp_count.  One stream per unit (row u of
// samp_idx / samp_count, the SplitMix64 stream of (seed, b, g, step)) or,
// with per_head, one per query head h of the group (row b Hq + g G + h, the
// stream of (seed, b, g G + h, step); s_copy unused).  chosen = the unit's kk
// chosen blocks in ascending order (shared or global memory, visible to
// every thread).  Draw i's rank r maps to the r-th tail position: tail =
// [s_eff, L - w_eff) minus the chosen blocks, and chosen block j starts
// after g_j = 16 c_j - s_eff - 16 j tail tokens.  Returns the count.
template <int NT>
__device__ __forceinline__ int unit_draws(const SetGeom& sg, const int32_t* chosen, int sample_b, int sample_cap,
                                          unsigned long long seed, int b, int g, int step, int u, int32_t* samp_idx,
                                          int32_t* samp_count, int* s_copy, int s_copy_cap, int G = 1,
                                          int per_head = 0, int Hq = 0) {
    const int nt = sg.n_t, kk = sg.kk;
    const int bdraw = (nt > 0) ? min(sample_b, sample_cap) : 0;
    const int ns = per_head ? G : 1;                         // streams
    if (threadIdx.x < ns) samp_count[per_head ? b * Hq + g * G + threadIdx.x : u] = bdraw;
    if (bdraw > 0) {
        for (int x = threadIdx.x; x < ns * bdraw; x += NT) {
            const int s = x / bdraw, i = x - s * bdraw;
            const int row = per_head ? b * Hq + g * G + s : u;
            const uint64_t key = unit_key(seed, (uint64_t)b, (uint64_t)(per_head ? g * G + s : g), (uint64_t)step);
            int32_t* out_s = samp_idx + (size_t)row * sample_cap;
            const int r = (int)draw_rank(key, (uint32_t)i, (uint32_t)nt);
            int lo_j = 0, hi_j = kk;             // count of j with g_j <= r
            while (lo_j < hi_j) {
                const int mid = (lo_j + hi_j) >> 1;
                const int gj = 16 * chosen[mid] - sg.s_eff - 16 * mid;
                if (gj <= r) lo_j = mid + 1; else hi_j = mid;
            }
            out_s[i] = sg.s_eff + r + 16 * lo_j;
            if (!per_head && s_copy != nullptr && bdraw <= s_copy_cap) s_copy[i] = sg.s_eff + r + 16 * lo_j;
        }
    }
    return bdraw;
}

// Inputs and outputs of one unit's selection (device pointers; the layouts
// of sa_select in sa_decode.h).
struct SelectIo {
    const void* q;
    const void* blk_mean;
    const int8_t* blk_code;
    const float4* blk_meta;
    int Hq, Hkv, L;
    int ld;                      // tokens per unit in the cache allocation (block rows ld / 16)
    SetGeom sg;
    int rows, nss;                        // candidate rows per split, splits per unit
    float* sc_lo_all;                     // [U][n_cand] lower bounds (split units)
    float* sc_up_all;                     // [U][n_cand] upper bounds (split units)
    unsigned long long* xkey;             // [U][n_cand] exact keys (very wide bands)
    unsigned* cnt;                        // [U] completion tickets
    int kb_stride;
    int32_t* blk_idx;
    int32_t* samp_idx;
    int32_t* samp_count;
    int32_t* n_rescored;
    int sample_b, sample_cap;
    unsigned long long seed;
    int step;
    unsigned* timeouts;                   // the library's count of abandoned waits (one per device)
    int per_head;                         // draws per query head (rows of samp_idx: B Hq)
};

// Shared memory the selection works in (the caller lays it out):
//   hist [256] (16-byte aligned), sw [NT/32 + 1], misc [3], qh [G*D] f32, qi
//   [2*D] (16-byte aligned), qc [3], ukeys [kSmemKeys], lkeys [kSmemKeys],
//   sorted [kWarpTopK], ring
//   (SketchRing::kRingBytes, 128-byte aligned, reused for the top-k and band
//   arrays after the scan), bar [kStages] mbarriers, samp [samp_cap] or null
//   (a shared copy of the draws).
struct SelectSmem {
    unsigned* hist;
    int* sw;
    int* misc;
    float* qh;
    int8_t* qi;
    float* qc;
    uint32_t* ukeys;
    uint32_t* lkeys;
    int* sorted;
    unsigned char* ring;
    uint64_t* bar;
    int* samp;
    int samp_cap;
};

// The kernel arguments of a selection call (workspace carved by its plan).
SelectIo select_io(const Dims& d, const SelectPlan& p, const SelectArgs& a);

// Which part of a unit's selection a call runs: everything (one CTA, or the
// split CTAs of a unit with the last one finishing), only the scan of this
// CTA's slice into the workspace bounds (a split unit whose finish runs in a
// kernel of its own), or only that finish (keys gathered from the workspace).
enum SelPhase { kPhAll = 0, kPhScan = 1, kPhFinish = 2 };

// done: this CTA finished the unit (false for a split CTA that was not the
// unit's last, or after an abandoned wait); sorted_smem: the chosen blocks
// (ascending) are in SelectSmem::sorted as well; bdraw: draws written.
struct SelectOutcome {
    bool done;
    bool sorted_smem;
    int bdraw;
};

// KEYS: capacity of SelectSmem::ukeys / lkeys (a unit's keys stay in shared
// memory when n_cand <= KEYS, else in place in the workspace).
template <typename T, int D, int G, int NT, int STAGES, int PHASE = kPhAll, int KEYS = kSmemKeys,
          int CC = kCandCap, bool BLOCKB = false>
__device__ __forceinline__ SelectOutcome select_unit(const SelectIo& io, const SelectSmem& sm, int u, int split) {
    constexpr int NW = NT / 32;
    using Ring = SketchRing<D, NW, STAGES>;
    constexpr int R = Ring::R, CPR = Ring::CPR, GPW = Ring::GPW;
    const T* __restrict__ q = static_cast<const T*>(io.q);
    const T* __restrict__ blk_mean = static_cast<const T*>(io.blk_mean);
    const int8_t* __restrict__ blk_code = io.blk_code;
    const float4* __restrict__ blk_meta = io.blk_meta;
    const int Hq = io.Hq, Hkv = io.Hkv, L = io.L, rows = io.rows, nss = io.nss;
    const SetGeom& sg = io.sg;
    unsigned* __restrict__ cnt = io.cnt;
    unsigned long long* __restrict__ xkey = io.xkey;
    const int kb_stride = io.kb_stride;
    int32_t* __restrict__ blk_idx = io.blk_idx;
    int32_t* __restrict__ samp_idx = io.samp_idx;
    int32_t* __restrict__ samp_count = io.samp_count;
    int32_t* __restrict__ n_rescored = io.n_rescored;
    const int sample_b = io.sample_b, sample_cap = io.sample_cap, step = io.step;
    const unsigned long long seed = io.seed;
    unsigned* hist = sm.hist;
    int* sw = sm.sw;
    int& s_digit = sm.misc[0];
    int& s_rem = sm.misc[1];
    int& s_nb = sm.misc[2];
    float* s_qh = sm.qh;
    int8_t* s_qi = sm.qi;
    float* s_qc = sm.qc;
    uint32_t* s_ukeys = sm.ukeys;
    uint32_t* s_lkeys = sm.lkeys;
    int* s_sorted = sm.sorted;
    unsigned char* s_ring = sm.ring;
    uint64_t* s_bar = sm.bar;
    constexpr int kCandWords = NW * kWarpTopK > CC ? NW * kWarpTopK : CC;
    unsigned long long* s_cand = reinterpret_cast<unsigned long long*>(s_ring);          // kCandWords
    constexpr int LISTN = BLOCKB ? (CC > kWarpTopK ? CC : kWarpTopK) : kWarpTopK;
    unsigned long long* s_list = s_cand + kCandWords;                                    // LISTN
    double* s_bx = reinterpret_cast<double*>(s_list + LISTN);                            // kBandCap
    int* s_bidx = reinterpret_cast<int*>(s_bx + kBandCap);                               // kBandCap
    unsigned char* s_bsel = reinterpret_cast<unsigned char*>(s_bidx + kBandCap);         // kBandCap
    uint32_t* s_u = reinterpret_cast<uint32_t*>(s_bsel + kBandCap);                      // CC

    const int b = u / Hkv, g = u - b * Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int li = lane % CPR, gsub = lane / CPR;
    const int nb = io.ld / 16;         // block rows per unit
    const int n = sg.n_cand, kk = sg.kk;
    const T* qg = q + ((size_t)b * Hq + (size_t)g * G) * D;
    float* sc_lo = io.sc_lo_all + (size_t)u * (n > 0 ? n : 1);
    float* sc_up = io.sc_up_all + (size_t)u * (n > 0 ? n : 1);
    // one CTA per unit: the keys never leave shared memory
    const bool local = PHASE == kPhAll && (nss == 1) && n <= KEYS;
    SelectOutcome res{false, false, 0};

    // ---- scan: score intervals of this CTA's slice ------------------------------
    // The slice's sketch rows are contiguous: thread 0 streams codes and
    // metadata through a ring of kStages shared-memory stages with bulk copies,
    // kStages stages in flight; all warps score each stage as it lands.
    const int r0 = split * rows, r1 = min(n, r0 + rows);
    const int nrows = max(0, r1 - r0);
    const int nst = PHASE == kPhFinish ? 0 : (nrows + Ring::SR - 1) / Ring::SR;
    const size_t row0 = (size_t)u * nb + sg.c_lo + r0;
    const int8_t* code0 = blk_code + row0 * D;
    const float4* meta0 = blk_meta + row0;
    const uint32_t ring = smem_addr(s_ring), bar0 = smem_addr(s_bar);
    if (threadIdx.x == 0) {
#pragma unroll
        for (int j = 0; j < Ring::kStages; ++j) mbar_init(bar0 + 8 * j, 1);
        mbar_init_fence();
    }
    __syncthreads();
    // the sketch is read once per step: evict-first in L2
    const uint64_t pol = l2_evict_first_policy();
    auto issue = [&](int j) {                      // thread 0
        if (j < nst) {
            const int rj = min(Ring::SR, nrows - j * Ring::SR);
            const uint32_t bar = bar0 + 8 * (j % Ring::kStages);
            const uint32_t dst = ring + (j % Ring::kStages) * Ring::kStageBytes;
            mbar_arrive_expect_tx(bar, (uint32_t)rj * (D + 16));
            bulk_g2s_hint(dst, code0 + (size_t)j * Ring::SR * D, (uint32_t)rj * D, bar, pol);
            bulk_g2s_hint(dst + Ring::kCodeBytes, meta0 + (size_t)j * Ring::SR, (uint32_t)rj * 16, bar, pol);
        }
    };
    if (threadIdx.x == 0)
        for (int j = 0; j < Ring::kStages; ++j) issue(j);
    __syncwarp();

    // The group query, exact per head (for rescoring) and as a 15-bit code of
    // qbar = sum_h q_h in two int8 halves: qbar64 (fp64), sq = fl32(max|qbar64|
    // / 127), qi1 = clamp(rint(qbar64 / sq), +-127), qi2 = clamp(rint((qbar64 -
    // sq qi1) / (sq / 128)), +-127), so qbar ~ sf Q with sf = sq / 128 and
    // Q = 128 qi1 + qi2.  For every candidate c with sketch (s, code, rn, kn)
    // of t_c = kbar_c - m (m the unit's centre, common to all c) and
    // z_c = qbar . t_c = x_c - qbar . m:
    //   z_c - sf s (Q . code) = qbar . (t_c - s code) + (qbar - sf Q) . (s code)
    //   |z_c - sf s (Q . code)| <= qn rn + rq kn,
    // qn >= ||qbar||_2, rq >= ||qbar - sf Q||_2 (both including the fp64
    // rounding of qbar64, at most (G-1) 2^-53 sum_h |q_h| per element).
    if (warp == 0) {
        constexpr int E = D / 32;
        double qb[E], qa[E];
        float amax = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) { qb[e] = 0.0; qa[e] = 0.0; }
#pragma unroll
        for (int h = 0; h < G; ++h) {
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const float f = to_f32<T>(qg[(size_t)h * D + lane * E + e]);
                s_qh[h * D + lane * E + e] = f;
                qb[e] += (double)f;
                qa[e] += (double)fabsf(f);
            }
        }
#pragma unroll
        for (int e = 0; e < E; ++e) amax = fmaxf(amax, (float)fabs(qb[e]));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        // amax may round below max|qbar64|: the clamps keep the codes in range
        const float sq = amax / 127.0f;
        const float sf = sq * 0x1p-7f;                 // exact
        double r2 = 0.0, n2 = 0.0, a2 = 0.0;
        uint32_t p1 = 0, p2 = 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            int c1 = 0, c2 = 0;
            if (sq > 0.f) {
                c1 = max(-127, min(127, (int)rint(qb[e] / (double)sq)));
                c2 = max(-127, min(127, (int)rint((qb[e] - (double)sq * c1) / (double)sf)));
            }
            p1 |= (uint32_t)(c1 & 0xff) << (8 * e);
            p2 |= (uint32_t)(c2 & 0xff) << (8 * e);
            const double r = qb[e] - (double)sf * (double)(128 * c1 + c2);
            r2 = fma(r, r, r2);
            n2 = fma(qb[e], qb[e], n2);
            a2 = fma(qa[e], qa[e], a2);
        }
        if constexpr (E == 4) {
            *reinterpret_cast<uint32_t*>(s_qi + lane * E) = p1;
            *reinterpret_cast<uint32_t*>(s_qi + D + lane * E) = p2;
        } else {
            *reinterpret_cast<uint16_t*>(s_qi + lane * E) = (uint16_t)p1;
            *reinterpret_cast<uint16_t*>(s_qi + D + lane * E) = (uint16_t)p2;
        }
        r2 = group_sum_f64<32>(r2);
        n2 = group_sum_f64<32>(n2);
        a2 = group_sum_f64<32>(a2);
        if (lane == 0) {
            // r is one fp64 rounding away from exact: 2^-52 ||qbar64|| covers it
            const double m = 1.0 + 0x1p-40;
            const double slack = (double)(G > 1 ? G - 1 : 0) * 0x1p-52 * sqrt(a2) * m;
            s_qc[0] = sf;
            s_qc[1] = __double2float_ru(sqrt(n2) * m + slack);
            s_qc[2] = __double2float_ru(sqrt(r2) * m + 0x1p-52 * sqrt(n2) * m + slack);
        }
    }
    __syncthreads();
    // the finish of split units coded the query while the scan ran; the
    // scan's bounds are complete and visible after this
    if constexpr (PHASE == kPhFinish) asm volatile("griddepcontrol.wait;\n" ::: "memory");

    bool failed = false;
    {
        const uint4 qv1 = *reinterpret_cast<const uint4*>(s_qi + li * 16);
        const uint4 qv2 = *reinterpret_cast<const uint4*>(s_qi + D + li * 16);
        const float sf = s_qc[0], qn = s_qc[1], rq = s_qc[2];
        // this warp's rows of a stage: warp * R * GPW + jj * GPW + gsub, jj < R
        const int wrow = warp * R * GPW + gsub;
        int j = 0;
        for (; j < nst; ++j) {
            const bool ok = mbar_wait(bar0 + 8 * (j % Ring::kStages), (uint32_t)(j / Ring::kStages) & 1u);
            const unsigned char* sb = s_ring + (size_t)(j % Ring::kStages) * Ring::kStageBytes;
            const int rows_j = min(Ring::SR, nrows - j * Ring::SR);
            // integer dot products Q . code of the lane's 16 codes (exact;
            // |Q . code| < 2^14 * 127 * D < 2^31)
            int x[R];
#pragma unroll
            for (int jj = 0; jj < R; ++jj) {
                const int rr = wrow + jj * GPW;
                const uint4 w = (rr < rows_j) ? *reinterpret_cast<const uint4*>(sb + (size_t)rr * D + li * 16)
                                              : make_uint4(0, 0, 0, 0);
                const int hi = __dp4a((int)w.x, (int)qv1.x, __dp4a((int)w.y, (int)qv1.y,
                               __dp4a((int)w.z, (int)qv1.z, __dp4a((int)w.w, (int)qv1.w, 0))));
                const int lo = __dp4a((int)w.x, (int)qv2.x, __dp4a((int)w.y, (int)qv2.y,
                               __dp4a((int)w.z, (int)qv2.z, __dp4a((int)w.w, (int)qv2.w, 0))));
                x[jj] = 128 * hi + lo;
            }
            // transposed reduction over the CPR lanes of the group: each of the
            // first log2(R) levels keeps half of the remaining rows, so the lane
            // bits select one row; the remaining levels add across lanes
            int row = 0;
#pragma unroll
            for (int half = R / 2, off = CPR / 2; half > 0; half >>= 1, off >>= 1) {
                const int bit = (li & off) ? 1 : 0;
#pragma unroll
                for (int jj = 0; jj < half; ++jj) {
                    const int send = bit ? x[jj] : x[jj + half];
                    const int keep = bit ? x[jj + half] : x[jj];
                    x[jj] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
                row = 2 * row + bit;
            }
#pragma unroll
            for (int off = CPR / (2 * R); off > 0; off >>= 1) x[0] += __shfl_xor_sync(0xffffffffu, x[0], off);
            const int rr = wrow + row * GPW;
            const int r = r0 + j * Ring::SR + rr;
            const bool owner = (li & (CPR / R - 1)) == 0 && rr < rows_j;
            // score interval: y = fl(fl(sf s) fl(y_int)) is three roundings,
            // within 2^-21 |y| of sf s y_int; 2^-100 covers an underflow of
            // sf s; every bound term is rounded up
            uint32_t lkey = 0u, ukey = 0u;
            if (owner) {
                const float4 m = *reinterpret_cast<const float4*>(sb + Ring::kCodeBytes + (size_t)rr * 16);
                const float y = __fmul_rn(__fmul_rn(sf, m.x), (float)x[0]);
                const float e = __fadd_ru(__fmaf_ru(qn, m.y, __fmaf_ru(rq, m.z, __fmul_ru(0x1p-21f, fabsf(y)))),
                                          0x1p-100f);
                const float lo = __fsub_rd(y, e), up = __fadd_ru(y, e);
                lkey = fkey(lo);
                ukey = fkey(up);
                if (local) {
                    s_ukeys[r] = ukey;
                    s_lkeys[r] = lkey;
                } else {
                    sc_lo[r] = lo;
                    sc_up[r] = up;
                }
            }
            // the stage is free once every warp has scored it
            if (__syncthreads_or(!ok)) { failed = true; break; }
            if (threadIdx.x == 0) issue(j + Ring::kStages);
            // warp 0 reconverges here: its other lanes must not spin on the
            // next stage's barrier while lane 0 still has the copy to issue
            __syncwarp();
        }
        if (failed) {
            // give the copies still in flight a bounded time to land, then
            // return with the unit's outputs marked invalid
            if (threadIdx.x == 0) {
                atomicAdd(io.timeouts, 1u);
                for (int jj = j; jj < min(nst, j + Ring::kStages); ++jj)
                    mbar_wait(bar0 + 8 * (jj % Ring::kStages), (uint32_t)(jj / Ring::kStages) & 1u, kDrainNs);
            }
        }
    }
    if (PHASE == kPhScan) {
        // the finish kernel learns of an abandoned wait from the unit's
        // (otherwise unused) selection ticket
        if (failed && threadIdx.x == 0) atomicAdd(cnt + u, 1u);
        return res;
    }
    if (failed) {
        int32_t* out_idx = blk_idx + (size_t)u * kb_stride;
        for (int i = threadIdx.x; i < kb_stride; i += NT) out_idx[i] = -1;
        if (threadIdx.x == 0) {
            samp_count[u] = 0;
            if (n_rescored != nullptr) n_rescored[u] = -1;
        }
        // keep the unit's completion count consistent for the next call
        if (!local && last_cta_of_unit(cnt + u, nss)) reset_counter(cnt + u);
        return res;
    }

    // counters of the group top-k (zero before the barrier that ends the gather)
    if (threadIdx.x == 0) {
        s_digit = 0;
        s_rem = 0;
    }
    // ---- gather the unit's keys --------------------------------------------------
    uint32_t* lk = s_lkeys;            // lower-bound keys: the ranking
    uint32_t* uk = s_ukeys;            // upper-bound keys: band membership
    if (local) {
        __syncthreads();
    } else {
        if (PHASE == kPhAll && !last_cta_of_unit(cnt + u, nss)) return res;
        if (PHASE == kPhFinish) {
            __shared__ unsigned s_bad;
            if (threadIdx.x == 0) s_bad = __ldcg(cnt + u);
            __syncthreads();
            if (s_bad != 0u) {               // a scan CTA of the unit gave up a wait
                int32_t* out_idx = blk_idx + (size_t)u * kb_stride;
                for (int i = threadIdx.x; i < kb_stride; i += NT) out_idx[i] = -1;
                if (threadIdx.x == 0) {
                    samp_count[u] = 0;
                    if (n_rescored != nullptr) n_rescored[u] = -1;
                    cnt[u] = 0u;
                }
                return res;
            }
        }
        // orderable keys, staged once: shared memory when they fit, else in
        // place over the unit's bounds in the workspace (each thread rewrites
        // only the entries it read)
        if (n > KEYS) {
            lk = reinterpret_cast<uint32_t*>(sc_lo);
            uk = reinterpret_cast<uint32_t*>(sc_up);
        }
        for (int i0 = 0; i0 < n; i0 += 4 * NT) {
            float ylo[4], yup[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = i0 + j * NT + threadIdx.x;
                ylo[j] = i < n ? ldcg(sc_lo + i) : 0.f;
                yup[j] = i < n ? ldcg(sc_up + i) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = i0 + j * NT + threadIdx.x;
                if (i < n) {
                    lk[i] = fkey(ylo[j]);
                    uk[i] = fkey(yup[j]);
                }
            }
        }
        __syncthreads();
    }

    // ---- top-k of the unit ------------------------------------------------------------
    int32_t* out_idx = blk_idx + (size_t)u * kb_stride;
    int rescored = 0;
    bool sorted_smem = false;          // the chosen indices are also in s_sorted
    if (kk > 0 && kk < n) {
        if (threadIdx.x == 0) s_nb = 0;        // band counter (barriers follow on every path)
        auto k32 = [&](int i) -> uint32_t { return lk[i]; };
        // the ranked list s_list[0..kk) comes from the group top-k (kk up to
        // LISTN) or, for kk <= 32 when it has too many candidates, from the
        // per-warp lists; otherwise a radix select finds thr
        const bool grp = kk <= LISTN && n <= KEYS;
        uint32_t thr = 0u;
        int need = 0;
        bool listed = false;            // band already listed (group path)
        bool have_list = false;         // s_list[0..kk) holds the top kk in rank order
        if (grp) {
            listed = topk_band<NT, KEYS, CC, BLOCKB>(lk, uk, n, kk, s_list, s_cand, s_u, sw,
                                                     reinterpret_cast<unsigned*>(&s_rem),
                                   s_bidx, &s_nb);
            have_list = listed;
            if (!listed && kk <= kWarpTopK) {
                warp_topk<NT, KEYS>(lk, n, kk, s_cand, s_list);
                have_list = true;
            }
        }
        if (have_list) {
            thr = (uint32_t)(s_list[kk - 1] >> 32);
            if (kk > kWarpTopK) {
                // the top kk's keys equal to thr are the lowest-index ones
                // among all keys equal to thr: emit_topk takes that many
                int c = 0;
                for (int r = threadIdx.x; r < kk; r += NT) c += ((uint32_t)(s_list[r] >> 32) == thr) ? 1 : 0;
                need = block_sum<NT>(c, sw);
            }
        } else {
            radix_select<NT, uint32_t>(k32, n, kk, &thr, &need, hist, &s_digit, &s_rem);
        }
        // thr = the kk-th largest lower bound.  A candidate whose upper bound is
        // below it is beaten strictly by kk others, so the exact top kk lies
        // in the band {upper >= thr}, which contains the kk best lower bounds.
        // Unless listed already, one pass counts the band and lists its
        // members (the first kBandCap of them, in no particular order) in s_bidx.
        if (!listed) {
            for (int i0 = warp * 32; i0 < n; i0 += NT) {
                const int i = i0 + lane;
                const bool in = i < n && uk[i] >= thr;
                const unsigned m = __ballot_sync(0xffffffffu, in);
                if (m != 0u) {
                    int base = 0;
                    if (lane == 0) base = atomicAdd(&s_nb, __popc(m));
                    base = __shfl_sync(0xffffffffu, base, 0);
                    if (in) {
                        const int pos = base + __popc(m & ((1u << lane) - 1u));
                        if (pos < kBandCap) s_bidx[pos] = i;
                    }
                }
            }
        }
        __syncthreads();
        const int band = s_nb;
        if (band == kk) {
            if (have_list && kk <= kWarpTopK) {
                emit_sorted_list(s_list, kk, sg.c_lo, out_idx, s_sorted);
                sorted_smem = true;
            }
            else emit_topk<NT, uint32_t>(k32, n, thr, need, kk, sg.c_lo, out_idx, sw);
        } else {
            // ambiguous: rescore the band members exactly and take the top k
            // among them by (x desc, index asc)
            rescored = band;
            const T* bm = blk_mean + ((size_t)u * nb + sg.c_lo) * D;
            if (band <= 32) {
                rescore_members<T, D, G, NW>(bm, s_bidx, band, s_qh, s_bx);
                __syncthreads();
                // one warp: lane j ranks member j, then the chosen are sorted by index
                if (warp == 0) {
                    const bool live = lane < band;
                    const double xj = live ? s_bx[lane] : -INFINITY;
                    const int ij = live ? s_bidx[lane] : 0x7fffffff;
                    int rank = 0;
                    for (int m = 0; m < band; ++m) {
                        const double xm = __shfl_sync(0xffffffffu, xj, m);
                        const int im = __shfl_sync(0xffffffffu, ij, m);
                        rank += (xm > xj || (xm == xj && im < ij)) ? 1 : 0;
                    }
                    const int v = warp_sort_asc((live && rank < kk) ? ij : 0x7fffffff);
                    if (lane < kk) {
                        out_idx[lane] = sg.c_lo + v;
                        s_sorted[lane] = sg.c_lo + v;
                    }
                }
                sorted_smem = true;
            } else if (band <= kBandCap) {
                // several rounds of members: their rows into L2 first
                if (band > 2 * NW) {
                    for (int j = threadIdx.x; j < band; j += NT) {
                        const char* r = reinterpret_cast<const char*>(bm + (size_t)s_bidx[j] * D);
#pragma unroll
                        for (int o = 0; o < (int)(D * sizeof(T)); o += 128)
                            asm volatile("prefetch.global.L2 [%0];" ::"l"(r + o));
                    }
                }
                rescore_members<T, D, G, NW>(bm, s_bidx, band, s_qh, s_bx);
                __syncthreads();
                for (int j = threadIdx.x; j < band; j += NT) {
                    const double xj = s_bx[j];
                    const int ij = s_bidx[j];
                    int rank = 0;
                    for (int m = 0; m < band; ++m) {
                        const double xm = s_bx[m];
                        rank += (xm > xj || (xm == xj && s_bidx[m] < ij)) ? 1 : 0;
                    }
                    s_bsel[j] = rank < kk ? 1 : 0;
                }
                __syncthreads();
                for (int j = threadIdx.x; j < band; j += NT) {
                    if (!s_bsel[j]) continue;
                    const int ij = s_bidx[j];
                    int pos = 0;
                    for (int m = 0; m < band; ++m) pos += (s_bsel[m] && s_bidx[m] < ij) ? 1 : 0;
                    if (pos < kk) {
                        out_idx[pos] = sg.c_lo + ij;
                        if (kk <= kWarpTopK) s_sorted[pos] = sg.c_lo + ij;
                    }
                }
                sorted_smem = kk <= kWarpTopK;
            } else {
                // very wide band (many near-equal scores): 64-bit keys for every
                // candidate in the workspace (0 outside the band), radix select
                __syncthreads();
                unsigned long long* xk = xkey + (size_t)u * n;
                for (int i = warp; i < n; i += NW) {
                    unsigned long long key = 0ull;
                    if (uk[i] >= thr) {                             // warp-uniform branch
                        const T* rows[1] = {bm + (size_t)i * D};
                        const bool live[1] = {true};
                        double x[1];
                        exact_scores<T, D, G, 1>(rows, live, s_qh, x);
                        key = dkey(x[0]);
                    }
                    if (lane == 0) xk[i] = key;
                }
                __threadfence_block();
                __syncthreads();
                auto k64 = [&](int i) -> unsigned long long { return xk[i]; };
                unsigned long long thr64;
                int need64;
                radix_select<NT, unsigned long long>(k64, n, kk, &thr64, &need64, hist, &s_digit, &s_rem);
                emit_topk<NT, unsigned long long>(k64, n, thr64, need64, kk, sg.c_lo, out_idx, sw);
            }
        }
    } else if (kk > 0) {       // every candidate is chosen
        for (int i = threadIdx.x; i < kk; i += NT) {
            out_idx[i] = sg.c_lo + i;
            if (kk <= kWarpTopK) s_sorted[i] = sg.c_lo + i;
        }
        sorted_smem = kk <= kWarpTopK;
    }
    for (int i = kk + threadIdx.x; i < kb_stride; i += NT) out_idx[i] = -1;
    if (n_rescored != nullptr && threadIdx.x == 0) n_rescored[u] = rescored;
    __threadfence_block();
    __syncthreads();

    // ---- tail draws -------------------------------------------------------------
    const int bdraw = unit_draws<NT>(sg, sorted_smem ? s_sorted : out_idx, sample_b, sample_cap, seed, b, g, step,
                                     u, samp_idx, samp_count, sm.samp, sm.samp_cap, G, io.per_head, Hq);
    if (!local) reset_counter(cnt + u);
    res.done = true;
    res.sorted_smem = sorted_smem;
    res.bdraw = bdraw;
    return res;
}


}  // namespace sa
