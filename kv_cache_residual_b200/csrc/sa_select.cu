// Per-step selection (vAttention, Method, overall framework: I_f = sink +
// local window + top-k; the top-k ranks 16-token blocks by their mean key, the
// block selection of Quest / ArkVale that RESA wraps).
//
// k_select: grid (nss, B*Hkv)
//   scan  : every CTA scores a slice of the unit's candidate blocks in fp32,
//           y_c = qbar . kbar_c with qbar = sum_{h in group} q_h, and stores y
//           in the workspace (the HBM-bound part: one read of the summaries);
//   top-k : the CTA that finishes the unit last (completion ticket, no wait)
//           finds the k-th largest y by a 4 x 8-bit radix select, takes ties at
//           the threshold by lowest block index, and checks the rounding bound
//           |y_c - x_c| <= E (x_c the exact score): every candidate with
//           y >= y_(k) - 2E may belong to the exact top-k; if more than k do,
//           those are rescored in fp64 and the top-k is re-taken over 64-bit
//           keys.  The decision is therefore the fp64 one.
//   draws : tail positions for the sampling estimator (SplitMix64 counters).
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int kSmemKeys = 4096;     // candidate keys staged in shared memory (16 KB)
constexpr int kBandCap = 512;       // band members ranked in shared memory

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

// Block-wide exclusive scan of one int per thread (thread order).  Returns
// this thread's exclusive prefix; *total gets the sum.  Uses sw[kWarps+1].
__device__ __forceinline__ int block_exscan(int v, int* sw, int* total) {
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
        for (int w = 0; w < kWarps; ++w) { const int c = sw[w]; sw[w] = s; s += c; }
        sw[kWarps] = s;
    }
    __syncthreads();
    const int r = sw[warp] + inc - v;
    *total = sw[kWarps];
    __syncthreads();
    return r;
}

__device__ __forceinline__ int block_sum(int v, int* sw) {
    int tot;
    (void)block_exscan(v, sw, &tot);
    return tot;
}

// Radix select (MSB first, 8 bits per pass) of the kk-th largest key among
// key(0..n-1).  On return *thr is that key and *need is how many of the keys
// equal to it belong to the top kk (the rest of the top kk is strictly above).
template <typename KT, typename KeyFn>
__device__ void radix_select(KeyFn key, int n, int kk, KT* thr, int* need, unsigned* hist,
                             int* s_digit, int* s_rem) {
    KT prefix = 0, mask = 0;
    int rem = kk;
    const int lane = threadIdx.x & 31;
    for (int shift = (int)sizeof(KT) * 8 - 8; shift >= 0; shift -= 8) {
        hist[threadIdx.x] = 0;   // kThreads == 256 bins
        __syncthreads();
        // warp-aggregated: lanes with equal digits add once (scores share their
        // top bits, so per-lane atomics would serialise on a few bins)
        for (int i0 = 0; i0 < n; i0 += kThreads) {
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
template <typename KT, typename KeyFn>
__device__ void emit_topk(KeyFn key, int n, KT thr, int need, int kk, int c_lo, int32_t* out_idx, int* sw) {
    const int C = (n + kThreads - 1) / kThreads;
    const int i0 = min(n, (int)threadIdx.x * C), i1 = min(n, i0 + C);
    int eqc = 0;
    for (int i = i0; i < i1; ++i) eqc += (key(i) == thr) ? 1 : 0;
    int tot;
    const int eq_before = block_exscan(eqc, sw, &tot);
    int selc = 0, r = eq_before;
    for (int i = i0; i < i1; ++i) {
        const KT kx = key(i);
        if (kx > thr) ++selc;
        else if (kx == thr) { if (r < need) ++selc; ++r; }
    }
    int p = block_exscan(selc, sw, &tot);
    r = eq_before;
    for (int i = i0; i < i1; ++i) {
        const KT kx = key(i);
        bool take = kx > thr;
        if (kx == thr) { take = r < need; ++r; }
        if (take && p < kk) out_idx[p++] = c_lo + i;
    }
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads)
k_select(const T* __restrict__ q, const T* __restrict__ blk_mean, const float* __restrict__ kbar_absmax,
         int Hq, int Hkv, int L, SetGeom sg, int rows, int nss,
         float* __restrict__ scores, unsigned long long* __restrict__ xkey, unsigned char* __restrict__ flags_ws,
         unsigned* __restrict__ cnt, int kb_stride, int32_t* __restrict__ blk_idx,
         int32_t* __restrict__ samp_idx, int32_t* __restrict__ samp_count, int32_t* __restrict__ n_rescored,
         int sample_b, int sample_cap, unsigned long long seed, int step) {
    using Gm = Geom<T, D>;
    constexpr int EPC = Gm::EPC, CPR = Gm::CPR, NG = Gm::NG;
    __shared__ unsigned hist[kThreads];
    __shared__ int sw[kWarps + 1];
    __shared__ int s_digit, s_rem, s_band;
    __shared__ double s_q64[D];
    __shared__ float s_qa[kWarps];
    __shared__ uint32_t s_keys[kSmemKeys];
    __shared__ int s_nb;
    __shared__ int s_bidx[kBandCap];
    __shared__ double s_bx[kBandCap];
    __shared__ unsigned char s_bsel[kBandCap];

    const int u = blockIdx.y, split = blockIdx.x;
    const int b = u / Hkv, g = u - b * Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int gi = warp * Gm::GPW + lane / CPR, li = lane % CPR;
    const int nb = L / 16;
    const int n = sg.n_cand, kk = sg.kk;
    const T* qg = q + ((size_t)b * Hq + (size_t)g * G) * D;
    float* sc = scores + (size_t)u * (n > 0 ? n : 1);

    // ---- scan: fp32 scores of this CTA's slice -------------------------------
    {
        float qb[EPC];
#pragma unroll
        for (int e = 0; e < EPC; ++e) qb[e] = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float f[EPC];
            unpack<T>(ld_nc16(qg + (size_t)h * D + li * EPC), f);
#pragma unroll
            for (int e = 0; e < EPC; ++e) qb[e] += f[e];
        }
        const T* base = blk_mean + ((size_t)u * nb + sg.c_lo) * D + li * EPC;
        const int r0 = split * rows, r1 = min(n, r0 + rows);
        const int gsub = lane / CPR;
        // warp-uniform loop: a warp step covers 4 x GPW rows (4 per lane group);
        // the next step's rows are loaded before this step's are reduced, so 8
        // rows per lane group are in flight; rows past the end load nothing
        auto load4 = [&](int wr, uint4 (&w)[4]) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = wr + j * Gm::GPW + gsub;
                w[j] = (r < r1) ? ld_stream16(base + (size_t)r * D) : make_uint4(0, 0, 0, 0);
            }
        };
        int wr = r0 + warp * 4 * Gm::GPW;
        uint4 cur[4];
        load4(wr, cur);
        for (; wr < r1; wr += 4 * NG) {
            uint4 nxt[4];
            load4(wr + 4 * NG, nxt);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = wr + j * Gm::GPW + gsub;
                float f[EPC];
                unpack<T>(cur[j], f);
                float x = 0.f;
#pragma unroll
                for (int e = 0; e < EPC; ++e) x = fmaf(qb[e], f[e], x);
                x = group_sum<CPR>(x);
                if (li == 0 && r < r1) sc[r] = x;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) cur[j] = nxt[j];
        }
    }
    if (!last_cta_of_unit(cnt + u, nss)) return;

    // ---- top-k of the unit (last CTA) ------------------------------------------
    int32_t* out_idx = blk_idx + (size_t)u * kb_stride;
    int rescored = 0;
    if (kk > 0 && kk < n) {
        // orderable keys, staged once: shared memory when they fit, else in
        // place over the unit's scores in the workspace
        uint32_t* keys = (n <= kSmemKeys) ? s_keys : reinterpret_cast<uint32_t*>(sc);
        for (int i0 = 0; i0 < n; i0 += 4 * kThreads) {
            float y[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = i0 + j * kThreads + threadIdx.x;
                y[j] = i < n ? ldcg(sc + i) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = i0 + j * kThreads + threadIdx.x;
                if (i < n) keys[i] = fkey(y[j]);
            }
        }
        __syncthreads();
        auto k32 = [&](int i) -> uint32_t { return keys[i]; };
        uint32_t thr;
        int need;
        radix_select<uint32_t>(k32, n, kk, &thr, &need, hist, &s_digit, &s_rem);
        // rounding bound of the fp32 scan: |y - x| <= (G + D) 2^-23 sum_i qa_i * max|kbar|
        float qa = 0.f;
        for (int i = threadIdx.x; i < D; i += kThreads) {
            float s = 0.f;
            for (int h = 0; h < G; ++h) s += fabsf(to_f32<T>(qg[(size_t)h * D + i]));
            qa += s;
        }
        for (int off = 16; off > 0; off >>= 1) qa += __shfl_xor_sync(0xffffffffu, qa, off);
        if (lane == 0) s_qa[warp] = qa;
        __syncthreads();
        float qsum = 0.f;
        for (int w = 0; w < kWarps; ++w) qsum += s_qa[w];
        const float E = (float)(G + D) * 0x1p-23f * qsum * kbar_absmax[u] * 1.0001f + 0x1p-100f;
        const uint32_t lo_key = fkey(fkey_inv(thr) - 2.f * E);
        int band = 0;
        for (int i = threadIdx.x; i < n; i += kThreads) band += (keys[i] >= lo_key) ? 1 : 0;
        band = block_sum(band, sw);
        if (band == kk) {
            emit_topk<uint32_t>(k32, n, thr, need, kk, sg.c_lo, out_idx, sw);
        } else {
            // ambiguous: the exact top-k lies inside the band; rescore the band
            // members in fp64 and take the top k among them by (x desc, index asc)
            rescored = band;
            for (int i = threadIdx.x; i < D; i += kThreads) {
                double s = 0.0;
                for (int h = 0; h < G; ++h) s += (double)to_f32<T>(qg[(size_t)h * D + i]);
                s_q64[i] = s;
            }
            const T* bm = blk_mean + ((size_t)u * nb + sg.c_lo) * D;
            auto dot64 = [&](int i) -> double {      // warp-collective fp64 score of candidate i
                double x = 0.0;
                for (int e = lane; e < D; e += 32) x += s_q64[e] * (double)to_f32<T>(bm[(size_t)i * D + e]);
                return group_sum_f64<32>(x) + 0.0;  // -0 -> +0
            };
            if (band <= kBandCap) {
                if (threadIdx.x == 0) s_nb = 0;
                __syncthreads();
                for (int i = threadIdx.x; i < n; i += kThreads)
                    if (keys[i] >= lo_key) s_bidx[atomicAdd(&s_nb, 1)] = i;
                __syncthreads();
                for (int j = warp; j < band; j += kWarps) {
                    const double x = dot64(s_bidx[j]);
                    if (lane == 0) s_bx[j] = x;
                }
                __syncthreads();
                for (int j = threadIdx.x; j < band; j += kThreads) {
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
                for (int j = threadIdx.x; j < band; j += kThreads) {
                    if (!s_bsel[j]) continue;
                    const int ij = s_bidx[j];
                    int pos = 0;
                    for (int m = 0; m < band; ++m) pos += (s_bsel[m] && s_bidx[m] < ij) ? 1 : 0;
                    if (pos < kk) out_idx[pos] = sg.c_lo + ij;
                }
            } else {
                // very wide band (many near-equal scores): 64-bit keys for every
                // candidate in the workspace (0 outside the band), radix select
                __syncthreads();
                unsigned long long* xk = xkey + (size_t)u * n;
                for (int i = warp; i < n; i += kWarps) {
                    unsigned long long key = 0ull;
                    if (keys[i] >= lo_key) key = dkey(dot64(i));   // warp-uniform branch
                    if (lane == 0) xk[i] = key;
                }
                __threadfence_block();
                __syncthreads();
                auto k64 = [&](int i) -> unsigned long long { return xk[i]; };
                unsigned long long thr64;
                int need64;
                radix_select<unsigned long long>(k64, n, kk, &thr64, &need64, hist, &s_digit, &s_rem);
                emit_topk<unsigned long long>(k64, n, thr64, need64, kk, sg.c_lo, out_idx, sw);
            }
        }
    } else if (kk > 0) {       // every candidate is chosen
        for (int i = threadIdx.x; i < kk; i += kThreads) out_idx[i] = sg.c_lo + i;
    }
    for (int i = kk + threadIdx.x; i < kb_stride; i += kThreads) out_idx[i] = -1;
    if (n_rescored != nullptr && threadIdx.x == 0) n_rescored[u] = rescored;
    __threadfence_block();
    __syncthreads();

    // ---- tail draws -------------------------------------------------------------
    const int nt = sg.n_t;
    const int bdraw = (nt > 0) ? min(sample_b, sample_cap) : 0;
    if (threadIdx.x == 0) samp_count[u] = bdraw;
    if (bdraw > 0) {
        const uint64_t key = unit_key(seed, (uint64_t)b, (uint64_t)g, (uint64_t)step);
        int32_t* out_s = samp_idx + (size_t)u * sample_cap;
        for (int i = threadIdx.x; i < bdraw; i += kThreads) {
            const int r = (int)draw_rank(key, (uint32_t)i, (uint32_t)nt);
            // tail = [s_eff, L - w_eff) minus the chosen blocks; chosen block j
            // starts after g_j = 16 c_j - s_eff - 16 j tail tokens
            int lo_j = 0, hi_j = kk;             // count of j with g_j <= r
            while (lo_j < hi_j) {
                const int mid = (lo_j + hi_j) >> 1;
                const int gj = 16 * out_idx[mid] - sg.s_eff - 16 * mid;
                if (gj <= r) lo_j = mid + 1; else hi_j = mid;
            }
            out_s[i] = sg.s_eff + r + 16 * lo_j;
        }
    }
    reset_counter(cnt + u);
}

template <typename T, int D, int G>
static cudaError_t select_t(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s) {
    char* ws = a.ws;
    k_select<T, D, G><<<dim3(p.nss, d.U()), kThreads, 0, s>>>(
        reinterpret_cast<const T*>(a.q), reinterpret_cast<const T*>(a.st.blk_mean), a.st.kbar_absmax,
        d.Hq, d.Hkv, d.L, p.g, p.rows_s, p.nss,
        reinterpret_cast<float*>(ws + p.off_scores), reinterpret_cast<unsigned long long*>(ws + p.off_xkey),
        reinterpret_cast<unsigned char*>(ws + p.off_flags), reinterpret_cast<unsigned*>(ws + p.off_cnt),
        a.sp.k_blocks, a.sel.blk_idx, a.sel.samp_idx, a.sel.samp_count, a.sel.n_rescored,
        a.sp.sample_b, a.sp.sample_cap, (unsigned long long)a.sp.seed, a.sp.step);
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t select_g(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s) {
    switch (d.G) {
        case 1: return select_t<T, D, 1>(d, p, a, s);
        case 2: return select_t<T, D, 2>(d, p, a, s);
        case 4: return select_t<T, D, 4>(d, p, a, s);
        case 8: return select_t<T, D, 8>(d, p, a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_select(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s) {
    if (d.bf16) return d.d == 128 ? select_g<__nv_bfloat16, 128>(d, p, a, s) : select_g<__nv_bfloat16, 64>(d, p, a, s);
    return d.d == 128 ? select_g<float, 128>(d, p, a, s) : select_g<float, 64>(d, p, a, s);
}

}  // namespace sa
