// Per-step selection by the two alternative block scores (the selectors the
// RESA page's related work builds on, and the GQA alternative to scoring a
// KV head by its group's summed query):
//   SA_SCORE_MEAN_MAX  score_c = max_{h in group} q_h . kbar_c
//   SA_SCORE_QUEST     score_c = sum_h sum_e max(q_he min_ce, q_he max_ce),
//                      min / max the elementwise key bounds of block c
//                      (Quest's criticality bound: for each head an upper
//                      bound of q_h . K_j over the block's tokens)
// Both rank by (score desc, block index asc) on the exact score rounded once,
// exactly as the default score does.
//
// k_select_var: one CTA of 256 threads per unit.
//   scan  : every candidate's summaries (one bf16 / fp32 row for MEAN_MAX,
//           the min and the max row for QUEST) are read once with 16-byte
//           loads, a lane group per row; fp32 products summed per head with
//           a running sum of their magnitudes A, so the exact score lies in
//           [y - e, y + e], e = A 2^-16 (MEAN_MAX: a length-d dot product
//           errs by at most gamma_d A < 2^-17 A at d <= 128) or A 2^-14
//           (QUEST: G d <= 1024 terms, gamma < 2^-14), plus 2^-100 for
//           underflow, all rounded outward.  MEAN_MAX takes the max over
//           heads of both ends.  Orderable 32-bit keys of both ends stay in
//           shared memory (n_cand <= kVarKeys).
//   top-k : radix select of the k-th largest lower key thr; the band
//           {upper >= thr} holds the exact top k.  A band of exactly k is the
//           answer; otherwise the band is rescored exactly (products exact in
//           fp64, double-double sums, one rounding; MEAN_MAX per head, then
//           the max) and ranked by (x desc, index asc); a band wider than
//           kBandCap gets 64-bit exact keys in the workspace and a second
//           radix select.
//   draws : unit_draws, as the default selection.
#include "sa_select_core.cuh"

namespace sa {

constexpr int kVarKeys = 16384;          // candidates per unit held in shared memory

struct VarIo {
    const void* q;
    const void* rows_a;                  // MEAN_MAX: block means; QUEST: block minima
    const void* rows_b;                  // QUEST: block maxima
    int Hq, Hkv, ld;
    SetGeom sg;
    unsigned long long* xkey;            // [U][n_cand] exact keys (very wide bands)
    int kb_stride;
    int32_t* blk_idx;
    int32_t* samp_idx;
    int32_t* samp_count;
    int32_t* n_rescored;
    int sample_b, sample_cap;
    unsigned long long seed;
    int step;
    int per_head;
};

// Exact score of one candidate (warp-collective; every lane gets it): the
// products of bf16 / fp32 values are exact in fp64 and are added in
// double-double, the lanes combined the same way, the two parts rounded
// together (as exact_scores in sa_select_core.cuh).
template <typename T, int D, int G, int SCORE>
__device__ __forceinline__ double exact_var(const T* ra, const T* rb, const float* s_qh) {
    const int lane = threadIdx.x & 31;
    constexpr int E = D / 32;
    float ka[E], kb[E];
#pragma unroll
    for (int i = 0; i < E; ++i) {
        ka[i] = to_f32<T>(ra[lane + 32 * i]);
        kb[i] = SCORE == SA_SCORE_QUEST ? to_f32<T>(rb[lane + 32 * i]) : 0.f;
    }
    if constexpr (SCORE == SA_SCORE_MEAN_MAX) {
        double best = -INFINITY;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            double s = 0.0, c = 0.0;
#pragma unroll
            for (int i = 0; i < E; ++i)
                two_sum_acc(s, c, __dmul_rn((double)s_qh[h * D + lane + 32 * i], (double)ka[i]));
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const double so = __shfl_xor_sync(0xffffffffu, s, off);
                const double co = __shfl_xor_sync(0xffffffffu, c, off);
                two_sum_acc(s, c, so);
                c = __dadd_rn(c, co);
            }
            best = fmax(best, __dadd_rn(s, c) + 0.0);
        }
        return best;
    } else {
        double s = 0.0, c = 0.0;
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int i = 0; i < E; ++i) {
                const float qv = s_qh[h * D + lane + 32 * i];
                // max(q mn, q mx) = q mx when q >= 0 (mx >= mn), else q mn
                two_sum_acc(s, c, __dmul_rn((double)qv, (double)(qv >= 0.f ? kb[i] : ka[i])));
            }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const double so = __shfl_xor_sync(0xffffffffu, s, off);
            const double co = __shfl_xor_sync(0xffffffffu, c, off);
            two_sum_acc(s, c, so);
            c = __dadd_rn(c, co);
        }
        return __dadd_rn(s, c) + 0.0;
    }
}

template <typename T, int D, int G, int SCORE>
__global__ void __launch_bounds__(kThreads)
k_select_var(VarIo io) {
    using Gm = Geom<T, D>;
    constexpr int EPC = Gm::EPC, CPR = Gm::CPR, GPW = Gm::GPW;
    constexpr int NT = kThreads, NW = kWarps;
    __shared__ __align__(16) unsigned hist[256];
    __shared__ int sw[NW + 1];
    __shared__ int misc[3];
    __shared__ __align__(16) float s_qh[G * D];
    __shared__ int s_sorted[kWarpTopK];
    __shared__ double s_bx[kBandCap];
    __shared__ int s_bidx[kBandCap];
    __shared__ unsigned char s_bsel[kBandCap];
    extern __shared__ __align__(16) uint32_t s_keys[];      // lower keys [n], then upper keys [n]
    // a decode launched as a programmatic dependent may start once every CTA
    // of this grid has begun; it waits for this grid before reading the result
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

    const int u = blockIdx.x;
    const int b = u / io.Hkv, g = u - b * io.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int li = lane % CPR, gsub = lane / CPR;
    const SetGeom& sg = io.sg;
    const int n = sg.n_cand, kk = sg.kk, nb = io.ld / 16;
    const T* qg = static_cast<const T*>(io.q) + ((size_t)b * io.Hq + (size_t)g * G) * D;
    for (int i = threadIdx.x; i < G * D; i += NT) s_qh[i] = to_f32<T>(qg[i]);
    int& s_digit = misc[0];
    int& s_rem = misc[1];
    int& s_nb = misc[2];
    if (threadIdx.x == 0) { s_digit = 0; s_rem = 0; s_nb = 0; }
    __syncthreads();
    uint32_t* lk = s_keys;
    uint32_t* uk = s_keys + n;

    // ---- scan: score intervals of every candidate --------------------------------
    const size_t row0 = (size_t)u * nb + sg.c_lo;
    const T* ra = static_cast<const T*>(io.rows_a) + row0 * D;
    const T* rb = SCORE == SA_SCORE_QUEST ? static_cast<const T*>(io.rows_b) + row0 * D : nullptr;
    float q[G][EPC];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < EPC; ++e) q[h][e] = s_qh[h * D + li * EPC + e];
    // rows in flight per lane group (measured: 16 single rows, 4 min / max
    // pairs; more pairs spill)
    constexpr int U4 = SCORE == SA_SCORE_QUEST ? 4 : 16;
    // the loop bound is the same for every lane of a warp (its GPW * U4 rows
    // start at rw), so the lane-group shuffles below always run on the full warp
    for (int rw = warp * GPW * U4; rw < n; rw += NW * GPW * U4) {
        uint4 wa[U4], wb[U4];
#pragma unroll
        for (int x = 0; x < U4; ++x) {
            const int r = rw + x * GPW + gsub;
            wa[x] = r < n ? ld_stream16(ra + (size_t)r * D + li * EPC) : make_uint4(0, 0, 0, 0);
            if constexpr (SCORE == SA_SCORE_QUEST)
                wb[x] = r < n ? ld_stream16(rb + (size_t)r * D + li * EPC) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int x = 0; x < U4; ++x) {
            float fa[EPC], fb[EPC];
            unpack<T>(wa[x], fa);
            if constexpr (SCORE == SA_SCORE_QUEST) unpack<T>(wb[x], fb);
            float y[G], a[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
                y[h] = 0.f;
                a[h] = 0.f;
#pragma unroll
                for (int e = 0; e < EPC; ++e) {
                    const float k = (SCORE == SA_SCORE_QUEST && q[h][e] >= 0.f) ? fb[e] : fa[e];
                    const float p = q[h][e] * k;
                    y[h] += p;
                    a[h] += fabsf(p);
                }
            }
#pragma unroll
            for (int off = CPR / 2; off > 0; off >>= 1)
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    y[h] += __shfl_xor_sync(0xffffffffu, y[h], off);
                    a[h] += __shfl_xor_sync(0xffffffffu, a[h], off);
                }
            const int r = rw + x * GPW + gsub;
            if (li == 0 && r < n) {
                float lo, up;
                if constexpr (SCORE == SA_SCORE_MEAN_MAX) {
                    lo = -INFINITY;
                    up = -INFINITY;
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        const float e = __fmaf_ru(a[h], 0x1p-16f, 0x1p-100f);
                        lo = fmaxf(lo, __fsub_rd(y[h], e));
                        up = fmaxf(up, __fadd_ru(y[h], e));
                    }
                } else {
                    float ys = 0.f, as = 0.f;
#pragma unroll
                    for (int h = 0; h < G; ++h) { ys += y[h]; as += a[h]; }
                    const float e = __fmaf_ru(as, 0x1p-14f, 0x1p-100f);
                    lo = __fsub_rd(ys, e);
                    up = __fadd_ru(ys, e);
                }
                lk[r] = fkey(lo);
                uk[r] = fkey(up);
            }
        }
    }
    __syncthreads();

    // ---- top-k -------------------------------------------------------------------------
    int32_t* out_idx = io.blk_idx + (size_t)u * io.kb_stride;
    int rescored = 0;
    bool sorted_smem = false;
    if (kk > 0 && kk < n) {
        auto k32 = [&](int i) -> uint32_t { return lk[i]; };
        uint32_t thr;
        int need;
        radix_select<NT, uint32_t>(k32, n, kk, &thr, &need, hist, &s_digit, &s_rem);
        // the band {upper >= thr}: its first kBandCap members listed, all counted
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
        __syncthreads();
        const int band = s_nb;
        if (band == kk) {
            emit_topk<NT, uint32_t>(k32, n, thr, need, kk, sg.c_lo, out_idx, sw);
        } else if (band <= kBandCap) {
            rescored = band;
            for (int j = warp; j < band; j += NW) {
                const int i = s_bidx[j];
                const double x = exact_var<T, D, G, SCORE>(ra + (size_t)i * D, rb + (size_t)(rb ? i : 0) * D, s_qh);
                if (lane == 0) s_bx[j] = x;
            }
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
            // very wide band: 64-bit exact keys for every candidate (0 outside
            // the band) in the workspace, radix select
            rescored = band;
            unsigned long long* xk = io.xkey + (size_t)u * n;
            for (int i = warp; i < n; i += NW) {
                unsigned long long key = 0ull;
                if (uk[i] >= thr)                               // warp-uniform
                    key = dkey(exact_var<T, D, G, SCORE>(ra + (size_t)i * D, rb + (size_t)(rb ? i : 0) * D, s_qh));
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
    } else if (kk > 0) {       // every candidate is chosen
        for (int i = threadIdx.x; i < kk; i += NT) {
            out_idx[i] = sg.c_lo + i;
            if (kk <= kWarpTopK) s_sorted[i] = sg.c_lo + i;
        }
        sorted_smem = kk <= kWarpTopK;
    }
    for (int i = kk + threadIdx.x; i < io.kb_stride; i += NT) out_idx[i] = -1;
    if (io.n_rescored != nullptr && threadIdx.x == 0) io.n_rescored[u] = rescored;
    __threadfence_block();
    __syncthreads();

    // ---- tail draws ------------------------------------------------------------------
    (void)unit_draws<NT>(sg, sorted_smem ? s_sorted : out_idx, io.sample_b, io.sample_cap, io.seed, b, g, io.step,
                         u, io.samp_idx, io.samp_count, nullptr, 0, G, io.per_head, io.Hq);
}

size_t select_var_smem(int n_cand) { return (size_t)8 * (size_t)(n_cand > 0 ? n_cand : 1); }

template <typename T, int D, int G, int SCORE>
static cudaError_t var_launch(const Dims& d, const VarIo& io, cudaStream_t s) {
    static std::atomic<unsigned long long> opted{0};
    cudaError_t e = opt_in_smem(k_select_var<T, D, G, SCORE>, select_var_smem(kVarKeys), opted);
    if (e != cudaSuccess) return e;
    k_select_var<T, D, G, SCORE><<<d.U(), kThreads, select_var_smem(io.sg.n_cand), s>>>(io);
    return cudaGetLastError();
}

template <typename T, int D, int G>
static cudaError_t var_s(const Dims& d, int score, const VarIo& io, cudaStream_t s) {
    if (score == SA_SCORE_MEAN_MAX) return var_launch<T, D, G, SA_SCORE_MEAN_MAX>(d, io, s);
    if (score == SA_SCORE_QUEST) return var_launch<T, D, G, SA_SCORE_QUEST>(d, io, s);
    return cudaErrorInvalidValue;
}

template <typename T, int D>
static cudaError_t var_g(const Dims& d, int score, const VarIo& io, cudaStream_t s) {
    switch (d.G) {
        case 1: return var_s<T, D, 1>(d, score, io, s);
        case 2: return var_s<T, D, 2>(d, score, io, s);
        case 4: return var_s<T, D, 4>(d, score, io, s);
        case 8: return var_s<T, D, 8>(d, score, io, s);
    }
    return cudaErrorInvalidValue;
}

bool select_var_ok(const SetGeom& g) { return g.n_cand <= kVarKeys; }

cudaError_t launch_select_var(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s) {
    VarIo io;
    io.q = a.q;
    io.rows_a = a.sp.score == SA_SCORE_QUEST ? a.st.blk_min : a.st.blk_mean;
    io.rows_b = a.sp.score == SA_SCORE_QUEST ? a.st.blk_max : nullptr;
    io.Hq = d.Hq; io.Hkv = d.Hkv; io.ld = d.ld;
    io.sg = p.g;
    io.xkey = reinterpret_cast<unsigned long long*>(a.ws + p.off_xkey);
    io.kb_stride = a.sp.k_blocks;
    io.blk_idx = a.sel.blk_idx;
    io.samp_idx = a.sel.samp_idx;
    io.samp_count = a.sel.samp_count;
    io.n_rescored = a.sel.n_rescored;
    io.sample_b = a.sp.clt_base > 0 ? a.sp.clt_base : a.sp.sample_b;
    io.sample_cap = a.sp.sample_cap;
    io.seed = (unsigned long long)a.sp.seed;
    io.step = a.sp.step;
    io.per_head = a.sp.per_head;
    const int sc = a.sp.score;
    if (d.bf16) return d.d == 128 ? var_g<__nv_bfloat16, 128>(d, sc, io, s) : var_g<__nv_bfloat16, 64>(d, sc, io, s);
    return d.d == 128 ? var_g<float, 128>(d, sc, io, s) : var_g<float, 64>(d, sc, io, s);
}

}  // namespace sa
