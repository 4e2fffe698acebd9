// Adaptive sampling budget (vAttention: Verified Sparse Attention via
// Sampling, Method, key designs 2 and 3), run after the selection kernel when
// clt_base > 0.
//
// The selection has written the unit's chosen blocks and its first b0 =
// clt_base draws (the base sample).  From the exactly read set I and the base
// sample this kernel estimates, per query head h of the group (logits
// l = s q_h . K_j, m a common shift, e = exp(l - m)):
//   N_hat = sum_I e V + (n_T / b0) sum_S e V,   D_hat = sum_I e + (n_T / b0) sum_S e,
//   Tr Sigma = sum over dims of the unbiased variance of e V over the sample,
//   var_D = the unbiased variance of e over the sample,
// and applies the lemma b >= (z n_T sqrt(Tr Sigma) / tau)^2 with
// tau = eps1 ||N_hat|| for the numerator and eps2 D_hat for the
// denominator, z = Phi^{-1}(1 - delta_i/2), under one of three rules:
//   SA_BUDGET_CLT         eps1 = eps2 = eps/4, delta1 = delta2 = delta/2 (an
//                         even split of Lemma 4.2's 2 (eps1 + eps2) = eps);
//   SA_BUDGET_CLT_SEARCH  the split searched (the reading of Theorem 4.3):
//                         eps1 = f eps/2, delta1 = g delta over the grid
//                         f, g in {1/20, ..., 19/20} (eps2 < 0.5), the
//                         smallest max over heads and bounds, ties to the
//                         first grid point in (f, g) order;
//   SA_BUDGET_HOEFFDING   the conservative bound (the page's appendix
//                         remark): b_D = n_T^2 ln(2/delta2) R_D^2 /
//                         (2 tau_D^2), b_N = d n_T^2 ln(2d/delta1) max_e
//                         R_e^2 / (2 tau_N^2), R the base sample's ranges of
//                         e and of each coordinate of e V, the even split.
// b = clamp(ceil(max over heads and both), b0, min(n_T, sample_cap)); draws
// b0 .. b-1 of the unit's stream are appended and samp_count = b.  The shift m cancels from both budgets (every term
// scales by e^-m), so the sums over I may be taken against any running
// maximum and rescaled; the sample terms use m = the maximum logit over I and
// the sample.  All of it in fp64.
//
// k_clt: grid (nsc, B*Hkv), 256 threads.  Split s of unit u takes tokens
// [s c, s c + c) of I (sink, window, chosen blocks): each warp scores 32
// tokens at a time, one token per lane (its key row against the G queries in
// shared memory, every product exact in fp64), keeps a running maximum per
// head, and accumulates e and e V (one lane per D/32 dims of the value
// rows), rescaling when the maximum rises.  The CTA's warps merge in warp
// order into a split record (m, sum e, sum e V per head).  The unit's last
// CTA (completion ticket) merges the records in split order, scores the base
// sample (one thread per draw), forms the sample sums and the two-pass
// variances, and sets the budget and the extra draws.
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int kCltMaxSamples = kCltMaxBase;     // base sample held in shared memory
constexpr int kCltBlkCache = 2048;              // chosen blocks staged for the draw mapping

// Shared layout (doubles unless noted): q [G][D], per-warp token weights
// e [W][32][G], per-warp state m, S [2][W][G], per-warp sums [W][G][D], the
// sample weights [G][kCltMaxSamples], vectors NS, DV, range [3][G][D], head
// values [12][G], the grid search's per-warp minima [2][W]; then the budget.
template <int D, int G>
struct CltSmem {
    static constexpr size_t kQ = 0;
    static constexpr size_t kE = kQ + (size_t)G * D;
    static constexpr size_t kMS = kE + (size_t)kWarps * 32 * G;
    static constexpr size_t kN = kMS + (size_t)2 * kWarps * G;
    static constexpr size_t kEs = kN + (size_t)kWarps * G * D;
    static constexpr size_t kVec = kEs + (size_t)G * kCltMaxSamples;
    static constexpr size_t kHead = kVec + (size_t)3 * G * D;
    static constexpr size_t kDoubles = kHead + (size_t)12 * G + 2 * kWarps;
    static constexpr size_t kBytes = kDoubles * 8 + 16;           // + the budget (int)
};

// logits of one key row against the G queries in shared memory (fp64, every
// product exact; the row is bf16 or fp32, 16-byte aligned)
template <typename T, int D, int G>
__device__ __forceinline__ void row_logits(const T* __restrict__ row, const double (*s_q)[D], double scale,
                                           double (&l)[G]) {
    constexpr int PER = 16 / (int)sizeof(T);          // elements per 16-byte load
#pragma unroll
    for (int h = 0; h < G; ++h) l[h] = 0.0;
    const uint4* r4 = reinterpret_cast<const uint4*>(row);
#pragma unroll 2
    for (int c = 0; c < D / PER; ++c) {
        const uint4 w = __ldg(r4 + c);
        float f[PER];
        if constexpr (PER == 8) {
            const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 x = __bfloat1622float2(b2[i]);
                f[2 * i] = x.x;
                f[2 * i + 1] = x.y;
            }
        } else {
            f[0] = __uint_as_float(w.x); f[1] = __uint_as_float(w.y);
            f[2] = __uint_as_float(w.z); f[3] = __uint_as_float(w.w);
        }
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int i = 0; i < PER; ++i) l[h] = fma(s_q[h][c * PER + i], (double)f[i], l[h]);
    }
#pragma unroll
    for (int h = 0; h < G; ++h) l[h] *= scale;
}

__device__ __forceinline__ double warp_max_f64(double x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x = fmax(x, __shfl_xor_sync(0xffffffffu, x, off));
    return x;
}

// e^(a - b) with e^(-inf - anything) = 0
__device__ __forceinline__ double exp_shift(double a, double b) { return a == -INFINITY ? 0.0 : exp(a - b); }

struct CltIo {
    const void* q;
    const void* k;
    const void* v;
    int Hq, Hkv, L, ld;
    SetGeom sg;
    const int32_t* blk_idx;
    int kb_stride;
    int32_t* samp_idx;
    int32_t* samp_count;
    int sample_cap, b0;
    double eps, delta, scale;
    int rule;                     // sa_budget
    int per_head;                 // a base sample, a budget and draws per query head
    unsigned long long seed;
    int step;
    int nsc, chunk, rec;          // splits per unit, I tokens per split, doubles per split record
    double* part;                 // [U][nsc][rec]: m[G], S[G], N[G][D]
    unsigned* cnt;                // [U] completion tickets
};

// E consecutive elements of a row, as floats
template <typename T, int E>
__device__ __forceinline__ void load_cols(const T* __restrict__ p, float (&x)[E]) {
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = to_f32<T>(p[e]);
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads)
k_clt(CltIo io) {
    constexpr int E = D / 32;                         // value dims per lane
    using SM = CltSmem<D, G>;
    extern __shared__ __align__(16) double smd[];
    double (*s_q)[D] = reinterpret_cast<double (*)[D]>(smd + SM::kQ);
    double (*s_e)[32][G] = reinterpret_cast<double (*)[32][G]>(smd + SM::kE);
    double (*s_ms)[kWarps][G] = reinterpret_cast<double (*)[kWarps][G]>(smd + SM::kMS);
    double (*s_n)[G][D] = reinterpret_cast<double (*)[G][D]>(smd + SM::kN);
    double (*s_es)[kCltMaxSamples] = reinterpret_cast<double (*)[kCltMaxSamples]>(smd + SM::kEs);
    double (*s_vec)[G][D] = reinterpret_cast<double (*)[G][D]>(smd + SM::kVec);
    double (*s_hd)[G] = reinterpret_cast<double (*)[G]>(smd + SM::kHead);
    double* s_gmin = smd + SM::kHead + 12 * G;        // [2][kWarps]: grid minimum, its index

    const int u = blockIdx.y, split = blockIdx.x;
    const int b = u / io.Hkv, g = u - b * io.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const SetGeom& sg = io.sg;
    const int nt = sg.n_t, b0 = io.b0;
    if (nt == 0 || b0 < 2) return;                    // (grid-uniform) the selection wrote the empty sample
    const T* K = reinterpret_cast<const T*>(io.k) + (size_t)u * io.ld * D;
    const T* V = reinterpret_cast<const T*>(io.v) + (size_t)u * io.ld * D;
    const int32_t* gblk = io.blk_idx + (size_t)u * io.kb_stride;
    const int32_t* gsamp = io.samp_idx + (size_t)u * io.sample_cap;
    const int n_indep = sg.s_eff + sg.w_eff, n_i = sg.n_i;
    const int win0 = io.L - sg.w_eff;
    auto pos_of = [&](int t) -> int {
        if (t < sg.s_eff) return t;
        if (t < n_indep) return win0 + (t - sg.s_eff);
        if (t < n_i) {
            const int j = t - n_indep;
            return 16 * __ldcg(gblk + (j >> 4)) + (j & 15);
        }
        return __ldcg(gsamp + (t - n_i));
    };
    const T* qg = reinterpret_cast<const T*>(io.q) + ((size_t)b * io.Hq + (size_t)g * G) * D;
    for (int i = threadIdx.x; i < G * D; i += kThreads) s_q[i / D][i % D] = (double)to_f32<T>(qg[i]);
    __syncthreads();

    // ---- this split's tokens of I: running maximum, sum e, sum e V ----------------
    const int t0 = split * io.chunk, t1 = min(n_i, t0 + io.chunk);
    double m[G], S[G], N[G][E];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m[h] = -INFINITY;
        S[h] = 0.0;
#pragma unroll
        for (int e = 0; e < E; ++e) N[h][e] = 0.0;
    }
    for (int tb = t0 + warp * 32; tb < t1; tb += kWarps * 32) {
        const int t = tb + lane;
        const int p = t < t1 ? pos_of(t) : 0;
        double l[G];
        if (t < t1) {
            row_logits<T, D, G>(K + (size_t)p * D, s_q, io.scale, l);
        } else {
#pragma unroll
            for (int h = 0; h < G; ++h) l[h] = -INFINITY;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const double mn = fmax(m[h], warp_max_f64(l[h]));
            const double sc = exp_shift(m[h], mn);
            S[h] *= sc;
#pragma unroll
            for (int e = 0; e < E; ++e) N[h][e] *= sc;
            m[h] = mn;
            const double w = exp_shift(l[h], mn);
            S[h] += w;
            s_e[warp][lane][h] = w;
        }
        __syncwarp();
        const int nb = min(32, t1 - tb);
        for (int j0 = 0; j0 < nb; j0 += 8) {
            // eight value rows in flight before their products
            float vx[8][E];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                const int pj = __shfl_sync(0xffffffffu, p, (j0 + jj) & 31);
                if (j0 + jj < nb) {
                    load_cols<T, E>(V + (size_t)pj * D + lane * E, vx[jj]);
                } else {
#pragma unroll
                    for (int e = 0; e < E; ++e) vx[jj][e] = 0.f;
                }
            }
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                if (j0 + jj >= nb) break;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    const double w = s_e[warp][j0 + jj][h];
#pragma unroll
                    for (int e = 0; e < E; ++e) N[h][e] = fma(w, (double)vx[jj][e], N[h][e]);
                }
            }
        }
        __syncwarp();                                 // s_e is rewritten by the next batch
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
        double s = S[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        if (lane == 0) {
            s_ms[0][warp][h] = m[h];
            s_ms[1][warp][h] = s;
        }
#pragma unroll
        for (int e = 0; e < E; ++e) s_n[warp][h][lane * E + e] = N[h][e];
    }
    __syncthreads();
    // the CTA's record: warps merged in warp order
    double* rec = io.part + ((size_t)u * io.nsc + split) * io.rec;
    for (int i = threadIdx.x; i < G * D; i += kThreads) {
        const int h = i / D, dim = i - h * D;
        double M = -INFINITY;
        for (int w = 0; w < kWarps; ++w) M = fmax(M, s_ms[0][w][h]);
        double A = 0.0;
        for (int w = 0; w < kWarps; ++w) A = fma(s_n[w][h][dim], exp_shift(s_ms[0][w][h], M), A);
        rec[2 * G + i] = A;
        if (dim == 0) {
            double Ss = 0.0;
            for (int w = 0; w < kWarps; ++w) Ss = fma(s_ms[1][w][h], exp_shift(s_ms[0][w][h], M), Ss);
            rec[h] = M;
            rec[G + h] = Ss;
        }
    }
    if (!last_cta_of_unit(io.cnt + u, (unsigned)io.nsc)) return;

    // ---- the unit's last CTA: merge the splits in split order ---------------------
    const double* recs = io.part + (size_t)u * io.nsc * io.rec;
    // per split and head the factor e^(m_s - M) (s_e reused as [split][head]
    // when it fits), M the maximum over the splits
    double* s_f = &s_e[0][0][0];
    const bool fcache = io.nsc * G <= kWarps * 32 * G;
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        double M = -INFINITY;
        for (int s = 0; s < io.nsc; ++s) M = fmax(M, ldcg(recs + (size_t)s * io.rec + h));
        double Ss = 0.0;
        for (int s = 0; s < io.nsc; ++s) {
            const double f = exp_shift(ldcg(recs + (size_t)s * io.rec + h), M);
            if (fcache) s_f[s * G + h] = f;
            Ss = fma(ldcg(recs + (size_t)s * io.rec + G + h), f, Ss);
        }
        s_hd[0][h] = M;                               // max logit over I
        s_hd[1][h] = Ss;                              // S_I relative to M
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * D; i += kThreads) {
        const int h = i / D, dim = i - h * D;
        double A = 0.0;
#pragma unroll 4
        for (int s = 0; s < io.nsc; ++s) {
            const double f = fcache ? s_f[s * G + h] : exp_shift(ldcg(recs + (size_t)s * io.rec + h), s_hd[0][h]);
            A = fma(ldcg(recs + (size_t)s * io.rec + 2 * G + i), f, A);
        }
        s_n[0][h][dim] = A;                           // N_I relative to M
    }
    // the base sample's logits, one thread per draw: one sample shared by the
    // heads, or (per_head) head h's own sample, row b Hq + g G + h
    const int ns = io.per_head ? G : 1;
    __shared__ int s_pos[G * kCltMaxSamples];
    for (int x = threadIdx.x; x < ns * b0; x += kThreads) {
        const int s = x / b0, i = x - s * b0;
        const int32_t* src = io.per_head ? io.samp_idx + ((size_t)b * io.Hq + g * G + s) * io.sample_cap : gsamp;
        double l[G];
        const int p = __ldcg(src + i);
        s_pos[s * kCltMaxSamples + i] = p;
        row_logits<T, D, G>(K + (size_t)p * D, s_q, io.scale, l);
        if (io.per_head) {
            s_es[s][i] = l[s];
        } else {
#pragma unroll
            for (int h = 0; h < G; ++h) s_es[h][i] = l[h];
        }
    }
    __syncthreads();
    // m = the maximum logit over I and the sample (one warp per head)
    for (int h = warp; h < G; h += kWarps) {
        double x = -INFINITY;
        for (int i = lane; i < b0; i += 32) x = fmax(x, s_es[h][i]);
        x = warp_max_f64(x);
        if (lane == 0) s_hd[2][h] = fmax(s_hd[0][h], x);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < G * b0; i += kThreads) {
        const int h = i / b0, j = i - h * b0;
        s_es[h][j] = exp_shift(s_es[h][j], s_hd[2][h]);
    }
    __syncthreads();
    // sample sums of e V, then the squared deviations from their mean (two
    // passes), over the sample's value rows staged in shared memory (one
    // sample at a time)
    T* s_vs = reinterpret_cast<T*>(reinterpret_cast<unsigned char*>(smd) + SM::kBytes);
    for (int s = 0; s < ns; ++s) {
    {
        constexpr int PER = 16 / (int)sizeof(T);
        for (int x = threadIdx.x; x < b0 * (D / PER); x += kThreads) {
            const int j = x / (D / PER), c = x - j * (D / PER);
            reinterpret_cast<uint4*>(s_vs + (size_t)j * D)[c] =
                __ldg(reinterpret_cast<const uint4*>(V + (size_t)s_pos[s * kCltMaxSamples + j] * D) + c);
        }
    }
    __syncthreads();
    const int nh = io.per_head ? 1 : G;             // heads that use this sample
    for (int i = threadIdx.x; i < nh * D; i += kThreads) {
        const int h = (io.per_head ? s : i / D), dim = i % D;
        double a = 0.0;
        for (int j = 0; j < b0; ++j) a = fma(s_es[h][j], (double)to_f32<T>(s_vs[(size_t)j * D + dim]), a);
        s_vec[0][h][dim] = a;
        const double mean = a / b0;
        double dv = 0.0, hi = -INFINITY, lo = INFINITY;
        for (int j = 0; j < b0; ++j) {
            const double r = s_es[h][j] * (double)to_f32<T>(s_vs[(size_t)j * D + dim]);
            const double dl = r - mean;
            dv = fma(dl, dl, dv);
            hi = fmax(hi, r);
            lo = fmin(lo, r);
        }
        s_vec[1][h][dim] = dv;
        s_vec[2][h][dim] = hi - lo;                   // the Hoeffding range of this coordinate
    }
    __syncthreads();                                  // the staged rows are rewritten by the next sample
    }
    // sum and unbiased variance of e over the sample (two passes), one warp per head
    for (int h = warp; h < G; h += kWarps) {
        double a = 0.0;
        for (int j = lane; j < b0; j += 32) a += s_es[h][j];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) a += __shfl_xor_sync(0xffffffffu, a, off);
        const double mean = a / b0;
        double ss = 0.0, hi = -INFINITY, lo = INFINITY;
        for (int j = lane; j < b0; j += 32) {
            const double dl = s_es[h][j] - mean;
            ss = fma(dl, dl, ss);
            hi = fmax(hi, s_es[h][j]);
            lo = fmin(lo, s_es[h][j]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, off);
            hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, off));
            lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        }
        if (lane == 0) {
            s_hd[3][h] = a;
            s_hd[4][h] = ss / (b0 - 1);
            s_hd[6][h] = hi - lo;                     // the Hoeffding range of e
        }
    }
    __syncthreads();

    // per head: ||N_hat||, D_hat, Tr Sigma and the largest squared coordinate
    // range (one warp per head)
    const double ratio = (double)nt / (double)b0;
    for (int h = warp; h < G; h += kWarps) {
        const double rI = exp_shift(s_hd[0][h], s_hd[2][h]);   // I's sums from their max to m
        double nn = 0.0, tr = 0.0, rn2 = 0.0;
        for (int e = lane; e < D; e += 32) {
            const double x = s_n[0][h][e] * rI + ratio * s_vec[0][h][e];
            nn = fma(x, x, nn);
            tr += s_vec[1][h][e];
            rn2 = fmax(rn2, s_vec[2][h][e] * s_vec[2][h][e]);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            nn += __shfl_xor_sync(0xffffffffu, nn, off);
            tr += __shfl_xor_sync(0xffffffffu, tr, off);
            rn2 = fmax(rn2, __shfl_xor_sync(0xffffffffu, rn2, off));
        }
        if (lane == 0) {
            s_hd[7][h] = sqrt(nn);                                   // ||N_hat||
            s_hd[8][h] = s_hd[1][h] * rI + ratio * s_hd[3][h];       // D_hat
            s_hd[9][h] = tr / (b0 - 1);                              // Tr Sigma
            s_hd[10][h] = rn2;
        }
    }
    __syncthreads();
    // the lemma's b for one estimate: (z(delta_i) n_T sqrt(spread) / tau)^2
    auto lemma = [&](double spread, double tau, double di) -> double {
        if (!(tau > 0.0)) return INFINITY;
        const double x = normcdfinv(1.0 - di / 2.0) * (double)nt * sqrt(fmax(spread, 0.0)) / tau;
        return x * x;
    };
    // the budget of each target: every head alone (per_head), or the group (the
    // max over its heads)
    __shared__ double s_best[G];
    const int nb = io.per_head ? G : 1;
    for (int tg = 0; tg < nb; ++tg) {
        const int h0 = io.per_head ? tg : 0, h1 = io.per_head ? tg + 1 : G;
        if (io.rule == SA_BUDGET_CLT_SEARCH) {
            // one thread per grid point (f, g); the smallest budget, first point on ties
            double bv = INFINITY;
            int bi = 0x7fffffff;
            for (int pnt = threadIdx.x; pnt < 19 * 19; pnt += kThreads) {
                const double f = (double)(pnt / 19 + 1) / 20.0, gg = (double)(pnt % 19 + 1) / 20.0;
                const double e1 = f * io.eps / 2.0, e2 = (1.0 - f) * io.eps / 2.0;
                if (e2 >= 0.5) continue;
                const double d1 = gg * io.delta, d2 = (1.0 - gg) * io.delta;
                double bb = 0.0;
                for (int h = h0; h < h1; ++h)
                    bb = fmax(bb, fmax(lemma(s_hd[9][h], e1 * s_hd[7][h], d1), lemma(s_hd[4][h], e2 * s_hd[8][h], d2)));
                if (bb < bv) { bv = bb; bi = pnt; }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const double ov = __shfl_xor_sync(0xffffffffu, bv, off);
                const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                if (ov < bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
            }
            if (lane == 0) {
                s_gmin[warp] = bv;
                s_gmin[kWarps + warp] = (double)bi;
            }
            __syncthreads();
            if (threadIdx.x == 0) {
                double v = INFINITY, vi = 1e30;
                for (int w = 0; w < kWarps; ++w)
                    if (s_gmin[w] < v || (s_gmin[w] == v && s_gmin[kWarps + w] < vi)) { v = s_gmin[w]; vi = s_gmin[kWarps + w]; }
                s_best[tg] = v;
            }
            __syncthreads();
        } else if (threadIdx.x == 0) {
            const double e1 = io.eps / 4.0, d1 = io.delta / 2.0;    // the even split, both estimates
            double best = 0.0;
            for (int h = h0; h < h1; ++h) {
                double bn, bd;
                if (io.rule == SA_BUDGET_HOEFFDING) {
                    const double tn = e1 * s_hd[7][h], td = e1 * s_hd[8][h];
                    const double dd = (double)D, n2 = (double)nt * (double)nt;
                    bn = tn > 0.0 ? dd * n2 * log(2.0 * dd / d1) * s_hd[10][h] / (2.0 * (tn * tn)) : INFINITY;
                    bd = td > 0.0 ? n2 * log(2.0 / d1) * (s_hd[6][h] * s_hd[6][h]) / (2.0 * (td * td)) : INFINITY;
                } else {
                    bn = lemma(s_hd[9][h], e1 * s_hd[7][h], d1);
                    bd = lemma(s_hd[4][h], e1 * s_hd[8][h], d1);
                }
                best = fmax(best, fmax(bn, bd));
            }
            s_best[tg] = best;
        }
    }
    __syncthreads();
    if (threadIdx.x < nb) {
        const double best = s_best[threadIdx.x];
        const int hi = min(nt, io.sample_cap);
        int bb;
        if (!(best < (double)hi)) bb = hi;                       // also inf / nan
        else bb = min(max((int)ceil(best), b0), hi);
        io.samp_count[io.per_head ? b * io.Hq + g * G + threadIdx.x : u] = bb;
    }
    if (threadIdx.x == 0) reset_counter(io.cnt + u);
}

// Draws b0 .. b-1 of each unit's stream, b = samp_count (set by k_clt):
// grid (ceil((sample_cap - b0) / kDrawsPerCta), B*Hkv), each CTA a range of
// draw indices.  Rank r of the tail maps past the chosen blocks j with g_j =
// 16 c_j - s_eff - 16 j <= r (binary search over the g_j, staged in shared
// memory when they fit).
constexpr int kDrawsPerCta = 2048;

template <int G>
__global__ void __launch_bounds__(kThreads)
k_clt_draws(CltIo io) {
    __shared__ int s_g[kCltBlkCache];
    const int u = blockIdx.y, b = u / io.Hkv, g = u - b * io.Hkv;
    const SetGeom& sg = io.sg;
    const int nt = sg.n_t, b0 = io.b0;
    if (nt == 0 || b0 < 2) return;
    const int32_t* gblk = io.blk_idx + (size_t)u * io.kb_stride;
    const bool cached = sg.kk <= kCltBlkCache;
    if (cached)
        for (int j = threadIdx.x; j < sg.kk; j += kThreads) s_g[j] = 16 * __ldcg(gblk + j) - sg.s_eff - 16 * j;
    __syncthreads();
    // one stream (the unit's) or one per query head of the group
    for (int s = 0; s < (io.per_head ? G : 1); ++s) {
    const int row = io.per_head ? b * io.Hq + g * G + s : u;
    const int bb = __ldcg(io.samp_count + row);
    const int i0 = b0 + blockIdx.x * kDrawsPerCta, i1 = min(bb, i0 + kDrawsPerCta);
    const uint64_t key = unit_key(io.seed, (uint64_t)b, (uint64_t)(io.per_head ? g * G + s : g), (uint64_t)io.step);
    int32_t* out_s = io.samp_idx + (size_t)row * io.sample_cap;
    for (int i = i0 + threadIdx.x; i < i1; i += kThreads) {
        const int r = (int)draw_rank(key, (uint32_t)i, (uint32_t)nt);
        int lo_j = 0, hi_j = sg.kk;                           // count of chosen j with g_j <= r
        while (lo_j < hi_j) {
            const int mid = (lo_j + hi_j) >> 1;
            const int gj = cached ? s_g[mid] : 16 * __ldcg(gblk + mid) - sg.s_eff - 16 * mid;
            if (gj <= r) lo_j = mid + 1; else hi_j = mid;
        }
        out_s[i] = sg.s_eff + r + 16 * lo_j;
    }
    }
}

template <typename T, int D, int G>
static cudaError_t clt_t(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s) {
    constexpr size_t smem = CltSmem<D, G>::kBytes;      // + the sample's value rows
    static std::atomic<unsigned long long> opted{0};
    cudaError_t e = opt_in_smem(k_clt<T, D, G>, smem + (size_t)kCltMaxSamples * D * sizeof(T), opted);
    if (e != cudaSuccess) return e;
    CltIo io;
    io.q = a.q; io.k = a.k; io.v = a.v;
    io.Hq = d.Hq; io.Hkv = d.Hkv; io.L = d.L; io.ld = d.ld;
    io.sg = p.g;
    io.blk_idx = a.sel.blk_idx; io.kb_stride = a.sp.k_blocks;
    io.samp_idx = a.sel.samp_idx; io.samp_count = a.sel.samp_count;
    io.sample_cap = a.sp.sample_cap; io.b0 = a.sp.clt_base;
    io.eps = (double)a.sp.eps; io.delta = (double)a.sp.delta; io.scale = (double)a.scale;
    io.rule = a.sp.budget;
    io.per_head = a.sp.per_head;
    io.seed = (unsigned long long)a.sp.seed; io.step = a.sp.step;
    io.nsc = p.nsc; io.chunk = p.clt_chunk; io.rec = p.clt_rec;
    io.part = reinterpret_cast<double*>(a.ws + p.off_clt);
    io.cnt = reinterpret_cast<unsigned*>(a.ws + p.off_cnt) + d.U();
    k_clt<T, D, G><<<dim3(p.nsc, d.U()), kThreads, smem + (size_t)io.b0 * D * sizeof(T), s>>>(io);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int nx = io.sample_cap > io.b0 ? cdiv(io.sample_cap - io.b0, kDrawsPerCta) : 0;
    if (nx > 0) k_clt_draws<G><<<dim3(nx, d.U()), kThreads, 0, s>>>(io);
    return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t clt_g(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s) {
    switch (d.G) {
        case 1: return clt_t<T, D, 1>(d, p, a, s);
        case 2: return clt_t<T, D, 2>(d, p, a, s);
        case 4: return clt_t<T, D, 4>(d, p, a, s);
        case 8: return clt_t<T, D, 8>(d, p, a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_clt(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s) {
    if (d.bf16) return d.d == 128 ? clt_g<__nv_bfloat16, 128>(d, p, a, s) : clt_g<__nv_bfloat16, 64>(d, p, a, s);
    return d.d == 128 ? clt_g<float, 128>(d, p, a, s) : clt_g<float, 64>(d, p, a, s);
}

}  // namespace sa
