// Adaptive sampling budget (vAttention: Verified Sparse Attention via
// Sampling, Method, key designs 2 and 3), one CTA per unit, run after the
// selection kernel when clt_base > 0.
//
// The selection has written the unit's chosen blocks and its first b0 =
// clt_base draws (the base sample).  From the exactly read set I and the base
// sample this kernel estimates, per query head h of the group (logits
// l = s q_h . K_j, m_h their maximum over I and the sample, e = exp(l - m_h)):
//   N_hat = sum_I e V + (n_T / b0) sum_S e V,   D_hat = sum_I e + (n_T / b0) sum_S e,
//   Tr Sigma = sum over dims of the unbiased variance of e V over the sample,
//   var_D = the unbiased variance of e over the sample,
// and applies the lemma b >= (z n_T sqrt(Tr Sigma) / tau)^2 with
// tau = (eps/4) ||N_hat|| for the numerator and (eps/4) D_hat for the
// denominator, z = Phi^{-1}(1 - delta/4) (eps and delta split evenly between
// them, Lemma 4.2).  b = clamp(ceil(max over heads and both), b0,
// min(n_T, sample_cap)); draws b0 .. b-1 of the unit's stream are appended
// and samp_count = b.  All of it in fp64: logits as sums of exact products,
// the sample variances in two passes (mean, then squared deviations).
#include "sa_common.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int kCltMaxSamples = kCltMaxBase;     // base sample held in shared memory

// Shared layout (doubles unless noted): q [G][D], warp maxima [W][G], sample
// weights e [G][kCltMaxSamples], cross-warp reduction [W][G][D], per-warp
// scalars [W][G][2], vectors NI, NS, NSD [3][G][D], head sums [4][G].
template <int D, int G>
struct CltSmem {
    static constexpr size_t kQ = 0;
    static constexpr size_t kM = kQ + (size_t)G * D;
    static constexpr size_t kEs = kM + (size_t)kWarps * G;
    static constexpr size_t kRed = kEs + (size_t)G * kCltMaxSamples;
    static constexpr size_t kSc = kRed + (size_t)kWarps * G * D;
    static constexpr size_t kVec = kSc + (size_t)kWarps * G * 2;
    static constexpr size_t kSum = kVec + (size_t)3 * G * D;
    static constexpr size_t kDoubles = kSum + (size_t)4 * G;
    static constexpr size_t kBytes = kDoubles * 8 + 16;           // + the budget (int)
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads)
k_clt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, int Hq, int Hkv, int L, int ld,
      SetGeom sg,
      const int32_t* __restrict__ blk_idx, int kb_stride, int32_t* __restrict__ samp_idx,
      int32_t* __restrict__ samp_count, int sample_cap, int b0, double eps, double delta, double scale,
      unsigned long long seed, int step) {
    constexpr int E = D / 32;                         // dims per lane
    using SM = CltSmem<D, G>;
    extern __shared__ __align__(16) double smd[];
    double (*s_q)[D] = reinterpret_cast<double (*)[D]>(smd + SM::kQ);
    double (*s_m)[G] = reinterpret_cast<double (*)[G]>(smd + SM::kM);
    double (*s_es)[kCltMaxSamples] = reinterpret_cast<double (*)[kCltMaxSamples]>(smd + SM::kEs);
    double (*s_red)[G][D] = reinterpret_cast<double (*)[G][D]>(smd + SM::kRed);
    double (*s_sc)[G][2] = reinterpret_cast<double (*)[G][2]>(smd + SM::kSc);
    double (*s_vec)[G][D] = reinterpret_cast<double (*)[G][D]>(smd + SM::kVec);
    double (*s_sum)[G] = reinterpret_cast<double (*)[G]>(smd + SM::kSum);
    int& s_b = *reinterpret_cast<int*>(smd + SM::kDoubles);

    const int u = blockIdx.x;
    const int b = u / Hkv, g = u - b * Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nt = sg.n_t;
    if (nt == 0 || b0 < 2) return;                    // the selection wrote the (empty) sample
    const T* K = k + (size_t)u * ld * D;
    const T* V = v + (size_t)u * ld * D;
    const int32_t* gblk = blk_idx + (size_t)u * kb_stride;
    const int32_t* gsamp = samp_idx + (size_t)u * sample_cap;
    const int n_indep = sg.s_eff + sg.w_eff, n_i = sg.n_i, n_tok = n_i + b0;
    const int win0 = L - sg.w_eff;
    auto pos_of = [&](int t) -> int {
        if (t < sg.s_eff) return t;
        if (t < n_indep) return win0 + (t - sg.s_eff);
        if (t < n_i) {
            const int j = t - n_indep;
            return 16 * __ldcg(gblk + (j >> 4)) + (j & 15);
        }
        return __ldcg(gsamp + (t - n_i));
    };
    for (int i = threadIdx.x; i < G * D; i += kThreads)
        s_q[i / D][i % D] = (double)to_f32<T>(q[((size_t)b * Hq + (size_t)g * G) * D + i]);
    __syncthreads();

    // logit of token t for every head (warp-collective; every lane gets them)
    auto logits = [&](int p, double (&l)[G]) {
        double kx[E];
#pragma unroll
        for (int e = 0; e < E; ++e) kx[e] = (double)to_f32<T>(K[(size_t)p * D + lane * E + e]);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            double x = 0.0;
#pragma unroll
            for (int e = 0; e < E; ++e) x = fma(s_q[h][lane * E + e], kx[e], x);
            l[h] = group_sum_f64<32>(x) * scale;
        }
    };

    // pass 1: the maximum logit per head over I and the sample
    double mx[G];
#pragma unroll
    for (int h = 0; h < G; ++h) mx[h] = -INFINITY;
    for (int t = warp; t < n_tok; t += kWarps) {
        double l[G];
        logits(pos_of(t), l);
#pragma unroll
        for (int h = 0; h < G; ++h) mx[h] = fmax(mx[h], l[h]);
    }
    if (lane == 0)
#pragma unroll
        for (int h = 0; h < G; ++h) s_m[warp][h] = mx[h];
    __syncthreads();
    if (threadIdx.x < G) {
        double m = -INFINITY;
        for (int w = 0; w < kWarps; ++w) m = fmax(m, s_m[w][threadIdx.x]);
        s_sum[3][threadIdx.x] = m;
    }
    __syncthreads();
    double m[G];
#pragma unroll
    for (int h = 0; h < G; ++h) m[h] = s_sum[3][h];

    // pass 2: sums over I and over the sample of e and e V (per warp, then
    // across warps in fixed warp order)
    double nI[G][E], nS[G][E], sI[G], sS[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        sI[h] = 0.0;
        sS[h] = 0.0;
#pragma unroll
        for (int e = 0; e < E; ++e) { nI[h][e] = 0.0; nS[h][e] = 0.0; }
    }
    for (int t = warp; t < n_tok; t += kWarps) {
        const int p = pos_of(t);
        double l[G];
        logits(p, l);
        double vx[E];
#pragma unroll
        for (int e = 0; e < E; ++e) vx[e] = (double)to_f32<T>(V[(size_t)p * D + lane * E + e]);
        const bool smp = t >= n_i;
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const double w = exp(l[h] - m[h]);
            if (smp) {
                sS[h] += w;
                if (lane == 0) s_es[h][t - n_i] = w;
#pragma unroll
                for (int e = 0; e < E; ++e) nS[h][e] = fma(w, vx[e], nS[h][e]);
            } else {
                sI[h] += w;
#pragma unroll
                for (int e = 0; e < E; ++e) nI[h][e] = fma(w, vx[e], nI[h][e]);
            }
        }
    }
    auto reduce_vec = [&](double (&a)[G][E], int slot) {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < E; ++e) s_red[warp][h][lane * E + e] = a[h][e];
        __syncthreads();
        for (int i = threadIdx.x; i < G * D; i += kThreads) {
            double x = 0.0;
            for (int w = 0; w < kWarps; ++w) x += s_red[w][i / D][i % D];
            s_vec[slot][i / D][i % D] = x;
        }
        __syncthreads();
    };
    reduce_vec(nI, 0);
    reduce_vec(nS, 1);
    if (lane == 0)
#pragma unroll
        for (int h = 0; h < G; ++h) { s_sc[warp][h][0] = sI[h]; s_sc[warp][h][1] = sS[h]; }
    __syncthreads();
    if (threadIdx.x < G) {
        const int h = threadIdx.x;
        double a = 0.0, c = 0.0;
        for (int w = 0; w < kWarps; ++w) { a += s_sc[w][h][0]; c += s_sc[w][h][1]; }
        s_sum[0][h] = a;
        s_sum[1][h] = c;
        // unbiased variance of e over the sample, two passes
        const double mean = c / b0;
        double ss = 0.0;
        for (int i = 0; i < b0; ++i) { const double dlt = s_es[h][i] - mean; ss = fma(dlt, dlt, ss); }
        s_sum[2][h] = ss / (b0 - 1);
    }
    __syncthreads();

    // pass 3 over the sample: squared deviations of e V from its mean
    double dv[G][E];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < E; ++e) dv[h][e] = 0.0;
    for (int t = n_i + warp; t < n_tok; t += kWarps) {
        const int p = pos_of(t);
        double vx[E];
#pragma unroll
        for (int e = 0; e < E; ++e) vx[e] = (double)to_f32<T>(V[(size_t)p * D + lane * E + e]);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            const double w = s_es[h][t - n_i];
#pragma unroll
            for (int e = 0; e < E; ++e) {
                const double dlt = w * vx[e] - s_vec[1][h][lane * E + e] / b0;
                dv[h][e] = fma(dlt, dlt, dv[h][e]);
            }
        }
    }
    reduce_vec(dv, 2);

    // the budget: one warp per head, then the maximum over heads
    const double ratio = (double)nt / (double)b0;
    const double tau_scale = eps / 4.0;
    const double z = normcdfinv(1.0 - delta / 4.0);     // two-sided quantile at delta/2
    for (int h = warp; h < G; h += kWarps) {
        double nn = 0.0, tr = 0.0;
        for (int e = lane; e < D; e += 32) {
            const double x = s_vec[0][h][e] + ratio * s_vec[1][h][e];
            nn = fma(x, x, nn);
            tr += s_vec[2][h][e];
        }
        nn = group_sum_f64<32>(nn);
        tr = group_sum_f64<32>(tr) / (b0 - 1);
        if (lane == 0) {
            const double dh = s_sum[0][h] + ratio * s_sum[1][h];
            const double tn = tau_scale * sqrt(nn), td = tau_scale * dh;
            const double bn = tn > 0.0 ? z * (double)nt * sqrt(fmax(tr, 0.0)) / tn : INFINITY;
            const double bd = td > 0.0 ? z * (double)nt * sqrt(fmax(s_sum[2][h], 0.0)) / td : INFINITY;
            s_sc[0][h][0] = fmax(bn * bn, bd * bd);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double best = 0.0;
        for (int h = 0; h < G; ++h) best = fmax(best, s_sc[0][h][0]);
        const int hi = min(nt, sample_cap);
        int bb;
        if (!(best < (double)hi)) bb = hi;                       // also inf / nan
        else bb = min(max((int)ceil(best), b0), hi);
        s_b = bb;
        samp_count[u] = bb;
    }
    __syncthreads();

    // draws b0 .. b-1 of the unit's stream
    const int bb = s_b;
    if (bb > b0) {
        const uint64_t key = unit_key(seed, (uint64_t)b, (uint64_t)g, (uint64_t)step);
        int32_t* out_s = samp_idx + (size_t)u * sample_cap;
        for (int i = b0 + threadIdx.x; i < bb; i += kThreads) {
            const int r = (int)draw_rank(key, (uint32_t)i, (uint32_t)nt);
            int lo_j = 0, hi_j = sg.kk;                           // count of chosen j with g_j <= r
            while (lo_j < hi_j) {
                const int mid = (lo_j + hi_j) >> 1;
                const int gj = 16 * __ldcg(gblk + mid) - sg.s_eff - 16 * mid;
                if (gj <= r) lo_j = mid + 1; else hi_j = mid;
            }
            out_s[i] = sg.s_eff + r + 16 * lo_j;
        }
    }
}

template <typename T, int D, int G>
static cudaError_t clt_t(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s) {
    constexpr size_t smem = CltSmem<D, G>::kBytes;
    static std::atomic<unsigned long long> opted{0};
    cudaError_t e = opt_in_smem(k_clt<T, D, G>, smem, opted);
    if (e != cudaSuccess) return e;
    k_clt<T, D, G><<<d.U(), kThreads, smem, s>>>(
        reinterpret_cast<const T*>(a.q), reinterpret_cast<const T*>(a.k), reinterpret_cast<const T*>(a.v), d.Hq,
        d.Hkv, d.L, d.ld, p.g, a.sel.blk_idx, a.sp.k_blocks, a.sel.samp_idx, a.sel.samp_count, a.sp.sample_cap,
        a.sp.clt_base, (double)a.sp.eps, (double)a.sp.delta, (double)a.scale, (unsigned long long)a.sp.seed,
        a.sp.step);
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
