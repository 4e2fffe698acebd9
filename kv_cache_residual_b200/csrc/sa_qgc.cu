// Query-geometry clustering of a cache at prefill (OpenAttention, method
// overview stage 01, QGC): the second moment of the unit's context queries,
// its leading eigenvectors (the QGS basis; the first 16 the clustering
// basis), and k-means (C clusters) of the keys projected on the first 16.
//
// k_qmoment (grid (splits, U)): M = (1/(G L)) sum q q^T over the unit's G L
//   context query rows; each CTA sums its rows into an 8 x 8 block of M per
//   thread (fp32, rows staged in shared memory) and the unit's last CTA
//   (completion ticket) adds the splits in split order in fp64.
// k_qbasis (one CTA per unit): simultaneous (subspace) iteration for the
//   32 leading eigenvectors in fp64: X <- M X, then CholeskyQR2 (twice: the
//   Gram matrix, its Cholesky factor R, X <- X R^-1), kQgcRounds rounds from
//   the first 32 unit vectors; the columns are then ordered by their
//   Rayleigh quotient x^T M x, largest first, and stored as fp32 rows.
// k_qproj (grid (splits, U)): y_j = U16 K_j for every token (fp32, workspace).
// k_kmeans (one CTA per unit): Lloyd's k-means of the y_j as the oracle runs
//   it (centroid c starts at y of position floor(c L / C); kKmeansRounds
//   rounds of nearest centroid, lowest index on ties, then means, an empty
//   cluster's centroid kept; a last assignment), the member sums kept in
//   64-bit fixed point so that the result does not depend on the order of
//   the atomic additions.
// The clusters' codes and sums then follow (k_cluster_codes,
// k_cluster_stats in sa_multi.cu).
#include "sa_cta.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int kBasisRank = 32;          // the QGS basis (r = 32)
constexpr int kClusterRank = 16;        // the QGC basis (its first 16 rows)
constexpr int kQgcRounds = 48;          // subspace iteration rounds
constexpr int kKmeansRounds = 10;
constexpr int kMomentRows = 32;         // query rows staged per tile

// ---- the second moment --------------------------------------------------------------

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
k_qmoment(const T* __restrict__ q_ctx, int Hq, int Hkv, int G, int L, int nsplit, int rows_per, float* part,
          unsigned* cnt, double* mom) {
    constexpr int TB = D / 16;                       // block edge per thread (16 x 16 threads)
    __shared__ float s_x[kMomentRows][D];
    const int u = blockIdx.y, split = blockIdx.x;
    const int b = u / Hkv, g = u - b * Hkv;
    const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
    const T* x0 = q_ctx + ((size_t)b * Hq + (size_t)g * G) * (size_t)L * D;   // G L contiguous rows
    const int n = G * L;
    const int r0 = split * rows_per, r1 = min(n, r0 + rows_per);
    float acc[TB][TB];
#pragma unroll
    for (int i = 0; i < TB; ++i)
#pragma unroll
        for (int j = 0; j < TB; ++j) acc[i][j] = 0.f;
    for (int rb = r0; rb < r1; rb += kMomentRows) {
        for (int x = threadIdx.x; x < kMomentRows * D; x += kThreads) {
            const int r = rb + x / D;
            s_x[x / D][x % D] = r < r1 ? to_f32<T>(x0[(size_t)r * D + x % D]) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int r = 0; r < kMomentRows; ++r) {
            float a[TB], c[TB];
#pragma unroll
            for (int i = 0; i < TB; ++i) { a[i] = s_x[r][ty * TB + i]; c[i] = s_x[r][tx * TB + i]; }
#pragma unroll
            for (int i = 0; i < TB; ++i)
#pragma unroll
                for (int j = 0; j < TB; ++j) acc[i][j] = fmaf(a[i], c[j], acc[i][j]);
        }
        __syncthreads();
    }
    float* pr = part + ((size_t)u * nsplit + split) * D * D;
#pragma unroll
    for (int i = 0; i < TB; ++i)
#pragma unroll
        for (int j = 0; j < TB; ++j) pr[(ty * TB + i) * D + tx * TB + j] = acc[i][j];
    if (!last_cta_of_unit(cnt + u, (unsigned)nsplit)) return;
    const float* pu = part + (size_t)u * nsplit * D * D;
    for (int x = threadIdx.x; x < D * D; x += kThreads) {
        double s = 0.0;
        for (int sp = 0; sp < nsplit; ++sp) s += (double)ldcg(pu + (size_t)sp * D * D + x);
        mom[(size_t)u * D * D + x] = s / (double)n;
    }
    reset_counter(cnt + u);
}

// ---- the leading eigenvectors --------------------------------------------------------

// One CholeskyQR pass over X [D][R] in shared memory: Gm = X^T X, R = chol(Gm),
// X <- X R^-1.  Every thread takes part.
template <int D, int R>
__device__ void cholqr(double* X, double* Gm) {
    for (int x = threadIdx.x; x < R * R; x += kThreads) {
        const int i = x / R, j = x % R;
        double s = 0.0;
        for (int r = 0; r < D; ++r) s = fma(X[r * R + i], X[r * R + j], s);
        Gm[x] = s;
    }
    __syncthreads();
    if (threadIdx.x < 32) {                           // Cholesky, one warp: lane i owns row i
        const int i = threadIdx.x;
        for (int k = 0; k < R; ++k) {
            double dk = 0.0;
            if (i == k) {
                double s = Gm[k * R + k];
                for (int m = 0; m < k; ++m) s -= Gm[k * R + m] * Gm[k * R + m];
                Gm[k * R + k] = sqrt(fmax(s, 1e-300));
            }
            __syncwarp();
            dk = Gm[k * R + k];
            if (i > k && i < R) {
                double s = Gm[i * R + k];
                for (int m = 0; m < k; ++m) s -= Gm[i * R + m] * Gm[k * R + m];
                Gm[i * R + k] = s / dk;               // lower factor: Gm = Lc Lc^T, R = Lc^T
            }
            __syncwarp();
        }
    }
    __syncthreads();
    // X <- X Lc^-T: row r solves y Lc^T = x, i.e. Lc y^T = x^T (forward substitution)
    for (int r = threadIdx.x; r < D; r += kThreads) {
        double y[R];
        for (int j = 0; j < R; ++j) {
            double s = X[r * R + j];
            for (int m = 0; m < j; ++m) s -= Gm[j * R + m] * y[m];
            y[j] = s / Gm[j * R + j];
        }
        for (int j = 0; j < R; ++j) X[r * R + j] = y[j];
    }
    __syncthreads();
}

template <int D>
__global__ void __launch_bounds__(kThreads)
k_qbasis(const double* __restrict__ mom, float* __restrict__ basis) {
    constexpr int R = kBasisRank;
    extern __shared__ __align__(16) double sm[];
    double* M = sm;                                   // [D][D]
    double* X = M + D * D;                            // [D][R]
    double* Y = X + D * R;                            // [D][R]
    double* Gm = Y + D * R;                           // [R][R]
    __shared__ double s_rq[R];
    __shared__ int s_ord[R];
    const int u = blockIdx.x;
    for (int x = threadIdx.x; x < D * D; x += kThreads) M[x] = mom[(size_t)u * D * D + x];
    for (int x = threadIdx.x; x < D * R; x += kThreads) X[x] = (x / R == x % R) ? 1.0 : 0.0;
    __syncthreads();
    for (int it = 0; it < kQgcRounds; ++it) {
        for (int x = threadIdx.x; x < D * R; x += kThreads) {
            const int r = x / R, j = x % R;
            double s = 0.0;
            for (int m = 0; m < D; ++m) s = fma(M[r * D + m], X[m * R + j], s);
            Y[x] = s;
        }
        __syncthreads();
        for (int x = threadIdx.x; x < D * R; x += kThreads) X[x] = Y[x];
        __syncthreads();
        cholqr<D, R>(X, Gm);
        cholqr<D, R>(X, Gm);
    }
    // Rayleigh quotients and the order, largest first (ties: lower column)
    for (int j = threadIdx.x; j < R; j += kThreads) {
        double s = 0.0;
        for (int r = 0; r < D; ++r) {
            double mx = 0.0;
            for (int m = 0; m < D; ++m) mx = fma(M[r * D + m], X[m * R + j], mx);
            s = fma(X[r * R + j], mx, s);
        }
        s_rq[j] = s;
    }
    __syncthreads();
    for (int j = threadIdx.x; j < R; j += kThreads) {
        int rank = 0;
        for (int m = 0; m < R; ++m) rank += (s_rq[m] > s_rq[j] || (s_rq[m] == s_rq[j] && m < j)) ? 1 : 0;
        s_ord[rank] = j;
    }
    __syncthreads();
    for (int x = threadIdx.x; x < R * D; x += kThreads) {
        const int i = x / D, e = x % D;
        basis[(size_t)u * R * D + x] = (float)X[e * R + s_ord[i]];
    }
}

// ---- projections and k-means ---------------------------------------------------------

template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
k_qproj(const T* __restrict__ k, const float* __restrict__ basis, int L, int ld, float* __restrict__ y) {
    __shared__ float s_u[kClusterRank][D];
    const int u = blockIdx.y;
    for (int x = threadIdx.x; x < kClusterRank * D; x += kThreads)
        s_u[x / D][x % D] = basis[(size_t)u * kBasisRank * D + x];
    __syncthreads();
    for (int j = blockIdx.x * kThreads + threadIdx.x; j < L; j += gridDim.x * kThreads) {
        const T* row = k + ((size_t)u * ld + j) * D;
        float acc[kClusterRank];
#pragma unroll
        for (int i = 0; i < kClusterRank; ++i) acc[i] = 0.f;
        for (int e0 = 0; e0 < D; e0 += 16 / (int)sizeof(T)) {
            float f[16 / sizeof(T)];
            unpack<T>(ld_nc16(row + e0), f);
#pragma unroll
            for (int x = 0; x < 16 / (int)sizeof(T); ++x)
#pragma unroll
                for (int i = 0; i < kClusterRank; ++i) acc[i] = fmaf(s_u[i][e0 + x], f[x], acc[i]);
        }
        float4* dst = reinterpret_cast<float4*>(y + ((size_t)u * ld + j) * kClusterRank);
#pragma unroll
        for (int i = 0; i < kClusterRank / 4; ++i)
            dst[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
    }
}

constexpr double kFixScale = 16777216.0;          // 2^24: member sums in 64-bit fixed point

constexpr int kKmThreads = 512;                   // k-means: one CTA of 16 warps per unit
constexpr int kKmCopies = 8;                      // copies of the member sums (warp w adds to w % 8)

__global__ void __launch_bounds__(kKmThreads, 1)
k_kmeans(const float* __restrict__ y, int L, int ld, int C, uint8_t* __restrict__ assign) {
    constexpr int R = kClusterRank;
    __shared__ __align__(16) float s_c[64][R];
    __shared__ float s_cn[64];                                  // |c|^2
    __shared__ long long s_sum[64][R];
    __shared__ int s_n[64];
    // each warp adds into its own copy (fewer colliding atomics), summed after
    extern __shared__ __align__(16) long long s_wsum[];         // [kKmCopies][64][R]
    int* s_wn = reinterpret_cast<int*>(s_wsum + kKmCopies * 64 * R);    // [kKmCopies][64]
    const int warp = (threadIdx.x >> 5) % kKmCopies;
    const int u = blockIdx.x;
    const float* yu = y + (size_t)u * ld * R;
    for (int x = threadIdx.x; x < C * R; x += kKmThreads) {
        const int c = x / R;
        s_c[c][x % R] = yu[(size_t)(((long long)c * L) / C) * R + x % R];
    }
    __syncthreads();
    auto norms = [&]() {
        for (int c = threadIdx.x; c < C; c += kKmThreads) {
            float t = 0.f;
#pragma unroll
            for (int i = 0; i < R; ++i) t = fmaf(s_c[c][i], s_c[c][i], t);
            s_cn[c] = t;
        }
    };
    // nearest centroid by |c|^2 - 2 v . c (|v - c|^2 less the common |v|^2),
    // first minimum (lowest index) on ties
    auto nearest = [&](const float (&v)[R]) -> int {
        float m2v[R];
#pragma unroll
        for (int i = 0; i < R; ++i) m2v[i] = -2.f * v[i];
        int best = 0;
        float bd = INFINITY;
        for (int c = 0; c < C; ++c) {
            float d2 = s_cn[c];
#pragma unroll
            for (int i = 0; i < R; i += 4) {
                const float4 cc = *reinterpret_cast<const float4*>(&s_c[c][i]);
                d2 = fmaf(m2v[i], cc.x, d2);
                d2 = fmaf(m2v[i + 1], cc.y, d2);
                d2 = fmaf(m2v[i + 2], cc.z, d2);
                d2 = fmaf(m2v[i + 3], cc.w, d2);
            }
            if (d2 < bd) { bd = d2; best = c; }
        }
        return best;
    };
    norms();
    __syncthreads();
    for (int round = 0; round < kKmeansRounds; ++round) {
        for (int x = threadIdx.x; x < kKmCopies * 64 * R; x += kKmThreads) s_wsum[x] = 0;
        for (int x = threadIdx.x; x < kKmCopies * 64; x += kKmThreads) s_wn[x] = 0;
        __syncthreads();
        for (int j = threadIdx.x; j < L; j += kKmThreads) {
            float v[R];
            const float4* src = reinterpret_cast<const float4*>(yu + (size_t)j * R);
#pragma unroll
            for (int i = 0; i < R / 4; ++i) {
                const float4 f = src[i];
                v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
            }
            const int c = nearest(v);
            atomicAdd(&s_wn[warp * 64 + c], 1);
#pragma unroll
            for (int i = 0; i < R; ++i)
                atomicAdd(reinterpret_cast<unsigned long long*>(&s_wsum[(warp * 64 + c) * R + i]),
                          (unsigned long long)llrint((double)v[i] * kFixScale));
        }
        __syncthreads();
        for (int x = threadIdx.x; x < C * R; x += kKmThreads) {
            long long t = 0;
            for (int w = 0; w < kKmCopies; ++w) t += s_wsum[(w * 64 + x / R) * R + x % R];
            s_sum[x / R][x % R] = t;
        }
        for (int x = threadIdx.x; x < C; x += kKmThreads) {
            int t = 0;
            for (int w = 0; w < kKmCopies; ++w) t += s_wn[w * 64 + x];
            s_n[x] = t;
        }
        __syncthreads();
        for (int x = threadIdx.x; x < C * R; x += kKmThreads) {
            const int c = x / R;
            if (s_n[c] > 0) s_c[c][x % R] = (float)((double)s_sum[c][x % R] / kFixScale / (double)s_n[c]);
        }
        __syncthreads();
        norms();
        __syncthreads();
    }
    for (int j = threadIdx.x; j < L; j += kKmThreads) {
        float v[R];
        const float4* src = reinterpret_cast<const float4*>(yu + (size_t)j * R);
#pragma unroll
        for (int i = 0; i < R / 4; ++i) {
            const float4 f = src[i];
            v[4 * i] = f.x; v[4 * i + 1] = f.y; v[4 * i + 2] = f.z; v[4 * i + 3] = f.w;
        }
        assign[(size_t)u * ld + j] = (uint8_t)nearest(v);
    }
}

// ---- plan and launch -----------------------------------------------------------------

QgcPlan qgc_plan(const Dims& d) {
    QgcPlan p;
    const int n = d.G * d.L;
    p.nsplit = clampi(cdiv(kSmTarget, d.U()), 1, cdiv(n, 1024));
    p.rows_per = cdiv(n, p.nsplit);
    p.nsplit = cdiv(n, p.rows_per);
    size_t off = 0;
    p.off_cnt = off;  off = align256(off + sizeof(unsigned) * (size_t)d.U());
    p.off_part = off; off = align256(off + sizeof(float) * (size_t)d.U() * p.nsplit * d.d * d.d);
    p.off_mom = off;  off = align256(off + sizeof(double) * (size_t)d.U() * d.d * d.d);
    p.off_y = off;    off = align256(off + sizeof(float) * (size_t)d.U() * d.ld * kClusterRank);
    p.bytes = off;
    return p;
}

template <typename T, int D>
static cudaError_t qgc_t(const Dims& d, const QgcPlan& p, const void* q_ctx, const void* k, const sa_clusters& cl,
                         bool basis_given, char* ws, cudaStream_t s) {
    cudaError_t e;
    if (!basis_given) {
        k_qmoment<T, D><<<dim3(p.nsplit, d.U()), kThreads, 0, s>>>(
            static_cast<const T*>(q_ctx), d.Hq, d.Hkv, d.G, d.L, p.nsplit, p.rows_per,
            reinterpret_cast<float*>(ws + p.off_part), reinterpret_cast<unsigned*>(ws + p.off_cnt),
            reinterpret_cast<double*>(ws + p.off_mom));
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        constexpr size_t smem = sizeof(double) * ((size_t)D * D + 2 * (size_t)D * kBasisRank + kBasisRank * kBasisRank);
        static std::atomic<unsigned long long> opted{0};
        e = opt_in_smem(k_qbasis<D>, smem, opted);
        if (e != cudaSuccess) return e;
        k_qbasis<D><<<d.U(), kThreads, smem, s>>>(reinterpret_cast<const double*>(ws + p.off_mom), cl.basis);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    const int gx = max(1, min(cdiv(d.L, kThreads), cdiv(4 * kSmTarget, d.U())));
    k_qproj<T, D><<<dim3(gx, d.U()), kThreads, 0, s>>>(static_cast<const T*>(k), cl.basis, d.L, d.ld,
                                                       reinterpret_cast<float*>(ws + p.off_y));
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    constexpr size_t ksm = sizeof(long long) * kKmCopies * 64 * kClusterRank + sizeof(int) * kKmCopies * 64;
    static std::atomic<unsigned long long> opted_k{0};
    e = opt_in_smem(k_kmeans, ksm, opted_k);
    if (e != cudaSuccess) return e;
    k_kmeans<<<d.U(), kKmThreads, ksm, s>>>(reinterpret_cast<const float*>(ws + p.off_y), d.L, d.ld, cl.n_clusters,
                                          cl.assign);
    return cudaGetLastError();
}

cudaError_t launch_cluster_build(const Dims& d, const QgcPlan& p, const void* q_ctx, const void* k,
                                 const sa_clusters& cl, bool basis_given, char* ws, cudaStream_t s) {
    if (d.bf16) return d.d == 128 ? qgc_t<__nv_bfloat16, 128>(d, p, q_ctx, k, cl, basis_given, ws, s)
                                  : qgc_t<__nv_bfloat16, 64>(d, p, q_ctx, k, cl, basis_given, ws, s);
    return d.d == 128 ? qgc_t<float, 128>(d, p, q_ctx, k, cl, basis_given, ws, s)
                      : qgc_t<float, 64>(d, p, q_ctx, k, cl, basis_given, ws, s);
}

}  // namespace sa
