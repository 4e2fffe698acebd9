// The OpenAttention multi-proxy path ("OpenAttention: One Percent Is Enough
// with Tail Proxies", method overview stages 01-04): query-geometry clusters
// of the cached keys, ErrorGate's split of the read budget over the
// clusters, the QGS int8 selector, and one count-aware mean proxy per
// cluster for its unread members, all in one online softmax.
//
// Per unit (sequence b, KV head g) the clusters are kept as (sa_clusters):
//   basis  [32][D] f32   the QGS basis (rows: the eigenvectors of the query
//                        second moment, decreasing eigenvalue; the first 16
//                        are the clustering basis)
//   assign [ld] u8       the token's cluster
//   order  [ld] i32, start [C+1] i32: the positions grouped by cluster
//                        (ascending within a cluster), cluster c at
//                        order[start[c] .. start[c+1])
//   codes  [ld][32] int8 and scales [ld] f32 in that order: each key in the
//          basis, z = basis . K_j (the exact sum rounded once), sigma =
//          fl32(max|z| / 127), code = clamp(rint(z / sigma), +-127)
//   count [C] i32, sum_k, sum_v, sum_k2 [C][D] f32   cluster sums
//
// Prefill: k_cluster_order (stable counting sort of the positions by
// cluster), k_cluster_codes (codes and scales), k_cluster_stats (counts and
// sums).
// Per step, two kernels (the second a programmatic dependent of the first):
// k_multi_gate (one CTA of 256 threads per unit):
//   1. the group's projected query p_i = basis_i . sum_h q_h (exact sums
//      rounded once), coded to 16 bits: sq = max |p| / 32767, qq = rint(p/sq);
//   2. ErrorGate: per cluster and head the member-logit mean mu = s q_h .
//      Kbar and variance var = s^2 sum_e q_he^2 var_e (diagonal), the proxy's
//      weight error n e^mu (e^(var/2) - 1) over the head's estimated mass
//      sum n e^(mu + var/2), summed over the heads; the errors made integers
//      w = rint(2^30 err / max err) and the budget E split exactly:
//      q_c = min(n_c, floor(E w_c / W)), the rest one token at a time by
//      largest remainder (E w_c mod W), lowest cluster first, round after
//      round; q_c, the clusters' offsets in the read list and the packed
//      query code go to the workspace.
// k_multi_pick (grid (C/8, U), a warp per cluster):
//   3. QGS: each member's score fl32(sigma_j (qq . code_j)) (exact integer
//      dot, dp4a) as an order-preserving 32-bit key; for q_c <= 32 (clusters
//      of at most kPickKeys members) q_c rounds of a warp argmax over (key
//      desc, member asc), else the q_c-th largest key by a 4-digit radix
//      select over the cluster's keys (shared memory, or the workspace for
//      larger clusters) and the members above it and the first of those
//      equal to it; either way ascending members are ascending positions,
//      which is the tie rule, and the taken positions are written to the
//      read list in position order;
//   4. the warp's read rows (lanes over the head dim, fp32 online softmax
//      per head) while summing their keys and values, then the cluster's proxy
//      for its n' = n_c - q_c unread members: key (sum_k - read keys) / n',
//      value likewise, logit s q . key + ln n'.  Warps merge in order into a
//      CTA record; the unit's last CTA (completion ticket) combines the
//      records in order; out = acc / l.
#include "sa_cta.cuh"
#include "sa_internal.h"
#include "sa_select_core.cuh"

namespace sa {

constexpr int kQgsRank = 32;            // QGS basis size (r = 32 on the page)
constexpr int kMaxClusters = 64;        // C = 64 on the page

struct MultiIo {
    const void* q;
    const void* k;
    const void* v;
    sa_clusters cl;
    int Hq, Hkv, L, ld, C, budget;
    float scale;
    int32_t* read;                      // [U][budget]
    int32_t* qcnt;                      // [U][C]
    float* out;                         // [B][Hq][D]
    // workspace
    int* wq;                            // [U][16]: the query code, 8 words of signed high bytes, 8 of low bytes
    int* woff;                          // [U][kMaxClusters + 1]: cluster offsets in the read list
    uint32_t* wkeys;                    // [U][ld]: score keys of clusters too large for shared memory
    float* part;                        // [U][kPickCtas][G (2 + D)]: CTA records
    unsigned* cnt;                      // [U]: completion tickets
    int npick;                          // pick CTAs per unit
};

// d = a . b + c over four byte lanes, a signed and b unsigned
__device__ __forceinline__ int dp4a_su(int a, unsigned b, int c) {
    int d;
    asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// E consecutive elements (4, 8 or 16 bytes, aligned) as floats
template <typename T, int E>
__device__ __forceinline__ void ld_dims(const T* __restrict__ p, float (&x)[E]) {
    constexpr int B = (int)sizeof(T) * E;
    static_assert(B == 4 || B == 8 || B == 16, "4, 8 or 16 bytes");
    if constexpr (B == 16) {
        unpack<T>(__ldg(reinterpret_cast<const uint4*>(p)), x);
    } else if constexpr (B == 8) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
        const T* t = reinterpret_cast<const T*>(&w);
#pragma unroll
        for (int e = 0; e < E; ++e) x[e] = to_f32<T>(t[e]);
    } else {
        const unsigned w = __ldg(reinterpret_cast<const unsigned*>(p));
        const T* t = reinterpret_cast<const T*>(&w);
#pragma unroll
        for (int e = 0; e < E; ++e) x[e] = to_f32<T>(t[e]);
    }
}

// ---- prefill: codes and cluster sums -----------------------------------------------

// One CTA per unit: a stable counting sort of the positions by cluster.  The
// counts give start[]; then 256 positions at a time (one per thread, in
// position order) each token's slot = its cluster's running offset + the
// members of its cluster before it in this chunk (earlier warps, then lower
// lanes of its own warp).
__global__ void __launch_bounds__(kThreads)
k_cluster_order(sa_clusters cl, int L, int ld, int C) {
    __shared__ int s_cnt[kMaxClusters];
    __shared__ int s_run[kMaxClusters];
    __shared__ int s_wc[kWarps][kMaxClusters];
    const int u = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint8_t* a = cl.assign + (size_t)u * ld;
    for (int c = threadIdx.x; c < kMaxClusters; c += kThreads) s_cnt[c] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < L; j += kThreads) {
        const int c = __ldg(a + j);
        if (c < C) atomicAdd(&s_cnt[c], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int off = 0;
        for (int c = 0; c < C; ++c) {
            cl.start[(size_t)u * (C + 1) + c] = off;
            s_run[c] = off;
            off += s_cnt[c];
        }
        cl.start[(size_t)u * (C + 1) + C] = off;
    }
    const unsigned lt = (1u << lane) - 1u;
    for (int j0 = 0; j0 < L; j0 += kThreads) {
        for (int x = threadIdx.x; x < kWarps * kMaxClusters; x += kThreads) (&s_wc[0][0])[x] = 0;
        __syncthreads();
        const int j = j0 + threadIdx.x;
        int c = j < L ? __ldg(a + j) : 255;
        if (c >= C) c = 255;                                     // outside the clusters: not placed
        const unsigned peers = __match_any_sync(0xffffffffu, c);
        const int rank = __popc(peers & lt);
        if (c != 255 && rank == 0) s_wc[warp][c] = __popc(peers);
        __syncthreads();
        int slot = 0;
        if (c != 255) {
            slot = s_run[c] + rank;
            for (int w = 0; w < warp; ++w) slot += s_wc[w][c];
        }
        __syncthreads();                                         // every slot read s_run before it moves
        if (c != 255) cl.order[(size_t)u * ld + slot] = j;
        for (int x = threadIdx.x; x < C; x += kThreads) {
            int t = 0;
            for (int w = 0; w < kWarps; ++w) t += s_wc[w][x];
            s_run[x] += t;
        }
        __syncthreads();
    }
}

// One warp per slot i (token j = order[i]): lane r forms z_r = basis_r . K_j
// in double-double (the products of fp32 and bf16 / fp32 values are exact in
// fp64), the scale and the codes follow, stored at slot i.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
k_cluster_codes(const T* __restrict__ k, sa_clusters cl, int L, int ld) {
    __shared__ float s_row[kWarps][D];
    __shared__ float s_b[kQgsRank][D + 1];           // the unit's basis, padded: lane i reads row i
    const int u = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const float* basis = cl.basis + (size_t)u * kQgsRank * D;
    for (int x = threadIdx.x; x < kQgsRank * D; x += kThreads) s_b[x / D][x % D] = basis[x];
    __syncthreads();
    for (int i = blockIdx.x * kWarps + warp; i < L; i += gridDim.x * kWarps) {
        const int j = __ldg(cl.order + (size_t)u * ld + i);           // slot i holds token j
        const T* row = k + ((size_t)u * ld + j) * D;
        for (int e = lane; e < D; e += 32) s_row[warp][e] = to_f32<T>(row[e]);
        __syncwarp();
        // four independent double-double chains over the dims, then combined
        double s[4] = {0.0, 0.0, 0.0, 0.0}, c[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
        for (int e = 0; e < D; e += 4)
#pragma unroll
            for (int x = 0; x < 4; ++x)
                two_sum_acc(s[x], c[x], __dmul_rn((double)s_b[lane][e + x], (double)s_row[warp][e + x]));
#pragma unroll
        for (int x = 1; x < 4; ++x) {
            two_sum_acc(s[0], c[0], s[x]);
            c[0] = __dadd_rn(c[0], c[x]);
        }
        const double z = __dadd_rn(s[0], c[0]);
        double amax = fabs(z);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) amax = fmax(amax, __shfl_xor_sync(0xffffffffu, amax, off));
        const float sig = __double2float_rn(amax / 127.0);
        int code = 0;
        if (sig > 0.f) code = max(-127, min(127, (int)rint(z / (double)sig)));
        cl.codes[((size_t)u * ld + i) * kQgsRank + lane] = (int8_t)code;
        if (lane == 0) cl.scales[(size_t)u * ld + i] = sig;
        __syncwarp();
    }
}

// One CTA per unit: thread e < D adds column e of every token, in position
// order, to its cluster's fp64 sums in shared memory (deterministic), then
// writes them as fp32 with the counts.
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
k_cluster_stats(const T* __restrict__ k, const T* __restrict__ v, sa_clusters cl, int L, int ld, int C) {
    extern __shared__ __align__(16) double s_sum[];          // [3][C][D]
    __shared__ int s_cnt[kMaxClusters];
    const int u = blockIdx.x;
    for (int x = threadIdx.x; x < 3 * C * D; x += kThreads) s_sum[x] = 0.0;
    for (int x = threadIdx.x; x < C; x += kThreads) s_cnt[x] = 0;
    __syncthreads();
    const uint8_t* a = cl.assign + (size_t)u * ld;
    const T* K = k + (size_t)u * ld * D;
    const T* V = v + (size_t)u * ld * D;
    const int e = threadIdx.x;
    if (e < D) {
        // eight tokens' loads in flight before their additions
        constexpr int TU = 8;
        for (int j0 = 0; j0 < L; j0 += TU) {
            int cc[TU];
            float kx[TU], vx[TU];
#pragma unroll
            for (int x = 0; x < TU; ++x) {
                const int j = j0 + x;
                cc[x] = j < L ? a[j] : -1;
                kx[x] = j < L ? to_f32<T>(K[(size_t)j * D + e]) : 0.f;
                vx[x] = j < L ? to_f32<T>(V[(size_t)j * D + e]) : 0.f;
            }
#pragma unroll
            for (int x = 0; x < TU; ++x) {
                const int c = cc[x];
                if (c < 0) break;
                const double kd = (double)kx[x], vd = (double)vx[x];
                s_sum[c * D + e] += kd;
                s_sum[(C + c) * D + e] += vd;
                s_sum[(2 * C + c) * D + e] = fma(kd, kd, s_sum[(2 * C + c) * D + e]);
                if (e == 0) s_cnt[c] += 1;
            }
        }
    }
    __syncthreads();
    for (int x = threadIdx.x; x < C * D; x += kThreads) {
        const size_t o = (size_t)u * C * D + x;
        cl.sum_k[o] = (float)s_sum[x];
        cl.sum_v[o] = (float)s_sum[C * D + x];
        cl.sum_k2[o] = (float)s_sum[2 * C * D + x];
    }
    for (int x = threadIdx.x; x < C; x += kThreads) cl.count[(size_t)u * C + x] = s_cnt[x];
}

// ---- per step: ErrorGate and the query code ----------------------------------------

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, 2)
k_multi_gate(MultiIo io) {
    constexpr int NT = kThreads, NW = kWarps;
    __shared__ float s_q[G][D];
    __shared__ double s_pp[NW][kQgsRank][2];               // partial projections (double-double)
    __shared__ int s_qq[kQgsRank];
    __shared__ int s_qh[kQgsRank / 4];                     // qq = 256 qh + ql, packed bytes
    __shared__ unsigned s_ql[kQgsRank / 4];
    __shared__ double s_mu[G][kMaxClusters], s_sg[G][kMaxClusters];
    __shared__ double s_err[kMaxClusters];
    __shared__ double s_eh[G][kMaxClusters];               // per head shares of the errors
    __shared__ int s_n[kMaxClusters];                      // cluster sizes
    __shared__ long long s_w[kMaxClusters];
    __shared__ int s_qc[kMaxClusters], s_off[kMaxClusters + 1], s_rem[kMaxClusters];
    // the pick kernel may start now: it waits for this grid before reading
    // what this kernel writes
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

    const int u = blockIdx.x, b = u / io.Hkv, g = u - b * io.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int C = io.C;
    const T* qg = static_cast<const T*>(io.q) + ((size_t)b * io.Hq + (size_t)g * G) * D;
    for (int i = threadIdx.x; i < G * D; i += NT) s_q[i / D][i % D] = to_f32<T>(qg[i]);
    for (int c = threadIdx.x; c < C; c += NT) s_n[c] = __ldg(io.cl.count + (size_t)u * C + c);
    __syncthreads();

    // 1. the projected group query: thread (warp w, lane i) sums dims
    // [w D/8, (w+1) D/8) of basis_i . qbar in double-double
    {
        const float* basis = io.cl.basis + (size_t)u * kQgsRank * D;
        constexpr int EW = D / NW;
        // the lane's EW basis entries, every load in flight at once
        float bv[EW];
#pragma unroll
        for (int j = 0; j < EW; j += 4) {
            const float4 f = __ldg(reinterpret_cast<const float4*>(basis + (size_t)lane * D + warp * EW + j));
            bv[j] = f.x; bv[j + 1] = f.y; bv[j + 2] = f.z; bv[j + 3] = f.w;
        }
        double s = 0.0, c = 0.0;
#pragma unroll
        for (int j = 0; j < EW; ++j) {
            const int e = warp * EW + j;
            double qb = 0.0;
#pragma unroll
            for (int h = 0; h < G; ++h) qb += (double)s_q[h][e];          // exact: G bf16 / fp32 values
            two_sum_acc(s, c, __dmul_rn(qb, (double)bv[j]));
        }
        s_pp[warp][lane][0] = s;
        s_pp[warp][lane][1] = c;
    }
    __syncthreads();
    if (warp == 0) {
        double s = 0.0, c = 0.0;
        for (int w = 0; w < NW; ++w) {
            two_sum_acc(s, c, s_pp[w][lane][0]);
            c = __dadd_rn(c, s_pp[w][lane][1]);
        }
        const double p = __dadd_rn(s, c);
        double top = fabs(p);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) top = fmax(top, __shfl_xor_sync(0xffffffffu, top, off));
        int qq = 0;
        if (top > 0.0) {
            const double sq = top / 32767.0;
            qq = (int)fmax(-32767.0, fmin(32767.0, rint(p / sq)));
        }
        s_qq[lane] = qq;
        // the 16-bit codes as a signed high byte and an unsigned low byte, packed
        // four to a word for dp4a
        const int qh = qq >> 8, ql = qq & 0xFF;
        unsigned wh = (unsigned)(qh & 0xFF) << (8 * (lane & 3)), wl = (unsigned)ql << (8 * (lane & 3));
        wh |= __shfl_xor_sync(0xffffffffu, wh, 1);
        wl |= __shfl_xor_sync(0xffffffffu, wl, 1);
        wh |= __shfl_xor_sync(0xffffffffu, wh, 2);
        wl |= __shfl_xor_sync(0xffffffffu, wl, 2);
        if ((lane & 3) == 0) {
            s_qh[lane >> 2] = (int)wh;
            s_ql[lane >> 2] = wl;
        }
    }

    // 2. ErrorGate: member-logit mean and variance per (cluster, head)
    const double scale = (double)io.scale;
    const int32_t* cnt = io.cl.count + (size_t)u * C;
    // the warp's clusters c = warp, warp + 8, ...: their counts and sums
    // loaded first, all in flight together
    constexpr int CPW = kMaxClusters / NW;
    int rn[CPW];
    float rk[CPW][D / 32], rk2[CPW][D / 32];
#pragma unroll
    for (int y = 0; y < CPW; ++y) {
        const int c = warp + y * NW;
        const bool ok = c < C;
        rn[y] = ok ? __ldg(cnt + c) : 0;
        const float* sk = io.cl.sum_k + ((size_t)u * C + (ok ? c : 0)) * D;
        const float* sk2 = io.cl.sum_k2 + ((size_t)u * C + (ok ? c : 0)) * D;
#pragma unroll
        for (int x = 0; x < D / 32; ++x) {
            rk[y][x] = ok ? __ldg(sk + lane + 32 * x) : 0.f;
            rk2[y][x] = ok ? __ldg(sk2 + lane + 32 * x) : 0.f;
        }
    }
#pragma unroll
    for (int y = 0; y < CPW; ++y) {
        const int c = warp + y * NW;
        if (c >= C) break;                                 // uniform in the warp
        const int n = rn[y];
        double mean[D / 32], var[D / 32];
#pragma unroll
        for (int x = 0; x < D / 32; ++x) {
            mean[x] = n > 0 ? (double)rk[y][x] / (double)n : 0.0;
            var[x] = n > 0 ? fmax((double)rk2[y][x] / (double)n - mean[x] * mean[x], 0.0) : 0.0;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
            double a = 0.0, a2 = 0.0;
#pragma unroll
            for (int x = 0; x < D / 32; ++x) {
                const double qv = (double)s_q[h][lane + 32 * x];
                a = fma(qv, mean[x], a);
                a2 = fma(qv * qv, var[x], a2);
            }
            a = group_sum_f64<32>(a);
            a2 = group_sum_f64<32>(a2);
            if (lane == 0) {
                s_mu[h][c] = n > 0 ? scale * a : -INFINITY;
                s_sg[h][c] = scale * scale * a2;
            }
        }
    }
    __syncthreads();
    // per head (warp h): the shift m, the estimated total mass and each
    // cluster's share of the weight error (lanes over clusters)
    if (warp < G) {
        const int h = warp;
        double m = -INFINITY;
        for (int c = lane; c < C; c += 32) m = fmax(m, s_mu[h][c] + s_sg[h][c] / 2);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
        double mass = 0.0;
        for (int c = lane; c < C; c += 32) {
            const int n = s_n[c];
            if (n > 0) mass += (double)n * exp(s_mu[h][c] + s_sg[h][c] / 2 - m);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mass += __shfl_xor_sync(0xffffffffu, mass, off);
        for (int c = lane; c < C; c += 32) {
            const int n = s_n[c];
            s_eh[h][c] = n > 0 ? (double)n * exp(s_mu[h][c] - m) * expm1(s_sg[h][c] / 2) / mass : 0.0;
        }
    }
    __syncthreads();
    if (warp == 0) {
        // the cluster's error: the heads' shares summed in head order
        for (int c = lane; c < C; c += 32) {
            double e = 0.0;
            for (int h = 0; h < G; ++h) e += s_eh[h][c];
            s_err[c] = e;
        }
        __syncwarp();
        // the clusters' weights as integers, their floors and remainders (the
        // lane of each cluster), then their order for the tokens left after
        // the floors: remainder desc, lowest cluster on ties (lanes rank two
        // clusters each against all, from shared memory)
        double top = 0.0;
        for (int c = lane; c < C; c += 32) top = fmax(top, s_err[c]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) top = fmax(top, __shfl_xor_sync(0xffffffffu, top, o));
        long long wl[kMaxClusters / 32], W = 0, total = 0;
#pragma unroll
        for (int x = 0; x < kMaxClusters / 32; ++x) {
            const int c = lane + 32 * x;
            wl[x] = (c < C && top > 0.0) ? (long long)rint(s_err[c] / top * 1073741824.0) : 0;
            W += wl[x];
            total += c < C ? s_n[c] : 0;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            W += __shfl_xor_sync(0xffffffffu, W, o);
            total += __shfl_xor_sync(0xffffffffu, total, o);
        }
        const long long E = min((long long)io.budget, total);
        long long floors = 0;
#pragma unroll
        for (int x = 0; x < kMaxClusters / 32; ++x) {
            const int c = lane + 32 * x;
            if (c < C) {
                const long long n = s_n[c];
                const long long qc = W > 0 ? min(n, E * wl[x] / W) : 0;
                s_qc[c] = (int)qc;
                s_w[c] = W > 0 ? (E * wl[x]) % W : 0;       // (the remainder)
                floors += qc;
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) floors += __shfl_xor_sync(0xffffffffu, floors, o);
        __syncwarp();
#pragma unroll
        for (int x = 0; x < kMaxClusters / 32; ++x) {
            const int c = lane + 32 * x;
            if (c < C) {
                const long long rc = s_w[c];
                int rank = 0;
                for (int o = 0; o < C; ++o) {
                    const long long ro = s_w[o];
                    rank += (ro > rc || (ro == rc && o < c)) ? 1 : 0;
                }
                s_rem[rank] = c;                      // (reused: the order)
            }
        }
        __syncwarp();
        if (lane == 0) {
            long long left = E - floors;
            // one token at a time in that order, round after round
            while (left > 0) {
                bool gave = false;
                for (int r = 0; r < C && left > 0; ++r) {
                    const int c = s_rem[r];
                    if (s_qc[c] < s_n[c]) {
                        s_qc[c] += 1;
                        --left;
                        gave = true;
                    }
                }
                if (!gave) break;
            }
            int off = 0;
            for (int c = 0; c < C; ++c) {
                s_off[c] = off;
                off += s_qc[c];
            }
            s_off[C] = off;
        }
    }
    __syncthreads();
    // the budgets, the offsets, the query code; -1 after the last read slot
    for (int c = threadIdx.x; c < C; c += NT) io.qcnt[(size_t)u * C + c] = s_qc[c];
    for (int c = threadIdx.x; c <= C; c += NT) io.woff[(size_t)u * (kMaxClusters + 1) + c] = s_off[c];
    if (threadIdx.x < kQgsRank / 4) {
        io.wq[(size_t)u * 16 + threadIdx.x] = s_qh[threadIdx.x];
        io.wq[(size_t)u * 16 + 8 + threadIdx.x] = (int)s_ql[threadIdx.x];
    }
    for (int r = s_off[C] + threadIdx.x; r < io.budget; r += NT) io.read[(size_t)u * io.budget + r] = -1;
}

// ---- per step: per-cluster top-q and the softmax with the proxies ----------------------

constexpr int kPickWarps = kWarps;      // clusters per CTA
constexpr int kPickCtas = kMaxClusters / kPickWarps;
constexpr int kPickKeys = 1024;         // keys per warp in shared memory

// dynamic shared memory of k_multi_pick: the keys and histograms (the
// cross-warp merge area aliases them), then the CTA record
template <int G, int D>
struct PickSmem {
    static constexpr size_t kPick = (size_t)kPickWarps * kPickKeys * 4 + (size_t)kPickWarps * 256 * 4;
    static constexpr size_t kMerge = (size_t)kWarps * G * (D + 2) * 4;
    static constexpr size_t kArea = kPick > kMerge ? kPick : kMerge;
    static constexpr size_t kBytes = kArea + (size_t)G * (2 + D) * 4;
};

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, G >= 8 ? 2 : 3)
k_multi_pick(MultiIo io) {
    constexpr int EPC = D / 32;           // dims per lane in the softmax (lanes over the head dim)
    extern __shared__ __align__(16) unsigned char smem[];
    uint32_t* s_keys = reinterpret_cast<uint32_t*>(smem);                       // [warps][kPickKeys]
    unsigned* s_hist = reinterpret_cast<unsigned*>(smem) + kPickWarps * kPickKeys;   // [warps][256]
    float* sm = reinterpret_cast<float*>(smem);                                // merge area (aliases)
    float* s_rec = reinterpret_cast<float*>(smem + PickSmem<G, D>::kArea);

    const int u = blockIdx.y, b = u / io.Hkv, g = u - b * io.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int C = io.C;
    const int c = blockIdx.x * kPickWarps + warp;
    const bool has = c < C;
    const float qscale = io.scale * kLog2e;
    const T* qg = static_cast<const T*>(io.q) + ((size_t)b * io.Hq + (size_t)g * G) * D;
    const T* K = static_cast<const T*>(io.k) + (size_t)u * io.ld * D + lane * EPC;
    const T* V = static_cast<const T*>(io.v) + (size_t)u * io.ld * D + lane * EPC;
    // what does not depend on the gate: the cluster's extent
    const int* st = io.cl.start + (size_t)u * (C + 1);
    const int n0 = has ? __ldg(st + c) : 0, n = has ? __ldg(st + c + 1) - n0 : 0;
    const int nc = has ? __ldg(io.cl.count + (size_t)u * C + c) : 0;
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    const int qc = has ? __ldcg(io.qcnt + (size_t)u * C + c) : 0;
    const int off = has ? __ldcg(io.woff + (size_t)u * (kMaxClusters + 1) + c) : 0;
    int32_t* rd = io.read + (size_t)u * io.budget + off;
    const int32_t* ord = io.cl.order + (size_t)u * io.ld + n0;
    const unsigned lt = (1u << lane) - 1u;

    // 3. the cluster's top qc (all of it when qc >= n)
    if (qc >= n) {
        for (int i = lane; i < n; i += 32) rd[i] = __ldg(ord + i);
    } else if (qc > 0) {
        int qh[kQgsRank / 4];
        unsigned ql[kQgsRank / 4];
#pragma unroll
        for (int x = 0; x < kQgsRank / 4; ++x) {
            qh[x] = __ldcg(io.wq + (size_t)u * 16 + x);
            ql[x] = (unsigned)__ldcg(io.wq + (size_t)u * 16 + 8 + x);
        }
        uint32_t* keys = n <= kPickKeys ? s_keys + warp * kPickKeys : io.wkeys + (size_t)u * io.ld + n0;
        const int8_t* codes = io.cl.codes + ((size_t)u * io.ld + n0) * kQgsRank;
        const float* sig = io.cl.scales + (size_t)u * io.ld + n0;
        constexpr int UN = 4;                        // tokens per lane in flight
        for (int i0 = lane; i0 < n; i0 += 32 * UN) {
            // an exact integer dot with the 16-bit query code (high bytes
            // signed, low bytes unsigned) times the token's scale, rounded once
            int4 cw[UN][kQgsRank / 16];
            float sg[UN];
#pragma unroll
            for (int j = 0; j < UN; ++j) {
                const int i = i0 + 32 * j;
                const int4* cr = reinterpret_cast<const int4*>(codes + (size_t)i * kQgsRank);
#pragma unroll
                for (int w4 = 0; w4 < kQgsRank / 16; ++w4) cw[j][w4] = i < n ? __ldg(cr + w4) : make_int4(0, 0, 0, 0);
                sg[j] = i < n ? __ldg(sig + i) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < UN; ++j) {
                const int i = i0 + 32 * j;
                int hi = 0, lo = 0;
#pragma unroll
                for (int w4 = 0; w4 < kQgsRank / 16; ++w4) {
                    const int wv[4] = {cw[j][w4].x, cw[j][w4].y, cw[j][w4].z, cw[j][w4].w};
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        hi = __dp4a(wv[y], qh[w4 * 4 + y], hi);
                        lo = dp4a_su(wv[y], ql[w4 * 4 + y], lo);
                    }
                }
                const int dot = 256 * hi + lo;
                if (i < n) keys[i] = fkey(__double2float_rn((double)sg[j] * (double)dot));
            }
        }
        __syncwarp();
        if (qc <= 32 && n <= kPickKeys) {
            // small q: q rounds of a warp argmax over (key desc, member asc);
            // lane l owns members l, l + 32, ... and keeps its best one not
            // yet taken (a taken key is zeroed: a finite score's key is never
            // 0); the round's winner rescans only its own members
            auto best_of = [&]() -> unsigned long long {
                unsigned long long b = 0ull;
                for (int i = lane; i < n; i += 32) {
                    const uint32_t key = keys[i];
                    const unsigned long long c = ((unsigned long long)key << 32) | (uint32_t)(~(uint32_t)i);
                    if (key != 0u && c > b) b = c;
                }
                return b;
            };
            unsigned long long mine = best_of();
            int chosen = 0x7fffffff;                 // lane r: the r-th member taken
            for (int r = 0; r < qc; ++r) {
                const unsigned long long w = warp_max_u64(mine);
                const int wi = (int)(~(uint32_t)w);
                if (lane == r) chosen = wi;
                if ((wi & 31) == lane) {
                    keys[wi] = 0u;
                    mine = best_of();
                }
                __syncwarp();
            }
            // members ascending = positions ascending (cluster-major order)
            chosen = warp_sort_asc(chosen);
            if (lane < qc) rd[lane] = __ldg(ord + chosen);
        } else {
            // radix select of the qc-th largest key, 8 bits at a time
            unsigned* hist = s_hist + warp * 256;
            uint32_t pre = 0u, mask = 0u;
            int rem = qc;
            for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
                for (int y = 0; y < 8; ++y) hist[lane * 8 + y] = 0u;
                __syncwarp();
                for (int i0 = 0; i0 < n; i0 += 32) {
                    const int i = i0 + lane;
                    const uint32_t key = i < n ? keys[i] : 0u;
                    const unsigned bin = (i < n && (key & mask) == pre) ? ((key >> shift) & 0xFFu) : 256u;
                    const unsigned peers = __match_any_sync(0xffffffffu, bin);
                    if (bin < 256u && (peers & lt) == 0u) atomicAdd(&hist[bin], (unsigned)__popc(peers));
                }
                __syncwarp();
                // lane l holds bins 255 - 8l - y; the digit where the count from the top reaches rem
                unsigned cc[8], loc = 0;
#pragma unroll
                for (int y = 0; y < 8; ++y) { cc[y] = hist[255 - 8 * lane - y]; loc += cc[y]; }
                unsigned inc = loc;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const unsigned t = __shfl_up_sync(0xffffffffu, inc, o);
                    if (lane >= o) inc += t;
                }
                unsigned ex = inc - loc;
                int dig = -1, nrem = 0;
                if (ex < (unsigned)rem && inc >= (unsigned)rem) {
#pragma unroll
                    for (int y = 0; y < 8; ++y) {
                        if (dig < 0 && ex + cc[y] >= (unsigned)rem) {
                            dig = 255 - 8 * lane - y;
                            nrem = rem - (int)ex;
                        }
                        if (dig < 0) ex += cc[y];
                    }
                }
                const unsigned who = __ballot_sync(0xffffffffu, dig >= 0);
                const int src = __ffs(who) - 1;
                dig = __shfl_sync(0xffffffffu, dig, src);
                rem = __shfl_sync(0xffffffffu, nrem, src);
                pre |= (uint32_t)dig << shift;
                mask |= 0xFFu << shift;
                __syncwarp();
            }
            // the keys above pre, and the first rem equal to it, in slot order
            int taken = 0, eqs = 0;
            for (int i0 = 0; i0 < n; i0 += 32 * 4) {
                int pos[4];                               // positions loaded ahead, all in flight
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = i0 + 32 * j + lane;
                    pos[j] = i < n ? __ldg(ord + i) : -1;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int i = i0 + 32 * j + lane;
                    const uint32_t key = i < n ? keys[i] : 0u;
                    const bool eq = i < n && key == pre;
                    const unsigned em = __ballot_sync(0xffffffffu, eq);
                    const bool take = (i < n && key > pre) || (eq && eqs + __popc(em & lt) < rem);
                    const unsigned tm = __ballot_sync(0xffffffffu, take);
                    if (take) rd[taken + __popc(tm & lt)] = pos[j];
                    taken += __popc(tm);
                    eqs += __popc(em);
                }
            }
        }
    }
    __syncwarp();                       // the warp's read list is visible to the warp

    // 4. exact rows of the cluster (two at a time, both rows' loads in
    // flight), then its proxy; each lane holds EPC dims of every head
    float qv[G][EPC];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float f[EPC];
        ld_dims<T, EPC>(qg + (size_t)h * D + lane * EPC, f);
#pragma unroll
        for (int e = 0; e < EPC; ++e) qv[h][e] = f[e] * qscale;
    }
    Online<G, EPC> os;
    os.init();
    const int q_eff = qc < n ? qc : n;
    float ks[EPC], vs[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) { ks[e] = 0.f; vs[e] = 0.f; }
    for (int r0 = 0; r0 < q_eff; r0 += 32) {
        const int nr = min(32, q_eff - r0);
        const int pl = lane < nr ? __ldcg(rd + r0 + lane) : 0;      // 32 positions at once
        for (int j0 = 0; j0 < nr; j0 += 2) {                         // warp-uniform
            float kf[2][EPC], vf[2][EPC];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int p = __shfl_sync(0xffffffffu, pl, (j0 + j) & 31);
                if (j0 + j < nr) {
                    ld_dims<T, EPC>(K + (size_t)p * D, kf[j]);
                    ld_dims<T, EPC>(V + (size_t)p * D, vf[j]);
                } else {
#pragma unroll
                    for (int e = 0; e < EPC; ++e) { kf[j][e] = 0.f; vf[j][e] = 0.f; }
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if (j0 + j < nr) {
#pragma unroll
                    for (int h = 0; h < G; ++h) {
                        float x = 0.f;
#pragma unroll
                        for (int e = 0; e < EPC; ++e) x = fmaf(qv[h][e], kf[j][e], x);
                        os.add(h, group_sum<32>(x), vf[j]);
                    }
#pragma unroll
                    for (int e = 0; e < EPC; ++e) { ks[e] += kf[j][e]; vs[e] += vf[j][e]; }
                }
            }
        }
    }
    const int n_un = nc - q_eff;
    if (has && n_un > 0) {
        const float* sk = io.cl.sum_k + ((size_t)u * C + c) * D + lane * EPC;
        const float* sv = io.cl.sum_v + ((size_t)u * C + c) * D + lane * EPC;
        const float inv = 1.f / (float)n_un;
        float kb[EPC], vb[EPC];
#pragma unroll
        for (int e = 0; e < EPC; ++e) {
            kb[e] = (__ldg(sk + e) - ks[e]) * inv;
            vb[e] = (__ldg(sv + e) - vs[e]) * inv;
        }
        const float lnn = log2f((float)n_un);
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float x = 0.f;
#pragma unroll
            for (int e = 0; e < EPC; ++e) x = fmaf(qv[h][e], kb[e], x);
            os.add(h, group_sum<32>(x) + lnn, vb);
        }
    }
    __syncthreads();                    // the merge area aliases the keys and histograms
    float* rec = io.npick == 1 ? s_rec : io.part + ((size_t)u * kPickCtas + blockIdx.x) * Rec<G, D>::kFloats;
    cta_merge_store<G, EPC, 32, D>(os, sm, rec);
    const float* recs = s_rec;
    if (io.npick > 1) {
        if (!last_cta_of_unit(io.cnt + u, (unsigned)io.npick)) return;
        // the CTAs' records into shared memory (over the merge area) with
        // every load in flight at once, then combined in CTA order
        constexpr int RF = Rec<G, D>::kFloats;
        const float* src = io.part + (size_t)u * kPickCtas * RF;
        for (int x0 = 0; x0 < io.npick * RF; x0 += 8 * kThreads) {
            float t[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int x = x0 + j * kThreads + threadIdx.x;
                t[j] = x < io.npick * RF ? __ldcg(src + x) : 0.f;
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int x = x0 + j * kThreads + threadIdx.x;
                if (x < io.npick * RF) sm[x] = t[j];
            }
        }
        __syncthreads();
        recs = sm;
    }
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
        const int h = idx / D, e = idx - h * D;
        constexpr int RF = Rec<G, D>::kFloats;
        float M = -INFINITY;
        for (int c = 0; c < io.npick; ++c) M = fmaxf(M, recs[c * RF + h]);
        float A = 0.f, Ls = 0.f;
        for (int c = 0; c < io.npick; ++c) {
            const float m = recs[c * RF + h];
            const float f = (m == -INFINITY) ? 0.f : ex2(m - M);
            A = fmaf(recs[c * RF + 2 * G + h * D + e], f, A);
            Ls = fmaf(recs[c * RF + G + h], f, Ls);
        }
        io.out[((size_t)b * io.Hq + g * G + h) * D + e] = Ls > 0.f ? A / Ls : 0.f;
    }
    if (io.npick > 1) reset_counter(io.cnt + u);
}

// ---- launchers ---------------------------------------------------------------------------

template <typename T, int D>
static cudaError_t prep_t(const Dims& d, const void* k, const void* v, const sa_clusters& cl, int C, cudaStream_t s) {
    k_cluster_order<<<d.U(), kThreads, 0, s>>>(cl, d.L, d.ld, C);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int gx = max(1, min(cdiv(d.L, kWarps), cdiv(4 * kSmTarget, d.U())));
    k_cluster_codes<T, D><<<dim3(gx, d.U()), kThreads, 0, s>>>(static_cast<const T*>(k), cl, d.L, d.ld);
    e = cudaGetLastError();
    if (e != cudaSuccess || v == nullptr) return e;
    const size_t smem = (size_t)3 * C * D * sizeof(double);
    static std::atomic<unsigned long long> opted{0};
    e = opt_in_smem(k_cluster_stats<T, D>, (size_t)3 * kMaxClusters * D * sizeof(double), opted);
    if (e != cudaSuccess) return e;
    k_cluster_stats<T, D><<<d.U(), kThreads, smem, s>>>(static_cast<const T*>(k), static_cast<const T*>(v), cl,
                                                        d.L, d.ld, C);
    return cudaGetLastError();
}

cudaError_t launch_cluster_prep(const Dims& d, const void* k, const void* v, const sa_clusters& cl, cudaStream_t s) {
    const int C = cl.n_clusters;
    if (d.bf16) return d.d == 128 ? prep_t<__nv_bfloat16, 128>(d, k, v, cl, C, s)
                                  : prep_t<__nv_bfloat16, 64>(d, k, v, cl, C, s);
    return d.d == 128 ? prep_t<float, 128>(d, k, v, cl, C, s) : prep_t<float, 64>(d, k, v, cl, C, s);
}

// workspace: tickets, query codes, offsets, keys, CTA records (largest G = 8)
struct MultiPlan {
    size_t off_cnt, off_q, off_off, off_keys, off_part, bytes;
};

static MultiPlan multi_plan(const Dims& d) {
    MultiPlan p;
    const size_t U = (size_t)d.U();
    size_t o = 0;
    p.off_cnt = o;  o = align256(o + 4 * U);
    p.off_q = o;    o = align256(o + 4 * 16 * U);
    p.off_off = o;  o = align256(o + 4 * (size_t)(kMaxClusters + 1) * U);
    p.off_keys = o; o = align256(o + 4 * U * d.ld);
    p.off_part = o; o = align256(o + 4 * U * kPickCtas * (size_t)(8 * (2 + d.d)));
    p.bytes = o;
    return p;
}

size_t multi_workspace(const Dims& d) { return multi_plan(d).bytes; }

template <typename T, int D, int G>
static cudaError_t multi_t(const Dims& d, const MultiIo& io, cudaStream_t s) {
    k_multi_gate<T, D, G><<<d.U(), kThreads, 0, s>>>(io);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    constexpr size_t smem = PickSmem<G, D>::kBytes;
    static std::atomic<unsigned long long> opted{0};
    e = opt_in_smem(k_multi_pick<T, D, G>, smem, opted);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(io.npick, d.U());
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_multi_pick<T, D, G>, io);
}

template <typename T, int D>
static cudaError_t multi_g(const Dims& d, const MultiIo& io, cudaStream_t s) {
    switch (d.G) {
        case 1: return multi_t<T, D, 1>(d, io, s);
        case 2: return multi_t<T, D, 2>(d, io, s);
        case 4: return multi_t<T, D, 4>(d, io, s);
        case 8: return multi_t<T, D, 8>(d, io, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_multi_step(const Dims& d, const void* q, const void* k, const void* v, const sa_clusters& cl,
                              int budget, float scale, int32_t* read, int32_t* qcnt, float* out, char* ws,
                              cudaStream_t s) {
    const MultiPlan p = multi_plan(d);
    MultiIo io;
    io.q = q; io.k = k; io.v = v; io.cl = cl;
    io.Hq = d.Hq; io.Hkv = d.Hkv; io.L = d.L; io.ld = d.ld; io.C = cl.n_clusters; io.budget = budget;
    io.scale = scale;
    io.read = read; io.qcnt = qcnt; io.out = out;
    io.cnt = reinterpret_cast<unsigned*>(ws + p.off_cnt);
    io.wq = reinterpret_cast<int*>(ws + p.off_q);
    io.woff = reinterpret_cast<int*>(ws + p.off_off);
    io.wkeys = reinterpret_cast<uint32_t*>(ws + p.off_keys);
    io.part = reinterpret_cast<float*>(ws + p.off_part);
    io.npick = cdiv(cl.n_clusters, kPickWarps);
    if (d.bf16) return d.d == 128 ? multi_g<__nv_bfloat16, 128>(d, io, s) : multi_g<__nv_bfloat16, 64>(d, io, s);
    return d.d == 128 ? multi_g<float, 128>(d, io, s) : multi_g<float, 64>(d, io, s);
}

}  // namespace sa
