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
//   codes  [ld][32] int8 and scales [ld] f32: each key in that basis,
//          z = basis . K_j (the exact sum rounded once), sigma = fl32(max|z| /
//          127), code = clamp(rint(z / sigma), +-127)
//   assign [ld] u8       the token's cluster
//   count [C] i32, sum_k, sum_v, sum_k2 [C][D] f32   cluster sums
//
// k_cluster_codes: codes and scales from the basis (prefill).
// k_cluster_stats: count and sums from the assignment (prefill).
// k_multi_select (per step, one CTA of 256 threads per unit):
//   1. the group's projected query p_i = basis_i . sum_h q_h (exact sums
//      rounded once), coded to 16 bits: sq = max |p| / 32767, qq = rint(p/sq);
//   2. ErrorGate: per cluster and head the member-logit mean mu = s q_h .
//      Kbar and variance var = s^2 sum_e q_he^2 var_e (diagonal), the proxy's
//      weight error n e^mu (e^(var/2) - 1) over the head's estimated mass
//      sum n e^(mu + var/2), summed over the heads; the errors made integers
//      w = rint(2^30 err / max err) and the budget E split exactly:
//      q_c = min(n_c, floor(E w_c / W)), the rest one token at a time by
//      largest remainder (E w_c mod W), lowest cluster first, round after round;
//   3. QGS: every token's score fl32(sigma_j (qq . code_j)) (exact integer dot)
//      as a 64-bit key (score, then lower position first); per cluster the
//      q_c-th largest key by an 8-digit radix select run for all clusters at
//      once (per-cluster histograms in shared memory, keys in the workspace);
//   4. the read tokens written grouped by cluster (cluster order, ascending
//      positions), and q_c.
// k_multi_decode (per step, one CTA of 256 threads per unit): each warp takes
//   clusters c = warp, warp + 8, ...: its read rows (lane groups over rows,
//   fp32 online softmax per head) while summing their keys and values, then
//   the cluster's proxy for its n' = n_c - q_c unread members: key (sum_k -
//   read keys) / n', value likewise, logit s q . key + ln n'.  Warps merge in
//   order; out = acc / l.
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
    unsigned long long* keys;           // [U][ld] workspace
    int* list;                          // [U][ld] workspace: the candidates left after two digits
    float* out;                         // [B][Hq][D]
};

// d = a . b + c over four byte lanes, a signed and b unsigned
__device__ __forceinline__ int dp4a_su(int a, unsigned b, int c) {
    int d;
    asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// ---- prefill: codes and cluster sums -----------------------------------------------

// One warp per token: lane i forms z_i = basis_i . K_j in double-double (the
// products of fp32 and bf16 / fp32 values are exact in fp64), the scale and
// the codes follow.
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
    for (int j = blockIdx.x * kWarps + warp; j < L; j += gridDim.x * kWarps) {
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
        cl.codes[((size_t)u * ld + j) * kQgsRank + lane] = (int8_t)code;
        if (lane == 0) cl.scales[(size_t)u * ld + j] = sig;
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

// ---- per step: the selection -----------------------------------------------------------

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads)
k_multi_select(MultiIo io) {
    constexpr int NT = kThreads, NW = kWarps;
    __shared__ float s_q[G][D];
    __shared__ double s_pp[NW][kQgsRank][2];               // partial projections (double-double)
    __shared__ int s_qq[kQgsRank];
    __shared__ int s_qh[kQgsRank / 4];                     // qq = 256 qh + ql, packed bytes
    __shared__ unsigned s_ql[kQgsRank / 4];
    __shared__ int s_nlist;
    __shared__ double s_mu[G][kMaxClusters], s_sg[G][kMaxClusters];
    __shared__ double s_err[kMaxClusters];
    __shared__ long long s_w[kMaxClusters];
    __shared__ int s_qc[kMaxClusters], s_off[kMaxClusters + 1], s_rem[kMaxClusters];
    __shared__ unsigned long long s_pre[kMaxClusters];
    extern __shared__ __align__(16) unsigned s_hist[];      // [C][256] (also [C][NT] counts at the end)
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");

    const int u = blockIdx.x, b = u / io.Hkv, g = u - b * io.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int C = io.C, L = io.L;
    const T* qg = static_cast<const T*>(io.q) + ((size_t)b * io.Hq + (size_t)g * G) * D;
    for (int i = threadIdx.x; i < G * D; i += NT) s_q[i / D][i % D] = to_f32<T>(qg[i]);
    __syncthreads();

    // 1. the projected group query: thread (warp w, lane i) sums dims
    // [w D/8, (w+1) D/8) of basis_i . qbar in double-double
    {
        const float* basis = io.cl.basis + (size_t)u * kQgsRank * D;
        constexpr int EW = D / NW;
        double s = 0.0, c = 0.0;
        for (int e = warp * EW; e < (warp + 1) * EW; ++e) {
            double qb = 0.0;
#pragma unroll
            for (int h = 0; h < G; ++h) qb += (double)s_q[h][e];          // exact: G bf16 / fp32 values
            two_sum_acc(s, c, __dmul_rn(qb, (double)basis[lane * D + e]));
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
    for (int c = warp; c < C; c += NW) {
        const int n = __ldg(cnt + c);
        const float* sk = io.cl.sum_k + ((size_t)u * C + c) * D;
        const float* sk2 = io.cl.sum_k2 + ((size_t)u * C + c) * D;
        double mean[D / 32], var[D / 32];
#pragma unroll
        for (int x = 0; x < D / 32; ++x) {
            const int e = lane + 32 * x;
            mean[x] = n > 0 ? (double)sk[e] / (double)n : 0.0;
            var[x] = n > 0 ? fmax((double)sk2[e] / (double)n - mean[x] * mean[x], 0.0) : 0.0;
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
    if (warp == 0) {
        // per head: the shift m and the estimated total mass (lanes over clusters)
        double err[kMaxClusters / 32];
#pragma unroll
        for (int x = 0; x < kMaxClusters / 32; ++x) err[x] = 0.0;
        for (int h = 0; h < G; ++h) {
            double m = -INFINITY;
            for (int c = lane; c < C; c += 32) m = fmax(m, s_mu[h][c] + s_sg[h][c] / 2);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, off));
            double mass = 0.0;
            for (int c = lane; c < C; c += 32) {
                const int n = __ldg(cnt + c);
                if (n > 0) mass += (double)n * exp(s_mu[h][c] + s_sg[h][c] / 2 - m);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) mass += __shfl_xor_sync(0xffffffffu, mass, off);
#pragma unroll
            for (int x = 0; x < kMaxClusters / 32; ++x) {
                const int c = lane + 32 * x;
                if (c < C) {
                    const int n = __ldg(cnt + c);
                    if (n > 0) err[x] += (double)n * exp(s_mu[h][c] - m) * expm1(s_sg[h][c] / 2) / mass;
                }
            }
        }
#pragma unroll
        for (int x = 0; x < kMaxClusters / 32; ++x)
            if (lane + 32 * x < C) s_err[lane + 32 * x] = err[x];
        __syncwarp();
        // the clusters' weights as integers, and their order for the tokens
        // left after the floors: remainder desc, lowest cluster on ties
        // (lanes rank two clusters each against all)
        double top = 0.0;
        for (int c = 0; c < C; ++c) top = fmax(top, s_err[c]);
        long long W = 0;
        for (int c = 0; c < C; ++c) W += top > 0.0 ? (long long)rint(s_err[c] / top * 1073741824.0) : 0;
        long long total = 0;
        for (int c = 0; c < C; ++c) total += __ldg(cnt + c);
        const long long E = min((long long)io.budget, total);
#pragma unroll
        for (int x = 0; x < kMaxClusters / 32; ++x) {
            const int c = lane + 32 * x;
            if (c < C) {
                const long long wc = top > 0.0 ? (long long)rint(s_err[c] / top * 1073741824.0) : 0;
                s_w[c] = wc;
                const long long rc = W > 0 ? (E * wc) % W : 0;
                int rank = 0;
                for (int o = 0; o < C; ++o) {
                    const long long wo = top > 0.0 ? (long long)rint(s_err[o] / top * 1073741824.0) : 0;
                    const long long ro = W > 0 ? (E * wo) % W : 0;
                    rank += (ro > rc || (ro == rc && o < c)) ? 1 : 0;
                }
                s_rem[rank] = c;                      // (reused: the order)
            }
        }
        __syncwarp();
        if (lane == 0) {
            // integer split of the budget (exact)
            for (int c = 0; c < C; ++c) top = fmax(top, s_err[c]);
            long long left = E;
            for (int c = 0; c < C; ++c) {
                const long long n = __ldg(cnt + c);
                const long long qc = W > 0 ? min(n, E * s_w[c] / W) : 0;
                s_qc[c] = (int)qc;
                left -= qc;
            }
            // one token at a time in that order, round after round
            while (left > 0) {
                bool gave = false;
                for (int r = 0; r < C && left > 0; ++r) {
                    const int c = s_rem[r];
                    if (s_qc[c] < __ldg(cnt + c)) {
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
                s_rem[c] = s_qc[c];
                s_pre[c] = 0ull;
            }
            s_off[C] = off;
        }
    }
    __syncthreads();

    // 3. scores as keys (score desc, position asc), and the per-cluster radix select
    const uint8_t* asg = io.cl.assign + (size_t)u * io.ld;
    const int8_t* codes = io.cl.codes + (size_t)u * io.ld * kQgsRank;
    const float* sig = io.cl.scales + (size_t)u * io.ld;
    unsigned long long* keys = io.keys + (size_t)u * io.ld;
    int* list = io.list + (size_t)u * io.ld;
    int qh[kQgsRank / 4];
    unsigned ql[kQgsRank / 4];
#pragma unroll
    for (int x = 0; x < kQgsRank / 4; ++x) { qh[x] = s_qh[x]; ql[x] = s_ql[x]; }
    if (threadIdx.x == 0) s_nlist = 0;
    unsigned long long mask = 0ull;
    for (int shift = 56; shift >= 0; shift -= 8) {
        for (int x = threadIdx.x; x < C * 256; x += NT) s_hist[x] = 0u;
        __syncthreads();
        // the first two digits over every token; then over the candidates
        // listed after them (those whose two top digits match their cluster's)
        const bool all = shift >= 48;
        const int n_it = all ? L : s_nlist;
        for (int x = threadIdx.x; x < ((n_it + 31) & ~31); x += NT) {      // warp-uniform trip count
            const bool live = x < n_it;
            const int j = all ? x : (live ? list[x] : 0);
            unsigned long long key = 0ull;
            if (live && shift == 56) {
                // the token's score: an exact integer dot with the 16-bit query
                // code (high bytes signed, low bytes unsigned) times its scale
                const int4* cr = reinterpret_cast<const int4*>(codes + (size_t)j * kQgsRank);
                int hi = 0, lo = 0;
#pragma unroll
                for (int w4 = 0; w4 < kQgsRank / 16; ++w4) {
                    const int4 cw = __ldg(cr + w4);
                    const int wv[4] = {cw.x, cw.y, cw.z, cw.w};
#pragma unroll
                    for (int y = 0; y < 4; ++y) {
                        hi = __dp4a(wv[y], qh[w4 * 4 + y], hi);
                        lo = dp4a_su(wv[y], ql[w4 * 4 + y], lo);
                    }
                }
                const int dot = 256 * hi + lo;
                const float sc = __double2float_rn((double)__ldg(sig + j) * (double)dot);   // exact product, one rounding
                key = ((unsigned long long)fkey(sc) << 32) | (unsigned long long)(~(uint32_t)j);
                keys[j] = key;
            } else if (live) {
                key = keys[j];
            }
            const int c = live ? __ldg(asg + j) : 0;
            int digit = 256;
            if (live && s_rem[c] > 0 && (key & mask) == s_pre[c]) digit = (int)((key >> shift) & 0xFF);
            const unsigned bin = digit < 256 ? (unsigned)(c * 256 + digit) : 0xffffffffu;
            const unsigned peers = __match_any_sync(0xffffffffu, bin);
            if (digit < 256 && lane == __ffs(peers) - 1) atomicAdd(&s_hist[bin], (unsigned)__popc(peers));
        }
        __syncthreads();
        // per cluster: the digit at which the count from the top reaches rem
        for (int c = warp; c < C; c += NW) {
            const int rem = s_rem[c];
            if (rem <= 0) continue;
            unsigned cc[8], loc = 0;
#pragma unroll
            for (int y = 0; y < 8; ++y) { cc[y] = s_hist[c * 256 + 255 - 8 * lane - y]; loc += cc[y]; }
            unsigned inc = loc;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const unsigned o = __shfl_up_sync(0xffffffffu, inc, off);
                if (lane >= off) inc += o;
            }
            unsigned ex = inc - loc;
            if (ex < (unsigned)rem && inc >= (unsigned)rem) {
#pragma unroll
                for (int y = 0; y < 8; ++y) {
                    if (ex + cc[y] >= (unsigned)rem) {
                        s_pre[c] |= (unsigned long long)(255 - 8 * lane - y) << shift;
                        s_rem[c] = rem - (int)ex;
                        break;
                    }
                    ex += cc[y];
                }
            }
        }
        mask |= 0xFFull << shift;
        __syncthreads();
        if (shift == 48) {
            // list the candidates still in play (order free: only counts follow)
            for (int x = threadIdx.x; x < ((L + 31) & ~31); x += NT) {
                bool in = false;
                if (x < L) {
                    const int c = __ldg(asg + x);
                    in = s_rem[c] > 0 && (keys[x] & mask) == s_pre[c];
                }
                const unsigned m = __ballot_sync(0xffffffffu, in);
                int base = 0;
                if (lane == 0 && m != 0u) base = atomicAdd(&s_nlist, __popc(m));
                base = __shfl_sync(0xffffffffu, base, 0);
                if (in) list[base + __popc(m & ((1u << lane) - 1u))] = x;
            }
            __threadfence_block();
            __syncthreads();
        }
    }

    // 4. the read tokens, grouped by cluster: each thread counts its chunk's
    // selected tokens per cluster, a scan per cluster gives the places
    const int chunk = (L + NT - 1) / NT;
    const int j0 = min(L, (int)threadIdx.x * chunk), j1 = min(L, j0 + chunk);
    unsigned* s_cnt = s_hist;                                 // [C][NT]
    for (int x = threadIdx.x; x < C * NT; x += NT) s_cnt[x] = 0u;
    __syncthreads();
    for (int j = j0; j < j1; ++j) {
        const int c = __ldg(asg + j);
        if (s_qc[c] > 0 && keys[j] >= s_pre[c]) s_cnt[c * NT + threadIdx.x] += 1u;
    }
    __syncthreads();
    for (int c = warp; c < C; c += NW) {                     // exclusive scan over threads, per cluster
        unsigned v[NT / 32], loc = 0;
#pragma unroll
        for (int y = 0; y < NT / 32; ++y) { v[y] = s_cnt[c * NT + lane * (NT / 32) + y]; loc += v[y]; }
        unsigned inc = loc;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const unsigned o = __shfl_up_sync(0xffffffffu, inc, off);
            if (lane >= off) inc += o;
        }
        unsigned ex = inc - loc + (unsigned)s_off[c];
#pragma unroll
        for (int y = 0; y < NT / 32; ++y) {
            const unsigned t = v[y];
            s_cnt[c * NT + lane * (NT / 32) + y] = ex;
            ex += t;
        }
    }
    __syncthreads();
    int32_t* rd = io.read + (size_t)u * io.budget;
    for (int j = j0; j < j1; ++j) {
        const int c = __ldg(asg + j);
        if (s_qc[c] > 0 && keys[j] >= s_pre[c]) {
            const unsigned p = s_cnt[c * NT + threadIdx.x]++;
            if (p < (unsigned)io.budget) rd[p] = j;
        }
    }
    for (int p = s_off[C] + threadIdx.x; p < io.budget; p += NT) rd[p] = -1;
    for (int c = threadIdx.x; c < C; c += NT) io.qcnt[(size_t)u * C + c] = s_qc[c];
}

// ---- per step: the decode ---------------------------------------------------------------

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads)
k_multi_decode(MultiIo io) {
    using Gm = Geom<T, D>;
    constexpr int EPC = Gm::EPC, CPR = Gm::CPR, GPW = Gm::GPW;
    __shared__ float sm[kWarps * G * (D + 2)];
    __shared__ float s_rec[G * (2 + D)];
    __shared__ int s_qc[kMaxClusters + 1];
    // the selection may still be running (programmatic dependent launch)
    asm volatile("griddepcontrol.wait;\n" ::: "memory");
    const int u = blockIdx.x, b = u / io.Hkv, g = u - b * io.Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int li = lane % CPR, gsub = lane / CPR;
    const int C = io.C;
    const float qscale = io.scale * kLog2e;
    const T* qg = static_cast<const T*>(io.q) + ((size_t)b * io.Hq + (size_t)g * G) * D;
    const T* K = static_cast<const T*>(io.k) + (size_t)u * io.ld * D + li * EPC;
    const T* V = static_cast<const T*>(io.v) + (size_t)u * io.ld * D + li * EPC;
    if (threadIdx.x == 0) {
        int off = 0;
        for (int c = 0; c < C; ++c) {
            s_qc[c] = off;
            off += __ldcg(io.qcnt + (size_t)u * C + c);
        }
        s_qc[C] = off;
    }
    __syncthreads();
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
    const int32_t* rd = io.read + (size_t)u * io.budget;
    for (int c = warp; c < C; c += kWarps) {
        const int r0 = s_qc[c], r1 = s_qc[c + 1];
        float ks[EPC], vs[EPC];
#pragma unroll
        for (int e = 0; e < EPC; ++e) { ks[e] = 0.f; vs[e] = 0.f; }
        for (int rb = r0; rb < r1; rb += GPW) {              // warp-uniform
            const int r = rb + gsub;
            const bool ok = r < r1;
            const int p = ok ? __ldcg(rd + r) : 0;
            float kf[EPC], vf[EPC];
            unpack<T>(ok ? ld_nc16(K + (size_t)p * D) : make_uint4(0, 0, 0, 0), kf);
            unpack<T>(ok ? ld_nc16(V + (size_t)p * D) : make_uint4(0, 0, 0, 0), vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float x = 0.f;
#pragma unroll
                for (int e = 0; e < EPC; ++e) x = fmaf(qv[h][e], kf[e], x);
                x = group_sum<CPR>(x);
                if (ok) os.add(h, x, vf);
            }
#pragma unroll
            for (int e = 0; e < EPC; ++e) { ks[e] += kf[e]; vs[e] += vf[e]; }
        }
        // the cluster's read sums in every lane group, then its proxy
#pragma unroll
        for (int off = CPR; off < 32; off <<= 1)
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                ks[e] += __shfl_xor_sync(0xffffffffu, ks[e], off);
                vs[e] += __shfl_xor_sync(0xffffffffu, vs[e], off);
            }
        const int n_un = __ldg(io.cl.count + (size_t)u * C + c) - (r1 - r0);
        if (n_un > 0) {
            const float* sk = io.cl.sum_k + ((size_t)u * C + c) * D + li * EPC;
            const float* sv = io.cl.sum_v + ((size_t)u * C + c) * D + li * EPC;
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
                x = group_sum<CPR>(x) + lnn;
                if (gsub == 0) os.add(h, x, vb);
            }
        }
    }
    warp_merge<G, EPC, CPR>(os);
    cta_merge_store<G, EPC, CPR, D>(os, sm, s_rec);
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
        const int h = idx / D, e = idx - h * D;
        const float l = s_rec[G + h];
        io.out[((size_t)b * io.Hq + g * G + h) * D + e] = l > 0.f ? s_rec[2 * G + idx] / l : 0.f;
    }
}

// ---- launchers ---------------------------------------------------------------------------

template <typename T, int D>
static cudaError_t prep_t(const Dims& d, const void* k, const void* v, const sa_clusters& cl, int C, cudaStream_t s) {
    const int gx = max(1, min(cdiv(d.L, kWarps), cdiv(4 * kSmTarget, d.U())));
    k_cluster_codes<T, D><<<dim3(gx, d.U()), kThreads, 0, s>>>(static_cast<const T*>(k), cl, d.L, d.ld);
    cudaError_t e = cudaGetLastError();
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

size_t multi_workspace(const Dims& d) {
    return align256(sizeof(unsigned long long) * (size_t)d.U() * d.ld) + align256(sizeof(int) * (size_t)d.U() * d.ld);
}

template <typename T, int D, int G>
static cudaError_t multi_t(const Dims& d, const MultiIo& io, cudaStream_t s) {
    const size_t hsm = (size_t)kMaxClusters * (kThreads > 256 ? kThreads : 256) * sizeof(unsigned);
    static std::atomic<unsigned long long> opted{0};
    cudaError_t e = opt_in_smem(k_multi_select<T, D, G>, hsm, opted);
    if (e != cudaSuccess) return e;
    k_multi_select<T, D, G><<<d.U(), kThreads, hsm, s>>>(io);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(d.U());
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_multi_decode<T, D, G>, io);
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
    MultiIo io;
    io.q = q; io.k = k; io.v = v; io.cl = cl;
    io.Hq = d.Hq; io.Hkv = d.Hkv; io.L = d.L; io.ld = d.ld; io.C = cl.n_clusters; io.budget = budget;
    io.scale = scale;
    io.read = read; io.qcnt = qcnt;
    io.keys = reinterpret_cast<unsigned long long*>(ws);
    io.list = reinterpret_cast<int*>(ws + align256(sizeof(unsigned long long) * (size_t)d.U() * d.ld));
    io.out = out;
    if (d.bf16) return d.d == 128 ? multi_g<__nv_bfloat16, 128>(d, io, s) : multi_g<__nv_bfloat16, 64>(d, io, s);
    return d.d == 128 ? multi_g<float, 128>(d, io, s) : multi_g<float, 64>(d, io, s);
}

}  // namespace sa
