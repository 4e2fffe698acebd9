// Tensor-core attention tile engine for bf16 caches (sm_100a, warp-level
// mma.sync m16n8k16 bf16 -> fp32, operands through ldmatrix).
//
// The contraction per unit is skinny (G <= 8 query heads against a run of
// keys), so tensor cores are used only to take the multiply-adds off the
// ALUs and keep the gather HBM-bound; the matrices are laid out so that
// nothing is converted on the way in (bf16 rows feed ldmatrix directly).
//
// One warp owns 16 cache rows (tokens) of a shared-memory tile:
//   S^T  = Q   K^T : A = query rows (heads in M, zero-padded to 16), B = K rows
//   O   += P   V   : A = softmax weights (heads in M), B = V rows (ldmatrix.trans)
// M rows 0..G-1 carry the exact logits / weights of the G heads.  For the RESA
// prior, a second A operand holds mu_Q split into bf16 hi (rows 0..G-1) and lo
// (rows 8..8+G-1) parts, so hi.K + lo.K gives the prior logit at fp32-level
// accuracy, and the PV step carries the prior weights in rows 8..8+G-1 of the
// same MMA.  Softmax weights P (in [0,1]) are split into bf16 hi + lo and
// multiplied twice, which keeps ~16 significant bits of each weight.
#pragma once

#include "sa_common.cuh"

namespace sa {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mma_bf16(float* c, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void cp16(uint32_t saddr, const void* g) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(saddr), "l"(g) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

__device__ __forceinline__ void st_zero16(uint32_t saddr) {
    asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(saddr), "r"(0) : "memory");
}

__device__ __forceinline__ uint32_t bf2(float lo_elem, float hi_elem) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
    return *reinterpret_cast<uint32_t*>(&v);
}

// x = hi + lo with hi, lo bf16 (both rounded to nearest)
__device__ __forceinline__ void split_bf2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<uint32_t*>(&h);
    lo = *reinterpret_cast<uint32_t*>(&l);
}

// Row pitch of a shared-memory tile in bf16 elements: 16 bytes of padding
// per row puts the 8 rows an ldmatrix reads in 8 different bank groups.
template <int D>
struct Pitch {
    static constexpr int kElems = D + 8;
    static constexpr int kBytes = kElems * 2;
};

// Per-warp online softmax state and accumulators for 16-token steps.
// Lane (g = lane/4, t = lane%4) holds head g (if g < G): its logits for the
// tokens 2t, 2t+1, 8+2t, 9+2t of each step, and o[nt][0..1] = exact
// accumulator of dims nt*8+2t, +1; o[nt][2..3] = prior accumulator.
template <int D, int G, bool PRIOR>
struct WarpAttn {
    static constexpr int KS = D / 16;   // k-steps over the head dim
    static constexpr int NT = D / 8;    // 8-wide output tiles
    uint32_t qa[KS][2];                 // exact A: a0 (dims 2t..), a2 (dims 8+2t..), rows 0..G-1
    uint32_t pa[PRIOR ? KS : 1][4];     // prior A: hi rows 0..G-1 (a0, a2), lo rows 8.. (a1, a3)
    float o[NT][4];
    float m, l, m0, l0;

    // q_row: pointer to the bf16 query of head g (only read when g < G; null
    // for none: zero logits);
    // mu_row: fp32 typical query of head g (PRIOR only)
    __device__ __forceinline__ void init(const __nv_bfloat16* q_row, const float* mu_row) {
        const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            uint32_t a0 = 0, a2 = 0;
            if (g < G && q_row != nullptr) {
                a0 = *reinterpret_cast<const uint32_t*>(q_row + ks * 16 + 2 * t);
                a2 = *reinterpret_cast<const uint32_t*>(q_row + ks * 16 + 8 + 2 * t);
            }
            qa[ks][0] = a0;
            qa[ks][1] = a2;
            if constexpr (PRIOR) {
                uint32_t h0 = 0, l0_ = 0, h2 = 0, l2 = 0;
                if (g < G) {
                    const float2 x = *reinterpret_cast<const float2*>(mu_row + ks * 16 + 2 * t);
                    const float2 y = *reinterpret_cast<const float2*>(mu_row + ks * 16 + 8 + 2 * t);
                    split_bf2(x.x, x.y, h0, l0_);
                    split_bf2(y.x, y.y, h2, l2);
                }
                pa[ks][0] = h0; pa[ks][1] = l0_; pa[ks][2] = h2; pa[ks][3] = l2;
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 4; ++j) o[nt][j] = 0.f;
        m = -INFINITY; l = 0.f; m0 = -INFINITY; l0 = 0.f;
    }

    // One online-softmax update of a head over 4 logits (x already in log2
    // units, -inf = masked); returns the weights through p and rescales acc
    // columns [c0, c0+2) of o by the change of maximum.
    __device__ __forceinline__ void online(float (&x)[4], float& mm, float& ll, int c0) {
        float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mn = fmaxf(mm, mx);
        const float sc = (mm == -INFINITY) ? 0.f : ex2(mm - mn);
        float ls = 0.f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            x[j] = (x[j] == -INFINITY) ? 0.f : ex2(x[j] - mn);
            ls += x[j];
        }
        ls += __shfl_xor_sync(0xffffffffu, ls, 1);
        ls += __shfl_xor_sync(0xffffffffu, ls, 2);
        if (mn != -INFINITY) {
            ll = ll * sc + ls;
            if (mm != mn) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) { o[nt][c0] *= sc; o[nt][c0 + 1] *= sc; }
            }
            mm = mn;
        }
    }

    // 16 tokens at shared rows [r0, r0+16) of the K and V tiles (byte
    // addresses of row 0).  xadd[j]: log2-weight added to token j's exact
    // logit (-inf masks it); in_i[j]: token j belongs to I (prior counts it).
    // Token order per lane: j=0,1 -> rows 2t, 2t+1; j=2,3 -> rows 8+2t, 9+2t.
    __device__ __forceinline__ void step16(uint32_t k_tile, uint32_t v_tile, int r0, const float (&xadd)[4],
                                           const bool (&in_i)[4], float qscale) {
        constexpr int P = Pitch<D>::kBytes;
        const int lane = threadIdx.x & 31, g = lane >> 2;
        float s[2][4], s0[2][4];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int j = 0; j < 4; ++j) { s[n][j] = 0.f; s0[n][j] = 0.f; }
#pragma unroll
        for (int kp = 0; kp < KS / 2; ++kp) {
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                uint32_t b[4];
                ldsm4(k_tile + (r0 + n * 8 + (lane & 7)) * P + (kp * 32 + (lane >> 3) * 8) * 2, b);
                mma_bf16(s[n], qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, b[0], b[1]);
                mma_bf16(s[n], qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, b[2], b[3]);
                if constexpr (PRIOR) {
                    mma_bf16(s0[n], pa[2 * kp][0], pa[2 * kp][1], pa[2 * kp][2], pa[2 * kp][3], b[0], b[1]);
                    mma_bf16(s0[n], pa[2 * kp + 1][0], pa[2 * kp + 1][1], pa[2 * kp + 1][2], pa[2 * kp + 1][3],
                             b[2], b[3]);
                }
            }
        }
        const bool head = g < G;
        float x[4], y[4];
#pragma unroll
        for (int n = 0; n < 2; ++n)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int i = 2 * n + j;
                x[i] = head ? fmaf(s[n][j], qscale, xadd[i]) : -INFINITY;
                if constexpr (PRIOR) y[i] = (head && in_i[i]) ? (s0[n][j] + s0[n][j + 2]) * qscale : -INFINITY;
            }
        online(x, m, l, 0);
        uint32_t ah[4], al[4];
        split_bf2(x[0], x[1], ah[0], al[0]);
        split_bf2(x[2], x[3], ah[2], al[2]);
        if constexpr (PRIOR) {
            online(y, m0, l0, 2);
            split_bf2(y[0], y[1], ah[1], al[1]);
            split_bf2(y[2], y[3], ah[3], al[3]);
        } else {
            ah[1] = al[1] = ah[3] = al[3] = 0u;
        }
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
            uint32_t b[4];
            ldsm4t(v_tile + (r0 + ((lane >> 3) & 1) * 8 + (lane & 7)) * P + (np * 16 + (lane >> 4) * 8) * 2, b);
            mma_bf16(o[2 * np], ah[0], ah[1], ah[2], ah[3], b[0], b[1]);
            mma_bf16(o[2 * np], al[0], al[1], al[2], al[3], b[0], b[1]);
            mma_bf16(o[2 * np + 1], ah[0], ah[1], ah[2], ah[3], b[2], b[3]);
            mma_bf16(o[2 * np + 1], al[0], al[1], al[2], al[3], b[2], b[3]);
        }
    }

    // Store this warp's state into shared arrays for the cross-warp merge:
    // ml[w][h][0..3] = m, l, m0, l0; acc[w][h][d] exact; acc0[w][h][d] prior.
    __device__ __forceinline__ void store(float* ml, float* acc, float* acc0) const {
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
        if (g < G) {
            float* a = acc + (warp * G + g) * D;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                a[nt * 8 + 2 * t] = o[nt][0];
                a[nt * 8 + 2 * t + 1] = o[nt][1];
            }
            if constexpr (PRIOR) {
                float* a0 = acc0 + (warp * G + g) * D;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    a0[nt * 8 + 2 * t] = o[nt][2];
                    a0[nt * 8 + 2 * t + 1] = o[nt][3];
                }
            }
            if (t == 0) {
                float* r = ml + (warp * G + g) * 4;
                r[0] = m; r[1] = l; r[2] = m0; r[3] = l0;
            }
        }
    }
};

// Tokens-on-M engine for G <= 4 (the usual GQA groups): the 16 tokens of a
// warp are the M rows, the query columns the N dimension, so no MMA row is
// spent on absent heads:
//   S^T = K Q^T : A = K rows (ldmatrix), B = query columns in registers
//                 (tile 0: q_0..q_{G-1}, then mu_Q hi of the G heads;
//                  tile 1, RESA only: mu_Q lo at the same columns)
//   O^T += V^T P^T : A = V rows (ldmatrix.trans), B = the weights, moved from
//                 the S layout to the B layout with movmatrix.trans
// Columns 0..G-1 carry the exact logits / weights and output, columns
// G..2G-1 the RESA prior ones, so one 8-column MMA holds both.  Lane
// (g = lane/4, t = lane%4) holds tokens g and g+8 of the step and columns
// 2t, 2t+1; its O^T entries are dims (16 mt + g, + 8) of those columns.
template <int D, int G, bool PRIOR>
struct WarpAttnT {
    static_assert(G <= 4, "the exact and prior columns share one 8-column tile");
    static constexpr int KS = D / 16;   // k-steps over the head dim
    static constexpr int MT = D / 16;   // 16-dim output tiles
    static constexpr int NQ = PRIOR ? 2 : 1;
    static constexpr int kRows = 2;     // token rows per lane per step
    uint32_t qb[NQ][KS][2];
    float o[MT][4];
    float m[2], l[2];

    // tile row of this lane's token j (0, 1) in the 16-token group at r0
    __device__ static __forceinline__ int row(int r0, int j) { return r0 + ((threadIdx.x & 31) >> 2) + 8 * j; }

    // init in two halves: load issues this lane's operand loads into raw
    // (qg: the G bf16 query rows of the unit, null for none (zero logits);
    // mu: the G fp32 typical queries, PRIOR only), finish forms the B fragments and clears the state once
    // they have landed, so other work can sit between the two.
    float2 raw[KS][2];
    __device__ __forceinline__ void load(const __nv_bfloat16* qg, const float* mu) {
        const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int dim = ks * 16 + 2 * t + 8 * half;
                float2 x = make_float2(0.f, 0.f);
                if (g < G) {
                    if (qg != nullptr) x.x = __uint_as_float(*reinterpret_cast<const uint32_t*>(qg + (size_t)g * D + dim));
                }
                else if (PRIOR && g < 2 * G)
                    x = *reinterpret_cast<const float2*>(mu + (size_t)(g - G) * D + dim);
                raw[ks][half] = x;
            }
        }
    }
    __device__ __forceinline__ void finish() {
        const int g = (threadIdx.x & 31) >> 2;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t v0 = 0u, v1 = 0u;
                if (g < G) v0 = __float_as_uint(raw[ks][half].x);
                else if (PRIOR && g < 2 * G) split_bf2(raw[ks][half].x, raw[ks][half].y, v0, v1);
                qb[0][ks][half] = v0;
                if constexpr (PRIOR) qb[NQ - 1][ks][half] = v1;
            }
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int j = 0; j < 4; ++j) o[mt][j] = 0.f;
        m[0] = m[1] = -INFINITY;
        l[0] = l[1] = 0.f;
    }
    __device__ __forceinline__ void init(const __nv_bfloat16* qg, const float* mu) {
        load(qg, mu);
        finish();
    }

    __device__ static __forceinline__ uint32_t trans8(uint32_t x) {
        uint32_t y;
        asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
        return y;
    }

    // 16 tokens at tile rows [r0, r0+16): xadd[j][e] = log2-weight added to
    // the exact logit of token row(r0, j) in this lane's column 2t + e (-inf
    // masks it for that head); in_i[j]: the token belongs to I
    __device__ __forceinline__ void step16(uint32_t k_tile, uint32_t v_tile, int r0, const float (&xadd)[2][2],
                                           const bool (&in_i)[2], float qscale) {
        constexpr int P = Pitch<D>::kBytes;
        const int lane = threadIdx.x & 31, t = lane & 3;
        // even and odd k-steps accumulate apart (two short MMA chains), summed after
        float s2[2][NQ][4];
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int nq = 0; nq < NQ; ++nq)
#pragma unroll
                for (int j = 0; j < 4; ++j) s2[c][nq][j] = 0.f;
        const uint32_t ka = k_tile + (r0 + (lane & 7) + ((lane >> 3) & 1) * 8) * P + (lane >> 4) * 16;
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
            uint32_t a[4];
            ldsm4(ka + ks * 32, a);
#pragma unroll
            for (int nq = 0; nq < NQ; ++nq)
                mma_bf16(s2[ks & 1][nq], a[0], a[1], a[2], a[3], qb[nq][ks][0], qb[nq][ks][1]);
        }
        float s[NQ][4];
#pragma unroll
        for (int nq = 0; nq < NQ; ++nq)
#pragma unroll
            for (int j = 0; j < 4; ++j) s[nq][j] = s2[0][nq][j] + s2[1][nq][j];
        // logits of the lane's two tokens (j) and two columns (e)
        float p[2][2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int c = 2 * t + e;
            float x[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                if (c < G) x[j] = fmaf(s[0][2 * j + e], qscale, xadd[j][e]);
                else if (PRIOR && c < 2 * G) x[j] = in_i[j] ? (s[0][2 * j + e] + s[NQ - 1][2 * j + e]) * qscale : -INFINITY;
                else x[j] = -INFINITY;
            }
            // online softmax of column c over the 16 tokens (lanes with this t)
            float mx = fmaxf(x[0], x[1]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 4));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
            const float mn = fmaxf(m[e], mx);
            const float sc = (m[e] == -INFINITY) ? 0.f : ex2(m[e] - mn);
#pragma unroll
            for (int j = 0; j < 2; ++j) p[j][e] = (x[j] == -INFINITY) ? 0.f : ex2(x[j] - mn);
            float ls = p[0][e] + p[1][e];
            ls += __shfl_xor_sync(0xffffffffu, ls, 4);
            ls += __shfl_xor_sync(0xffffffffu, ls, 8);
            ls += __shfl_xor_sync(0xffffffffu, ls, 16);
            if (mn != -INFINITY) {
                l[e] = l[e] * sc + ls;
                if (m[e] != mn) {
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) { o[mt][e] *= sc; o[mt][2 + e] *= sc; }
                }
                m[e] = mn;
            }
        }
        // weights -> bf16 hi + lo, S layout (token, column pair) -> B layout
        uint32_t h0, l0, h1, l1;
        split_bf2(p[0][0], p[0][1], h0, l0);      // token g
        split_bf2(p[1][0], p[1][1], h1, l1);      // token g + 8
        const uint32_t bh0 = trans8(h0), bh1 = trans8(h1), bl0 = trans8(l0), bl1 = trans8(l1);
        const uint32_t va = v_tile + (r0 + (lane & 7) + ((lane >> 4) & 1) * 8) * P + ((lane >> 3) & 1) * 16;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            uint32_t a[4];
            ldsm4t(va + mt * 32, a);
            mma_bf16(o[mt], a[0], a[1], a[2], a[3], bh0, bh1);
            mma_bf16(o[mt], a[0], a[1], a[2], a[3], bl0, bl1);
        }
    }

    // this warp's state into the arrays merge_warps reads (as WarpAttn::store)
    __device__ __forceinline__ void store(float* ml, float* acc, float* acc0) const {
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, g = lane >> 2, t = lane & 3;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int c = 2 * t + e;
            const bool exact = c < G, prior = PRIOR && c >= G && c < 2 * G;
            if (!exact && !prior) continue;
            const int h = exact ? c : c - G;
            float* a = (exact ? acc : acc0) + (warp * G + h) * D;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                a[mt * 16 + g] = o[mt][e];
                a[mt * 16 + g + 8] = o[mt][2 + e];
            }
            if (g == 0) {
                float* r = ml + (warp * G + h) * 4 + (exact ? 0 : 2);
                r[0] = m[e];
                r[1] = l[e];
            }
        }
        if constexpr (!PRIOR) {
            if (lane < G) {                      // the prior slots of a record without prior
                float* r = ml + (warp * G + lane) * 4;
                r[2] = -INFINITY;
                r[3] = 0.f;
            }
        }
    }
};

// Merge the stored states of `nw` warps (fixed warp order) into a split record
// m[G], l[G], acc[G][D] (and the prior record right after it when PRIOR).
template <int D, int G, bool PRIOR>
__device__ __forceinline__ void merge_warps(const float* ml, const float* acc, const float* acc0, int nw,
                                            float* rec) {
    for (int idx = threadIdx.x; idx < G * D * (PRIOR ? 2 : 1); idx += blockDim.x) {
        const int pr = idx >= G * D;
        const int r = idx - pr * G * D;
        const int h = r / D, e = r - h * D;
        float M = -INFINITY;
        for (int w = 0; w < nw; ++w) M = fmaxf(M, ml[(w * G + h) * 4 + 2 * pr]);
        float A = 0.f, Ls = 0.f;
        for (int w = 0; w < nw; ++w) {
            const float mw = ml[(w * G + h) * 4 + 2 * pr];
            const float f = (mw == -INFINITY) ? 0.f : ex2(mw - M);
            A = fmaf((pr ? acc0 : acc)[(w * G + h) * D + e], f, A);
            Ls = fmaf(ml[(w * G + h) * 4 + 2 * pr + 1], f, Ls);
        }
        float* rr = rec + pr * G * (2 + D);
        rr[2 * G + h * D + e] = A;
        if (e == 0) { rr[h] = M; rr[G + h] = Ls; }
    }
}

}  // namespace tc
}  // namespace sa
