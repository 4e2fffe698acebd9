// Sparse decode with the residual folded into the same pass, and the dense
// flash-decode reference.
//
// k_decode<MODE>: grid (nsd, B*Hkv).  The unit's token list is
//   [sink 0..s_eff) [chosen blocks, ascending] [window L-w_eff..L) [draws]
// split evenly over the CTAs of the unit.  Each lane group gathers one token
// row at a time (16-byte loads), computes the G logits of the group's query
// heads, and keeps an fp32 online softmax (OpenAttention page: exact tokens and
// the tail handled in one online softmax).  Mode extras in the same pass:
//   RESA  : a second online softmax of the prior logits s mu_Q . K_j over I
//           (the prior terms the RESA delta merge removes at I);
//   PROXY : the sums of K and V over I (tail sums = totals minus these);
//   SAMPLE: draws enter the softmax with logit + ln(n_T / b) (vAttention
//           eq. 3 reweighting).
// The CTA that finishes the unit last combines the splits in split order and
// applies the residual (RESA Online Aggregator; proxy token) -> out[b, h, :].
//
// k_dense: grid (nsdn, B*Hkv), the same engine over all L tokens.
#include "sa_decode_core.cuh"

#include <type_traits>


namespace sa {

template <typename T, int D, int G, int MODE>
__global__ void __launch_bounds__(kThreads)
k_decode(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, sa_stats st,
         const int32_t* __restrict__ blk_idx, int kb_stride, const int32_t* __restrict__ samp_idx,
         const int32_t* __restrict__ samp_count, int sample_cap, int Hq, int Hkv, int L, int ld, SetGeom sg,
         int tok, int nsd, int rec, float qscale, float scale, float lambda,
         float* __restrict__ part, unsigned* __restrict__ cnt, float* __restrict__ out, int per_head) {
    constexpr bool PRIOR = (MODE == SA_RESA);
    constexpr bool SUMS = (MODE == SA_PROXY);
    constexpr bool SAMP = (MODE == SA_SAMPLE);
    using Gm = Geom<T, D>;
    constexpr int EPC = Gm::EPC, CPR = Gm::CPR, GPW = Gm::GPW, NG = Gm::NG;
    constexpr int kSmW = (G * (D + 2) > 2 * D) ? G * (D + 2) : 2 * D;   // per warp
    __shared__ float sm[kWarps * kSmW];
    __shared__ float s_acc[G * D];
    __shared__ float s_acc0[PRIOR ? G * D : 1];
    __shared__ float s_ml[4 * G];
    __shared__ float s_t[2 * D];
    __shared__ float s_hs[G];

    const int u = blockIdx.y, split = blockIdx.x;
    const int b = u / Hkv, g = u - b * Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int li = lane % CPR, gsub = lane / CPR;
    const size_t ubase = (size_t)u * ld * D;
    const T* K = k + ubase + li * EPC;
    const T* V = v + ubase + li * EPC;
    const T* qg = q + ((size_t)b * Hq + (size_t)g * G) * D;

    const int nt = sg.n_t;
    const bool PH = SAMP && per_head != 0;
    const int bu = (SAMP && nt > 0 && !PH) ? min(__ldg(samp_count + u), sample_cap) : 0;
    TokenMap tm;
    tm.s_eff = sg.s_eff; tm.w_eff = sg.w_eff; tm.kk = sg.kk; tm.n_i = sg.n_i; tm.win0 = L - sg.w_eff;
    tm.blk = blk_idx + (size_t)u * kb_stride;
    tm.samp = samp_idx + (size_t)u * (sample_cap > 0 ? sample_cap : 0);
    tm.lw_samp = bu > 0 ? log2f((float)nt / (float)bu) : 0.f;
    // per-head draws: head h's list (row b Hq + g G + h) follows head h-1's,
    // and a drawn token enters the softmax of its head alone
    int ph_pre[G + 1];
    float ph_lw[G];
    ph_pre[0] = 0;
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const int bh = (PH && nt > 0) ? min(__ldg(samp_count + (size_t)b * Hq + g * G + h), sample_cap) : 0;
        ph_pre[h + 1] = ph_pre[h] + bh;
        ph_lw[h] = bh > 0 ? log2f((float)nt / (float)bh) : 0.f;
    }
    const int32_t* gsamp_ph = samp_idx + ((size_t)b * Hq + (size_t)g * G) * (sample_cap > 0 ? sample_cap : 0);
    const int n_tok = sg.n_i + (PH ? ph_pre[G] : bu);

    float qv[G][EPC];
    float q0[PRIOR ? G : 1][EPC];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        float f[EPC];
        unpack<T>(ld_nc16(qg + (size_t)h * D + li * EPC), f);
#pragma unroll
        for (int e = 0; e < EPC; ++e) qv[h][e] = f[e] * qscale;
        if constexpr (PRIOR) {
#pragma unroll
            for (int e = 0; e < EPC; ++e)
                q0[h][e] = st.mu_q[((size_t)b * Hq + g * G + h) * D + li * EPC + e] * qscale;
        }
    }
    Online<G, EPC> os;
    os.init();
    Online<PRIOR ? G : 1, EPC> os0;
    os0.init();
    float ks[EPC], vs[EPC];
#pragma unroll
    for (int e = 0; e < EPC; ++e) { ks[e] = 0.f; vs[e] = 0.f; }

    const int t0 = split * tok, t1 = min(n_tok, t0 + tok);
    // warp-uniform: a warp step covers 2 x GPW tokens (2 per lane group)
    for (int wt = t0 + warp * 2 * GPW; wt < t1; wt += 2 * NG) {
        uint4 wk[2], wv[2];
        float lw[2];
        bool ok[2];
        int tag[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int t = wt + j * GPW + gsub;
            ok[j] = t < t1;
            lw[j] = 0.f;
            tag[j] = -1;
            int p = 0;
            if (ok[j] && PH && t >= sg.n_i) {
                const int x = t - sg.n_i;
                int h = 0;
#pragma unroll
                for (int y = 1; y < G; ++y) h += (x >= ph_pre[y]) ? 1 : 0;
                tag[j] = h;
#pragma unroll
                for (int y = 0; y < G; ++y) lw[j] = (y == h) ? ph_lw[y] : lw[j];
                p = __ldg(gsamp_ph + (size_t)h * sample_cap + (x - ph_pre[h]));
            } else if (ok[j]) {
                p = tm.pos(t, lw[j]);
            }
            ok[j] = ok[j] && (unsigned)p < (unsigned)L;   // a position outside the cache is skipped
            if (ok[j]) {
                const size_t off = (size_t)p * D;
                wk[j] = ld_nc16(K + off);
                wv[j] = ld_nc16(V + off);
            } else {
                wk[j] = make_uint4(0, 0, 0, 0);
                wv[j] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int t = wt + j * GPW + gsub;
            float kf[EPC], vf[EPC];
            unpack<T>(wk[j], kf);
            unpack<T>(wv[j], vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float x = 0.f;
#pragma unroll
                for (int e = 0; e < EPC; ++e) x = fmaf(qv[h][e], kf[e], x);
                x = group_sum<CPR>(x) + lw[j];
                if (ok[j] && (tag[j] < 0 || tag[j] == h)) os.add(h, x, vf);
            }
            if constexpr (PRIOR) {
                const bool exact = ok[j] && t < sg.n_i;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                    float x = 0.f;
#pragma unroll
                    for (int e = 0; e < EPC; ++e) x = fmaf(q0[h][e], kf[e], x);
                    x = group_sum<CPR>(x);
                    if (exact) os0.add(h, x, vf);
                }
            }
            if constexpr (SUMS) {
                if (ok[j] && t < sg.n_i) {
#pragma unroll
                    for (int e = 0; e < EPC; ++e) { ks[e] += kf[e]; vs[e] += vf[e]; }
                }
            }
        }
    }

    // ---- publish this split ------------------------------------------------------
    float* r = part + ((size_t)u * nsd + split) * rec;
    warp_merge<G, EPC, CPR>(os);
    cta_merge_store<G, EPC, CPR, D>(os, sm, r);
    if constexpr (PRIOR) {
        warp_merge<G, EPC, CPR>(os0);
        cta_merge_store<G, EPC, CPR, D>(os0, sm, r + G * (2 + D));
    }
    if constexpr (SUMS) {
#pragma unroll
        for (int off = CPR; off < 32; off <<= 1)
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                ks[e] += __shfl_xor_sync(0xffffffffu, ks[e], off);
                vs[e] += __shfl_xor_sync(0xffffffffu, vs[e], off);
            }
        if (lane < CPR) {
#pragma unroll
            for (int e = 0; e < EPC; ++e) {
                sm[warp * 2 * D + li * EPC + e] = ks[e];
                sm[warp * 2 * D + D + li * EPC + e] = vs[e];
            }
        }
        __syncthreads();
        for (int c = threadIdx.x; c < 2 * D; c += kThreads) {
            float s = 0.f;
            for (int w = 0; w < kWarps; ++w) s += sm[w * 2 * D + c];
            r[2 * G * (2 + D) + c] = s;
        }
    }

    if (!last_cta_of_unit(cnt + u, nsd)) return;
    decode_epilogue<T, D, G, MODE>(part + (size_t)u * nsd * rec, nsd, rec, qg, st, u, b, g, Hq, sg.n_t, scale,
                                   lambda, out, s_acc, s_acc0, s_ml, s_t, s_hs);
    reset_counter(cnt + u);
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads)
k_dense(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, int Hq, int Hkv,
        int L, int ld, int tok, int nsdn, int rec, float qscale, float* __restrict__ part,
        unsigned* __restrict__ cnt, float* __restrict__ out) {
    using Gm = Geom<T, D>;
    constexpr int EPC = Gm::EPC, CPR = Gm::CPR, GPW = Gm::GPW, NG = Gm::NG;
    __shared__ float sm[kWarps * G * (D + 2)];
    const int u = blockIdx.y, split = blockIdx.x;
    const int b = u / Hkv, g = u - b * Hkv;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int li = lane % CPR, gsub = lane / CPR;
    const size_t ubase = (size_t)u * ld * D;
    const T* K = k + ubase + li * EPC;
    const T* V = v + ubase + li * EPC;
    const T* qg = q + ((size_t)b * Hq + (size_t)g * G) * D;
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
    const int t0 = split * tok, t1 = min(L, t0 + tok);
    for (int wt = t0 + warp * 4 * GPW; wt < t1; wt += 4 * NG) {
        uint4 wk[4], wv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = wt + j * GPW + gsub;
            const bool ok = t < t1;
            wk[j] = ok ? ld_stream16(K + (size_t)t * D) : make_uint4(0, 0, 0, 0);
            wv[j] = ok ? ld_stream16(V + (size_t)t * D) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const bool ok = wt + j * GPW + gsub < t1;
            float kf[EPC], vf[EPC];
            unpack<T>(wk[j], kf);
            unpack<T>(wv[j], vf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float x = 0.f;
#pragma unroll
                for (int e = 0; e < EPC; ++e) x = fmaf(qv[h][e], kf[e], x);
                x = group_sum<CPR>(x);
                if (ok) os.add(h, x, vf);
            }
        }
    }
    float* r = part + ((size_t)u * nsdn + split) * rec;
    warp_merge<G, EPC, CPR>(os);
    cta_merge_store<G, EPC, CPR, D>(os, sm, r);
    if (!last_cta_of_unit(cnt + u, nsdn)) return;
    const float* recs = part + (size_t)u * nsdn * rec;
    for (int idx = threadIdx.x; idx < G * D; idx += kThreads) {
        const int h = idx / D, e = idx - h * D;
        float M, Ls;
        const float A = combine_splits<G, D>(recs, nsdn, rec, h, e, M, Ls);
        out[((size_t)b * Hq + g * G + h) * D + e] = A / Ls;
    }
    reset_counter(cnt + u);
}


// ---- dispatch ----------------------------------------------------------------

template <int D, int G, int MODE>
static cudaError_t stream_launch(const Dims& d, dim3 grid, const void* q, const void* k, const void* v,
                                 const sa_stats& st, const sa_selection& sel, const sa_select_params& sp,
                                 const SetGeom& sg, int tpc, int nchunk, int rec, float scale, float lambda,
                                 char* part, char* cnt, float* out, bool pdl, cudaStream_t s) {
    constexpr size_t sm = stream_smem<D, G, MODE>();
    static std::atomic<unsigned long long> opted{0};
    cudaError_t e = opt_in_smem(k_stream_tc<D, G, MODE>, sm, opted);
    if (e != cudaSuccess) return e;
    StreamIo io;
    io.q = reinterpret_cast<const __nv_bfloat16*>(q);
    io.k = reinterpret_cast<const __nv_bfloat16*>(k);
    io.v = reinterpret_cast<const __nv_bfloat16*>(v);
    io.st = st;
    io.blk_idx = sel.blk_idx;
    io.kb_stride = sp.k_blocks;
    io.samp_idx = sel.samp_idx;
    io.samp_count = sel.samp_count;
    io.sample_cap = sp.sample_cap;
    io.Hq = d.Hq; io.Hkv = d.Hkv; io.L = d.L; io.ld = d.ld;
    io.sg = sg;
    io.tpc = tpc; io.nchunk = nchunk; io.rec = rec;
    io.qscale = scale * kLog2e; io.scale = scale; io.lambda = lambda;
    io.part = reinterpret_cast<float*>(part);
    io.cnt = reinterpret_cast<unsigned*>(cnt);
    io.out = out;
    io.per_head = sp.per_head;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = sm;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_stream_tc<D, G, MODE>, io);
}

template <typename T, int D, int G, int MODE>
static cudaError_t decode_m(const Dims& d, const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        return stream_launch<D, G, MODE>(d, dim3(p.nsd, d.U()), a.q, a.k, a.v, a.st, a.sel, a.sp, p.g, p.tok_d,
                                         p.nsd, p.rec, a.scale, a.dp.lambda, a.ws + p.off_part, a.ws + p.off_cnt,
                                         a.out, a.pdl, s);
    } else {
        k_decode<T, D, G, MODE><<<dim3(p.nsd, d.U()), kThreads, 0, s>>>(
            reinterpret_cast<const T*>(a.q), reinterpret_cast<const T*>(a.k), reinterpret_cast<const T*>(a.v),
            a.st, a.sel.blk_idx, a.sp.k_blocks, a.sel.samp_idx, a.sel.samp_count, a.sp.sample_cap,
            d.Hq, d.Hkv, d.L, d.ld, p.g, p.tok_d, p.nsd, p.rec, a.scale * kLog2e, a.scale, a.dp.lambda,
            reinterpret_cast<float*>(a.ws + p.off_part), reinterpret_cast<unsigned*>(a.ws + p.off_cnt), a.out,
            a.sp.per_head);
        return cudaGetLastError();
    }
}

template <typename T, int D, int G>
static cudaError_t decode_t(const Dims& d, const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
    switch (a.dp.mode) {
        case SA_DROP: return decode_m<T, D, G, SA_DROP>(d, p, a, s);
        case SA_RESA: return decode_m<T, D, G, SA_RESA>(d, p, a, s);
        case SA_PROXY: return decode_m<T, D, G, SA_PROXY>(d, p, a, s);
        case SA_SAMPLE: return decode_m<T, D, G, SA_SAMPLE>(d, p, a, s);
    }
    return cudaErrorInvalidValue;
}

template <typename T, int D>
static cudaError_t decode_g(const Dims& d, const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
    switch (d.G) {
        case 1: return decode_t<T, D, 1>(d, p, a, s);
        case 2: return decode_t<T, D, 2>(d, p, a, s);
        case 4: return decode_t<T, D, 4>(d, p, a, s);
        case 8: return decode_t<T, D, 8>(d, p, a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const Dims& d, const DecodePlan& p, const DecodeArgs& a, cudaStream_t s) {
    if (d.bf16) return d.d == 128 ? decode_g<__nv_bfloat16, 128>(d, p, a, s) : decode_g<__nv_bfloat16, 64>(d, p, a, s);
    return d.d == 128 ? decode_g<float, 128>(d, p, a, s) : decode_g<float, 64>(d, p, a, s);
}

template <int D, int G>
static cudaError_t prefill_stream_t(const Dims& d, const PrefillPlan& p, const void* k, const void* v,
                                    const sa_stats& st, float scale, char* part, char* cnt, cudaStream_t s) {
    SetGeom sg{};
    sa_selection sel{};
    sa_select_params sp{};
    return stream_launch<D, G, kPrefillMode>(d, dim3(p.nsp, d.U()), nullptr, k, v, st, sel, sp, sg, p.tpc, p.nsp,
                                             p.rec_p, scale, 1.f, part, cnt, nullptr, false, s);
}

template <int D>
static cudaError_t prefill_stream_g(const Dims& d, const PrefillPlan& p, const void* k, const void* v,
                                    const sa_stats& st, float scale, char* part, char* cnt, cudaStream_t s) {
    switch (d.G) {
        case 1: return prefill_stream_t<D, 1>(d, p, k, v, st, scale, part, cnt, s);
        case 2: return prefill_stream_t<D, 2>(d, p, k, v, st, scale, part, cnt, s);
        case 4: return prefill_stream_t<D, 4>(d, p, k, v, st, scale, part, cnt, s);
        case 8: return prefill_stream_t<D, 8>(d, p, k, v, st, scale, part, cnt, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_prefill_stream(const Dims& d, const PrefillPlan& p, const void* k, const void* v,
                                  const sa_stats& st, float scale, char* part, char* cnt, cudaStream_t s) {
    if (!d.bf16) return cudaErrorInvalidValue;
    return d.d == 128 ? prefill_stream_g<128>(d, p, k, v, st, scale, part, cnt, s)
                      : prefill_stream_g<64>(d, p, k, v, st, scale, part, cnt, s);
}

template <typename T, int D, int G>
static cudaError_t dense_t(const Dims& d, const DensePlan& p, const DenseArgs& a, cudaStream_t s) {
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        SetGeom sg{};
        sa_stats st{};
        sa_selection sel{};
        sa_select_params sp{};
        return stream_launch<D, G, kDenseMode>(d, dim3(p.nsdn, d.U()), a.q, a.k, a.v, st, sel, sp, sg,
                                               p.tok / kTcTile, p.nsdn, p.rec, a.scale, 1.f, a.ws + p.off_part,
                                               a.ws + p.off_cnt, a.out, false, s);
    } else {
        k_dense<T, D, G><<<dim3(p.nsdn, d.U()), kThreads, 0, s>>>(
            reinterpret_cast<const T*>(a.q), reinterpret_cast<const T*>(a.k), reinterpret_cast<const T*>(a.v),
            d.Hq, d.Hkv, d.L, d.ld, p.tok, p.nsdn, p.rec, a.scale * kLog2e,
            reinterpret_cast<float*>(a.ws + p.off_part), reinterpret_cast<unsigned*>(a.ws + p.off_cnt), a.out);
        return cudaGetLastError();
    }
}

template <typename T, int D>
static cudaError_t dense_g(const Dims& d, const DensePlan& p, const DenseArgs& a, cudaStream_t s) {
    switch (d.G) {
        case 1: return dense_t<T, D, 1>(d, p, a, s);
        case 2: return dense_t<T, D, 2>(d, p, a, s);
        case 4: return dense_t<T, D, 4>(d, p, a, s);
        case 8: return dense_t<T, D, 8>(d, p, a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_dense(const Dims& d, const DensePlan& p, const DenseArgs& a, cudaStream_t s) {
    if (d.bf16) return d.d == 128 ? dense_g<__nv_bfloat16, 128>(d, p, a, s) : dense_g<__nv_bfloat16, 64>(d, p, a, s);
    return d.d == 128 ? dense_g<float, 128>(d, p, a, s) : dense_g<float, 64>(d, p, a, s);
}

}  // namespace sa
