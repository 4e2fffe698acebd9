// C ABI of libsa_b200.so (declared in include/sa_decode.h): argument checks,
// workspace sizing, and dispatch to the kernel launchers.  Every check runs
// before anything is enqueued, so a rejected call leaves the stream untouched.
#include <math.h>
#include <nvtx3/nvToolsExt.h>

#include "sa_internal.h"

using namespace sa;

namespace {

struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

sa_status check_shape(const sa_shape* s, Dims* d) {
    if (s == nullptr) return SA_ERR_INVALID_ARG;
    if (s->B < 1 || s->Hkv < 1 || s->Hq < 1 || s->L < 16 || s->d < 1) return SA_ERR_INVALID_ARG;
    const int ld = s->ld == 0 ? s->L : s->ld;
    if (s->Hq % s->Hkv != 0 || ld % 16 != 0 || ld < s->L) return SA_ERR_INVALID_ARG;
    if (s->dtype != SA_F32 && s->dtype != SA_BF16) return SA_ERR_INVALID_ARG;
    const int G = s->Hq / s->Hkv;
    if (G != 1 && G != 2 && G != 4 && G != 8) return SA_ERR_UNSUPPORTED;
    if (s->d != 64 && s->d != 128) return SA_ERR_UNSUPPORTED;
    if ((long long)ld * s->d >= (1LL << 31) || (long long)s->B * s->Hq >= 65536 ||
        (long long)s->B * s->Hkv >= 65536)
        return SA_ERR_UNSUPPORTED;
    d->B = s->B; d->Hq = s->Hq; d->Hkv = s->Hkv; d->G = G; d->d = s->d; d->L = s->L; d->ld = ld;
    d->bf16 = s->dtype == SA_BF16;
    return SA_OK;
}

sa_status check_select_params(const sa_select_params* p) {
    if (p == nullptr) return SA_ERR_INVALID_ARG;
    if (p->sink < 0 || p->local < 0 || p->k_blocks < 0 || p->sample_b < 0 || p->sample_cap < 0 ||
        p->clt_base < 0)
        return SA_ERR_INVALID_ARG;
    if (p->sample_b > p->sample_cap) return SA_ERR_INVALID_ARG;
    if (p->score != SA_SCORE_MEAN_SUM && p->score != SA_SCORE_MEAN_MAX && p->score != SA_SCORE_QUEST)
        return SA_ERR_INVALID_ARG;
    if (p->budget != SA_BUDGET_CLT && p->budget != SA_BUDGET_CLT_SEARCH && p->budget != SA_BUDGET_HOEFFDING)
        return SA_ERR_INVALID_ARG;
    if (p->per_head != 0 && p->per_head != 1) return SA_ERR_INVALID_ARG;
    if (p->clt_base > 0) {
        if (p->clt_base < 2 || p->clt_base > p->sample_cap) return SA_ERR_INVALID_ARG;
        if (!(p->eps > 0.f) || !(p->delta > 0.f && p->delta < 1.f)) return SA_ERR_INVALID_ARG;
        if (p->clt_base > kCltMaxBase) return SA_ERR_UNSUPPORTED;
    }
    return SA_OK;
}

bool check_stats(const sa_stats* st, bool need_all) {
    if (st == nullptr) return false;
    // the block bounds come as a pair, or not at all
    if ((st->blk_min == nullptr) != (st->blk_max == nullptr)) return false;
    if (st->blk_min != nullptr && (!aligned16(st->blk_min) || !aligned16(st->blk_max))) return false;
    if (!aligned16(st->blk_mean) || !aligned4(st->kbar_absmax) || !aligned16(st->blk_code) ||
        !aligned16(st->blk_meta))
        return false;
    if (need_all) {
        if (!aligned16(st->mu_q) || !aligned16(st->o_est) || !aligned4(st->log_z0) ||
            !aligned16(st->mu_k) || !aligned16(st->sum_k) || !aligned16(st->sum_v))
            return false;
    }
    return true;
}

float resolve_scale(float scale, int d) { return scale > 0.f ? scale : (float)(1.0 / sqrt((double)d)); }

}  // namespace

extern "C" {

sa_status sa_wait_timeouts(unsigned* count) {
    if (count == nullptr) return SA_ERR_INVALID_ARG;
    return sa::select_wait_timeouts(count) == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

const char* sa_status_string(sa_status s) {
    switch (s) {
        case SA_OK: return "ok";
        case SA_ERR_INVALID_ARG: return "invalid argument";
        case SA_ERR_UNSUPPORTED: return "unsupported configuration";
        case SA_ERR_WORKSPACE: return "workspace missing or too small";
        case SA_ERR_CUDA: return "CUDA launch failed";
    }
    return "unknown status";
}

size_t sa_workspace_size(const sa_shape* shape, const sa_select_params* params, int op) {
    Dims d;
    if (check_shape(shape, &d) != SA_OK) return 0;
    switch (op) {
        case SA_OP_PREFILL: return prefill_plan(d).bytes;
        case SA_OP_DENSE: return dense_plan(d).bytes;
        case SA_OP_SELECT:
            if (check_select_params(params) != SA_OK) return 0;
            return select_plan(d, *params).bytes;
        case SA_OP_DECODE:
            if (check_select_params(params) != SA_OK) return 0;
            return decode_plan(d, *params).bytes;
        case SA_OP_STEP:
            if (check_select_params(params) != SA_OK) return 0;
            return select_plan(d, *params).bytes + decode_plan(d, *params).bytes;
        case SA_OP_MULTI: return multi_workspace(d);
        case SA_OP_CLUSTER: return qgc_plan(d).bytes;
    }
    return 0;
}

sa_status sa_prefill_stats(const sa_shape* shape, const void* q_ctx, const void* k, const void* v,
                           const sa_stats* out, float scale, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange r("sa_prefill_stats");
    Dims d;
    sa_status e = check_shape(shape, &d);
    if (e != SA_OK) return e;
    if (d.L % 16 != 0) return SA_ERR_INVALID_ARG;     // the statistics cover whole blocks
    if (!aligned16(q_ctx) || !aligned16(k) || !aligned16(v) || !check_stats(out, true) || scale < 0.f)
        return SA_ERR_INVALID_ARG;
    const PrefillPlan p = prefill_plan(d);
    if (ws == nullptr || ws_bytes < p.bytes || !aligned16(ws)) return SA_ERR_WORKSPACE;
    PrefillArgs a{q_ctx, k, v, *out, resolve_scale(scale, d.d), static_cast<char*>(ws)};
    return launch_prefill(d, p, a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status sa_block_summaries(const sa_shape* shape, const void* k, int blk_begin, int blk_end, void* blk_mean,
                             float* kbar_absmax, const float* mu_k, int8_t* blk_code, float* blk_meta,
                             void* stream) {
    NvtxRange r("sa_block_summaries");
    Dims d;
    sa_status e = check_shape(shape, &d);
    if (e != SA_OK) return e;
    if (!aligned16(k) || !aligned16(blk_mean) || !aligned4(kbar_absmax) || !aligned4(mu_k) ||
        !aligned16(blk_code) || !aligned16(blk_meta))
        return SA_ERR_INVALID_ARG;
    if (blk_begin < 0 || blk_end > d.nb() || blk_begin > blk_end) return SA_ERR_INVALID_ARG;
    if (blk_begin == blk_end) return SA_OK;
    return launch_block_summaries(d, k, blk_begin, blk_end, blk_mean, kbar_absmax, mu_k, blk_code, blk_meta,
                                  static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SA_OK
               : SA_ERR_CUDA;
}

sa_status sa_append(const sa_shape* shape, const void* k_new, const void* v_new, void* k, void* v,
                    const sa_stats* stats, float scale, void* stream) {
    NvtxRange r("sa_append");
    Dims d;
    sa_status e = check_shape(shape, &d);
    if (e != SA_OK) return e;
    if (d.L >= d.ld) return SA_ERR_INVALID_ARG;       // no room for the token
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k) || !aligned16(v) || !check_stats(stats, true) ||
        scale < 0.f)
        return SA_ERR_INVALID_ARG;
    return launch_append(d, k_new, v_new, k, v, *stats, resolve_scale(scale, d.d),
                         static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SA_OK
               : SA_ERR_CUDA;
}

sa_status sa_block_minmax(const sa_shape* shape, const void* k, int blk_begin, int blk_end, void* blk_min,
                          void* blk_max, void* stream) {
    NvtxRange r("sa_block_minmax");
    Dims d;
    sa_status e = check_shape(shape, &d);
    if (e != SA_OK) return e;
    if (!aligned16(k) || !aligned16(blk_min) || !aligned16(blk_max)) return SA_ERR_INVALID_ARG;
    if (blk_begin < 0 || blk_end > d.nb() || blk_begin > blk_end) return SA_ERR_INVALID_ARG;
    if (blk_begin == blk_end) return SA_OK;
    return launch_block_minmax(d, k, blk_begin, blk_end, blk_min, blk_max, static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? SA_OK
               : SA_ERR_CUDA;
}

sa_status sa_block_sketch(const sa_shape* shape, const void* blk_mean, const float* mu_k, int blk_begin,
                          int blk_end, int8_t* blk_code, float* blk_meta, void* stream) {
    NvtxRange r("sa_block_sketch");
    Dims d;
    sa_status e = check_shape(shape, &d);
    if (e != SA_OK) return e;
    if (!aligned16(blk_mean) || !aligned4(mu_k) || !aligned16(blk_code) || !aligned16(blk_meta))
        return SA_ERR_INVALID_ARG;
    if (blk_begin < 0 || blk_end > d.nb() || blk_begin > blk_end) return SA_ERR_INVALID_ARG;
    if (blk_begin == blk_end) return SA_OK;
    return launch_block_sketch(d, blk_mean, mu_k, blk_begin, blk_end, blk_code, blk_meta,
                               static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SA_OK
               : SA_ERR_CUDA;
}

}  // extern "C"

namespace {

sa_status prep_select(const sa_shape* shape, const sa_select_params* params, const void* q, const sa_stats* stats,
                      const void* k, const void* v, const sa_selection* out, float scale, Dims* d,
                      SelectPlan* p, SelectArgs* a) {
    sa_status e = check_shape(shape, d);
    if (e != SA_OK) return e;
    e = check_select_params(params);
    if (e != SA_OK) return e;
    if (!aligned16(q) || !check_stats(stats, false) || out == nullptr || scale < 0.f) return SA_ERR_INVALID_ARG;
    *p = select_plan(*d, *params);
    if (params->score == SA_SCORE_QUEST && stats->blk_min == nullptr) return SA_ERR_INVALID_ARG;
    if (params->score != SA_SCORE_MEAN_SUM && !select_var_ok(p->g)) return SA_ERR_UNSUPPORTED;
    if (p->g.kk > 0 && !aligned4(out->blk_idx)) return SA_ERR_INVALID_ARG;
    if (params->k_blocks > 0 && out->blk_idx == nullptr) return SA_ERR_INVALID_ARG;
    if (!aligned4(out->samp_count)) return SA_ERR_INVALID_ARG;
    if (params->sample_b > 0 && !aligned4(out->samp_idx)) return SA_ERR_INVALID_ARG;
    if (out->n_rescored != nullptr && !aligned4(out->n_rescored)) return SA_ERR_INVALID_ARG;
    if (params->clt_base > 0 && (!aligned16(k) || !aligned16(v) || !aligned4(out->samp_idx)))
        return SA_ERR_INVALID_ARG;                  // the CLT budget reads K and V
    *a = SelectArgs{q, *stats, k, v, *out, *params, resolve_scale(scale, d->d), nullptr};
    return SA_OK;
}

sa_status prep_decode(const sa_shape* shape, const sa_decode_params* dparams, const sa_select_params* sparams,
                      const void* q, const void* k, const void* v, const sa_stats* stats, const sa_selection* sel,
                      float* out, Dims* d, DecodePlan* p, size_t* need, DecodeArgs* a) {
    sa_status e = check_shape(shape, d);
    if (e != SA_OK) return e;
    e = check_select_params(sparams);
    if (e != SA_OK) return e;
    if (dparams == nullptr) return SA_ERR_INVALID_ARG;
    const sa_mode m = dparams->mode;
    if (m != SA_DROP && m != SA_RESA && m != SA_PROXY && m != SA_SAMPLE) return SA_ERR_INVALID_ARG;
    if (!(dparams->lambda >= 0.f && dparams->lambda <= 1.f) || dparams->scale < 0.f) return SA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || sel == nullptr)
        return SA_ERR_INVALID_ARG;
    // stats: RESA reads mu_q, o_est, log_z0, mu_k; PROXY reads sum_k, sum_v
    sa_stats st{};
    if (m == SA_RESA || m == SA_PROXY) {
        if (stats == nullptr) return SA_ERR_INVALID_ARG;
        st = *stats;
        if (m == SA_RESA && (!aligned16(st.mu_q) || !aligned16(st.o_est) || !aligned4(st.log_z0) ||
                             !aligned16(st.mu_k)))
            return SA_ERR_INVALID_ARG;
        if (m == SA_PROXY && (!aligned16(st.sum_k) || !aligned16(st.sum_v))) return SA_ERR_INVALID_ARG;
    }
    *p = decode_plan(*d, *sparams, (int)m);
    *need = decode_plan(*d, *sparams).bytes;
    if (p->g.kk > 0 && !aligned4(sel->blk_idx)) return SA_ERR_INVALID_ARG;
    if (m == SA_SAMPLE && (sparams->sample_cap < 1 || !aligned4(sel->samp_idx) || !aligned4(sel->samp_count)))
        return SA_ERR_INVALID_ARG;
    *a = DecodeArgs{q, k, v, st, *sel, *sparams, *dparams, resolve_scale(dparams->scale, d->d), out, nullptr, false};
    return SA_OK;
}

}  // namespace

sa_status sa::check_select_call(const sa_shape* shape, const sa_select_params* params, const void* q,
                                const sa_stats* stats, const void* k, const void* v, const sa_selection* out,
                                float scale) {
    Dims d;
    SelectPlan p;
    SelectArgs a;
    return prep_select(shape, params, q, stats, k, v, out, scale, &d, &p, &a);
}

extern "C" {

sa_status sa_select(const sa_shape* shape, const sa_select_params* params, const void* q,
                    const sa_stats* stats, const void* k, const void* v, const sa_selection* out,
                    float scale, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange r("sa_select");
    Dims d;
    SelectPlan p;
    SelectArgs a;
    sa_status e = prep_select(shape, params, q, stats, k, v, out, scale, &d, &p, &a);
    if (e != SA_OK) return e;
    if (ws == nullptr || ws_bytes < p.bytes || !aligned16(ws)) return SA_ERR_WORKSPACE;
    a.ws = static_cast<char*>(ws);
    if (launch_select(d, p, a, static_cast<cudaStream_t>(stream)) != cudaSuccess) return SA_ERR_CUDA;
    if (params->clt_base > 0 && launch_clt(d, p, a, static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return SA_ERR_CUDA;
    return SA_OK;
}

sa_status sa_decode(const sa_shape* shape, const sa_decode_params* dparams, const sa_select_params* sparams,
                    const void* q, const void* k, const void* v, const sa_stats* stats,
                    const sa_selection* sel, float* out, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange r("sa_decode");
    Dims d;
    DecodePlan p;
    size_t need;
    DecodeArgs a;
    sa_status e = prep_decode(shape, dparams, sparams, q, k, v, stats, sel, out, &d, &p, &need, &a);
    if (e != SA_OK) return e;
    if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return SA_ERR_WORKSPACE;
    a.ws = static_cast<char*>(ws);
    return launch_decode(d, p, a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status sa_step(const sa_shape* shape, const sa_decode_params* dparams, const sa_select_params* sparams,
                  const void* q, const void* k, const void* v, const sa_stats* stats, const sa_selection* sel,
                  float* out, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange r("sa_step");
    Dims d;
    SelectPlan ps;
    SelectArgs as;
    const float scale = dparams != nullptr ? dparams->scale : 0.f;
    sa_status e = prep_select(shape, sparams, q, stats, k, v, sel, scale, &d, &ps, &as);
    if (e != SA_OK) return e;
    DecodePlan pd;
    size_t need;
    DecodeArgs ad;
    e = prep_decode(shape, dparams, sparams, q, k, v, stats, sel, out, &d, &pd, &need, &ad);
    if (e != SA_OK) return e;
    if (ws == nullptr || ws_bytes < ps.bytes + need || !aligned16(ws)) return SA_ERR_WORKSPACE;
    as.ws = static_cast<char*>(ws);
    ad.ws = static_cast<char*>(ws) + ps.bytes;
    ad.pdl = true;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (launch_select(d, ps, as, s) != cudaSuccess) return SA_ERR_CUDA;
    if (sparams->clt_base > 0) {
        // the budget kernel sits between: the decode waits for it as usual
        if (launch_clt(d, ps, as, s) != cudaSuccess) return SA_ERR_CUDA;
    }
    return launch_decode(d, pd, ad, s) == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

namespace {
bool check_clusters(const sa_clusters* cl) {
    if (cl == nullptr || cl->n_clusters < 1 || cl->n_clusters > 64) return false;
    const void* p[] = {cl->basis, cl->assign, cl->codes, cl->scales, cl->count,
                       cl->sum_k, cl->sum_v, cl->sum_k2, cl->order, cl->start};
    for (const void* x : p)
        if (x == nullptr || !aligned16(x)) return false;
    return true;
}
}  // namespace

sa_status sa_cluster_prep(const sa_shape* shape, const void* k, const void* v, const sa_clusters* cl, void* stream) {
    NvtxRange r("sa_cluster_prep");
    Dims d;
    sa_status e = check_shape(shape, &d);
    if (e != SA_OK) return e;
    if (!aligned16(k) || !aligned16(v) || !check_clusters(cl)) return SA_ERR_INVALID_ARG;
    if (d.ld >= (1 << 24)) return SA_ERR_UNSUPPORTED;
    return launch_cluster_prep(d, k, v, *cl, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status sa_cluster_build(const sa_shape* shape, const void* q_ctx, const void* k, const void* v,
                           const sa_clusters* cl, int basis_given, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange r("sa_cluster_build");
    Dims d;
    sa_status e = check_shape(shape, &d);
    if (e != SA_OK) return e;
    if ((basis_given != 0 && basis_given != 1) || (!basis_given && !aligned16(q_ctx)) || !aligned16(k) ||
        !aligned16(v) || !check_clusters(cl))
        return SA_ERR_INVALID_ARG;
    if (d.ld >= (1 << 24)) return SA_ERR_UNSUPPORTED;
    const QgcPlan p = qgc_plan(d);
    if (ws == nullptr || ws_bytes < p.bytes || !aligned16(ws)) return SA_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (launch_cluster_build(d, p, q_ctx, k, *cl, basis_given != 0, static_cast<char*>(ws), s) != cudaSuccess)
        return SA_ERR_CUDA;
    return launch_cluster_prep(d, k, v, *cl, s) == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

sa_status sa_multi_step(const sa_shape* shape, const void* q, const void* k, const void* v, const sa_clusters* cl,
                        int budget, float scale, int32_t* read, int32_t* read_count, float* out, void* ws,
                        size_t ws_bytes, void* stream) {
    NvtxRange r("sa_multi_step");
    Dims d;
    sa_status e = check_shape(shape, &d);
    if (e != SA_OK) return e;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !check_clusters(cl) || budget < 1 ||
        !aligned4(read) || !aligned4(read_count) || !aligned16(out) || scale < 0.f)
        return SA_ERR_INVALID_ARG;
    const size_t need = multi_workspace(d);
    if (ws == nullptr || ws_bytes < need || !aligned16(ws)) return SA_ERR_WORKSPACE;
    return launch_multi_step(d, q, k, v, *cl, budget, resolve_scale(scale, d.d), read, read_count, out,
                             static_cast<char*>(ws), static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? SA_OK
               : SA_ERR_CUDA;
}

sa_status sa_dense_decode(const sa_shape* shape, const void* q, const void* k, const void* v, float* out,
                          float scale, void* ws, size_t ws_bytes, void* stream) {
    NvtxRange r("sa_dense_decode");
    Dims d;
    sa_status e = check_shape(shape, &d);
    if (e != SA_OK) return e;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || scale < 0.f)
        return SA_ERR_INVALID_ARG;
    const DensePlan p = dense_plan(d);
    if (ws == nullptr || ws_bytes < p.bytes || !aligned16(ws)) return SA_ERR_WORKSPACE;
    DenseArgs a{q, k, v, resolve_scale(scale, d.d), out, static_cast<char*>(ws)};
    return launch_dense(d, p, a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}

}  // extern "C"
