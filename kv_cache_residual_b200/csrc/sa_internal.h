// Host-side plans shared by the C ABI and the kernel launchers: split counts
// and workspace offsets.  The same functions size the workspace and lay it
// out at launch, so the two can never disagree.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sa_decode.h"

#include <atomic>

namespace sa {

constexpr int kSmTarget = 148 * 4;   // CTAs to aim for: 4 per SM on B200
constexpr int kStreamSlots = 148 * 2; // resident CTAs of the bf16 stream kernel (2 per SM)
constexpr int kSelectSlots = 148 * 2; // resident scanning CTAs of the selection (2 per SM): one wave
constexpr int kMinChunkTiles = 8;     // fewest 64-token tiles per CTA when a decode unit is split

struct Dims {
    int B, Hq, Hkv, G, d, L;
    int ld;            // tokens per unit in the cache allocation (>= L, multiple of 16)
    int bf16;          // 1: bf16 cache and queries, 0: fp32
    int U() const { return B * Hkv; }
    int nb() const { return L / 16; }      // complete blocks of the current length
    int nbl() const { return ld / 16; }    // block rows per unit in the summary arrays
};

// Exactly-read set geometry of a unit (same for all units of a shape).
struct SetGeom {
    int s_eff;       // sink tokens actually read: min(sink, L)
    int w_eff;       // window tokens read, disjoint from the sink
    int c_lo, c_hi;  // candidate blocks [c_lo, c_hi)
    int n_cand;
    int kk;          // blocks chosen per unit
    int n_i;         // |I|
    int n_t;         // L - |I|
};

inline SetGeom set_geom(const Dims& d, int sink, int local, int k_blocks) {
    SetGeom g;
    g.s_eff = sink < d.L ? sink : d.L;
    int w = local < d.L ? local : d.L;
    g.w_eff = w < d.L - g.s_eff ? w : d.L - g.s_eff;
    g.c_lo = (sink + 15) / 16;
    int hi = d.L - local;
    g.c_hi = hi > 0 ? hi / 16 : 0;
    if (g.c_hi < g.c_lo) g.c_hi = g.c_lo;
    g.n_cand = g.c_hi - g.c_lo;
    g.kk = k_blocks < g.n_cand ? k_blocks : g.n_cand;
    g.n_i = g.s_eff + g.w_eff + 16 * g.kk;
    g.n_t = d.L - g.n_i;
    return g;
}

inline int clampi(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }
inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
inline int cdiv(int a, int b) { return (a + b - 1) / b; }

struct PrefillPlan {
    int nsq, rows_q;             // q-mean splits per (b, h), rows per split
    int nskv, tok_kv;            // KV-pass splits per unit, tokens per split (x16)
    size_t off_qpart, off_qcnt, off_kvpart, off_kvcnt, bytes;
    int kv_stride;               // floats per KV-pass partial record
    // bf16 caches: the KV pass on the tensor-core stream kernel, chunks of
    // tpc 64-token tiles (about one wave), rec floats per chunk record (in
    // the off_kvpart area)
    int nsp, tpc, rec_p;
};

inline PrefillPlan prefill_plan(const Dims& d) {
    PrefillPlan p;
    const int BH = d.B * d.Hq;
    p.nsq = clampi(cdiv(kSmTarget, BH), 1, d.L / 256 > 0 ? d.L / 256 : 1);
    p.rows_q = cdiv(d.L, p.nsq);
    p.nsq = cdiv(d.L, p.rows_q);
    p.nskv = clampi(cdiv(kSmTarget, d.U()), 1, d.L / 256 > 0 ? d.L / 256 : 1);
    p.tok_kv = cdiv(d.nb(), p.nskv) * 16;
    p.nskv = cdiv(d.L, p.tok_kv);
    // m[G], l[G], acc[G][d], vsum[d], absmax, pad to even, then ksum[d] as f64
    int f = 2 * d.G + d.G * d.d + d.d + 1;
    f = (f + 1) & ~1;
    p.kv_stride = f + 2 * d.d;
    // completion counters first: their place never depends on split counts
    size_t off = 0;
    p.off_qcnt = off;  off = align256(off + sizeof(unsigned) * (size_t)BH);
    p.off_kvcnt = off; off = align256(off + sizeof(unsigned) * (size_t)d.U());
    p.off_qpart = off; off = align256(off + sizeof(float) * (size_t)BH * p.nsq * d.d);
    // bf16: the stream kernel's chunks (as the dense pass) and records of
    // the exact and prior states, fp64 key sums, absmax
    const int ntiles = cdiv(d.L, 64);
    p.nsp = clampi(kStreamSlots / d.U(), 1, ntiles);
    p.tpc = cdiv(ntiles, p.nsp);
    p.nsp = cdiv(ntiles, p.tpc);
    p.rec_p = (2 * d.G * (2 + d.d) + 2 * d.d + 1 + 3) & ~3;
    const size_t kv_floats = (size_t)d.U() * (size_t)(d.bf16 ? p.nsp * p.rec_p : p.nskv * p.kv_stride);
    p.off_kvpart = off; off = align256(off + sizeof(float) * kv_floats);
    p.bytes = off;
    return p;
}

struct SelectPlan {
    SetGeom g;
    int nss, rows_s;             // scan splits per unit, candidate rows per split
    int nsc, clt_chunk, clt_rec; // CLT budget: splits per unit, I tokens per split, doubles per record
    size_t off_scores, off_scores_up, off_xkey, off_cnt, off_clt, bytes;
};

inline SelectPlan select_plan(const Dims& d, const sa_select_params& sp) {
    SelectPlan p;
    p.g = set_geom(d, sp.sink, sp.local, sp.k_blocks);
    const int nc = p.g.n_cand > 0 ? p.g.n_cand : 1;
    // enough units to fill the GPU: one CTA per unit (scores stay on chip);
    // otherwise split units so the grid is one wave, >= 32 rows per CTA
    p.nss = d.U() >= 148 ? 1 : clampi(kSelectSlots / d.U(), 1, cdiv(nc, 32));
    p.rows_s = cdiv(nc, p.nss);
    p.nss = cdiv(nc, p.rows_s);
    size_t off = 0;
    // completion tickets: the selection's [0, U), the CLT budget's [U, 2U)
    p.off_cnt = off;    off = align256(off + sizeof(unsigned) * 2 * (size_t)d.U());
    p.off_scores = off; off = align256(off + sizeof(float) * (size_t)d.U() * nc);
    p.off_scores_up = off; off = align256(off + sizeof(float) * (size_t)d.U() * nc);
    p.off_xkey = off;   off = align256(off + sizeof(unsigned long long) * (size_t)d.U() * nc);
    // CLT budget (clt_base > 0): the read set split over about one wave of
    // CTAs, >= 128 tokens per split; one record per split (m, S, N per head)
    p.nsc = 0; p.clt_chunk = 0; p.clt_rec = 0; p.off_clt = off;
    if (sp.clt_base > 0) {
        const int ni = p.g.n_i > 0 ? p.g.n_i : 1;
        p.nsc = clampi(kSmTarget / d.U(), 1, cdiv(ni, 128));
        p.clt_chunk = cdiv(ni, p.nsc);
        p.nsc = cdiv(ni, p.clt_chunk);
        p.clt_rec = 2 * d.G + d.G * d.d;
        off = align256(off + sizeof(double) * (size_t)d.U() * p.nsc * p.clt_rec);
    }
    p.bytes = off;
    return p;
}

struct DecodePlan {
    SetGeom g;
    int n_tok_max;               // |I| + sample capacity
    int nsd, tok_d;              // splits per unit, tokens per split (bf16: tiles per chunk)
    int rec;                     // floats per partial record
    size_t off_part, off_cnt, bytes;
};

// mode < 0: the largest plan over all modes (workspace sizing); otherwise the
// launch plan of that mode (only SA_SAMPLE reads the draws).  Counters sit at
// offset 0 and records after them, so a smaller launch plan fits in the
// workspace sized by the largest.
inline DecodePlan decode_plan(const Dims& d, const sa_select_params& sp, int mode = -1) {
    DecodePlan p;
    p.g = set_geom(d, sp.sink, sp.local, sp.k_blocks);
    const bool draws = mode < 0 || mode == SA_SAMPLE;
    // per-head draws: G lists of up to sample_cap each follow I
    p.n_tok_max = p.g.n_i + (draws && sp.sample_cap > 0 ? (sp.per_head ? d.G : 1) * sp.sample_cap : 0);
    const int nt = p.n_tok_max > 0 ? p.n_tok_max : 1;
    if (d.bf16) {                  // stream kernel: chunks of 64-token tiles, ~one wave
        // at least kMinChunkTiles tiles per chunk: a unit split over several
        // CTAs pays a record, a ticket and the last CTA's combine (~10 us on
        // one sequence), more than a CTA spends on that many tiles
        const int ntiles = cdiv(nt, 64);
        p.nsd = clampi(kStreamSlots / d.U(), 1, cdiv(ntiles, kMinChunkTiles));
        p.tok_d = cdiv(ntiles, p.nsd);          // tiles per chunk
        p.nsd = cdiv(ntiles, p.tok_d);
    } else {
        p.nsd = clampi(cdiv(kSmTarget, d.U()), 1, cdiv(nt, 32));
        p.tok_d = cdiv(nt, p.nsd);
        p.nsd = cdiv(nt, p.tok_d);
    }
    // exact (m,l,acc) + prior (m0,l0,acc0) per head, then ksum, vsum
    p.rec = 2 * d.G * (2 + d.d) + 2 * d.d;
    size_t off = 0;
    p.off_cnt = off;  off = align256(off + sizeof(unsigned) * (size_t)d.U());
    p.off_part = off; off = align256(off + sizeof(float) * (size_t)d.U() * p.nsd * p.rec);
    p.bytes = off;
    return p;
}

struct DensePlan {
    int nsdn, tok;
    int rec;
    size_t off_part, off_cnt, bytes;
};

inline DensePlan dense_plan(const Dims& d) {
    DensePlan p;
    if (d.bf16) {                  // stream kernel: chunks of 64-token tiles, ~one wave
        const int ntiles = cdiv(d.L, 64);
        p.nsdn = clampi(kStreamSlots / d.U(), 1, ntiles);
        p.tok = cdiv(ntiles, p.nsdn) * 64;
        p.nsdn = cdiv(d.L, p.tok);
    } else {
        p.nsdn = clampi(cdiv(2 * kSmTarget, d.U()), 1, d.L / 256 > 0 ? d.L / 256 : 1);
        p.tok = cdiv(d.nb(), p.nsdn) * 16;
        p.nsdn = cdiv(d.L, p.tok);
    }
    p.rec = d.G * (2 + d.d);
    size_t off = 0;
    p.off_cnt = off;  off = align256(off + sizeof(unsigned) * (size_t)d.U());
    p.off_part = off; off = align256(off + sizeof(float) * (size_t)d.U() * p.nsdn * p.rec);
    p.bytes = off;
    return p;
}

// ---- launchers (one per .cu file) -----------------------------------------

struct PrefillArgs {
    const void* q_ctx; const void* k; const void* v;
    sa_stats st; float scale; char* ws;
};
cudaError_t launch_prefill(const Dims& d, const PrefillPlan& p, const PrefillArgs& a, cudaStream_t s);
cudaError_t launch_block_summaries(const Dims& d, const void* k, int blk_begin, int blk_end, void* blk_mean,
                                   float* kbar_absmax, const float* centre, int8_t* blk_code, float* blk_meta,
                                   cudaStream_t s);
// elementwise key min / max of blocks [blk_begin, blk_end) (sa_prefill.cu)
cudaError_t launch_block_minmax(const Dims& d, const void* k, int blk_begin, int blk_end, void* blk_min,
                                void* blk_max, cudaStream_t s);
cudaError_t launch_block_sketch(const Dims& d, const void* blk_mean, const float* centre, int blk_begin, int blk_end,
                                int8_t* blk_code, float* blk_meta, cudaStream_t s);
// one token per unit at position d.L (sa_append.cu)
cudaError_t launch_append(const Dims& d, const void* k_new, const void* v_new, void* k, void* v,
                          const sa_stats& st, float scale, cudaStream_t s);

struct SelectArgs {
    const void* q; sa_stats st; const void* k; const void* v;
    sa_selection sel; sa_select_params sp; float scale; char* ws;
};
// Raises a kernel's dynamic shared-memory limit to `bytes` once per device
// (the attribute lives in the device's context; `done` holds one bit per
// device id < 64, larger ids set it on every call).
template <typename K>
inline cudaError_t opt_in_smem(K kernel, size_t bytes, std::atomic<unsigned long long>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? 1ull << dev : 0ull;
    if (bit != 0ull && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

cudaError_t launch_select(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s);
// the alternative block scores (sa_select_var.cu): whether the shape fits
// (candidate keys in shared memory), and the launch
bool select_var_ok(const SetGeom& g);
cudaError_t launch_select_var(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s);
// selection CTAs (on the current device) that gave up a bounded wait
cudaError_t select_wait_timeouts(unsigned* count);
// sa_select's argument checks alone (nothing is enqueued): SA_OK when
// sa_select would accept these arguments with a large enough workspace
sa_status check_select_call(const sa_shape* shape, const sa_select_params* params, const void* q,
                            const sa_stats* stats, const void* k, const void* v, const sa_selection* out,
                            float scale);
// The CLT sampling budget (sa_clt.cu), after the selection when clt_base > 0.
constexpr int kCltMaxBase = 256;     // largest base sample
cudaError_t launch_clt(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s);


struct DecodeArgs {
    const void* q; const void* k; const void* v; sa_stats st; sa_selection sel;
    sa_select_params sp; sa_decode_params dp; float scale; float* out; char* ws;
    bool pdl;          // launched as a programmatic dependent of the selection kernel
};
cudaError_t launch_decode(const Dims& d, const DecodePlan& p, const DecodeArgs& a, cudaStream_t s);

// Query-geometry clustering at prefill (sa_qgc.cu): workspace layout and launch
struct QgcPlan {
    int nsplit, rows_per;       // second-moment splits per unit, query rows per split
    size_t off_cnt, off_part, off_mom, off_y, bytes;
};
QgcPlan qgc_plan(const Dims& d);
cudaError_t launch_cluster_build(const Dims& d, const QgcPlan& p, const void* q_ctx, const void* k,
                                 const sa_clusters& cl, bool basis_given, char* ws, cudaStream_t s);

// The multi-proxy path (sa_multi.cu)
// The prefill KV pass of bf16 caches on the tensor-core stream kernel (prior
// state of mu_Q, totals, block means, largest |block mean|): st.mu_q must be
// set; part / cnt: records and tickets of the prefill plan.
cudaError_t launch_prefill_stream(const Dims& d, const PrefillPlan& p, const void* k, const void* v,
                                  const sa_stats& st, float scale, char* part, char* cnt, cudaStream_t s);
cudaError_t launch_cluster_prep(const Dims& d, const void* k, const void* v, const sa_clusters& cl, cudaStream_t s);
size_t multi_workspace(const Dims& d);
cudaError_t launch_multi_step(const Dims& d, const void* q, const void* k, const void* v, const sa_clusters& cl,
                              int budget, float scale, int32_t* read, int32_t* qcnt, float* out, char* ws,
                              cudaStream_t s);

struct DenseArgs {
    const void* q; const void* k; const void* v; float scale; float* out; char* ws;
};
cudaError_t launch_dense(const Dims& d, const DensePlan& p, const DenseArgs& a, cudaStream_t s);

}  // namespace sa
