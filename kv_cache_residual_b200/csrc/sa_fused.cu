// One whole decode step per unit in one kernel: the selection (sketch scan,
// certified top-k, tail draws) and then the sparse decode with the residual
// estimator, by the same CTA, with the chosen blocks and draws handed over in
// shared memory (vAttention, Method, overall framework: I_f = sink + local
// window + top-k, then attention over I_f and the sampled tail; RESA, Method:
// the prior merge over I).
//
// k_step_fused: grid (B*Hkv), 128 threads, two CTAs per SM.  Used, when the
// environment variable SA_FUSED_STEP is 1, where every unit gets a CTA of its
// own (enough units to fill the GPU), the cache is bf16, k <= 32 blocks and
// the draws fit a shared list; otherwise sa_step runs the selection and
// decode kernels as a programmatic pair.  The results are
// the ones of the two kernels: the same device code (select_unit,
// stream_unit) runs on the same data in the same order.
//
// Shared memory: one dynamic area used first by the selection (sketch ring +
// barriers + score-bound keys) and then by the stream pass (tile stages, then
// the merge and epilogue scratch), plus small static arrays that carry the
// selection across (chosen blocks, draws).  The sink and window rows, which do
// not depend on the selection, are prefetched into L2 with bulk prefetches at
// the start, so the stream pass finds them there.
#include <cstdlib>

#include "sa_decode_core.cuh"
#include "sa_select_core.cuh"

namespace sa {

constexpr int kFusedStages = 4;     // sketch ring stages (18 KB each at d = 128)

template <int D>
using FusedRing = SketchRing<D, kTcWarps, kFusedStages>;

template <int D>
constexpr size_t fused_select_smem() {   // ring, its barriers (padded to 128 B), upper- and lower-bound keys
    return (size_t)FusedRing<D>::kRingBytes + 128 + (size_t)kSmemKeys * 8;
}

template <int D, int G, int MODE>
constexpr size_t fused_smem() {
    constexpr size_t a = fused_select_smem<D>(), b = stream_area_smem<D, G, MODE>();
    return a > b ? a : b;
}

template <int D, int G, int MODE>
__global__ void __launch_bounds__(kTcThreads, 2)
k_step_fused(SelectIo sio, StreamIo dio) {
    using Ring = FusedRing<D>;
    __shared__ __align__(16) unsigned hist[256];
    __shared__ int sw[kTcWarps + 1];
    __shared__ int misc[3];
    __shared__ float s_qh[G * D];
    __shared__ __align__(16) int8_t s_qi[2 * D];
    __shared__ float s_qc[3];
    __shared__ int s_sorted[kWarpTopK];
    __shared__ int s_samp[kSampCache];
    extern __shared__ __align__(128) unsigned char fsmem[];
    unsigned char* smem = fsmem;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + Ring::kRingBytes);
    uint32_t* ukeys = reinterpret_cast<uint32_t*>(smem + Ring::kRingBytes + 128);
    uint32_t* lkeys = ukeys + kSmemKeys;
    const int u = blockIdx.x;

    // the rows every step reads whatever the selection: sink and window
    if (threadIdx.x == 0) {
        const SetGeom& g = dio.sg;
        const size_t ubase = (size_t)u * dio.ld * D;
        const uint32_t rb = D * 2;                      // bf16 row bytes
        if (g.s_eff > 0) {
            bulk_prefetch_l2(dio.k + ubase, (uint32_t)g.s_eff * rb);
            bulk_prefetch_l2(dio.v + ubase, (uint32_t)g.s_eff * rb);
        }
        if (g.w_eff > 0) {
            const size_t w0 = ubase + (size_t)(dio.L - g.w_eff) * D;
            bulk_prefetch_l2(dio.k + w0, (uint32_t)g.w_eff * rb);
            bulk_prefetch_l2(dio.v + w0, (uint32_t)g.w_eff * rb);
        }
        // and the decode's per-unit statistics
        const int b = u / dio.Hkv, gg = u - b * dio.Hkv;
        const size_t qh0 = (size_t)b * dio.Hq + (size_t)gg * G;
        if constexpr (MODE == SA_RESA) {
            bulk_prefetch_l2(dio.st.mu_q + qh0 * D, G * D * 4);
            bulk_prefetch_l2(dio.st.o_est + qh0 * D, G * D * 4);
            bulk_prefetch_l2(dio.st.mu_k + (size_t)u * D, D * 4);
            prefetch_l2(dio.st.log_z0 + qh0);
        }
        if constexpr (MODE == SA_PROXY) {
            bulk_prefetch_l2(dio.st.sum_k + (size_t)u * D, D * 4);
            bulk_prefetch_l2(dio.st.sum_v + (size_t)u * D, D * 4);
        }
    }

    const SelectSmem sm{hist, sw, misc, s_qh, s_qi, s_qc, ukeys, lkeys, s_sorted, smem, bar, s_samp, kSampCache};
    const SelectOutcome r = select_unit<__nv_bfloat16, D, G, kTcThreads, kFusedStages>(sio, sm, u, 0);
    if (!r.done) return;                 // an abandoned wait: the unit's selection is marked invalid
    if (threadIdx.x == 0)
        for (int j = 0; j < kFusedStages; ++j) mbar_inval(smem_addr(bar + j));
    if (!r.sorted_smem) {
        // the chosen blocks went to global memory only (very wide band): this
        // CTA wrote them before select_unit's closing barrier
        const int32_t* gblk = sio.blk_idx + (size_t)u * sio.kb_stride;
        for (int i = threadIdx.x; i < sio.sg.kk; i += kTcThreads) s_sorted[i] = __ldcg(gblk + i);
    }
    __syncthreads();
    stream_unit<D, G, MODE>(dio, smem, s_sorted, s_samp, u, 0, r.bdraw);
}

// Whether the fused kernel applies (see the file comment); the decode plan
// must be a single chunk per unit so that the result is the two kernels' one.
bool fused_step_ok(const Dims& d, const SelectPlan& sp, const DecodePlan& dp, const sa_select_params& prm,
                   int mode) {
    // opt-in: on the 32-sequence 32K workload the programmatic pair of kernels
    // is faster (the fused CTA has 4 warps for the latency-bound decode)
    const char* env = getenv("SA_FUSED_STEP");
    if (env == nullptr || env[0] != '1') return false;
    if (!d.bf16 || sp.nss != 1 || sp.g.n_cand > kSmemKeys || sp.g.kk > kWarpTopK || dp.nsd != 1) return false;
    if (mode == SA_SAMPLE && prm.sample_cap > kSampCache) return false;
    if (prm.clt_base > 0) return false;             // the budget kernel runs between
    return true;
}

template <int D, int G, int MODE>
static cudaError_t fused_launch(const Dims& d, const SelectIo& sio, const StreamIo& dio, cudaStream_t s) {
    constexpr size_t smem = fused_smem<D, G, MODE>();
    static std::atomic<unsigned long long> opted{0};
    cudaError_t e = opt_in_smem(k_step_fused<D, G, MODE>, smem, opted);
    if (e != cudaSuccess) return e;
    k_step_fused<D, G, MODE><<<d.U(), kTcThreads, smem, s>>>(sio, dio);
    return cudaGetLastError();
}

template <int D, int G>
static cudaError_t fused_m(const Dims& d, int mode, const SelectIo& sio, const StreamIo& dio, cudaStream_t s) {
    switch (mode) {
        case SA_DROP: return fused_launch<D, G, SA_DROP>(d, sio, dio, s);
        case SA_RESA: return fused_launch<D, G, SA_RESA>(d, sio, dio, s);
        case SA_PROXY: return fused_launch<D, G, SA_PROXY>(d, sio, dio, s);
        case SA_SAMPLE: return fused_launch<D, G, SA_SAMPLE>(d, sio, dio, s);
    }
    return cudaErrorInvalidValue;
}

template <int D>
static cudaError_t fused_g(const Dims& d, int mode, const SelectIo& sio, const StreamIo& dio, cudaStream_t s) {
    switch (d.G) {
        case 1: return fused_m<D, 1>(d, mode, sio, dio, s);
        case 2: return fused_m<D, 2>(d, mode, sio, dio, s);
        case 4: return fused_m<D, 4>(d, mode, sio, dio, s);
        case 8: return fused_m<D, 8>(d, mode, sio, dio, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t launch_step_fused(const Dims& d, const SelectPlan& sp, const SelectArgs& sa_, const DecodePlan& dp,
                              const DecodeArgs& da, cudaStream_t s) {
    const SelectIo sio = select_io(d, sp, sa_);
    StreamIo dio;
    dio.q = reinterpret_cast<const __nv_bfloat16*>(da.q);
    dio.k = reinterpret_cast<const __nv_bfloat16*>(da.k);
    dio.v = reinterpret_cast<const __nv_bfloat16*>(da.v);
    dio.st = da.st;
    dio.blk_idx = da.sel.blk_idx;
    dio.kb_stride = da.sp.k_blocks;
    dio.samp_idx = da.sel.samp_idx;
    dio.samp_count = da.sel.samp_count;
    dio.sample_cap = da.sp.sample_cap;
    dio.Hq = d.Hq; dio.Hkv = d.Hkv; dio.L = d.L; dio.ld = d.ld;
    dio.sg = dp.g;
    dio.tpc = dp.tok_d; dio.nchunk = dp.nsd; dio.rec = dp.rec;
    dio.qscale = da.scale * kLog2e; dio.scale = da.scale; dio.lambda = da.dp.lambda;
    dio.part = reinterpret_cast<float*>(da.ws + dp.off_part);
    dio.cnt = reinterpret_cast<unsigned*>(da.ws + dp.off_cnt);
    dio.out = da.out;
    return d.d == 128 ? fused_g<128>(d, da.dp.mode, sio, dio, s) : fused_g<64>(d, da.dp.mode, sio, dio, s);
}

}  // namespace sa
