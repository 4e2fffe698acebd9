// Per-step selection: one CTA of 256 threads per unit when the unit's
// candidate keys fit its shared memory and there are enough units to fill
// the GPU (k_select runs the whole selection); otherwise the units are split
// over several scanning CTAs (k_select in its scan phase, bounds into the
// workspace) and a second kernel, k_select_finish, one 512-thread CTA per
// unit with up to 16K keys in shared memory, gathers the bounds and runs the
// top-k, the exact band and the draws (select_unit in its finish phase).  The
// finish kernel is a programmatic dependent of the scan.
#include "sa_select_core.cuh"

namespace sa {

// selection CTAs that abandoned a bounded wait, since the library was loaded
// (the only definition: every selection kernel counts into it through
// SelectIo::timeouts)
__device__ unsigned g_wait_timeouts;

namespace {
std::atomic<unsigned*> g_timeouts_ptr[64];
}

// device address of this device's counter, looked up once per device
static unsigned* wait_counter() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
    if (dev < 64) {
        unsigned* p = g_timeouts_ptr[dev].load(std::memory_order_acquire);
        if (p != nullptr) return p;
    }
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_wait_timeouts) != cudaSuccess) return nullptr;
    if (dev < 64) g_timeouts_ptr[dev].store(static_cast<unsigned*>(p), std::memory_order_release);
    return static_cast<unsigned*>(p);
}

constexpr int kSelStages = 4;      // 4 x 18 KB ring at d = 128 (split units' scan, the finish)
// One CTA per unit: a 3-stage ring, the candidates' keys sized to the unit
// (dynamic) and at most 80 registers, so that two selection CTAs leave room
// on an SM for a decode CTA (a programmatic dependent), which streams its
// selection-independent rows meanwhile
constexpr int kSelStagesAll = 3;

template <int PHASE>
__host__ __device__ constexpr int sel_stages() { return PHASE == kPhAll ? kSelStagesAll : kSelStages; }

template <int D, int PHASE>
__host__ __device__ constexpr size_t sel_ring_smem() {      // the ring and its barriers, 16-byte aligned
    return (SketchRing<D, kWarps, sel_stages<PHASE>()>::kSmem + 15) & ~(size_t)15;
}
constexpr int kFinThreads = 512;
constexpr int kFinishKeys = 16384; // keys of one unit in the finish kernel's shared memory
constexpr int kFinCand = 1024;     // top-k candidates ranked in shared memory
constexpr int kFinAlias = 32768;   // bytes for the top-k / band arrays (select_unit's ring aliases)

template <typename T, int D, int G, int PHASE>
__global__ void __launch_bounds__(kThreads, PHASE == kPhAll ? 3 : 2)
k_select(SelectIo io) {
    using Ring = SketchRing<D, kWarps, sel_stages<PHASE>()>;
    __shared__ __align__(16) unsigned hist[256];
    __shared__ int sw[kWarps + 1];
    __shared__ int misc[3];
    __shared__ float s_qh[G * D];
    __shared__ __align__(16) int8_t s_qi[2 * D];
    __shared__ float s_qc[3];
    __shared__ int s_sorted[kWarpTopK];
    extern __shared__ __align__(128) unsigned char s_ring[];
    // one CTA per unit: the upper and lower keys of its candidates after the
    // ring (a split unit's scan keeps its bounds in the workspace)
    const int kcap = PHASE == kPhAll ? (io.sg.n_cand + 3) & ~3 : 0;
    uint32_t* s_ukeys = reinterpret_cast<uint32_t*>(s_ring + sel_ring_smem<D, PHASE>());
    uint32_t* s_lkeys = s_ukeys + kcap;
    // a decode kernel launched as a programmatic dependent may start as soon as
    // every CTA of this grid has begun; it waits for this grid's completion
    // before reading the selection
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    const SelectSmem sm{hist, sw, misc, s_qh, s_qi, s_qc, s_ukeys, s_lkeys, s_sorted, s_ring,
                        reinterpret_cast<uint64_t*>(s_ring + Ring::kRingBytes), nullptr, 0};
    (void)select_unit<T, D, G, kThreads, sel_stages<PHASE>(), PHASE>(io, sm, blockIdx.y, blockIdx.x);
}

// The finish of split units; dynamic shared memory: the alias area
// (kFinAlias bytes), then upper- and lower-bound keys (n_cand each, when
// n_cand <= kFinishKeys).
template <typename T, int D, int G>
__global__ void __launch_bounds__(kFinThreads, 1)
k_select_finish(SelectIo io) {
    constexpr int NW = kFinThreads / 32;
    __shared__ __align__(16) unsigned hist[256];
    __shared__ int sw[NW + 1];
    __shared__ int misc[3];
    __shared__ float s_qh[G * D];
    __shared__ __align__(16) int8_t s_qi[2 * D];
    __shared__ float s_qc[3];
    __shared__ int s_sorted[kWarpTopK];
    __shared__ uint64_t s_bar[kSelStages];
    extern __shared__ __align__(128) unsigned char s_fin[];
    asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
    // (select_unit waits for the scan kernel once the query is coded)
    const int nk = io.sg.n_cand <= kFinishKeys ? io.sg.n_cand : 0;
    uint32_t* ukeys = reinterpret_cast<uint32_t*>(s_fin + kFinAlias);
    const SelectSmem sm{hist, sw, misc, s_qh, s_qi, s_qc, ukeys, ukeys + nk, s_sorted, s_fin, s_bar, nullptr, 0};
    (void)select_unit<T, D, G, kFinThreads, kSelStages, kPhFinish, kFinishKeys, kFinCand, true>(io, sm,
                                                                                                blockIdx.x, 0);
}

SelectIo select_io(const Dims& d, const SelectPlan& p, const SelectArgs& a) {
    char* ws = a.ws;
    SelectIo io;
    io.q = a.q;
    io.blk_mean = a.st.blk_mean;
    io.blk_code = a.st.blk_code;
    io.blk_meta = reinterpret_cast<const float4*>(a.st.blk_meta);
    io.Hq = d.Hq; io.Hkv = d.Hkv; io.L = d.L; io.ld = d.ld;
    io.sg = p.g;
    io.rows = p.rows_s; io.nss = p.nss;
    io.sc_lo_all = reinterpret_cast<float*>(ws + p.off_scores);
    io.sc_up_all = reinterpret_cast<float*>(ws + p.off_scores_up);
    io.xkey = reinterpret_cast<unsigned long long*>(ws + p.off_xkey);
    io.cnt = reinterpret_cast<unsigned*>(ws + p.off_cnt);
    io.kb_stride = a.sp.k_blocks;
    io.blk_idx = a.sel.blk_idx;
    io.samp_idx = a.sel.samp_idx;
    io.samp_count = a.sel.samp_count;
    io.n_rescored = a.sel.n_rescored;
    // with the CLT budget the selection draws the base sample only
    io.sample_b = a.sp.clt_base > 0 ? a.sp.clt_base : a.sp.sample_b;
    io.sample_cap = a.sp.sample_cap;
    io.seed = (unsigned long long)a.sp.seed;
    io.step = a.sp.step;
    io.timeouts = wait_counter();
    io.per_head = a.sp.per_head;
    return io;
}

template <typename T, int D, int G>
static cudaError_t select_t(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s) {
    constexpr size_t smem = sel_ring_smem<D, kPhScan>();
    const SelectIo io = select_io(d, p, a);
    if (io.timeouts == nullptr) return cudaErrorInvalidDevice;
    if (p.nss == 1 && p.g.n_cand <= kSmemKeys) {
        static std::atomic<unsigned long long> opted{0};
        constexpr size_t all_max = sel_ring_smem<D, kPhAll>() + (size_t)2 * kSmemKeys * 4;
        cudaError_t e = opt_in_smem(k_select<T, D, G, kPhAll>, all_max, opted);
        if (e != cudaSuccess) return e;
        const size_t all = sel_ring_smem<D, kPhAll>() + (size_t)2 * ((p.g.n_cand + 3) & ~3) * 4;
        k_select<T, D, G, kPhAll><<<dim3(p.nss, d.U()), kThreads, all, s>>>(io);
        return cudaGetLastError();
    }
    static std::atomic<unsigned long long> opted_scan{0}, opted_fin{0};
    cudaError_t e = opt_in_smem(k_select<T, D, G, kPhScan>, smem, opted_scan);
    if (e != cudaSuccess) return e;
    k_select<T, D, G, kPhScan><<<dim3(p.nss, d.U()), kThreads, smem, s>>>(io);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    constexpr size_t fin_max = (size_t)kFinAlias + (size_t)kFinishKeys * 8;
    e = opt_in_smem(k_select_finish<T, D, G>, fin_max, opted_fin);
    if (e != cudaSuccess) return e;
    const int nk = p.g.n_cand <= kFinishKeys ? p.g.n_cand : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(d.U());
    cfg.blockDim = dim3(kFinThreads);
    cfg.dynamicSmemBytes = (size_t)kFinAlias + (size_t)nk * 8;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_select_finish<T, D, G>, io);
}

template <typename T, int D>
static cudaError_t select_g(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s) {
    switch (d.G) {
        case 1: return select_t<T, D, 1>(d, p, a, s);
        case 2: return select_t<T, D, 2>(d, p, a, s);
        case 4: return select_t<T, D, 4>(d, p, a, s);
        case 8: return select_t<T, D, 8>(d, p, a, s);
    }
    return cudaErrorInvalidValue;
}

cudaError_t select_wait_timeouts(unsigned* count) {
    return cudaMemcpyFromSymbol(count, g_wait_timeouts, sizeof(unsigned));
}

cudaError_t launch_select(const Dims& d, const SelectPlan& p, const SelectArgs& a, cudaStream_t s) {
    if (a.sp.score != SA_SCORE_MEAN_SUM) return launch_select_var(d, p, a, s);
    if (d.bf16) return d.d == 128 ? select_g<__nv_bfloat16, 128>(d, p, a, s) : select_g<__nv_bfloat16, 64>(d, p, a, s);
    return d.d == 128 ? select_g<float, 128>(d, p, a, s) : select_g<float, 64>(d, p, a, s);
}

}  // namespace sa
