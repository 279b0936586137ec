// C ABI of the tensor-parallel MLP block: argument checks, planning and
// kernel launches. See include/tpmlp.h for the contract of each entry point.
//
// The forward runs two GEMMs (page "Megatron", section "张量并行 / 数学原理"):
//   F1  column-parallel  H, Y = X·A + a, GeLU(·)   output tiles never straddle
//                        the shard boundary's meaning: every column of H is
//                        independent, so shards are just column ranges
//   F2  row-parallel     Z = Σ_i Y_i·B_i + b       the K loop runs over the
//                        shards in ascending order (in tensor memory); where
//                        a tile's K range is split over several work units
//                        (a stream-K tail, or one unit per shard group),
//                        their fp32 partials are added in ascending order
//                        inside the same kernel, before the bias
// and the backward four GEMMs plus two column sums (chain rule):
//   B2  dH = (dZ·Bᵀ) ⊙ GeLU′(H)   B3  dB = Yᵀ·dZ   B4  dA = Xᵀ·dH
//   B5  dX = Σ_i dH_i·A_iᵀ (ordered shard sum, as F2)   db, da column sums
// (for long K the B2 epilogue itself writes da's per-32-row partials, and
// only their ordered sum remains).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/tpmlp.h"
#include "aux_kernels.cuh"
#include "gemm_tc.cuh"
#include "gemm_tc2.cuh"
#include "simt.cuh"

namespace tpmlp {
namespace {

constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;
constexpr int64_t kColsumRowsPerChunk = 128;
constexpr int kMaxDevices = 64;

std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitLimitNs};
std::atomic<int> g_split_policy{0};
std::atomic<bool> g_overlap{true};  // programmatic dependent launches
std::atomic<bool> g_dynamic{true};  // dynamic tile schedule for the longest products

struct DeviceInfo {
    bool init = false;
    int cc_major = 0;
    int num_sms = 0;
    bool attr_set[128] = {};       // per one-CTA tensor-core kernel instantiation
    bool attr_set_pair[128] = {};  // per CTA-pair kernel instantiation
    int max_pairs[128] = {};       // co-resident CTA pairs per pair-kernel instantiation
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

const DeviceInfo* device_info() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceInfo& d = g_dev[dev];
    if (!d.init) {
        if (cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
            return nullptr;
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return nullptr;
        d.init = true;
    }
    return &d;
}

// --------------------------------------------------------------- tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Row-major bf16 matrix with `rows` rows of `cols` elements, read in boxes
// of box_rows × 64 columns with the 128-byte swizzle (64 bf16 = 128 bytes).
// Out-of-range box elements read as zero.
bool make_map(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output of the epilogue's bulk stores: a row-major M × N matrix of bf16 or
// fp32, written in 32 × 32 boxes; bf16 boxes are 64-byte rows with the
// 64-byte swizzle, fp32 boxes 128-byte rows with the 128-byte swizzle (the
// layouts the epilogue stages in shared memory). Box elements outside
// M × N are not written. (The map is 3-D with one plane.)
bool make_out_map(CUtensorMap* m, void* ptr, int64_t rows, int64_t cols, bool f32) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t esize = f32 ? 4 : 2;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), 1};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols) * esize,
                             static_cast<cuuint64_t>(rows) * static_cast<cuuint64_t>(cols) * esize};
    cuuint32_t box[3] = {32u, 32u, 1u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, ptr, dims,
              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI>
bool make_out_maps(CUtensorMap* o0, CUtensorMap* o1, const GemmArgs& g, int M, int N) {
    const bool f32 = (EPI == EPI_F32);
    if (!make_out_map(o0, g.out0, M, N, f32)) return false;
    if (EpiTraits<EPI>::kAct) return make_out_map(o1, g.out1, M, N, false);
    *o1 = *o0;
    return true;
}

tpmlp_status check_launch() {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError() == cudaSuccess ? TPMLP_OK : TPMLP_ERR_CUDA;
}

// Launch a kernel that orders itself after its predecessor with
// grid_dep_wait() before it reads any global memory. With launch overlap on
// it goes out as a programmatic dependent launch: its CTAs take the SMs the
// predecessor's finished CTAs leave and run their prologue (barriers, tensor
// memory, descriptor prefetch) while the predecessor's last CTAs still run;
// launch latency and prologue leave the critical path. Counts the launch;
// maps errors.
template <typename... KArgs, typename... Args>
tpmlp_status launch_dep(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                        Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = g_overlap.load(std::memory_order_relaxed) ? 1 : 0;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return TPMLP_ERR_CUDA;
    }
    return cudaGetLastError() == cudaSuccess ? TPMLP_OK : TPMLP_ERR_CUDA;
}

// ------------------------------------------------------- per-kernel timing

enum Kind : int {
    K_F1 = 0, K_F2, K_B1_DB, K_B2, K_B2_DA, K_B3, K_B4, K_B34, K_B5, K_MISC,
    K_L_FWD, K_L_DB, K_L_DW, K_L_DX, K_RECOMP, K_CTR, K_B12, K_COUNT
};
const char* const kKindNames[K_COUNT] = {
    "F1.col_gemm_bias_gelu", "F2.row_gemm_shard_sum", "B1.db_colsum",
    "B2.dgrad_gelu_grad",    "B2.da_colsum",          "B3.wgrad_dB",     "B4.wgrad_dA",
    "B3+B4.wgrad_dB_dA",     "B5.dgrad_dX_shard_sum", "misc",
    "L.fwd_gemm_bias",       "L.dbias_colsum",        "L.wgrad_dW",      "L.dgrad_dX",
    "R.recompute_activation", "S.counter_reset",  "B1+B2.db_da_colsum",
};

struct KindTotals {
    uint64_t launches = 0;
    double ms = 0, flops = 0, bytes = 0;
};
struct PendingRec {
    cudaEvent_t a, b;
    int kind;
    double flops, bytes;
};
// Timing state, shared by every host thread that calls the library: the
// flag is atomic, the records and the event pool are guarded by g_prof_mutex.
std::atomic<bool> g_prof_on{false};
std::mutex g_prof_mutex;
KindTotals g_prof[K_COUNT];
std::vector<PendingRec> g_pending;
std::vector<cudaEvent_t> g_event_pool;

// Caller holds g_prof_mutex.
cudaEvent_t pool_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

// Run `fn` (which enqueues one step's kernels on `st`); when timing is on,
// bracket it with two events and remember the step's algorithmic work.
template <class Fn>
tpmlp_status timed(int kind, double flops, double bytes, cudaStream_t st, Fn&& fn) {
    if (!g_prof_on.load(std::memory_order_relaxed)) return fn();
    cudaEvent_t a, b;
    {
        std::lock_guard<std::mutex> lock(g_prof_mutex);
        a = pool_event();
        b = pool_event();
        if (a == nullptr || b == nullptr) {
            if (a) g_event_pool.push_back(a);
            if (b) g_event_pool.push_back(b);
            return TPMLP_ERR_CUDA;
        }
    }
    cudaEventRecord(a, st);
    tpmlp_status s = fn();
    cudaEventRecord(b, st);
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    g_pending.push_back({a, b, kind, flops, bytes});
    return s;
}

// ------------------------------------------------------ tensor-core launches

// Index of a tensor-core kernel instantiation (0..95) for per-device caches.
template <int BN, bool A_MN, bool B_MN, int EPI, bool RELAY, bool LONG = false>
constexpr int kernel_id() {
    static_assert(BN == 256, "the launchers use 256-column tiles");
    return ((EPI * 4 + (A_MN ? 2 : 0) + (B_MN ? 1 : 0)) * 2 + (RELAY ? 1 : 0)) * 2 + (LONG ? 1 : 0);
}

// How a GEMM launch cuts its work into units (see next_unit).
struct SchedReq {
    int kind = SCHED_TILES;  // SCHED_TILES, SCHED_GROUPS or SCHED_STREAMK
    int groups = 1;          // SCHED_GROUPS: consecutive k ranges per tile
    bool force = false;      // SCHED_STREAMK even where the time model says it does not pay
    bool dyn = false;        // items handed out dynamically (CTA pairs; needs the counters)
};

// Shortest stream-K segment allowed, and the tail's extra cost (partial
// stores, the last unit's reads and sums, the counter reset), both in
// k-block times of one worker. Measured on CTA pairs: forcing the tail cost
// 27–36 µs per product where it saves nothing (7B-class shapes, ~0.43 µs per
// k-block at power-capped clocks), i.e. ~80 k-blocks.
constexpr int64_t kSkMinSegmentKb = 4;
constexpr double kSkOverheadKb = 80.0;

// Whether the stream-K tail is valid for `tiles` output tiles of `kb`
// k-blocks on P workers and (unless forced) faster than whole tiles. In
// k-block times of one worker: whole tiles take ceil(tiles/P)·kb; the tail
// takes floor(tiles/P)·kb + ceil(W/P) + overhead, W = (tiles mod P)·kb.
bool streamk_pays(int64_t tiles, int64_t kb, int64_t P, bool force) {
    if (P < 1) return false;
    const int64_t rem = tiles % P;
    if (rem == 0) return false;
    const int64_t W = rem * kb;
    if (W < P * kSkMinSegmentKb) return false;
    if (force) return true;
    const double whole = static_cast<double>((tiles + P - 1) / P) * static_cast<double>(kb);
    const double tail = static_cast<double>(tiles / P) * static_cast<double>(kb) +
                        static_cast<double>((W + P - 1) / P) + kSkOverheadKb;
    return tail < 0.985 * whole;
}

// Fill g's schedule for at most P workers; returns the number of workers
// to launch. A split schedule needs the partial-tile workspace, a kernel
// instantiation that can finish split tiles, and no column-sum output.
int resolve_sched(GemmArgs& g, const SchedReq& req, int64_t P, bool splittable) {
    const int64_t tiles = static_cast<int64_t>(g.num_m_blocks) * g.num_n_blocks;
    g.sched = SCHED_TILES;
    g.groups = 1;
    g.kb_per_group = g.k_blocks;
    if (g.second) {  // a grouped launch: whole tiles of both products
        const int64_t all = tiles + static_cast<int64_t>(g.num_m_blocks2) * g.num_n_blocks2;
        return static_cast<int>(std::min(all, P));
    }
    const bool have_ws = g.partials != nullptr && g.counters != nullptr && splittable &&
                         g.colsum_out == nullptr;
    if (req.kind == SCHED_GROUPS && have_ws && req.groups > 1 && g.k_blocks % req.groups == 0) {
        g.sched = SCHED_GROUPS;
        g.groups = req.groups;
        g.kb_per_group = g.k_blocks / req.groups;
        return static_cast<int>(std::min(tiles * req.groups, P));
    }
    if (req.kind == SCHED_STREAMK && have_ws && streamk_pays(tiles, g.k_blocks, P, req.force)) {
        g.sched = SCHED_STREAMK;
        return static_cast<int>(P);
    }
    return static_cast<int>(std::min(tiles, P));
}

// D[M, N] = Aop·Bop with Aop stored [M][K] (A_MN = false) or [K][M], Bop
// stored [N][K] (B_MN = false) or [K][N].
template <int BN, bool A_MN, bool B_MN, int EPI, bool RELAY>
tpmlp_status gemm_tc_launch(const void* Aop, const void* Bop, int M, int N, int K,
                            const SchedReq& req, GemmArgs g, cudaStream_t st) {
    using Cfg = TileCfg<BN>;
    const DeviceInfo* dev = device_info();
    if (dev == nullptr) return TPMLP_ERR_CUDA;
    CUtensorMap tmA, tmB;
    const bool okA = A_MN ? make_map(&tmA, Aop, K, M, 64) : make_map(&tmA, Aop, M, K, kBM);
    const bool okB = B_MN ? make_map(&tmB, Bop, K, N, 64) : make_map(&tmB, Bop, N, K, BN);
    CUtensorMap tmO0, tmO1;
    if (!okA || !okB || !make_out_maps<EPI>(&tmO0, &tmO1, g, M, N)) return TPMLP_ERR_CUDA;
    g.M = M;
    g.N = N;
    g.K = K;
    g.num_m_blocks = (M + kBM - 1) / kBM;
    g.num_n_blocks = (N + BN - 1) / BN;
    g.k_blocks = (K + kBK - 1) / kBK;
    g.wait_limit_ns = g_wait_limit_ns.load();
    auto kern = gemm_tc_kernel<BN, A_MN, B_MN, EPI, RELAY>;
    constexpr int id = kernel_id<BN, A_MN, B_MN, EPI, RELAY>();
    {
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        int devn = 0;
        if (cudaGetDevice(&devn) != cudaSuccess || devn < 0 || devn >= kMaxDevices)
            return TPMLP_ERR_CUDA;
        if (!g_dev[devn].attr_set[id]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Cfg::SMEM_BYTES) != cudaSuccess)
                return TPMLP_ERR_CUDA;
            g_dev[devn].attr_set[id] = true;
        }
    }
    const int grid = resolve_sched(g, req, dev->num_sms, kSplittable<EPI, RELAY>);
    g.dyn_counter = nullptr;  // the one-CTA kernel runs the static schedule
    return launch_dep(kern, dim3(grid), dim3(kThreads), Cfg::SMEM_BYTES, st, tmA, tmB, tmO0, tmO1, g);
}

// A second product launched with the first (grouped launch, whole tiles):
// Aop2 · Bop2 into the M2 × N2 fp32 matrix out2, same K and layouts.
struct SecondProduct {
    const void* A;
    const void* B;
    int M, N;
    void* out;
};

// Same product on CTA pairs: 256 × BN tiles, grid = 2 × (co-resident pairs).
// LONG: the long-product variant (double epilogue staging; the only one that
// runs the dynamic schedule: other variants run req's schedule statically).
template <int BN, bool A_MN, bool B_MN, int EPI, bool RELAY, bool LONG = false>
tpmlp_status gemm_tc2_launch(const void* Aop, const void* Bop, int M, int N, int K,
                             const SchedReq& req, GemmArgs g, cudaStream_t st,
                             const SecondProduct* second = nullptr) {
    using Cfg = Tile2Cfg<BN, LONG>;
    const DeviceInfo* dev = device_info();
    if (dev == nullptr) return TPMLP_ERR_CUDA;
    CUtensorMap tmA, tmB;
    const bool okA = A_MN ? make_map(&tmA, Aop, K, M, 64) : make_map(&tmA, Aop, M, K, kBM);
    const bool okB = B_MN ? make_map(&tmB, Bop, K, N, 64) : make_map(&tmB, Bop, N, K, BN / 2);
    CUtensorMap tmO0, tmO1;
    if (!okA || !okB || !make_out_maps<EPI>(&tmO0, &tmO1, g, M, N)) return TPMLP_ERR_CUDA;
    CUtensorMap tmA2 = tmA, tmB2 = tmB;
    if (second != nullptr) {
        // the second product's output takes the second output map
        if constexpr (EpiTraits<EPI>::kAct) return TPMLP_ERR_INVALID;
        const SecondProduct& q = *second;
        const bool ok2 = (A_MN ? make_map(&tmA2, q.A, K, q.M, 64) : make_map(&tmA2, q.A, q.M, K, kBM)) &&
                         (B_MN ? make_map(&tmB2, q.B, K, q.N, 64) : make_map(&tmB2, q.B, q.N, K, BN / 2)) &&
                         make_out_map(&tmO1, q.out, q.M, q.N, EPI == EPI_F32);
        if (!ok2) return TPMLP_ERR_CUDA;
        g.second = 1;
        g.M2 = q.M;
        g.N2 = q.N;
        g.num_m_blocks2 = (q.M + kPairM - 1) / kPairM;
        g.num_n_blocks2 = (q.N + BN - 1) / BN;
    }
    g.M = M;
    g.N = N;
    g.K = K;
    g.num_m_blocks = (M + kPairM - 1) / kPairM;
    g.num_n_blocks = (N + BN - 1) / BN;
    g.k_blocks = (K + kBK - 1) / kBK;
    g.wait_limit_ns = g_wait_limit_ns.load();
    auto kern = gemm_tc2_kernel<BN, A_MN, B_MN, EPI, RELAY, LONG>;
    constexpr int id = kernel_id<BN, A_MN, B_MN, EPI, RELAY, LONG>();
    int max_pairs = 0;
    {
        std::lock_guard<std::mutex> lock(g_dev_mutex);
        int devn = 0;
        if (cudaGetDevice(&devn) != cudaSuccess || devn < 0 || devn >= kMaxDevices)
            return TPMLP_ERR_CUDA;
        DeviceInfo& d = g_dev[devn];
        if (!d.attr_set_pair[id]) {
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Cfg::SMEM_BYTES) != cudaSuccess)
                return TPMLP_ERR_CUDA;
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(static_cast<unsigned>(2 * (d.num_sms / 2)));
            cfg.blockDim = dim3(kThreads);
            cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
            cudaLaunchAttribute attr;
            attr.id = cudaLaunchAttributeClusterDimension;
            attr.val.clusterDim.x = 2;
            attr.val.clusterDim.y = 1;
            attr.val.clusterDim.z = 1;
            cfg.attrs = &attr;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) return TPMLP_ERR_CUDA;
            d.max_pairs[id] = n;
            d.attr_set_pair[id] = true;
        }
        max_pairs = d.max_pairs[id];
    }
    // never more workers than the plan sized the workspace for (num_sms / 2)
    const int pairs = resolve_sched(g, req, std::min(max_pairs, dev->num_sms / 2), kSplittable<EPI, RELAY>);
    if (!LONG || !req.dyn) g.dyn_counter = nullptr;
    return launch_dep(kern, dim3(2 * pairs), dim3(kThreads), Cfg::SMEM_BYTES, st, tmA, tmB, tmO0, tmO1,
                      tmA2, tmB2, g);
}

// Algorithmic bytes of one GEMM: both operands read once (bf16), the
// outputs written once, plus the epilogue's extra input (saved H) and the
// second output (Y) where the epilogue has them.
template <int EPI>
double gemm_bytes(double M, double N, double K) {
    double b = 2.0 * (M * K + K * N);
    if (EpiTraits<EPI>::kAct) b += 2.0 * 2.0 * M * N;
    if (EPI == EPI_BIAS) b += 2.0 * M * N;
    if (EpiTraits<EPI>::kDAct) b += 2.0 * 2.0 * M * N;
    if (EPI == EPI_F32) b += 4.0 * M * N;
    return b;
}

// Relay the epilogue (see epilogue_role) only when the K loop of a work unit
// is long enough to hide the doubled work of the computing warps. Measured
// (CTA pairs, 256 × 256 tiles): GeLU 0.622 -> 0.577 ms at K = 4096, even at
// K = 2048, 0.033 -> 0.053 ms at K = 768; fp32 store 0.318 -> 0.299 ms at
// K = 2048; bias store 0.548 -> 0.543 ms at K = 4096, 0.021 -> 0.027 ms at
// K = 768.
// The long-product kernel variant (two epilogue staging slots per warp, paid
// with one ring stage; able to run the dynamic schedule) for a bf16-output
// product on CTA pairs of at least 64 k-blocks per tile and 4 waves of tiles.
// Measured on B200 (same runs alternating): double staging is 1.5–3.5% faster
// for every such product of the 7B- and 175B-class workloads, and 6–15% slower
// for the GPT-2-small and 350M ones (12–64 k-blocks, 0.6–5 waves), where the
// producer's look-ahead across short tiles needs the sixth stage.
int plan_num_sms();

bool long_product(int epi, int64_t M, int64_t N, int64_t K) {
    if (epi == EPI_F32 || M <= kBM) return false;
    if (epi == EPI_F32) return false;
    const int64_t tiles = ((int64_t(M) + kPairM - 1) / kPairM) * ((int64_t(N) + 255) / 256);
    return (K + kBK - 1) / kBK >= 64 && tiles >= 4 * (plan_num_sms() / 2);
}

template <int BN, bool A_MN, bool B_MN, int EPI, bool RELAY>
tpmlp_status gemm_tc_pick(const void* Aop, const void* Bop, int M, int N, int K, const SchedReq& req,
                          const GemmArgs& g, cudaStream_t st) {
    // CTA pairs whenever a 256-row tile is not mostly padding
    if (M > kBM) {
        if constexpr (EPI != EPI_F32) {
            if (long_product(EPI, M, N, K))
                return gemm_tc2_launch<BN, A_MN, B_MN, EPI, RELAY, true>(Aop, Bop, M, N, K, req, g, st);
        }
        return gemm_tc2_launch<BN, A_MN, B_MN, EPI, RELAY>(Aop, Bop, M, N, K, req, g, st);
    }
    return gemm_tc_launch<BN, A_MN, B_MN, EPI, RELAY>(Aop, Bop, M, N, K, req, g, st);
}

// Shortest K loop per work unit for which the relaying epilogue pays
// (measured on the 7B-class and GPT-2-class shapes).
constexpr int kRelayMinKAct = 3072;    // GeLU and GeLU′ epilogues
constexpr int kRelayMinKPlain = 2048;  // bias and fp32 epilogues

// The relay also needs work to hide behind: it keeps the sub-partitions of
// the producer and the MMA issuer free for the next unit's K loop, but it
// halves the warps that compute and store, and a pair's last unit's epilogue
// overlaps nothing. With at most two units per CTA pair (on CTA pairs: M >
// 128) the full-width epilogue is faster. Measured on B200, alternating runs,
// bit-identical results: GPT-2-small step 698–709 → 736–742 TFLOP/s (Y·B and
// dH·Aᵀ, 48 tiles, 7–10% faster; the weight gradients, 72 tiles, 6%), 350M
// 987–995 → 1002–1012 (96 and 128 tiles, 2–4%); the 7B- and 175B-class
// products (≥ 512 tiles) keep the relay. The GeLU′ epilogue keeps the K rule
// alone: its da column sums are fused only into the relaying form.
bool relay_has_work(int64_t M, int64_t units) {
    return M <= kBM || units > 2 * static_cast<int64_t>(plan_num_sms() / 2);
}

int64_t pair_tiles(int64_t M, int64_t N) { return ((M + kPairM - 1) / kPairM) * ((N + 255) / 256); }

template <int BN, bool A_MN, bool B_MN, int EPI>
tpmlp_status gemm_tc(int kind, const void* Aop, const void* Bop, int M, int N, int K,
                     const SchedReq& req, GemmArgs g, cudaStream_t st) {
    return timed(kind, 2.0 * M * N * K, gemm_bytes<EPI>(M, N, K), st, [&] {
        const int k_per_unit = req.kind == SCHED_GROUPS && req.groups > 1 ? K / req.groups : K;
        const int threshold =
            (EpiTraits<EPI>::kAct || EpiTraits<EPI>::kDAct) ? kRelayMinKAct : kRelayMinKPlain;
        const int64_t units = pair_tiles(M, N) * (req.kind == SCHED_GROUPS ? req.groups : 1);
        if (k_per_unit < threshold || (!EpiTraits<EPI>::kDAct && !relay_has_work(M, units)))
            return gemm_tc_pick<BN, A_MN, B_MN, EPI, false>(Aop, Bop, M, N, K, req, g, st);
        return gemm_tc_pick<BN, A_MN, B_MN, EPI, true>(Aop, Bop, M, N, K, req, g, st);
    });
}

// Two products of the same kernel (fp32 epilogue) and K in one launch, as
// one list of whole tiles on the CTA pairs (both M > 128): the second's
// tiles follow the first's, so a short product no longer leaves half the
// GPU idle for its whole duration.
template <int BN, bool A_MN, bool B_MN>
tpmlp_status gemm_tc_grouped(int kind, const void* A0, const void* B0, int M0, int N0, void* out0,
                             const void* A1, const void* B1, int M1, int N1, void* out1, int K,
                             cudaStream_t st) {
    const double flops = 2.0 * (double(M0) * N0 + double(M1) * N1) * K;
    const double bytes = gemm_bytes<EPI_F32>(M0, N0, K) + gemm_bytes<EPI_F32>(M1, N1, K);
    return timed(kind, flops, bytes, st, [&] {
        GemmArgs g{};
        g.out0 = out0;
        g.ld_out = N0;
        const SchedReq req;  // whole tiles, static (fp32 outputs: no long-product variant)
        const SecondProduct second{A1, B1, M1, N1, out1};
        if (K < kRelayMinKPlain || !relay_has_work(M0, pair_tiles(M0, N0) + pair_tiles(M1, N1)))
            return gemm_tc2_launch<BN, A_MN, B_MN, EPI_F32, false>(A0, B0, M0, N0, K, req, g, st,
                                                                 &second);
        return gemm_tc2_launch<BN, A_MN, B_MN, EPI_F32, true>(A0, B0, M0, N0, K, req, g, st,
                                                            &second);
    });
}

template <typename T, int EPI>
tpmlp_status gemm_simt(int kind, const SimtArgs& a, cudaStream_t st) {
    const double flops = 2.0 * a.M * a.N * a.K;
    const double bytes = sizeof(T) * (1.0 * a.M * a.K + 1.0 * a.K * a.N) +
                         (EPI == EPI_F32 ? 4.0 : sizeof(T) * (EPI == EPI_BIAS ? 1.0 : 2.0)) * a.M * a.N;
    return timed(kind, flops, bytes, st, [&] {
        dim3 grid((a.N + 15) / 16, (a.M + 15) / 16);
        simt_gemm_kernel<T, EPI><<<grid, 256, 0, st>>>(a);
        return check_launch();
    });
}

// ---------------------------------------------------------------- planning

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Partial rows of da written by the relaying GeLU′ epilogue: two per 128-row
// CTA tile (one per computing warp, 64 rows each).
int64_t da_partial_rows(int64_t T) { return T > 0 ? 2 * ((T + kBM - 1) / kBM) : 1; }

// Workspace a call's split tiles need: fp32 partial tiles and arrival
// counters (16 per split tile). Shared by the call's products, which run
// one after another on the stream; every counter is back at zero when a
// launch completes, and the call zeroes them once before its first launch.
struct SplitSpace {
    size_t partial_bytes = 0, counter_bytes = 0;
    void need(size_t part, size_t ctr) {
        partial_bytes = std::max(partial_bytes, part);
        counter_bytes = std::max(counter_bytes, ctr);
    }
};

// Two ints after the split counters: the dynamic schedule's item counter and
// its count of finished pairs (zero at every launch; the last pair resets them).
constexpr size_t kDynCounterInts = 2;

// Whether a product runs the dynamic schedule: a long product (long_product,
// the only kernel variant that carries it) with at least 4 waves of items,
// at least kDynMinTileKBlocks k-blocks per tile (each item's hand-off costs
// a fixed time: 6% slower at 32 k-blocks, launches timed alone) and at least
// kDynMinPairKBlocks k-blocks of work per CTA pair. The last one is where
// the schedule pays: under a static round-robin the pairs drift apart in
// proportion to the work each runs (the slowest take ~5% longer per tile),
// and pairs that share an operand panel then read it from DRAM more than
// once. Measured on B200 in forward + backward steps of 1.7 s at the power
// limit (alternating runs, on against off): 175B-class, ~3990 k-blocks per
// pair in all four row products: step 0.5% faster, DRAM reads of X·A 40%
// lower (ncu); 7B-class Y·B and dH·Aᵀ, ~1770 k-blocks per pair: 0.7% slower
// each.
constexpr int64_t kDynMinTileKBlocks = 192;
constexpr int64_t kDynMinPairKBlocks = 3072;

bool wants_dynamic(int epi, int64_t M, int64_t N, int64_t items, int64_t K, int num_sms) {
    const int64_t kb = (K + kBK - 1) / kBK;
    const int64_t pairs = num_sms / 2;
    return g_dynamic.load() && long_product(epi, M, N, K) && items >= 4 * pairs &&
           kb >= kDynMinTileKBlocks && pair_tiles(M, N) * kb >= kDynMinPairKBlocks * pairs;
}

// Schedule of one tensor-core product (M × N output, K deep) under the
// current policy (tpmlp_set_split_policy):
//   0  stream-K tail where the time model says it pays (streamk_pays);
//   1  whole tiles only;
//   2  a row-parallel product (shard_groups > 1: p shards of whole k-blocks)
//      as one unit per shard and tile, the shards' partials added in
//      ascending order; other products as whole tiles;
//   3  stream-K tail wherever it is valid (for tests and measurement).
// The geometry is the launcher's: CTA pairs with 256-row tiles and
// num_sms / 2 workers when M > 128, else one CTA per 128-row tile and
// num_sms workers; 256-column tiles.
SchedReq plan_sched(int64_t M, int64_t N, int64_t K, int shard_groups, int num_sms, SplitSpace* sp,
                    bool may_split = true) {
    SchedReq r;
    const int policy = may_split ? g_split_policy.load() : 1;
    const bool pairs = M > kBM;
    const int64_t tile_rows = pairs ? kPairM : kBM;
    const int64_t workers = pairs ? num_sms / 2 : num_sms;
    const int64_t tiles = ((M + tile_rows - 1) / tile_rows) * ((N + 255) / 256);
    const int64_t kb = (K + kBK - 1) / kBK;
    const size_t tile_bytes = static_cast<size_t>(tile_rows) * 256 * sizeof(float);
    if (policy == 2 && shard_groups > 1 && kb % shard_groups == 0) {
        r.kind = SCHED_GROUPS;
        r.groups = shard_groups;
        sp->need(static_cast<size_t>(tiles) * shard_groups * tile_bytes,
                 static_cast<size_t>(tiles) * 16 * sizeof(int));
        return r;
    }
    if ((policy == 0 || policy == 3) && streamk_pays(tiles, kb, workers, policy == 3)) {
        r.kind = SCHED_STREAMK;
        r.force = (policy == 3);
        sp->need(static_cast<size_t>(2 * workers) * tile_bytes,
                 static_cast<size_t>(workers) * 16 * sizeof(int));
    }
    return r;
}

// Shard groups of a row-parallel product whose K = p shards of Fp: p when
// every shard is whole k-blocks, else none (the K loop runs through all shards).
int shard_groups(int64_t K, int p) {
    return (p > 1 && K % p == 0 && (K / p) % kBK == 0) ? p : 0;
}

int plan_num_sms() {
    if (const DeviceInfo* d = device_info()) return d->num_sms;
    return 148;
}

struct Plan {
    bool tc = false;    // tensor-core path (bf16, h % 8 == 0, F % 8 == 0)
    SchedReq f1, f2, b2, b3, b4, b5;
    bool fwd_split = false, bwd_split = false;  // some product of the call splits tiles
    bool fwd_dyn = false, bwd_dyn = false;      // some product of the call is dynamic
    bool group34 = false;                       // B3 and B4 in one launch
    int64_t chunks = 1; // column-sum row chunks
    size_t off_part = 0, off_ctr = 0, off_dyn = 0, ctr_bytes = 0, off_cs_h = 0, off_cs_f = 0, total = 0;
};

bool make_plan(int64_t T, int64_t h, int64_t F, int p, tpmlp_dtype dt, Plan* pl) {
    if (T < 0 || h < 1 || F < 1 || p < 1 || F % p != 0) return false;
    if (dt != TPMLP_BF16 && dt != TPMLP_FP32) return false;
    pl->tc = (dt == TPMLP_BF16) && (h % 8 == 0) && (F % 8 == 0);
    SplitSpace sp;
    if (pl->tc && T > 0) {
        const int sms = plan_num_sms();
        // X·A: whole tiles when the GeLU epilogue relays (K = h ≥ 3072), whose
        // kernel has no split path
        pl->f1 = plan_sched(T, F, h, 0, sms, &sp, h < kRelayMinKAct);
        pl->f2 = plan_sched(T, h, F, shard_groups(F, p), sms, &sp);  // Σ Y_i·B_i
        // dZ·Bᵀ: whole tiles when its relaying epilogue also sums da's columns
        // (those sums pair the rows of two warps, which a split tile, finished
        // warp by warp, does not have together)
        pl->b2 = plan_sched(T, F, h, 0, sms, &sp, h < kRelayMinKAct);
        pl->b3 = plan_sched(F, h, T, 0, sms, &sp);                   // Yᵀ·dZ
        pl->b4 = plan_sched(h, F, T, 0, sms, &sp);                   // Xᵀ·dH
        pl->b5 = plan_sched(T, h, F, shard_groups(F, p), sms, &sp);  // Σ dH_i·A_iᵀ
        pl->fwd_split = pl->f1.kind != SCHED_TILES || pl->f2.kind != SCHED_TILES;
        pl->bwd_split = pl->b2.kind != SCHED_TILES || pl->b3.kind != SCHED_TILES ||
                        pl->b4.kind != SCHED_TILES || pl->b5.kind != SCHED_TILES;
        pl->group34 = pl->b3.kind == SCHED_TILES && pl->b4.kind == SCHED_TILES && F > kBM && h > kBM;
        // items of each product (a split tile's units count as items too)
        auto items = [&](const SchedReq& r, int64_t M, int64_t N) {
            return pair_tiles(M, N) * (r.kind == SCHED_GROUPS ? r.groups : 1);
        };
        pl->f1.dyn = wants_dynamic(EPI_GELU, T, F, items(pl->f1, T, F), h, sms);
        pl->f2.dyn = wants_dynamic(EPI_BIAS, T, h, items(pl->f2, T, h), F, sms);
        pl->b2.dyn = wants_dynamic(EPI_DGELU, T, F, items(pl->b2, T, F), h, sms);
        // the weight gradients (fp32 outputs) always run statically
        pl->b3.dyn = pl->b4.dyn = false;
        pl->b5.dyn = wants_dynamic(EPI_BIAS, T, h, items(pl->b5, T, h), F, sms);
        pl->fwd_dyn = pl->f1.dyn || pl->f2.dyn;
        pl->bwd_dyn = pl->b2.dyn || pl->b3.dyn || pl->b4.dyn || pl->b5.dyn;
    }
    pl->chunks = T > 0 ? (T + kColsumRowsPerChunk - 1) / kColsumRowsPerChunk : 1;
    size_t off = 0;
    pl->off_part = off;
    off += round256(sp.partial_bytes);
    pl->off_ctr = off;
    pl->off_dyn = pl->off_ctr + sp.counter_bytes;  // the dynamic schedule's two ints
    pl->ctr_bytes = (pl->fwd_dyn || pl->bwd_dyn)
                        ? round256(sp.counter_bytes + kDynCounterInts * sizeof(int))
                        : round256(sp.counter_bytes);
    off += pl->ctr_bytes;
    pl->off_cs_h = off;
    off += round256(static_cast<size_t>(pl->chunks) * h * sizeof(float));
    pl->off_cs_f = off;
    // tensor-core path: da's partials come from the GeLU′ epilogue (two rows per
    // 128 token rows) or from the column-sum kernel (one per 128); plain path:
    // the column-sum kernel
    off += round256(static_cast<size_t>(pl->tc ? da_partial_rows(T) : pl->chunks) * F * sizeof(float));
    pl->total = off;
    return true;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Blocks of `threads` threads that the device holds at once for KERNEL (per
// SM from the occupancy calculator, cached per kernel). Grid-stride kernels
// launch no more than this, so that no block waits for a second wave.
template <auto KERNEL>
int64_t resident_blocks(int threads) {
    static std::atomic<int> cached{0};
    int per_sm = cached.load(std::memory_order_relaxed);
    if (per_sm == 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, KERNEL, threads, 0) !=
                cudaSuccess || per_sm < 1) {
            cudaGetLastError();
            per_sm = 1;
        }
        cached.store(per_sm, std::memory_order_relaxed);
    }
    const DeviceInfo* d = device_info();
    return static_cast<int64_t>(per_sm) * (d ? d->num_sms : 148);
}

int64_t clamp_grid(int64_t blocks, int64_t cap) {
    if (blocks > cap) blocks = cap;
    return blocks < 1 ? 1 : blocks;
}

template <typename T>
tpmlp_status colsum_launch(const T* X, int64_t R, int64_t C, int64_t chunks, float* partial,
                           float* out, cudaStream_t st) {
    dim3 grid(static_cast<unsigned>((C + 255) / 256), static_cast<unsigned>(chunks));
    dim3 block(32, 8);
    const tpmlp_status s =
        (C % 8 == 0 && aligned16(X))
            ? launch_dep(colsum_partial_kernel<T, true>, grid, block, 0, st, X, R, C,
                         kColsumRowsPerChunk, partial)
            : launch_dep(colsum_partial_kernel<T, false>, grid, block, 0, st, X, R, C,
                         kColsumRowsPerChunk, partial);
    if (s != TPMLP_OK) return s;
    return launch_dep(colsum_final_kernel, dim3(static_cast<unsigned>((C + 31) / 32)), dim3(32, 8), 0,
                      st, static_cast<const float*>(partial), static_cast<int>(chunks), C, out);
}

// out = 1ᵀ·X for X: R × C; algorithmic bytes = X read once + out written.
template <typename T>
tpmlp_status colsum(int kind, const T* X, int64_t R, int64_t C, int64_t chunks, float* partial,
                    float* out, cudaStream_t st) {
    return timed(kind, 0.0, sizeof(T) * double(R) * C + 4.0 * C, st,
                 [&] { return colsum_launch(X, R, C, chunks, partial, out, st); });
}

// Both bias gradients' column sums in two launches instead of four: pass 1
// over X1 (R × C1) and X2 (R × C2) in one grid, then pass 2 of both. Each
// column's sum is computed exactly as colsum computes it.
template <typename T>
tpmlp_status colsum2(int kind, const T* X1, int64_t C1, float* partial1, float* out1, const T* X2,
                     int64_t C2, float* partial2, float* out2, int64_t R, int64_t chunks,
                     cudaStream_t st) {
    return timed(kind, 0.0, sizeof(T) * double(R) * (C1 + C2) + 4.0 * (C1 + C2), st, [&] {
        dim3 grid(static_cast<unsigned>((C1 + 255) / 256 + (C2 + 255) / 256),
                  static_cast<unsigned>(chunks));
        const bool vec = C1 % 8 == 0 && C2 % 8 == 0 && aligned16(X1) && aligned16(X2);
        const tpmlp_status s =
            vec ? launch_dep(colsum_partial2_kernel<T, true>, grid, dim3(32, 8), 0, st, X1, C1,
                             partial1, X2, C2, partial2, R, kColsumRowsPerChunk)
                : launch_dep(colsum_partial2_kernel<T, false>, grid, dim3(32, 8), 0, st, X1, C1,
                             partial1, X2, C2, partial2, R, kColsumRowsPerChunk);
        if (s != TPMLP_OK) return s;
        return launch_dep(colsum_final2_kernel,
                          dim3(static_cast<unsigned>((C1 + 31) / 32 + (C2 + 31) / 32)), dim3(32, 8), 0,
                          st, static_cast<const float*>(partial1), static_cast<int>(chunks), C1, out1,
                          static_cast<const float*>(partial2), static_cast<int>(chunks), C2, out2);
    });
}

// Pass 1 alone (its pass 2 runs later through colsum_finish2).
template <typename T>
tpmlp_status colsum_first(int kind, const T* X, int64_t R, int64_t C, int64_t chunks, float* partial,
                          cudaStream_t st) {
    return timed(kind, 0.0, sizeof(T) * double(R) * C + 4.0 * double(chunks) * C, st, [&] {
        dim3 grid(static_cast<unsigned>((C + 255) / 256), static_cast<unsigned>(chunks));
        return (C % 8 == 0 && aligned16(X))
                   ? launch_dep(colsum_partial_kernel<T, true>, grid, dim3(32, 8), 0, st, X, R, C,
                                kColsumRowsPerChunk, partial)
                   : launch_dep(colsum_partial_kernel<T, false>, grid, dim3(32, 8), 0, st, X, R, C,
                                kColsumRowsPerChunk, partial);
    });
}

// Pass 2 of two sets of partials in one launch: out1[c] = Σ_r partial1[r][c]
// over rows1 rows and out2 likewise, each in ascending r.
tpmlp_status colsum_finish2(int kind, const float* partial1, int64_t rows1, int64_t C1, float* out1,
                            const float* partial2, int64_t rows2, int64_t C2, float* out2,
                            cudaStream_t st) {
    return timed(kind, 0.0, 4.0 * (double(rows1) * C1 + double(rows2) * C2 + C1 + C2), st, [&] {
        return launch_dep(colsum_final2_kernel,
                          dim3(static_cast<unsigned>((C1 + 31) / 32 + (C2 + 31) / 32)), dim3(32, 8), 0,
                          st, partial1, static_cast<int>(rows1), C1, out1, partial2,
                          static_cast<int>(rows2), C2, out2);
    });
}

// One launch of recompute_act_kernel over n elements: a thread-iteration
// takes two 8-element groups (VEC) or one element; no more blocks than the
// device holds at once.
template <typename T, bool TANH, bool VEC>
tpmlp_status launch_recompute(const void* H, void* Y, int64_t n, cudaStream_t st) {
    const int64_t work = VEC ? (n / 8 + 1) / 2 : n;
    const unsigned nb = static_cast<unsigned>(
        clamp_grid((work + 255) / 256, resident_blocks<recompute_act_kernel<T, TANH, VEC>>(256)));
    return launch_dep(recompute_act_kernel<T, TANH, VEC>, dim3(nb), dim3(256), 0, st,
                      static_cast<const T*>(H), static_cast<T*>(Y), n);
}

tpmlp_status zero_f32(float* p, int64_t n, cudaStream_t st, int kind = K_MISC) {
    if (n <= 0) return TPMLP_OK;
    return timed(kind, 0.0, 4.0 * n, st, [&] {
        const int64_t blocks = clamp_grid((n + 255) / 256, resident_blocks<zero_f32_kernel>(256));
        return launch_dep(zero_f32_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, st, p, n);
    });
}

// Arrival counters of split tiles: zeroed once at the start of a call whose
// plan splits tiles (each launch leaves them at zero again).
tpmlp_status reset_counters(void* workspace, size_t off, size_t bytes, cudaStream_t st) {
    float* p = reinterpret_cast<float*>(static_cast<char*>(workspace) + off);  // 0.0f is all-zero bits
    return zero_f32(p, static_cast<int64_t>(bytes / sizeof(float)), st, K_CTR);
}

// Workspace pointers of a call's split tiles.
void set_split_space(GemmArgs& g, void* workspace, size_t off_part, size_t off_ctr) {
    g.partials = reinterpret_cast<float*>(static_cast<char*>(workspace) + off_part);
    g.counters = reinterpret_cast<int*>(static_cast<char*>(workspace) + off_ctr);
}

// The dynamic schedule's counters (used only by a launch whose request says so).
int* dyn_space(void* workspace, size_t off_dyn) {
    return reinterpret_cast<int*>(static_cast<char*>(workspace) + off_dyn);
}

// The counters must be zero before the first product of a call that splits
// tiles. `g` is the call's first GEMM (launched next, with schedule `req`):
// if it runs whole tiles, its own kernel zeroes them for the later products
// (no extra launch); otherwise a reset kernel runs first.
tpmlp_status zero_counters_before(GemmArgs& g, const SchedReq& req, void* workspace, size_t off_ctr,
                                  size_t bytes, cudaStream_t st) {
    if (req.kind == SCHED_TILES) {
        g.zero_counters = reinterpret_cast<int*>(static_cast<char*>(workspace) + off_ctr);
        g.zero_count = static_cast<int>(bytes / sizeof(int));
        return TPMLP_OK;
    }
    return reset_counters(workspace, off_ctr, bytes, st);
}

#define TPMLP_TRY(expr)                         \
    do {                                        \
        tpmlp_status _s = (expr);               \
        if (_s != TPMLP_OK) return _s;          \
    } while (0)

tpmlp_status common_checks(int64_t T, int64_t h, int64_t F, int p, tpmlp_dtype dt, Plan* pl,
                           void* ws, size_t ws_bytes, bool need_ws = true) {
    if (!make_plan(T, h, F, p, dt, pl)) return TPMLP_ERR_INVALID;
    // the kernels index rows, columns and tiles with 32-bit integers
    if (T >= (int64_t(1) << 31) || h >= (int64_t(1) << 31) || F >= (int64_t(1) << 31))
        return TPMLP_ERR_UNSUPPORTED;
    const DeviceInfo* d = device_info();
    if (d == nullptr) return TPMLP_ERR_CUDA;
    if (d->cc_major != 10) return TPMLP_ERR_UNSUPPORTED;
    if (need_ws && pl->total > 0 && (ws == nullptr || ws_bytes < pl->total))
        return TPMLP_ERR_WORKSPACE;
    if (ws != nullptr && !aligned16(ws)) return TPMLP_ERR_ALIGN;
    return TPMLP_OK;
}

// ------------------------------------------------ tensor-parallel linear

// Plan of a linear layer Y = X·W + bias (X: T × K, W: K × N), W split into
// p shards by columns (split 0) or rows (split 1). The product carrying a
// shard sum (the forward for rows, dX of the backward for columns) may run
// one unit per shard and tile like the MLP's row-parallel products; every
// product may take a stream-K tail.
struct LinPlan {
    bool tc = false;
    SchedReq fwd, dw, dx;
    bool fwd_split = false, bwd_split = false;
    int64_t chunks = 1;
    size_t off_part = 0, off_ctr = 0, ctr_bytes = 0, off_cs = 0, total = 0;
};

bool make_lin_plan(int64_t T, int64_t K, int64_t N, int p, int split, tpmlp_dtype dt, LinPlan* pl) {
    if (T < 0 || K < 1 || N < 1 || p < 1 || (split != 0 && split != 1)) return false;
    if (split == 0 && N % p != 0) return false;
    if (split == 1 && K % p != 0) return false;
    if (dt != TPMLP_BF16 && dt != TPMLP_FP32) return false;
    pl->tc = (dt == TPMLP_BF16) && (K % 8 == 0) && (N % 8 == 0);
    SplitSpace sp;
    if (pl->tc && T > 0) {
        const int sms = plan_num_sms();
        pl->fwd = plan_sched(T, N, K, split == 1 ? shard_groups(K, p) : 0, sms, &sp);
        pl->dw = plan_sched(K, N, T, 0, sms, &sp);
        pl->dx = plan_sched(T, K, N, split == 0 ? shard_groups(N, p) : 0, sms, &sp);
        pl->fwd_split = pl->fwd.kind != SCHED_TILES;
        pl->bwd_split = pl->dw.kind != SCHED_TILES || pl->dx.kind != SCHED_TILES;
    }
    pl->chunks = T > 0 ? (T + kColsumRowsPerChunk - 1) / kColsumRowsPerChunk : 1;
    pl->off_part = 0;
    pl->off_ctr = round256(sp.partial_bytes);
    pl->ctr_bytes = round256(sp.counter_bytes);
    pl->off_cs = pl->off_ctr + pl->ctr_bytes;
    pl->total = pl->off_cs + round256(static_cast<size_t>(pl->chunks) * N * sizeof(float));
    return true;
}

tpmlp_status lin_checks(int64_t T, int64_t K, int64_t N, int p, int split, tpmlp_dtype dt,
                        LinPlan* pl, void* ws, size_t ws_bytes) {
    if (!make_lin_plan(T, K, N, p, split, dt, pl)) return TPMLP_ERR_INVALID;
    if (T >= (int64_t(1) << 31) || K >= (int64_t(1) << 31) || N >= (int64_t(1) << 31))
        return TPMLP_ERR_UNSUPPORTED;
    const DeviceInfo* d = device_info();
    if (d == nullptr) return TPMLP_ERR_CUDA;
    if (d->cc_major != 10) return TPMLP_ERR_UNSUPPORTED;
    if (pl->total > 0 && (ws == nullptr || ws_bytes < pl->total))
        return TPMLP_ERR_WORKSPACE;
    if (ws != nullptr && !aligned16(ws)) return TPMLP_ERR_ALIGN;
    return TPMLP_OK;
}

tpmlp_status linear_fwd_impl(const void* X, const void* W, const void* bias, void* Y, int64_t T,
                             int64_t K, int64_t N, int p, int split, tpmlp_dtype dt, void* workspace,
                             size_t workspace_bytes, cudaStream_t st) {
    LinPlan pl;
    TPMLP_TRY(lin_checks(T, K, N, p, split, dt, &pl, workspace, workspace_bytes));
    if (T == 0) return TPMLP_OK;
    if (!X || !W || !Y) return TPMLP_ERR_INVALID;
    const int iT = static_cast<int>(T), iK = static_cast<int>(K), iN = static_cast<int>(N);
    if (pl.tc) {
        for (const void* q : {X, W, bias, static_cast<const void*>(Y)})
            if (q && !aligned16(q)) return TPMLP_ERR_ALIGN;
        if (pl.fwd_split) TPMLP_TRY(reset_counters(workspace, pl.off_ctr, pl.ctr_bytes, st));
        // Aop = X [T][K] (K-major), Bop = W [K][N] (MN-major); for the row split
        // the K loop (or the units' partials) runs through the shards in order
        GemmArgs g{};
        set_split_space(g, workspace, pl.off_part, pl.off_ctr);
        g.out0 = Y;
        g.ld_out = N;
        g.bias = static_cast<const __nv_bfloat16*>(bias);
        return gemm_tc<256, false, true, EPI_BIAS>(K_L_FWD, X, W, iT, iN, iK, pl.fwd, g, st);
    }
    SimtArgs a{};
    a.M = iT; a.N = iN; a.K = iK;
    a.A = X; a.sam = K; a.sak = 1;
    a.B = W; a.sbk = N; a.sbn = 1;
    a.out0 = Y; a.ld_out = N; a.bias = bias;
    if (dt == TPMLP_FP32) return gemm_simt<float, EPI_BIAS>(K_L_FWD, a, st);
    return gemm_simt<__nv_bfloat16, EPI_BIAS>(K_L_FWD, a, st);
}

tpmlp_status linear_bwd_impl(const void* dY, const void* X, const void* W, void* dX, float* dW,
                             float* dbias, int64_t T, int64_t K, int64_t N, int p, int split,
                             tpmlp_dtype dt, void* workspace, size_t workspace_bytes,
                             cudaStream_t st) {
    LinPlan pl;
    TPMLP_TRY(lin_checks(T, K, N, p, split, dt, &pl, workspace, workspace_bytes));
    if (!dW || !dbias) return TPMLP_ERR_INVALID;
    if (T == 0) {
        TPMLP_TRY(zero_f32(dW, K * N, st));
        return zero_f32(dbias, N, st);
    }
    if (!dY || !X || !W || !dX) return TPMLP_ERR_INVALID;
    float* cs = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.off_cs);
    const int iT = static_cast<int>(T), iK = static_cast<int>(K), iN = static_cast<int>(N);
    if (pl.tc) {
        for (const void* q : {dY, X, W, static_cast<const void*>(dX), static_cast<const void*>(dW),
                              static_cast<const void*>(dbias)})
            if (!aligned16(q)) return TPMLP_ERR_ALIGN;
        TPMLP_TRY(colsum(K_L_DB, static_cast<const __nv_bfloat16*>(dY), T, N, pl.chunks, cs, dbias, st));
        // dW = Xᵀ·dY: Aop = X [T][K] (MN-major, M = K), Bop = dY [T][N] (MN-major)
        GemmArgs gw{};
        set_split_space(gw, workspace, pl.off_part, pl.off_ctr);
        if (pl.bwd_split) TPMLP_TRY(zero_counters_before(gw, pl.dw, workspace, pl.off_ctr, pl.ctr_bytes, st));
        gw.out0 = dW;
        gw.ld_out = N;
        TPMLP_TRY((gemm_tc<256, true, true, EPI_F32>(K_L_DW, X, dY, iK, iN, iT, pl.dw, gw, st)));
        // dX = dY·Wᵀ: Aop = dY [T][N] (K-major), Bop = W [K][N] read as [N' = K][K' = N] (K-major);
        // for the column split this is the shard sum over the N dimension
        GemmArgs gx{};
        set_split_space(gx, workspace, pl.off_part, pl.off_ctr);
        gx.out0 = dX;
        gx.ld_out = K;
        return gemm_tc<256, false, false, EPI_BIAS>(K_L_DX, dY, W, iT, iK, iN, pl.dx, gx, st);
    }
    // dW = Xᵀ·dY: Aop(k, t) = X[t][k], Bop(t, n) = dY[t][n]
    SimtArgs w{};
    w.M = iK; w.N = iN; w.K = iT;
    w.A = X; w.sam = 1; w.sak = K;
    w.B = dY; w.sbk = N; w.sbn = 1;
    w.out0 = dW; w.ld_out = N;
    // dX = dY·Wᵀ: Aop(t, n) = dY[t][n], Bop(n, k) = W[k][n]
    SimtArgs x{};
    x.M = iT; x.N = iK; x.K = iN;
    x.A = dY; x.sam = N; x.sak = 1;
    x.B = W; x.sbk = 1; x.sbn = N;
    x.out0 = dX; x.ld_out = K;
    if (dt == TPMLP_FP32) {
        TPMLP_TRY(colsum(K_L_DB, static_cast<const float*>(dY), T, N, pl.chunks, cs, dbias, st));
        TPMLP_TRY((gemm_simt<float, EPI_F32>(K_L_DW, w, st)));
        return gemm_simt<float, EPI_BIAS>(K_L_DX, x, st);
    }
    TPMLP_TRY(colsum(K_L_DB, static_cast<const __nv_bfloat16*>(dY), T, N, pl.chunks, cs, dbias, st));
    TPMLP_TRY((gemm_simt<__nv_bfloat16, EPI_F32>(K_L_DW, w, st)));
    return gemm_simt<__nv_bfloat16, EPI_BIAS>(K_L_DX, x, st);
}

// Forward with activation epilogue EPI_ACT (EPI_GELU or EPI_GELU_TANH).
// with_f2 = false runs F1 alone (H and Y from X; B, b and Z unused).
template <int EPI_ACT>
tpmlp_status fwd_impl(const void* X, const void* A, const void* a, const void* B, const void* b,
                      void* H, void* Y, void* Z, int64_t T, int64_t h, int64_t F, int p,
                      tpmlp_dtype dt, void* workspace, size_t workspace_bytes, void* stream,
                      bool with_f2 = true) {
    cudaGetLastError();  // start from a clean (non-sticky) error state
    Plan pl;
    TPMLP_TRY(common_checks(T, h, F, p, dt, &pl, workspace, workspace_bytes, with_f2));
    if (T == 0) return TPMLP_OK;
    if (!X || !A || !H || !Y) return TPMLP_ERR_INVALID;
    if (with_f2 && (!B || !Z)) return TPMLP_ERR_INVALID;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (pl.tc) {
        for (const void* q : {X, A, a, B, b, static_cast<const void*>(H), static_cast<const void*>(Y),
                              static_cast<const void*>(Z)})
            if (q && !aligned16(q)) return TPMLP_ERR_ALIGN;
        const int iT = static_cast<int>(T), ih = static_cast<int>(h), iF = static_cast<int>(F);
        // without F2 (activation recompute) there is no workspace: whole tiles
        const SchedReq f1 = with_f2 ? pl.f1 : SchedReq{};
        // F1: H = X·A + a, Y = GeLU(H). Aop = X [T][h] (K-major), Bop = A [h][F] (MN-major).
        GemmArgs g1{};
        if (with_f2) {
            set_split_space(g1, workspace, pl.off_part, pl.off_ctr);
            g1.dyn_counter = dyn_space(workspace, pl.off_dyn);
        }
        if (with_f2 && pl.fwd_dyn)  // the first product itself needs them zero
            TPMLP_TRY(reset_counters(workspace, pl.off_ctr, pl.ctr_bytes, st));
        else if (with_f2 && pl.fwd_split)
            TPMLP_TRY(zero_counters_before(g1, f1, workspace, pl.off_ctr, pl.ctr_bytes, st));
        g1.out0 = H;
        g1.out1 = Y;
        g1.ld_out = F;
        g1.bias = static_cast<const __nv_bfloat16*>(a);
        TPMLP_TRY((gemm_tc<256, false, true, EPI_ACT>(K_F1, X, A, iT, iF, ih, f1, g1, st)));
        if (!with_f2) return TPMLP_OK;
        // F2: Z = Σ_i Y_i·B_i + b. Aop = Y [T][F] (K-major), Bop = B [F][h] (MN-major).
        // Each tile's K loop runs through the shards in ascending order; where
        // the schedule splits a tile, the units' partials are added in ascending
        // order in the epilogue of the last one, then b once.
        GemmArgs g2{};
        set_split_space(g2, workspace, pl.off_part, pl.off_ctr);
        g2.dyn_counter = dyn_space(workspace, pl.off_dyn);
        g2.out0 = Z;
        g2.ld_out = h;
        g2.bias = static_cast<const __nv_bfloat16*>(b);
        TPMLP_TRY((gemm_tc<256, false, true, EPI_BIAS>(K_F2, Y, B, iT, ih, iF, pl.f2, g2, st)));
        return TPMLP_OK;
    }
    // plain CUDA-core path: fp32, or bf16 with h or F not a multiple of 8
    SimtArgs s1{};
    s1.M = static_cast<int>(T); s1.N = static_cast<int>(F); s1.K = static_cast<int>(h);
    s1.A = X; s1.sam = h; s1.sak = 1;
    s1.B = A; s1.sbk = F; s1.sbn = 1;
    s1.out0 = H; s1.out1 = Y; s1.ld_out = F; s1.bias = a;
    SimtArgs s2{};
    s2.M = static_cast<int>(T); s2.N = static_cast<int>(h); s2.K = static_cast<int>(F);
    s2.A = Y; s2.sam = F; s2.sak = 1;
    s2.B = B; s2.sbk = h; s2.sbn = 1;
    s2.out0 = Z; s2.ld_out = h; s2.bias = b;
    if (dt == TPMLP_FP32) {
        TPMLP_TRY((gemm_simt<float, EPI_ACT>(K_F1, s1, st)));
        if (with_f2) TPMLP_TRY((gemm_simt<float, EPI_BIAS>(K_F2, s2, st)));
    } else {
        TPMLP_TRY((gemm_simt<__nv_bfloat16, EPI_ACT>(K_F1, s1, st)));
        if (with_f2) TPMLP_TRY((gemm_simt<__nv_bfloat16, EPI_BIAS>(K_F2, s2, st)));
    }
    return TPMLP_OK;
}

// Backward with activation-derivative epilogue EPI_DACT (EPI_DGELU or EPI_DGELU_TANH).
template <int EPI_DACT>
tpmlp_status bwd_impl(const void* dZ, const void* X, const void* A, const void* B, const void* H,
                      const void* Y, void* dX, float* dA, float* da, float* dB, float* db,
                      void* dH, int64_t T, int64_t h, int64_t F, int p, tpmlp_dtype dt,
                      void* workspace, size_t workspace_bytes, void* stream) {
    cudaGetLastError();
    Plan pl;
    TPMLP_TRY(common_checks(T, h, F, p, dt, &pl, workspace, workspace_bytes));
    if (!dA || !da || !dB || !db) return TPMLP_ERR_INVALID;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        TPMLP_TRY(zero_f32(dA, h * F, st));
        TPMLP_TRY(zero_f32(da, F, st));
        TPMLP_TRY(zero_f32(dB, F * h, st));
        TPMLP_TRY(zero_f32(db, h, st));
        return TPMLP_OK;
    }
    if (!dZ || !X || !A || !B || !H || !Y || !dX || !dH) return TPMLP_ERR_INVALID;
    float* cs_h = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.off_cs_h);
    float* cs_f = reinterpret_cast<float*>(static_cast<char*>(workspace) + pl.off_cs_f);
    if (pl.tc) {
        for (const void* q : {dZ, X, A, B, H, Y, static_cast<const void*>(dX),
                              static_cast<const void*>(dA), static_cast<const void*>(da),
                              static_cast<const void*>(dB), static_cast<const void*>(db),
                              static_cast<const void*>(dH)})
            if (!aligned16(q)) return TPMLP_ERR_ALIGN;
        const int iT = static_cast<int>(T), ih = static_cast<int>(h), iF = static_cast<int>(F);
        const __nv_bfloat16* dZb = static_cast<const __nv_bfloat16*>(dZ);
        int* dyn = dyn_space(workspace, pl.off_dyn);
        if (pl.bwd_dyn) TPMLP_TRY(reset_counters(workspace, pl.off_ctr, pl.ctr_bytes, st));
        // B2: dH = (dZ·Bᵀ) ⊙ GeLU′(H). Aop = dZ [T][h] (K-major), Bop = B [F][h] (K-major).
        // With the relaying epilogue (long K) the computing warps have room to
        // also leave the column sums of dH in cs_f (two partial rows per
        // 128-row tile); da then needs only their ordered sum. With short K
        // the extra epilogue work costs more than the separate pass, and db
        // (which nothing in the backward reads) waits for it: both column
        // sums then take one two-pass pair of launches after B2. With da
        // fused, db's first pass runs before B2 and its second shares one
        // launch with da's ordered sum after it.
        const bool fused_da = h >= kRelayMinKAct;
        // db = 1ᵀ·dZ, pass 1
        if (fused_da) TPMLP_TRY(colsum_first(K_B1_DB, dZb, T, h, pl.chunks, cs_h, st));
        GemmArgs g2{};
        set_split_space(g2, workspace, pl.off_part, pl.off_ctr);
        g2.dyn_counter = dyn;
        if (pl.bwd_split && !pl.bwd_dyn)
            TPMLP_TRY(zero_counters_before(g2, pl.b2, workspace, pl.off_ctr, pl.ctr_bytes, st));
        g2.out0 = dH;
        g2.ld_out = F;
        g2.aux = static_cast<const __nv_bfloat16*>(H);
        g2.colsum_out = fused_da ? cs_f : nullptr;
        TPMLP_TRY((gemm_tc<256, false, false, EPI_DACT>(K_B2, dZ, B, iT, iF, ih, pl.b2, g2, st)));
        // da = 1ᵀ·dH and db's pass 2 (or both whole column sums)
        if (fused_da)
            TPMLP_TRY(colsum_finish2(K_B12, cs_h, pl.chunks, h, db, cs_f, da_partial_rows(T), F, da, st));
        else
            TPMLP_TRY(colsum2(K_B12, dZb, h, cs_h, db, static_cast<const __nv_bfloat16*>(dH), F, cs_f,
                              da, T, pl.chunks, st));
        // B3: dB = Yᵀ·dZ. Aop = Y [T][F] (MN-major, M = F), Bop = dZ [T][h] (MN-major).
        // B4: dA = Xᵀ·dH. Aop = X [T][h] (MN-major, M = h), Bop = dH [T][F] (MN-major).
        // Same kernel and K = T: one launch of both when both run whole tiles.
        if (pl.group34) {
            TPMLP_TRY((gemm_tc_grouped<256, true, true>(K_B34, Y, dZ, iF, ih, dB, X, dH, ih, iF, dA,
                                                        iT, st)));
        } else {
            GemmArgs g3{};
            set_split_space(g3, workspace, pl.off_part, pl.off_ctr);
            g3.out0 = dB;
            g3.ld_out = h;
            TPMLP_TRY((gemm_tc<256, true, true, EPI_F32>(K_B3, Y, dZ, iF, ih, iT, pl.b3, g3, st)));
            GemmArgs g4{};
            set_split_space(g4, workspace, pl.off_part, pl.off_ctr);
            g4.out0 = dA;
            g4.ld_out = F;
            TPMLP_TRY((gemm_tc<256, true, true, EPI_F32>(K_B4, X, dH, ih, iF, iT, pl.b4, g4, st)));
        }
        // B5: dX = Σ_i dH_i·A_iᵀ. Aop = dH [T][F] (K-major), Bop = A [h][F] (K-major).
        GemmArgs g5{};
        set_split_space(g5, workspace, pl.off_part, pl.off_ctr);
        g5.dyn_counter = dyn;
        g5.out0 = dX;
        g5.ld_out = h;
        TPMLP_TRY((gemm_tc<256, false, false, EPI_BIAS>(K_B5, dH, A, iT, ih, iF, pl.b5, g5, st)));
        return TPMLP_OK;
    }
    const int iT = static_cast<int>(T), ih = static_cast<int>(h), iF = static_cast<int>(F);
    // B2: dH = (dZ·Bᵀ) ⊙ GeLU′(H): Aop(t, j) = dZ[t][j], Bop(j, f) = B[f][j]
    SimtArgs s2{};
    s2.M = iT; s2.N = iF; s2.K = ih;
    s2.A = dZ; s2.sam = h; s2.sak = 1;
    s2.B = B; s2.sbk = 1; s2.sbn = h;
    s2.out0 = dH; s2.ld_out = F; s2.aux = H;
    // B3: dB = Yᵀ·dZ: Aop(f, t) = Y[t][f], Bop(t, j) = dZ[t][j]
    SimtArgs s3{};
    s3.M = iF; s3.N = ih; s3.K = iT;
    s3.A = Y; s3.sam = 1; s3.sak = F;
    s3.B = dZ; s3.sbk = h; s3.sbn = 1;
    s3.out0 = dB; s3.ld_out = h;
    // B4: dA = Xᵀ·dH: Aop(k, t) = X[t][k], Bop(t, f) = dH[t][f]
    SimtArgs s4{};
    s4.M = ih; s4.N = iF; s4.K = iT;
    s4.A = X; s4.sam = 1; s4.sak = h;
    s4.B = dH; s4.sbk = F; s4.sbn = 1;
    s4.out0 = dA; s4.ld_out = F;
    // B5: dX = dH·Aᵀ: Aop(t, f) = dH[t][f], Bop(f, k) = A[k][f]
    SimtArgs s5{};
    s5.M = iT; s5.N = ih; s5.K = iF;
    s5.A = dH; s5.sam = F; s5.sak = 1;
    s5.B = A; s5.sbk = 1; s5.sbn = F;
    s5.out0 = dX; s5.ld_out = h;
    if (dt == TPMLP_FP32) {
        TPMLP_TRY(colsum(K_B1_DB, static_cast<const float*>(dZ), T, h, pl.chunks, cs_h, db, st));
        TPMLP_TRY((gemm_simt<float, EPI_DACT>(K_B2, s2, st)));
        TPMLP_TRY(colsum(K_B2_DA, static_cast<const float*>(dH), T, F, pl.chunks, cs_f, da, st));
        TPMLP_TRY((gemm_simt<float, EPI_F32>(K_B3, s3, st)));
        TPMLP_TRY((gemm_simt<float, EPI_F32>(K_B4, s4, st)));
        TPMLP_TRY((gemm_simt<float, EPI_BIAS>(K_B5, s5, st)));
    } else {
        TPMLP_TRY(colsum(K_B1_DB, static_cast<const __nv_bfloat16*>(dZ), T, h, pl.chunks, cs_h, db, st));
        TPMLP_TRY((gemm_simt<__nv_bfloat16, EPI_DACT>(K_B2, s2, st)));
        TPMLP_TRY(colsum(K_B2_DA, static_cast<const __nv_bfloat16*>(dH), T, F, pl.chunks, cs_f, da, st));
        TPMLP_TRY((gemm_simt<__nv_bfloat16, EPI_F32>(K_B3, s3, st)));
        TPMLP_TRY((gemm_simt<__nv_bfloat16, EPI_F32>(K_B4, s4, st)));
        TPMLP_TRY((gemm_simt<__nv_bfloat16, EPI_BIAS>(K_B5, s5, st)));
    }
    return TPMLP_OK;
}

}  // namespace
}  // namespace tpmlp

using namespace tpmlp;

extern "C" {

size_t tpmlp_workspace_size(int64_t T, int64_t h, int64_t F, int p, tpmlp_dtype dt) {
    Plan pl;
    if (!make_plan(T, h, F, p, dt, &pl)) return 0;
    return pl.total;
}

tpmlp_status tp_mlp_fwd(const void* X, const void* A, const void* a, const void* B, const void* b,
                        void* H, void* Y, void* Z, int64_t T, int64_t h, int64_t F, int p,
                        tpmlp_dtype dt, void* workspace, size_t workspace_bytes, void* stream) {
    return fwd_impl<EPI_GELU>(X, A, a, B, b, H, Y, Z, T, h, F, p, dt, workspace, workspace_bytes,
                              stream);
}

tpmlp_status tp_mlp_fwd_ex(const void* X, const void* A, const void* a, const void* B,
                           const void* b, void* H, void* Y, void* Z, int64_t T, int64_t h,
                           int64_t F, int p, tpmlp_dtype dt, tpmlp_activation act, void* workspace,
                           size_t workspace_bytes, void* stream) {
    switch (act) {
        case TPMLP_GELU_ERF:
            return fwd_impl<EPI_GELU>(X, A, a, B, b, H, Y, Z, T, h, F, p, dt, workspace,
                                      workspace_bytes, stream);
        case TPMLP_GELU_TANH:
            return fwd_impl<EPI_GELU_TANH>(X, A, a, B, b, H, Y, Z, T, h, F, p, dt, workspace,
                                           workspace_bytes, stream);
    }
    return TPMLP_ERR_INVALID;
}

tpmlp_status tp_mlp_bwd(const void* dZ, const void* X, const void* A, const void* B, const void* H,
                        const void* Y, void* dX, float* dA, float* da, float* dB, float* db,
                        void* dH, int64_t T, int64_t h, int64_t F, int p, tpmlp_dtype dt,
                        void* workspace, size_t workspace_bytes, void* stream) {
    return bwd_impl<EPI_DGELU>(dZ, X, A, B, H, Y, dX, dA, da, dB, db, dH, T, h, F, p, dt, workspace,
                               workspace_bytes, stream);
}

tpmlp_status tp_mlp_bwd_ex(const void* dZ, const void* X, const void* A, const void* B,
                           const void* H, const void* Y, void* dX, float* dA, float* da, float* dB,
                           float* db, void* dH, int64_t T, int64_t h, int64_t F, int p,
                           tpmlp_dtype dt, tpmlp_activation act, void* workspace,
                           size_t workspace_bytes, void* stream) {
    switch (act) {
        case TPMLP_GELU_ERF:
            return bwd_impl<EPI_DGELU>(dZ, X, A, B, H, Y, dX, dA, da, dB, db, dH, T, h, F, p, dt,
                                       workspace, workspace_bytes, stream);
        case TPMLP_GELU_TANH:
            return bwd_impl<EPI_DGELU_TANH>(dZ, X, A, B, H, Y, dX, dA, da, dB, db, dH, T, h, F, p,
                                            dt, workspace, workspace_bytes, stream);
    }
    return TPMLP_ERR_INVALID;
}

size_t tpmlp_linear_workspace_size(int64_t T, int64_t K, int64_t N, int p, tpmlp_split split,
                                   tpmlp_dtype dt) {
    LinPlan pl;
    if (!make_lin_plan(T, K, N, p, static_cast<int>(split), dt, &pl)) return 0;
    return pl.total;
}

tpmlp_status tp_linear_fwd(const void* X, const void* W, const void* bias, void* Y, int64_t T,
                           int64_t K, int64_t N, int p, tpmlp_split split, tpmlp_dtype dt,
                           void* workspace, size_t workspace_bytes, void* stream) {
    cudaGetLastError();
    return linear_fwd_impl(X, W, bias, Y, T, K, N, p, static_cast<int>(split), dt, workspace,
                           workspace_bytes, static_cast<cudaStream_t>(stream));
}

tpmlp_status tp_linear_bwd(const void* dY, const void* X, const void* W, void* dX, float* dW,
                           float* dbias, int64_t T, int64_t K, int64_t N, int p, tpmlp_split split,
                           tpmlp_dtype dt, void* workspace, size_t workspace_bytes, void* stream) {
    cudaGetLastError();
    return linear_bwd_impl(dY, X, W, dX, dW, dbias, T, K, N, p, static_cast<int>(split), dt,
                           workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

tpmlp_status tp_mlp_recompute_hidden(const void* X, const void* A, const void* a, void* H, void* Y,
                                     int64_t T, int64_t h, int64_t F, int p, tpmlp_dtype dt,
                                     tpmlp_activation act, void* stream) {
    switch (act) {
        case TPMLP_GELU_ERF:
            return fwd_impl<EPI_GELU>(X, A, a, nullptr, nullptr, H, Y, nullptr, T, h, F, p, dt,
                                      nullptr, 0, stream, false);
        case TPMLP_GELU_TANH:
            return fwd_impl<EPI_GELU_TANH>(X, A, a, nullptr, nullptr, H, Y, nullptr, T, h, F, p,
                                           dt, nullptr, 0, stream, false);
    }
    return TPMLP_ERR_INVALID;
}

tpmlp_status tp_mlp_recompute_activation(const void* H, void* Y, int64_t n, tpmlp_dtype dt,
                                         tpmlp_activation act, void* stream) {
    cudaGetLastError();
    if (n < 0 || (dt != TPMLP_BF16 && dt != TPMLP_FP32)) return TPMLP_ERR_INVALID;
    if (act != TPMLP_GELU_ERF && act != TPMLP_GELU_TANH) return TPMLP_ERR_INVALID;
    if (n == 0) return TPMLP_OK;
    if (!H || !Y) return TPMLP_ERR_INVALID;
    const DeviceInfo* d = device_info();
    if (d == nullptr) return TPMLP_ERR_CUDA;
    if (d->cc_major != 10) return TPMLP_ERR_UNSUPPORTED;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t esize = dt == TPMLP_BF16 ? 2 : 4;
    const bool vec = (n % 8 == 0) && aligned16(H) && aligned16(Y);
    const bool tanh_form = (act == TPMLP_GELU_TANH);
    return timed(K_RECOMP, 0.0, 2.0 * esize * static_cast<double>(n), st, [&] {
        using B = __nv_bfloat16;
        if (dt == TPMLP_BF16) {
            if (vec)
                return tanh_form ? launch_recompute<B, true, true>(H, Y, n, st)
                                 : launch_recompute<B, false, true>(H, Y, n, st);
            return tanh_form ? launch_recompute<B, true, false>(H, Y, n, st)
                             : launch_recompute<B, false, false>(H, Y, n, st);
        }
        if (vec)
            return tanh_form ? launch_recompute<float, true, true>(H, Y, n, st)
                             : launch_recompute<float, false, true>(H, Y, n, st);
        return tanh_form ? launch_recompute<float, true, false>(H, Y, n, st)
                         : launch_recompute<float, false, false>(H, Y, n, st);
    });
}

const char* tpmlp_strerror(tpmlp_status s) {
    switch (s) {
        case TPMLP_OK: return "ok";
        case TPMLP_ERR_INVALID: return "invalid argument (size, p, null pointer or dtype)";
        case TPMLP_ERR_ALIGN: return "pointer not 16-byte aligned";
        case TPMLP_ERR_UNSUPPORTED: return "unsupported device or size";
        case TPMLP_ERR_WORKSPACE: return "workspace missing or too small";
        case TPMLP_ERR_CUDA: return "CUDA runtime or launch error";
        case TPMLP_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    }
    return "unknown status";
}

tpmlp_status tpmlp_last_device_status(void* stream) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TPMLP_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return TPMLP_ERR_CUDA;
    if (v != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess)
        return TPMLP_ERR_CUDA;
    return v == 0 ? TPMLP_OK : static_cast<tpmlp_status>(v);
}

tpmlp_status tpmlp_set_split_policy(int policy) {
    if (policy < 0 || policy > 3) return TPMLP_ERR_INVALID;
    g_split_policy.store(policy);
    return TPMLP_OK;
}

int tpmlp_get_split_policy(void) { return g_split_policy.load(); }

void tpmlp_set_launch_overlap(int on) { g_overlap.store(on != 0); }

void tpmlp_set_dynamic_schedule(int on) { g_dynamic.store(on != 0); }

int tpmlp_get_dynamic_schedule(void) { return g_dynamic.load() ? 1 : 0; }

int tpmlp_get_launch_overlap(void) { return g_overlap.load() ? 1 : 0; }

void tpmlp_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns == 0 ? kDefaultWaitLimitNs : ns); }

tpmlp_status tpmlp_wait_selftest(uint64_t limit_ns, void* stream) {
    cudaGetLastError();
    wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
    return check_launch();
}

uint64_t tpmlp_launch_count(void) { return g_launches.load(); }

tpmlp_status tpmlp_eval_activation(const float* x, float* y, float* dy, int64_t n, int form,
                                   void* stream) {
    cudaGetLastError();
    if (n < 0 || form < 0 || form > 3) return TPMLP_ERR_INVALID;
    if (n == 0) return TPMLP_OK;
    if (!x || !y || !dy) return TPMLP_ERR_INVALID;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 4096) blocks = 4096;
    eval_activation_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        x, y, dy, n, form);
    return check_launch();
}

void tpmlp_profile_enable(int on) { g_prof_on.store(on != 0); }

int tpmlp_profile_collect(void) {
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    int rc = K_COUNT;
    for (const PendingRec& r : g_pending) {
        float ms = 0.0f;
        if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
            rc = -1;
        } else {
            KindTotals& t = g_prof[r.kind];
            t.launches += 1;
            t.ms += ms;
            t.flops += r.flops;
            t.bytes += r.bytes;
        }
        g_event_pool.push_back(r.a);
        g_event_pool.push_back(r.b);
    }
    g_pending.clear();
    return rc;
}

int tpmlp_profile_kinds(void) { return K_COUNT; }

const char* tpmlp_profile_name(int kind) {
    return (kind >= 0 && kind < K_COUNT) ? kKindNames[kind] : "unknown";
}

tpmlp_status tpmlp_profile_read(int kind, uint64_t* launches, double* total_ms, double* flops,
                                double* bytes) {
    if (kind < 0 || kind >= K_COUNT) return TPMLP_ERR_INVALID;
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    const KindTotals& t = g_prof[kind];
    if (launches) *launches = t.launches;
    if (total_ms) *total_ms = t.ms;
    if (flops) *flops = t.flops;
    if (bytes) *bytes = t.bytes;
    return TPMLP_OK;
}

void tpmlp_profile_reset(void) {
    std::lock_guard<std::mutex> lock(g_prof_mutex);
    for (KindTotals& t : g_prof) t = KindTotals{};
}

int64_t tpmlp_schedule_units(int sched, int m_blocks, int n_blocks, int k_blocks, int groups,
                             int workers, int64_t* out, int64_t max_units) {
    if (m_blocks < 1 || n_blocks < 1 || k_blocks < 1 || workers < 1 || max_units < 0) return -1;
    if (max_units > 0 && out == nullptr) return -1;
    GemmArgs g{};
    g.num_m_blocks = m_blocks;
    g.num_n_blocks = n_blocks;
    g.k_blocks = k_blocks;
    g.groups = 1;
    g.kb_per_group = k_blocks;
    const int64_t tiles = static_cast<int64_t>(m_blocks) * n_blocks;
    if (tiles > (int64_t(1) << 30)) return -1;
    if (sched == SCHED_TILES) {
        g.sched = SCHED_TILES;
    } else if (sched == SCHED_GROUPS) {
        if (groups < 2 || k_blocks % groups != 0) return -1;
        g.sched = SCHED_GROUPS;
        g.groups = groups;
        g.kb_per_group = k_blocks / groups;
    } else if (sched == SCHED_STREAMK) {
        if (!streamk_pays(tiles, k_blocks, workers, true)) return -1;
        g.sched = SCHED_STREAMK;
    } else {
        return -1;
    }
    int64_t n = 0;
    for (int wk = 0; wk < workers; ++wk) {
        WorkIter it = work_iter(wk, workers);
        WorkUnit w;
        for (int local = 0; next_unit(g, it, w); ++local, ++n) {
            if (n >= max_units) continue;
            int64_t* r = out + 10 * n;
            r[0] = wk;
            r[1] = local;
            r[2] = w.mb;
            r[3] = w.nb;
            r[4] = w.kb0;
            r[5] = w.kb1;
            r[6] = w.pieces;
            r[7] = w.piece;
            r[8] = w.pieces > 1 ? w.key : -1;
            r[9] = w.pieces > 1 ? partial_slot(g, w, w.piece, workers) : -1;
        }
    }
    return n;
}

tpmlp_status tpmlp_plan_schedules(int64_t T, int64_t h, int64_t F, int p, tpmlp_dtype dt, int* kinds) {
    Plan pl;
    if (kinds == nullptr || !make_plan(T, h, F, p, dt, &pl)) return TPMLP_ERR_INVALID;
    const SchedReq* r[6] = {&pl.f1, &pl.f2, &pl.b2, &pl.b3, &pl.b4, &pl.b5};
    for (int i = 0; i < 6; ++i) kinds[i] = r[i]->kind;
    return TPMLP_OK;
}

tpmlp_status tpmlp_plan_dynamic(int64_t T, int64_t h, int64_t F, int p, tpmlp_dtype dt, int* dyn) {
    Plan pl;
    if (dyn == nullptr || !make_plan(T, h, F, p, dt, &pl)) return TPMLP_ERR_INVALID;
    const SchedReq* r[6] = {&pl.f1, &pl.f2, &pl.b2, &pl.b3, &pl.b4, &pl.b5};
    for (int i = 0; i < 6; ++i) dyn[i] = r[i]->dyn ? 1 : 0;
    return TPMLP_OK;
}

int tpmlp_version(void) { return 200; }

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward without any caller-provided memory beyond inputs and outputs.
//
// Some callers cannot allocate device memory when they call the backward:
// a plugin running inside another framework that owns every device
// allocation and gives its extensions no allocator, or a runtime with a
// fixed memory budget that forbids allocation after start-up (cudaMalloc
// and cudaFree may also synchronize the device, which such callers avoid).
// tp_mlp_bwd_noalloc serves them: its only scratch, the partial column sums
// of the two bias gradients, lives in a fixed array compiled into this
// library, and it always uses the unsplit schedule for dX (each output tile
// loops over the shards in ascending order in tensor memory), which needs
// no scratch.
namespace tpmlp {
namespace {

// 8 MiB, resident on every GPU that loads this library until the process
// exits. The column-sum partials of a call need
// 4·ceil(T/128)·h + 4·ceil(T/128)·F bytes (each part rounded up to 256).
constexpr size_t kNoallocScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// Device address of g_noalloc_scratch, per device. In host code the
// array's name is only a host-side stand-in, so the address is looked up
// with cudaGetSymbolAddress, once per device, with that device current.
void* g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mutex;

tpmlp_status noalloc_scratch_ptr(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TPMLP_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
            return TPMLP_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return TPMLP_OK;
}

}  // namespace
}  // namespace tpmlp

extern "C" {

size_t tpmlp_noalloc_scratch_bytes(void) { return kNoallocScratchBytes; }

tpmlp_status tp_mlp_bwd_noalloc(const void* dZ, const void* X, const void* A, const void* B,
                                const void* H, const void* Y, void* dX, float* dA, float* da,
                                float* dB, float* db, void* dH, int64_t T, int64_t h, int64_t F,
                                int p, tpmlp_dtype dt, void* stream) {
    cudaGetLastError();
    Plan pl;
    if (!make_plan(T, h, F, p, dt, &pl)) return TPMLP_ERR_INVALID;
    if (T >= (int64_t(1) << 31) || h >= (int64_t(1) << 31) || F >= (int64_t(1) << 31))
        return TPMLP_ERR_UNSUPPORTED;
    const DeviceInfo* d = device_info();
    if (d == nullptr) return TPMLP_ERR_CUDA;
    if (d->cc_major != 10) return TPMLP_ERR_UNSUPPORTED;
    const size_t cs_h_bytes = round256(static_cast<size_t>(pl.chunks) * h * sizeof(float));
    const size_t cs_f_bytes = round256(static_cast<size_t>(pl.chunks) * F * sizeof(float));
    if (cs_h_bytes + cs_f_bytes > kNoallocScratchBytes) return TPMLP_ERR_WORKSPACE;
    if (!dA || !da || !dB || !db) return TPMLP_ERR_INVALID;
    if (T > 0 && (!dZ || !X || !A || !B || !H || !Y || !dX || !dH)) return TPMLP_ERR_INVALID;
    if (pl.tc && T > 0) {
        for (const void* q : {dZ, X, A, B, H, Y, static_cast<const void*>(dX),
                              static_cast<const void*>(dA), static_cast<const void*>(da),
                              static_cast<const void*>(dB), static_cast<const void*>(db),
                              static_cast<const void*>(dH)})
            if (!aligned16(q)) return TPMLP_ERR_ALIGN;
    }
    void* scratch = nullptr;
    TPMLP_TRY(noalloc_scratch_ptr(&scratch));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        TPMLP_TRY(zero_f32(dA, h * F, st));
        TPMLP_TRY(zero_f32(da, F, st));
        TPMLP_TRY(zero_f32(dB, F * h, st));
        TPMLP_TRY(zero_f32(db, h, st));
        return TPMLP_OK;
    }
    // Every partial the column sums use is written before it is read, so
    // nothing in the scratch has to start at zero. Every product runs as
    // whole tiles (no partial tiles, no counters).
    float* cs_h = static_cast<float*>(scratch);
    float* cs_f = reinterpret_cast<float*>(static_cast<char*>(scratch) + cs_h_bytes);
    const int iT = static_cast<int>(T), ih = static_cast<int>(h), iF = static_cast<int>(F);
    if (pl.tc) {
        TPMLP_TRY(colsum(K_B1_DB, static_cast<const __nv_bfloat16*>(dZ), T, h, pl.chunks, cs_h, db, st));
        GemmArgs g2{};
        g2.out0 = dH;
        g2.ld_out = F;
        g2.aux = static_cast<const __nv_bfloat16*>(H);
        TPMLP_TRY((gemm_tc<256, false, false, EPI_DGELU>(K_B2, dZ, B, iT, iF, ih, SchedReq{}, g2, st)));
        TPMLP_TRY(colsum(K_B2_DA, static_cast<const __nv_bfloat16*>(dH), T, F, pl.chunks, cs_f, da, st));
        GemmArgs g3{};
        g3.out0 = dB;
        g3.ld_out = h;
        TPMLP_TRY((gemm_tc<256, true, true, EPI_F32>(K_B3, Y, dZ, iF, ih, iT, SchedReq{}, g3, st)));
        GemmArgs g4{};
        g4.out0 = dA;
        g4.ld_out = F;
        TPMLP_TRY((gemm_tc<256, true, true, EPI_F32>(K_B4, X, dH, ih, iF, iT, SchedReq{}, g4, st)));
        GemmArgs g5{};
        g5.out0 = dX;
        g5.ld_out = h;
        TPMLP_TRY((gemm_tc<256, false, false, EPI_BIAS>(K_B5, dH, A, iT, ih, iF, SchedReq{}, g5, st)));
        return TPMLP_OK;
    }
    SimtArgs s2{};
    s2.M = iT; s2.N = iF; s2.K = ih;
    s2.A = dZ; s2.sam = h; s2.sak = 1;
    s2.B = B; s2.sbk = 1; s2.sbn = h;
    s2.out0 = dH; s2.ld_out = F; s2.aux = H;
    SimtArgs s3{};
    s3.M = iF; s3.N = ih; s3.K = iT;
    s3.A = Y; s3.sam = 1; s3.sak = F;
    s3.B = dZ; s3.sbk = h; s3.sbn = 1;
    s3.out0 = dB; s3.ld_out = h;
    SimtArgs s4{};
    s4.M = ih; s4.N = iF; s4.K = iT;
    s4.A = X; s4.sam = 1; s4.sak = h;
    s4.B = dH; s4.sbk = F; s4.sbn = 1;
    s4.out0 = dA; s4.ld_out = F;
    SimtArgs s5{};
    s5.M = iT; s5.N = ih; s5.K = iF;
    s5.A = dH; s5.sam = F; s5.sak = 1;
    s5.B = A; s5.sbk = 1; s5.sbn = F;
    s5.out0 = dX; s5.ld_out = h;
    if (dt == TPMLP_FP32) {
        TPMLP_TRY(colsum(K_B1_DB, static_cast<const float*>(dZ), T, h, pl.chunks, cs_h, db, st));
        TPMLP_TRY((gemm_simt<float, EPI_DGELU>(K_B2, s2, st)));
        TPMLP_TRY(colsum(K_B2_DA, static_cast<const float*>(dH), T, F, pl.chunks, cs_f, da, st));
        TPMLP_TRY((gemm_simt<float, EPI_F32>(K_B3, s3, st)));
        TPMLP_TRY((gemm_simt<float, EPI_F32>(K_B4, s4, st)));
        TPMLP_TRY((gemm_simt<float, EPI_BIAS>(K_B5, s5, st)));
    } else {
        TPMLP_TRY(colsum(K_B1_DB, static_cast<const __nv_bfloat16*>(dZ), T, h, pl.chunks, cs_h, db, st));
        TPMLP_TRY((gemm_simt<__nv_bfloat16, EPI_DGELU>(K_B2, s2, st)));
        TPMLP_TRY(colsum(K_B2_DA, static_cast<const __nv_bfloat16*>(dH), T, F, pl.chunks, cs_f, da, st));
        TPMLP_TRY((gemm_simt<__nv_bfloat16, EPI_F32>(K_B3, s3, st)));
        TPMLP_TRY((gemm_simt<__nv_bfloat16, EPI_F32>(K_B4, s4, st)));
        TPMLP_TRY((gemm_simt<__nv_bfloat16, EPI_BIAS>(K_B5, s5, st)));
    }
    return TPMLP_OK;
}

}  // extern "C"
