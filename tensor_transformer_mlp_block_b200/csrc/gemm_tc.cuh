// Persistent tcgen05 GEMM for sm_100a with fused epilogues.
//
//   D[M, N] = Σ_k Aop[m, k] · Bop[k, n]      (bf16 operands, fp32 accumulate)
//
// Operands are row-major tensors in global memory read by TMA in either
// orientation: Aop is "K-major" when stored as [M][K] and "MN-major" when
// stored as [K][M] (the transposed operand of a weight-gradient product);
// likewise Bop is K-major when stored as [N][K] and MN-major as [K][N]. The
// tensor cores read both orientations directly from 128-byte-swizzled shared
// memory, so no transposed copy is ever made.
//
// CTA organisation (320 threads, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: fills a STAGES-deep ring of (A, B) k-blocks
//   warp 1      tensor-memory allocator and MMA issuer (one thread)
//   warps 2..9  epilogue: tensor memory -> registers -> fused math -> global
// The accumulator is double-buffered in tensor memory (2 × BN fp32 columns
// of 128 lanes), so the epilogue of one tile overlaps the next tile's
// main loop. Work units follow one of three schedules (next_unit), which
// every role of a CTA walks in the same order:
//   whole tiles    unit u = tile u, handed out round-robin over the CTAs;
//   shard groups   every tile's K range cut into `groups` equal consecutive
//                  parts (the row-parallel products' shard groups);
//   stream-K tail  whole tiles in full waves, then the k-blocks of the
//                  remaining tiles cut into one equal segment per CTA (pair),
//                  so that the last wave has no idle SMs.
// A unit that covers only part of a tile's K range writes its fp32 partial
// to the workspace and arrives on the tile's counters; the last unit to
// arrive adds all partials of the tile in ascending k order and runs the
// epilogue. No unit waits for another, so the sum is the same whichever
// unit finishes last, and no CTA depends on another CTA being resident.
//
// Every wait is bounded (mbar_wait_bounded); a wait that runs out records
// a timeout in the device status word and the CTA winds down: the producer
// waits for its copies in flight, the MMA thread for its tensor-core work,
// and tensor memory is freed before the CTA exits.
#pragma once

#include "ptx.cuh"

namespace tpmlp {

enum EpiKind : int {
    EPI_GELU = 0,        // out0 = H = acc + bias (bf16), out1 = Y = GeLU(H) (bf16)
    EPI_BIAS = 1,        // out0 = acc + bias (element type); bias may be null
    EPI_DGELU = 2,       // out0 = dH = acc · GeLU′(aux) (bf16), aux = saved H (bf16)
    EPI_F32 = 3,         // out0 = acc (fp32)
    EPI_GELU_TANH = 4,   // as EPI_GELU with the tanh approximation of GeLU
    EPI_DGELU_TANH = 5,  // as EPI_DGELU with the tanh approximation's derivative
};

// Epilogue classes: activation forward (two outputs), activation backward
// (reads the saved pre-activation), and the tanh forms of both.
template <int EPI>
struct EpiTraits {
    static constexpr bool kAct = (EPI == EPI_GELU || EPI == EPI_GELU_TANH);
    static constexpr bool kDAct = (EPI == EPI_DGELU || EPI == EPI_DGELU_TANH);
    static constexpr bool kTanh = (EPI == EPI_GELU_TANH || EPI == EPI_DGELU_TANH);
    static constexpr bool kBias = (EPI == EPI_BIAS) || kAct;
};

// Work-unit schedules (see next_unit).
enum SchedKind : int {
    SCHED_TILES = 0,    // one unit per output tile
    SCHED_GROUPS = 1,   // every tile in `groups` consecutive k ranges
    SCHED_STREAMK = 2,  // whole tiles in full waves, then a stream-K tail
};

struct GemmArgs {
    int M, N, K;
    int num_m_blocks, num_n_blocks;
    int k_blocks;      // ceil(K / BK)
    int sched;         // SchedKind
    int groups;        // SCHED_GROUPS: k ranges per tile
    int kb_per_group;  // SCHED_GROUPS: k-blocks per range
    void* out0;
    void* out1;
    int64_t ld_out;        // row stride (elements) of out0, out1 and aux
    const __nv_bfloat16* bias;
    const __nv_bfloat16* aux;
    uint64_t wait_limit_ns;
    // GeLU′ epilogues with the relay: if set, column sums of the stored (bf16)
    // output go to colsum_out[r·N + col] (fp32), one row r per 64 rows a
    // computing warp handles in a 128-row CTA tile (see epilogue_role)
    float* colsum_out;
    // Tiles split over several units (SCHED_GROUPS, the stream-K tail):
    // fp32 partial tiles (partial_chunk) and 16 arrival counters per split
    // tile (one per CTA of the pair and epilogue warp), all zero at launch.
    // (colsum_out must be null: a split tile is finished warp by warp.)
    float* partials;
    int* counters;
    // Counters of a later launch on the same stream, zeroed by this one
    // (which must not split tiles itself): zero_count ints at zero_counters.
    int* zero_counters;
    int zero_count;
    // A second product in the same launch (CTA-pair kernel, whole tiles, same
    // K and fp32 epilogue; operands in tmA2 / tmB2, output in tmO1): its
    // M2 × N2 tiles follow the first product's. second = 0: none.
    int second;
    int M2, N2, num_m_blocks2, num_n_blocks2;
    // Dynamic schedule (CTA-pair kernel; null: static round-robin). Work
    // items are taken in order from dyn_counter[0] by each pair's leader
    // producer and handed to the pair's other roles through a shared-memory
    // queue; the last pair to finish puts dyn_counter[0..1] back to zero.
    // Both must be zero at launch.
    int* dyn_counter;
};

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kEpiWarps = 8;  // two per SM sub-partition, each half of the columns
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kGroupM = 16;  // m-blocks per raster group (L2 reuse of Bop)
// Shared-memory staging for the epilogue's bulk stores: one 4 KB slot per
// epilogue warp (a 32 × 32 fp32 chunk, or two 32 × 32 bf16 chunks).
constexpr int kEpiSlotBytes = 4096;
constexpr int kEpiStagingBytes = kEpiWarps * kEpiSlotBytes;

template <int BN>
struct TileCfg {
    static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "BN must be 64..256, multiple of 64");
    static constexpr int A_BYTES = kBM * kBK * 2;  // 16 KB
    static constexpr int B_BYTES = BN * kBK * 2;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
    static constexpr int STAGES = (196608 / STAGE_BYTES) > 8 ? 8 : (196608 / STAGE_BYTES);
    // tensor-memory columns: two accumulators, rounded up to a power of two
    static constexpr int TMEM_COLS = (2 * BN <= 128) ? 128 : (2 * BN <= 256 ? 256 : 512);
    static constexpr int BAR_BYTES = 8 * (2 * STAGES + 5 + 8) + 16;
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + kEpiStagingBytes + BAR_BYTES;
};

// The work schedule below is plain integer arithmetic, compiled for the host
// too so that the library can list the units it would run (a diagnostic).
#define TPMLP_HD __host__ __device__ __forceinline__

// Output tile t in grouped raster order: kGroupM m-blocks per group,
// m fastest inside a group, so that neighbouring units share Bop panels.
TPMLP_HD void tile_coords_of(int num_m_blocks, int num_n_blocks, int t, int& mb, int& nb) {
    const int per_group = kGroupM * num_n_blocks;
    const int group = t / per_group;
    const int first_m = group * kGroupM;
    const int rem_m = num_m_blocks - first_m;
    const int gm = rem_m < kGroupM ? rem_m : kGroupM;
    const int idx = t - group * per_group;
    mb = first_m + idx % gm;
    nb = idx / gm;
}

TPMLP_HD void tile_coords(const GemmArgs& g, int t, int& mb, int& nb) {
    tile_coords_of(g.num_m_blocks, g.num_n_blocks, t, mb, nb);
}

struct WorkUnit {
    int prob;      // 0, or 1 for the second product of a grouped launch
    int mb, nb;    // output tile
    int kb0, kb1;  // k-blocks [kb0, kb1) of this unit
    int pieces;    // units sharing the tile (1: the whole K range)
    int piece;     // this unit's place among them, in ascending k
    int key;       // split tiles: index of the tile's counters
    int seg_lo;    // stream-K tail: first segment covering the tile
};

// Position of one worker (a CTA pair, or a CTA of the one-CTA kernel) in
// its sequence of units.
struct WorkIter {
    int worker, nworkers;
    int next;       // whole-tile / group units taken so far
    bool tail;      // in the stream-K segment
    int64_t cur, end;
};

TPMLP_HD WorkIter work_iter(int worker, int nworkers) {
    WorkIter it;
    it.worker = worker;
    it.nworkers = nworkers;
    it.next = 0;
    it.tail = false;
    it.cur = it.end = 0;
    return it;
}

// Stream-K tail: W k-blocks of the tail tiles (tile-major, k fastest) are cut
// into P segments; segment j is [begin(j), begin(j + 1)). With W ≥ P no
// segment is empty. seg_of(x) is the segment that holds k-block x.
TPMLP_HD int64_t sk_begin(int64_t j, int64_t W, int P) { return j * W / P; }
TPMLP_HD int sk_seg_of(int64_t x, int64_t W, int P) {
    return static_cast<int>(((x + 1) * P - 1) / W);
}
TPMLP_HD int sk_whole_tiles(const GemmArgs& g, int P) {
    const int tiles = g.num_m_blocks * g.num_n_blocks;
    return (tiles / P) * P;
}
TPMLP_HD int64_t sk_work(const GemmArgs& g, int P) {
    const int tiles = g.num_m_blocks * g.num_n_blocks;
    return static_cast<int64_t>(tiles - sk_whole_tiles(g, P)) * g.k_blocks;
}

// The next unit of this worker; false when it has none left.
TPMLP_HD bool next_unit(const GemmArgs& g, WorkIter& it, WorkUnit& w) {
    const int tiles = g.num_m_blocks * g.num_n_blocks;
    if (g.sched == SCHED_GROUPS) {
        const int u = it.worker + it.next * it.nworkers;
        if (u >= tiles * g.groups) return false;
        ++it.next;
        const int s = u / tiles;
        const int t = u - s * tiles;
        tile_coords(g, t, w.mb, w.nb);
        w.prob = 0;
        w.kb0 = s * g.kb_per_group;
        w.kb1 = w.kb0 + g.kb_per_group < g.k_blocks ? w.kb0 + g.kb_per_group : g.k_blocks;
        w.pieces = g.groups;
        w.piece = s;
        w.key = t;
        w.seg_lo = 0;
        return true;
    }
    const int whole = g.sched == SCHED_STREAMK ? sk_whole_tiles(g, it.nworkers) : tiles;
    if (!it.tail) {
        const int u = it.worker + it.next * it.nworkers;
        const int tiles2 = (g.second && g.sched == SCHED_TILES) ? g.num_m_blocks2 * g.num_n_blocks2 : 0;
        if (u < whole + tiles2) {
            ++it.next;
            w.prob = u < whole ? 0 : 1;
            if (w.prob == 0)
                tile_coords(g, u, w.mb, w.nb);
            else
                tile_coords_of(g.num_m_blocks2, g.num_n_blocks2, u - whole, w.mb, w.nb);
            w.kb0 = 0;
            w.kb1 = g.k_blocks;
            w.pieces = 1;
            w.piece = 0;
            w.key = 0;
            w.seg_lo = 0;
            return true;
        }
        if (g.sched != SCHED_STREAMK) return false;
        it.tail = true;
        const int64_t W = sk_work(g, it.nworkers);
        it.cur = sk_begin(it.worker, W, it.nworkers);
        it.end = sk_begin(it.worker + 1, W, it.nworkers);
    }
    if (it.cur >= it.end) return false;
    const int64_t W = sk_work(g, it.nworkers);
    const int kb = g.k_blocks;
    const int st = static_cast<int>(it.cur / kb);  // tail tile
    const int64_t first = static_cast<int64_t>(st) * kb;
    w.kb0 = static_cast<int>(it.cur - first);
    const int64_t room = w.kb0 + (it.end - it.cur);
    w.kb1 = static_cast<int>(room < kb ? room : kb);
    tile_coords(g, whole + st, w.mb, w.nb);
    w.prob = 0;
    w.seg_lo = sk_seg_of(first, W, it.nworkers);
    w.pieces = sk_seg_of(first + kb - 1, W, it.nworkers) - w.seg_lo + 1;
    w.piece = it.worker - w.seg_lo;
    w.key = st;
    it.cur += w.kb1 - w.kb0;
    return true;
}

// ------------------------------------------------- dynamic schedule (pairs)
// A tile costs the same on every SM, but the SMs do not run at the same
// speed (measured: the slowest CTA pairs take ~5% longer per tile, the same
// pairs in every product). With a static round-robin the product ends with
// its slowest pair; with items taken in order from a global counter, fast
// pairs take more of them. Items are the schedule's units (whole tiles, shard
// group units) or, for the stream-K tail, whole tiles and then one item per
// segment, which expands into the segment's pieces in every role the same
// way. Results do not depend on which pair runs an item.

constexpr int kQueue = 8;  // item slots of a pair's queue

TPMLP_HD int dyn_items(const GemmArgs& g, int P) {
    const int tiles = g.num_m_blocks * g.num_n_blocks;
    if (g.sched == SCHED_GROUPS) return tiles * g.groups;
    if (g.sched == SCHED_STREAMK) return sk_whole_tiles(g, P) + (sk_work(g, P) > 0 ? P : 0);
    return tiles + (g.second ? g.num_m_blocks2 * g.num_n_blocks2 : 0);
}

// The first unit of item `id`. For a stream-K segment, `it` yields its other
// pieces afterwards (seg = true); any other item is a single unit.
TPMLP_HD bool dyn_item_first(const GemmArgs& g, int P, int id, WorkIter& it, bool& seg, WorkUnit& w) {
    seg = false;
    if (g.sched == SCHED_STREAMK && id >= sk_whole_tiles(g, P)) {
        const int j = id - sk_whole_tiles(g, P);  // the segment, as the static schedule's worker j
        it = work_iter(j, P);
        it.tail = true;
        const int64_t W = sk_work(g, P);
        it.cur = sk_begin(j, W, P);
        it.end = sk_begin(j + 1, W, P);
        seg = true;
        return next_unit(g, it, w);
    }
    it = work_iter(id, P);  // the static schedule's unit number `id`
    return next_unit(g, it, w);
}

// This CTA's view of its pair's item queue.
struct PairQueue {
    uint32_t items;  // shared address of kQueue item ids (this CTA's copy)
    uint32_t full;   // kQueue barriers of this CTA: slot s holds an item
    uint32_t empty;  // kQueue barriers of the leader: every role has read slot s
    bool leader;     // this CTA is the pair's leader
};

// A consumer role (the leader's MMA thread and epilogue warps, the other
// CTA's producer and epilogue warps) takes the id in slot n mod kQueue.
// WARP: all lanes wait and read; lane 0 arrives. False: a wait gave up.
template <bool WARP>
__device__ __forceinline__ bool queue_take(const PairQueue& q, int n, int& id, volatile int* abort,
                                           uint64_t limit) {
    const int s = n % kQueue;
    const uint32_t par = static_cast<uint32_t>(n / kQueue) & 1u;
    // the other CTA's copy arrives with a release at cluster scope
    bool got = mbar_wait_bounded_cluster(q.full + 8 * s, par, abort, limit);
    if (WARP) got = __all_sync(0xffffffffu, got);
    if (!got) return false;
    id = static_cast<int>(ld_shared_u32(q.items + 4 * s));
    if (!WARP || (threadIdx.x & 31) == 0) {
        const uint32_t e = q.empty + 8 * s;
        if (q.leader)
            mbar_arrive(e);
        else
            mbar_arrive_cluster(mapa_shared(e, 0));
    }
    if (WARP) __syncwarp();
    return true;
}

// The leader's producer puts item `id` (-1: past the end) into slot
// n mod kQueue of both CTAs' queues, once every role has read the slot's
// previous item.
__device__ __forceinline__ bool queue_publish(const PairQueue& q, int n, int id, volatile int* abort,
                                              uint64_t limit) {
    const int s = n % kQueue;
    const uint32_t par = static_cast<uint32_t>(n / kQueue) & 1u;
    if (!mbar_wait_bounded_cluster(q.empty + 8 * s, par ^ 1u, abort, limit)) return false;
    const uint32_t slot = q.items + 4 * s;
    asm volatile("st.volatile.shared.u32 [%0], %1;" ::"r"(slot), "r"(id) : "memory");
    st_shared_cluster_u32(mapa_shared(slot, 1), static_cast<uint32_t>(id));
    mbar_arrive(q.full + 8 * s);
    mbar_arrive_cluster(mapa_shared(q.full + 8 * s, 1));
    return true;
}

// Where a role's units come from: the static sequence of its worker, or
// the items of the pair's queue (dynamic schedule).
struct UnitCursor {
    WorkIter it;   // static: the worker's sequence; dynamic: the current segment's pieces
    bool dyn;
    bool seg;      // dynamic: `it` may have pieces of the current item left
    int n;         // dynamic: items taken (consumers) or published (leader's producer)
    // leader's producer: the item published one ahead of the one it loads,
    // and the counter value drawn for the item after that (still in flight)
    int ahead, pend;
    bool started;
};

__device__ __forceinline__ UnitCursor unit_cursor(int worker, int nworkers, bool dyn) {
    UnitCursor c;
    c.it = work_iter(worker, nworkers);
    c.dyn = dyn;
    c.seg = false;
    c.n = 0;
    c.ahead = -1;
    c.pend = -1;
    c.started = false;
    return c;
}

// The leader's producer: the next item to load. Items are published one
// ahead of the one being loaded, and the counter draw for the item after
// that is issued right away and used one item later, so the atomic's latency
// hides behind the current item's loads (a tile's loads never wait for it).
__device__ __forceinline__ bool give_next_item(const GemmArgs& g, int items, UnitCursor& c, int& id,
                                               const PairQueue& q, volatile int* abort,
                                               uint64_t limit) {
    if (!c.started) {
        c.started = true;
        int first = atomicAdd(g.dyn_counter, 1);
        if (first >= items) first = -1;
        if (!queue_publish(q, c.n++, first, abort, limit)) return false;
        c.ahead = first;
        c.pend = first >= 0 ? atomicAdd(g.dyn_counter, 1) : -1;
    }
    id = c.ahead;
    if (id < 0) return true;
    int next = c.pend;
    if (next >= items) next = -1;
    if (!queue_publish(q, c.n++, next, abort, limit)) return false;
    c.ahead = next;
    c.pend = next >= 0 ? atomicAdd(g.dyn_counter, 1) : -1;
    return true;
}

// The whole tile numbered u of a whole-tile schedule (the second product's
// tiles follow the first's).
__device__ __forceinline__ void whole_tile_unit(const GemmArgs& g, int u, WorkUnit& w) {
    const int tiles = g.num_m_blocks * g.num_n_blocks;
    w.prob = u < tiles ? 0 : 1;
    if (w.prob == 0)
        tile_coords(g, u, w.mb, w.nb);
    else
        tile_coords_of(g.num_m_blocks2, g.num_n_blocks2, u - tiles, w.mb, w.nb);
    w.kb0 = 0;
    w.kb1 = g.k_blocks;
    w.pieces = 1;
    w.piece = 0;
    w.key = 0;
    w.seg_lo = 0;
}

// The next unit of a role; false at the end, or (ok = false) when a wait gave
// up. GIVE: the leader's producer, which draws the items. TILES_ONLY: the
// kernel runs whole-tile schedules only (fewer registers live).
template <bool GIVE, bool WARP, bool TILES_ONLY = false>
__device__ __forceinline__ bool cursor_next(const GemmArgs& g, int P, UnitCursor& c, WorkUnit& w,
                                            const PairQueue* q, bool& ok, volatile int* abort,
                                            uint64_t limit) {
    if constexpr (TILES_ONLY) {
        int u;
        if (!c.dyn) {
            u = c.it.worker + c.it.next * c.it.nworkers;
            ++c.it.next;
            const int all = g.num_m_blocks * g.num_n_blocks +
                            (g.second ? g.num_m_blocks2 * g.num_n_blocks2 : 0);
            if (u >= all) return false;
        } else {
            const bool got = GIVE ? give_next_item(g, dyn_items(g, P), c, u, *q, abort, limit)
                                  : queue_take<WARP>(*q, c.n, u, abort, limit);
            if (!got) {
                ok = false;
                return false;
            }
            if (!GIVE) ++c.n;
            if (u < 0) return false;
        }
        whole_tile_unit(g, u, w);
        return true;
    }
    if (!c.dyn) return next_unit(g, c.it, w);
    for (;;) {
        if (c.seg) {
            if (next_unit(g, c.it, w)) return true;
            c.seg = false;
        }
        int id = -1;
        const bool got = GIVE ? give_next_item(g, dyn_items(g, P), c, id, *q, abort, limit)
                              : queue_take<WARP>(*q, c.n, id, abort, limit);
        if (!got) {
            ok = false;
            return false;
        }
        if (!GIVE) ++c.n;
        if (id < 0) return false;
        bool seg = false;
        if (dyn_item_first(g, P, id, c.it, seg, w)) {
            c.seg = seg;
            return true;
        }
    }
}

// Workspace slot (one partial tile) of piece q of a split tile. Shard groups:
// one slot per (tile, group). Stream-K tail: two per segment, 2j for the
// piece that starts where segment j starts, 2j + 1 for the piece that starts
// at a tile boundary inside it (a segment has at most these two partial
// pieces; the tiles wholly inside it need no partial).
TPMLP_HD int64_t partial_slot(const GemmArgs& g, const WorkUnit& w, int q,
                                                int nworkers) {
    if (g.sched == SCHED_GROUPS) return static_cast<int64_t>(w.key) * g.groups + q;
    const int j = w.seg_lo + q;
    const int64_t begin = sk_begin(j, sk_work(g, nworkers), nworkers);
    return 2 * static_cast<int64_t>(j) + (begin >= static_cast<int64_t>(w.key) * g.k_blocks ? 0 : 1);
}

// The 32 × 32 fp32 chunk of a partial tile at tile rows r0.., columns c0..
// (r0, c0 multiples of 32; a pair tile counts rows over both CTAs): 1024
// floats in the order the epilogue's registers hold them, float4 j of lane
// l (row l, columns 4j..4j+3) at index 4·(32·j + l), so that a warp's
// accesses of one j are 512 contiguous bytes.
__device__ __forceinline__ float* partial_chunk(const GemmArgs& g, int64_t slot, int tile_rows,
                                                int bn, int r0, int c0) {
    return g.partials + slot * static_cast<int64_t>(tile_rows) * bn +
           static_cast<int64_t>((r0 / 32) * (bn / 32) + c0 / 32) * 1024;
}

__device__ __forceinline__ void partial_store(float* chunk, const uint32_t (&acc)[32], int lane) {
    float4* p = reinterpret_cast<float4*>(chunk);
#pragma unroll
    for (int j = 0; j < 8; ++j)
        __stcg(p + 32 * j + lane, make_float4(__uint_as_float(acc[4 * j]), __uint_as_float(acc[4 * j + 1]),
                                              __uint_as_float(acc[4 * j + 2]),
                                              __uint_as_float(acc[4 * j + 3])));
}

// acc = Σ_{q = 0 .. pieces-1} partial q, added in ascending q (ascending k).
// The partials sit in L2, written by other SMs (one round trip per piece, its
// 8 loads per lane in flight together). Piece own_q (if ≥ 0) is this unit's
// own, still in tensor memory at t_chunk: it is read from there at its place
// in the order, so the sum is the same as from memory.
__device__ __forceinline__ void partial_sum(const GemmArgs& g, const WorkUnit& w, int nworkers,
                                            int tile_rows, int bn, int r0, int c0,
                                            uint32_t (&acc)[32], int lane, int own_q,
                                            uint32_t t_chunk) {
#pragma unroll 1
    for (int q = 0; q < w.pieces; ++q) {
        uint32_t x[32];
        if (q == own_q) {
            tmem_ld_32x32b_x32(t_chunk, x);
            tmem_wait_ld();
        } else {
            const uint4* p = reinterpret_cast<const uint4*>(
                partial_chunk(g, partial_slot(g, w, q, nworkers), tile_rows, bn, r0, c0));
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint4 v = __ldcg(p + 32 * j + lane);
                x[4 * j] = v.x;
                x[4 * j + 1] = v.y;
                x[4 * j + 2] = v.z;
                x[4 * j + 3] = v.w;
            }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i)
            acc[i] = q == 0 ? x[i] : __float_as_uint(__uint_as_float(acc[i]) + __uint_as_float(x[i]));
    }
}

__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Arrival of one epilogue warp on its counter of a split tile, after
// writing its partial chunks. Returns true (in every lane) for the warp of
// the last unit to arrive, which then reads every partial of the tile; it
// also puts the counter back to zero for the next launch.
__device__ __forceinline__ bool partial_arrive(int* ctr, int pieces, int lane) {
    __threadfence();  // this lane's partial stores are visible device-wide
    __syncwarp();
    int old = 0;
    if (lane == 0) {
        old = atomicAdd(ctr, 1);
        __threadfence();  // later loads of the other units' partials see them
    }
    old = __shfl_sync(0xffffffffu, old, 0);
    const bool last = (old == pieces - 1);
    if (last && lane == 0) atomicExch(ctr, 0);
    __syncwarp();
    return last;
}

// GeLU and its derivative through CUDA's erff/expf (the plain path).
__device__ __forceinline__ float gelu_f32(float x) {
    return 0.5f * x * (1.0f + erff(x * 0.70710678118654752f));
}

__device__ __forceinline__ float gelu_grad_f32(float x) {
    const float cdf = 0.5f * (1.0f + erff(x * 0.70710678118654752f));
    const float pdf = 0.39894228040143268f * expf(-0.5f * x * x);
    return cdf + x * pdf;
}

// Two fp32 values in one 64-bit register: sm_100's fma.rn.f32x2 and
// mul.rn.f32x2 work on both halves in one instruction, which halves the FP32
// issue slots the epilogue's activation math takes.
__device__ __forceinline__ uint64_t f2_pack(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_splat(float a) { return f2_pack(a, a); }
__device__ __forceinline__ void f2_unpack(uint64_t v, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float exp2_approx(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Φ(x) and g = exp(−x²/2) of two values at once for the
// tensor-core epilogues, from the rational
// approximation of erf by C. Hastings as printed in Abramowitz & Stegun,
// Handbook of Mathematical Functions, eq. 7.1.26:
//   erf(z) = 1 − (a1·t + a2·t² + a3·t³ + a4·t⁴ + a5·t⁵)·exp(−z²),
//   t = 1/(1 + p·z), z ≥ 0, |error| ≤ 1.5e−7.
// With z = |x|/√2, exp(−z²) = exp(−x²/2) is the same factor the normal
// density needs, so Φ and φ = g/√(2π) cost one exponential and one
// reciprocal. Φ(−|x|) = ½·(1 − erf(z)); Φ(x) = 1 − Φ(−x).
// In the code the coefficients a1..a5 are halved, so that poly(t)·g is
// Φ(−|x|) itself, and exp(−x²/2) = 2^(−x²·log2(e)/2).
__device__ __forceinline__ void normal_cdf_and_gauss_x2(uint64_t x, float x0, float x1,
                                                        uint64_t& cdf, uint64_t& g) {
    const uint64_t z = f2_mul(f2_pack(fabsf(x0), fabsf(x1)), f2_splat(0.70710678118654752f));
    float d0, d1;
    f2_unpack(f2_fma(z, f2_splat(0.3275911f), f2_splat(1.0f)), d0, d1);
    const uint64_t t = f2_pack(rcp_approx(d0), rcp_approx(d1));
    uint64_t poly = f2_fma(f2_splat(0.5307027145f), t, f2_splat(-0.7265760135f));
    poly = f2_fma(poly, t, f2_splat(0.7107068705f));
    poly = f2_fma(poly, t, f2_splat(-0.142248368f));
    poly = f2_fma(poly, t, f2_splat(0.127414796f));
    poly = f2_mul(poly, t);
    float m0, m1;
    f2_unpack(f2_mul(f2_mul(x, x), f2_splat(-0.72134752044448170f)), m0, m1);
    g = f2_pack(exp2_approx(m0), exp2_approx(m1));
    float q0, q1;  // Φ(−|x|)
    f2_unpack(f2_mul(poly, g), q0, q1);
    cdf = f2_pack(x0 >= 0.0f ? 1.0f - q0 : q0, x1 >= 0.0f ? 1.0f - q1 : q1);
}

// GeLU(x0), GeLU(x1) and GeLU′(x0), GeLU′(x1) of the tensor-core epilogues.
__device__ __forceinline__ void gelu_fast_x2(float x0, float x1, float& y0, float& y1) {
    const uint64_t x = f2_pack(x0, x1);
    uint64_t cdf, g;
    normal_cdf_and_gauss_x2(x, x0, x1, cdf, g);
    f2_unpack(f2_mul(x, cdf), y0, y1);
}

__device__ __forceinline__ void gelu_grad_fast_x2(float x0, float x1, float& d0, float& d1) {
    const uint64_t x = f2_pack(x0, x1);
    uint64_t cdf, g;
    normal_cdf_and_gauss_x2(x, x0, x1, cdf, g);
    f2_unpack(f2_fma(f2_mul(x, f2_splat(0.39894228040143268f)), g, cdf), d0, d1);
}

// The tanh approximation of GeLU, ½·x·(1 + tanh u), u = √(2/π)·(x + 0.044715·x³),
// for two values at once. ½·(1 + tanh u) is the logistic function
// s = 1/(1 + exp(−2u)), so GeLU_tanh(x) = x·s: one exp2 and one reciprocal,
// with no cancellation for negative x (exp(−2u) = ∞ gives s = 0).
// The derivative, ½(1 + tanh u) + ½·x·(1 − tanh² u)·u′, is
// s + x·s·(1 − s)·2u′ with 2u′ = 2√(2/π)·(1 + 3·0.044715·x²).
__device__ __forceinline__ uint64_t logistic_2u_x2(uint64_t x, uint64_t x2) {
    // −2u·log2(e) = x·(1 + 0.044715·x²)·(−2√(2/π)·log2(e))
    const uint64_t inner = f2_fma(x2, f2_splat(0.044715f), f2_splat(1.0f));
    float m0, m1;
    f2_unpack(f2_mul(f2_mul(x, inner), f2_splat(-2.3022082f)), m0, m1);
    const uint64_t e = f2_pack(exp2_approx(m0), exp2_approx(m1));
    float d0, d1;
    f2_unpack(f2_fma(e, f2_splat(1.0f), f2_splat(1.0f)), d0, d1);
    return f2_pack(rcp_approx(d0), rcp_approx(d1));
}

__device__ __forceinline__ void gelu_tanh_fast_x2(float x0, float x1, float& y0, float& y1) {
    const uint64_t x = f2_pack(x0, x1);
    const uint64_t s = logistic_2u_x2(x, f2_mul(x, x));
    f2_unpack(f2_mul(x, s), y0, y1);
}

__device__ __forceinline__ void gelu_tanh_grad_fast_x2(float x0, float x1, float& d0, float& d1) {
    const uint64_t x = f2_pack(x0, x1);
    const uint64_t x2 = f2_mul(x, x);
    const uint64_t s = logistic_2u_x2(x, x2);
    // 2u′ = 2√(2/π) + 2√(2/π)·0.134145·x²
    const uint64_t du2 = f2_fma(x2, f2_splat(0.21406445f), f2_splat(1.5957691f));
    const uint64_t one_minus_s = f2_fma(s, f2_splat(-1.0f), f2_splat(1.0f));
    const uint64_t t = f2_mul(f2_mul(x, s), one_minus_s);
    f2_unpack(f2_fma(t, du2, s), d0, d1);
}

// The same two functions through CUDA's tanhf (the plain path).
__device__ __forceinline__ float gelu_tanh_f32(float x) {
    const float u = 0.79788456080286536f * (x + 0.044715f * x * x * x);
    return 0.5f * x * (1.0f + tanhf(u));
}

__device__ __forceinline__ float gelu_tanh_grad_f32(float x) {
    const float u = 0.79788456080286536f * (x + 0.044715f * x * x * x);
    const float th = tanhf(u);
    const float du = 0.79788456080286536f * (1.0f + 0.134145f * x * x);
    return 0.5f * (1.0f + th) + 0.5f * x * (1.0f - th * th) * du;
}

// Activation of the tensor-core epilogues for epilogue kind EPI.
template <int EPI>
__device__ __forceinline__ void act_fast_x2(float x0, float x1, float& y0, float& y1) {
    if constexpr (EpiTraits<EPI>::kTanh) {
        gelu_tanh_fast_x2(x0, x1, y0, y1);
    } else {
        gelu_fast_x2(x0, x1, y0, y1);
    }
}

template <int EPI>
__device__ __forceinline__ void act_grad_fast_x2(float x0, float x1, float& d0, float& d1) {
    if constexpr (EpiTraits<EPI>::kTanh) {
        gelu_tanh_grad_fast_x2(x0, x1, d0, d1);
    } else {
        gelu_grad_fast_x2(x0, x1, d0, d1);
    }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Column sums of a 32 × 32 block held one row per lane (x[j] = column j of
// this lane's row): lane l returns the sum of column l over the 32 rows. Five
// exchange rounds; in each, a lane keeps half of its remaining columns and
// adds its partner's values of them, so the adds follow a fixed pairwise tree
// over the rows and the result is the same on every run.
__device__ __forceinline__ float warp_column_sums32(float (&x)[32], int lane) {
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1) {
        const bool upper = (lane & w) != 0;
#pragma unroll
        for (int i = 0; i < w; ++i) {
            const float send = upper ? x[i] : x[i + w];
            const float keep = upper ? x[i + w] : x[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
        }
    }
    return x[0];
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& v, float* f) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(p[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

// Epilogue of one 32 × 32 chunk of the accumulator: this warp's 32 rows
// row0 .. row0+31 (lane i holds row row0 + i) and columns col0 .. col0+31.
// The results are written row by row into the warp's shared-memory staging
// slot in the swizzled layout the output tensor map expects (bf16: 64-byte
// rows, 64-byte swizzle; fp32: 128-byte rows, 128-byte swizzle, which makes
// the 16-byte shared stores of a warp bank-conflict free), then one lane
// stores the whole chunk with a TMA bulk tensor store, which clips rows and
// columns outside the output. The slot is reused only after the previous
// store of this warp has finished reading it.
// DBL: the warp stages chunks alternately in two slots (slot_base and the
// 4 KB after it), so a chunk's bulk store may still be reading one slot while
// the next chunk is staged in the other; sbuf is the warp's toggle. It flips
// only when a store group is committed (a chunk wholly outside the output
// stores nothing), so the most recent group always read the other slot and
// waiting for all but one group frees this one.
// cs_mode (GeLU′ epilogues with colsum_out): 0 = none; 1 = keep this chunk's
// stored values in csx; 2 = add them to csx, reduce csx over the 32 lanes
// and write the column sums to colsum_out row cs_row (if cs_row ≥ 0).
template <int EPI, bool DBL>
__device__ __forceinline__ void epilogue_chunk(const GemmArgs& g, const CUtensorMap* tmO0,
                                               const CUtensorMap* tmO1, const uint32_t (&acc)[32],
                                               int row0, int col0, int M, int N, uint32_t slot_base,
                                               uint32_t& sbuf, int lane, float (&csx)[32],
                                               int cs_mode, int64_t cs_row) {
    const uint32_t slot = DBL ? slot_base + sbuf * kEpiSlotBytes : slot_base;
    const int row = row0 + lane;
    const bool any = (row0 < M) && (col0 < N);
    if constexpr (EPI == EPI_F32) {
        if (lane == 0) {
            if (DBL) bulk_wait_read1();
            else bulk_wait_read0();
        }
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint4 v = make_uint4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
            st_shared_v4(slot + lane * 128 + ((j ^ (lane & 7)) << 4), v);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && any) {
            tma_store_3d(tmO0, slot, col0, row0, 0);
            bulk_commit();
        }
        if (DBL && any) sbuf ^= 1u;
    } else {
        uint4 o0[4], o1[4];
        const int64_t off = static_cast<int64_t>(row) * g.ld_out + col0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int c = col0 + 8 * q;
            float v[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(acc[8 * q + i]);
            if constexpr (EpiTraits<EPI>::kBias) {
                if (g.bias != nullptr && c < N) {
                    float bb[8];
                    unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(g.bias + c)), bb);
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] += bb[i];
                }
            }
            if constexpr (EpiTraits<EPI>::kDAct) {
                float hh[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                if (row < M && c < N)
                    unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(g.aux + off + 8 * q)), hh);
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                    float d0, d1;
                    act_grad_fast_x2<EPI>(hh[i], hh[i + 1], d0, d1);
                    f2_unpack(f2_mul(f2_pack(v[i], v[i + 1]), f2_pack(d0, d1)), v[i], v[i + 1]);
                }
            }
            o0[q].x = pack_bf16x2(v[0], v[1]);
            o0[q].y = pack_bf16x2(v[2], v[3]);
            o0[q].z = pack_bf16x2(v[4], v[5]);
            o0[q].w = pack_bf16x2(v[6], v[7]);
            if constexpr (EpiTraits<EPI>::kAct) {
                float y[8];
#pragma unroll
                for (int i = 0; i < 8; i += 2) act_fast_x2<EPI>(v[i], v[i + 1], y[i], y[i + 1]);
                o1[q].x = pack_bf16x2(y[0], y[1]);
                o1[q].y = pack_bf16x2(y[2], y[3]);
                o1[q].z = pack_bf16x2(y[4], y[5]);
                o1[q].w = pack_bf16x2(y[6], y[7]);
            }
        }
        if (lane == 0) {
            if (DBL) bulk_wait_read1();
            else bulk_wait_read0();
        }
        __syncwarp();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t a = lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4);
            st_shared_v4(slot + a, o0[q]);
            if constexpr (EpiTraits<EPI>::kAct) st_shared_v4(slot + 2048 + a, o1[q]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && any) {
            tma_store_3d(tmO0, slot, col0, row0, 0);
            if constexpr (EpiTraits<EPI>::kAct) tma_store_3d(tmO1, slot + 2048, col0, row0, 0);
            bulk_commit();
        }
        if (DBL && any) sbuf ^= 1u;
        if constexpr (EpiTraits<EPI>::kDAct) {
            // da's partial from the values just stored (rows beyond M and
            // columns beyond N hold zeros): this lane's row of the chunk, then
            // with cs_mode 2 the sum over both chunks' 64 rows per column
            if (cs_mode != 0) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float x[8];
                    unpack_bf16x8(o0[q], x);
#pragma unroll
                    for (int i = 0; i < 8; ++i) csx[8 * q + i] = cs_mode == 1 ? x[i] : csx[8 * q + i] + x[i];
                }
                if (cs_mode == 2) {
                    const float s = warp_column_sums32(csx, lane);
                    if (cs_row >= 0 && col0 + lane < N) g.colsum_out[cs_row * N + col0 + lane] = s;
                }
            }
        }
    }
}

// The epilogue warps' loop over this CTA's work units (shared by the
// one-CTA and the CTA-pair kernels). Each warp may read only the tensor-memory
// lanes of its SM sub-partition (warp index mod 4), 32 accumulator rows.
//
// The sub-partitions that also host the TMA producer (warp 0) and the MMA
// issuer (warp 1) should stay lightly loaded: epilogue math and store traffic
// there delay those latency-critical single threads and the tensor pipe
// idles (measured: up to 0.1 ms per 7B GEMM for GeLU, 4–6% for fp32
// outputs). With RELAY, the 4 epilogue warps of sub-partitions 0 and 1
// are relays: they drain their rows from tensor memory and pass each raw
// fp32 32 × 32 chunk through their shared-memory slot (128-byte swizzle,
// conflict-free) to a partner warp in sub-partition 2 or 3, which computes
// and stores both its own chunk and the relayed one. Hand-offs use one
// full/empty mbarrier pair per relay (bounded waits). Relaying doubles the
// work of the computing warps, so it pays only when a tile's main loop is
// long enough to hide it; the host picks the instantiation per launch.
// Whether an instantiation can finish split tiles. The relaying GeLU′
// epilogue sums da's columns over the rows of two warps, which a split tile
// (finished warp by warp) does not have together; the relaying GeLU epilogue
// has no registers to spare for the split path (it would spill in the
// whole-tile path too). Their launches always run whole tiles (the host keeps
// them so), and the split path is compiled out of them.
template <int EPI, bool RELAY>
constexpr bool kSplittable = !((EpiTraits<EPI>::kDAct || EpiTraits<EPI>::kAct) && RELAY);

template <int BN, int EPI, bool PAIR, bool RELAY, bool DBL = false>
__device__ __forceinline__ void epilogue_role(const GemmArgs& g, const CUtensorMap* tmO0,
                                              const CUtensorMap* tmO1, uint32_t tmem_base,
                                              uint64_t* tfull, uint64_t* tempty, uint64_t* xfull,
                                              uint64_t* xempty, uint8_t* sEpi, int worker,
                                              int nworkers, int tile_rows, int cta_row_off,
                                              volatile int* abort, uint64_t limit, int warp,
                                              int lane, const PairQueue* queue = nullptr) {
    constexpr int kChunks = BN / 64;  // 32-column chunks per half of the tile
    const int quad = warp & 3;          // tensor-memory lanes this warp may access
    const int half = (warp - 2) / 4;    // which half of the tile's columns
    const bool relay = RELAY && quad < 2;
    const int pair_id = (quad & 1) + 2 * half;  // relay (quad 0/1) <-> math (quad 2/3)
    constexpr int kSlotsPerWarp = DBL ? 2 : 1;
    const uint32_t slot = smem_u32(sEpi + kSlotsPerWarp * (warp - 2) * kEpiSlotBytes);
    uint32_t sbuf = 0;  // DBL: which of the warp's two slots stages the next chunk
    // a math warp's (quad 2/3) partner relay is warp 2 + 4·half + quad (quad - 2,
    // same half), whose slot index is 4·half + quad
    const uint32_t partner_slot = smem_u32(sEpi + kSlotsPerWarp * (4 * half + quad) * kEpiSlotBytes);
    if (lane == 0 && !relay) {
        tma_prefetch_desc(tmO0);
        if (EpiTraits<EPI>::kAct || g.second) tma_prefetch_desc(tmO1);
    }
    uint32_t xcount = 0;
    bool stored = false;  // a relay warp has bulk stores of a split tile in flight
    UnitCursor cur = unit_cursor(worker, nworkers, queue != nullptr);
    WorkUnit w;
    bool qok = true;
    for (int local = 0;
         cursor_next<false, true, !kSplittable<EPI, RELAY>>(g, nworkers, cur, w, queue, qok, abort, limit);
         ++local) {
        const int buf = local & 1;
        const uint32_t aphase = (local >> 1) & 1;
        // every lane waits; the warp proceeds only if all lanes saw the
        // phase complete, so the .sync.aligned loads below never diverge
        const bool ok = mbar_wait_bounded(smem_u32(&tfull[buf]), aphase, abort, limit);
        if (!__all_sync(0xffffffffu, ok)) {
            raise_timeout(abort);
            break;
        }
        tc_fence_after();
        const int tile_row0 = w.mb * tile_rows + cta_row_off;
        const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                               static_cast<uint32_t>(buf * BN);
        // the unit's product: sizes and output map (a grouped launch's second
        // product stores through tmO1; grouping is for single-output epilogues)
        const int uM = w.prob ? g.M2 : g.M;
        const int uN = w.prob ? g.N2 : g.N;
        const CUtensorMap* uO = w.prob ? tmO1 : tmO0;
        if (kSplittable<EPI, RELAY> && w.pieces > 1) {
            // A split tile. Every epilogue warp (no relay) takes its own 32
            // rows and half of the columns; the warp of the last unit to arrive
            // adds the tile's partials in ascending k order and runs the
            // epilogue for those rows.
            const int own_r = cta_row_off + quad * 32;
            // one counter per split tile, CTA of the pair and epilogue warp
            int* ctr = g.counters + (static_cast<int64_t>(w.key) * 2 + cta_row_off / kBM) * 8 + (warp - 2);
            // If every other unit of the tile has arrived already, this one is
            // the last for certain: it neither stores its partial nor arrives,
            // and takes its own part from tensor memory while summing.
            int seen = 0;
            if (lane == 0) seen = ld_acquire_gpu(ctr);
            seen = __shfl_sync(0xffffffffu, seen, 0);
            const bool sure_last = (seen == w.pieces - 1);
            bool last = sure_last;
            if (!sure_last) {
                const int64_t my_slot = partial_slot(g, w, w.piece, nworkers);
#pragma unroll 1
                for (int i = 0; i < kChunks; ++i) {
                    const int c = half * kChunks + i;
                    uint32_t acc[32];
                    tmem_ld_32x32b_x32(t_row + c * 32, acc);
                    tmem_wait_ld();
                    if (i == kChunks - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if constexpr (PAIR)
                                mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
                            else
                                mbar_arrive(smem_u32(&tempty[buf]));
                        }
                    }
                    partial_store(partial_chunk(g, my_slot, tile_rows, BN, own_r, c * 32), acc, lane);
                }
                last = partial_arrive(ctr, w.pieces, lane);
            }
            if (last) {
                if (RELAY && relay) {
                    // The slot may still hold the last chunk this warp relayed
                    // on an earlier whole tile: it is staged over only once the
                    // partner has taken that chunk (the wait passes at once if
                    // it has, or if nothing was relayed yet).
                    const bool got = mbar_wait_bounded(smem_u32(&xempty[pair_id]), (xcount & 1u) ^ 1u,
                                                       abort, limit);
                    if (!__all_sync(0xffffffffu, got)) {
                        raise_timeout(abort);
                        break;
                    }
                }
                float csx[32];  // unused: no column sums on split tiles
#pragma unroll 1
                for (int i = 0; i < kChunks; ++i) {
                    const int c = half * kChunks + i;
                    uint32_t acc[32];
                    partial_sum(g, w, nworkers, tile_rows, BN, own_r, c * 32, acc, lane,
                                sure_last ? w.piece : -1, t_row + c * 32);
                    epilogue_chunk<EPI, DBL>(g, uO, tmO1, acc, tile_row0 + quad * 32, w.nb * BN + c * 32,
                                             uM, uN, slot, sbuf, lane, csx, 0, -1);
                }
                if (sure_last) {
                    // the accumulator was read in the loop above: release it, and
                    // put the counter (at pieces - 1) back to zero
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if constexpr (PAIR)
                            mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
                        else
                            mbar_arrive(smem_u32(&tempty[buf]));
                        atomicExch(ctr, 0);
                    }
                }
                stored = true;
            }
            continue;
        }
        if (RELAY && relay && stored) {
            // the slot becomes a hand-off buffer again: the split tile's bulk
            // stores must have finished reading it
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
            stored = false;
        }
        bool failed = false;
        float csx[32];  // da partial of the current columns (relay, GeLU′ only)
        // da partials (relay only): the own rows and the partner's rows of these
        // columns form one row of colsum_out per computing warp and CTA tile
        const bool cs_on = RELAY && g.colsum_out != nullptr;
        const int64_t cs_row =
            tile_row0 < uM ? static_cast<int64_t>(tile_row0 / kBM) * 2 + (quad - 2) : -1;
#pragma unroll 1
        for (int i = 0; i < kChunks; ++i) {
            const int c = half * kChunks + i;
            const int col0 = w.nb * BN + c * 32;
            uint32_t acc[32];
            tmem_ld_32x32b_x32(t_row + c * 32, acc);
            tmem_wait_ld();
            if (i == kChunks - 1) {
                // this warp's part of the accumulator is in registers: release it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (PAIR)
                        mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
                    else
                        mbar_arrive(smem_u32(&tempty[buf]));
                }
            }
            if (RELAY && relay) {
                const bool got = mbar_wait_bounded(smem_u32(&xempty[pair_id]), (xcount & 1u) ^ 1u,
                                                   abort, limit);
                if (!__all_sync(0xffffffffu, got)) {
                    failed = true;
                    break;
                }
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    st_shared_v4(slot + lane * 128 + ((j ^ (lane & 7)) << 4),
                                 make_uint4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]));
                mbar_arrive(smem_u32(&xfull[pair_id]));
                ++xcount;
                continue;
            }
            epilogue_chunk<EPI, DBL>(g, uO, tmO1, acc, tile_row0 + quad * 32, col0, uM, uN, slot, sbuf,
                                     lane, csx, cs_on ? 1 : 0, cs_row);
            if constexpr (RELAY) {
                // the partner relay's chunk: same columns, rows of quad - 2
                const bool got = mbar_wait_bounded(smem_u32(&xfull[pair_id]), xcount & 1u, abort, limit);
                if (!__all_sync(0xffffffffu, got)) {
                    failed = true;
                    break;
                }
                uint32_t pacc[32];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint4 v = ld_shared_v4(partner_slot + lane * 128 + ((j ^ (lane & 7)) << 4));
                    pacc[4 * j] = v.x;
                    pacc[4 * j + 1] = v.y;
                    pacc[4 * j + 2] = v.z;
                    pacc[4 * j + 3] = v.w;
                }
                mbar_arrive(smem_u32(&xempty[pair_id]));
                ++xcount;
                epilogue_chunk<EPI, DBL>(g, uO, tmO1, pacc, tile_row0 + (quad - 2) * 32, col0, uM, uN,
                                         slot, sbuf, lane, csx, cs_on ? 2 : 0, cs_row);
            }
        }
        if (failed) {
            raise_timeout(abort);
            break;
        }
    }
    if (!qok) raise_timeout(abort);
    if (lane == 0) bulk_wait0();  // this warp's stores are complete before exit
    __syncwarp();
}

// Counters of a later launch (GemmArgs::zero_counters), zeroed by the idle
// lanes of warp 0 of every CTA after the wait for the predecessor.
__device__ __forceinline__ void zero_later_counters(const GemmArgs& g, int lane) {
    if (g.zero_counters == nullptr || lane == 0) return;
    for (int i = blockIdx.x * 31 + lane - 1; i < g.zero_count; i += gridDim.x * 31) g.zero_counters[i] = 0;
}

template <int BN, bool A_MN, bool B_MN, int EPI, bool RELAY>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmO0, const __grid_constant__ CUtensorMap tmO1,
                   const GemmArgs g) {
    using C = TileCfg<BN>;
    constexpr int STAGES = C::STAGES;
    constexpr uint32_t IDESC = idesc_bf16_f32(kBM, BN, A_MN, B_MN);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * C::A_BYTES;
    uint8_t* sEpi = sB + STAGES * C::B_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + kEpiStagingBytes);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* tfull = bars + 2 * STAGES;
    uint64_t* tempty = bars + 2 * STAGES + 2;
    uint64_t* drain = bars + 2 * STAGES + 4;
    uint64_t* xfull = bars + 2 * STAGES + 5;   // relay hand-off, 4 pairs
    uint64_t* xempty = bars + 2 * STAGES + 9;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 13);
    volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int x = 0; x < 4; ++x) {
            mbar_init(smem_u32(&xfull[x]), 32);
            mbar_init(smem_u32(&xempty[x]), 32);
        }
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(smem_u32(&tfull[b]), 1);
            mbar_init(smem_u32(&tempty[b]), kEpiWarps);
        }
        mbar_init(smem_u32(drain), 1);
        *abort = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // launched as a programmatic dependent: the prologue above overlaps the
    // predecessor's last CTAs; its outputs are read only after this wait
    grid_dep_wait();
    grid_dep_launch();

    const uint64_t limit = g.wait_limit_ns;
    if (warp == 0) zero_later_counters(g, lane);

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmA);
            tma_prefetch_desc(&tmB);
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;
            bool ok = true;
            WorkIter it = work_iter(blockIdx.x, gridDim.x);
            WorkUnit w;
            while (ok && next_unit(g, it, w)) {
                const int mb = w.mb, nb = w.nb;
                for (int kb = w.kb0; kb < w.kb1; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&empty[stage]), phase ^ 1u, abort, limit)) {
                        raise_timeout(abort);
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&full[stage]);
                    mbar_arrive_expect_tx(fb, C::STAGE_BYTES);
                    const uint32_t a_dst = smem_u32(sA + stage * C::A_BYTES);
                    const uint32_t b_dst = smem_u32(sB + stage * C::B_BYTES);
                    if constexpr (!A_MN) {
                        tma_load_2d(a_dst, &tmA, fb, kb * kBK, mb * kBM);
                    } else {
                        tma_load_2d(a_dst, &tmA, fb, mb * kBM, kb * kBK);
                        tma_load_2d(a_dst + 8192, &tmA, fb, mb * kBM + 64, kb * kBK);
                    }
                    if constexpr (!B_MN) {
                        tma_load_2d(b_dst, &tmB, fb, kb * kBK, nb * BN);
                    } else {
#pragma unroll
                        for (int j = 0; j < BN / 64; ++j)
                            tma_load_2d(b_dst + j * 8192, &tmB, fb, nb * BN + j * 64, kb * kBK);
                    }
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (ok && !*abort) {
                // Producer tail: wait until the MMA thread has released every
                // slot, so no tensor-core completion is still due to arrive on
                // this CTA's barriers when it exits.
                int s = stage;
                uint32_t ph = phase;
                for (int i = 0; i < STAGES && ok; ++i) {
                    if (!mbar_wait_bounded(smem_u32(&empty[s]), ph ^ 1u, abort, limit)) {
                        raise_timeout(abort);
                        ok = false;
                    }
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok || *abort) {
                // Wind down: wait (bounded) for the copies still in flight, the
                // most recent load of each of the last min(issued, STAGES) slots.
                int s = stage;
                uint32_t ph = phase;
                const int n = issued < STAGES ? issued : STAGES;
                for (int i = 0; i < n; ++i) {
                    if (--s < 0) {
                        s = STAGES - 1;
                        ph ^= 1u;
                    }
                    volatile int never = 0;
                    mbar_wait_bounded(smem_u32(&full[s]), ph, &never, limit);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            WorkIter it = work_iter(blockIdx.x, gridDim.x);
            WorkUnit w;
            for (int local = 0; ok && next_unit(g, it, w); ++local) {
                const int kb0 = w.kb0, kb1 = w.kb1;
                const int buf = local & 1;
                const uint32_t aphase = (local >> 1) & 1;
                if (!mbar_wait_bounded(smem_u32(&tempty[buf]), aphase ^ 1u, abort, limit)) {
                    raise_timeout(abort);
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * BN);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait_bounded(smem_u32(&full[stage]), phase, abort, limit)) {
                        raise_timeout(abort);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_base = smem_u32(sA + stage * C::A_BYTES);
                    const uint32_t b_base = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k) {
                        // K-major: the 16-element k slice is 32 bytes further along
                        // each 128-byte swizzled row. MN-major: it is 16 rows of
                        // 128 bytes further down; 64-wide MN chunks are 8 KB apart.
                        const uint64_t ad = A_MN ? smem_desc_sw128(a_base + k * 2048, 8192, 1024)
                                                 : smem_desc_sw128(a_base + k * 32, 16, 1024);
                        const uint64_t bd = B_MN ? smem_desc_sw128(b_base + k * 2048, 8192, 1024)
                                                 : smem_desc_sw128(b_base + k * 32, 16, 1024);
                        umma_bf16(d_tmem, ad, bd, IDESC, (kb > kb0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit(smem_u32(&empty[stage]));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                umma_commit(smem_u32(&tfull[buf]));
            }
            if (!ok || *abort) {
                // Wind down: wait (bounded) for every MMA issued so far.
                umma_commit(smem_u32(drain));
                volatile int never = 0;
                mbar_wait_bounded(smem_u32(drain), 0, &never, limit);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue warps
        epilogue_role<BN, EPI, false, RELAY>(g, &tmO0, &tmO1, tmem_base, tfull, tempty, xfull, xempty, sEpi,
                                             blockIdx.x, gridDim.x, kBM, 0, abort, limit, warp, lane);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

}  // namespace tpmlp
