/*
 * tpmlp — tensor-parallel Transformer MLP block on one B200 (sm_100a).
 *
 * The block is Z = GeLU(X·A + a)·B + b with A (h × F) split by columns into p
 * shards and B (F × h) split by rows into the matching p shards, forward and
 * backward (page "Megatron", zzmblog.top, section "张量并行 / 数学原理" for the
 * two splits; section "Transformer层的张量并行实现" for their pairing in the MLP;
 * section "实战使用 / 基础训练示例" for activation_func = "gelu"). All p shards
 * live on one GPU, so the all-reduce of the row-parallel partials happens
 * inside the library as an ordered shard reduction.
 *
 * Conventions for every entry point below:
 *  - Matrices are dense, row-major, with no padding between rows.
 *  - Pointers are DEVICE pointers owned by the caller, except where a
 *    comment says otherwise. The library never allocates or frees memory.
 *  - The pointers and `stream` belong to the device that is current on the
 *    calling thread (cudaSetDevice); the library reads that device's
 *    properties and launches there.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream). Work is enqueued asynchronously on it; the call returns once
 *    the launches are enqueued.
 *  - All argument checks happen before the first launch: a call that
 *    returns an error has enqueued nothing.
 *  - Results are deterministic: the same inputs and p give bit-identical
 *    outputs on every run.
 *  - The library keeps a small amount of process-wide state (the split
 *    policy, the wait limit, a launch counter, per-device caches, one device
 *    status word per device). Its caches are guarded, so host threads may
 *    call it at the same time, each on its own stream; the settings and the
 *    status word are shared by all of them.
 */
#ifndef TPMLP_H
#define TPMLP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum tpmlp_status {
    TPMLP_OK = 0,
    TPMLP_ERR_INVALID = 1,     /* bad size, p, null pointer or dtype code */
    TPMLP_ERR_ALIGN = 2,       /* a bf16 pointer is not 16-byte aligned */
    TPMLP_ERR_UNSUPPORTED = 3, /* no GPU of compute capability 10.x, or sizes beyond int32 */
    TPMLP_ERR_WORKSPACE = 4,   /* workspace null or smaller than tpmlp_workspace_size() */
    TPMLP_ERR_CUDA = 5,        /* a CUDA runtime/driver call or a launch failed */
    TPMLP_ERR_TIMEOUT = 6      /* a kernel gave up a bounded wait (device status word) */
} tpmlp_status;

/* Element type of X, A, a, B, b, H, Y, Z, dZ, dH and dX. Weight and bias
 * gradients (dA, da, dB, db) are always fp32 ("weight update in full
 * precision", page "Megatron", section "其他关键技术 / 混合精度训练").
 * TPMLP_BF16 accumulates in fp32 on the tensor cores; TPMLP_FP32 uses fp32
 * FFMA throughout (no TF32). */
typedef enum tpmlp_dtype { TPMLP_BF16 = 0, TPMLP_FP32 = 1 } tpmlp_dtype;

/* Activation of the block. TPMLP_GELU_ERF is the exact GeLU x·Φ(x), the form
 * tp_mlp_fwd and tp_mlp_bwd use (the pages name the activation only as
 * "gelu"). TPMLP_GELU_TANH is the tanh approximation
 * ½·x·(1 + tanh(√(2/π)·(x + 0.044715·x³))) (Hendrycks & Gimpel, 2016). */
typedef enum tpmlp_activation { TPMLP_GELU_ERF = 0, TPMLP_GELU_TANH = 1 } tpmlp_activation;

/* Bytes of device workspace that tp_mlp_fwd and tp_mlp_bwd need for these
 * sizes under the current split policy and dynamic-schedule setting (the
 * larger of the two calls' needs). Returns 0 for invalid sizes. Holds, each
 * part rounded up to 256 bytes: the fp32 partial tiles and the arrival
 * counters of products whose output tiles are split over several work units
 * (see tpmlp_set_split_policy; none when no product splits), followed by the
 * dynamic schedule's two int counters when some product runs it (see
 * tpmlp_set_dynamic_schedule), and the partial column sums of the bias
 * gradients. The contents need no initialisation: a call that splits tiles
 * or runs the dynamic schedule first zeroes the counters itself. Changing
 * either setting can change the size: query it after setting them. */
size_t tpmlp_workspace_size(int64_t T, int64_t h, int64_t F, int p, tpmlp_dtype dt);

/* Forward (column-parallel, then row-parallel):
 *   H[:, i·Fp:(i+1)·Fp] = X·A_i + a_i        for shard i = 1..p, Fp = F/p
 *   Y = GeLU(H) = ½·H·(1 + erf(H/√2))         (exact erf form)
 *   Z = Σ_{i=1..p} Y_i·B_i + b                summed over shards in ascending i
 * X: T×h. A: h×F. a: F (may be NULL = zero). B: F×h. b: h (may be NULL).
 * H, Y: T×F outputs (H, the pre-activation, and Y are both kept for the
 * backward). Z: T×h output. All of dtype `dt`.
 * Requires T ≥ 0, h ≥ 1, F ≥ 1, p ≥ 1, F % p == 0. For TPMLP_BF16 the
 * pointers must be 16-byte aligned; when h % 8 != 0 or F % 8 != 0 a plain
 * (slower) GPU kernel path serves the call.
 * workspace: device buffer of at least tpmlp_workspace_size() bytes (may be
 * NULL when that size is 0). */
tpmlp_status tp_mlp_fwd(const void* X, const void* A, const void* a, const void* B,
                        const void* b, void* H, void* Y, void* Z, int64_t T, int64_t h,
                        int64_t F, int p, tpmlp_dtype dt, void* workspace,
                        size_t workspace_bytes, void* stream);

/* Backward, given the upstream gradient dZ (T×h) and the forward's X, A, B,
 * H and Y (chain rule on the forward above):
 *   db = 1ᵀ·dZ                       (h, fp32)
 *   dB_i = Y_iᵀ·dZ                   (F×h, fp32; row block i per shard)
 *   dH_i = (dZ·B_iᵀ) ⊙ GeLU′(H_i)    (T×F, dtype dt; written to dH)
 *   da = 1ᵀ·dH                       (F, fp32)
 *   dA_i = Xᵀ·dH_i                   (h×F, fp32; column block i per shard)
 *   dX = Σ_{i=1..p} dH_i·A_iᵀ        (T×h, dtype dt; ascending i)
 * GeLU′(x) = Φ(x) + x·φ(x). X is replicated across shards, so its gradient
 * is the sum over shards: the backward counterpart of the forward all-reduce.
 * dH is an output the caller owns (T×F). Same requirements as tp_mlp_fwd.
 * With T == 0 the gradients dA, da, dB, db are set to zero. */
tpmlp_status tp_mlp_bwd(const void* dZ, const void* X, const void* A, const void* B,
                        const void* H, const void* Y, void* dX, float* dA, float* da,
                        float* dB, float* db, void* dH, int64_t T, int64_t h, int64_t F,
                        int p, tpmlp_dtype dt, void* workspace, size_t workspace_bytes,
                        void* stream);

/* tp_mlp_fwd and tp_mlp_bwd with a selectable activation (GeLU in the
 * forward, its derivative in the backward); same arguments, requirements
 * and workspace, plus `act`. The backward must use the forward's `act`.
 * Returns TPMLP_ERR_INVALID for an unknown `act`. */
tpmlp_status tp_mlp_fwd_ex(const void* X, const void* A, const void* a, const void* B,
                           const void* b, void* H, void* Y, void* Z, int64_t T, int64_t h,
                           int64_t F, int p, tpmlp_dtype dt, tpmlp_activation act, void* workspace,
                           size_t workspace_bytes, void* stream);
tpmlp_status tp_mlp_bwd_ex(const void* dZ, const void* X, const void* A, const void* B,
                           const void* H, const void* Y, void* dX, float* dA, float* da, float* dB,
                           float* db, void* dH, int64_t T, int64_t h, int64_t F, int p,
                           tpmlp_dtype dt, tpmlp_activation act, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Tensor-parallel linear layer Y = X·W + bias, X: T×K, W: K×N, bias: N (may
 * be NULL), all of dtype dt; the attention layer's use of the two splits
 * (page "Megatron", section "Transformer层的张量并行实现": the QKV projection is
 * split by columns, the output projection by rows; section "张量并行 /
 * 数学原理" for the splits themselves).
 *   TPMLP_SPLIT_COLUMNS: W = [W_1 … W_p] (N % p == 0). Forward Y_i = X·W_i +
 *     bias_i side by side, no exchange. Backward dW_i = Xᵀ·dY_i, dbias_i =
 *     1ᵀ·dY_i and, X being replicated, dX = Σ_{i=1..p} dY_i·W_iᵀ summed in
 *     ascending i.
 *   TPMLP_SPLIT_ROWS: W = [W_1; …; W_p] (K % p == 0), X split into the
 *     matching column blocks X_i. Forward Y = Σ_{i=1..p} X_i·W_i + bias,
 *     ascending i, bias once. Backward dX_i = dY·W_iᵀ (no exchange), dW_i =
 *     X_iᵀ·dY, dbias = 1ᵀ·dY.
 * dW (K×N) and dbias (N) are fp32; dX (T×K) and Y (T×N) have dtype dt.
 * Requirements, alignment and error behaviour as tp_mlp_fwd, with K and N in
 * place of h and F. With T == 0, dW and dbias are set to zero. */
typedef enum tpmlp_split { TPMLP_SPLIT_COLUMNS = 0, TPMLP_SPLIT_ROWS = 1 } tpmlp_split;

size_t tpmlp_linear_workspace_size(int64_t T, int64_t K, int64_t N, int p, tpmlp_split split,
                                   tpmlp_dtype dt);
tpmlp_status tp_linear_fwd(const void* X, const void* W, const void* bias, void* Y, int64_t T,
                           int64_t K, int64_t N, int p, tpmlp_split split, tpmlp_dtype dt,
                           void* workspace, size_t workspace_bytes, void* stream);
tpmlp_status tp_linear_bwd(const void* dY, const void* X, const void* W, void* dX, float* dW,
                           float* dbias, int64_t T, int64_t K, int64_t N, int p, tpmlp_split split,
                           tpmlp_dtype dt, void* workspace, size_t workspace_bytes, void* stream);

/* Activation recompute (page "Megatron", section "其他关键技术 / 激活重计算":
 * keep fewer forward activations and recompute them in the backward). A
 * caller that keeps only the pre-activation H after tp_mlp_fwd(_ex) rebuilds
 * Y = act(H) here just before tp_mlp_bwd(_ex):
 *   Y[i] = act(H[i]), i < n (n = T·F), H and Y device arrays of dtype dt,
 *   act = the forward's activation.
 * One bandwidth-bound pass (n reads, n writes). Y rebuilt from the stored H
 * (rounded to dt) can differ from the forward's Y (computed from the fp32
 * accumulator) by the effect of that one rounding. Returns
 * TPMLP_ERR_INVALID for n < 0, null pointers, or an unknown dt or act. */
tpmlp_status tp_mlp_recompute_activation(const void* H, void* Y, int64_t n, tpmlp_dtype dt,
                                         tpmlp_activation act, void* stream);

/* Activation recompute from the block's input (same section): a caller that
 * keeps only X rebuilds H = X·A + a and Y = act(H) before the backward, the
 * forward's first product (column split, no shard sum) without the second.
 * Arguments, layouts, requirements and errors as tp_mlp_fwd_ex, without B,
 * b, Z and the workspace (this product needs none). H and Y are bitwise
 * those of tp_mlp_fwd_ex on the same inputs. Costs 2·T·h·F flops. */
tpmlp_status tp_mlp_recompute_hidden(const void* X, const void* A, const void* a, void* H, void* Y,
                                     int64_t T, int64_t h, int64_t F, int p, tpmlp_dtype dt,
                                     tpmlp_activation act, void* stream);

/* Static, NUL-terminated description of a status code. */
const char* tpmlp_strerror(tpmlp_status s);

/* Synchronizes `stream`, then reads and clears the current device's status
 * word. Returns TPMLP_ERR_TIMEOUT if a kernel launched since the last read
 * gave up a bounded wait (its outputs are then undefined), TPMLP_ERR_CUDA if
 * the synchronization itself failed, else TPMLP_OK. */
tpmlp_status tpmlp_last_device_status(void* stream);

/* How the tensor-core products are cut into work units. By default every
 * output tile is one unit whose K loop runs through all k-blocks (for the
 * two row-parallel products, Z = Σ Y_i·B_i and dX = Σ dH_i·A_iᵀ, through
 * the shards in ascending order), accumulating in tensor memory. A tile may
 * instead be split over several units, each covering a consecutive k range;
 * each writes an fp32 partial, and the last of them to finish adds all the
 * tile's partials in ascending k order inside the same kernel, then applies
 * the epilogue (bias, activation, rounding). No unit waits for another.
 *   0 = automatic: whole tiles in full waves of the GPU's CTA pairs, and
 *       the remaining tiles' k-blocks cut into one equal segment per pair (a
 *       stream-K tail) wherever a time model says that is faster,
 *   1 = whole tiles only,
 *   2 = the two row-parallel products as one unit per shard and tile when
 *       F/p is a multiple of 64 (the shards' partials summed in ascending
 *       shard order, the literal form of the pages' all-reduce); the other
 *       products as whole tiles,
 *   3 = the stream-K tail wherever it is valid (for tests and measurement).
 * Every schedule is deterministic: the same inputs, sizes, policy and GPU
 * model give bit-identical results. Different schedules agree within
 * rounding. Returns TPMLP_ERR_INVALID for other values. The workspace size
 * depends on it. */
tpmlp_status tpmlp_set_split_policy(int policy);
int tpmlp_get_split_policy(void);

/* Launch overlap (default on): the library's tensor-core and helper kernels
 * go out as programmatic dependent launches (CUDA's
 * cudaLaunchAttributeProgrammaticStreamSerialization). A kernel's CTAs may
 * then start, and set up their barriers and tensor memory, on SMs its
 * predecessor on the stream has already left; each waits for the
 * predecessor to complete before it reads or writes global memory. Results
 * are bit-identical with overlap on or off, and the first kernel of a call
 * never reads the caller's data before the caller's preceding work has
 * finished. Off: ordinary stream order. */
void tpmlp_set_launch_overlap(int on);
int tpmlp_get_launch_overlap(void);

/* Dynamic tile schedule (default on). The SMs of a GPU do not all run a
 * tile in the same time (measured on B200: the slowest CTA pairs take ~5%
 * longer, the same pairs in every product), so with a static round-robin of
 * tiles a long product ends with its slowest pair. With this on, the
 * tensor-core products with bf16 outputs that run at least 4 waves of tiles
 * on CTA pairs, at least 192 k-blocks (12288 of K) per tile and at least
 * 3072 k-blocks of work per CTA pair hand their tiles (and their stream-K
 * segments) out in order from a counter in the workspace: faster pairs take
 * more, and the pairs that share an operand panel stay closer together in
 * time (fewer DRAM re-reads). Which pair computes a tile does not change the
 * arithmetic: results are bit-identical with it on or off. A call that uses
 * it zeroes its counters with one small kernel first. (Measured on B200 in
 * power-limited full steps: the 175B-class step, ~3990 k-blocks per pair,
 * 0.5% faster; the 7B-class row products, ~1770, 0.7% slower each with it;
 * hence the thresholds.) */
void tpmlp_set_dynamic_schedule(int on);
int tpmlp_get_dynamic_schedule(void);

/* Upper bound, in nanoseconds, on any single wait inside a kernel (for data
 * from the tensor-memory accelerator, for the tensor cores, between warps).
 * Default 2e9 (2 s). A wait that runs out sets the device status word to
 * TPMLP_ERR_TIMEOUT and the kernel winds down and returns. 0 restores the
 * default. */
void tpmlp_set_wait_limit_ns(uint64_t ns);

/* Launches one kernel that waits, with limit `limit_ns`, on a barrier that
 * nothing ever completes, so that the bounded-wait path can be tested: after
 * it, tpmlp_last_device_status() returns TPMLP_ERR_TIMEOUT and the context
 * stays usable. */
tpmlp_status tpmlp_wait_selftest(uint64_t limit_ns, void* stream);

/* Number of kernels this library has launched in this process. */
uint64_t tpmlp_launch_count(void);

/* Evaluates GeLU(x[i]) into y[i] and GeLU′(x[i]) into dy[i] (fp32 device
 * arrays of n elements) with one of the forms the kernels use, so the
 * approximations can be checked against CUDA's functions:
 *   form 0: exact GeLU as the tensor-core epilogues compute it, Φ(x) from
 *           the rational erf approximation of C. Hastings (Abramowitz &
 *           Stegun, Handbook of Mathematical Functions, eq. 7.1.26,
 *           |error| ≤ 1.5e−7) sharing exp(−x²/2) with φ(x);
 *   form 1: exact GeLU through CUDA's erff and expf (the plain path);
 *   form 2: the tanh approximation as the tensor-core epilogues compute it,
 *           ½(1 + tanh u) = 1/(1 + exp(−2u));
 *   form 3: the tanh approximation through CUDA's tanhf (the plain path).
 * Returns TPMLP_ERR_INVALID for n < 0, null pointers or another form. */
tpmlp_status tpmlp_eval_activation(const float* x, float* y, float* dy, int64_t n, int form,
                                   void* stream);

/* Per-kernel timing on the launching stream, for measurement tools. While
 * enabled (on != 0), every kernel launch is bracketed by a pair of CUDA
 * events on its stream and tagged with its step (F1 column GEMM, F2 row
 * GEMM, B1..B5, and the helper kernels). tpmlp_profile_collect() waits for
 * the recorded events and adds their elapsed times into per-kind totals,
 * together with each launch's algorithmic flops (2·M·N·K for a GEMM) and
 * algorithmic bytes (every operand read once, every output written once).
 * Returns the number of kinds, or -1 if a CUDA call failed.
 * tpmlp_profile_read(kind, ...) returns those totals (any out-pointer may be
 * NULL); tpmlp_profile_name(kind) its static name; tpmlp_profile_reset()
 * clears them. The calls may come from several host threads (the state is
 * guarded by a lock); the timing events are created on the current device,
 * so one process times launches on one device. */
void tpmlp_profile_enable(int on);
int tpmlp_profile_collect(void);
int tpmlp_profile_kinds(void);
const char* tpmlp_profile_name(int kind);
tpmlp_status tpmlp_profile_read(int kind, uint64_t* launches, double* total_ms, double* flops,
                                double* bytes);
void tpmlp_profile_reset(void);

/* Backward that allocates nothing and takes no workspace. The pages have no
 * counterpart: this entry point exists for callers that cannot allocate
 * device memory when they run the backward, such as a plugin inside another
 * framework that owns all device allocations and offers extensions no
 * allocator, or a runtime with a fixed memory budget that forbids
 * allocation after start-up (cudaMalloc and cudaFree can also synchronize
 * the device, which such callers must avoid).
 * Computes the same gradients as tp_mlp_bwd, with the same arguments minus
 * the workspace, and the same requirements. The results agree within the
 * library's stated tolerance but not always bit for bit, because the order
 * of two accumulations can differ: da is summed from per-128-row column-sum
 * chunks here (tp_mlp_bwd sums two 64-row partials per tile that its GeLU′
 * epilogue writes when h ≥ 3072), and dX always runs each output tile's K
 * loop through all shards in tensor memory (tp_mlp_bwd may split that loop
 * and add the pieces' fp32 partials in ascending order). Its only scratch, the partial
 * column sums of db and da, is a fixed 8 MiB array inside this library
 * (tpmlp_noalloc_scratch_bytes()), held on every GPU that loads the library
 * until the process exits; dX always uses the unsplit schedule (each output
 * tile loops over the shards in ascending order), which needs no scratch.
 * The call needs 4·ceil(T/128)·h + 4·ceil(T/128)·F bytes of it (each part
 * rounded up to a multiple of 256); larger sizes return TPMLP_ERR_WORKSPACE
 * before any launch. It calls no allocating routine.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture. The address is kept for the life of the
 * process: after cudaDeviceReset on a device, the cached address belongs to
 * the destroyed context, so do not call this entry point on that device
 * again in the same process. Every call shares the one array: calls whose
 * kernels overlap on the GPU (on different streams or host threads) race on
 * it and give undefined gradients. Nothing in the array needs to start at
 * zero; each call writes every partial before reading it. */
tpmlp_status tp_mlp_bwd_noalloc(const void* dZ, const void* X, const void* A, const void* B,
                                const void* H, const void* Y, void* dX, float* dA, float* da,
                                float* dB, float* db, void* dH, int64_t T, int64_t h, int64_t F,
                                int p, tpmlp_dtype dt, void* stream);

/* Size in bytes of the fixed scratch array tp_mlp_bwd_noalloc uses. */
size_t tpmlp_noalloc_scratch_bytes(void);

/* Diagnostic, host only (launches nothing): the work units the tensor-core
 * GEMM kernels run for an output of m_blocks × n_blocks tiles and k_blocks
 * 64-deep k-blocks on `workers` CTA pairs (or single CTAs), under schedule
 * `sched`: 0 whole tiles; 1 every tile cut into `groups` equal consecutive
 * k ranges (one per shard group of a row-parallel product); 2 whole tiles
 * in full waves, then the remaining tiles' k-blocks cut into one equal
 * segment per worker (a stream-K tail). Writes up to max_units records of
 * 10 int64 to `out`, in each worker's order: worker, its unit index, m
 * block, n block, first k-block, end k-block, units sharing the tile,
 * this unit's place among them (ascending k), the tile's counter index and
 * this unit's partial-tile slot (both -1 for a whole tile). Returns the
 * total number of units (which may exceed max_units), or -1 for arguments
 * the kernels would not run with (a stream-K tail needs tiles not a
 * multiple of workers and at least 4 k-blocks per segment; shard groups
 * need k_blocks divisible by groups). */
int64_t tpmlp_schedule_units(int sched, int m_blocks, int n_blocks, int k_blocks, int groups,
                             int workers, int64_t* out, int64_t max_units);

/* Diagnostic, host only: the schedule (0 whole tiles, 1 shard groups,
 * 2 stream-K tail; as tpmlp_schedule_units) that tp_mlp_fwd / tp_mlp_bwd
 * plan for each of the block's six products, in the order F1 (X·A),
 * F2 (Σ Y_i·B_i), B2 (dZ·Bᵀ), B3 (Yᵀ·dZ), B4 (Xᵀ·dH), B5 (Σ dH_i·A_iᵀ),
 * under the current split policy, on the current device (148 SMs when no
 * device is present). Writes 6 ints to `kinds`. */
tpmlp_status tpmlp_plan_schedules(int64_t T, int64_t h, int64_t F, int p, tpmlp_dtype dt, int* kinds);

/* Diagnostic, host only: for the same six products in the same order,
 * whether each runs the dynamic tile schedule (1) or a static one (0), under
 * the current split policy and tpmlp_set_dynamic_schedule setting, on the
 * current device (148 SMs when no device is present). Writes 6 ints to
 * `dyn`. */
tpmlp_status tpmlp_plan_dynamic(int64_t T, int64_t h, int64_t F, int p, tpmlp_dtype dt, int* dyn);

/* Library version, major·10000 + minor·100 + patch. */
int tpmlp_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TPMLP_H */
