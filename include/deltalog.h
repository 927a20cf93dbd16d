/*
 * deltalog.h -- C ABI of a B200 (sm_100a) library for the batched recurrent-state
 * decode step of linear-attention models, executed base + log ("DeltaLog").
 *
 * Passages this interface follows (DeltaLog: Deferred Materialization of
 * Recurrent States for Linear Attention Decoding, Lin, Sun, Sun):
 *  - Background, Eq. 3 (the common decode form): per slot, layer and head,
 *        S_t = Diag(exp(lambda_t)) S_{t-1} + a_t b_t^T,   o_t = S_t^T q_t,
 *    with a_t = k_t; b_t = v_t for additive operators (linear attention, RetNet,
 *    GLA, RWKV6) and b_t = beta_t (v_t - Shat^T k_t) for delta-rule operators
 *    (DeltaNet, GDN, KDA), Shat = Diag(exp(lambda_t)) S_{t-1} by default.
 *    Scalar decay shares one lambda over all d_k coordinates; diagonal decay
 *    uses a per-key vector.
 *  - Section 3 (append-merge cycle, Algorithm 1): append steps record the
 *    compact factors in a bounded log and leave the dense base untouched; every
 *    merge interval the log is folded into the base and cleared.
 *  - Section 3 (physical state): dense fp32 base state, cumulative log-decay,
 *    key/value log buffers, one log-decay snapshot per entry, live-log length.
 *  - Section 3 (traffic model, logical state): the base plus the log represents
 *        S = D(lbar) Sbar + sum_{i<live} D(lbar - Lambda_i) a_i b_i^T,
 *    D(x) = Diag(exp(x)), at every step.
 *  - Section 3.3 (GPU execution): value-tiled work units over (slot, head,
 *    value tile); key-side replay coefficients q^T a_i and k^T a_i with the
 *    row rescaling D(lbar - Lambda_i); a single owner commits the shared log
 *    metadata; Merge rewrites each dense fp32 tile once.
 *  - Section 4 (serving integration): prefill initialises the base; a fresh or
 *    reused slot starts with an empty log.
 *
 * Memory.  The library allocates no device memory.  Every buffer below is
 * caller-owned device memory (for example torch tensors) and must stay alive
 * while a pool that names it is in use.  All float buffers are fp32, row-major,
 * 16-byte aligned.
 *
 * Streams.  Every call is asynchronous on the given cudaStream_t (passed as
 * void*, NULL = legacy default stream) except dl_read_error, which
 * synchronises that stream.  Calls on the same (pool, layer) must be ordered
 * on one stream; different layers may run concurrently.  The whole-head decode
 * kernel is launched with programmatic stream serialization: it may start while
 * the previous kernel on its stream finishes, and reads no global memory before
 * that kernel has completed.  Each of its CTAs (one per SM) holds all of that SM's
 * tensor memory while it runs, so a kernel on another stream that holds tensor
 * memory on the same SM delays it until those columns are released.
 *
 * Errors.  Argument problems found on the host are returned as a dl_status
 * before anything is launched.  Problems only the device can see (a slot id out
 * of range, a full log, a corrupt log length, an eager step on a slot with a
 * live log) set a bit in the pool's sticky device error word and the affected
 * work item is skipped; nothing traps.  Read the word with dl_read_error.
 */
#ifndef DELTALOG_H
#define DELTALOG_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DL_OK = 0,
    DL_ERR_INVALID_ARG = 1,  /* null pointer, bad enum, misaligned buffer, bad layer */
    DL_ERR_SHAPE = 2,        /* dimension outside the supported set               */
    DL_ERR_DTYPE = 3,        /* input dtype not supported                         */
    DL_ERR_UNSUPPORTED = 4,  /* operation needs a log but the pool has none       */
    DL_ERR_CUDA = 5,         /* a CUDA runtime call or a launch failed            */
    DL_ERR_DEVICE = 6        /* dl_read_error found device error bits set         */
} dl_status;

/* Decay granularity of lambda_t (Background, Table 1 as restated in the text). */
typedef enum {
    DL_DECAY_NONE = 0,    /* lambda = 0: linear attention, DeltaNet                 */
    DL_DECAY_SCALAR = 1,  /* one value per head: RetNet, GDN                        */
    DL_DECAY_DIAG = 2     /* one value per key coordinate: GLA, RWKV6, KDA          */
} dl_decay;

/* Update semantics: how b_t is formed (Background; Section 3.4 per operator). */
typedef enum {
    DL_UPDATE_ADD = 0,             /* b_t = v_t                                        */
    DL_UPDATE_DELTA = 1,           /* b_t = beta_t (v_t - (Diag(exp lambda_t) S_{t-1})^T k_t) */
    DL_UPDATE_DELTA_UNDECAYED = 2  /* b_t = beta_t (v_t - S_{t-1}^T k_t)               */
} dl_update;

typedef enum { DL_F32 = 0, DL_BF16 = 1 } dl_dtype;

/* Log entry layout.  The deferred log is that of the Design section; the narrower
 * factor storage follows the per-operator instantiations of Section 3.4, which keep
 * a_t in 16-bit storage (GDN, KDA), b_t in FP32 under the delta rule and both
 * factors in BF16 for RWKV6, with the decay metadata in FP32.
 *  DL_LOG_FP32     [a_i | b_i | Lambda_i] in fp32, 2*d_k + d_v floats per entry.
 *  DL_LOG_COMPACT  [a_i bf16 x d_k | b_i | Lambda_i], where b_i is bf16 x d_v under
 *                  DL_UPDATE_ADD and fp32 x d_v under the delta rule, and Lambda_i is
 *                  fp32 x d_k (per-key decay), fp32 x 4 (scalar decay: Lambda_0 and 3
 *                  pad floats) or absent (no decay).  a_t = k_t and, without the delta
 *                  rule, b_t = v_t are bf16 inputs, so the narrower storage is exact:
 *                  a compact pool computes the same values as an fp32 one while moving
 *                  17-50% fewer log bytes.  Decode and append steps on a compact pool
 *                  require in_dtype == DL_BF16 (else DL_ERR_DTYPE).
 * dl_log_bytes gives the size of the log buffer either layout needs. */
typedef enum { DL_LOG_FP32 = 0, DL_LOG_COMPACT = 1 } dl_log_format;

/* Where the value-tiled kernel forms the key-side replay coefficients (ReplayPrep,
 * Section 3.3: q^T A'_i and k^T A'_i, with A'_i for a merge).  The whole-head kernel
 * (tile_v 128) always forms them once per head, in the head's warp.
 *  DL_REPLAY_PER_TILE  every value tile forms all of them itself (default; the fused,
 *                      redundant form).
 *  DL_REPLAY_CLUSTER   the d_v / B_V tiles of a head run as one thread-block cluster
 *                      (when that is 2..8 CTAs); each tile forms a share of the entries
 *                      and reads the rest from the others' shared memory.
 * Measured on B200 the cluster form is slower for most launches (co-scheduling the
 * cluster and its two barriers cost more than the redundant replay) and faster only
 * for the smallest launches with long logs; it is kept for that case and for the
 * ablation of Section 3.3's staged ReplayPrep. */
typedef enum { DL_REPLAY_PER_TILE = 0, DL_REPLAY_CLUSTER = 1 } dl_replay_mode;

/* Sticky device error bits (dl_read_error). */
#define DL_EBIT_SLOT_RANGE 0x1  /* a slot id outside [0, n_slots)                    */
#define DL_EBIT_LOG_FULL 0x2    /* append / decode without auto-merge on a full log   */
#define DL_EBIT_LIVE_LOG 0x4    /* eager step on a slot whose log is not empty        */
#define DL_EBIT_LOG_LEN 0x8     /* a stored live-log length outside [0, log_cap]     */
#define DL_EBIT_TIMEOUT 0x10    /* a pipeline wait inside a kernel ran out of time and
                                   the kernel abandoned the call (a library fault)    */

/* Pool descriptor.  One pool covers n_slots request slots x n_layers
 * linear-attention layers x n_heads value heads.
 *
 *  d_k in {16, 64, 128}; d_v a multiple of 16 in [16, 1024];
 *  n_kheads divides n_heads (grouped value attention: v-head h reads the q/k of
 *  k-head h / (n_heads / n_kheads));  1 <= log_cap <= 64.
 *
 *  state    [n_slots][n_layers][n_heads][d_k][d_v]  fp32 dense base state.  The
 *           caller writes prefill states here, then resets the slot's log.
 *  log      [n_slots][n_layers][n_heads][log_cap][entry] ring, 16-byte aligned.  Row i
 *           holds entry i.  With log_format DL_LOG_FP32 an entry is
 *           [a_i (d_k) | b_i (d_v) | Lambda_i (d_k)] fp32; scalar decay uses
 *           Lambda_i[0] only; no decay leaves Lambda unused.  DL_LOG_COMPACT is
 *           described at dl_log_format.  NULL makes an eager-only pool
 *           (decode/append/merge/materialize then return DL_ERR_UNSUPPORTED).
 *  log_len  [n_slots][n_layers] int32 live-log length (entries 0..log_len-1 live).
 *           Required with a log; optional (NULL) for an eager-only pool.
 *  arrive   [n_slots][n_layers] int32 arrival counters used to commit log_len once
 *           per call.  Must be zero when the pool is created; the library returns
 *           them to zero at the end of every call.  Required with a log.
 *  err_word [1] int32 sticky device error bits; zero it before first use.
 *  tile_v   value-tile width B_V of a work unit (Section 3.3): 16 or 32 columns;
 *           128 for whole-head work units, each owned by one warp of the
 *           warp-per-head decode kernel (needs d_k = d_v = 128; it serves decode
 *           and eager steps whose q, k, v, per-key lambda and out are 16-byte
 *           aligned, and other calls of such a pool use 16/32-wide tiles); 0 to
 *           choose per launch (whole heads for decode steps when those conditions
 *           hold and there are at least as many heads as SMs, else 32 columns
 *           unless that leaves SMs idle, else 16).  32 needs d_k >= 64 and d_v a
 *           multiple of 32.
 *  log_format dl_log_format of the log (DL_LOG_FP32 or DL_LOG_COMPACT).
 *  replay_mode dl_replay_mode (DL_REPLAY_PER_TILE or DL_REPLAY_CLUSTER).
 *
 * The cumulative log-decay lbar of a slot is not stored separately: it equals
 * Lambda of the newest live entry (0 when the log is empty).
 */
typedef struct {
    int32_t n_slots, n_layers, n_heads, n_kheads, d_k, d_v, log_cap;
    dl_decay decay;
    dl_update update;
    int32_t tile_v;
    int32_t log_format;   /* dl_log_format */
    int32_t replay_mode;  /* dl_replay_mode */
    float *state;
    float *log;
    int32_t *log_len;
    int32_t *arrive;
    int32_t *err_word;
} dl_pool_desc;

typedef struct dl_pool dl_pool;  /* opaque host-side handle */

/* Inputs of one decode step of one layer for a batch of slots.
 *  slots   device [batch] int32 slot ids, distinct within one call.  Row b of
 *          every per-row tensor below belongs to slot slots[b].
 *  q, k    device [batch][n_kheads][d_k] (in_dtype).  k is the key factor a_t.
 *  v       device [batch][n_heads][d_v] (in_dtype).
 *  lambda  fp32 log-decay (<= 0 for a decaying state):
 *            lambda_per_head == 0: [batch][n_heads] (scalar) | [batch][n_heads][d_k] (diag)
 *            lambda_per_head == 1: [n_heads] (scalar) | [n_heads][d_k] (diag), the
 *                                  same for every row and step (RetNet)
 *          NULL iff decay == DL_DECAY_NONE.
 *  beta    device [batch][n_heads] fp32, delta rule only (else ignored).
 *  out     device [batch][n_heads][d_v] fp32 output o_t.  Ignored by dl_append.
 */
typedef struct {
    const int32_t *slots;
    int32_t batch;
    const void *q, *k, *v;
    dl_dtype in_dtype;
    const float *lambda;
    int32_t lambda_per_head;
    const float *beta;
    float *out;
} dl_step_args;

/* Bytes of the log buffer a descriptor needs: n_slots * n_layers * n_heads *
 * log_cap entries of the layout its log_format, decay and update select (every
 * entry a multiple of 16 bytes).  Reads only the shape fields and log_format;
 * DL_ERR_SHAPE / DL_ERR_INVALID_ARG as dl_create_pool for those.  No CUDA call. */
dl_status dl_log_bytes(const dl_pool_desc *desc, int64_t *bytes);

/* Validate a descriptor and return a host handle recording it.  No device
 * memory is allocated and no CUDA call is made. */
dl_status dl_create_pool(const dl_pool_desc *desc, dl_pool **out_pool);
dl_status dl_destroy_pool(dl_pool *pool);

/* Merge policy of dl_decode_step (its auto_merge argument). */
#define DL_MERGE_NONE 0         /* never merge; a full log is an error                  */
#define DL_MERGE_AT_CAPACITY 1  /* merge on the slot's log_cap-th step (any other
                                   non-zero value except DL_MERGE_ADAPTIVE means this)  */
#define DL_MERGE_ADAPTIVE 2     /* as DL_MERGE_AT_CAPACITY, except that a launch too
                                   small to fill the GPU merges every slot on every step */

/* One decode step (Section 3.3, AppendDecode + Finalize, and the merge step of
 * the append-merge cycle).  For each slot with c live entries:
 *   c < log_cap - 1, or auto_merge == DL_MERGE_NONE and c < log_cap:
 *       read o_t and, for the delta rule, the correction (Shat^T k_t) off the
 *       read-only base plus the decayed log; append (k_t, b_t, lbar + lambda_t)
 *       as entry c; live length c + 1.
 *   auto_merge != DL_MERGE_NONE and c >= log_cap - 1 (the slot's merge step):
 *       compute o_t the same way and write the fully materialised state S_t
 *       (base, log and the token) to the base; live length 0.
 *   auto_merge == DL_MERGE_NONE and c == log_cap: DL_EBIT_LOG_FULL, slot skipped.
 * So with auto_merge the merge interval equals log_cap, and log_cap == 1 is
 * the eager recurrence.
 *
 * DL_MERGE_ADAPTIVE: when batch * n_heads is below a few heads per SM of the
 * current device (dl_merge_policy tells), the launch is latency-bound: its time
 * is one head's chain of dependent loads plus, on a merge step, that head's
 * write-back, not the bytes it moves.  Every slot of such a launch then takes the
 * merge step (folding whatever its log holds), so after the first such step the
 * launch is the eager recurrence with an empty log, run by the value-tiled kernel.
 * The outputs and logical states are the same under every policy (the
 * logical-state equation); only the split between base and log differs. */
dl_status dl_decode_step(dl_pool *pool, int32_t layer, const dl_step_args *args,
                         int32_t auto_merge, void *stream);

/* Whether dl_decode_step with this batch, head count and auto_merge value merges
 * every slot on every step (*merges_every_step = 1) on the current device.
 * DL_ERR_INVALID_ARG for a NULL output, batch < 0 or n_heads <= 0.  Reads the
 * device's SM count (148 when no device is visible). */
dl_status dl_merge_policy(int32_t batch, int32_t n_heads, int32_t auto_merge,
                          int32_t *merges_every_step);

/* Append the step's factors only (no output, never merges).  For the delta rule
 * the base is still read to form b_t.  A full log sets DL_EBIT_LOG_FULL. */
dl_status dl_append(dl_pool *pool, int32_t layer, const dl_step_args *args, void *stream);

/* Merge (Section 3.3): for each listed slot fold its live log into the base,
 *   Sbar <- D(lbar) Sbar + sum_i D(lbar - Lambda_i) a_i b_i^T,
 * one read-modify-write pass per value tile, then reset the live length. */
dl_status dl_merge(dl_pool *pool, int32_t layer, const int32_t *slots, int32_t batch,
                   void *stream);

/* Eager dense step (Background: one read-modify-write of the full state per
 * token), the in-library comparison path.  Requires an empty log on every
 * listed slot (else DL_EBIT_LIVE_LOG and the slot is skipped). */
dl_status dl_eager_step(dl_pool *pool, int32_t layer, const dl_step_args *args, void *stream);

/* Empty the logs of the listed slots on every layer (Section 4: a fresh or
 * reused slot starts with an empty auxiliary representation; the base, which
 * prefill writes, is left alone). */
dl_status dl_reset_slots(dl_pool *pool, const int32_t *slots, int32_t batch, void *stream);

/* Write the logical state of the listed slots (logical-state equation) to
 * dense_out [batch][n_heads][d_k][d_v] fp32 (device); the pool is unchanged. */
dl_status dl_materialize(dl_pool *pool, int32_t layer, const int32_t *slots, int32_t batch,
                         float *dense_out, void *stream);

/* Synchronise `stream`, copy the device error word to *bits, and, when `clear` is
 * non-zero, clear the bits just read (an atomic AND on the device, ordered on
 * `stream`, then a second synchronisation): a bit that a kernel on another stream
 * sets between the copy and the clear stays set for the next read.  Returns
 * DL_ERR_DEVICE when any bit was set.
 *
 * After any bit is reported, prefill and reset (dl_reset_slots) the affected slots
 * before their next step.  A skipped work item leaves its slot as it was, but a
 * kernel that abandoned a call (DL_EBIT_TIMEOUT) can leave a slot's base, log and
 * arrival counters part-way through the step. */
dl_status dl_read_error(dl_pool *pool, int32_t *bits, int32_t clear, void *stream);

/* Fault injection for tests (the paper has no counterpart).  While limit_ns > 0
 * (process-wide, for launches issued after the call), every launch of the
 * whole-head decode kernel makes the first warp of its first CTA wait, bounded by
 * limit_ns, on a barrier that nothing completes, before that warp consumes any of
 * the bulk copies it has already issued.  The wait runs out: the kernel sets
 * DL_EBIT_TIMEOUT, the warp stops, waits with the normal 100 ms bound for its own
 * copies still in flight, the CTA frees its tensor memory and returns, and the
 * context stays usable.  The heads of that warp are left unprocessed, so the
 * call's slots must be prefilled and reset afterwards (see dl_read_error).
 * limit_ns <= 0 switches it off.  Always DL_OK; makes no CUDA call. */
dl_status dl_debug_stall(int64_t limit_ns);

/* Decode step that allocates nothing.  The paper has no counterpart: this entry
 * point exists for integration only.
 *
 * Who needs it.  dl_decode_step needs one small buffer besides the state, the
 * log and the step's inputs and outputs: the per-(slot, layer) arrival counters
 * (pool `arrive`) that let the last work unit of a slot commit its new live-log
 * length.  Some callers cannot provide even that.  One example is a serving engine
 * whose memory manager has already divided the whole device among its own pools
 * and refuses further cudaMalloc calls.  Another is a host runtime that reaches the
 * GPU only through buffers it was handed at start-up.  This call keeps the
 * counters in a fixed array compiled into the library instead, so such a caller
 * passes only memory it already owns.
 *
 * Arguments and results are those of dl_decode_step, except that the pool is a
 * descriptor (checked on every call with the rules of dl_create_pool; no handle
 * is made) and its `arrive` field is ignored and may be NULL.  The descriptor must
 * name a log.
 *
 * Limits and sharing:
 *  - n_slots * n_layers <= DL_NOALLOC_MAX_COUNTERS, else DL_ERR_SHAPE.  The array
 *    (DL_NOALLOC_MAX_COUNTERS int32, 256 KiB) occupies every GPU that loads the
 *    library until the process exits.
 *  - All calls share that one array.  Each call first clears the counters it uses
 *    (an asynchronous memset on `stream`), so calls that overlap on the GPU (two
 *    streams, or two host threads) race; issue them in order on one stream.
 *  - Every call looks up the array's address in the current device's context
 *    (cudaGetSymbolAddress; nothing is cached between calls).  The first lookup on
 *    a device can load the module, so make the first call on each device before
 *    any stream capture.
 *  - It calls no cudaMalloc, cudaFree or other allocating routine. */
#define DL_NOALLOC_MAX_COUNTERS 65536
dl_status dl_decode_step_noalloc(const dl_pool_desc *desc, int32_t layer,
                                 const dl_step_args *args, int32_t auto_merge, void *stream);

/* Static description of a status code. */
const char *dl_status_string(dl_status status);

#ifdef __cplusplus
}
#endif
#endif /* DELTALOG_H */
