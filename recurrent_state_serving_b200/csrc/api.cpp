// C ABI of the base + log recurrent-state decode library: argument validation,
// launch-shape selection and error reporting.  The arithmetic lives in the
// kernels (dl_kernels.cuh); nothing here computes on the host.
#include <atomic>
#include <cstdint>
#include <cstring>
#include <new>

#include <cuda_runtime.h>

#include "deltalog.h"
#include "dl_internal.h"

#define DL_API extern "C" __attribute__((visibility("default")))

struct dl_pool {
    dl_pool_desc d;
};

namespace {

std::atomic<unsigned long long> g_stall_ns{0};

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool dk_supported(int dk) { return dk == 16 || dk == 64 || dk == 128; }

// Log entry layout of a descriptor (dl_log_format in deltalog.h), in floats.
struct LogLayout {
    int E, boff, loff, a16, b16;
};
LogLayout log_layout(const dl_pool_desc &d) {
    LogLayout l;
    if (d.log_format == DL_LOG_COMPACT) {
        l.a16 = 1;
        l.b16 = d.update == DL_UPDATE_ADD ? 1 : 0;
        l.boff = d.d_k / 2;
        l.loff = l.boff + (l.b16 ? d.d_v / 2 : d.d_v);
        l.E = l.loff + (d.decay == DL_DECAY_DIAG ? d.d_k : d.decay == DL_DECAY_SCALAR ? 4 : 0);
    } else {
        l.a16 = l.b16 = 0;
        l.boff = d.d_k;
        l.loff = d.d_k + d.d_v;
        l.E = 2 * d.d_k + d.d_v;
    }
    return l;
}

dl::KParams base_params(const dl_pool_desc &d, int layer) {
    dl::KParams p;
    std::memset(&p, 0, sizeof(p));
    p.state = d.state;
    p.log = d.log;
    p.log_len = d.log_len;
    p.arrive = d.arrive;
    p.err = d.err_word;
    p.n_slots = d.n_slots;
    p.n_layers = d.n_layers;
    p.H = d.n_heads;
    p.Hk = d.n_kheads;
    p.dk = d.d_k;
    p.dv = d.d_v;
    p.L = d.log_cap;
    const LogLayout l = log_layout(d);
    p.E = l.E;
    p.boff = l.boff;
    p.loff = l.loff;
    p.a16 = l.a16;
    p.b16 = l.b16;
    p.layer = layer;
    p.cl = 1;
    p.stall_ns = dl::stall_ns();
    return p;
}

void set_tiles(const dl_pool_desc &d, dl::KParams &p, int batch, int &bv) {
    bv = (d.tile_v == 16 || d.tile_v == 32) ? d.tile_v
                                           : dl::pick_bv(p.dk, p.dv, (long long)batch * p.H * (p.dv / 32));
    p.nv = p.dv / bv;
}

// Whole-head work units (warp-per-head kernel) for a decode or eager step?  That
// kernel streams token rows and writes outputs with 128-bit accesses, so it needs
// 16-byte aligned q, k, v, per-key lambda and out; calls whose buffers are only
// element-aligned run the value-tiled kernel.
bool use_whole_head(const dl_pool_desc &d, const dl_step_args *a, bool want_out, bool rewrites_all) {
    if (!want_out || !dl::whole_head_supported(d.d_k, d.d_v)) return false;
    if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->v, 16) || !aligned(a->out, 16))
        return false;
    if (d.decay == DL_DECAY_DIAG && !aligned(a->lambda, 16)) return false;
    if (d.tile_v == 128) return true;
    if (d.tile_v != 0) return false;
    // A step that rewrites every head (eager, or merging every slot) goes to the
    // value-tiled kernel, which keeps its tile in registers between the read and
    // the write and measured faster for it.
    if (rewrites_all) return false;
    return (long long)a->batch * d.n_heads >= (long long)dl::device_sm_count();
}

dl_status check_step(const dl_pool *P, int32_t layer, const dl_step_args *a, bool need_out,
                     bool uses_log) {
    if (!P || !a) return DL_ERR_INVALID_ARG;
    const dl_pool_desc &d = P->d;
    if (layer < 0 || layer >= d.n_layers) return DL_ERR_INVALID_ARG;
    if (a->batch < 0) return DL_ERR_SHAPE;
    if (a->batch == 0) return DL_OK;
    if (a->batch > d.n_slots) return DL_ERR_SHAPE;
    if (!a->slots || !a->q || !a->k || !a->v) return DL_ERR_INVALID_ARG;
    if (a->in_dtype != DL_F32 && a->in_dtype != DL_BF16) return DL_ERR_DTYPE;
    // the compact log stores a_t = k_t (and b_t = v_t) in bf16: exact only for bf16 inputs
    if (uses_log && d.log_format == DL_LOG_COMPACT && a->in_dtype != DL_BF16) return DL_ERR_DTYPE;
    const uintptr_t esz = a->in_dtype == DL_F32 ? 4 : 2;
    if (!aligned(a->q, esz) || !aligned(a->k, esz) || !aligned(a->v, esz)) return DL_ERR_INVALID_ARG;
    if (d.decay != DL_DECAY_NONE && (!a->lambda || !aligned(a->lambda, 4))) return DL_ERR_INVALID_ARG;
    if (a->lambda_per_head != 0 && a->lambda_per_head != 1) return DL_ERR_INVALID_ARG;
    if (d.update != DL_UPDATE_ADD && (!a->beta || !aligned(a->beta, 4))) return DL_ERR_INVALID_ARG;
    if (need_out && (!a->out || !aligned(a->out, 4))) return DL_ERR_INVALID_ARG;
    if (!aligned(a->slots, 4)) return DL_ERR_INVALID_ARG;
    return DL_OK;
}

dl_status run_step(dl_pool *P, int32_t layer, const dl_step_args *a, bool want_out,
                   int32_t auto_merge, bool eager, void *stream) {
    const dl_pool_desc &d = P->d;
    dl::KParams p = base_params(d, layer);
    p.slots = a->slots;
    p.batch = a->batch;
    p.q = a->q;
    p.k = a->k;
    p.v = a->v;
    p.lam = d.decay == DL_DECAY_NONE ? nullptr : a->lambda;
    p.lam_const = a->lambda_per_head;
    p.beta = d.update == DL_UPDATE_ADD ? nullptr : a->beta;
    p.out = want_out ? a->out : nullptr;
    p.auto_merge = auto_merge ? 1 : 0;
    p.merge_every = (!eager && auto_merge == DL_MERGE_ADAPTIVE &&
                     dl::adaptive_merges_every_step(a->batch, d.n_heads)) ? 1 : 0;
    p.eager = eager ? 1 : 0;
    p.want_out = want_out ? 1 : 0;
    p.undecayed = d.update == DL_UPDATE_DELTA_UNDECAYED ? 1 : 0;
    cudaError_t e;
    if (use_whole_head(d, a, want_out, eager || p.merge_every)) {
        p.nv = 1;
        e = dl::launch_whole_head(p, d.decay, d.update != DL_UPDATE_ADD, a->in_dtype == DL_BF16,
                                  static_cast<cudaStream_t>(stream));
    } else {
        int bv = 32;
        set_tiles(d, p, a->batch, bv);
        // ReplayPrep shared by the head's value tiles as one cluster (2..8 CTAs); an
        // eager step has no log to replay
        p.cl = (d.replay_mode == DL_REPLAY_CLUSTER && !eager && p.nv >= 2 && p.nv <= 8) ? p.nv : 1;
        e = dl::launch_step(p, bv, d.decay, d.update != DL_UPDATE_ADD, a->in_dtype == DL_BF16,
                            static_cast<cudaStream_t>(stream));
    }
    return e == cudaSuccess ? DL_OK : DL_ERR_CUDA;
}

}  // namespace

DL_API dl_status dl_log_bytes(const dl_pool_desc *desc, int64_t *bytes) {
    if (!desc || !bytes) return DL_ERR_INVALID_ARG;
    const dl_pool_desc &d = *desc;
    if (d.n_slots <= 0 || d.n_layers <= 0 || d.n_heads <= 0) return DL_ERR_SHAPE;
    if (!dk_supported(d.d_k) || d.d_v < 16 || d.d_v > 1024 || d.d_v % 16) return DL_ERR_SHAPE;
    if (d.log_cap < 1 || d.log_cap > 64) return DL_ERR_SHAPE;
    if ((int)d.decay < DL_DECAY_NONE || (int)d.decay > DL_DECAY_DIAG) return DL_ERR_INVALID_ARG;
    if ((int)d.update < DL_UPDATE_ADD || (int)d.update > DL_UPDATE_DELTA_UNDECAYED)
        return DL_ERR_INVALID_ARG;
    if (d.log_format != DL_LOG_FP32 && d.log_format != DL_LOG_COMPACT) return DL_ERR_INVALID_ARG;
    *bytes = (int64_t)d.n_slots * d.n_layers * d.n_heads * d.log_cap * log_layout(d).E * 4;
    return DL_OK;
}

DL_API dl_status dl_create_pool(const dl_pool_desc *desc, dl_pool **out_pool) {
    if (!desc || !out_pool) return DL_ERR_INVALID_ARG;
    *out_pool = nullptr;
    const dl_pool_desc &d = *desc;
    if (d.n_slots <= 0 || d.n_layers <= 0 || d.n_heads <= 0 || d.n_kheads <= 0)
        return DL_ERR_SHAPE;
    if (d.n_heads % d.n_kheads) return DL_ERR_SHAPE;
    if (!dk_supported(d.d_k)) return DL_ERR_SHAPE;
    if (d.d_v < 16 || d.d_v > 1024 || d.d_v % 16) return DL_ERR_SHAPE;
    if (d.log_cap < 1 || d.log_cap > 64) return DL_ERR_SHAPE;
    if (d.tile_v != 0 && d.tile_v != 16 && d.tile_v != 32 && d.tile_v != 128) return DL_ERR_SHAPE;
    if (d.tile_v == 32 && (d.d_k < 64 || d.d_v % 32)) return DL_ERR_SHAPE;
    if (d.tile_v == 128 && !dl::whole_head_supported(d.d_k, d.d_v)) return DL_ERR_SHAPE;
    if ((int)d.decay < DL_DECAY_NONE || (int)d.decay > DL_DECAY_DIAG) return DL_ERR_INVALID_ARG;
    if ((int)d.update < DL_UPDATE_ADD || (int)d.update > DL_UPDATE_DELTA_UNDECAYED)
        return DL_ERR_INVALID_ARG;
    if (d.log_format != DL_LOG_FP32 && d.log_format != DL_LOG_COMPACT) return DL_ERR_INVALID_ARG;
    if (d.replay_mode != DL_REPLAY_PER_TILE && d.replay_mode != DL_REPLAY_CLUSTER) return DL_ERR_INVALID_ARG;
    if (!d.state || !aligned(d.state, 16) || !d.err_word || !aligned(d.err_word, 4))
        return DL_ERR_INVALID_ARG;
    if (d.log && (!aligned(d.log, 16) || !d.log_len || !d.arrive)) return DL_ERR_INVALID_ARG;
    if ((d.log_len && !aligned(d.log_len, 4)) || (d.arrive && !aligned(d.arrive, 4)))
        return DL_ERR_INVALID_ARG;
    // launch grids are one CTA per (row, head, 16-column tile)
    if ((long long)d.n_slots * d.n_heads * (d.d_v / 16) > 0x7fffffffLL) return DL_ERR_SHAPE;
    dl_pool *p = new (std::nothrow) dl_pool;
    if (!p) return DL_ERR_INVALID_ARG;
    p->d = d;
    *out_pool = p;
    return DL_OK;
}

DL_API dl_status dl_destroy_pool(dl_pool *pool) {
    if (!pool) return DL_ERR_INVALID_ARG;
    delete pool;
    return DL_OK;
}

DL_API dl_status dl_decode_step(dl_pool *pool, int32_t layer, const dl_step_args *args,
                                int32_t auto_merge, void *stream) {
    const dl_status s = check_step(pool, layer, args, true, true);
    if (s != DL_OK || args->batch == 0) return s;
    if (!pool->d.log) return DL_ERR_UNSUPPORTED;
    return run_step(pool, layer, args, true, auto_merge, false, stream);
}

DL_API dl_status dl_append(dl_pool *pool, int32_t layer, const dl_step_args *args, void *stream) {
    const dl_status s = check_step(pool, layer, args, false, true);
    if (s != DL_OK || args->batch == 0) return s;
    if (!pool->d.log) return DL_ERR_UNSUPPORTED;
    return run_step(pool, layer, args, false, DL_MERGE_NONE, false, stream);
}

DL_API dl_status dl_eager_step(dl_pool *pool, int32_t layer, const dl_step_args *args,
                               void *stream) {
    const dl_status s = check_step(pool, layer, args, true, false);
    if (s != DL_OK || args->batch == 0) return s;
    return run_step(pool, layer, args, true, DL_MERGE_NONE, true, stream);
}

static dl_status merge_like(dl_pool *pool, int32_t layer, const int32_t *slots, int32_t batch,
                            float *dense_out, bool materialize, void *stream) {
    if (!pool) return DL_ERR_INVALID_ARG;
    const dl_pool_desc &d = pool->d;
    if (layer < 0 || layer >= d.n_layers) return DL_ERR_INVALID_ARG;
    if (batch < 0 || batch > d.n_slots) return DL_ERR_SHAPE;
    if (batch == 0) return DL_OK;
    if (!slots || !aligned(slots, 4)) return DL_ERR_INVALID_ARG;
    if (materialize && (!dense_out || !aligned(dense_out, 16))) return DL_ERR_INVALID_ARG;
    if (!d.log) return DL_ERR_UNSUPPORTED;
    dl::KParams p = base_params(d, layer);
    p.slots = slots;
    p.batch = batch;
    p.dense_out = dense_out;
    cudaError_t e;
    if (dl::whole_head_supported(d.d_k, d.d_v) && d.tile_v != 16 && d.tile_v != 32) {
        e = dl::launch_merge_head(p, d.decay, materialize, static_cast<cudaStream_t>(stream));
    } else {
        int bv = 32;
        set_tiles(d, p, batch, bv);
        e = dl::launch_merge(p, bv, d.decay, materialize, static_cast<cudaStream_t>(stream));
    }
    return e == cudaSuccess ? DL_OK : DL_ERR_CUDA;
}

DL_API dl_status dl_merge(dl_pool *pool, int32_t layer, const int32_t *slots, int32_t batch,
                          void *stream) {
    return merge_like(pool, layer, slots, batch, nullptr, false, stream);
}

DL_API dl_status dl_materialize(dl_pool *pool, int32_t layer, const int32_t *slots,
                                int32_t batch, float *dense_out, void *stream) {
    return merge_like(pool, layer, slots, batch, dense_out, true, stream);
}

DL_API dl_status dl_reset_slots(dl_pool *pool, const int32_t *slots, int32_t batch,
                                void *stream) {
    if (!pool) return DL_ERR_INVALID_ARG;
    const dl_pool_desc &d = pool->d;
    if (batch < 0 || batch > d.n_slots) return DL_ERR_SHAPE;
    if (batch == 0) return DL_OK;
    if (!slots || !aligned(slots, 4)) return DL_ERR_INVALID_ARG;
    if (!d.log_len) return DL_OK;  // eager-only pool without a log: nothing to reset
    const cudaError_t e = dl::launch_reset(slots, batch, d.n_slots, d.n_layers, d.log_len,
                                           d.arrive, d.err_word,
                                           static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DL_OK : DL_ERR_CUDA;
}

DL_API dl_status dl_read_error(dl_pool *pool, int32_t *bits, int32_t clear, void *stream) {
    if (!pool || !bits) return DL_ERR_INVALID_ARG;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t host = 0;
    if (cudaMemcpyAsync(&host, pool->d.err_word, sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
        cudaSuccess)
        return DL_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DL_ERR_CUDA;
    if (clear && host) {
        // clear only the bits just read, atomically: a bit another stream's kernel
        // sets in the meantime stays set for the next read
        if (dl::launch_clear_bits(pool->d.err_word, host, st) != cudaSuccess) return DL_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return DL_ERR_CUDA;
    }
    *bits = host;
    return host ? DL_ERR_DEVICE : DL_OK;
}

DL_API dl_status dl_merge_policy(int32_t batch, int32_t n_heads, int32_t auto_merge,
                                 int32_t *merges_every_step) {
    if (!merges_every_step || batch < 0 || n_heads <= 0) return DL_ERR_INVALID_ARG;
    *merges_every_step = (auto_merge == DL_MERGE_ADAPTIVE && batch > 0 &&
                          dl::adaptive_merges_every_step(batch, n_heads)) ? 1 : 0;
    return DL_OK;
}

DL_API dl_status dl_debug_stall(int64_t limit_ns) {
    g_stall_ns.store(limit_ns > 0 ? (unsigned long long)limit_ns : 0ull);
    return DL_OK;
}

DL_API const char *dl_status_string(dl_status status) {
    switch (status) {
    case DL_OK: return "ok";
    case DL_ERR_INVALID_ARG: return "invalid argument";
    case DL_ERR_SHAPE: return "unsupported or inconsistent shape";
    case DL_ERR_DTYPE: return "unsupported dtype";
    case DL_ERR_UNSUPPORTED: return "operation not supported by this pool";
    case DL_ERR_CUDA: return "CUDA error";
    case DL_ERR_DEVICE: return "device error bits set";
    }
    return "unknown status";
}

namespace dl {

unsigned long long stall_ns() { return g_stall_ns.load(); }

// A decode launch with fewer than this many heads per SM is latency-bound: its time
// is the dependent chain of one head (slot id, live length, log, tile) and, when a
// slot merges, that head's write-back, not the bytes.  Measured on B200 (RetNet,
// L = 32): 3.5 heads per SM ran faster merging every step (the eager recurrence),
// 14 heads per SM faster deferred.
constexpr int kAdaptiveHeadsPerSm = 6;

bool adaptive_merges_every_step(long long batch, int n_heads) {
    return batch * (long long)n_heads < (long long)kAdaptiveHeadsPerSm * device_sm_count();
}

// Checks a bare descriptor with the rules of dl_create_pool, except that its
// arrival-counter buffer is not looked at (the entry point that allocates nothing
// supplies its own).  Makes no CUDA call.
dl_status check_desc_without_arrive(const dl_pool_desc &d) {
    if (d.n_slots <= 0 || d.n_layers <= 0 || d.n_heads <= 0 || d.n_kheads <= 0)
        return DL_ERR_SHAPE;
    if (d.n_heads % d.n_kheads) return DL_ERR_SHAPE;
    if (!dk_supported(d.d_k)) return DL_ERR_SHAPE;
    if (d.d_v < 16 || d.d_v > 1024 || d.d_v % 16) return DL_ERR_SHAPE;
    if (d.log_cap < 1 || d.log_cap > 64) return DL_ERR_SHAPE;
    if (d.tile_v != 0 && d.tile_v != 16 && d.tile_v != 32 && d.tile_v != 128) return DL_ERR_SHAPE;
    if (d.tile_v == 32 && (d.d_k < 64 || d.d_v % 32)) return DL_ERR_SHAPE;
    if (d.tile_v == 128 && !dl::whole_head_supported(d.d_k, d.d_v)) return DL_ERR_SHAPE;
    if ((int)d.decay < DL_DECAY_NONE || (int)d.decay > DL_DECAY_DIAG) return DL_ERR_INVALID_ARG;
    if ((int)d.update < DL_UPDATE_ADD || (int)d.update > DL_UPDATE_DELTA_UNDECAYED)
        return DL_ERR_INVALID_ARG;
    if (d.log_format != DL_LOG_FP32 && d.log_format != DL_LOG_COMPACT) return DL_ERR_INVALID_ARG;
    if (d.replay_mode != DL_REPLAY_PER_TILE && d.replay_mode != DL_REPLAY_CLUSTER) return DL_ERR_INVALID_ARG;
    if (!d.state || !aligned(d.state, 16) || !d.err_word || !aligned(d.err_word, 4))
        return DL_ERR_INVALID_ARG;
    if (!d.log || !aligned(d.log, 16) || !d.log_len || !aligned(d.log_len, 4))
        return DL_ERR_INVALID_ARG;
    if ((long long)d.n_slots * d.n_heads * (d.d_v / 16) > 0x7fffffffLL) return DL_ERR_SHAPE;
    return DL_OK;
}

// The host-side checks of dl_decode_step for a descriptor (no CUDA call).
dl_status check_decode_args(const dl_pool_desc &desc, int32_t layer, const dl_step_args *args) {
    dl_pool stack_pool;
    stack_pool.d = desc;
    return check_step(&stack_pool, layer, args, true, true);
}

// Runs dl_decode_step for a checked descriptor with the given arrival counters,
// through a pool handle held on the stack (nothing is allocated).
dl_status decode_step_on_desc(const dl_pool_desc &desc, int32_t *arrive, int32_t layer,
                              const dl_step_args *args, int32_t auto_merge, void *stream) {
    dl_pool stack_pool;
    stack_pool.d = desc;
    stack_pool.d.arrive = arrive;
    return dl_decode_step(&stack_pool, layer, args, auto_merge, stream);
}

}  // namespace dl
