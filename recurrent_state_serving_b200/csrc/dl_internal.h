// Internal interface between the C ABI (api.cpp) and the sm_100a kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "deltalog.h"

namespace dl {

// Everything a launch needs, passed by value as the kernel parameter.
struct KParams {
    // pool
    float *state;
    float *log;
    int32_t *log_len;
    int32_t *arrive;
    int32_t *err;
    int n_slots, n_layers, H, Hk, dk, dv, L;
    int E;      // floats per log entry (the layout's entry bytes / 4)
    int boff;   // offset of b_i in an entry, in floats
    int loff;   // offset of Lambda_i in an entry, in floats
    int a16;    // a_i stored as bf16 (compact layout)
    int b16;    // b_i stored as bf16 (compact layout without the delta rule)
    int cl;     // value tiles of a head sharing ReplayPrep as one cluster (1: each alone)
    int nv;     // value tiles per head: d_v / B_V
    int layer;
    // batch
    const int32_t *slots;
    int batch;
    const void *q, *k, *v;
    const float *lam;
    int lam_const;
    const float *beta;
    float *out;
    float *dense_out;
    // behaviour
    int auto_merge;  // decode step: the slot's merge step writes the materialised state
    int merge_every; // decode step with auto_merge: every slot merges on every step
    int eager;       // eager step: c = 0 and always write back, no log
    int want_out;    // write o_t
    int undecayed;   // delta correction from S_{t-1} instead of Diag(e^lambda) S_{t-1}
    unsigned long long stall_ns;  // timeout test: 0, or the bound of a wait that never completes
};

// dl_debug_stall's setting for launches issued now (0: off).
unsigned long long stall_ns();

// Does a dl_decode_step of `batch` slots x `n_heads` heads under DL_MERGE_ADAPTIVE
// merge every slot on every step (a launch too small to fill the GPU)?
bool adaptive_merges_every_step(long long batch, int n_heads);

// Value-tile width chosen for a launch (16 or 32 columns).
int pick_bv(int dk, int dv, long long work_items_at_32);

cudaError_t launch_step(const KParams &p, int bv, int decay, bool delta, bool bf16,
                        cudaStream_t st);
// Warp-per-head step for full 128 x 128 heads (dl_warp_head.cuh).
bool whole_head_supported(int dk, int dv);
int device_sm_count();
cudaError_t launch_whole_head(const KParams &p, int decay, bool delta, bool bf16, cudaStream_t st);

cudaError_t launch_merge(const KParams &p, int bv, int decay, bool materialize,
                         cudaStream_t st);
// Merge / materialise of whole 128 x 128 heads, one CTA per head.
cudaError_t launch_merge_head(const KParams &p, int decay, bool materialize, cudaStream_t st);
cudaError_t launch_reset(const int32_t *slots, int batch, int n_slots, int n_layers,
                         int32_t *log_len, int32_t *arrive, int32_t *err, cudaStream_t st);
// Atomically clears `bits` in the error word (bits set meanwhile by other launches survive).
cudaError_t launch_clear_bits(int32_t *err, int32_t bits, cudaStream_t st);

// Floats of dynamic shared memory a launch needs.
inline size_t dyn_floats(int L, int dk, int bv, bool need_A) {
    const size_t L4 = (size_t)((L + 3) & ~3);
    return 2 * L4 + (size_t)L * bv + (need_A ? (size_t)L * dk : 0);
}

}  // namespace dl
