// Merge / materialise / reset kernels, and the step-kernel dispatch over d_k.
#include "dl_kernels.cuh"

namespace dl {

cudaError_t launch_step_dk16(const KParams &, int, int, bool, bool, cudaStream_t);
cudaError_t launch_step_dk64(const KParams &, int, int, bool, bool, cudaStream_t);
cudaError_t launch_step_dk128(const KParams &, int, int, bool, bool, cudaStream_t);

int pick_bv(int dk, int dv, long long work_items_at_32) {
    if (dk == 16) return 16;
    if (dv % 32) return 16;
    // Narrow tiles double the CTA count when 32-wide tiles would leave SMs idle
    // (148 SMs; two waves of at least one CTA each).
    return work_items_at_32 < 2LL * 148 ? 16 : 32;
}

cudaError_t launch_step(const KParams &p, int bv, int decay, bool delta, bool bf16,
                        cudaStream_t st) {
    switch (p.dk) {
    case 16: return launch_step_dk16(p, bv, decay, delta, bf16, st);
    case 64: return launch_step_dk64(p, bv, decay, delta, bf16, st);
    case 128: return launch_step_dk128(p, bv, decay, delta, bf16, st);
    default: return cudaErrorInvalidValue;
    }
}

namespace {

template <int DK, int BV, int DECAY>
cudaError_t merge_one(const KParams &p, bool materialize, cudaStream_t st) {
    using Sh = TileShape<DK, BV>;
    const size_t smem = dyn_floats(p.L, DK, BV, true) * sizeof(float);
    const long long grid = (long long)p.batch * p.H * p.nv;
    merge_kernel<DK, BV, DECAY><<<(unsigned)grid, Sh::NT, smem, st>>>(p, materialize ? 1 : 0);
    return cudaGetLastError();
}

template <int DK, int BV>
cudaError_t merge_decay(const KParams &p, int decay, bool materialize, cudaStream_t st) {
    switch (decay) {
    case DL_DECAY_NONE: return merge_one<DK, BV, DL_DECAY_NONE>(p, materialize, st);
    case DL_DECAY_SCALAR: return merge_one<DK, BV, DL_DECAY_SCALAR>(p, materialize, st);
    case DL_DECAY_DIAG: return merge_one<DK, BV, DL_DECAY_DIAG>(p, materialize, st);
    default: return cudaErrorInvalidValue;
    }
}

__global__ void reset_kernel(const int32_t *slots, int batch, int n_slots, int n_layers,
                             int32_t *log_len, int32_t *arrive, int32_t *err) {
    const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= (long long)batch * n_layers) return;
    const int b = (int)(idx / n_layers), l = (int)(idx % n_layers);
    const int s = slots[b];
    if (s < 0 || s >= n_slots) {
        atomicOr(err, DL_EBIT_SLOT_RANGE);
        return;
    }
    log_len[(size_t)s * n_layers + l] = 0;
    arrive[(size_t)s * n_layers + l] = 0;
}

__global__ void clear_bits_kernel(int32_t *err, int32_t bits) { atomicAnd(err, ~bits); }

}  // namespace

cudaError_t launch_clear_bits(int32_t *err, int32_t bits, cudaStream_t st) {
    clear_bits_kernel<<<1, 1, 0, st>>>(err, bits);
    return cudaGetLastError();
}

namespace {

template <int DECAY>
cudaError_t merge_head_one(const KParams &p, bool materialize, cudaStream_t st) {
    // A'^T and b (2 x L x 128 floats) and the raw entries (L x E floats)
    const size_t smem = ((size_t)2 * p.L * 128 + (size_t)p.L * p.E) * sizeof(float);
    auto kern = merge_head_kernel<DECAY>;
    static bool configured = false;  // per instantiation: room for the largest log (64 fp32 entries)
    if (!configured) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   (2 * 64 * 128 + 64 * 384) * (int)sizeof(float));
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const long long grid = (long long)p.batch * p.H;
    kern<<<(unsigned)grid, MH_NT, smem, st>>>(p, materialize ? 1 : 0);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_merge_head(const KParams &p, int decay, bool materialize, cudaStream_t st) {
    if (p.dk != 128 || p.dv != 128) return cudaErrorInvalidValue;
    switch (decay) {
    case DL_DECAY_NONE: return merge_head_one<DL_DECAY_NONE>(p, materialize, st);
    case DL_DECAY_SCALAR: return merge_head_one<DL_DECAY_SCALAR>(p, materialize, st);
    case DL_DECAY_DIAG: return merge_head_one<DL_DECAY_DIAG>(p, materialize, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_merge(const KParams &p, int bv, int decay, bool materialize, cudaStream_t st) {
    if (p.dk == 16 && bv == 16) return merge_decay<16, 16>(p, decay, materialize, st);
    if (p.dk == 64 && bv == 16) return merge_decay<64, 16>(p, decay, materialize, st);
    if (p.dk == 64 && bv == 32) return merge_decay<64, 32>(p, decay, materialize, st);
    if (p.dk == 128 && bv == 16) return merge_decay<128, 16>(p, decay, materialize, st);
    if (p.dk == 128 && bv == 32) return merge_decay<128, 32>(p, decay, materialize, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_reset(const int32_t *slots, int batch, int n_slots, int n_layers,
                         int32_t *log_len, int32_t *arrive, int32_t *err, cudaStream_t st) {
    const long long n = (long long)batch * n_layers;
    const int threads = 256;
    reset_kernel<<<(unsigned)((n + threads - 1) / threads), threads, 0, st>>>(
        slots, batch, n_slots, n_layers, log_len, arrive, err);
    return cudaGetLastError();
}

}  // namespace dl
