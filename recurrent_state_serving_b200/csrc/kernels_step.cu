// Instantiations and dispatch of the decode / append / eager step kernel for one
// key dimension.  The build compiles this file once per supported d_k
// (-DDL_STEP_DK=16|64|128) so the variants compile in parallel.
#include "dl_kernels.cuh"

#ifndef DL_STEP_DK
#error "DL_STEP_DK must be defined"
#endif

namespace dl {

namespace {

template <int BV, int DECAY, bool DELTA, typename IT>
cudaError_t launch_one(const KParams &p, cudaStream_t st) {
    using Sh = TileShape<DL_STEP_DK, BV>;
    // merge-every launches with scalar decay form A' without shared memory (step_kernel)
    const bool need_A = p.auto_merge != 0 && !(p.merge_every && DECAY == DL_DECAY_SCALAR);
    const size_t smem = dyn_floats(p.L, DL_STEP_DK, BV, need_A) * sizeof(float);
    const long long grid = (long long)p.batch * p.H * p.nv;
    auto kern = step_kernel<DL_STEP_DK, BV, DECAY, DELTA, IT>;
    if (p.cl <= 1) {
        kern<<<(unsigned)grid, Sh::NT, smem, st>>>(p);
        return cudaGetLastError();
    }
    // a head's p.cl = p.nv value tiles (adjacent in blockIdx) as one cluster
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(Sh::NT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)p.cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int BV, int DECAY>
cudaError_t by_update(const KParams &p, bool delta, bool bf16, cudaStream_t st) {
    if (delta)
        return bf16 ? launch_one<BV, DECAY, true, __nv_bfloat16>(p, st)
                    : launch_one<BV, DECAY, true, float>(p, st);
    return bf16 ? launch_one<BV, DECAY, false, __nv_bfloat16>(p, st)
                : launch_one<BV, DECAY, false, float>(p, st);
}

template <int BV>
cudaError_t by_decay(const KParams &p, int decay, bool delta, bool bf16, cudaStream_t st) {
    switch (decay) {
    case DL_DECAY_NONE: return by_update<BV, DL_DECAY_NONE>(p, delta, bf16, st);
    case DL_DECAY_SCALAR: return by_update<BV, DL_DECAY_SCALAR>(p, delta, bf16, st);
    case DL_DECAY_DIAG: return by_update<BV, DL_DECAY_DIAG>(p, delta, bf16, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

#define DL_CAT2(a, b) a##b
#define DL_CAT(a, b) DL_CAT2(a, b)

cudaError_t DL_CAT(launch_step_dk, DL_STEP_DK)(const KParams &p, int bv, int decay, bool delta,
                                               bool bf16, cudaStream_t st) {
#if DL_STEP_DK == 16
    if (bv == 16) return by_decay<16>(p, decay, delta, bf16, st);
#else
    if (bv == 16) return by_decay<16>(p, decay, delta, bf16, st);
    if (bv == 32) return by_decay<32>(p, decay, delta, bf16, st);
#endif
    return cudaErrorInvalidValue;
}

}  // namespace dl
