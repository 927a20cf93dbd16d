// Launch of the persistent TMA-staged decode step (dl_persistent.cuh).
#include "dl_persistent.cuh"

namespace dl {

int device_sm_count() {
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            return 148;
        cached[dev] = n;
    }
    return cached[dev];
}

bool persistent_supported(int dk, int dv, int log_cap) {
    return dk == pk::DK && dv == pk::DV && log_cap <= pk::LMAX;
}

namespace {

// Shared memory for two CTAs per SM: 228 KB per SM less 1 KB reserved per CTA.
constexpr size_t kSmemPerCta = 115712;

template <int DECAY, bool DELTA, typename IT>
cudaError_t launch_one(KParams p, cudaStream_t st) {
    auto kern = pk::persistent_step_kernel<DECAY, DELTA, IT>;
    const size_t fixed = pk::Layout(0, p.L).total;
    int ns = (int)((kSmemPerCta - fixed) / pk::CBYTES);
    ns = ns < pk::NCHUNK ? pk::NCHUNK : (ns > 8 ? 8 : ns);
    p.ns = ns;
    const size_t smem = pk::Layout(ns, p.L).total;
    static size_t configured = 0;  // per instantiation
    if (smem > configured) {
        const cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        configured = smem;
    }
    const long long items = (long long)p.batch * p.H;
    const long long cap = 2LL * device_sm_count();
    const int grid = (int)(items < cap ? items : cap);
    kern<<<grid, pk::NTHREADS, smem, st>>>(p);
    return cudaGetLastError();
}

template <int DECAY>
cudaError_t by_update(const KParams &p, bool delta, bool bf16, cudaStream_t st) {
    if (delta)
        return bf16 ? launch_one<DECAY, true, __nv_bfloat16>(p, st)
                    : launch_one<DECAY, true, float>(p, st);
    return bf16 ? launch_one<DECAY, false, __nv_bfloat16>(p, st)
                : launch_one<DECAY, false, float>(p, st);
}

}  // namespace

cudaError_t launch_persistent(const KParams &p, int decay, bool delta, bool bf16, cudaStream_t st) {
    switch (decay) {
    case DL_DECAY_NONE: return by_update<DL_DECAY_NONE>(p, delta, bf16, st);
    case DL_DECAY_SCALAR: return by_update<DL_DECAY_SCALAR>(p, delta, bf16, st);
    case DL_DECAY_DIAG: return by_update<DL_DECAY_DIAG>(p, delta, bf16, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace dl
