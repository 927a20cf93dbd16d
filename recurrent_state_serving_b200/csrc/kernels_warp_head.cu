// Launch of the warp-per-head decode step (dl_warp_head.cuh).
#include "dl_warp_head.cuh"

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

bool whole_head_supported(int dk, int dv) { return dk == wh::DK && dv == wh::DV; }

namespace {

template <int DECAY, bool DELTA, typename IT, int FMT>
cudaError_t launch_one(const KParams &p, cudaStream_t st) {
    // the kernel's compile-time entry layout must be the one the pool was given
    using LC = wh::LogCopy<DECAY, FMT, DELTA>;
    if (p.log && (p.E != LC::E_F || p.boff != LC::B_OFF || p.loff != LC::L_OFF || p.a16 != (int)LC::A16 ||
                  p.b16 != (int)LC::B16))
        return cudaErrorInvalidValue;
    auto kern = wh::warp_head_kernel<DECAY, DELTA, IT, FMT>;
    static bool configured = false;  // per instantiation
    if (!configured) {
        const cudaError_t e =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)wh::SMEM);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const long long items = (long long)p.batch * p.H;
    const long long sms = device_sm_count();
    const int grid = (int)(items < sms ? items : sms);
    // programmatic stream serialization: the launch may overlap the end of the
    // previous kernel in the stream; the kernel waits for it (griddepcontrol.wait)
    // before its first global memory access
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(wh::NTHREADS);
    cfg.dynamicSmemBytes = wh::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int DECAY>
cudaError_t by_update(const KParams &p, bool delta, bool bf16, cudaStream_t st) {
    if (p.a16) {  // compact log: bf16 inputs only (checked at the ABI)
        if (!bf16) return cudaErrorInvalidValue;
        return delta ? launch_one<DECAY, true, __nv_bfloat16, 1>(p, st)
                     : launch_one<DECAY, false, __nv_bfloat16, 1>(p, st);
    }
    if (delta)
        return bf16 ? launch_one<DECAY, true, __nv_bfloat16, 0>(p, st)
                    : launch_one<DECAY, true, float, 0>(p, st);
    return bf16 ? launch_one<DECAY, false, __nv_bfloat16, 0>(p, st)
                : launch_one<DECAY, false, float, 0>(p, st);
}

}  // namespace

cudaError_t launch_whole_head(const KParams &p, int decay, bool delta, bool bf16, cudaStream_t st) {
    switch (decay) {
    case DL_DECAY_NONE: return by_update<DL_DECAY_NONE>(p, delta, bf16, st);
    case DL_DECAY_SCALAR: return by_update<DL_DECAY_SCALAR>(p, delta, bf16, st);
    case DL_DECAY_DIAG: return by_update<DL_DECAY_DIAG>(p, delta, bf16, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace dl
