// decode.cu -- dispatch of the fused decode kernel (instantiations live in
// decode_gdn.cu and decode_mamba2.cu).
#include <cuda_runtime.h>

#include "rsq_internal.h"

namespace rsq {

int decode_info_gdn(int dk, int ub, bool f32state, bool sr, int* threads, size_t* smem, const void** func);
int decode_info_mamba2(int dk, int ub, bool f32state, bool sr, int* threads, size_t* smem,
                       const void** func);

int decode_kernel_info(int family, int dk, int ub, bool f32state, bool sr, int* threads, size_t* smem,
                       const void** func) {
    if (family == RSQ_GDN) return decode_info_gdn(dk, ub, f32state, sr, threads, smem, func);
    return decode_info_mamba2(dk, ub, f32state, sr, threads, smem, func);
}

int launch_decode(int family, int dk, int ub, bool f32state, bool sr, const DecodeParams& p,
                  void* stream) {
    int threads;
    size_t smem;
    const void* func;
    if (decode_kernel_info(family, dk, ub, f32state, sr, &threads, &smem, &func) != 0)
        return static_cast<int>(cudaErrorInvalidValue);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    void* args[] = {const_cast<DecodeParams*>(&p)};
    return static_cast<int>(cudaLaunchKernelExC(&cfg, func, args));
}

}  // namespace rsq
