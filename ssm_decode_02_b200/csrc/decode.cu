// decode.cu -- dispatch of the fused decode kernel (the instantiations live in
// decode_<family>.cu and decode_<family>_bdr.cu).
#include <cuda_runtime.h>

#include "rsq_internal.h"
#include "rsq_tile.cuh"

namespace rsq {

// One pair of lookup functions per family (plain rules / directional rules),
// each defined in its own translation unit.
using InfoFn = int (*)(int, int, int, bool, int, int*, size_t*, const void**);
#define RSQ_DECLARE(NAME) int NAME(int dk, int ub, int bpw, bool f32state, int rnd, int* threads, size_t* smem, \
                                   const void** func);
RSQ_DECLARE(decode_info_gdn)
RSQ_DECLARE(decode_info_gdn_bdr)
RSQ_DECLARE(decode_info_mamba2)
RSQ_DECLARE(decode_info_mamba2_bdr)
RSQ_DECLARE(decode_info_gla)
RSQ_DECLARE(decode_info_gla_bdr)
RSQ_DECLARE(decode_info_kda)
RSQ_DECLARE(decode_info_kda_bdr)
RSQ_DECLARE(decode_info_gdn_copy)
RSQ_DECLARE(decode_info_gdn_copy_bdr)
RSQ_DECLARE(decode_info_mamba2_copy)
RSQ_DECLARE(decode_info_mamba2_copy_bdr)
RSQ_DECLARE(decode_info_gla_copy)
RSQ_DECLARE(decode_info_gla_copy_bdr)
RSQ_DECLARE(decode_info_kda_copy)
RSQ_DECLARE(decode_info_kda_copy_bdr)
RSQ_DECLARE(decode_info_gdn_pw4)
RSQ_DECLARE(decode_info_gdn_pw8)
RSQ_DECLARE(decode_info_gdn_pw16)
#undef RSQ_DECLARE

int decode_kernel_info(int family, int dk, int ub, int bpw, bool f32state, int rnd, int* threads, size_t* smem,
                       const void** func) {
    // [family][rule group]: plain, BDR, copy scale, copy scale + BDR
    static const InfoFn table[4][4] = {
        {decode_info_gdn, decode_info_gdn_bdr, decode_info_gdn_copy, decode_info_gdn_copy_bdr},
        {decode_info_mamba2, decode_info_mamba2_bdr, decode_info_mamba2_copy, decode_info_mamba2_copy_bdr},
        {decode_info_gla, decode_info_gla_bdr, decode_info_gla_copy, decode_info_gla_copy_bdr},
        {decode_info_kda, decode_info_kda_bdr, decode_info_kda_copy, decode_info_kda_copy_bdr}};
    if (rnd < 0 || rnd > 15) return -1;
    const int group = f32state ? 0 : (((rnd & kRndBdr) ? 1 : 0) + ((rnd & kRndCopy) ? 2 : 0));
    if (is_pw_family(family)) {  // pure-write window: plain rules only
        static const InfoFn pw[3] = {decode_info_gdn_pw4, decode_info_gdn_pw8, decode_info_gdn_pw16};
        return group == 0 ? pw[family - kFamGdnPw](dk, ub, bpw, f32state, rnd, threads, smem, func) : -1;
    }
    if (family < 0 || family > 3) return -1;
    return table[family][group](dk, ub, bpw, f32state, rnd, threads, smem, func);
}

int launch_decode(int family, int dk, int ub, int bpw, bool f32state, int rnd, const DecodeParams& p,
                  void* stream) {
    int threads;
    size_t smem;
    const void* func;
    if (decode_kernel_info(family, dk, ub, bpw, f32state, rnd, &threads, &smem, &func) != 0)
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
