// decode_mamba2.cu -- Mamba-2 instantiations of the fused decode kernel.
#include "decode_kernel.cuh"

namespace rsq {
int decode_info_mamba2(int dk, int ub, bool f32state, bool sr, int* threads, size_t* smem,
                       const void** func) {
    return decode_info_family<RSQ_MAMBA2>(dk, ub, f32state, sr, threads, smem, func);
}
}  // namespace rsq
