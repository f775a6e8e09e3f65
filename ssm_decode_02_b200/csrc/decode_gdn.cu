// decode_gdn.cu -- Gated DeltaNet instantiations of the fused decode kernel.
#include "decode_kernel.cuh"

namespace rsq {
int decode_info_gdn(int dk, int ub, bool f32state, bool sr, int* threads, size_t* smem,
                    const void** func) {
    return decode_info_family<RSQ_GDN>(dk, ub, f32state, sr, threads, smem, func);
}
}  // namespace rsq
