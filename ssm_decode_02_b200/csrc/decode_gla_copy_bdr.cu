// decode_gla_copy_bdr.cu -- GLA instantiations of the fused decode
// kernel with the copy scale and Bounded Directional Rounding.
#include "decode_kernel.cuh"

namespace rsq {
int decode_info_gla_copy_bdr(int dk, int ub, int bpw, bool f32state, int rnd, int* threads, size_t* smem,
                             const void** func) {
    return decode_info_family<RSQ_GLA, kRndCopy | kRndBdr, kRndCopy | kRndBdr | kRndSr, kRndCopy | kRndBdr | kRndSr | kRndU8>(
        dk, ub, bpw, f32state, rnd, threads, smem, func);
}
}  // namespace rsq
