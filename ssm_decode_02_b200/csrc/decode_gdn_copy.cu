// decode_gdn_copy.cu -- Gated DeltaNet instantiations of the fused decode kernel
// with the copy scale (scales from an unquantized copy's column maxima), with
// nearest and stochastic rounding.
#include "decode_kernel.cuh"

namespace rsq {
int decode_info_gdn_copy(int dk, int ub, int bpw, bool f32state, int rnd, int* threads, size_t* smem,
                         const void** func) {
    return decode_info_family<RSQ_GDN, kRndCopy, kRndCopy | kRndSr, kRndCopy | kRndSr | kRndU8>(dk, ub, bpw, f32state, rnd, threads,
                                                                   smem, func);
}
}  // namespace rsq
