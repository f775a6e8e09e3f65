// decode_gla.cu -- GLA instantiations of the fused decode kernel with
// nearest and stochastic rounding, 16- and 8-bit uniforms (and the full-precision state).
#include "decode_kernel.cuh"

namespace rsq {
int decode_info_gla(int dk, int ub, int bpw, bool f32state, int rnd, int* threads, size_t* smem,
                    const void** func) {
    return decode_info_family<RSQ_GLA, 0, kRndSr, kRndSr | kRndU8>(dk, ub, bpw, f32state, rnd, threads, smem, func);
}
}  // namespace rsq
