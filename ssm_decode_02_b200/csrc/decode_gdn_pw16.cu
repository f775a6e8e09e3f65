// decode_gdn_pw16.cu -- Gated DeltaNet with a 16-slot pure-write window:
// instantiations of the fused decode kernel with nearest and stochastic
// rounding (and the full-precision history).
#include "decode_kernel.cuh"

namespace rsq {
int decode_info_gdn_pw16(int dk, int ub, int bpw, bool f32state, int rnd, int* threads, size_t* smem,
                        const void** func) {
    return decode_info_family<kFamGdnPw + 2, 0, kRndSr, kRndSr | kRndU8>(dk, ub, bpw, f32state, rnd, threads, smem, func);
}
}  // namespace rsq
