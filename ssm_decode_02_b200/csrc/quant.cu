// quant.cu -- standalone quantize / dequantize / drift kernels (sm_100a).
//
// rsq_quantize converts a full-precision state into the stored format with the
// same per-column absmax scale and rounding as the decode step (initialisation,
// checkpoint load).  rsq_dequantize expands codes * scales back to floats.
// rsq_state_drift accumulates the per-head squared error of a quantized state
// against a full-precision trajectory (relative state drift).
#include <cuda_runtime.h>

#include "rsq_internal.h"
#include "rsq_tile.cuh"

namespace rsq {

template <int DK, int CB, int BITS>
__device__ __forceinline__ void quantize_unit(const QuantParams& p, int hu, int cb, int b, int h,
                                              float* red, int warp, int rgl, int cw, int rho) {
    using L = Layout<DK, CB>;
    constexpr int R = L::R, RPT = L::RPT;
    const float* src = p.S + (long long)hu * DK * p.dv + cb * CB + 4 * cw;
    float S[RPT][4];
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(src + (long long)(rho + R * k) * p.dv));
        S[k][0] = t.x; S[k][1] = t.y; S[k][2] = t.z; S[k][3] = t.w;
    }
    const uint32_t code_bytes = static_cast<uint32_t>(DK * CB * BITS / 8);
    uint8_t* dst = p.codes + (long long)b * p.row_bytes + p.head_off[h] + (long long)cb * code_bytes;
    if constexpr (BITS == 32) {
#pragma unroll
        for (int k = 0; k < RPT; ++k)
            *reinterpret_cast<float4*>(dst + ((rho + R * k) * CB + 4 * cw) * 4) =
                make_float4(S[k][0], S[k][1], S[k][2], S[k][3]);
        return;
    } else {
        float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k + 1 < RPT; k += 2)
#pragma unroll
            for (int j = 0; j < 4; ++j) m[j] = max3_nan(m[j], fabsf(S[k][j]), fabsf(S[k + 1][j]));
        const float4 m4 = colmax<L::LPR, L::W, CB>(make_float4(m[0], m[1], m[2], m[3]), red, warp, rgl, cw);
        const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
        float sn[4], inv[4];
        unsigned bad = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) scale_and_inv<BITS>(mv[j], sn[j], inv[j], bad, j);
        const long long col0 = (long long)hu * p.dv + cb * CB + 4 * cw;
        if (rho == 0) *reinterpret_cast<float4*>(p.scales + col0) = make_float4(sn[0], sn[1], sn[2], sn[3]);
        if (bad && rho == 0) atomicOr(p.flag, kFlagNonFinite);
        const uint32_t g = static_cast<uint32_t>(cb * (CB / 4) + cw);
        if (p.sr)
            requantize_store<BITS, true, R, RPT, CB>(S, inv, dst, rho, cw, g, h, b, p.step, p.key0,
                                                     p.key1, bad);
        else
            requantize_store<BITS, false, R, RPT, CB>(S, inv, dst, rho, cw, g, h, b, p.step,
                                                      p.key0, p.key1, bad);
    }
}

template <int DK, int CB>
__global__ void __launch_bounds__(Layout<DK, CB>::NT) rsq_quantize_kernel(const __grid_constant__ QuantParams p) {
    using L = Layout<DK, CB>;
    __shared__ __align__(16) float red[L::W * CB];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cw = lane % L::LPR, rgl = lane / L::LPR, rho = warp * L::RPW + rgl;
    for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
        const int hu = u / p.ncb, cb = u - hu * p.ncb, b = hu / p.H, h = hu - b * p.H;
        const int bits = p.head_bits[h];
        if (bits == 8) quantize_unit<DK, CB, 8>(p, hu, cb, b, h, red, warp, rgl, cw, rho);
        else if (bits == 4) quantize_unit<DK, CB, 4>(p, hu, cb, b, h, red, warp, rgl, cw, rho);
        else quantize_unit<DK, CB, 32>(p, hu, cb, b, h, red, warp, rgl, cw, rho);
        __syncthreads();
    }
}

template <int DK, int CB, int BITS>
__device__ __forceinline__ void dequantize_unit(const DequantParams& p, int hu, int cb, int b, int h,
                                                int cw, int rho) {
    using L = Layout<DK, CB>;
    constexpr int R = L::R, RPT = L::RPT;
    const uint32_t code_bytes = static_cast<uint32_t>(DK * CB * BITS / 8);
    const uint8_t* src = p.codes + (long long)b * p.row_bytes + p.head_off[h] + (long long)cb * code_bytes;
    float* dst = p.S + (long long)hu * DK * p.dv + cb * CB + 4 * cw;
    float S[RPT][4];
    if constexpr (BITS == 32) {
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const float4 t = *reinterpret_cast<const float4*>(src + ((rho + R * k) * CB + 4 * cw) * 4);
            S[k][0] = t.x; S[k][1] = t.y; S[k][2] = t.z; S[k][3] = t.w;
        }
    } else {
        load_codes<BITS, R, RPT, CB>(src, rho, cw, S);
        const float4 s = *reinterpret_cast<const float4*>(p.scales + (long long)hu * p.dv + cb * CB + 4 * cw);
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            S[k][0] = __fmul_rn(S[k][0], s.x);
            S[k][1] = __fmul_rn(S[k][1], s.y);
            S[k][2] = __fmul_rn(S[k][2], s.z);
            S[k][3] = __fmul_rn(S[k][3], s.w);
        }
    }
#pragma unroll
    for (int k = 0; k < RPT; ++k)
        *reinterpret_cast<float4*>(dst + (long long)(rho + R * k) * p.dv) =
            make_float4(S[k][0], S[k][1], S[k][2], S[k][3]);
}

template <int DK, int CB>
__global__ void __launch_bounds__(Layout<DK, CB>::NT) rsq_dequantize_kernel(const __grid_constant__ DequantParams p) {
    using L = Layout<DK, CB>;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cw = lane % L::LPR, rgl = lane / L::LPR, rho = warp * L::RPW + rgl;
    const int units = p.B * p.H * p.ncb;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int hu = u / p.ncb, cb = u - hu * p.ncb, b = hu / p.H, h = hu - b * p.H;
        const int bits = p.head_bits[h];
        if (bits == 8) dequantize_unit<DK, CB, 8>(p, hu, cb, b, h, cw, rho);
        else if (bits == 4) dequantize_unit<DK, CB, 4>(p, hu, cb, b, h, cw, rho);
        else dequantize_unit<DK, CB, 32>(p, hu, cb, b, h, cw, rho);
    }
}

// One CTA per head: sums of squared differences in double.
__global__ void __launch_bounds__(256) rsq_drift_kernel(const __grid_constant__ DriftParams p) {
    __shared__ double red[2][8];
    const int hu = blockIdx.x;
    const int b = hu / p.H, h = hu - b * p.H;
    const int bits = p.q_head_bits[h];
    const int CB = p.dv < 64 ? p.dv : 64;
    const long long n = (long long)p.dk * p.dv;
    const uint8_t* q = p.q_codes + (long long)b * p.q_row_bytes + p.q_head_off[h];
    const float* f = reinterpret_cast<const float*>(p.f_codes + (long long)b * p.f_row_bytes +
                                                    (long long)h * n * 4);
    const float* sc = p.q_scales + (long long)hu * p.dv;
    double e2 = 0.0, f2 = 0.0;
    for (long long e = threadIdx.x; e < n; e += blockDim.x) {
        // e walks the stored (column-block) order: block, row, column within block
        const long long cb = e / ((long long)p.dk * CB);
        const long long rem = e - cb * p.dk * CB;
        const int jj = static_cast<int>(rem % CB);
        const int j = static_cast<int>(cb) * CB + jj;
        int c;
        if (bits == 8) {
            c = static_cast<int>(q[e]) - 128;
        } else {
            const uint8_t byte = q[e >> 1];
            c = static_cast<int>((e & 1) ? (byte >> 4) : (byte & 0xF)) - 8;
        }
        const double sh = static_cast<double>(__fmul_rn(static_cast<float>(c), sc[j]));
        const double fv = static_cast<double>(f[e]);
        e2 += (sh - fv) * (sh - fv);
        f2 += fv * fv;
    }
    for (int off = 16; off > 0; off >>= 1) {
        e2 += __shfl_xor_sync(0xffffffffu, e2, off);
        f2 += __shfl_xor_sync(0xffffffffu, f2, off);
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) {
        red[0][warp] = e2;
        red[1][warp] = f2;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double a = 0.0, c2 = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
            a += red[0][w];
            c2 += red[1][w];
        }
        p.sums[2 * hu] = a;
        p.sums[2 * hu + 1] = c2;
    }
}

// ---------------------------------------------------------------------------
template <int DK, int CB>
static int launch_q(const QuantParams& p, void* stream) {
    const int grid = p.units < 148 * 16 ? p.units : 148 * 16;
    rsq_quantize_kernel<DK, CB><<<grid, Layout<DK, CB>::NT, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return static_cast<int>(cudaGetLastError());
}
template <int DK, int CB>
static int launch_dq(const DequantParams& p, void* stream) {
    const int units = p.B * p.H * p.ncb;
    const int grid = units < 148 * 16 ? units : 148 * 16;
    rsq_dequantize_kernel<DK, CB><<<grid, Layout<DK, CB>::NT, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return static_cast<int>(cudaGetLastError());
}

#define RSQ_DISPATCH(FN, P)                                                                   \
    switch (dk * 1000 + cb) {                                                                \
        case 16016: return FN<16, 16>(P, stream);   case 16032: return FN<16, 32>(P, stream);   \
        case 16064: return FN<16, 64>(P, stream);   case 32016: return FN<32, 16>(P, stream);   \
        case 32032: return FN<32, 32>(P, stream);   case 32064: return FN<32, 64>(P, stream);   \
        case 64016: return FN<64, 16>(P, stream);   case 64032: return FN<64, 32>(P, stream);   \
        case 64064: return FN<64, 64>(P, stream);   case 128016: return FN<128, 16>(P, stream); \
        case 128032: return FN<128, 32>(P, stream); case 128064: return FN<128, 64>(P, stream); \
        case 256016: return FN<256, 16>(P, stream); case 256032: return FN<256, 32>(P, stream); \
        case 256064: return FN<256, 64>(P, stream);                                          \
        default: return static_cast<int>(cudaErrorInvalidValue);                               \
    }

int launch_quantize(int dk, int cb, const QuantParams& p, void* stream) { RSQ_DISPATCH(launch_q, p) }
int launch_dequantize(int dk, int cb, const DequantParams& p, void* stream) { RSQ_DISPATCH(launch_dq, p) }

int launch_drift(const DriftParams& p, void* stream) {
    rsq_drift_kernel<<<p.B * p.H, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return static_cast<int>(cudaGetLastError());
}

}  // namespace rsq
