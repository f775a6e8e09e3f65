// quant.cu -- standalone quantize / dequantize / drift kernels (sm_100a).
//
// rsq_quantize converts a full-precision state into the stored format with the
// same per-column absmax scale and rounding as the decode step (initialisation,
// checkpoint load).  rsq_dequantize expands codes * scales back to floats.
// rsq_state_drift accumulates the per-head squared error of a quantized state
// against a full-precision trajectory (relative state drift).  All three walk
// the stored 16-column blocks with one warp per block.
#include <cuda_runtime.h>

#include "rsq_internal.h"
#include "rsq_tile.cuh"

namespace rsq {

constexpr int kWarpsPerCta = 4;

struct BlockIdx {
    int b, h, hu, blk;
};

__device__ __forceinline__ BlockIdx block_of(long long gb, int H, int nblk) {
    BlockIdx r;
    r.hu = static_cast<int>(gb / nblk);
    r.blk = static_cast<int>(gb - (long long)r.hu * nblk);
    r.b = r.hu / H;
    r.h = r.hu - r.b * H;
    return r;
}

template <int DK, int BITS>
__device__ __forceinline__ void quantize_block(const QuantParams& p, const BlockIdx& bi, int lane, int g,
                                               int cw) {
    constexpr int RPT = Layout<DK>::RPT;
    const int j0 = bi.blk * kBlockCols;
    const float* src = p.S + (long long)bi.hu * DK * p.dv + j0 + 4 * cw;
    uint64_t S2[RPT][2];
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const ulonglong2 t = __ldg(reinterpret_cast<const ulonglong2*>(src + (long long)(g + kR * k) * p.dv));
        S2[k][0] = t.x;
        S2[k][1] = t.y;
    }
    constexpr int BLOCK_BYTES = DK * kBlockCols * BITS / 8;
    uint8_t* dst = p.codes + (long long)bi.b * p.row_bytes + p.head_off[bi.h] + (long long)bi.blk * BLOCK_BYTES;
    if constexpr (BITS == 32) {
#pragma unroll
        for (int k = 0; k < RPT; ++k)
            *reinterpret_cast<ulonglong2*>(dst + ((g + kR * k) * 16 + 4 * cw) * 4) = make_ulonglong2(S2[k][0], S2[k][1]);
    } else {
        float4 m4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const float4 s = unpk4(S2[k][0], S2[k][1]);
            m4.x = max_nan(m4.x, fabsf(s.x));
            m4.y = max_nan(m4.y, fabsf(s.y));
            m4.z = max_nan(m4.z, fabsf(s.z));
            m4.w = max_nan(m4.w, fabsf(s.w));
        }
        const float m = reduce_scatter4(m4, g, MaxOp());
        const float mine = scale_or_inv<BITS>(m, g);
        const long long col = (long long)bi.hu * p.dv + j0 + 4 * cw + col_of(g);
        if (g < 4) p.scales[col] = mine;
        const float4 iv = gather_cols(mine, cw, 16);
        const bool any_nonfinite = is_neg_zero(iv.x) || is_neg_zero(iv.y) || is_neg_zero(iv.z) || is_neg_zero(iv.w);
        if (any_nonfinite) {
            atomicOr(p.flag, kFlagNonFinite);
            clear_nonfinite_columns<RPT>(S2, iv);
        }
        const uint32_t gcol = static_cast<uint32_t>(j0 / 4 + cw);
        // no previous state: the base rounding of the context's rule
        const BdrRef none{};
        if (p.rnd == (kRndSr | kRndU8))
            requantize_store<BITS, kRndSr | kRndU8, RPT>(S2, iv, dst, g, cw, gcol, bi.h, bi.b, p.step, p.rk, none);
        else if (p.rnd == kRndSr)
            requantize_store<BITS, kRndSr, RPT>(S2, iv, dst, g, cw, gcol, bi.h, bi.b, p.step, p.rk, none);
        else
            requantize_store<BITS, 0, RPT>(S2, iv, dst, g, cw, gcol, bi.h, bi.b, p.step, p.rk, none);
    }
}

template <int DK>
__global__ void __launch_bounds__(32 * kWarpsPerCta) rsq_quantize_kernel(const __grid_constant__ QuantParams p) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int g = lane >> 2, cw = lane & 3;
    const int nblk = p.dv / kBlockCols;
    const long long total = (long long)p.B * p.H * nblk;
    for (long long gb = (long long)blockIdx.x * kWarpsPerCta + w; gb < total; gb += (long long)gridDim.x * kWarpsPerCta) {
        const BlockIdx bi = block_of(gb, p.H, nblk);
        const int bits = p.head_bits[bi.h];
        if (bits == 8) quantize_block<DK, 8>(p, bi, lane, g, cw);
        else if (bits == 4) quantize_block<DK, 4>(p, bi, lane, g, cw);
        else quantize_block<DK, 32>(p, bi, lane, g, cw);
    }
}

template <int DK, int BITS>
__device__ __forceinline__ void dequantize_block(const DequantParams& p, const BlockIdx& bi, int g, int cw) {
    constexpr int RPT = Layout<DK>::RPT;
    constexpr int BLOCK_BYTES = DK * kBlockCols * BITS / 8;
    const int j0 = bi.blk * kBlockCols;
    const uint8_t* src = p.codes + (long long)bi.b * p.row_bytes + p.head_off[bi.h] + (long long)bi.blk * BLOCK_BYTES;
    float* dst = p.S + (long long)bi.hu * DK * p.dv + j0 + 4 * cw;
    uint64_t S2[RPT][2];
    if constexpr (BITS == 32) {
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const ulonglong2 t = *reinterpret_cast<const ulonglong2*>(src + ((g + kR * k) * 16 + 4 * cw) * 4);
            S2[k][0] = t.x;
            S2[k][1] = t.y;
        }
    } else {
        load_codes<BITS, RPT>(src, g, cw, S2);
        if (p.key_axis) {
            // one scale per key row
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                const float si = p.scales[(long long)bi.hu * DK + g + kR * k];
                const uint64_t ss = pk(si, si);
                S2[k][0] = mul2(S2[k][0], ss);
                S2[k][1] = mul2(S2[k][1], ss);
            }
        } else {
            const float4 s = *reinterpret_cast<const float4*>(p.scales + (long long)bi.hu * p.dv + j0 + 4 * cw);
            const uint64_t s01 = pk(s.x, s.y), s23 = pk(s.z, s.w);
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                S2[k][0] = mul2(S2[k][0], s01);
                S2[k][1] = mul2(S2[k][1], s23);
            }
        }
    }
    if (p.absmax != nullptr) {
        // column maxima of |S| (NaN-propagating), one lane per column after the reduce-scatter
        float4 m4 = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const float4 v = unpk4(S2[k][0], S2[k][1]);
            m4.x = max_nan(m4.x, fabsf(v.x));
            m4.y = max_nan(m4.y, fabsf(v.y));
            m4.z = max_nan(m4.z, fabsf(v.z));
            m4.w = max_nan(m4.w, fabsf(v.w));
        }
        const float m = reduce_scatter4(m4, g, MaxOp());
        if (g < 4) p.absmax[(long long)bi.hu * p.dv + j0 + 4 * cw + col_of(g)] = m;
        return;
    }
#pragma unroll
    for (int k = 0; k < RPT; ++k)
        *reinterpret_cast<ulonglong2*>(dst + (long long)(g + kR * k) * p.dv) = make_ulonglong2(S2[k][0], S2[k][1]);
}

template <int DK>
__global__ void __launch_bounds__(32 * kWarpsPerCta) rsq_dequantize_kernel(const __grid_constant__ DequantParams p) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int g = lane >> 2, cw = lane & 3;
    const int nblk = p.dv / kBlockCols;
    const long long total = (long long)p.B * p.H * nblk;
    for (long long gb = (long long)blockIdx.x * kWarpsPerCta + w; gb < total; gb += (long long)gridDim.x * kWarpsPerCta) {
        const BlockIdx bi = block_of(gb, p.H, nblk);
        const int bits = p.head_bits[bi.h];
        if (bits == 8) dequantize_block<DK, 8>(p, bi, g, cw);
        else if (bits == 4) dequantize_block<DK, 4>(p, bi, g, cw);
        else dequantize_block<DK, 32>(p, bi, g, cw);
    }
}

// One CTA per head: sums of squared differences in double.
__global__ void __launch_bounds__(256) rsq_drift_kernel(const __grid_constant__ DriftParams p) {
    __shared__ double red[2][8];
    const int hu = blockIdx.x;
    const int b = hu / p.H, h = hu - b * p.H;
    const int bits = p.q_head_bits[h];
    const long long n = (long long)p.dk * p.dv;
    const uint8_t* q = p.q_codes + (long long)b * p.q_row_bytes + p.q_head_off[h];
    const float* f = reinterpret_cast<const float*>(p.f_codes + (long long)b * p.f_row_bytes +
                                                    (long long)h * n * 4);
    const float* sc = p.q_scales + (long long)hu * p.dv;
    double e2 = 0.0, f2 = 0.0;
    for (long long e = threadIdx.x; e < n; e += blockDim.x) {
        // e walks the stored order: block of 16 columns, row, column within block
        const long long blk = e / ((long long)p.dk * kBlockCols);
        const int jj = static_cast<int>(e % kBlockCols);
        const int j = static_cast<int>(blk) * kBlockCols + jj;
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
static int grid_for(long long blocks) {
    const long long ctas = (blocks + kWarpsPerCta - 1) / kWarpsPerCta;
    return static_cast<int>(ctas < 148 * 16 ? ctas : 148 * 16);
}

int launch_quantize(int dk, const QuantParams& p, void* stream) {
    const int grid = grid_for((long long)p.B * p.H * (p.dv / kBlockCols));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (dk) {
        case 16: rsq_quantize_kernel<16><<<grid, 32 * kWarpsPerCta, 0, st>>>(p); break;
        case 32: rsq_quantize_kernel<32><<<grid, 32 * kWarpsPerCta, 0, st>>>(p); break;
        case 64: rsq_quantize_kernel<64><<<grid, 32 * kWarpsPerCta, 0, st>>>(p); break;
        case 128: rsq_quantize_kernel<128><<<grid, 32 * kWarpsPerCta, 0, st>>>(p); break;
        case 256: rsq_quantize_kernel<256><<<grid, 32 * kWarpsPerCta, 0, st>>>(p); break;
        default: return static_cast<int>(cudaErrorInvalidValue);
    }
    return static_cast<int>(cudaGetLastError());
}

int launch_dequantize(int dk, const DequantParams& p, void* stream) {
    const int grid = grid_for((long long)p.B * p.H * (p.dv / kBlockCols));
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    switch (dk) {
        case 16: rsq_dequantize_kernel<16><<<grid, 32 * kWarpsPerCta, 0, st>>>(p); break;
        case 32: rsq_dequantize_kernel<32><<<grid, 32 * kWarpsPerCta, 0, st>>>(p); break;
        case 64: rsq_dequantize_kernel<64><<<grid, 32 * kWarpsPerCta, 0, st>>>(p); break;
        case 128: rsq_dequantize_kernel<128><<<grid, 32 * kWarpsPerCta, 0, st>>>(p); break;
        case 256: rsq_dequantize_kernel<256><<<grid, 32 * kWarpsPerCta, 0, st>>>(p); break;
        default: return static_cast<int>(cudaErrorInvalidValue);
    }
    return static_cast<int>(cudaGetLastError());
}

int launch_drift(const DriftParams& p, void* stream) {
    rsq_drift_kernel<<<p.B * p.H, 256, 0, static_cast<cudaStream_t>(stream)>>>(p);
    return static_cast<int>(cudaGetLastError());
}

}  // namespace rsq
