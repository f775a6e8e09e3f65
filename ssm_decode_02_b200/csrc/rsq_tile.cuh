// rsq_tile.cuh -- thread layout, column reductions and the requantizer shared by
// the decode, quantize and dequantize kernels.
//
// Work unit: one column block of one head, i.e. all dk rows of CB = min(64, dv)
// consecutive value columns (the scale groups of the value-axis grouping are
// columns, so a unit's reductions never leave the unit).  Thread layout inside
// a unit: a thread owns 4 consecutive columns (4*cw .. 4*cw+3) of the rows
// i = rho, rho + R, rho + 2R, ... (RPT rows), where R = 8 (dk <= 128) or 16.
// Lanes of a warp cover LPR = CB/4 column groups of RPW = 32/LPR consecutive
// rho, so every warp-wide shared-memory access reads consecutive rows without
// bank conflicts.
#pragma once

#include "rsq_device.cuh"

namespace rsq {

constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: ulp 1, integers land in the low mantissa bits
constexpr uint32_t kMagicBits = 0x4B400000u;
constexpr uint32_t kSrBits8 = 0x43000000u;  // 128.0f: SR offset of 8-bit codes
constexpr uint32_t kSrBits4 = 0x43080000u;  // 136.0f: SR offset of 4-bit codes

template <int DK, int CB>
struct Layout {
    static constexpr int R = DK <= 128 ? 8 : 16;  // partial sums over the key axis
    static constexpr int RPT = DK / R;            // rows per thread (even)
    static constexpr int LPR = CB / 4;            // lanes per row
    static constexpr int RPW = 32 / LPR;          // rows per warp instruction
    static constexpr int NT = LPR * R;            // threads per unit
    static constexpr int W = NT / 32;             // warps per unit
    static_assert(RPT % 2 == 0, "rows per thread must pair up for the SR counter");
    static_assert(W * RPW == R, "layout");
};

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
    return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z),
                       __fadd_rn(a.w, b.w));
}
__device__ __forceinline__ float4 max4(float4 a, float4 b) {
    return make_float4(max_nan(a.x, b.x), max_nan(a.y, b.y), max_nan(a.z, b.z), max_nan(a.w, b.w));
}

// Sum of a per-thread partial over the R partials (rho), in the fixed order:
// XOR butterfly over rho with d = 1, 2, ..., R/2.  Low rho bits live in the
// lanes (shuffles), high bits in the warps (shared memory `red`, [W][CB]).
// Every thread returns the full sum for its 4 columns.  Contains one
// __syncthreads when W > 1.
template <int LPR, int W, int CB>
__device__ __forceinline__ float4 colsum(float4 v, float* red, int warp, int rgl, int cw) {
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
        v.x = __fadd_rn(v.x, __shfl_xor_sync(0xffffffffu, v.x, off));
        v.y = __fadd_rn(v.y, __shfl_xor_sync(0xffffffffu, v.y, off));
        v.z = __fadd_rn(v.z, __shfl_xor_sync(0xffffffffu, v.z, off));
        v.w = __fadd_rn(v.w, __shfl_xor_sync(0xffffffffu, v.w, off));
    }
    if constexpr (W > 1) {
        if (rgl == 0) *reinterpret_cast<float4*>(red + warp * CB + 4 * cw) = v;
        __syncthreads();
        float4 P[W];
#pragma unroll
        for (int w = 0; w < W; ++w) P[w] = *reinterpret_cast<const float4*>(red + w * CB + 4 * cw);
#pragma unroll
        for (int d = 1; d < W; d <<= 1)
#pragma unroll
            for (int w = 0; w < W; w += 2 * d) P[w] = add4(P[w], P[w + d]);
        v = P[0];
    }
    return v;
}

// Column sum and column max together (one barrier).
template <int LPR, int W, int CB>
__device__ __forceinline__ void colsum_max(float4& v, float4& m, float* red_s, float* red_m,
                                           int warp, int rgl, int cw) {
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
        v.x = __fadd_rn(v.x, __shfl_xor_sync(0xffffffffu, v.x, off));
        v.y = __fadd_rn(v.y, __shfl_xor_sync(0xffffffffu, v.y, off));
        v.z = __fadd_rn(v.z, __shfl_xor_sync(0xffffffffu, v.z, off));
        v.w = __fadd_rn(v.w, __shfl_xor_sync(0xffffffffu, v.w, off));
        m.x = max_nan(m.x, __shfl_xor_sync(0xffffffffu, m.x, off));
        m.y = max_nan(m.y, __shfl_xor_sync(0xffffffffu, m.y, off));
        m.z = max_nan(m.z, __shfl_xor_sync(0xffffffffu, m.z, off));
        m.w = max_nan(m.w, __shfl_xor_sync(0xffffffffu, m.w, off));
    }
    if constexpr (W > 1) {
        if (rgl == 0) {
            *reinterpret_cast<float4*>(red_s + warp * CB + 4 * cw) = v;
            *reinterpret_cast<float4*>(red_m + warp * CB + 4 * cw) = m;
        }
        __syncthreads();
        float4 P[W], Q[W];
#pragma unroll
        for (int w = 0; w < W; ++w) {
            P[w] = *reinterpret_cast<const float4*>(red_s + w * CB + 4 * cw);
            Q[w] = *reinterpret_cast<const float4*>(red_m + w * CB + 4 * cw);
        }
#pragma unroll
        for (int d = 1; d < W; d <<= 1)
#pragma unroll
            for (int w = 0; w < W; w += 2 * d) {
                P[w] = add4(P[w], P[w + d]);
                Q[w] = max4(Q[w], Q[w + d]);
            }
        v = P[0];
        m = Q[0];
    }
}

// Column max only.
template <int LPR, int W, int CB>
__device__ __forceinline__ float4 colmax(float4 m, float* red_m, int warp, int rgl, int cw) {
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
        m.x = max_nan(m.x, __shfl_xor_sync(0xffffffffu, m.x, off));
        m.y = max_nan(m.y, __shfl_xor_sync(0xffffffffu, m.y, off));
        m.z = max_nan(m.z, __shfl_xor_sync(0xffffffffu, m.z, off));
        m.w = max_nan(m.w, __shfl_xor_sync(0xffffffffu, m.w, off));
    }
    if constexpr (W > 1) {
        if (rgl == 0) *reinterpret_cast<float4*>(red_m + warp * CB + 4 * cw) = m;
        __syncthreads();
        float4 Q[W];
#pragma unroll
        for (int w = 0; w < W; ++w) Q[w] = *reinterpret_cast<const float4*>(red_m + w * CB + 4 * cw);
#pragma unroll
        for (int d = 1; d < W; d <<= 1)
#pragma unroll
            for (int w = 0; w < W; w += 2 * d) Q[w] = max4(Q[w], Q[w + d]);
        m = Q[0];
    }
    return m;
}

// Per-column scale s = m / r and multiplier inv = r / m rounded toward zero
// (0 for an all-zero or non-finite column).  Sets bit j of `bad` for a
// non-finite column.
template <int BITS>
__device__ __forceinline__ void scale_and_inv(float m, float& s, float& inv, unsigned& bad, int j) {
    constexpr float r = float((1 << (BITS - 1)) - 1);
    s = __fdiv_rn(m, r);
    const bool finite = isfinite(m);
    inv = (m > 0.0f && finite) ? __fdiv_rz(r, m) : 0.0f;
    if (!finite) bad |= 1u << j;
}

// Decode RPT rows of 4 codes (this thread's part of a unit tile in shared
// memory) into exact float codes c.
template <int BITS, int R, int RPT, int CB>
__device__ __forceinline__ void load_codes(const uint8_t* tile, int rho, int cw, float (&c)[RPT][4]) {
    if constexpr (BITS == 8) {
        const uint64_t off = pk(-(kMagic + 128.0f), -(kMagic + 128.0f));
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(tile + (rho + R * k) * CB + 4 * cw);
            const uint64_t f01 = pk(__uint_as_float(prmt(w, kMagicBits, 0x7650u)),
                                    __uint_as_float(prmt(w, kMagicBits, 0x7651u)));
            const uint64_t f23 = pk(__uint_as_float(prmt(w, kMagicBits, 0x7652u)),
                                    __uint_as_float(prmt(w, kMagicBits, 0x7653u)));
            upk(add2(f01, off), c[k][0], c[k][1]);
            upk(add2(f23, off), c[k][2], c[k][3]);
        }
    } else {
        const uint64_t off = pk(-(kMagic + 8.0f), -(kMagic + 8.0f));
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const uint32_t h16 =
                *reinterpret_cast<const uint16_t*>(tile + (rho + R * k) * (CB / 2) + 2 * cw);
            const uint32_t lo = h16 & 0x0F0Fu;         // columns 0 and 2
            const uint32_t hi = (h16 >> 4) & 0x0F0Fu;  // columns 1 and 3
            const uint64_t f01 = pk(__uint_as_float(prmt(lo, kMagicBits, 0x7650u)),
                                    __uint_as_float(prmt(hi, kMagicBits, 0x7650u)));
            const uint64_t f23 = pk(__uint_as_float(prmt(lo, kMagicBits, 0x7651u)),
                                    __uint_as_float(prmt(hi, kMagicBits, 0x7651u)));
            upk(add2(f01, off), c[k][0], c[k][1]);
            upk(add2(f23, off), c[k][2], c[k][3]);
        }
    }
}

// Pack the 4 codes of one row held in the low byte (fill=0) or byte 2 of
// four floats into the stored representation.
template <int BITS>
__device__ __forceinline__ uint32_t pack_row(uint32_t t0, uint32_t t1, uint32_t t2, uint32_t t3,
                                             bool byte2) {
    if constexpr (BITS == 8) {
        // byte 0 of each float holds c + 128
        const uint32_t a = prmt(t0, t1, 0x0040u);
        const uint32_t b = prmt(t2, t3, 0x0040u);
        return prmt(a, b, 0x5410u);
    } else {
        // the code nibble c + 8 sits in byte 0 (RTN) or byte 2 (SR)
        const uint32_t sel = byte2 ? 0x0062u : 0x0040u;
        const uint32_t a = prmt(t0, t2, sel);  // columns 0, 2
        const uint32_t b = prmt(t1, t3, sel);  // columns 1, 3
        return a + (b << 4);                   // low 16 bits are the two stored bytes
    }
}

// Requantize this thread's RPT x 4 block of the full-precision state S and
// store it to the unit tile `dst` in global memory.
//   RTN: nearest integer of the exact S*inv (fma with a magic offset).
//   SR : t = fma(S, inv, o + u/2^16), c = floor(t) - o, u from Philox4x32-10.
// Columns flagged in `bad` get the zero code.
template <int BITS, bool SR, int R, int RPT, int CB>
__device__ __forceinline__ void requantize_store(const float (&S)[RPT][4], const float (&inv)[4],
                                                 uint8_t* dst, int rho, int cw, uint32_t g,
                                                 uint32_t h, uint32_t b, uint32_t step,
                                                 uint32_t key0, uint32_t key1, unsigned bad) {
    const uint64_t inv01 = pk(inv[0], inv[1]);
    const uint64_t inv23 = pk(inv[2], inv[3]);
    // stored-code masks for non-finite columns: keep good columns, fill bad ones with zero code
    uint32_t keep = 0xFFFFFFFFu, fill = 0u;
    if (bad) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (bad & (1u << j)) {
                if constexpr (BITS == 8) {
                    keep &= ~(0xFFu << (8 * j));
                    fill |= 0x80u << (8 * j);
                } else {
                    keep &= ~(0xFu << (4 * j));
                    fill |= 0x8u << (4 * j);
                }
            }
    }
    auto store_row = [&](int k, uint32_t word) {
        word = (word & keep) | fill;
        const int i = rho + R * k;
        if constexpr (BITS == 8)
            *reinterpret_cast<uint32_t*>(dst + i * CB + 4 * cw) = word;
        else
            *reinterpret_cast<uint16_t*>(dst + i * (CB / 2) + 2 * cw) = static_cast<uint16_t>(word);
    };
    if constexpr (!SR) {
        const float o = (BITS == 8) ? kMagic + 128.0f : kMagic + 8.0f;
        const uint64_t oo = pk(o, o);
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            float t0, t1, t2, t3;
            upk(fma2(pk(S[k][0], S[k][1]), inv01, oo), t0, t1);
            upk(fma2(pk(S[k][2], S[k][3]), inv23, oo), t2, t3);
            store_row(k, pack_row<BITS>(__float_as_uint(t0), __float_as_uint(t1),
                                        __float_as_uint(t2), __float_as_uint(t3), false));
        }
    } else {
        constexpr uint32_t vb = (BITS == 8) ? kSrBits8 : kSrBits4;
        const uint64_t mm = pk(kMagic, kMagic);
#pragma unroll
        for (int k = 0; k < RPT / 2; ++k) {
            const uint32_t i = static_cast<uint32_t>(rho + R * k);  // i < dk/2; partner i + dk/2
            const U4 rnd = philox4x32_10(U4{i | (g << 16), h, b, step}, key0, key1);
            const uint32_t u[2][2] = {{rnd.x, rnd.y}, {rnd.z, rnd.w}};
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int kk = k + half * (RPT / 2);
                const uint32_t w0 = u[half][0], w1 = u[half][1];
                const uint64_t V01 = pk(__uint_as_float(vb | (w0 & 0xFFFFu)), __uint_as_float(vb | (w0 >> 16)));
                const uint64_t V23 = pk(__uint_as_float(vb | (w1 & 0xFFFFu)), __uint_as_float(vb | (w1 >> 16)));
                uint64_t t01 = fma2(pk(S[kk][0], S[kk][1]), inv01, V01);
                uint64_t t23 = fma2(pk(S[kk][2], S[kk][3]), inv23, V23);
                if constexpr (BITS == 8) {
                    // floor(t) + magic: byte 0 = floor(t) = c + 128
                    t01 = add2_rm(t01, mm);
                    t23 = add2_rm(t23, mm);
                }
                float t0, t1, t2, t3;
                upk(t01, t0, t1);
                upk(t23, t2, t3);
                // 4-bit: t in [129, 144) so byte 2 of t is floor(t) - 128 = c + 8
                store_row(kk, pack_row<BITS>(__float_as_uint(t0), __float_as_uint(t1),
                                             __float_as_uint(t2), __float_as_uint(t3), BITS == 4));
            }
        }
    }
}

}  // namespace rsq
