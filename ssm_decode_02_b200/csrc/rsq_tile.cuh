// rsq_tile.cuh -- warp tile layout, in-warp column reductions and the
// requantizer shared by the decode, quantize and dequantize kernels.
//
// A head's value columns are stored in blocks of 16 (the scale groups of the
// value-axis grouping are columns, so a block carries everything its
// reductions need).  One warp owns one block: all dk rows x 16 columns.  Lane
// (cw, g) with cw = lane % 4 and g = lane / 4 holds columns 4cw..4cw+3 of the
// rows i = g, g+8, g+16, ... (RPT = dk/8 rows).  Sums over the key axis are
// therefore R = 8 partials p = i mod 8 (the lane's row group), each
// accumulated in increasing i, then combined by the XOR butterfly over p with
// d = 1, 2, 4 -- shuffles across lanes 4, 8, 16 apart.  A warp-wide shared load
// of one row per lane group reads 8 consecutive rows: no bank conflicts.
// The decode kernel at dk = 256 splits a block over two warps: each lane then
// holds the rows g + 8hh + 16k (row stride RS = 16), giving R = 16 partials
// p = i mod 16; the helpers below take the lane's first row and RS.
#pragma once

#include "rsq_device.cuh"

namespace rsq {

constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: ulp 1, integers land in the low mantissa bits
constexpr uint32_t kMagicBits = 0x4B400000u;
constexpr uint32_t kSrBits8 = 0x43000000u;  // 128.0f: SR offset of 8-bit codes (16-bit uniforms)
constexpr uint32_t kSrBits4 = 0x43080000u;  // 136.0f: SR offset of 4-bit codes (16-bit uniforms)
// 8-bit uniforms: t = S*inv + 2^15 + o + u/2^8 lies in [2^15, 2^16), where the
// ulp is 2^-8: u fills the low byte of the offset and floor(t) - 2^15 = c + o
// lands in byte 1 of t.  o = 128 (8-bit codes) or 8 (4-bit codes).
constexpr uint32_t kSr8Bits8 = 0x47008000u;  // 32896.0f
constexpr uint32_t kSr8Bits4 = 0x47000800u;  // 32776.0f

// Requantization rule of a kernel instance: bit 0 = stochastic base rounding
// (else nearest), bit 1 = Bounded Directional Rounding on top of it, bit 2 =
// 8-bit uniforms for the stochastic rounding (else 16-bit), bit 3 = scales
// from the column maxima of an unquantized copy (copy scale).  Bits 0-2 are
// the public rsq_rounding value.
constexpr int kRndSr = 1;
constexpr int kRndBdr = 2;
constexpr int kRndU8 = 4;
constexpr int kRndCopy = 8;

constexpr int kBlockCols = 16;  // columns per stored block (one warp)
constexpr int kR = 8;           // partial sums over the key axis (row groups)

template <int DK>
struct Layout {
    static constexpr int R = kR;
    static constexpr int RPT = DK / kR;  // rows per lane
    static_assert(RPT >= 2 && RPT % 2 == 0, "rows per lane must pair up for the SR counter");
};

__device__ __forceinline__ float4 unpk4(uint64_t a, uint64_t b) {
    float4 r;
    upk(a, r.x, r.y);
    upk(b, r.z, r.w);
    return r;
}

// Reduce-scatter over the 8 row groups of a column group.  Afterwards lane
// (cw, g) holds the total of column 4cw + col_of(g), col_of(g) = 2*(g&1) +
// ((g>>1)&1); lanes g and g^4 hold the same column.  Every addition pairs the
// same two partials as the butterfly d = 1, 2, 4 (floating-point addition is
// commutative), so each column total is bit-identical to the butterfly's.
__device__ __forceinline__ int col_of(int g) { return 2 * (g & 1) + ((g >> 1) & 1); }

template <class Op>
__device__ __forceinline__ float reduce_scatter4(const float4& v, int g, Op op) {
    const bool b0 = (g & 1) != 0, b1 = (g & 2) != 0;
    // d = 1 (lanes 4 apart): keep columns {0,1} (b0 = 0) or {2,3} (b0 = 1)
    const float send0 = b0 ? v.x : v.z, send1 = b0 ? v.y : v.w;
    const float keep0 = b0 ? v.z : v.x, keep1 = b0 ? v.w : v.y;
    const float a0 = op(keep0, __shfl_xor_sync(0xffffffffu, send0, 4));
    const float a1 = op(keep1, __shfl_xor_sync(0xffffffffu, send1, 4));
    // d = 2 (lanes 8 apart): keep column 2*b0 (b1 = 0) or 2*b0 + 1 (b1 = 1)
    const float send = b1 ? a0 : a1, keep = b1 ? a1 : a0;
    const float c = op(keep, __shfl_xor_sync(0xffffffffu, send, 8));
    // d = 4 (lanes 16 apart): both hold the same column
    return op(c, __shfl_xor_sync(0xffffffffu, c, 16));
}
struct AddOp {
    __device__ __forceinline__ float operator()(float a, float b) const { return __fadd_rn(a, b); }
};
struct MaxOp {
    __device__ __forceinline__ float operator()(float a, float b) const { return max_nan(a, b); }
};

// Values of this lane's 4 columns 4cw..4cw+3 after a reduce-scatter: column j
// sits on the lanes with col_of(g) = j, i.e. g = 0, 2, 1, 3 (+ base).
__device__ __forceinline__ float4 gather_cols(float mine, int cw, int base) {
    float4 r;
    r.x = __shfl_sync(0xffffffffu, mine, base + cw);
    r.y = __shfl_sync(0xffffffffu, mine, base + cw + 8);
    r.z = __shfl_sync(0xffffffffu, mine, base + cw + 4);
    r.w = __shfl_sync(0xffffffffu, mine, base + cw + 12);
    return r;
}

// Column finalisation after the reduce-scatter (m = absmax of this lane's
// column): lanes g < 4 compute the scale s = m / r, lanes g >= 4 the multiplier
// inv = r / m rounded toward zero -- 0 for an all-zero column and -0.0 for a
// non-finite one (so the caller can find non-finite columns from the
// multipliers alone).  Every lane performs one round-to-nearest division (no
// divergence); the multiplier lanes then step the quotient toward zero when it
// was rounded up, which the exact sign of fma(q, m, -r) = q*m - r tells.
template <int BITS>
__device__ __forceinline__ float scale_or_inv(float m, int g) {
    constexpr float r = float((1 << (BITS - 1)) - 1);
    const bool finite = isfinite(m);
    const bool scale_lane = g < 4;
    const float q = __fdiv_rn(scale_lane ? m : r, scale_lane ? r : m);
    const bool rounded_up = __fmaf_rn(q, m, -r) > 0.0f;
    const float q_rz = rounded_up ? __uint_as_float(__float_as_uint(q) - 1u) : q;
    const float inv = !finite ? -0.0f : (m > 0.0f ? q_rz : 0.0f);
    return scale_lane ? q : inv;
}

__device__ __forceinline__ bool is_neg_zero(float x) { return __float_as_uint(x) == 0x80000000u; }

// Decode this lane's RPT rows of 4 codes of a stored block into exact float
// codes, kept as packed pairs: S2[k][0] = columns 0,1 and S2[k][1] = columns
// 2,3 of row g + RS k (g: the lane's first row; RS: the row stride, 8 when one
// warp holds every row of the block, 16 when two warps share it).
template <int BITS, int RPT, int RS = kR>
__device__ __forceinline__ void load_codes(const uint8_t* blk, int g, int cw, uint64_t (&S2)[RPT][2]) {
    if constexpr (BITS == 8) {
        const uint64_t off = pk(-(kMagic + 128.0f), -(kMagic + 128.0f));
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const uint32_t w = *reinterpret_cast<const uint32_t*>(blk + (g + RS * k) * 16 + 4 * cw);
            const uint64_t f01 = pk(__uint_as_float(prmt(w, kMagicBits, 0x7650u)),
                                    __uint_as_float(prmt(w, kMagicBits, 0x7651u)));
            const uint64_t f23 = pk(__uint_as_float(prmt(w, kMagicBits, 0x7652u)),
                                    __uint_as_float(prmt(w, kMagicBits, 0x7653u)));
            S2[k][0] = add2(f01, off);
            S2[k][1] = add2(f23, off);
        }
    } else {
        // Nibble t of the row's 16 bits (column t, bits 4t..4t+3) is OR-ed in place
        // into the float 2^E_t with E_t = 23 - 4t, whose ulp is 2^(4t) there: the
        // float is exactly 2^E_t + (c + 8), one logic operation per code.
        const uint64_t off01 = pk(-(8388608.0f + 8.0f), -(524288.0f + 8.0f));  // 2^23, 2^19
        const uint64_t off23 = pk(-(32768.0f + 8.0f), -(2048.0f + 8.0f));      // 2^15, 2^11
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const uint32_t h16 = *reinterpret_cast<const uint16_t*>(blk + (g + RS * k) * 8 + 2 * cw);
            const uint64_t f01 = pk(__uint_as_float(and_or<0x000Fu>(h16, 0x4B000000u)),
                                    __uint_as_float(and_or<0x00F0u>(h16, 0x49000000u)));
            const uint64_t f23 = pk(__uint_as_float(and_or<0x0F00u>(h16, 0x47000000u)),
                                    __uint_as_float(and_or<0xF000u>(h16, 0x45000000u)));
            S2[k][0] = add2(f01, off01);
            S2[k][1] = add2(f23, off23);
        }
    }
}

// Exact float codes of row g + RS k of a stored block (this lane's 4 columns).
template <int BITS, int RS = kR>
__device__ __forceinline__ void load_code_row(const uint8_t* blk, int g, int cw, int k, uint64_t& c01,
                                              uint64_t& c23) {
    uint64_t S2[1][2];
    if constexpr (BITS == 8)
        load_codes<8, 1>(blk + RS * k * 16, g, cw, S2);
    else
        load_codes<4, 1>(blk + RS * k * 8, g, cw, S2);
    c01 = S2[0][0];
    c23 = S2[0][1];
}

// Pack the 4 codes of one row held in byte B of four floats (byte 0: nearest
// rounding and 8-bit codes with 16-bit uniforms; byte 1: 8-bit uniforms;
// byte 2: 4-bit codes with 16-bit uniforms) into the stored representation.
template <int BITS, int B>
__device__ __forceinline__ uint32_t pack_row(uint32_t t0, uint32_t t1, uint32_t t2, uint32_t t3) {
    if constexpr (BITS == 8 && B == 0) {
        // Byte 0 of each float holds c + 128 and byte 1 is zero, so t1*256 + t0
        // (mod 2^32) carries (byte0(t1), byte0(t0)) in its low 16 bits without any
        // carry between them; one byte permute joins the two halves.
        const uint32_t a = t1 * 256u + t0;
        const uint32_t b = t3 * 256u + t2;
        return prmt(a, b, 0x5410u);
    } else if constexpr (BITS == 8) {
        constexpr uint32_t sel = (4u + B) << 4 | B;  // bytes B of the two operands
        return prmt(prmt(t0, t1, sel), prmt(t2, t3, sel), 0x5410u);
    } else {
        // the code nibble c + 8 sits in byte B
        constexpr uint32_t sel = (4u + B) << 4 | B;
        const uint32_t a = prmt(t0, t2, sel);  // columns 0, 2
        const uint32_t b = prmt(t1, t3, sel);  // columns 1, 3
        return a + (b << 4);                   // low 16 bits are the two stored bytes
    }
}

// Stochastic rounding with 8-bit uniforms: the Philox4x32-10 words of this
// lane's rows.  One block with counter {i mod dk/4 | (j/4) << 16, h, b, step}
// serves rows i, i + dk/4, i + dk/2, i + 3dk/4 of four columns: word
// i div (dk/4), byte j mod 4.  The lane's rows are g + RS k (k < RPT), so the
// block of counter row g + RS k (k < RPT/4) gives rows k + q RPT/4 word q;
// with two rows per lane (dk = 16) both rows share counter row g mod 4.
// row_fn(k, word) is called once per row.
template <int RPT, int RS, class PhiloxKeysT, class F>
__device__ __forceinline__ void sr8_words(int g, uint32_t gcol, uint32_t h, uint32_t b, uint32_t step,
                                          const PhiloxKeysT& rk, F&& row_fn) {
    if constexpr (RPT >= 4) {
        constexpr int Q = RPT / 4;
#pragma unroll
        for (int k = 0; k < Q; ++k) {
            const uint32_t i = static_cast<uint32_t>(g + RS * k);
            const U4 rnd = philox4x32_10(U4{i | (gcol << 16), h, b, step}, rk.k0, rk.k1);
            row_fn(k, rnd.x);
            row_fn(k + Q, rnd.y);
            row_fn(k + 2 * Q, rnd.z);
            row_fn(k + 3 * Q, rnd.w);
        }
    } else {
        static_assert(RPT == 2 && RS == 8, "two rows per lane only at dk = 16");
        const U4 rnd = philox4x32_10(U4{static_cast<uint32_t>(g & 3) | (gcol << 16), h, b, step}, rk.k0, rk.k1);
        const bool upper = g >= 4;  // rows g, g + 8 are words g/4 and g/4 + 2
        row_fn(0, upper ? rnd.y : rnd.x);
        row_fn(1, upper ? rnd.w : rnd.z);
    }
}

// The offsets 2^15 + o + u/2^8 of one row's four columns, u = byte jj of the
// row's Philox word (column 4cw + jj), as two packed pairs.
__device__ __forceinline__ void sr8_offsets(uint32_t word, uint32_t vb, uint64_t& V01, uint64_t& V23) {
    V01 = pk(__uint_as_float(prmt(word, vb, 0x7650u)), __uint_as_float(prmt(word, vb, 0x7651u)));
    V23 = pk(__uint_as_float(prmt(word, vb, 0x7652u)), __uint_as_float(prmt(word, vb, 0x7653u)));
}

// Non-finite columns (multiplier -0.0) must come out as the zero code; their
// state values would not, so clear them (used on the rare path only).
template <int RPT>
__device__ __forceinline__ void clear_nonfinite_columns(uint64_t (&S2)[RPT][2], const float4& iv) {
    const bool b0 = is_neg_zero(iv.x), b1 = is_neg_zero(iv.y), b2 = is_neg_zero(iv.z), b3 = is_neg_zero(iv.w);
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const float4 s = unpk4(S2[k][0], S2[k][1]);
        S2[k][0] = pk(b0 ? 0.0f : s.x, b1 ? 0.0f : s.y);
        S2[k][1] = pk(b2 ? 0.0f : s.z, b3 ? 0.0f : s.w);
    }
}

// What Bounded Directional Rounding needs besides the new state: the previous
// codes (the stage's copy of the stored block) and scales, and the new scales.
struct BdrRef {
    const uint8_t* old_block;  // stored block as loaded (shared memory)
    uint64_t s_old01, s_old23;  // previous scales of this lane's 4 columns
    uint64_t s_new01, s_new23;  // new scales of this lane's 4 columns
};

// Bounded Directional Rounding of one element, in the magic domain T = c + M
// (M = 1.5 * 2^23 + code offset): the base code tb stands unless its value
// c * s_new lies strictly on the other side of the previous value prev than
// the new state S does; then the integer next to x = S * inv on the update's
// side (tu = ceil, td = floor) replaces it.
__device__ __forceinline__ float bdr_pick(float S, float prev, float now, float tb, float tu, float td) {
    const bool up = (S > prev) && (now < prev);
    const bool down = (S < prev) && (now > prev);
    return up ? tu : (down ? td : tb);
}

// Requantize this lane's RPT x 4 part of the full-precision state and store it
// to the block `dst` (global memory).
//   RTN: nearest integer of the exact S*inv (fma with a magic offset).
//   SR : t = fma(S, inv, o + u/2^16), c = floor(t) - o, u a 16-bit uniform from
//        Philox4x32-10 with counter {i mod dk/2 | (j/4) << 16, h, b, step}.
//   SR, 8-bit uniforms: t = fma(S, inv, 2^15 + o + u/2^8) in [2^15, 2^16),
//        c = floor(t) - 2^15 - o (byte 1 of t), u from sr8_words.
//   +BDR: the base code is replaced by ceil / floor of the exact S*inv when it
//        moves the element opposite to its update (see bdr_pick).
// `gcol` is j/4 of this lane's first column; the lane's rows are g + RS k
// (RS: as for load_codes; RS * RPT / 2 = dk / 2, so rows k and k + RPT/2 are
// the pair i, i + dk/2 that one 16-bit-uniform Philox call serves).
template <int BITS, int RND, int RPT, class PhiloxKeysT, int RS = kR>
__device__ __forceinline__ void requantize_store(const uint64_t (&S2)[RPT][2], const float4& iv,
                                                 uint8_t* dst, int g, int cw, uint32_t gcol,
                                                 uint32_t h, uint32_t b, uint32_t step,
                                                 const PhiloxKeysT& rk, const BdrRef& bdr) {
    constexpr bool SR = (RND & kRndSr) != 0;
    constexpr bool BDR = (RND & kRndBdr) != 0;
    constexpr bool U8 = SR && (RND & kRndU8) != 0;
    constexpr float kOff = (BITS == 8) ? 128.0f : 8.0f;  // stored code = c + kOff
    const uint64_t inv01 = pk(iv.x, iv.y), inv23 = pk(iv.z, iv.w);
    // this lane's first row; row k sits k * RS rows further
    uint8_t* const row0 = dst + (BITS == 8 ? g * 16 + 4 * cw : g * 8 + 2 * cw);
    auto store_row = [&](int k, uint32_t word) {
        if constexpr (BITS == 8)
            *reinterpret_cast<uint32_t*>(row0 + k * (RS * 16)) = word;
        else
            *reinterpret_cast<uint16_t*>(row0 + k * (RS * 8)) = static_cast<uint16_t>(word);
    };
    const uint64_t moff = pk(kMagic + kOff, kMagic + kOff);
    // Row k with its base codes T = c + M + kOff (two packed pairs): apply the
    // directional correction if enabled, then pack and store (low byte = c + kOff).
    auto finish_row = [&](int k, uint64_t T01, uint64_t T23) {
        if constexpr (BDR) {
            const uint64_t nmoff = pk(-(kMagic + kOff), -(kMagic + kOff));
            uint64_t c01, c23;
            load_code_row<BITS, RS>(bdr.old_block, g, cw, k, c01, c23);
            const float4 prev = unpk4(mul2(c01, bdr.s_old01), mul2(c23, bdr.s_old23));
            const float4 now = unpk4(mul2(add2(T01, nmoff), bdr.s_new01), mul2(add2(T23, nmoff), bdr.s_new23));
            const float4 tu = unpk4(fma2_rp(S2[k][0], inv01, moff), fma2_rp(S2[k][1], inv23, moff));
            const float4 td = unpk4(fma2_rm(S2[k][0], inv01, moff), fma2_rm(S2[k][1], inv23, moff));
            const float4 S = unpk4(S2[k][0], S2[k][1]);
            const float4 tb = unpk4(T01, T23);
            T01 = pk(bdr_pick(S.x, prev.x, now.x, tb.x, tu.x, td.x), bdr_pick(S.y, prev.y, now.y, tb.y, tu.y, td.y));
            T23 = pk(bdr_pick(S.z, prev.z, now.z, tb.z, tu.z, td.z), bdr_pick(S.w, prev.w, now.w, tb.w, tu.w, td.w));
        }
        float t0, t1, t2, t3;
        upk(T01, t0, t1);
        upk(T23, t2, t3);
        store_row(k, pack_row<BITS, 0>(__float_as_uint(t0), __float_as_uint(t1), __float_as_uint(t2),
                                       __float_as_uint(t3)));
    };
    if constexpr (!SR) {
#pragma unroll
        for (int k = 0; k < RPT; ++k) finish_row(k, fma2(S2[k][0], inv01, moff), fma2(S2[k][1], inv23, moff));
    } else if constexpr (U8) {
        constexpr uint32_t vb = (BITS == 8) ? kSr8Bits8 : kSr8Bits4;
        sr8_words<RPT, RS>(g, gcol, h, b, step, rk, [&](int kk, uint32_t word) {
            uint64_t V01, V23;
            sr8_offsets(word, vb, V01, V23);
            const uint64_t t01 = fma2(S2[kk][0], inv01, V01);
            const uint64_t t23 = fma2(S2[kk][1], inv23, V23);
            if constexpr (BDR) {
                // floor(t) - 2^15 + M: the magic domain of the directional rounding
                const uint64_t to_magic = pk(kMagic - 32768.0f, kMagic - 32768.0f);
                finish_row(kk, add2_rm(t01, to_magic), add2_rm(t23, to_magic));
            } else {
                float t0, t1, t2, t3;
                upk(t01, t0, t1);
                upk(t23, t2, t3);
                store_row(kk, pack_row<BITS, 1>(__float_as_uint(t0), __float_as_uint(t1), __float_as_uint(t2),
                                                __float_as_uint(t3)));
            }
        });
    } else {
        constexpr uint32_t vb = (BITS == 8) ? kSrBits8 : kSrBits4;
        const uint64_t mm = pk(kMagic, kMagic);
#pragma unroll
        for (int k = 0; k < RPT / 2; ++k) {
            const uint32_t i = static_cast<uint32_t>(g + RS * k);  // i < dk/2; partner i + dk/2
            const U4 rnd = philox4x32_10(U4{i | (gcol << 16), h, b, step}, rk.k0, rk.k1);
            const uint32_t u[2][2] = {{rnd.x, rnd.y}, {rnd.z, rnd.w}};
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int kk = k + half * (RPT / 2);
                const uint32_t w0 = u[half][0], w1 = u[half][1];
                // offset + u/2^16: the low half by a mask, the high half as
                // hi(w * 2^16) + offset bits (a multiply-add, off the logic pipe)
                const uint64_t V01 = pk(__uint_as_float(vb | (w0 & 0xFFFFu)), __uint_as_float(umulhi_add(w0, 0x10000u, vb)));
                const uint64_t V23 = pk(__uint_as_float(vb | (w1 & 0xFFFFu)), __uint_as_float(umulhi_add(w1, 0x10000u, vb)));
                uint64_t t01 = fma2(S2[kk][0], inv01, V01);
                uint64_t t23 = fma2(S2[kk][1], inv23, V23);
                if constexpr (BITS == 8 || BDR) {
                    // floor(t) + magic = c + o + magic
                    t01 = add2_rm(t01, mm);
                    t23 = add2_rm(t23, mm);
                }
                if constexpr (BITS == 8) {
                    // o = 128 = kOff: byte 0 already holds c + 128
                    finish_row(kk, t01, t23);
                } else if constexpr (BDR) {
                    // o = 136 = kOff + 128
                    const uint64_t m128 = pk(-128.0f, -128.0f);
                    finish_row(kk, add2(t01, m128), add2(t23, m128));
                } else {
                    // 4-bit: t in [129, 144) so byte 2 of t is floor(t) - 128 = c + 8
                    float t0, t1, t2, t3;
                    upk(t01, t0, t1);
                    upk(t23, t2, t3);
                    store_row(kk, pack_row<BITS, 2>(__float_as_uint(t0), __float_as_uint(t1),
                                                    __float_as_uint(t2), __float_as_uint(t3)));
                }
            }
        }
    }
}

}  // namespace rsq
