// decode_kernel.cuh -- fused quantized recurrent-state decode step (sm_100a).
//
// A work unit is one to four 16-column blocks of one head (all dk rows); up to
// dk = 128 the CTA has one warp per block (or, on large steps with units of
// four blocks, one warp per two blocks, taken one after the other), and each
// warp owns its block's columns outright, so every reduction over the key axis
// stays inside the warp and the loop has no CTA-wide barrier.  At dk = 256 two
// warps share a block (half of the rows each) and combine their column totals
// through shared memory behind a per-block mbarrier.  Persistent CTAs walk the
// units with a grid stride.
// Units arrive in an NS-stage shared-memory ring filled by bulk asynchronous
// (TMA) copies; the last warp to finish with a stage refills it with the unit
// NS ahead.  Per block a warp:
//   1. decodes the codes to exact floats (packed pairs),
//   2. (Gated DeltaNet) forms u = S^T k as s_j * sum_i c_ij k_i,
//   3. updates the state in registers (full precision, packed f32x2),
//   4. reads out o = S^T q (GDN, GLA, KDA) or y = S^T C + D x (Mamba-2) from
//      that state,
//   5. takes each column's absmax as its new scale (the dynamic "noisy" scale;
//      or the column maxima of an unquantized copy: the copy scale),
//   6. requantizes (round-to-nearest or Philox stochastic rounding, optionally
//      with Bounded Directional Rounding) and stores.
// Template parameters: the family (GDN, Mamba-2, GLA, KDA, or GDN with a 4-,
// 8- or 16-slot pure-write window), dk, the blocks per unit, a full-precision
// state, and the rule bits (stochastic, BDR, copy scale).
// Method: LoReS ("Quantizing Recurrent Language Models Is Easier Than You
// Think", sections "LoReS: State Quantization", "(1/4) Scale grouping", "(3/4)
// Rounding", "(4/4) Rotations"); recurrences and BDR as named in "Preserving
// Updates in Low-Bit Recurrent State Quantization" (abstract); the pure-write
// window of "Low-Bit GDN Recurrent-State Quantization: Global Gradient-aware
// Allocation and Pure-Write Sliding Windows" (abstract).  No tensor cores: per
// head this is two matrix-vector products over a state read once from HBM.
#pragma once

#include <cuda_runtime.h>

#include "rsq_internal.h"
#include "rsq_tile.cuh"

namespace rsq {

template <int FAM, int DK, int UB, bool F32STATE, int BPW_ = 1>
struct DecodeCfg {
    // warps per 16-column block: one holds all rows up to d_k = 128; at d_k = 256
    // two warps share the block, warp half hh holding the rows i with
    // (i mod 16) div 8 = hh (the register footprint of d_k = 128)
    static constexpr int SPLIT = DK > 128 ? 2 : 1;
    using L = Layout<DK / SPLIT>;
    static constexpr int RS = kR * SPLIT;      // row stride of a lane's rows
    // blocks each warp takes per unit: one, or two (BPW = 2, units of four
    // one-warp blocks): a warp's per-unit work -- its pair arrays, the stage
    // wait and release -- then serves two blocks
    static constexpr int BPW = BPW_;
    static constexpr int NW = UB * SPLIT / BPW;  // warps per CTA
    static constexpr int NT = 32 * NW;
    static constexpr int UCOLS = 16 * UB;      // columns per unit
    // pipeline stages (KDA's extra pair array leaves room for three; two-block
    // warps keep two so that eight 64-thread CTAs fit an SM)
    static constexpr int NS = F32STATE ? 2 : (BPW == 2 ? 2 : ((FAM == RSQ_KDA || is_pw_family(FAM)) ? 3 : 4));
    static constexpr int CODE_BYTES = F32STATE ? DK * UCOLS * 4 : DK * UCOLS;  // largest tile (8-bit)
    static constexpr int OFF_SCALES = CODE_BYTES;
    static constexpr int OFF_VA = OFF_SCALES + UCOLS * 4;  // GDN q / Mamba-2 C   (<= DK floats)
    static constexpr int OFF_VB = OFF_VA + DK * 4;         // GDN k / Mamba-2 B
    static constexpr int OFF_VC = OFF_VB + DK * 4;         // GDN v / Mamba-2 x   (<= UCOLS floats)
    static constexpr int OFF_VD = OFF_VC + UCOLS * 4;      // GLA / KDA decay per key channel (DK floats)
    static constexpr bool DIAG = (FAM == RSQ_GLA || FAM == RSQ_KDA);
    // pure-write window: the whole v (<= 256 floats), the slots' a codes and
    // scales, this unit's b codes (W x 16 per block) and the b scales
    static constexpr bool PW = is_pw_family(FAM);
    static constexpr int WIN = pw_window(FAM);  // window slots
    static constexpr int OFF_VF = OFF_VD;
    static constexpr int OFF_WA = OFF_VF + 256 * 4;
    static constexpr int OFF_WAS = OFF_WA + kMaxWindow * DK;
    static constexpr int OFF_WB = OFF_WAS + kMaxWindow * 4;
    static constexpr int OFF_WBS = OFF_WB + UB * kMaxWindow * 16;
    // the slot pass's results, shared by the unit's warps: z_w and the leaving
    // slot's propagated a as duplicated pairs (row-group layout of the pairs)
    static constexpr int OFF_WZ = OFF_WBS + kMaxWindow * 4;
    static constexpr int OFF_WM = OFF_WZ + kMaxWindow * 4;
    static constexpr int END_BASE = DIAG ? OFF_VD + DK * 4 : OFF_VD;
    static constexpr int STAGE = ((PW ? OFF_WM + kR * (DK / kR + 2) * 8 : END_BASE) + 127) / 128 * 128;
    // warps that run the slot passes (passes of 4 slots spread over the unit's warps)
    static constexpr int NPROD = PW ? (WIN / 4 < UB ? WIN / 4 : UB) : 0;
    // per warp: the two key-axis vectors as duplicated pairs (x, x), one row of
    // PST pairs per row group (padded so the row groups hit different banks)
    static constexpr int PST = L::RPT + 2;
    // pair arrays: q, k (+ the decay per key channel for GLA, + decay and
    // decay * k for KDA)
    static constexpr int NPAIR = FAM == RSQ_KDA ? 4 : (DIAG ? 3 : 2);
    static constexpr int P_WARP = NPAIR * kR * PST * 8;
    static constexpr int OFF_P = NS * STAGE;
    static constexpr int OFF_CNT = OFF_P + NW * P_WARP;  // NS release counters
    static constexpr int OFF_BAR = OFF_CNT + 16;
    static constexpr int OFF_SBAR = OFF_BAR + NS * 8;  // window: "slot results ready" per stage
    // d_k = 256: the two warps of a block exchange column totals (k^T S, the
    // readout, the absmax) in three slots of 2 x 16 floats, behind one mbarrier
    // per block (two arrivals per phase)
    static constexpr int OFF_XCH = OFF_SBAR + (PW ? NS * 8 : 0);
    static constexpr int OFF_XBAR = OFF_XCH + (SPLIT > 1 ? UB * 3 * 32 * 4 : 0);
    static constexpr int SMEM = OFF_XBAR + (SPLIT > 1 ? UB * 8 : 0);
    // resident CTAs per SM the register budget is sized for: shared memory holds
    // four 128-thread CTAs per SM (4 x ~50 KB), so 128 registers per thread
    static constexpr int MINB = F32STATE ? 1 : (NT < 128 ? 8 : 512 / NT);
    static_assert(!PW || SPLIT == 1, "the pure-write window is built for d_k <= 128");
    static_assert(BPW == 1 || (BPW == 2 && SPLIT == 1 && UB == 4 && !F32STATE && !PW),
                  "two blocks per warp only for units of four one-warp blocks");
    // the shared-memory layout, checked for every instance at compile time
    static_assert(SMEM <= 227 * 1024, "shared memory beyond the per-CTA limit");
    static_assert(STAGE % 128 == 0 && OFF_P >= NS * STAGE, "stages overlap the pair arrays");
    static_assert(OFF_SCALES % 16 == 0 && OFF_VA % 16 == 0 && OFF_VB % 16 == 0 && OFF_VC % 16 == 0 &&
                      OFF_VD % 16 == 0, "bulk-copy destinations must be 16-byte aligned");
    static_assert(P_WARP % 16 == 0 && OFF_P % 16 == 0 && OFF_CNT - OFF_P >= NW * P_WARP,
                  "one 16-byte aligned pair-array set per warp");
    static_assert(OFF_BAR >= OFF_CNT + 4 * NS && OFF_BAR % 8 == 0 && OFF_SBAR % 8 == 0 && OFF_XBAR % 8 == 0,
                  "mbarriers need their own 8-byte aligned words");
    static_assert(L::RPT * RS == DK && RS * (L::RPT / 2) == DK / 2,
                  "a lane's rows cover the block once, Philox row pairs are i and i + dk/2");
    static_assert(PST > (DK - 1) / RS, "pair arrays hold a lane's rows");
};

// Grid-stride walk over units without divisions: (b, h, cb) advance by the
// grid size G, precomputed by the host as (gb, gh, gcb).
struct UnitIt {
    int u, b, h, cb;
    __device__ __forceinline__ void init(int u0, const DecodeParams& p) {
        u = u0;
        const int hu = u0 / p.ncb;
        cb = u0 - hu * p.ncb;
        b = hu / p.H;
        h = hu - b * p.H;
    }
    __device__ __forceinline__ void advance(const DecodeParams& p) {
        u += p.grid;
        cb += p.gcb;
        h += p.gh;
        b += p.gb;
        if (cb >= p.ncb) { cb -= p.ncb; ++h; }
        if (h >= p.H) { h -= p.H; ++b; }
    }
    __device__ __forceinline__ int hu(const DecodeParams& p) const { return b * p.H + h; }
};

// Issue the bulk copies of one unit into a stage (one thread).
template <int FAM, int DK, int UB, bool F32STATE, int BPW>
__device__ __forceinline__ void issue_unit(const DecodeParams& p, const UnitIt& un, uint8_t* stage,
                                           uint32_t bar) {
    using C = DecodeCfg<FAM, DK, UB, F32STATE, BPW>;
    constexpr int UCOLS = C::UCOLS;
    const int bits = F32STATE ? 32 : p.head_bits[un.h];
    const int hu = un.hu(p);
    const uint32_t code_bytes = static_cast<uint32_t>(DK * UCOLS * bits / 8);
    const uint32_t esz = p.in_bf16 ? 2u : 4u;
    const uint32_t W = static_cast<uint32_t>(C::WIN);
    const uint32_t total = code_bytes + (F32STATE ? 0u : UCOLS * 4u) + 2u * DK * esz + UCOLS * esz +
                           (C::DIAG ? DK * 4u : 0u) +
                           (C::PW ? p.dv * esz + W * DK + 2u * W * 4u + UB * W * 16u : 0u);
    const uint8_t* codes = p.codes_in + (long long)un.b * p.row_bytes + p.head_off[un.h] +
                           (long long)un.cb * code_bytes;
    const uint32_t s = smem_u32(stage);
    mbar_arrive_expect_tx(bar, total);
    bulk_g2s(s, codes, code_bytes, bar);
    if (!F32STATE)
        bulk_g2s(s + C::OFF_SCALES, p.scales_in + (long long)hu * p.dv + un.cb * UCOLS, UCOLS * 4u, bar);
    const char* vA = static_cast<const char*>(p.vA);
    const char* vB = static_cast<const char*>(p.vB);
    const char* vC = static_cast<const char*>(p.vC);
    const long long rowA = (FAM != RSQ_MAMBA2)
                               ? (long long)hu * DK  // q and k of this head
                               : ((long long)un.b * p.ngroups + un.h / p.heads_per_group) * DK;
    bulk_g2s(s + C::OFF_VA, vA + rowA * esz, DK * esz, bar);
    bulk_g2s(s + C::OFF_VB, vB + rowA * esz, DK * esz, bar);
    bulk_g2s(s + C::OFF_VC, vC + ((long long)hu * p.dv + un.cb * UCOLS) * esz, UCOLS * esz, bar);
    if constexpr (C::DIAG) bulk_g2s(s + C::OFF_VD, p.vD + (long long)hu * DK, DK * 4u, bar);
    if constexpr (C::PW) {
        const long long nblk = p.dv / kBlockCols;
        bulk_g2s(s + C::OFF_VF, vC + (long long)hu * p.dv * esz, p.dv * esz, bar);
        bulk_g2s(s + C::OFF_WA, p.win_a_in + (long long)hu * W * DK, W * DK, bar);
        bulk_g2s(s + C::OFF_WAS, p.win_as_in + (long long)hu * W, W * 4u, bar);
        bulk_g2s(s + C::OFF_WB, p.win_b_in + ((long long)hu * nblk + (long long)un.cb * UB) * W * 16, UB * W * 16u, bar);
        bulk_g2s(s + C::OFF_WBS, p.win_bs_in + (long long)hu * W, W * 4u, bar);
    }
}

__device__ __forceinline__ float ld_vec(const uint8_t* base, int e, bool bf16) {
    if (bf16) return bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(base)[e]);
    return reinterpret_cast<const float*>(base)[e];
}

// Four consecutive elements e..e+3 of a vector in the stage, widened.
__device__ __forceinline__ float4 ld_vec4(const uint8_t* base, int e, bool bf16) {
    if (bf16) {
        const uint2 w = *reinterpret_cast<const uint2*>(base + 2 * e);
        return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u),
                           __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u));
    }
    return *reinterpret_cast<const float4*>(base + 4 * e);
}

// Per-unit scalars fetched one unit ahead.
struct Gates {
    float g0, g1, A, D;
};

template <int FAM>
__device__ __forceinline__ Gates load_gates(const DecodeParams& p, const UnitIt& un) {
    Gates g;
    const int hu = un.hu(p);
    g.g0 = (FAM == RSQ_GLA || FAM == RSQ_KDA) ? 0.f : __ldg(p.g0 + hu);
    g.g1 = (FAM != RSQ_GLA && p.g1) ? __ldg(p.g1 + hu) : 0.f;
    g.A = (FAM == RSQ_MAMBA2) ? __ldg(p.A + un.h) : 0.f;
    g.D = (FAM == RSQ_MAMBA2) ? __ldg(p.D + un.h) : 0.f;
    return g;
}

// Pure-write window ("Low-Bit GDN Recurrent-State Quantization: ... Pure-Write
// Sliding Windows", abstract), for the slot passes given to this warp: each
// slot's a vector goes through
// the step's transition a <- alpha (a - beta k (k.a)); the slot `ps` leaving
// the window leaves its propagated a in the pair array `pm` (rows as
// duplicated pairs) for the merge into the history; z_w = a_w . q (slot ps:
// k . q, its new write) goes to `zs`.  Lane (slot group, chunk) handles rows
// [chunk * DK/8, (chunk+1) * DK/8) of one slot; the dot products sum each
// chunk in increasing row order and combine the 8 chunks by the XOR butterfly
// d = 1, 2, 4.  The writer warp also encodes the new a vectors (FP8 E4M3, one
// scale = max|a| / 448 per vector).
// Widened elements [i0, i0 + N) of a key-axis vector in the stage.
template <int N>
__device__ __forceinline__ void ld_chunk(const uint8_t* base, int i0, bool bf16, float (&x)[N]) {
    if constexpr (N % 4 == 0) {
#pragma unroll
        for (int t = 0; t < N; t += 4) {
            const float4 v = ld_vec4(base, i0 + t, bf16);
            x[t] = v.x; x[t + 1] = v.y; x[t + 2] = v.z; x[t + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int t = 0; t < N; ++t) x[t] = ld_vec(base, i0 + t, bf16);
    }
}

// One slot of the pure-write window for this lane's chunk of rows: decode a,
// propagate a' = alpha * fma(-beta (k.a), k, a), and z = a'.q (k.q for the
// slot that takes the new write).  Dots: each chunk in increasing row order,
// the 8 chunks combined by the XOR butterfly d = 1, 2, 4.
template <int CH>
__device__ __forceinline__ float pw_slot(const uint8_t* stage, int off_wa, int off_was, int slot, int dk,
                                         int i0, const float (&kk)[CH], const float (&qq)[CH], float alpha,
                                         float beta, bool merging, float (&a)[CH]) {
    const float as = reinterpret_cast<const float*>(stage + off_was)[slot];
    const uint16_t* ab = reinterpret_cast<const uint16_t*>(stage + off_wa + slot * dk + i0);
#pragma unroll
    for (int t = 0; t < CH; t += 2) {
        float lo, hi;
        e4m3x2_to_f32(ab[t / 2], lo, hi);
        a[t] = __fmul_rn(lo, as);
        a[t + 1] = __fmul_rn(hi, as);
    }
    float ka = 0.f;
#pragma unroll
    for (int t = 0; t < CH; ++t) ka = __fmaf_rn(kk[t], a[t], ka);
#pragma unroll
    for (int d = 1; d < 8; d <<= 1) ka = __fadd_rn(ka, __shfl_xor_sync(0xffffffffu, ka, d));
    const float gg = __fmul_rn(beta, ka);
    float z = 0.f;
#pragma unroll
    for (int t = 0; t < CH; ++t) {
        a[t] = __fmul_rn(alpha, __fmaf_rn(-gg, kk[t], a[t]));
        z = __fmaf_rn(merging ? kk[t] : a[t], qq[t], z);
    }
#pragma unroll
    for (int d = 1; d < 8; d <<= 1) z = __fadd_rn(z, __shfl_xor_sync(0xffffffffu, z, d));
    return z;
}

// Pure-write window ("Low-Bit GDN Recurrent-State Quantization: ... Pure-Write
// Sliding Windows", abstract), for the slot passes given to this warp: each
// slot's a vector goes through
// the step's transition a <- alpha (a - beta k (k.a)); the slot `ps` leaving
// the window leaves its propagated a in the pair array `pm` (rows as
// duplicated pairs) for the merge into the history; z_w = a_w . q (slot ps:
// k . q, its new write) goes to `zs`.  Lane (slot group, chunk) handles rows
// [chunk * DK/8, (chunk+1) * DK/8) of the slots (slot group) + 4 * pass.  In a
// writer unit the warp also encodes its slots' new a vectors (FP8 E4M3, one
// scale = max|a| / 448).
template <int DK, int PST, int WIN>
__device__ __forceinline__ void pw_slots(const DecodeParams& p, const uint8_t* stage, int off_wa,
                                         int off_was, int off_va, int off_vb, int hu, int ps,
                                         float alpha, float beta, int pass0, int pstep, bool writer,
                                         uint64_t* pm, float* zs, int lane) {
    constexpr int CH = DK / 8;
    const bool bf16 = p.in_bf16 != 0;
    const int sl = lane >> 3, chunk = lane & 7, i0 = chunk * CH;
    float kk[CH], qq[CH];
    ld_chunk<CH>(stage + off_vb, i0, bf16, kk);
    ld_chunk<CH>(stage + off_va, i0, bf16, qq);
    auto finish = [&](int slot, float z, float (&a)[CH]) {
        const bool merging = (slot == ps);
        if (merging) {
#pragma unroll
            for (int t = 0; t < CH; ++t) {
                const int i = i0 + t;
                pm[(i & (kR - 1)) * PST + i / kR] = pk(a[t], a[t]);
            }
        }
        if (chunk == 0) zs[slot] = z;
        if (writer) {
            // the stored a: propagated for the slots that stay, k for the new write
            float m = 0.f;
#pragma unroll
            for (int t = 0; t < CH; ++t) {
                if (merging) a[t] = kk[t];
                m = max_nan(m, fabsf(a[t]));
            }
#pragma unroll
            for (int d = 1; d < 8; d <<= 1) m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, d));
            const float inv = (m > 0.f && isfinite(m)) ? __fdiv_rn(448.f, m) : 0.f;
            uint8_t* dst = p.win_a_out + ((long long)hu * WIN + slot) * DK + i0;
#pragma unroll
            for (int t = 0; t < CH; t += 2) {
                const uint32_t two = e4m3x2_from_f32(__fmul_rn(a[t + 1], inv), __fmul_rn(a[t], inv));
                *reinterpret_cast<uint16_t*>(dst + t) = static_cast<uint16_t>(two);
            }
            if (chunk == 0) p.win_as_out[(long long)hu * WIN + slot] = __fdiv_rn(m, 448.f);
        }
    };
    // passes pass0, pass0 + pstep, ... of 4 slots each; two slots per lane at a
    // time where possible (independent dependency chains)
    constexpr int NPASS = WIN / 4;
    int pass = pass0;
    for (; pass + pstep < NPASS; pass += 2 * pstep) {
        const int s0 = pass * 4 + sl, s1 = (pass + pstep) * 4 + sl;
        float a0[CH], a1[CH];
        const float z0 = pw_slot<CH>(stage, off_wa, off_was, s0, DK, i0, kk, qq, alpha, beta, s0 == ps, a0);
        const float z1 = pw_slot<CH>(stage, off_wa, off_was, s1, DK, i0, kk, qq, alpha, beta, s1 == ps, a1);
        finish(s0, z0, a0);
        finish(s1, z1, a1);
    }
    for (; pass < NPASS; pass += pstep) {
        const int s0 = pass * 4 + sl;
        float a0[CH];
        const float z0 = pw_slot<CH>(stage, off_wa, off_was, s0, DK, i0, kk, qq, alpha, beta, s0 == ps, a0);
        finish(s0, z0, a0);
    }
}

// Two warps sharing a block (d_k = 256): combine this lane's column total v
// (after the in-warp reduce-scatter) with the other warp's total of the same
// column, through exchange slot `xs` (2 x 16 floats) and the block's mbarrier.
// Both warps compute op(v_0, v_1) with operands in the same order as the
// butterfly's last stage d = 8 (partials p and p ^ 8).  False if the bounded
// wait ran out.
template <class Op>
__device__ __forceinline__ bool pair_combine(const DecodeParams& p, float& v, float* xs, uint32_t xbar,
                                             uint32_t& xphase, int hh, int col16, int lane, int g, Op op) {
    if (g < 4) xs[hh * 16 + col16] = v;  // lanes g and g ^ 4 hold the same column
    __syncwarp();
    // (failure-detection tests: the second warp withholds its arrival, so the
    // phase never completes and both warps' bounded waits run out)
    if (lane == 0 && !(p.withhold && hh == 1)) mbar_arrive(xbar);
    const bool ok = mbar_wait(xbar, xphase & 1u, p.wait_iters);
    ++xphase;
    if (!__all_sync(0xffffffffu, ok)) return false;
    const float other = xs[(hh ^ 1) * 16 + col16];
    v = hh == 0 ? op(v, other) : op(other, v);
    return true;
}

// One 16-column block of one unit, processed by warp w (with d_k = 256, by
// warps w and w + UB, each with half of the rows).
template <int FAM, int DK, int UB, bool F32STATE, int RND, int BITS, int BPW>
__device__ __forceinline__ bool process_block(const DecodeParams& p, const UnitIt& un, uint8_t* stage,
                                              uint8_t* smem, int stage_idx, uint32_t bar, uint32_t parity,
                                              uint32_t& xphase, const Gates& gt, int w, int lane, int g,
                                              int cw, int wblk) {
    using C = DecodeCfg<FAM, DK, UB, F32STATE, BPW>;
    using L = typename C::L;
    constexpr int RPT = L::RPT;
    constexpr int RS = C::RS;
    constexpr int BLOCK_BYTES = DK * kBlockCols * BITS / 8;
    const bool bf16 = p.in_bf16 != 0;
    const int hu = un.hu(p);
    const int hh = (C::SPLIT > 1) ? w / UB : 0;  // which rows of the block (d_k = 256)
    const int wb = (C::SPLIT > 1) ? w - hh * UB : w + wblk * C::NW;  // block within the unit (warp's wblk-th)
    const int gr = g + kR * hh;                  // this lane's first row
    const int blk = un.cb * UB + wb;  // block index within the head
    const int j0 = blk * kBlockCols;  // its first column
    const int col16 = 4 * cw + col_of(g);  // the column this lane finalises (within the block)
    // Addresses are a per-unit base (the same in every thread of the CTA) plus a
    // per-thread offset that does not change from unit to unit.
    const long long unit_code = (long long)un.b * p.row_bytes + p.head_off[un.h] +
                                (long long)(un.cb * UB) * BLOCK_BYTES;
    const long long unit_col = (long long)hu * p.dv + un.cb * C::UCOLS;
    const int lane_col = kBlockCols * wb + 4 * cw;  // this lane's first column within the unit
    float* xs = reinterpret_cast<float*>(smem + C::OFF_XCH) + wb * 96;
    const uint32_t xbar = smem_u32(smem + C::OFF_XBAR) + 8 * wb;

    // ---- this warp's copy of the key-axis vectors as duplicated pairs --------
    uint64_t* pa = reinterpret_cast<uint64_t*>(smem + C::OFF_P + w * C::P_WARP);
    uint64_t* pb = pa + kR * C::PST;
    uint64_t* pc = pb + kR * C::PST;  // GLA / KDA: decay alpha_i
    uint64_t* pd = pc + kR * C::PST;  // KDA: alpha_i * k_i
#pragma unroll
    for (int i = lane; i < DK; i += 32) {
        if (wblk != 0) break;  // built once per unit, for the warp's first block
        if (C::SPLIT > 1 && ((i / kR) & 1) != hh) continue;  // the other warp's rows
        const float a = ld_vec(stage + C::OFF_VA, i, bf16);
        const float b = ld_vec(stage + C::OFF_VB, i, bf16);
        const int pos = (i & (kR - 1)) * C::PST + i / RS;
        pa[pos] = pk(a, a);
        pb[pos] = pk(b, b);
        if constexpr (C::DIAG) {
            const float d = reinterpret_cast<const float*>(stage + C::OFF_VD)[i];
            pc[pos] = pk(d, d);
            if constexpr (FAM == RSQ_KDA) {
                const float ak = __fmul_rn(d, b);
                pd[pos] = pk(ak, ak);
            }
        }
    }
    __syncwarp();
    // window: z_w and the leaving slot's propagated a, computed by the unit's
    // first NPROD warps into the stage and published through a stage barrier
    float* zs = reinterpret_cast<float*>(stage + C::OFF_WZ);
    const int ps = C::PW ? static_cast<int>(p.step % static_cast<uint32_t>(C::WIN)) : 0;  // slot leaving
    if constexpr (C::PW) {
        const uint32_t sbar = smem_u32(smem + C::OFF_SBAR) + 8 * stage_idx;
        if (w < C::NPROD) {
            pw_slots<DK, C::PST, C::WIN>(p, stage, C::OFF_WA, C::OFF_WAS, C::OFF_VA, C::OFF_VB, hu, ps, gt.g0,
                                         gt.g1, w, C::NPROD, un.cb == 0,
                                         reinterpret_cast<uint64_t*>(stage + C::OFF_WM), zs, lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(sbar);
        }
        const bool ok = mbar_wait(sbar, parity, p.wait_iters);
        if (!__all_sync(0xffffffffu, ok)) return false;
    }
    const uint64_t* qa = pa + g * C::PST;  // q (GDN, GLA, KDA) / C (Mamba-2) of rows g + 8k
    const uint64_t* kb = pb + g * C::PST;  // k / B
    const uint64_t* ga = pc + g * C::PST;  // decay per key channel (GLA, KDA)
    const uint64_t* gk = pd + g * C::PST;  // decay * k (KDA)

    // ---- state block -> registers (packed pairs) ------------------------------
    const uint8_t* tile = stage + wb * BLOCK_BYTES;
    uint64_t S2[RPT][2];
    if constexpr (BITS == 32) {
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const ulonglong2 t = *reinterpret_cast<const ulonglong2*>(tile + ((gr + RS * k) * 16 + 4 * cw) * 4);
            S2[k][0] = t.x;
            S2[k][1] = t.y;
        }
    } else {
        load_codes<BITS, RPT, RS>(tile, gr, cw, S2);  // exact float codes c
    }
    // scales and v (GDN) / x (Mamba-2) of this lane's columns, read where needed
    // (keeping them live across the reductions costs registers)
    auto load_s4 = [&]() {
        if constexpr (BITS != 32)
            return *reinterpret_cast<const float4*>(stage + C::OFF_SCALES + (16 * wb + 4 * cw) * 4);
        else
            return make_float4(1.f, 1.f, 1.f, 1.f);
    };
    auto load_vc = [&]() { return ld_vec4(stage + C::OFF_VC, 16 * wb + 4 * cw, bf16); };

    // ---- state update ---------------------------------------------------------
    if constexpr (FAM == RSQ_GDN || C::PW) {
        const float alpha = gt.g0, beta = gt.g1;
        uint64_t a01 = pk(0.f, 0.f), a23 = pk(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < RPT; k += 2) {
            const ulonglong2 kk = *reinterpret_cast<const ulonglong2*>(kb + k);
            a01 = fma2(S2[k][0], kk.x, a01);
            a23 = fma2(S2[k][1], kk.x, a23);
            a01 = fma2(S2[k + 1][0], kk.y, a01);
            a23 = fma2(S2[k + 1][1], kk.y, a23);
        }
        float cpart = reduce_scatter4(unpk4(a01, a23), g, AddOp());
        if constexpr (C::SPLIT > 1)
            if (!pair_combine(p, cpart, xs, xbar, xphase, hh, col16, lane, g, AddOp())) return false;
        const float4 ck = gather_cols(cpart, cw, 0);
        // reload the k pairs below instead of keeping 16 of them live across the
        // reduction (register pressure)
        asm volatile("" ::: "memory");
        // u = s*ck, w = beta*(v - alpha*u), a = alpha*s  (full-precision state: u = ck, a = alpha)
        const float4 s4 = load_s4();
        const float4 vc = load_vc();
        const float ckv[4] = {ck.x, ck.y, ck.z, ck.w};
        const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
        // (with a pure-write window the new write goes to the window: v = 0 here)
        const float vv[4] = {C::PW ? 0.f : vc.x, C::PW ? 0.f : vc.y, C::PW ? 0.f : vc.z, C::PW ? 0.f : vc.w};
        float wj[4], aj[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float u = (BITS == 32) ? ckv[j] : __fmul_rn(sv[j], ckv[j]);
            wj[j] = __fmul_rn(beta, __fmaf_rn(-alpha, u, vv[j]));
            aj[j] = (BITS == 32) ? alpha : __fmul_rn(alpha, sv[j]);
        }
        const uint64_t W01 = pk(wj[0], wj[1]), W23 = pk(wj[2], wj[3]);
        const uint64_t A01 = pk(aj[0], aj[1]), A23 = pk(aj[2], aj[3]);
#pragma unroll
        for (int k = 0; k < RPT; k += 2) {
            const ulonglong2 kk = *reinterpret_cast<const ulonglong2*>(kb + k);
            // S = c*(alpha s) + k*w   (full-precision state: alpha*S + k*w)
            S2[k][0] = fma2(S2[k][0], A01, mul2(kk.x, W01));
            S2[k][1] = fma2(S2[k][1], A23, mul2(kk.x, W23));
            S2[k + 1][0] = fma2(S2[k + 1][0], A01, mul2(kk.y, W01));
            S2[k + 1][1] = fma2(S2[k + 1][1], A23, mul2(kk.y, W23));
        }
        if constexpr (C::PW) {
            // the slot leaving the window merges into the history: S += a'_ps b_ps^T
            const float bsc = reinterpret_cast<const float*>(stage + C::OFF_WBS)[ps];
            const uint32_t b4 = *reinterpret_cast<const uint32_t*>(stage + C::OFF_WB + (w * C::WIN + ps) * 16 + 4 * cw);
            float b0, b1, b2, b3;
            e4m3x2_to_f32(b4 & 0xFFFFu, b0, b1);
            e4m3x2_to_f32(b4 >> 16, b2, b3);
            const uint64_t B01 = pk(__fmul_rn(b0, bsc), __fmul_rn(b1, bsc));
            const uint64_t B23 = pk(__fmul_rn(b2, bsc), __fmul_rn(b3, bsc));
            const uint64_t* mg = reinterpret_cast<const uint64_t*>(stage + C::OFF_WM) + g * C::PST;
#pragma unroll
            for (int k = 0; k < RPT; k += 2) {
                const ulonglong2 aa = *reinterpret_cast<const ulonglong2*>(mg + k);
                S2[k][0] = fma2(aa.x, B01, S2[k][0]);
                S2[k][1] = fma2(aa.x, B23, S2[k][1]);
                S2[k + 1][0] = fma2(aa.y, B01, S2[k + 1][0]);
                S2[k + 1][1] = fma2(aa.y, B23, S2[k + 1][1]);
            }
        }
    } else if constexpr (C::DIAG) {
        // GLA: w = v.  KDA: u = s * sum_i c_ij (alpha_i k_i), w = beta (v - u).
        const float4 s4 = load_s4();
        const float4 vc = load_vc();
        const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
        const float vv[4] = {vc.x, vc.y, vc.z, vc.w};
        float wj[4] = {vv[0], vv[1], vv[2], vv[3]};
        if constexpr (FAM == RSQ_KDA) {
            uint64_t a01 = pk(0.f, 0.f), a23 = pk(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < RPT; k += 2) {
                const ulonglong2 kk = *reinterpret_cast<const ulonglong2*>(gk + k);  // alpha_i k_i
                a01 = fma2(S2[k][0], kk.x, a01);
                a23 = fma2(S2[k][1], kk.x, a23);
                a01 = fma2(S2[k + 1][0], kk.y, a01);
                a23 = fma2(S2[k + 1][1], kk.y, a23);
            }
            float cpart = reduce_scatter4(unpk4(a01, a23), g, AddOp());
            if constexpr (C::SPLIT > 1)
                if (!pair_combine(p, cpart, xs, xbar, xphase, hh, col16, lane, g, AddOp())) return false;
            const float4 ck = gather_cols(cpart, cw, 0);
            asm volatile("" ::: "memory");
            const float ckv[4] = {ck.x, ck.y, ck.z, ck.w};
            const float beta = gt.g1;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float u = (BITS == 32) ? ckv[j] : __fmul_rn(sv[j], ckv[j]);
                wj[j] = __fmul_rn(beta, __fsub_rn(vv[j], u));
            }
        }
        const uint64_t W01 = pk(wj[0], wj[1]), W23 = pk(wj[2], wj[3]);
        const uint64_t S01 = pk(sv[0], sv[1]), S23 = pk(sv[2], sv[3]);
#pragma unroll
        for (int k = 0; k < RPT; k += 2) {
            const ulonglong2 kk = *reinterpret_cast<const ulonglong2*>(kb + k);
            const ulonglong2 aa = *reinterpret_cast<const ulonglong2*>(ga + k);
            // S = c*(alpha_i s_j) + k_i w_j   (full-precision state: S*alpha_i + k_i w_j)
            if constexpr (BITS == 32) {
                S2[k][0] = fma2(S2[k][0], aa.x, mul2(kk.x, W01));
                S2[k][1] = fma2(S2[k][1], aa.x, mul2(kk.x, W23));
                S2[k + 1][0] = fma2(S2[k + 1][0], aa.y, mul2(kk.y, W01));
                S2[k + 1][1] = fma2(S2[k + 1][1], aa.y, mul2(kk.y, W23));
            } else {
                S2[k][0] = fma2(S2[k][0], mul2(aa.x, S01), mul2(kk.x, W01));
                S2[k][1] = fma2(S2[k][1], mul2(aa.x, S23), mul2(kk.x, W23));
                S2[k + 1][0] = fma2(S2[k + 1][0], mul2(aa.y, S01), mul2(kk.y, W01));
                S2[k + 1][1] = fma2(S2[k + 1][1], mul2(aa.y, S23), mul2(kk.y, W23));
            }
        }
    } else {
        const float dt = gt.g0;
        const float a = (p.g1 != nullptr) ? gt.g1 : expf(__fmul_rn(dt, gt.A));
        const float4 s4 = load_s4();
        const float4 vc = load_vc();
        const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
        const float xv[4] = {vc.x, vc.y, vc.z, vc.w};
        float xd[4], gj[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            xd[j] = __fmul_rn(dt, xv[j]);
            gj[j] = (BITS == 32) ? a : __fmul_rn(a, sv[j]);
        }
        const uint64_t X01 = pk(xd[0], xd[1]), X23 = pk(xd[2], xd[3]);
        const uint64_t G01 = pk(gj[0], gj[1]), G23 = pk(gj[2], gj[3]);
#pragma unroll
        for (int k = 0; k < RPT; k += 2) {
            const ulonglong2 bb = *reinterpret_cast<const ulonglong2*>(kb + k);
            // S = c*(a s) + B*(dt x)   (full-precision state: a*S + B*(dt x))
            S2[k][0] = fma2(S2[k][0], G01, mul2(bb.x, X01));
            S2[k][1] = fma2(S2[k][1], G23, mul2(bb.x, X23));
            S2[k + 1][0] = fma2(S2[k + 1][0], G01, mul2(bb.y, X01));
            S2[k + 1][1] = fma2(S2[k + 1][1], G23, mul2(bb.y, X23));
        }
    }

    // ---- readout and column absmax ----------------------------------------------
    // From here to the code stores the block is branch-free, so the compiler can
    // overlap the reductions' shuffle and division latency with Philox work.
    uint64_t o01 = pk(0.f, 0.f), o23 = pk(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < RPT; k += 2) {
        const ulonglong2 qq = *reinterpret_cast<const ulonglong2*>(qa + k);
        o01 = fma2(S2[k][0], qq.x, o01);
        o23 = fma2(S2[k][1], qq.x, o23);
        o01 = fma2(S2[k + 1][0], qq.y, o01);
        o23 = fma2(S2[k + 1][1], qq.y, o23);
    }
    const int c = col_of(g);  // the column this lane finalises
    float o = reduce_scatter4(unpk4(o01, o23), g, AddOp());
    if constexpr (C::SPLIT > 1)
        if (!pair_combine(p, o, xs + 32, xbar, xphase, hh, col16, lane, g, AddOp())) return false;
    if constexpr (FAM == RSQ_MAMBA2) o = __fmaf_rn(gt.D, ld_vec(stage + C::OFF_VC, 16 * wb + 4 * cw + c, bf16), o);
    if constexpr (C::PW) {
        // the window's part of the readout: o_j += b_w,j z_w in slot order
        const float vcol = ld_vec(stage + C::OFF_VC, 16 * wb + 4 * cw + c, bf16);
        const uint8_t* bcol = stage + C::OFF_WB + w * C::WIN * 16 + 4 * cw + c;
        const float* bscale = reinterpret_cast<const float*>(stage + C::OFF_WBS);
#pragma unroll
        for (int ws = 0; ws < C::WIN; ++ws) {
            float bw, unused;
            e4m3x2_to_f32(bcol[ws * 16], bw, unused);
            bw = (ws == ps) ? __fmul_rn(gt.g1, vcol) : __fmul_rn(bw, bscale[ws]);
            o = __fmaf_rn(bw, zs[ws], o);
        }
    }
    const long long col = unit_col + (lane_col + c);
    if (g < 4 && hh == 0) p.out[col] = o;
    float4 iv = make_float4(0.f, 0.f, 0.f, 0.f);
    float mine_scale = 0.f;  // the scale (lanes g < 4) or multiplier (g >= 4) of this lane's column
    if constexpr (BITS != 32) {
        float m0 = 0.f, m1 = 0.f, m2 = 0.f, m3 = 0.f;
#pragma unroll
        for (int k = 0; k < RPT; k += 2) {
            const float4 x = unpk4(S2[k][0], S2[k][1]);
            const float4 y = unpk4(S2[k + 1][0], S2[k + 1][1]);
            m0 = max3_nan(m0, fabsf(x.x), fabsf(y.x));
            m1 = max3_nan(m1, fabsf(x.y), fabsf(y.y));
            m2 = max3_nan(m2, fabsf(x.z), fabsf(y.z));
            m3 = max3_nan(m3, fabsf(x.w), fabsf(y.w));
        }
        float m = reduce_scatter4(make_float4(m0, m1, m2, m3), g, MaxOp());
        if constexpr (C::SPLIT > 1)
            if (!pair_combine(p, m, xs + 64, xbar, xphase, hh, col16, lane, g, MaxOp())) return false;
        if constexpr ((RND & kRndCopy) == 0) {
            mine_scale = scale_or_inv<BITS>(m, g);
        } else {
            // copy scale: the column maximum of an unquantized copy of the state;
            // the column's own maximum still decides whether it is finite
            mine_scale = scale_or_inv<BITS>(__ldg(p.copy_absmax + col), g);
            if (g >= 4 && !isfinite(m)) mine_scale = -0.0f;
        }
        if (g < 4 && hh == 0) p.scales_out[col] = mine_scale;
        iv = gather_cols(mine_scale, cw, 16);
    }

    // ---- store ------------------------------------------------------------------
    uint8_t* dst = p.codes_out + unit_code + wb * BLOCK_BYTES;
    const uint32_t gcol = static_cast<uint32_t>(un.cb * (C::UCOLS / 4)) + static_cast<uint32_t>(lane_col / 4);
    if constexpr (BITS == 32) {
#pragma unroll
        for (int k = 0; k < RPT; ++k)
            *reinterpret_cast<ulonglong2*>(dst + ((gr + RS * k) * 16 + 4 * cw) * 4) =
                make_ulonglong2(S2[k][0], S2[k][1]);
    } else {
        BdrRef bdr{};
        if constexpr ((RND & kRndBdr) != 0) {
            const float4 so = load_s4();
            const float4 sn = gather_cols(mine_scale, cw, 0);
            bdr.old_block = tile;
            bdr.s_old01 = pk(so.x, so.y);
            bdr.s_old23 = pk(so.z, so.w);
            bdr.s_new01 = pk(sn.x, sn.y);
            bdr.s_new23 = pk(sn.z, sn.w);
        }
        if constexpr ((RND & kRndCopy) != 0) {
            // a copy scale can lie below the state's own maximum: the state is
            // clipped to the copy's range first, so every code stays within +-r
            const float4 mc = __ldg(reinterpret_cast<const float4*>(p.copy_absmax + unit_col + lane_col));
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                const float4 v = unpk4(S2[k][0], S2[k][1]);
                S2[k][0] = pk(fminf(fmaxf(v.x, -mc.x), mc.x), fminf(fmaxf(v.y, -mc.y), mc.y));
                S2[k][1] = pk(fminf(fmaxf(v.z, -mc.z), mc.z), fminf(fmaxf(v.w, -mc.w), mc.w));
            }
        }
        requantize_store<BITS, RND, RPT, PhiloxKeys, RS>(S2, iv, dst, gr, cw, gcol, un.h, un.b, p.step, p.rk, bdr);
        // rare: a non-finite column (multiplier -0.0) is stored as the zero code
        if (is_neg_zero(iv.x) || is_neg_zero(iv.y) || is_neg_zero(iv.z) || is_neg_zero(iv.w)) {
            atomicOr(p.flag, kFlagNonFinite);
            clear_nonfinite_columns<RPT>(S2, iv);
            requantize_store<BITS, RND, RPT, PhiloxKeys, RS>(S2, iv, dst, gr, cw, gcol, un.h, un.b, p.step, p.rk,
                                                             bdr);
        }
    }

    if constexpr (C::PW) {
        // window b codes of this block: the slots that stay are copied, the new
        // write (slot ps) is encoded with one scale over the whole vector beta v
        const float beta = gt.g1;
        float mb = 0.f;
        for (int j = lane; j < p.dv; j += 32)
            mb = max_nan(mb, fabsf(__fmul_rn(beta, ld_vec(stage + C::OFF_VF, j, bf16))));
#pragma unroll
        for (int d = 16; d >= 1; d >>= 1) mb = max_nan(mb, __shfl_xor_sync(0xffffffffu, mb, d));
        const float invb = (mb > 0.f && isfinite(mb)) ? __fdiv_rn(448.f, mb) : 0.f;
        const long long nblk = p.dv / kBlockCols;
        uint8_t* bdst = p.win_b_out + ((long long)hu * nblk + blk) * C::WIN * 16;
        if (lane < C::WIN) {
            // the slots that stay: copied
            if (lane != ps)
                *reinterpret_cast<uint4*>(bdst + lane * 16) =
                    *reinterpret_cast<const uint4*>(stage + C::OFF_WB + (w * C::WIN + lane) * 16);
            if (un.cb == 0 && w == 0)
                p.win_bs_out[(long long)hu * C::WIN + lane] =
                    (lane == ps) ? __fdiv_rn(mb, 448.f) : reinterpret_cast<const float*>(stage + C::OFF_WBS)[lane];
        } else if (lane >= 16) {
            // the new write: one column per lane
            const int jj = lane - 16;
            const float x = __fmul_rn(__fmul_rn(beta, ld_vec(stage + C::OFF_VF, j0 + jj, bf16)), invb);
            bdst[ps * 16 + jj] = static_cast<uint8_t>(e4m3x2_from_f32(0.f, x));
        }
    }

    // ---- release the stage; the last warp refills it with the unit NS ahead ----
    // (the warp's reads of the stage are ordered before its release by the
    // __syncwarp and the release half of the counter update; the last warp's
    // acquire half orders every warp's reads before its refill)
    __syncwarp();
    if (wblk == C::BPW - 1 && lane == 0) {  // after the warp's last block of the unit
        uint32_t* cnt = reinterpret_cast<uint32_t*>(smem + C::OFF_CNT) + stage_idx;
        if (atom_add_acq_rel_cta(cnt, 1u) == C::NW - 1) {
            *cnt = 0u;
            UnitIt refill = un;  // the unit NS ahead of this one
#pragma unroll
            for (int s = 0; s < C::NS; ++s) refill.advance(p);
            if (refill.u < p.units) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                issue_unit<FAM, DK, UB, F32STATE, BPW>(p, refill, stage, bar);
            }
        }
    }
    return true;
}

// Resident CTAs per SM the register budget is sized for: Bounded Directional
// Rounding re-decodes the previous codes while requantizing and needs more
// registers than the plain rules.
template <int FAM, int DK, int UB, bool F32STATE, int RND, int BPW>
constexpr int decode_min_blocks() {
    using C = DecodeCfg<FAM, DK, UB, F32STATE, BPW>;
    // BDR: about 168 registers per thread (65536 / (168 * 128) = 3 CTAs of 128 threads)
    // (the pure-write window's slot pass needs as many, and so does stochastic
    // rounding at dk = 256 with its pair exchanges, run with two blocks per unit)
    constexpr bool wide = (RND & kRndBdr) != 0 || is_pw_family(FAM) || (C::SPLIT > 1 && (RND & kRndSr) != 0);
    return wide ? 384 / C::NT : C::MINB;
}

template <int FAM, int DK, int UB, bool F32STATE, int RND, int BPW>
__global__ void __launch_bounds__(DecodeCfg<FAM, DK, UB, F32STATE, BPW>::NT,
                                  (decode_min_blocks<FAM, DK, UB, F32STATE, RND, BPW>()))
    rsq_decode_kernel(const __grid_constant__ DecodeParams p) {
    using C = DecodeCfg<FAM, DK, UB, F32STATE, BPW>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x;
    const int lane = tid & 31, w = tid >> 5;
    const int g = lane >> 2, cw = lane & 3;
    const uint32_t bar0 = smem_u32(smem + C::OFF_BAR);

    if (tid == 0) {
        uint32_t* cnt = reinterpret_cast<uint32_t*>(smem + C::OFF_CNT);
        for (int s = 0; s < C::NS; ++s) {
            mbar_init(bar0 + 8 * s, 1);
            if constexpr (C::PW) mbar_init(smem_u32(smem + C::OFF_SBAR) + 8 * s, C::NPROD);
            cnt[s] = 0u;
        }
        if constexpr (C::SPLIT > 1)
            for (int b = 0; b < UB; ++b) mbar_init(smem_u32(smem + C::OFF_XBAR) + 8 * b, C::SPLIT);
        fence_mbar_init();
    }
    __syncthreads();
    UnitIt cur;
    cur.init(blockIdx.x, p);
    if (tid == 0) {
        UnitIt it = cur;
        for (int s = 0; s < C::NS; ++s) {
            if (it.u < p.units) issue_unit<FAM, DK, UB, F32STATE, BPW>(p, it, smem + s * C::STAGE, bar0 + 8 * s);
            it.advance(p);
        }
    }
    Gates gt = {0.f, 0.f, 0.f, 0.f};
    if (cur.u < p.units) gt = load_gates<FAM>(p, cur);
    int stage = 0;
    uint32_t parity = 0;
    uint32_t xphase = 0;  // phases of the block's exchange barrier (d_k = 256)
    // A warp that stops early (a bounded wait ran out) first waits, again
    // bounded, for the stage copies that may still be in flight towards this
    // CTA's shared memory: at every stage whose next unit exists, the phase
    // this warp would wait for next (a copy not yet issued, which a slower
    // warp may still issue, is waited for by that warp when it stops).  The
    // last warp of the CTA to stop has then seen every copy the CTA issued land
    // (or given up on it after the limit).
    auto stop = [&](const UnitIt& at, int stage_now, uint32_t parity_now) {
        if (lane == 0) atomicOr(p.flag, kFlagTimeout);
        for (int s = 0; s < C::NS; ++s) {
            const int ahead = (s - stage_now + C::NS) % C::NS;  // units between this one and stage s's next
            if (static_cast<long long>(at.u) + static_cast<long long>(ahead) * p.grid >= p.units) continue;
            mbar_wait(bar0 + 8 * s, s >= stage_now ? parity_now : (parity_now ^ 1u), kDrainIters);
        }
        __syncwarp();
    };
    while (cur.u < p.units) {
        UnitIt nxt = cur;
        nxt.advance(p);
        Gates ng = gt;
        if (nxt.u < p.units) ng = load_gates<FAM>(p, nxt);
        const uint32_t bar = bar0 + 8 * stage;
        const bool ok = mbar_wait(bar, parity, p.wait_iters);
        if (__any_sync(0xffffffffu, !ok)) {
            stop(cur, stage, parity);
            return;  // this warp stops; the others see their own waits expire
        }
        uint8_t* st = smem + stage * C::STAGE;
        bool done = true;
#pragma unroll 1
        for (int wblk = 0; wblk < C::BPW && done; ++wblk) {
            if constexpr (F32STATE) {
                done = process_block<FAM, DK, UB, true, 0, 32, BPW>(p, cur, st, smem, stage, bar, parity, xphase, gt,
                                                                    w, lane, g, cw, wblk);
            } else {
                if (p.head_bits[cur.h] == 8)
                    done = process_block<FAM, DK, UB, false, RND, 8, BPW>(p, cur, st, smem, stage, bar, parity, xphase,
                                                                          gt, w, lane, g, cw, wblk);
                else
                    done = process_block<FAM, DK, UB, false, RND, 4, BPW>(p, cur, st, smem, stage, bar, parity, xphase,
                                                                          gt, w, lane, g, cw, wblk);
            }
        }
        if (!done) {  // a bounded wait inside the block ran out (window slot results, pair exchange)
            stop(cur, stage, parity);
            return;
        }
        cur = nxt;
        gt = ng;
        if (++stage == C::NS) {
            stage = 0;
            parity ^= 1u;
        }
    }
}

// Kernel attributes for one instantiation.
template <int FAM, int DK, int UB, bool F32, int RND, int BPW = 1>
int decode_info_one(int* threads, size_t* smem, const void** func) {
    using C = DecodeCfg<FAM, DK, UB, F32, BPW>;
    *threads = C::NT;
    *smem = C::SMEM;
    *func = reinterpret_cast<const void*>(&rsq_decode_kernel<FAM, DK, UB, F32, RND, BPW>);
    return 0;
}

// All (dk, blocks per unit, blocks per warp) instantiations of one family for
// the rounding rules RND0, RNDS... (a full-precision state ignores the
// rounding: it is built with the first rule only, when that rule is plain
// nearest rounding).  The rules are split over translation units so the
// instantiations compile in parallel.
template <int FAM, int DK, int UB, int BPW, int RND0, int... RNDS>
int decode_info_rules(bool f32state, int rnd, int* threads, size_t* smem, const void** func) {
    if (f32state) {
        if constexpr (RND0 == 0 && BPW == 1)
            return decode_info_one<FAM, DK, UB, true, 0>(threads, smem, func);
        else
            return -1;
    }
    int found = -1;
    if (rnd == RND0) found = decode_info_one<FAM, DK, UB, false, RND0, BPW>(threads, smem, func);
    ((found != 0 && rnd == RNDS ? (found = decode_info_one<FAM, DK, UB, false, RNDS, BPW>(threads, smem, func)) : 0),
     ...);
    return found;
}

// Two blocks per warp are built for d_k = 128 units of four blocks, but not for
// the pure-write window nor for Bounded Directional Rounding: its second decode
// of the previous codes does not fit two blocks' work into the registers of
// six 64-thread CTAs per SM (the instances spilled 400-550 bytes per thread).
template <int FAM, int... RNDS>
int decode_info_family(int dk, int ub, int bpw, bool f32state, int rnd, int* threads, size_t* smem,
                       const void** func) {
    constexpr bool kAnyBdr = (((RNDS & kRndBdr) != 0) || ...);
    if (bpw == 2) {
        if constexpr (!is_pw_family(FAM) && !kAnyBdr) {
            if (dk == 128 && ub == 4 && !f32state)
                return decode_info_rules<FAM, 128, 4, 2, RNDS...>(f32state, rnd, threads, smem, func);
        }
        return -1;
    }
    if (bpw != 1) return -1;
#define RSQ_CASE(DK_, UB_)                                                                 \
    if (dk == DK_ && ub == UB_) return decode_info_rules<FAM, DK_, UB_, 1, RNDS...>(f32state, rnd, threads, smem, func);
    RSQ_CASE(16, 1) RSQ_CASE(16, 2) RSQ_CASE(16, 4)
    RSQ_CASE(32, 1) RSQ_CASE(32, 2) RSQ_CASE(32, 4)
    RSQ_CASE(64, 1) RSQ_CASE(64, 2) RSQ_CASE(64, 4)
    RSQ_CASE(128, 1) RSQ_CASE(128, 2) RSQ_CASE(128, 4)
    if constexpr (!is_pw_family(FAM)) {
        RSQ_CASE(256, 1)
        // BDR at d_k = 256 runs one block per unit (the host never picks more)
        if constexpr (!kAnyBdr) {
            RSQ_CASE(256, 2) RSQ_CASE(256, 4)
        }
    }
#undef RSQ_CASE
    return -1;
}

}  // namespace rsq
