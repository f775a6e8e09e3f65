// decode_ka.cu -- Gated DeltaNet decode step with key-axis scale groups.
//
// The grouping ablation of LoReS ("Quantizing Recurrent Language Models Is
// Easier Than You Think", section "(1/4) Scale grouping"): one scale per key
// row, s_i = max_j |S_ij| / r, instead of one per value column.  A row's
// maximum runs over all d_v columns of the head, so a CTA works on one head at
// a time: warp w holds the 16-column block w (the same lane tile as the
// value-axis kernel), the row maxima of the warps meet in shared memory, and
// CTA barriers separate the phases.  CTAs are persistent and walk the heads
// with a grid stride; each head (its codes, row scales, q, k and v) arrives in
// a two-stage shared-memory ring by bulk asynchronous copies, so the next
// head's copy overlaps this head's arithmetic.  Every thread takes the same
// path through the barriers: the one early exit (a stage wait that ran out) is
// decided for the whole CTA at once, at the head's first barrier.
//
// Per head, in the canonical order the oracle follows:
//   u_j = sum_i c_ij (s_i k_i)  (8 partials + XOR butterfly),
//   w_j = beta * fma(-alpha, u_j, v_j),   S_ij = fma(c_ij, alpha s_i, k_i w_j),
//   o_j = sum_i S_ij q_i,   m_i = max_j |S_ij|,   s_i = m_i / r,
//   inv_i = r / m_i rounded toward zero,   codes as in the value-axis kernel.
#include <cuda_runtime.h>

#include "rsq_internal.h"
#include "rsq_tile.cuh"

namespace rsq {
namespace {

template <int DK>
struct KaCfg {
    static constexpr int RPT = DK / kR;
    static constexpr int PST = RPT + 2;          // padded row-group stride of the pair arrays
    static constexpr int PAIRS = kR * PST;        // uint64 per pair array
};

// One head in a stage: codes (sized for 8-bit heads), the row scales, q and k
// (d_k each) and v (d_v), the vectors as delivered (bf16 or f32); every part
// at a 16-byte aligned offset.
constexpr int kKaStages = 2;
struct KaStage {
    int off_s, off_q, off_k, off_v, bytes;
    __host__ __device__ KaStage(int dk, int dv) {
        off_s = dk * dv;
        off_q = off_s + dk * 4;
        off_k = off_q + dk * 4;
        off_v = off_k + dk * 4;
        bytes = (off_v + dv * 4 + 127) / 128 * 128;
    }
};

__device__ __forceinline__ float ka_vec(const void* base, long long e, bool bf16) {
    if (bf16) return bf16_bits_to_f32(static_cast<const uint16_t*>(base)[e]);
    return static_cast<const float*>(base)[e];
}

// Requantize this lane's rows with one multiplier per row (pairs (inv_i, inv_i)
// at invp[k] for row g + 8k) and store them; nearest or Philox stochastic
// rounding (16- or 8-bit uniforms: rule bits RND) as in the value-axis
// requantizer.
template <int BITS, int RND, int RPT>
__device__ __forceinline__ void ka_requantize_store(const uint64_t (&S2)[RPT][2], const uint64_t* invp,
                                                    uint8_t* dst, int g, int cw, uint32_t gcol,
                                                    uint32_t h, uint32_t b, uint32_t step,
                                                    const PhiloxKeys& rk) {
    constexpr bool SR = (RND & kRndSr) != 0;
    constexpr bool U8 = SR && (RND & kRndU8) != 0;
    uint8_t* const row0 = dst + (BITS == 8 ? g * 16 + 4 * cw : g * 8 + 2 * cw);
    auto store_row = [&](int k, uint32_t word) {
        if constexpr (BITS == 8)
            *reinterpret_cast<uint32_t*>(row0 + k * (kR * 16)) = word;
        else
            *reinterpret_cast<uint16_t*>(row0 + k * (kR * 8)) = static_cast<uint16_t>(word);
    };
    constexpr float kOff = (BITS == 8) ? 128.0f : 8.0f;
    if constexpr (!SR) {
        const uint64_t moff = pk(kMagic + kOff, kMagic + kOff);
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            float t0, t1, t2, t3;
            upk(fma2(S2[k][0], invp[k], moff), t0, t1);
            upk(fma2(S2[k][1], invp[k], moff), t2, t3);
            store_row(k, pack_row<BITS, 0>(__float_as_uint(t0), __float_as_uint(t1), __float_as_uint(t2),
                                           __float_as_uint(t3)));
        }
    } else if constexpr (U8) {
        constexpr uint32_t vb = (BITS == 8) ? kSr8Bits8 : kSr8Bits4;
        sr8_words<RPT, kR>(g, gcol, h, b, step, rk, [&](int kk, uint32_t word) {
            uint64_t V01, V23;
            sr8_offsets(word, vb, V01, V23);
            float t0, t1, t2, t3;
            upk(fma2(S2[kk][0], invp[kk], V01), t0, t1);
            upk(fma2(S2[kk][1], invp[kk], V23), t2, t3);
            store_row(kk, pack_row<BITS, 1>(__float_as_uint(t0), __float_as_uint(t1), __float_as_uint(t2),
                                            __float_as_uint(t3)));
        });
    } else {
        constexpr uint32_t vb = (BITS == 8) ? kSrBits8 : kSrBits4;
        const uint64_t mm = pk(kMagic, kMagic);
#pragma unroll
        for (int k = 0; k < RPT / 2; ++k) {
            const uint32_t i = static_cast<uint32_t>(g + kR * k);  // partner row i + dk/2
            const U4 rnd = philox4x32_10(U4{i | (gcol << 16), h, b, step}, rk.k0, rk.k1);
            const uint32_t u[2][2] = {{rnd.x, rnd.y}, {rnd.z, rnd.w}};
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int kk = k + half * (RPT / 2);
                const uint32_t w0 = u[half][0], w1 = u[half][1];
                const uint64_t V01 = pk(__uint_as_float(vb | (w0 & 0xFFFFu)), __uint_as_float(umulhi_add(w0, 0x10000u, vb)));
                const uint64_t V23 = pk(__uint_as_float(vb | (w1 & 0xFFFFu)), __uint_as_float(umulhi_add(w1, 0x10000u, vb)));
                uint64_t t01 = fma2(S2[kk][0], invp[kk], V01);
                uint64_t t23 = fma2(S2[kk][1], invp[kk], V23);
                if constexpr (BITS == 8) {
                    t01 = add2_rm(t01, mm);
                    t23 = add2_rm(t23, mm);
                }
                float t0, t1, t2, t3;
                upk(t01, t0, t1);
                upk(t23, t2, t3);
                if constexpr (BITS == 8)
                    store_row(kk, pack_row<8, 0>(__float_as_uint(t0), __float_as_uint(t1), __float_as_uint(t2),
                                                 __float_as_uint(t3)));
                else
                    store_row(kk, pack_row<4, 2>(__float_as_uint(t0), __float_as_uint(t1), __float_as_uint(t2),
                                                 __float_as_uint(t3)));
            }
        }
    }
}

// Issue the bulk copies of head hu into a stage (one thread).
template <int DK>
__device__ __forceinline__ void ka_issue(const DecodeParams& p, int hu, uint8_t* st, uint32_t bar,
                                         const KaStage& L) {
    const int b = hu / p.H, h = hu - b * p.H;
    const uint32_t cb = static_cast<uint32_t>(DK * p.dv * p.head_bits[h] / 8);
    const uint32_t esz = p.in_bf16 ? 2u : 4u;
    const uint32_t vk = DK * esz, vv = static_cast<uint32_t>(p.dv) * esz;
    const uint32_t s = smem_u32(st);
    mbar_arrive_expect_tx(bar, cb + DK * 4u + 2u * vk + vv);
    bulk_g2s(s, p.codes_in + (long long)b * p.row_bytes + p.head_off[h], cb, bar);
    bulk_g2s(s + L.off_s, p.scales_in + (long long)hu * DK, DK * 4u, bar);
    bulk_g2s(s + L.off_q, static_cast<const char*>(p.vA) + (long long)hu * vk, vk, bar);
    bulk_g2s(s + L.off_k, static_cast<const char*>(p.vB) + (long long)hu * vk, vk, bar);
    bulk_g2s(s + L.off_v, static_cast<const char*>(p.vC) + (long long)hu * vv, vv, bar);
}

// One head from its stage.  `ok`: this thread's wait for the stage succeeded;
// the first barrier also decides, for the whole CTA, whether every thread's did
// (false: nothing was computed, the caller stops).  After the row-maxima barrier
// no thread reads the stage again, so thread 0 refills it there with head
// `refill` (if any).  alpha, beta: the head's gates, loaded one head ahead.
template <int DK, int BITS, int RND>
__device__ __forceinline__ bool ka_head(const DecodeParams& p, uint8_t* st, const KaStage& L, uint8_t* work,
                                        uint32_t bar, int b, int h, int hu, int refill, bool ok, float alpha,
                                        float beta) {
    using K = KaCfg<DK>;
    constexpr int RPT = K::RPT;
    constexpr int BLOCK_BYTES = DK * kBlockCols * BITS / 8;
    constexpr float r = float((1 << (BITS - 1)) - 1);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nt = blockDim.x, nw = nt >> 5;
    const int g = lane >> 2, cw = lane & 3;
    const bool bf16 = p.in_bf16 != 0;
    uint64_t* pq = reinterpret_cast<uint64_t*>(work);
    uint64_t* pkk = pq + K::PAIRS;   // k
    uint64_t* pks = pkk + K::PAIRS;  // s_i k_i
    uint64_t* pas = pks + K::PAIRS;  // alpha s_i
    uint64_t* pin = pas + K::PAIRS;  // inv_i (after the row maxima)
    float* rowmax = reinterpret_cast<float*>(pin + K::PAIRS);  // [nw][DK]

    // ---- key-axis vectors and row scales as duplicated pairs (shared by all warps)
    for (int i = tid; i < DK && ok; i += nt) {
        const float q = ka_vec(st + L.off_q, i, bf16);
        const float k = ka_vec(st + L.off_k, i, bf16);
        const float s = reinterpret_cast<const float*>(st + L.off_s)[i];
        const int pos = (i & (kR - 1)) * K::PST + i / kR;
        const float ks = __fmul_rn(s, k), as = __fmul_rn(alpha, s);
        pq[pos] = pk(q, q);
        pkk[pos] = pk(k, k);
        pks[pos] = pk(ks, ks);
        pas[pos] = pk(as, as);
    }
    if (!__syncthreads_and(ok)) return false;

    // ---- this warp's block: decode, update, read out -------------------------
    const int j0 = w * kBlockCols;
    uint64_t S2[RPT][2];
    load_codes<BITS, RPT>(st + w * BLOCK_BYTES, g, cw, S2);
    const uint64_t* kq = pq + g * K::PST;
    const uint64_t* kk = pkk + g * K::PST;
    const uint64_t* kks = pks + g * K::PST;
    const uint64_t* kas = pas + g * K::PST;
    uint64_t a01 = pk(0.f, 0.f), a23 = pk(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < RPT; k += 2) {
        const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(kks + k);
        a01 = fma2(S2[k][0], x.x, a01);
        a23 = fma2(S2[k][1], x.x, a23);
        a01 = fma2(S2[k + 1][0], x.y, a01);
        a23 = fma2(S2[k + 1][1], x.y, a23);
    }
    const float4 u4 = gather_cols(reduce_scatter4(unpk4(a01, a23), g, AddOp()), cw, 0);
    const float uv[4] = {u4.x, u4.y, u4.z, u4.w};
    float wj[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float v = ka_vec(st + L.off_v, j0 + 4 * cw + j, bf16);
        wj[j] = __fmul_rn(beta, __fmaf_rn(-alpha, uv[j], v));
    }
    const uint64_t W01 = pk(wj[0], wj[1]), W23 = pk(wj[2], wj[3]);
#pragma unroll
    for (int k = 0; k < RPT; k += 2) {
        const ulonglong2 ka = *reinterpret_cast<const ulonglong2*>(kas + k);
        const ulonglong2 kv = *reinterpret_cast<const ulonglong2*>(kk + k);
        S2[k][0] = fma2(S2[k][0], ka.x, mul2(kv.x, W01));
        S2[k][1] = fma2(S2[k][1], ka.x, mul2(kv.x, W23));
        S2[k + 1][0] = fma2(S2[k + 1][0], ka.y, mul2(kv.y, W01));
        S2[k + 1][1] = fma2(S2[k + 1][1], ka.y, mul2(kv.y, W23));
    }
    uint64_t o01 = pk(0.f, 0.f), o23 = pk(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < RPT; k += 2) {
        const ulonglong2 x = *reinterpret_cast<const ulonglong2*>(kq + k);
        o01 = fma2(S2[k][0], x.x, o01);
        o23 = fma2(S2[k][1], x.x, o23);
        o01 = fma2(S2[k + 1][0], x.y, o01);
        o23 = fma2(S2[k + 1][1], x.y, o23);
    }
    const float o = reduce_scatter4(unpk4(o01, o23), g, AddOp());
    if (g < 4) p.out[(long long)hu * p.dv + j0 + 4 * cw + col_of(g)] = o;

    // ---- row maxima: this warp's 16 columns, then across the warps -----------
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const float4 x = unpk4(S2[k][0], S2[k][1]);
        float m = max3_nan(fabsf(x.x), fabsf(x.y), max_nan(fabsf(x.z), fabsf(x.w)));
        m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, 2));
        if (cw == 0) rowmax[w * DK + g + kR * k] = m;
    }
    __syncthreads();
    // every read of the stage is behind the barrier above: refill it (the
    // proxy fence orders those generic-proxy reads before the async writes)
    if (tid == 0 && refill >= 0) {
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        ka_issue<DK>(p, refill, st, bar, L);
    }
    for (int i = tid; i < DK; i += nt) {
        float m = 0.f;
        for (int ww = 0; ww < nw; ++ww) m = max_nan(m, rowmax[ww * DK + i]);
        const float s = __fdiv_rn(m, r);
        float inv = 0.f;
        if (!isfinite(m)) {
            inv = -0.0f;  // marks a non-finite row
        } else if (m > 0.f) {
            const float q = __fdiv_rn(r, m);
            inv = (__fmaf_rn(q, m, -r) > 0.f) ? __uint_as_float(__float_as_uint(q) - 1u) : q;
        }
        p.scales_out[(long long)hu * DK + i] = s;
        pin[(i & (kR - 1)) * K::PST + i / kR] = pk(inv, inv);
    }
    __syncthreads();

    // ---- requantize with the row multipliers ----------------------------------
    const uint64_t* ki = pin + g * K::PST;
    uint64_t invp[RPT];
#pragma unroll
    for (int k = 0; k < RPT; ++k) invp[k] = ki[k];
    const long long rowoff = (long long)b * p.row_bytes + p.head_off[h] + (long long)w * BLOCK_BYTES;
    uint8_t* dst = p.codes_out + rowoff;
    const uint32_t gcol = static_cast<uint32_t>(j0 / 4 + cw);
    ka_requantize_store<BITS, RND, RPT>(S2, invp, dst, g, cw, gcol, h, b, p.step, p.rk);
    // rare: non-finite rows (multiplier -0.0) are stored as the zero code
    bool bad = false;
#pragma unroll
    for (int k = 0; k < RPT; ++k) bad |= is_neg_zero(__uint_as_float(static_cast<uint32_t>(invp[k])));
    if (bad) {
        if (cw == 0 && g == 0) atomicOr(p.flag, kFlagNonFinite);
#pragma unroll
        for (int k = 0; k < RPT; ++k)
            if (is_neg_zero(__uint_as_float(static_cast<uint32_t>(invp[k])))) {
                S2[k][0] = pk(0.f, 0.f);
                S2[k][1] = pk(0.f, 0.f);
            }
        ka_requantize_store<BITS, RND, RPT>(S2, invp, dst, g, cw, gcol, h, b, p.step, p.rk);
    }
    return true;
}

// Shared memory: the stages, then the pair arrays and row maxima of the head in
// work, then one mbarrier per stage.
template <int DK>
__host__ __device__ inline size_t ka_work_bytes(int nw) {
    return 5 * KaCfg<DK>::PAIRS * sizeof(uint64_t) + static_cast<size_t>(nw) * DK * sizeof(float);
}
template <int DK>
__host__ __device__ inline size_t ka_smem(int dv) {
    return static_cast<size_t>(kKaStages) * KaStage(DK, dv).bytes + ka_work_bytes<DK>(dv / kBlockCols) +
           kKaStages * 8;
}

template <int DK, int RND>
__global__ void __launch_bounds__(512) rsq_decode_ka_kernel(const __grid_constant__ DecodeParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x;
    const int heads = p.B * p.H, grid = static_cast<int>(gridDim.x);
    const KaStage L(DK, p.dv);
    uint8_t* work = smem + kKaStages * L.bytes;
    const uint32_t bar0 = smem_u32(work + ka_work_bytes<DK>(p.dv / kBlockCols));
    if (tid == 0) {
        for (int s = 0; s < kKaStages; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncthreads();
    // (failure-detection tests: with p.withhold the first stage is never
    // filled, so its wait runs out while the second stage's copies are in flight)
    if (tid == 0)
        for (int s = 0; s < kKaStages; ++s) {
            const int hu = static_cast<int>(blockIdx.x) + s * grid;
            if (hu < heads && !(p.withhold && s == 0)) ka_issue<DK>(p, hu, smem + s * L.bytes, bar0 + 8 * s, L);
        }
    int stage = 0;
    uint32_t parity = 0;
    // the gates of the CTA's first head; each iteration loads the next head's
    float alpha = 0.f, beta = 0.f;
    if (static_cast<int>(blockIdx.x) < heads) {
        alpha = __ldg(p.g0 + blockIdx.x);
        beta = __ldg(p.g1 + blockIdx.x);
    }
    for (int hu = static_cast<int>(blockIdx.x); hu < heads; hu += grid) {
        const uint32_t bar = bar0 + 8 * stage;
        const bool ok = mbar_wait(bar, parity, p.wait_iters);
        float na = 0.f, nb = 0.f;
        if (hu + grid < heads) {
            na = __ldg(p.g0 + hu + grid);
            nb = __ldg(p.g1 + hu + grid);
        }
        const int b = hu / p.H, h = hu - b * p.H;
        const long long next = static_cast<long long>(hu) + static_cast<long long>(kKaStages) * grid;
        const int refill = next < heads ? static_cast<int>(next) : -1;
        uint8_t* st = smem + stage * L.bytes;
        const bool done = (p.head_bits[h] == 8)
                              ? ka_head<DK, 8, RND>(p, st, L, work, bar, b, h, hu, refill, ok, alpha, beta)
                              : ka_head<DK, 4, RND>(p, st, L, work, bar, b, h, hu, refill, ok, alpha, beta);
        if (!done) {
            // a stage wait ran out (decided for the whole CTA): the CTA leaves,
            // first waiting (bounded) for every stage copy it issued that has
            // not landed, so none writes into a CTA that is gone
            if (tid == 0) {
                atomicOr(p.flag, kFlagTimeout);
                for (int s = 0; s < kKaStages; ++s) {
                    const int ahead = (s - stage + kKaStages) % kKaStages;
                    if (static_cast<long long>(hu) + static_cast<long long>(ahead) * grid >= heads) continue;
                    mbar_wait(bar0 + 8 * s, s >= stage ? parity : (parity ^ 1u), kDrainIters);
                }
            }
            return;
        }
        alpha = na;
        beta = nb;
        if (++stage == kKaStages) {
            stage = 0;
            parity ^= 1u;
        }
    }
}

// Quantize a full-precision head (natural [dk][dv] layout) with key-axis
// scales: warp w owns block w, row maxima meet in shared memory.
template <int DK, int BITS, int RND>
__device__ __forceinline__ void ka_quantize_head(const QuantParams& p, uint8_t* smem, int b, int h, int hu) {
    using K = KaCfg<DK>;
    constexpr int RPT = K::RPT;
    constexpr int BLOCK_BYTES = DK * kBlockCols * BITS / 8;
    constexpr float r = float((1 << (BITS - 1)) - 1);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, nt = blockDim.x, nw = nt >> 5;
    const int g = lane >> 2, cw = lane & 3;
    uint64_t* pin = reinterpret_cast<uint64_t*>(smem);
    float* rowmax = reinterpret_cast<float*>(pin + K::PAIRS);
    const int j0 = w * kBlockCols;
    const float* src = p.S + (long long)hu * DK * p.dv + j0 + 4 * cw;
    uint64_t S2[RPT][2];
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const ulonglong2 t = __ldg(reinterpret_cast<const ulonglong2*>(src + (long long)(g + kR * k) * p.dv));
        S2[k][0] = t.x;
        S2[k][1] = t.y;
        const float4 x = unpk4(t.x, t.y);
        float m = max3_nan(fabsf(x.x), fabsf(x.y), max_nan(fabsf(x.z), fabsf(x.w)));
        m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = max_nan(m, __shfl_xor_sync(0xffffffffu, m, 2));
        if (cw == 0) rowmax[w * DK + g + kR * k] = m;
    }
    __syncthreads();
    for (int i = tid; i < DK; i += nt) {
        float m = 0.f;
        for (int ww = 0; ww < nw; ++ww) m = max_nan(m, rowmax[ww * DK + i]);
        float inv = 0.f;
        if (!isfinite(m)) {
            inv = -0.0f;
        } else if (m > 0.f) {
            const float q = __fdiv_rn(r, m);
            inv = (__fmaf_rn(q, m, -r) > 0.f) ? __uint_as_float(__float_as_uint(q) - 1u) : q;
        }
        p.scales[(long long)hu * DK + i] = __fdiv_rn(m, r);
        pin[(i & (kR - 1)) * K::PST + i / kR] = pk(inv, inv);
    }
    __syncthreads();
    uint64_t invp[RPT];
    bool bad = false;
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        invp[k] = pin[g * K::PST + k];
        if (is_neg_zero(__uint_as_float(static_cast<uint32_t>(invp[k])))) {
            bad = true;
            S2[k][0] = pk(0.f, 0.f);
            S2[k][1] = pk(0.f, 0.f);
        }
    }
    if (bad && cw == 0 && g == 0) atomicOr(p.flag, kFlagNonFinite);
    uint8_t* dst = p.codes + (long long)b * p.row_bytes + p.head_off[h] + (long long)w * BLOCK_BYTES;
    ka_requantize_store<BITS, RND, RPT>(S2, invp, dst, g, cw, static_cast<uint32_t>(j0 / 4 + cw), h, b, p.step,
                                       p.rk);
}

template <int DK>
__global__ void __launch_bounds__(512) rsq_quantize_ka_kernel(const __grid_constant__ QuantParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int hu = blockIdx.x;
    const int b = hu / p.H, h = hu - b * p.H;
    const bool bits8 = p.head_bits[h] == 8;
    constexpr int kSr8 = kRndSr | kRndU8;
    if (p.rnd == kSr8) {
        if (bits8) ka_quantize_head<DK, 8, kSr8>(p, smem, b, h, hu);
        else ka_quantize_head<DK, 4, kSr8>(p, smem, b, h, hu);
    } else if (p.rnd == kRndSr) {
        if (bits8) ka_quantize_head<DK, 8, kRndSr>(p, smem, b, h, hu);
        else ka_quantize_head<DK, 4, kRndSr>(p, smem, b, h, hu);
    } else {
        if (bits8) ka_quantize_head<DK, 8, 0>(p, smem, b, h, hu);
        else ka_quantize_head<DK, 4, 0>(p, smem, b, h, hu);
    }
}

template <int DK>
int launch_quantize_ka_dk(const QuantParams& p, void* stream) {
    const int nw = p.dv / kBlockCols;
    const size_t smem = KaCfg<DK>::PAIRS * sizeof(uint64_t) + static_cast<size_t>(nw) * DK * sizeof(float);
    rsq_quantize_ka_kernel<DK><<<p.B * p.H, 32 * nw, smem, static_cast<cudaStream_t>(stream)>>>(p);
    return static_cast<int>(cudaGetLastError());
}

template <int DK>
const void* ka_func(int rnd) {
    constexpr int kSr8 = kRndSr | kRndU8;
    return rnd == kSr8    ? reinterpret_cast<const void*>(&rsq_decode_ka_kernel<DK, kSr8>)
           : rnd == kRndSr ? reinterpret_cast<const void*>(&rsq_decode_ka_kernel<DK, kRndSr>)
                           : reinterpret_cast<const void*>(&rsq_decode_ka_kernel<DK, 0>);
}

template <int DK>
int launch_ka_dk(const DecodeParams& p, void* stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(32 * (p.dv / kBlockCols));
    cfg.dynamicSmemBytes = ka_smem<DK>(p.dv);
    cfg.stream = static_cast<cudaStream_t>(stream);
    void* args[] = {const_cast<DecodeParams*>(&p)};
    return static_cast<int>(cudaLaunchKernelExC(&cfg, ka_func<DK>(p.rnd), args));
}

template <int DK>
int ka_info_dk(int dv, int rnd, int* threads, size_t* smem, const void** func) {
    *threads = 32 * (dv / kBlockCols);
    *smem = ka_smem<DK>(dv);
    *func = ka_func<DK>(rnd);
    return 0;
}

}  // namespace

int launch_quantize_ka(int dk, const QuantParams& p, void* stream) {
    switch (dk) {
        case 16: return launch_quantize_ka_dk<16>(p, stream);
        case 32: return launch_quantize_ka_dk<32>(p, stream);
        case 64: return launch_quantize_ka_dk<64>(p, stream);
        case 128: return launch_quantize_ka_dk<128>(p, stream);
        default: return static_cast<int>(cudaErrorInvalidValue);
    }
}

int decode_ka_info(int dk, int dv, int rnd, int* threads, size_t* smem, const void** func) {
    switch (dk) {
        case 16: return ka_info_dk<16>(dv, rnd, threads, smem, func);
        case 32: return ka_info_dk<32>(dv, rnd, threads, smem, func);
        case 64: return ka_info_dk<64>(dv, rnd, threads, smem, func);
        case 128: return ka_info_dk<128>(dv, rnd, threads, smem, func);
        default: return -1;
    }
}

int launch_decode_ka(int dk, const DecodeParams& p, void* stream) {
    switch (dk) {
        case 16: return launch_ka_dk<16>(p, stream);
        case 32: return launch_ka_dk<32>(p, stream);
        case 64: return launch_ka_dk<64>(p, stream);
        case 128: return launch_ka_dk<128>(p, stream);
        default: return static_cast<int>(cudaErrorInvalidValue);
    }
}

}  // namespace rsq
