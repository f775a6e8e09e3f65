// decode.cu -- fused quantized recurrent-state decode step (sm_100a).
//
// One persistent CTA per resident slot walks the work units (b, h, column
// block) with a grid stride.  Per unit it:
//   1. receives the unit's code tile, scales and input vectors in a shared-
//      memory stage filled by bulk asynchronous copies (issued NS units ahead),
//   2. decodes the codes to exact floats,
//   3. (Gated DeltaNet) forms u = S^T k as s_j * sum_i c_ij k_i,
//   4. updates the state in registers (full precision),
//   5. reads out o = S^T q (GDN) or y = S^T C + D x (Mamba-2) from that FP32 state,
//   6. takes each column's absmax as its new scale (the dynamic "noisy" scale),
//   7. requantizes (round-to-nearest or Philox stochastic rounding) and stores.
// Method: LoReS ("Quantizing Recurrent Language Models Is Easier Than You
// Think", sections "LoReS: State Quantization", "(1/4) Scale grouping", "(3/4)
// Rounding"); recurrences as named in "Preserving Updates in Low-Bit Recurrent
// State Quantization" (abstract).  No tensor cores: per head this is two
// matrix-vector products over a state read once from HBM.
#include <cuda_runtime.h>

#include "rsq_internal.h"
#include "rsq_tile.cuh"

namespace rsq {

constexpr uint32_t kWaitIters = 1u << 22;  // bounded mbarrier waits (error flag on expiry)

template <int FAM, int DK, int CB, bool F32STATE>
struct DecodeCfg {
    using L = Layout<DK, CB>;
    static constexpr int NS = F32STATE ? 3 : 4;                      // pipeline stages
    static constexpr int CODE_BYTES = F32STATE ? DK * CB * 4 : DK * CB;  // largest tile (8-bit)
    static constexpr int OFF_SCALES = CODE_BYTES;
    static constexpr int OFF_VA = OFF_SCALES + CB * 4;   // GDN q / Mamba-2 C   (<= DK floats)
    static constexpr int OFF_VB = OFF_VA + DK * 4;       // GDN k / Mamba-2 B
    static constexpr int OFF_VC = OFF_VB + DK * 4;       // GDN v / Mamba-2 x   (<= CB floats)
    static constexpr int STAGE = (OFF_VC + CB * 4 + 127) / 128 * 128;
    static constexpr int OFF_VF = NS * STAGE;            // converted vectors: 2 x DK floats
    static constexpr int OFF_RED = OFF_VF + 2 * DK * 4;  // 3 x [W][CB] floats
    static constexpr int OFF_BAR = OFF_RED + 3 * L::W * CB * 4;
    static constexpr int SMEM = OFF_BAR + NS * 8;
};

struct Unit {
    int b, h, hu, cb, bits;
};

__device__ __forceinline__ Unit unit_of(const DecodeParams& p, int u, bool f32state) {
    Unit r;
    r.hu = u / p.ncb;
    r.cb = u - r.hu * p.ncb;
    r.b = r.hu / p.H;
    r.h = r.hu - r.b * p.H;
    r.bits = f32state ? 32 : p.head_bits[r.h];
    return r;
}

// Issue the bulk copies of unit u into a stage (one thread).
template <int FAM, int DK, int CB, bool F32STATE>
__device__ __forceinline__ void issue_unit(const DecodeParams& p, int u, uint8_t* stage, uint32_t bar) {
    using C = DecodeCfg<FAM, DK, CB, F32STATE>;
    const Unit un = unit_of(p, u, F32STATE);
    const uint32_t code_bytes = static_cast<uint32_t>(DK * CB * un.bits / 8);
    const uint32_t esz = p.in_bf16 ? 2u : 4u;
    const uint32_t total = code_bytes + (F32STATE ? 0u : CB * 4u) + 2u * DK * esz + CB * esz;
    const uint8_t* codes = p.codes_in + (long long)un.b * p.row_bytes + p.head_off[un.h] +
                           (long long)un.cb * code_bytes;
    const uint32_t s = smem_u32(stage);
    mbar_arrive_expect_tx(bar, total);
    bulk_g2s(s, codes, code_bytes, bar);
    if (!F32STATE)
        bulk_g2s(s + C::OFF_SCALES, p.scales_in + (long long)un.hu * p.dv + un.cb * CB, CB * 4u, bar);
    const char* vA = static_cast<const char*>(p.vA);
    const char* vB = static_cast<const char*>(p.vB);
    const char* vC = static_cast<const char*>(p.vC);
    long long rowA;
    if (FAM == RSQ_GDN) {
        rowA = (long long)un.hu * DK;  // q and k rows of this head
    } else {
        rowA = ((long long)un.b * p.ngroups + un.h / p.heads_per_group) * DK;  // C and B of the group
    }
    bulk_g2s(s + C::OFF_VA, vA + rowA * esz, DK * esz, bar);
    bulk_g2s(s + C::OFF_VB, vB + rowA * esz, DK * esz, bar);
    bulk_g2s(s + C::OFF_VC, vC + ((long long)un.hu * p.dv + un.cb * CB) * esz, CB * esz, bar);
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

// This thread's RPT consecutive entries of a permuted vector (16-byte loads when
// RPT is a multiple of 4; RPT = 2 uses one 8-byte load, aligned since rho*RPT is even).
template <int RPT>
__device__ __forceinline__ void load_rows(const float* src, float (&v)[RPT]) {
    if constexpr (RPT % 4 == 0) {
#pragma unroll
        for (int k = 0; k < RPT; k += 4) {
            const float4 t = *reinterpret_cast<const float4*>(src + k);
            v[k] = t.x; v[k + 1] = t.y; v[k + 2] = t.z; v[k + 3] = t.w;
        }
    } else {
        static_assert(RPT == 2, "rows per thread");
        const float2 t = *reinterpret_cast<const float2*>(src);
        v[0] = t.x; v[1] = t.y;
    }
}

template <int FAM, int DK, int CB, bool F32STATE, int BITS>
__device__ __forceinline__ void process_unit(const DecodeParams& p, const Unit& un,
                                             const uint8_t* stage, const float* vf, float* red,
                                             uint8_t* issue_stage, uint32_t issue_bar,
                                             int next_issue, float g0, float g1, int tid, int warp,
                                             int rgl, int cw, int rho) {
    using L = Layout<DK, CB>;
    using C = DecodeCfg<FAM, DK, CB, F32STATE>;
    constexpr int R = L::R, RPT = L::RPT;
    const bool bf16 = p.in_bf16 != 0;
    const float* fA = vf;            // permuted [R][RPT]: q (GDN) / C (Mamba-2)
    const float* fB = vf + DK;       // permuted: k (GDN) / B (Mamba-2)
    float* redA = red;
    float* redS = red + L::W * CB;
    float* redM = red + 2 * L::W * CB;

    // this thread's rows of the key-side vector
    float kv[RPT];
    load_rows<RPT>(fB + rho * RPT, kv);
    const float4 vc = ld_vec4(stage + C::OFF_VC, 4 * cw, bf16);  // v (GDN) / x (Mamba-2)
    const float vcol[4] = {vc.x, vc.y, vc.z, vc.w};

    float S[RPT][4];
    if constexpr (BITS == 32) {
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const float4 t = *reinterpret_cast<const float4*>(stage + ((rho + R * k) * CB + 4 * cw) * 4);
            S[k][0] = t.x; S[k][1] = t.y; S[k][2] = t.z; S[k][3] = t.w;
        }
    } else {
        load_codes<BITS, R, RPT, CB>(stage, rho, cw, S);  // S holds the float codes c for now
    }
    float s4[4] = {1.f, 1.f, 1.f, 1.f};
    if constexpr (BITS != 32) {
        const float4 t = *reinterpret_cast<const float4*>(stage + C::OFF_SCALES + 16 * cw);
        s4[0] = t.x; s4[1] = t.y; s4[2] = t.z; s4[3] = t.w;
    }

    // ---- state update in registers ----------------------------------------
    if constexpr (FAM == RSQ_GDN) {
        const float alpha = g0, beta = g1;
        // sum_i c_ij k_i (or sum_i S_ij k_i for a full-precision state)
        uint64_t a01 = pk(0.f, 0.f), a23 = pk(0.f, 0.f);
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const uint64_t kk = pk(kv[k], kv[k]);
            a01 = fma2(pk(S[k][0], S[k][1]), kk, a01);
            a23 = fma2(pk(S[k][2], S[k][3]), kk, a23);
        }
        float4 ck;
        upk(a01, ck.x, ck.y);
        upk(a23, ck.z, ck.w);
        ck = colsum<L::LPR, L::W, CB>(ck, redA, warp, rgl, cw);
        const float ckv[4] = {ck.x, ck.y, ck.z, ck.w};
        float wj[4], aj[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float u = (BITS == 32) ? ckv[j] : __fmul_rn(s4[j], ckv[j]);
            wj[j] = __fmul_rn(beta, __fmaf_rn(-alpha, u, vcol[j]));
            aj[j] = (BITS == 32) ? alpha : __fmul_rn(alpha, s4[j]);
        }
        const uint64_t w01 = pk(wj[0], wj[1]), w23 = pk(wj[2], wj[3]);
        const uint64_t A01 = pk(aj[0], aj[1]), A23 = pk(aj[2], aj[3]);
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const uint64_t kk = pk(kv[k], kv[k]);
            // S = c*(alpha s) + k*w   (full-precision state: alpha*S + k*w)
            const uint64_t n01 = fma2(pk(S[k][0], S[k][1]), A01, mul2(kk, w01));
            const uint64_t n23 = fma2(pk(S[k][2], S[k][3]), A23, mul2(kk, w23));
            upk(n01, S[k][0], S[k][1]);
            upk(n23, S[k][2], S[k][3]);
        }
    } else {
        const float dt = g0;
        const float a = (p.g1 != nullptr) ? g1 : expf(__fmul_rn(dt, p.A[un.h]));
        float xd[4], gj[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            xd[j] = __fmul_rn(dt, vcol[j]);
            gj[j] = (BITS == 32) ? a : __fmul_rn(a, s4[j]);
        }
        const uint64_t x01 = pk(xd[0], xd[1]), x23 = pk(xd[2], xd[3]);
        const uint64_t G01 = pk(gj[0], gj[1]), G23 = pk(gj[2], gj[3]);
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const uint64_t bb = pk(kv[k], kv[k]);
            // S = c*(a s) + B*(dt x)   (full-precision state: a*S + B*(dt x))
            const uint64_t n01 = fma2(pk(S[k][0], S[k][1]), G01, mul2(bb, x01));
            const uint64_t n23 = fma2(pk(S[k][2], S[k][3]), G23, mul2(bb, x23));
            upk(n01, S[k][0], S[k][1]);
            upk(n23, S[k][2], S[k][3]);
        }
    }

    // ---- readout (and column absmax) ---------------------------------------
    float qv[RPT];
    load_rows<RPT>(fA + rho * RPT, qv);
    uint64_t o01 = pk(0.f, 0.f), o23 = pk(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < RPT; ++k) {
        const uint64_t qq = pk(qv[k], qv[k]);
        o01 = fma2(pk(S[k][0], S[k][1]), qq, o01);
        o23 = fma2(pk(S[k][2], S[k][3]), qq, o23);
    }
    float4 o4;
    upk(o01, o4.x, o4.y);
    upk(o23, o4.z, o4.w);
    float4 m4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (BITS != 32) {
        float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k + 1 < RPT; k += 2)
#pragma unroll
            for (int j = 0; j < 4; ++j) m[j] = max3_nan(m[j], fabsf(S[k][j]), fabsf(S[k + 1][j]));
        m4 = make_float4(m[0], m[1], m[2], m[3]);
        colsum_max<L::LPR, L::W, CB>(o4, m4, redS, redM, warp, rgl, cw);
    } else {
        o4 = colsum<L::LPR, L::W, CB>(o4, redS, warp, rgl, cw);
    }
    // a single-warp unit has no barrier inside the reductions: add one so that
    // every lane's reads of the stage precede its refill
    if constexpr (L::W == 1) __syncthreads();
    // every read of this stage is done: refill it with the unit NS ahead
    if (tid == 0 && next_issue >= 0)
        issue_unit<FAM, DK, CB, F32STATE>(p, next_issue, issue_stage, issue_bar);

    const long long col0 = (long long)un.hu * p.dv + un.cb * CB + 4 * cw;
    if (FAM == RSQ_MAMBA2) {
        const float D = p.D[un.h];
        o4.x = __fmaf_rn(D, vcol[0], o4.x);
        o4.y = __fmaf_rn(D, vcol[1], o4.y);
        o4.z = __fmaf_rn(D, vcol[2], o4.z);
        o4.w = __fmaf_rn(D, vcol[3], o4.w);
    }
    if (rho == 0) *reinterpret_cast<float4*>(p.out + col0) = o4;

    const uint32_t code_bytes = static_cast<uint32_t>(DK * CB * BITS / 8);
    uint8_t* dst = p.codes_out + (long long)un.b * p.row_bytes + p.head_off[un.h] +
                   (long long)un.cb * code_bytes;
    if constexpr (BITS == 32) {
#pragma unroll
        for (int k = 0; k < RPT; ++k)
            *reinterpret_cast<float4*>(dst + ((rho + R * k) * CB + 4 * cw) * 4) =
                make_float4(S[k][0], S[k][1], S[k][2], S[k][3]);
    } else {
        const float mv[4] = {m4.x, m4.y, m4.z, m4.w};
        float sn[4], inv[4];
        unsigned bad = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) scale_and_inv<BITS>(mv[j], sn[j], inv[j], bad, j);
        if (rho == 0) *reinterpret_cast<float4*>(p.scales_out + col0) = make_float4(sn[0], sn[1], sn[2], sn[3]);
        if (bad && rho == 0) atomicOr(p.flag, kFlagNonFinite);
        const uint32_t g = static_cast<uint32_t>(un.cb * (CB / 4) + cw);
        if (p.sr)
            requantize_store<BITS, true, R, RPT, CB>(S, inv, dst, rho, cw, g, un.h, un.b, p.step,
                                                     p.key0, p.key1, bad);
        else
            requantize_store<BITS, false, R, RPT, CB>(S, inv, dst, rho, cw, g, un.h, un.b, p.step,
                                                      p.key0, p.key1, bad);
    }
}

template <int FAM, int DK, int CB, bool F32STATE>
__global__ void __launch_bounds__(Layout<DK, CB>::NT)
    rsq_decode_kernel(const __grid_constant__ DecodeParams p) {
    using L = Layout<DK, CB>;
    using C = DecodeCfg<FAM, DK, CB, F32STATE>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int cw = lane % L::LPR, rgl = lane / L::LPR;
    const int rho = warp * L::RPW + rgl;
    float* vf = reinterpret_cast<float*>(smem + C::OFF_VF);
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
    const uint32_t bar0 = smem_u32(smem + C::OFF_BAR);

    if (tid == 0) {
        for (int s = 0; s < C::NS; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncthreads();
    const int G = gridDim.x;
    if (tid == 0) {
        for (int s = 0; s < C::NS; ++s) {
            const int u = blockIdx.x + s * G;
            if (u < p.units) issue_unit<FAM, DK, CB, F32STATE>(p, u, smem + s * C::STAGE, bar0 + 8 * s);
        }
    }
    // gates of the first unit
    float g0 = 0.f, g1 = 0.f;
    if (blockIdx.x < p.units) {
        const Unit un = unit_of(p, blockIdx.x, F32STATE);
        g0 = __ldg(p.g0 + un.hu);
        g1 = p.g1 ? __ldg(p.g1 + un.hu) : 0.f;
    }
    for (int n = 0;; ++n) {
        const int u = blockIdx.x + n * G;
        if (u >= p.units) break;
        const int stage = n % C::NS;
        const uint32_t bar = bar0 + 8 * stage;
        const Unit un = unit_of(p, u, F32STATE);
        // prefetch the next unit's gates
        float ng0 = 0.f, ng1 = 0.f;
        if (u + G < p.units) {
            const Unit nx = unit_of(p, u + G, F32STATE);
            ng0 = __ldg(p.g0 + nx.hu);
            ng1 = p.g1 ? __ldg(p.g1 + nx.hu) : 0.f;
        }
        const bool ok = mbar_wait(bar, (n / C::NS) & 1, kWaitIters);
        const uint8_t* st = smem + stage * C::STAGE;
        // widen the two key-axis vectors into permuted float buffers [R][RPT]
        if (ok) {
            const bool bf16 = p.in_bf16 != 0;
            for (int e = tid; e < DK; e += L::NT) {
                const int pos = (e % L::R) * L::RPT + e / L::R;
                vf[pos] = ld_vec(st + C::OFF_VA, e, bf16);
                vf[DK + pos] = ld_vec(st + C::OFF_VB, e, bf16);
            }
        }
        if (__syncthreads_or(!ok)) {
            if (tid == 0) atomicOr(p.flag, kFlagTimeout);
            return;
        }
        const int nxt = (u + C::NS * G < p.units) ? u + C::NS * G : -1;
        if constexpr (F32STATE) {
            process_unit<FAM, DK, CB, true, 32>(p, un, st, vf, red, smem + stage * C::STAGE, bar, nxt,
                                                g0, g1, tid, warp, rgl, cw, rho);
        } else {
            if (un.bits == 8)
                process_unit<FAM, DK, CB, false, 8>(p, un, st, vf, red, smem + stage * C::STAGE, bar,
                                                    nxt, g0, g1, tid, warp, rgl, cw, rho);
            else
                process_unit<FAM, DK, CB, false, 4>(p, un, st, vf, red, smem + stage * C::STAGE, bar,
                                                    nxt, g0, g1, tid, warp, rgl, cw, rho);
        }
        g0 = ng0;
        g1 = ng1;
    }
}

// ---------------------------------------------------------------------------
// Instantiation table
// ---------------------------------------------------------------------------
template <int FAM, int DK, int CB, bool F32>
static int info_one(int* threads, size_t* smem, const void** func) {
    using C = DecodeCfg<FAM, DK, CB, F32>;
    *threads = Layout<DK, CB>::NT;
    *smem = C::SMEM;
    *func = reinterpret_cast<const void*>(&rsq_decode_kernel<FAM, DK, CB, F32>);
    return 0;
}

template <int FAM, bool F32>
static int info_dk_cb(int dk, int cb, int* threads, size_t* smem, const void** func) {
#define RSQ_CASE(DK_, CB_) \
    if (dk == DK_ && cb == CB_) return info_one<FAM, DK_, CB_, F32>(threads, smem, func);
    RSQ_CASE(16, 16) RSQ_CASE(16, 32) RSQ_CASE(16, 64)
    RSQ_CASE(32, 16) RSQ_CASE(32, 32) RSQ_CASE(32, 64)
    RSQ_CASE(64, 16) RSQ_CASE(64, 32) RSQ_CASE(64, 64)
    RSQ_CASE(128, 16) RSQ_CASE(128, 32) RSQ_CASE(128, 64)
    RSQ_CASE(256, 16) RSQ_CASE(256, 32) RSQ_CASE(256, 64)
#undef RSQ_CASE
    return -1;
}

int decode_kernel_info(int family, int dk, int cb, bool f32state, int* threads, size_t* smem,
                       const void** func) {
    if (family == RSQ_GDN)
        return f32state ? info_dk_cb<RSQ_GDN, true>(dk, cb, threads, smem, func)
                        : info_dk_cb<RSQ_GDN, false>(dk, cb, threads, smem, func);
    return f32state ? info_dk_cb<RSQ_MAMBA2, true>(dk, cb, threads, smem, func)
                    : info_dk_cb<RSQ_MAMBA2, false>(dk, cb, threads, smem, func);
}

int launch_decode(int family, int dk, int cb, bool f32state, const DecodeParams& p, int grid,
                  void* stream) {
    int threads;
    size_t smem;
    const void* func;
    if (decode_kernel_info(family, dk, cb, f32state, &threads, &smem, &func) != 0)
        return static_cast<int>(cudaErrorInvalidValue);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = static_cast<cudaStream_t>(stream);
    void* args[] = {const_cast<DecodeParams*>(&p)};
    return static_cast<int>(cudaLaunchKernelExC(&cfg, func, args));
}

}  // namespace rsq
