// rsq_internal.h -- parameter blocks shared by the host API and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>

#include "../../include/rsq.h"

namespace rsq {

// Internal family values of Gated DeltaNet with a pure-write window of 4, 8
// or 16 slots (the public family is RSQ_GDN with rsq_config.window > 0).
constexpr int kFamGdnPw = 4;  // + log2(W / 4)
constexpr int kMaxWindow = 16;
constexpr bool is_pw_family(int fam) { return fam >= kFamGdnPw && fam < kFamGdnPw + 3; }
constexpr int pw_window(int fam) { return is_pw_family(fam) ? 4 << (fam - kFamGdnPw) : 0; }

constexpr unsigned kFlagNonFinite = 1u;  // a column's absmax was inf or NaN
constexpr unsigned kFlagTimeout = 2u;    // a bounded barrier wait ran out
constexpr uint32_t kWaitIters = 1u << 22;  // default limit of a bounded barrier wait (polls)
constexpr uint32_t kDrainIters = 1u << 16; // wait for in-flight stage copies before a CTA leaves early

// The ten round keys of Philox4x32-10 for one (key0, key1): round r uses
// key0 + r * 0x9E3779B9 and key1 + r * 0xBB67AE85 (mod 2^32).  Computed once on
// the host so the kernel reads them as constants.
struct PhiloxKeys {
    uint32_t k0[10];
    uint32_t k1[10];
};

inline PhiloxKeys philox_round_keys(uint32_t key0, uint32_t key1) {
    PhiloxKeys r;
    for (int i = 0; i < 10; ++i) {
        r.k0[i] = key0 + static_cast<uint32_t>(i) * 0x9E3779B9u;
        r.k1[i] = key1 + static_cast<uint32_t>(i) * 0xBB67AE85u;
    }
    return r;
}

// Everything one decode launch needs, passed by value as a __grid_constant__.
struct DecodeParams {
    int B, H, dk, dv, ncb, units;  // units = B * H * ncb column blocks
    int grid;                      // persistent grid size G
    int gcb, gh, gb;               // G decomposed as (batch, head, column block) steps
    int ngroups, heads_per_group;
    int in_bf16;                   // vector inputs are bf16 (else float)
    int rnd;                       // base rounding: 0 nearest, kRndSr (16-bit uniforms),
                                   // kRndSr | kRndU8 (8-bit uniforms)
    long long row_bytes;           // code bytes per batch row
    const uint8_t* codes_in;
    uint8_t* codes_out;
    const float* scales_in;
    float* scales_out;
    const void* vA;                // GDN q      | Mamba-2 C
    const void* vB;                // GDN k      | Mamba-2 B
    const void* vC;                // GDN v      | Mamba-2 x
    const float* vD;               // GLA / KDA decay per key channel [B][H][dk]
    const float* g0;               // GDN alpha  | Mamba-2 dt                          | GLA, KDA: unused
    const float* g1;               // GDN beta   | Mamba-2 decay override (may be null) | KDA beta
    const float* A;                // Mamba-2 A [H]
    const float* D;                // Mamba-2 D [H]
    float* out;                    // [B][H][dv]
    const float* copy_absmax;      // copy scale: column maxima [B][H][dv] of an unquantized copy, or null
    // pure-write window (GDN): W slots; a [B][H][W][dk] FP8 + as [B][H][W],
    // b [B][H][dv/16][W][16] FP8 + bs [B][H][W]; in and out buffers differ
    int W;
    const uint8_t* win_a_in;
    const float* win_as_in;
    const uint8_t* win_b_in;
    const float* win_bs_in;
    uint8_t* win_a_out;
    float* win_as_out;
    uint8_t* win_b_out;
    float* win_bs_out;
    unsigned* flag;
    uint32_t step, key0, key1;
    PhiloxKeys rk;                 // Philox round keys of (key0, key1)
    // bounded waits: polls before a barrier wait gives up (sets kFlagTimeout);
    // withhold = 1 (failure-detection tests only): the second warp of a
    // two-warp block never arrives on the block's exchange barrier, and the
    // key-axis kernel never fills its first stage
    uint32_t wait_iters;
    int withhold;
    uint32_t head_off[RSQ_MAX_HEADS];  // byte offset of each head in a batch row
    uint8_t head_bits[RSQ_MAX_HEADS];
};

struct QuantParams {
    int B, H, dk, dv, ncb, units;
    int rnd;                       // base rounding bits, as DecodeParams::rnd
    long long row_bytes;
    const float* S;                // natural [B][H][dk][dv]
    uint8_t* codes;
    float* scales;
    unsigned* flag;
    uint32_t step, key0, key1;
    PhiloxKeys rk;
    uint32_t head_off[RSQ_MAX_HEADS];
    uint8_t head_bits[RSQ_MAX_HEADS];
};

struct DequantParams {
    int B, H, dk, dv, ncb;
    long long row_bytes;
    const uint8_t* codes;
    const float* scales;
    float* S;                      // natural [B][H][dk][dv] (dequantize), or null
    float* absmax;                 // [B][H][dv] column maxima of |S| (column_absmax), or null
    int key_axis;                  // scales are per key row ([B][H][dk]) instead of per column
    uint32_t head_off[RSQ_MAX_HEADS];
    uint8_t head_bits[RSQ_MAX_HEADS];
};

struct DriftParams {
    int B, H, dk, dv, ncb;
    long long q_row_bytes, f_row_bytes;
    const uint8_t* q_codes;
    const float* q_scales;
    const uint8_t* f_codes;
    double* sums;                  // [B][H][2]
    uint32_t q_head_off[RSQ_MAX_HEADS];
    uint8_t q_head_bits[RSQ_MAX_HEADS];
};

// Launchers (defined in the .cu files).  Return a cudaError_t value.
// ub = 16-column blocks per decode work unit (1, 2 or 4); bpw = blocks each
// warp takes per unit (1, or 2 for d_k = 128 units of four blocks)
int launch_decode(int family, int dk, int ub, int bpw, bool f32state, int rnd, const DecodeParams& p,
                  void* stream);
int decode_kernel_info(int family, int dk, int ub, int bpw, bool f32state, int rnd, int* threads, size_t* smem,
                       const void** func);
int launch_quantize(int dk, const QuantParams& p, void* stream);
int launch_dequantize(int dk, const DequantParams& p, void* stream);
// key-axis scale groups (one head at a time per CTA; the decode kernel is
// persistent over p.grid CTAs)
int launch_decode_ka(int dk, const DecodeParams& p, void* stream);
int decode_ka_info(int dk, int dv, int rnd, int* threads, size_t* smem, const void** func);
int launch_quantize_ka(int dk, const QuantParams& p, void* stream);
int launch_drift(const DriftParams& p, void* stream);

}  // namespace rsq
