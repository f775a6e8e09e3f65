/*
 * rsq_oracle.c -- CPU oracle for the quantized recurrent-state decode step.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline / reference arm may load this library.  The product
 * path (the CUDA library) never calls it and shares no code with it.
 *
 * Plain, single-threaded, obviously-correct C.  Every function cites the passage
 * of the method description it follows, and every function is pinned by a
 * test against something other than itself.  Parity unpinned: the drift
 * *values* of the long-horizon study, which the pages describe only in words
 * (the steps that produce them are pinned).  Sources:
 *   [LoReS]  "Quantizing Recurrent Language Models Is Easier Than You Think"
 *            (blog post of the LoReS paper): sections "(1/4) Scale grouping",
 *            "(2/4) Mixed precision", "(3/4) Rounding", "(4/4) Rotations".
 *   [LRB]    "Preserving Updates in Low-Bit Recurrent State Quantization",
 *            abstract (state requantized after every update).
 *   [FEED]   "When Dynamic Scaling Fails: A Scale-State Feedback Governs
 *            Recurrent-State Quantization ...", key points (dynamic scale).
 *   [BDR]    "Preserving Updates in Low-Bit Recurrent State Quantization",
 *            abstract: Bounded Directional Rounding -- an element whose
 *            rounding moves it opposite to its update is rounded toward the
 *            update instead, with no extra storage.
 *   [PW]     "Low-Bit GDN Recurrent-State Quantization: Global Gradient-aware
 *            Allocation and Pure-Write Sliding Windows", abstract: recent pure
 *            writes kept as FP8 vector pairs, propagated through the full GDN
 *            transition, merged into the low-bit state when they leave the
 *            window.
 *   [OCP8]   OCP 8-bit floating point specification, E4M3 format (bias 7,
 *            no infinities, max normal 448, subnormals m * 2^-9).
 *   [PHILOX] Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as
 *            1, 2, 3", SC'11 -- Philox4x32-10 block function.
 *   Recurrences: gated delta rule and Mamba-2 scalar-decay SSM as named in
 *   [LRB] abstract and [LoReS] Table 1; GLA (gated linear attention, a decay
 *   per key channel) and KDA (the delta rule with a decay per key channel),
 *   the diagonal-decay mixers of [LoReS] Table 1 / "Decayed recurrences are
 *   robust" (RetNet and plain linear attention are the Mamba-2 step with a
 *   constant decay, dt = 1 and D = 0).
 *
 * Orientation.  The state of one head is stored with the key / SSM-state axis i
 * as rows (dk rows) and the value / head-dim axis j as columns (dv columns):
 *     GDN     S_t = alpha*(I - beta k k^T) S_{t-1} + beta k v^T,   o_j = sum_i S_ij q_i
 *     Mamba-2 S_t = exp(dt*A) S_{t-1} + dt B x^T,                  y_j = sum_i S_ij C_i + D x_j
 * A value channel is a column; its scale is s_j = max_i |S_ij| / r with
 * r = 2^(b-1) - 1 ([LoReS] (1/4), Proposition "per-channel readout error").
 *
 * Two evaluation modes, both in binary32 (the workloads fix FP32 math):
 *   ORC_PLAIN      the literal definition: dequantize (c*s), sequential sums
 *                  over i, update, read out from the full-precision S_t,
 *                  quantize x = S/s with round-to-nearest or floor(x + U), clamp.
 *   ORC_CANONICAL  the same mathematics in the fixed FP32 evaluation order of
 *                  the GPU library (partial sums over i = rho (mod R) merged by
 *                  an XOR butterfly; c-form update; reciprocal multiplier
 *                  rounded toward zero), so results can be compared bit for bit.
 * In exact arithmetic both modes compute the same thing.
 *
 * Build: gcc -O1 -fPIC -shared -ffp-contract=off -fno-fast-math (see build.py).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_PLAIN 0
#define ORC_CANONICAL 1
/* Rounding: bit 0 selects the base rounding (0 nearest, 1 stochastic); bit 1
 * adds the directional correction of [BDR] on top of it; bit 2 makes the
 * stochastic rounding's uniforms 8 bits wide instead of 16.                 */
#define ORC_RTN 0
#define ORC_SR 1
#define ORC_BDR 2
#define ORC_U8 4
#define ORC_SR_BASE(rnd) ((rnd) & 1)
#define ORC_HAS_BDR(rnd) (((rnd) & 2) != 0)
#define ORC_UBITS(rnd) (((rnd) & ORC_U8) ? 8 : 16)

/* ------------------------------------------------------------------------- */
/* Philox4x32-10 [PHILOX]: 10 rounds of two 32x32->64 multiplies; the key is
 * bumped by the Weyl constants between rounds.                              */
/* ------------------------------------------------------------------------- */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
    const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += W0;
            k1 += W1;
        }
        uint64_t p0 = (uint64_t)M0 * (uint64_t)x0;
        uint64_t p1 = (uint64_t)M1 * (uint64_t)x2;
        uint32_t y0 = (uint32_t)(p1 >> 32) ^ x1 ^ k0;
        uint32_t y1 = (uint32_t)p1;
        uint32_t y2 = (uint32_t)(p0 >> 32) ^ x3 ^ k1;
        uint32_t y3 = (uint32_t)p0;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* The 16-bit uniform that stochastic rounding of element (i, j) of head (b, h)
 * at decode step `step` consumes.  One Philox block serves 8 elements: rows
 * i' and i' + dk/2 (i' = i mod dk/2) of the four columns 4g..4g+3 (g = j/4).
 *   counter = { i' | g << 16, h, b, step },  key = { seed_lo, seed_hi }
 *   chunk   = 4*[i >= dk/2] + (j mod 4);  word chunk/2, low half first.    */
uint32_t orc_sr_uniform16(uint64_t seed, uint32_t b, uint32_t h, uint32_t step,
                          int dk, int i, int j)
{
    int half = dk / 2;
    uint32_t ip = (uint32_t)(i % half);
    uint32_t g = (uint32_t)(j / 4);
    uint32_t ctr[4] = {ip | (g << 16), h, b, step};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    orc_philox4x32_10(ctr, key, out);
    int chunk = 4 * (i >= half ? 1 : 0) + (j % 4);
    uint32_t word = out[chunk / 2];
    return (chunk % 2 == 0) ? (word & 0xFFFFu) : (word >> 16);
}

/* The 8-bit uniform of element (i, j) of head (b, h) at decode step `step`
 * (stochastic rounding with 8-bit uniforms).  One Philox block serves 16
 * elements: rows i', i' + dk/4, i' + dk/2, i' + 3dk/4 (i' = i mod dk/4) of the
 * four columns 4g..4g+3 (g = j/4).
 *   counter = { i' | g << 16, h, b, step },  key = { seed_lo, seed_hi }
 *   word i div (dk/4), byte j mod 4 (lowest byte first).                   */
uint32_t orc_sr_uniform8(uint64_t seed, uint32_t b, uint32_t h, uint32_t step,
                         int dk, int i, int j)
{
    int quarter = dk / 4;
    uint32_t ip = (uint32_t)(i % quarter);
    uint32_t g = (uint32_t)(j / 4);
    uint32_t ctr[4] = {ip | (g << 16), h, b, step};
    uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
    uint32_t out[4];
    orc_philox4x32_10(ctr, key, out);
    uint32_t word = out[i / quarter];
    return (word >> (8 * (j % 4))) & 0xFFu;
}

/* The uniform stochastic rounding of element (i, j) consumes under rule `rnd`. */
static uint32_t orc_sr_uniform(int rnd, uint64_t seed, uint32_t b, uint32_t h, uint32_t step,
                               int dk, int i, int j)
{
    return (rnd & ORC_U8) ? orc_sr_uniform8(seed, b, h, step, dk, i, j)
                          : orc_sr_uniform16(seed, b, h, step, dk, i, j);
}

/* bfloat16 -> binary32 widening (exact): the bf16 bits are the upper half. */
void orc_bf16_to_f32(const uint16_t* src, float* dst, int64_t n)
{
    for (int64_t t = 0; t < n; ++t) {
        uint32_t u = (uint32_t)src[t] << 16;
        memcpy(&dst[t], &u, 4);
    }
}

/* ------------------------------------------------------------------------- */
/* Sums over the key axis.                                                    */
/* ------------------------------------------------------------------------- */

/* sum_i a[i*stride] * b[i] accumulated with one fused multiply-add per term.
 * R == 1: sequential in increasing i.  R > 1 (canonical order): partial p sums
 * rows i = p, p+R, p+2R, ... sequentially; then for d = 1, 2, ..., R/2 every
 * partial p becomes P[p] + P[p ^ d]; the result is P[0].                     */
static float orc_dot_rows(const float* a, int stride, const float* b, int n, int R)
{
    float part[64];
    for (int p = 0; p < R; ++p) {
        float acc = 0.0f;
        for (int i = p; i < n; i += R)
            acc = fmaf(a[(int64_t)i * stride], b[i], acc);
        part[p] = acc;
    }
    for (int d = 1; d < R; d *= 2) {
        float next[64];
        for (int p = 0; p < R; ++p)
            next[p] = part[p] + part[p ^ d];
        memcpy(part, next, sizeof(float) * (size_t)R);
    }
    return part[0];
}

/* ------------------------------------------------------------------------- */
/* Per-column scale and quantizer ([LoReS] (1/4), (3/4); [FEED]).             */
/* ------------------------------------------------------------------------- */

/* Largest representable code r = 2^(b-1) - 1 ([LoReS] (1/4), below the
 * proposition).  Codes are symmetric in [-r, r].                            */
static int orc_rmax(int bits) { return (1 << (bits - 1)) - 1; }

/* Reciprocal multiplier r/m rounded toward zero (canonical mode).  With it
 * |S| * inv <= r for every |S| <= m, so no code exceeds r.                  */
static float orc_inv_rz(float r, float m)
{
    float q = r / m; /* round to nearest */
    if ((double)q * (double)m > (double)r)
        q = nextafterf(q, 0.0f);
    return q;
}

/* Quantize one element S of a column whose absolute maximum is m (> 0 and
 * finite) to a symmetric b-bit code.  `u` is the element's uniform (used by
 * stochastic rounding only): 16 bits wide, or 8 bits under ORC_U8.
 *   plain:      x = S / s with s = m / r;  RTN: nearest (ties to even);
 *               SR, 16-bit u: floor(x + u/2^16), up with probability frac(x)
 *               to within 2^-16 ([LoReS] (3/4): SR is conditionally unbiased);
 *               SR, 8-bit u: floor(x + (u + 1/2)/2^8), up with probability
 *               frac(x) rounded to a multiple of 2^-8 (within 2^-9), and a
 *               value within 2^-9 of an integer stays on it;  clamp to [-r, r].
 *   canonical:  inv = r/m rounded toward zero;  RTN: nearest integer (ties to
 *               even) of the exact product S*inv;  SR: t = S*inv + (o + u/U)
 *               rounded once to binary32, c = floor(t) - o, with U = 2^16 and
 *               the offset o = 128 (8-bit codes) or 136 (4-bit codes), so that
 *               t stays in [1, 256), or U = 2^8 and o = 2^15 + 128 or 2^15 + 8,
 *               so that t stays in [2^15, 2^16) where the rounding of t to a
 *               multiple of 2^-8 adds the half of (u + 1/2).                 */
/* S / s of the plain order, made safe to convert to an integer.  When the
 * scale s = m / r underflows to zero (m below r * 2^-150, deep in the
 * subnormal range) S / s is +-inf, which the clamp to [-r, r] turns into +-r,
 * or 0 / 0 for an element that is zero, whose code is 0.  Values beyond
 * +-(r + 1) clamp to +-r either way, so they are cut there first.         */
static float orc_plain_ratio(float S, float s, int r)
{
    const float x = S / s;
    const float lim = (float)(r + 1);
    if (isnan(x)) return 0.0f;
    if (x > lim) return lim;
    if (x < -lim) return -lim;
    return x;
}

int orc_quantize_scalar(float S, float m, int bits, int rounding, int mode, uint32_t u)
{
    const int r = orc_rmax(bits);
    const float rf = (float)r;
    const int u8 = (rounding & ORC_U8) != 0;
    int c;
    if (mode == ORC_PLAIN) {
        const float s = m / rf;
        const float x = orc_plain_ratio(S, s, r);
        if (!ORC_SR_BASE(rounding))
            c = (int)rintf(x);
        else if (u8)
            c = (int)floor((double)x + ((double)u + 0.5) / 256.0);
        else
            c = (int)floor((double)x + (double)u / 65536.0);
        if (c > r) c = r;
        if (c < -r) c = -r;
    } else {
        const float inv = orc_inv_rz(rf, m);
        if (!ORC_SR_BASE(rounding)) {
            c = (int)rint((double)S * (double)inv);
        } else {
            const float off = u8 ? ((bits == 8) ? 32896.0f : 32776.0f)
                                 : ((bits == 8) ? 128.0f : 136.0f);
            const float V = off + (float)u / (u8 ? 256.0f : 65536.0f); /* exact */
            const float t = fmaf(S, inv, V);
            c = (int)floorf(t) - (int)off;
        }
    }
    return c;
}

/* Bounded Directional Rounding [BDR].  c is the base code of S (column maximum
 * m, stored scale s_new = m / r); prev is the element's previous dequantized
 * value c_{t-1} * s_{t-1}.  The update moves the element from prev to S; when
 * the rounded value c * s_new lies strictly on the other side of prev (a
 * reversal), the code becomes the integer next to x on the update's side:
 * ceil(x) for an upward update, floor(x) for a downward one, so the rounding
 * error stays below one step ("bounded").  x is S / s (plain) or the exact
 * product S * inv (canonical), as in the base rounding.                     */
int orc_bdr_adjust(int c, float S, float prev, float m, int bits, int mode)
{
    const float rf = (float)orc_rmax(bits);
    const float s_new = m / rf;
    const float now = (float)c * s_new;
    const int up = (S > prev) && (now < prev);
    const int down = (S < prev) && (now > prev);
    if (!up && !down) return c;
    const double x = (mode == ORC_PLAIN) ? (double)orc_plain_ratio(S, s_new, orc_rmax(bits))
                                         : (double)S * (double)orc_inv_rz(rf, m);
    int d = up ? (int)ceil(x) : (int)floor(x);
    const int r = orc_rmax(bits);
    if (d > r) d = r;
    if (d < -r) d = -r;
    return d;
}

/* Quantize column j of the full-precision state S (dk x dv, row-major) with
 * the dynamic scale computed from S itself: the "noisy" scale of [LoReS]
 * (4/4), through which earlier errors feed back [FEED].
 * Copy scale ([LoReS] (4/4), animation details; the ablation of [FEED]): when
 * m_copy is given, the scale is *m_copy / r, the column maximum of an
 * unquantized copy of the state, instead; the state is first clipped to
 * [-m_copy, m_copy], so elements beyond it get the codes +-r.  The column's
 * own maximum still decides whether it is finite.                          */
static void orc_quantize_column(const float* S, const float* prev, const float* m_copy, int dk,
                                int dv, int j, int bits, int rounding, int mode, uint64_t seed,
                                uint32_t b, uint32_t h, uint32_t step, int8_t* codes,
                                float* scale_out)
{
    const float rf = (float)orc_rmax(bits);
    /* m_j = max_i |S_ij|; a NaN anywhere in the column makes m NaN. */
    float m = 0.0f;
    for (int i = 0; i < dk; ++i) {
        float a = fabsf(S[(int64_t)i * dv + j]);
        if (isnan(a) || isnan(m))
            m = NAN;
        else if (a > m)
            m = a;
    }
    const float ms = m_copy ? *m_copy : m; /* the maximum the scale is taken from */
    *scale_out = ms / rf;                  /* s_j = max_i |S_ij| / r */
    /* An all-zero column has scale 0 and codes 0; a non-finite column keeps
     * its non-finite scale and gets codes 0.                                */
    const int usable = (ms > 0.0f) && isfinite(ms) && isfinite(m);
    const int r = orc_rmax(bits);
    for (int i = 0; i < dk; ++i) {
        int c = 0;
        if (usable) {
            float x = S[(int64_t)i * dv + j];
            if (m_copy) x = fminf(fmaxf(x, -ms), ms); /* clip to the copy's range */
            uint32_t u = ORC_SR_BASE(rounding) ? orc_sr_uniform(rounding, seed, b, h, step, dk, i, j) : 0u;
            c = orc_quantize_scalar(x, ms, bits, rounding, mode, u);
            /* without a previous state (initial quantization) there is no
             * update direction and the base rounding stands */
            if (ORC_HAS_BDR(rounding) && prev)
                c = orc_bdr_adjust(c, x, prev[(int64_t)i * dv + j], ms, bits, mode);
            if (c > r) c = r; /* plain order: S/s may exceed r by a rounding */
            if (c < -r) c = -r;
        }
        codes[(int64_t)i * dv + j] = (int8_t)c;
    }
}

/* ------------------------------------------------------------------------- */
/* One decode step of one head.                                              */
/* ------------------------------------------------------------------------- */
typedef struct {
    int dk, dv;       /* rows (key / SSM-state axis) and columns (value / head-dim axis) */
    int bits;         /* 4, 8 (quantized) or 32 (full-precision state) */
    int rounding;     /* ORC_RTN or ORC_SR, optionally | ORC_BDR */
    int mode;         /* ORC_PLAIN or ORC_CANONICAL */
    int R;            /* canonical partial-sum count (power of two, <= 64); 1 = sequential */
    uint64_t seed;    /* stochastic-rounding key */
    uint32_t b, h, step;
    const float* m_copy; /* copy scale: dv column maxima of an unquantized copy, or NULL */
} orc_head;

/* Gated delta rule decode step ([LRB] abstract: Gated DeltaNet; the LoReS
 * scheme keeps the update in full precision and quantizes the stored state,
 * [LoReS] "LoReS: State Quantization").
 *   inputs  c_in (dk*dv codes) + s_in (dv scales) for bits 4/8, or f_in (dk*dv floats) for 32;
 *           q, k (dk), v (dv) widened to binary32; alpha, beta gates.
 *   outputs c_out + s_out (or f_out), o (dv): readout from the FP32 S_t.    */
int orc_gdn_head_step(const orc_head* hd, const int8_t* c_in, const float* s_in,
                      const float* f_in, const float* q, const float* k, const float* v,
                      float alpha, float beta, int8_t* c_out, float* s_out, float* f_out,
                      float* o)
{
    const int dk = hd->dk, dv = hd->dv;
    const int R = (hd->mode == ORC_PLAIN) ? 1 : hd->R;
    float* S = (float*)malloc(sizeof(float) * (size_t)dk * (size_t)dv);
    float* Sh = (float*)malloc(sizeof(float) * (size_t)dk * (size_t)dv);
    float* cf = (float*)malloc(sizeof(float) * (size_t)dk * (size_t)dv);
    if (!S || !Sh || !cf) { free(S); free(Sh); free(cf); return 1; }

    if (hd->bits == 32) {
        /* Full-precision state: S_t = alpha*S + k w^T with w = beta*(v - alpha*S^T k). */
        for (int64_t t = 0; t < (int64_t)dk * dv; ++t) Sh[t] = f_in[t];
        for (int j = 0; j < dv; ++j) {
            float u = orc_dot_rows(Sh + j, dv, k, dk, R);
            float w = beta * fmaf(-alpha, u, v[j]);
            for (int i = 0; i < dk; ++i)
                S[(int64_t)i * dv + j] = fmaf(alpha, Sh[(int64_t)i * dv + j], k[i] * w);
        }
    } else if (hd->mode == ORC_PLAIN) {
        /* Dequantize: S^_ij = c_ij * s_j. */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                Sh[(int64_t)i * dv + j] = (float)c_in[(int64_t)i * dv + j] * s_in[j];
        for (int j = 0; j < dv; ++j) {
            float u = orc_dot_rows(Sh + j, dv, k, dk, 1);        /* u = S^T k */
            float w = beta * fmaf(-alpha, u, v[j]);            /* w = beta (v - alpha u) */
            for (int i = 0; i < dk; ++i)                        /* S = alpha S^ + k w^T */
                S[(int64_t)i * dv + j] = fmaf(alpha, Sh[(int64_t)i * dv + j], k[i] * w);
        }
    } else {
        /* Canonical c-form: u_j = s_j * sum_i c_ij k_i, S_ij = c_ij*(alpha s_j) + k_i w_j. */
        for (int64_t t = 0; t < (int64_t)dk * dv; ++t) cf[t] = (float)c_in[t];
        for (int j = 0; j < dv; ++j) {
            float ck = orc_dot_rows(cf + j, dv, k, dk, R);
            float u = s_in[j] * ck;
            float w = beta * fmaf(-alpha, u, v[j]);
            float a = alpha * s_in[j];
            for (int i = 0; i < dk; ++i)
                S[(int64_t)i * dv + j] = fmaf(cf[(int64_t)i * dv + j], a, k[i] * w);
        }
    }
    /* Readout from the full-precision S_t: o_j = sum_i S_ij q_i. */
    for (int j = 0; j < dv; ++j)
        o[j] = orc_dot_rows(S + j, dv, q, dk, R);

    if (hd->bits == 32) {
        for (int64_t t = 0; t < (int64_t)dk * dv; ++t) f_out[t] = S[t];
    } else {
        /* previous dequantized values c_{t-1} s_{t-1} (the directional rounding's reference) */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                Sh[(int64_t)i * dv + j] = (float)c_in[(int64_t)i * dv + j] * s_in[j];
        for (int j = 0; j < dv; ++j)
            orc_quantize_column(S, Sh, hd->m_copy ? hd->m_copy + j : NULL, dk, dv, j, hd->bits,
                                hd->rounding, hd->mode, hd->seed,
                                hd->b, hd->h, hd->step, c_out, &s_out[j]);
    }
    free(S); free(Sh); free(cf);
    return 0;
}

/* Mamba-2 scalar-decay decode step ([LRB] abstract: Mamba2; [LoReS] Table 1).
 *   decay a = exp(dt*A) (computed here with libm expf unless `decay` >= 0 is
 *   given), x (dv = P), Bv, Cv (dk = N), D.                                 */
int orc_mamba2_head_step(const orc_head* hd, const int8_t* c_in, const float* s_in,
                         const float* f_in, const float* x, const float* Bv, const float* Cv,
                         float dt, float A, float D, float decay, int8_t* c_out,
                         float* s_out, float* f_out, float* y)
{
    const int dk = hd->dk, dv = hd->dv;
    const int R = (hd->mode == ORC_PLAIN) ? 1 : hd->R;
    float* S = (float*)malloc(sizeof(float) * (size_t)dk * (size_t)dv);
    float* cf = (float*)malloc(sizeof(float) * (size_t)dk * (size_t)dv);
    float* Sh = (float*)malloc(sizeof(float) * (size_t)dk * (size_t)dv);
    if (!S || !cf || !Sh) { free(S); free(cf); free(Sh); return 1; }
    const float a = (decay >= 0.0f) ? decay : expf(dt * A);

    if (hd->bits == 32) {
        for (int j = 0; j < dv; ++j) {
            float xd = dt * x[j];
            for (int i = 0; i < dk; ++i)
                S[(int64_t)i * dv + j] = fmaf(a, f_in[(int64_t)i * dv + j], Bv[i] * xd);
        }
    } else if (hd->mode == ORC_PLAIN) {
        for (int j = 0; j < dv; ++j) {
            float xd = dt * x[j];
            for (int i = 0; i < dk; ++i) {
                float sh = (float)c_in[(int64_t)i * dv + j] * s_in[j];      /* dequantize */
                S[(int64_t)i * dv + j] = fmaf(a, sh, Bv[i] * xd);           /* a S^ + dt x B^T */
            }
        }
    } else {
        for (int64_t t = 0; t < (int64_t)dk * dv; ++t) cf[t] = (float)c_in[t];
        for (int j = 0; j < dv; ++j) {
            float xd = dt * x[j];
            float g = a * s_in[j];
            for (int i = 0; i < dk; ++i)
                S[(int64_t)i * dv + j] = fmaf(cf[(int64_t)i * dv + j], g, Bv[i] * xd);
        }
    }
    /* y_j = sum_i S_ij C_i + D x_j, from the full-precision S_t. */
    for (int j = 0; j < dv; ++j)
        y[j] = fmaf(D, x[j], orc_dot_rows(S + j, dv, Cv, dk, R));

    if (hd->bits == 32) {
        for (int64_t t = 0; t < (int64_t)dk * dv; ++t) f_out[t] = S[t];
    } else {
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                Sh[(int64_t)i * dv + j] = (float)c_in[(int64_t)i * dv + j] * s_in[j];
        for (int j = 0; j < dv; ++j)
            orc_quantize_column(S, Sh, hd->m_copy ? hd->m_copy + j : NULL, dk, dv, j, hd->bits,
                                hd->rounding, hd->mode, hd->seed,
                                hd->b, hd->h, hd->step, c_out, &s_out[j]);
    }
    free(S); free(cf); free(Sh);
    return 0;
}

/* Diagonal-decay recurrences ([LoReS] Table 1: GLA, KDA).  alpha is the decay
 * vector over the key axis (dk entries in (0, 1)).
 *   GLA:  S_t = diag(alpha) S_{t-1} + k v^T,                         o = S_t^T q
 *   KDA:  S_t = (I - beta k k^T) diag(alpha) S_{t-1} + beta k v^T,    o = S_t^T q
 * KDA in steps: D = diag(alpha) S^, u = D^T k, w = beta (v - u), S = D + k w^T.
 * Canonical c-form (s_j = 1 for a full-precision state):
 *   GLA  S_ij = fma(c_ij, alpha_i s_j, k_i v_j)
 *   KDA  u_j = s_j * sum_i c_ij (alpha_i k_i),  w_j = beta (v_j - u_j),
 *        S_ij = fma(c_ij, alpha_i s_j, k_i w_j)
 * Plain: dequantize S^ = c s, then D_ij = alpha_i S^_ij, sequential sums,
 * S_ij = fma(k_i, w_j, D_ij).                                              */
int orc_diag_head_step(const orc_head* hd, int delta, const int8_t* c_in, const float* s_in,
                       const float* f_in, const float* q, const float* k, const float* v,
                       const float* alpha, float beta, int8_t* c_out, float* s_out,
                       float* f_out, float* o)
{
    const int dk = hd->dk, dv = hd->dv;
    const int R = (hd->mode == ORC_PLAIN) ? 1 : hd->R;
    const size_t n = (size_t)dk * (size_t)dv;
    float* S = (float*)malloc(sizeof(float) * n);
    float* Sh = (float*)malloc(sizeof(float) * n);
    float* cf = (float*)malloc(sizeof(float) * n);
    float* ak = (float*)malloc(sizeof(float) * (size_t)dk);
    if (!S || !Sh || !cf || !ak) { free(S); free(Sh); free(cf); free(ak); return 1; }
    for (int i = 0; i < dk; ++i) ak[i] = alpha[i] * k[i];

    if (hd->bits != 32 && hd->mode == ORC_PLAIN) {
        /* dequantize, decay, then the (delta) update in the literal order */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                Sh[(int64_t)i * dv + j] = alpha[i] * ((float)c_in[(int64_t)i * dv + j] * s_in[j]);
        for (int j = 0; j < dv; ++j) {
            float w = v[j];
            if (delta) {
                const float u = orc_dot_rows(Sh + j, dv, k, dk, 1); /* u = D^T k */
                w = beta * (v[j] - u);
            }
            for (int i = 0; i < dk; ++i)
                S[(int64_t)i * dv + j] = fmaf(k[i], w, Sh[(int64_t)i * dv + j]);
        }
    } else {
        /* canonical c-form; a full-precision state is its own "code" with s = 1 */
        for (size_t t = 0; t < n; ++t) cf[t] = (hd->bits == 32) ? f_in[t] : (float)c_in[t];
        for (int j = 0; j < dv; ++j) {
            const float sj = (hd->bits == 32) ? 1.0f : s_in[j];
            float w = v[j];
            if (delta) {
                const float ck = orc_dot_rows(cf + j, dv, ak, dk, R);
                const float u = (hd->bits == 32) ? ck : sj * ck;
                w = beta * (v[j] - u);
            }
            for (int i = 0; i < dk; ++i) {
                const float a = (hd->bits == 32) ? alpha[i] : alpha[i] * sj;
                S[(int64_t)i * dv + j] = fmaf(cf[(int64_t)i * dv + j], a, k[i] * w);
            }
        }
    }
    for (int j = 0; j < dv; ++j)
        o[j] = orc_dot_rows(S + j, dv, q, dk, R);

    if (hd->bits == 32) {
        for (size_t t = 0; t < n; ++t) f_out[t] = S[t];
    } else {
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                Sh[(int64_t)i * dv + j] = (float)c_in[(int64_t)i * dv + j] * s_in[j];
        for (int j = 0; j < dv; ++j)
            orc_quantize_column(S, Sh, hd->m_copy ? hd->m_copy + j : NULL, dk, dv, j, hd->bits,
                                hd->rounding, hd->mode, hd->seed,
                                hd->b, hd->h, hd->step, c_out, &s_out[j]);
    }
    free(S); free(Sh); free(cf); free(ak);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Key-axis scale groups ([LoReS] (1/4) Scale grouping: the alternative to the */
/* value-axis groups; one scale per key row i, s_i = max_j |S_ij| / r).       */
/* ------------------------------------------------------------------------- */
/* Quantize row i of S (dk x dv) with its own maximum; same rounding rules as
 * a column.  Non-finite rows keep their scale and get codes 0.             */
static void orc_quantize_row(const float* S, int dk, int dv, int i, int bits, int rounding,
                             int mode, uint64_t seed, uint32_t b, uint32_t h, uint32_t step,
                             int8_t* codes, float* scale_out)
{
    const float rf = (float)orc_rmax(bits);
    float m = 0.0f;
    for (int j = 0; j < dv; ++j) {
        const float a = fabsf(S[(int64_t)i * dv + j]);
        if (isnan(a) || isnan(m)) m = NAN;
        else if (a > m) m = a;
    }
    *scale_out = m / rf;
    const int usable = (m > 0.0f) && isfinite(m);
    for (int j = 0; j < dv; ++j) {
        int c = 0;
        if (usable) {
            const uint32_t u = ORC_SR_BASE(rounding) ? orc_sr_uniform(rounding, seed, b, h, step, dk, i, j) : 0u;
            c = orc_quantize_scalar(S[(int64_t)i * dv + j], m, bits, rounding, mode, u);
        }
        codes[(int64_t)i * dv + j] = (int8_t)c;
    }
}

/* Gated DeltaNet decode step with key-axis scales s_in[dk] (everything else as
 * orc_gdn_head_step).  Canonical c-form with a per-row scale:
 *   u_j = sum_i c_ij (s_i k_i),  w_j = beta * fma(-alpha, u_j, v_j),
 *   S_ij = fma(c_ij, alpha s_i, k_i w_j),  o_j = sum_i S_ij q_i,
 * then each row is requantized with its own maximum.                       */
int orc_gdn_ka_head_step(const orc_head* hd, const int8_t* c_in, const float* s_in,
                         const float* q, const float* k, const float* v, float alpha, float beta,
                         int8_t* c_out, float* s_out, float* o)
{
    const int dk = hd->dk, dv = hd->dv;
    const int R = (hd->mode == ORC_PLAIN) ? 1 : hd->R;
    const size_t n = (size_t)dk * (size_t)dv;
    float* S = (float*)malloc(sizeof(float) * n);
    float* cf = (float*)malloc(sizeof(float) * n);
    float* ks = (float*)malloc(sizeof(float) * (size_t)dk);
    if (!S || !cf || !ks) { free(S); free(cf); free(ks); return 1; }
    if (hd->mode == ORC_PLAIN) {
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j)
                cf[(int64_t)i * dv + j] = (float)c_in[(int64_t)i * dv + j] * s_in[i];  /* S^ */
        for (int j = 0; j < dv; ++j) {
            const float u = orc_dot_rows(cf + j, dv, k, dk, 1);
            const float w = beta * fmaf(-alpha, u, v[j]);
            for (int i = 0; i < dk; ++i)
                S[(int64_t)i * dv + j] = fmaf(alpha, cf[(int64_t)i * dv + j], k[i] * w);
        }
    } else {
        for (size_t t = 0; t < n; ++t) cf[t] = (float)c_in[t];
        for (int i = 0; i < dk; ++i) ks[i] = s_in[i] * k[i];
        for (int j = 0; j < dv; ++j) {
            const float u = orc_dot_rows(cf + j, dv, ks, dk, R);
            const float w = beta * fmaf(-alpha, u, v[j]);
            for (int i = 0; i < dk; ++i)
                S[(int64_t)i * dv + j] = fmaf(cf[(int64_t)i * dv + j], alpha * s_in[i], k[i] * w);
        }
    }
    for (int j = 0; j < dv; ++j) o[j] = orc_dot_rows(S + j, dv, q, dk, R);
    for (int i = 0; i < dk; ++i)
        orc_quantize_row(S, dk, dv, i, hd->bits, hd->rounding & ~ORC_BDR, hd->mode, hd->seed, hd->b,
                         hd->h, hd->step, c_out, &s_out[i]);
    free(S); free(cf); free(ks);
    return 0;
}

/* Quantize a full-precision head with key-axis scales. */
int orc_quantize_ka_head(const orc_head* hd, const float* S, int8_t* c_out, float* s_out)
{
    if (hd->bits != 4 && hd->bits != 8) return 1;
    for (int i = 0; i < hd->dk; ++i)
        orc_quantize_row(S, hd->dk, hd->dv, i, hd->bits, hd->rounding & ~ORC_BDR, hd->mode, hd->seed,
                         hd->b, hd->h, hd->step, c_out, &s_out[i]);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* FP8 E4M3 [OCP8]: round to nearest even, saturating to +-448.              */
/* ------------------------------------------------------------------------- */
uint8_t orc_e4m3_encode(float x)
{
    if (isnan(x)) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0) return sign | 0x7E;                  /* saturate */
    if (a < 0.015625) {                                   /* below the smallest normal 2^-6 */
        const double m = nearbyint(a * 512.0);            /* subnormal steps of 2^-9 */
        return sign | (uint8_t)m;                         /* m = 8 is the smallest normal, 0x08 */
    }
    int e;
    const double fr = frexp(a, &e);                       /* a = fr * 2^e, fr in [0.5, 1) */
    int E = e - 1;                                        /* a = (2 fr) * 2^E, 2 fr in [1, 2) */
    double m = nearbyint((2.0 * fr - 1.0) * 8.0);         /* 3 mantissa bits */
    if (m == 8.0) { m = 0.0; E += 1; }
    if (E > 8 || (E == 8 && m > 6.0)) return sign | 0x7E;
    return sign | (uint8_t)(((E + 7) << 3) | (int)m);
}

float orc_e4m3_decode(uint8_t v)
{
    const int e = (v >> 3) & 15, m = v & 7;
    if (e == 15 && m == 7) return NAN;
    const double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (float)((v & 0x80) ? -mag : mag);
}

/* FP8 vector with one scale [PW]: s = max|x| / 448, codes e4m3(x_i * (448 / max|x|)). */
static void orc_fp8_vector_encode(const float* x, int n, uint8_t* q, float* scale)
{
    float m = 0.0f;
    for (int i = 0; i < n; ++i) {
        const float a = fabsf(x[i]);
        if (isnan(a) || isnan(m)) m = NAN;
        else if (a > m) m = a;
    }
    *scale = m / 448.0f;
    const float inv = (m > 0.0f && isfinite(m)) ? 448.0f / m : 0.0f;
    for (int i = 0; i < n; ++i) q[i] = orc_e4m3_encode(x[i] * inv);
}

/* Window dot product: 8 partials over contiguous chunks of n/8 entries, each
 * summed in increasing index, then combined by the XOR butterfly d = 1, 2, 4. */
static float orc_dot_chunks(const float* a, const float* b, int n)
{
    float part[8];
    const int len = n / 8;
    for (int p = 0; p < 8; ++p) {
        float acc = 0.0f;
        for (int t = 0; t < len; ++t) acc = fmaf(a[p * len + t], b[p * len + t], acc);
        part[p] = acc;
    }
    for (int d = 1; d < 8; d <<= 1)
        for (int p = 0; p < 8; ++p)
            if ((p & d) == 0) part[p] = part[p] + part[p | d];
    return part[0];
}

/* Gated DeltaNet decode step with a pure-write window [PW] of W slots.
 *
 * The full state is S_t = H_t + sum_w a_w b_w^T: H is the low-bit historical
 * state, slot w holds a recent pure write beta v k^T as the pair (a = k
 * propagated to the current step, b = beta v), each vector in FP8 with one
 * scale (fp8 = 0) or in binary32 (fp8 = 1 keeps them exact for the pins).
 * Step t uses slot p = t mod W: its write (from step t - W) leaves the window.
 *   1. H: the GDN transition of the dequantized history (no new write):
 *        u_j = s_j sum_i c_ij k_i,  w_j = beta * (-alpha u_j),
 *        S_ij = fma(c_ij, alpha s_j, k_i w_j)          (c-form, as GDN)
 *   2. every slot: a <- alpha (a - beta k (k^T a)):
 *        g = beta * dot(k, a),  a'_i = alpha * fma(-g, k_i, a_i)
 *   3. slot p leaves: S_ij = fma(a'_p,i, b_p,j, S_ij)
 *   4. slot p takes the new write: a = k, b = beta v
 *   5. readout from the full-precision state:
 *        o_j = sum_i S_ij q_i, then for w = 0..W-1: o_j = fma(b_w,j, z_w, o_j)
 *        with z_w = dot(a'_w, q) (slot p: dot(k, q))
 *   6. requantize H (rounding as configured, no BDR), encode the window.
 * Window layout: a [W][dk] codes + [W] scales, b [W][dv] codes + [W] scales
 * (binary32 arrays when fp32window).  Dots over the window use
 * orc_dot_chunks; sums over the state the canonical R-partial order.       */
int orc_gdn_pw_head_step(const orc_head* hd, int W, int fp32window, const int8_t* c_in,
                         const float* s_in, const float* f_in, const void* a_in,
                         const float* as_in, const void* b_in, const float* bs_in,
                         const float* q, const float* k, const float* v, float alpha, float beta,
                         int8_t* c_out, float* s_out, float* f_out, void* a_out, float* as_out,
                         void* b_out, float* bs_out, float* o)
{
    const int dk = hd->dk, dv = hd->dv;
    const int R = (hd->mode == ORC_PLAIN) ? 1 : hd->R;
    const int p = (int)(hd->step % (uint32_t)W);
    const size_t n = (size_t)dk * (size_t)dv;
    float* S = (float*)malloc(sizeof(float) * n);
    float* cf = (float*)malloc(sizeof(float) * n);
    float* A = (float*)malloc(sizeof(float) * (size_t)W * dk);   /* propagated a'_w */
    float* Bv = (float*)malloc(sizeof(float) * (size_t)W * dv);  /* decoded b_w */
    float* z = (float*)malloc(sizeof(float) * (size_t)W);
    if (!S || !cf || !A || !Bv || !z) { free(S); free(cf); free(A); free(Bv); free(z); return 1; }

    /* decode the window */
    for (int w = 0; w < W; ++w) {
        for (int i = 0; i < dk; ++i)
            A[w * dk + i] = fp32window ? ((const float*)a_in)[w * dk + i]
                                       : orc_e4m3_decode(((const uint8_t*)a_in)[w * dk + i]) * as_in[w];
        for (int j = 0; j < dv; ++j)
            Bv[w * dv + j] = fp32window ? ((const float*)b_in)[w * dv + j]
                                        : orc_e4m3_decode(((const uint8_t*)b_in)[w * dv + j]) * bs_in[w];
    }
    /* 1. history: the GDN transition without a write */
    for (size_t t = 0; t < n; ++t) cf[t] = (hd->bits == 32) ? f_in[t] : (float)c_in[t];
    for (int j = 0; j < dv; ++j) {
        const float sj = (hd->bits == 32) ? 1.0f : s_in[j];
        const float ck = orc_dot_rows(cf + j, dv, k, dk, R);
        const float u = (hd->bits == 32) ? ck : sj * ck;
        const float wj = beta * fmaf(-alpha, u, 0.0f);
        const float a = (hd->bits == 32) ? alpha : alpha * sj;
        for (int i = 0; i < dk; ++i)
            S[(int64_t)i * dv + j] = fmaf(cf[(int64_t)i * dv + j], a, k[i] * wj);
    }
    /* 2. propagate every slot through the transition */
    for (int w = 0; w < W; ++w) {
        const float g = beta * orc_dot_chunks(k, A + w * dk, dk);
        for (int i = 0; i < dk; ++i) A[w * dk + i] = alpha * fmaf(-g, k[i], A[w * dk + i]);
    }
    /* 3. slot p leaves the window into the history */
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            S[(int64_t)i * dv + j] = fmaf(A[p * dk + i], Bv[p * dv + j], S[(int64_t)i * dv + j]);
    /* 4. the new write takes slot p */
    for (int i = 0; i < dk; ++i) A[p * dk + i] = k[i];
    for (int j = 0; j < dv; ++j) Bv[p * dv + j] = beta * v[j];
    /* 5. readout */
    for (int w = 0; w < W; ++w) z[w] = orc_dot_chunks(A + w * dk, q, dk);
    for (int j = 0; j < dv; ++j) {
        float acc = orc_dot_rows(S + j, dv, q, dk, R);
        for (int w = 0; w < W; ++w) acc = fmaf(Bv[w * dv + j], z[w], acc);
        o[j] = acc;
    }
    /* 6. requantize the history, encode the window */
    if (hd->bits == 32) {
        for (size_t t = 0; t < n; ++t) f_out[t] = S[t];
    } else {
        for (int j = 0; j < dv; ++j)
            orc_quantize_column(S, NULL, hd->m_copy ? hd->m_copy + j : NULL, dk, dv, j, hd->bits,
                                hd->rounding & ~ORC_BDR, hd->mode, hd->seed, hd->b, hd->h, hd->step,
                                c_out, &s_out[j]);
    }
    for (int w = 0; w < W; ++w) {
        if (fp32window) {
            memcpy((float*)a_out + w * dk, A + w * dk, sizeof(float) * dk);
            memcpy((float*)b_out + w * dv, Bv + w * dv, sizeof(float) * dv);
            continue;
        }
        orc_fp8_vector_encode(A + w * dk, dk, (uint8_t*)a_out + w * dk, &as_out[w]);
        if (w == p) {
            orc_fp8_vector_encode(Bv + w * dv, dv, (uint8_t*)b_out + w * dv, &bs_out[w]);
        } else {
            memcpy((uint8_t*)b_out + w * dv, (const uint8_t*)b_in + w * dv, (size_t)dv);
            bs_out[w] = bs_in[w];
        }
    }
    free(S); free(cf); free(A); free(Bv); free(z);
    return 0;
}

/* Quantize a full-precision head state (initialisation / checkpoint), with the
 * same per-column scale and rounding as the decode step.                    */
int orc_quantize_head(const orc_head* hd, const float* S, int8_t* c_out, float* s_out)
{
    if (hd->bits != 4 && hd->bits != 8) return 1;
    for (int j = 0; j < hd->dv; ++j)
        orc_quantize_column(S, NULL, hd->m_copy ? hd->m_copy + j : NULL, hd->dk, hd->dv, j,
                            hd->bits, hd->rounding, hd->mode, hd->seed, hd->b, hd->h, hd->step,
                            c_out, &s_out[j]);
    return 0;
}

/* Dequantize: S^_ij = c_ij * s_j. */
void orc_dequantize_head(int dk, int dv, const int8_t* c, const float* s, float* S)
{
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j)
            S[(int64_t)i * dv + j] = (float)c[(int64_t)i * dv + j] * s[j];
}

/* ------------------------------------------------------------------------- */
/* Storage format of the library, written out independently.                 */
/*   A head's dv columns are cut into blocks of CB = 16 columns.  Block cb     */
/*   holds rows i = 0..dk-1 of columns cb*CB .. cb*CB+CB-1, row by row.  8-bit code c is stored as the byte c + 128; 4-bit codes as the     */
/*   nibble c + 8, column 2t in the low nibble of byte t of the row segment   */
/*   and column 2t+1 in the high nibble.  32-bit heads store binary32 values  */
/*   in the same block order.                                                 */
/* ------------------------------------------------------------------------- */
static int orc_cb(int dv) { (void)dv; return 16; }

int64_t orc_head_bytes(int dk, int dv, int bits) { return (int64_t)dk * dv * bits / 8; }

void orc_pack_head(int dk, int dv, int bits, const int8_t* c, const float* f, uint8_t* out)
{
    const int CB = orc_cb(dv);
    int64_t pos = 0;
    for (int cb = 0; cb < dv / CB; ++cb) {
        for (int i = 0; i < dk; ++i) {
            for (int jj = 0; jj < CB; ++jj) {
                int j = cb * CB + jj;
                int64_t e = (int64_t)i * dv + j;
                if (bits == 8) {
                    out[pos++] = (uint8_t)(c[e] + 128);
                } else if (bits == 4) {
                    uint8_t nib = (uint8_t)(c[e] + 8);
                    if (jj % 2 == 0) out[pos] = nib;
                    else out[pos++] |= (uint8_t)(nib << 4);
                } else {
                    memcpy(out + pos, &f[e], 4);
                    pos += 4;
                }
            }
        }
    }
}

void orc_unpack_head(int dk, int dv, int bits, const uint8_t* in, int8_t* c, float* f)
{
    const int CB = orc_cb(dv);
    int64_t pos = 0;
    for (int cb = 0; cb < dv / CB; ++cb) {
        for (int i = 0; i < dk; ++i) {
            for (int jj = 0; jj < CB; ++jj) {
                int j = cb * CB + jj;
                int64_t e = (int64_t)i * dv + j;
                if (bits == 8) {
                    c[e] = (int8_t)((int)in[pos++] - 128);
                } else if (bits == 4) {
                    int nib = (jj % 2 == 0) ? (in[pos] & 0xF) : (in[pos++] >> 4);
                    c[e] = (int8_t)(nib - 8);
                } else {
                    memcpy(&f[e], in + pos, 4);
                    pos += 4;
                }
            }
        }
    }
}

/* Decay-based mixed precision ([LoReS] (2/4): more bits for the slowest-
 * decaying heads).  Brute force: head h gets `hi` bits when fewer than
 * n_hi heads have a larger decay score (ties: the lower head index ranks
 * first), otherwise `lo` bits.                                               */
void orc_allocate_bits(const double* score, int H, int n_hi, int hi, int lo, int8_t* bits)
{
    for (int h = 0; h < H; ++h) {
        int ahead = 0;
        for (int g = 0; g < H; ++g)
            if (score[g] > score[h] || (score[g] == score[h] && g < h)) ++ahead;
        bits[h] = (int8_t)(ahead < n_hi ? hi : lo);
    }
}
