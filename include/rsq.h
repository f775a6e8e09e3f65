/*
 * rsq.h -- quantized recurrent-state decode step for NVIDIA B200 (sm_100a).
 *
 * One decode step of a linear-attention / SSM layer whose recurrent state is
 * stored in low precision between steps: the stored state is dequantized,
 * advanced by one token with the layer's recurrence, read out, given fresh
 * per-value-channel absmax scales and requantized, in one fused pass.
 *
 * Method sources (cited below by tag):
 *   [LoReS] "Quantizing Recurrent Language Models Is Easier Than You Think"
 *           (LoReS blog post): "LoReS: State Quantization" (full-precision
 *           updates, quantized stored state), "(1/4) Scale grouping"
 *           (value-axis scales, r = 2^(b-1) - 1), "(2/4) Mixed precision"
 *           (more bits for the slowest-decaying heads), "(3/4) Rounding"
 *           (stochastic rounding), "(4/4) Rotations" (noisy vs copy scale).
 *   [LRB]   "Preserving Updates in Low-Bit Recurrent State Quantization",
 *           abstract: the state is requantized after every update; Gated
 *           DeltaNet, GLA, Mamba2 and RetNet recurrences.
 *   [FEED]  "When Dynamic Scaling Fails: A Scale-State Feedback Governs
 *           Recurrent-State Quantization ...", key points: the dynamic scale
 *           is derived from the state it quantizes.
 *   [PW]    "Low-Bit GDN Recurrent-State Quantization: Global Gradient-aware
 *           Allocation and Pure-Write Sliding Windows", abstract: recent pure
 *           writes kept as FP8 vector pairs beside the low-bit state.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All buffers are caller-owned.  Pointers marked "device" must point to
 *    CUDA device memory of the current device, 16-byte aligned.  Pointers
 *    marked "host" are ordinary host memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call that takes a stream is asynchronous on that stream
 *    and never synchronizes, except rsq_check_flags.  rsq_decode_step,
 *    rsq_decode_step_window, rsq_quantize and rsq_dequantize may be captured
 *    into CUDA graphs (the benchmark replays them from graphs).
 *  - Host-side validation happens before any CUDA call; a failing check
 *    returns RSQ_E_INVAL or RSQ_E_UNSUPPORTED and touches no memory.  A
 *    failed launch returns RSQ_E_CUDA.  rsq_last_error() then holds a
 *    human-readable reason (thread-local).
 *  - A context is immutable after rsq_create and may be used from several
 *    host threads and streams at once.
 *
 * State orientation (both families)
 * ---------------------------------
 *  One head's state is a dk x dv matrix S with rows i (GDN key axis / Mamba-2
 *  SSM state axis N) and columns j (GDN value axis / Mamba-2 head-dim axis P).
 *  A value channel is a column: it has one scale s_j = max_i |S_ij| / r with
 *  r = 2^(b-1) - 1 (127 for 8-bit, 7 for 4-bit) ([LoReS] (1/4)).  Codes are
 *  symmetric integers in [-r, r].
 *
 * State storage format (rsq_state)
 * --------------------------------
 *  codes: device bytes [batch][row_bytes].  Within a batch row the heads are
 *    concatenated in order; head h occupies dk*dv*bits_h/8 bytes.  A head's
 *    columns are cut into blocks of 16 columns; block cb (cb = 0 .. dv/16-1)
 *    stores rows i = 0..dk-1 of columns 16cb..16cb+15 row after row, so every
 *    block is one contiguous run of dk*16*bits/8 bytes.  Inside a row segment:
 *      8-bit : byte = c + 128                       (one per column)
 *      4-bit : byte t = (c_{2t} + 8) | (c_{2t+1} + 8) << 4
 *      32-bit: IEEE binary32 value of S_ij          (full-precision state)
 *  scales: device float [batch][heads][dv], s_j per column (unused for 32-bit).
 *  The all-zero state S_0 = 0 is codes "zero code" (128 / 0x88) with scales 0;
 *  rsq_quantize of a zero tensor produces it.
 *
 * Arithmetic (binary32 throughout; fixed evaluation order, see rsq_decode_step)
 * ------------------------------------------------------------------------
 *  Sums over the key axis i use R = rsq_reduction_partials(dk) partial sums
 *  (8 up to dk = 128, 16 for dk = 256): partial p accumulates rows i = p, p+R, p+2R, ... in increasing i with
 *  one fused multiply-add per term; then for d = 1, 2, ..., R/2 every partial p
 *  becomes P[p] + P[p^d]; the sum is P[0].
 */
#ifndef RSQ_H
#define RSQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RSQ_MAX_HEADS 512

typedef enum {
    RSQ_OK = 0,
    RSQ_E_INVAL = 1,       /* bad argument: null / misaligned pointer, bad size or enum */
    RSQ_E_UNSUPPORTED = 2, /* valid but not built: a dk/dv/bit-width combination */
    RSQ_E_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
    RSQ_E_NOMEM = 4,       /* the context's own small allocation failed */
    RSQ_E_NONFINITE = 5    /* rsq_check_flags: a non-finite state column was seen */
} rsq_status;

/* Recurrence of the layer.  RSQ_GDN: gated delta rule; RSQ_MAMBA2: scalar
 * decay (RetNet and plain linear attention are this step with B = k, C = q,
 * x = v, dt = 1, decay = gamma (resp. 1), D = 0 and ngroups = heads);
 * RSQ_GLA: S_t = diag(alpha) S_{t-1} + k v^T with a decay per key channel;
 * RSQ_KDA: S_t = (I - beta k k^T) diag(alpha) S_{t-1} + beta k v^T.  GLA and
 * KDA are the diagonal-decay mixers of [LoReS] Table 1. */
typedef enum { RSQ_GDN = 0, RSQ_MAMBA2 = 1, RSQ_GLA = 2, RSQ_KDA = 3 } rsq_family;
/* Requantization rule.  RSQ_RTN: nearest code (ties to even).  RSQ_SR8:
 * stochastic rounding with an 8-bit Philox uniform per element, up with
 * probability frac(x) rounded to a multiple of 2^-8 ([LoReS] (3/4)); RSQ_SR:
 * the same with a 16-bit uniform per element, up with probability frac(x) to
 * within 2^-16 (twice the random bits, twice the Philox work per element).
 * Bit 0 = stochastic, bit 1 = directional correction, bit 2 = 8-bit uniforms.
 * RSQ_BDR / RSQ_SR_BDR / RSQ_SR8_BDR: the same base rounding followed by
 * Bounded Directional Rounding ("Preserving Updates in Low-Bit Recurrent State
 * Quantization", abstract): when the rounded value c_t s_t lies strictly on
 * the other side of the previous value c_{t-1} s_{t-1} than the updated state
 * S_t does (the element moved against its update), the code becomes the
 * integer next to S_t / s_t on the update's side (ceil for an upward update,
 * floor for a downward one), so the error stays below one step.  No extra
 * storage.  rsq_quantize has no previous state and applies the base rounding. */
typedef enum {
    RSQ_RTN = 0,
    RSQ_SR = 1,
    RSQ_BDR = 2,
    RSQ_SR_BDR = 3,
    RSQ_SR8 = 5,
    RSQ_SR8_BDR = 7
} rsq_rounding;
typedef enum { RSQ_F32 = 0, RSQ_BF16 = 1 } rsq_dtype;

/* Device allocator hook for the context's own allocation (its 4-byte flag
 * word).  alloc returns device memory of at least `bytes` bytes, 16-byte
 * aligned, on the current device, or NULL when it cannot (rsq_create then
 * returns RSQ_E_NOMEM and allocates nothing else); release gives it back and
 * is called once, by rsq_destroy or by a failing rsq_create.  `user` is
 * rsq_config.alloc_user, passed through.  Both NULL: cudaMalloc / cudaFree.
 * The hook lets a caller place the word in its own pool, and lets a test
 * make the allocation fail. */
typedef void* (*rsq_alloc_fn)(size_t bytes, void* user);
typedef void (*rsq_release_fn)(void* ptr, void* user);

/* Layer configuration, read once by rsq_create. */
typedef struct {
    int family;      /* rsq_family */
    int batch;       /* B >= 1 independent requests */
    int heads;       /* H, 1..RSQ_MAX_HEADS */
    int dk;          /* rows: GDN key dim d_k / Mamba-2 state dim N; one of 16, 32, 64, 128,
                        256 (256: no pure-write window, no key-axis scales) */
    int dv;          /* columns: GDN value dim d_v / Mamba-2 head dim P; one of 16,32,64,128,256 */
    int ngroups;     /* Mamba-2 B/C groups (divides heads); ignored for GDN */
    const int8_t* head_bits; /* host [heads]: each 4 or 8, or every entry 32 (full-precision
                                state).  NULL = all 8.  Copied by rsq_create. */
    int rounding;    /* rsq_rounding: requantization rule */
    int in_dtype;    /* rsq_dtype of the vector inputs (q, k, v / x, B, C) */
    uint64_t seed;   /* stochastic-rounding key */
    int window;      /* pure-write window slots W for Gated DeltaNet ([PW]): 0 (none), 4, 8
                        or 16; needs RSQ_RTN, RSQ_SR or RSQ_SR8 and rsq_decode_step_window */
    int key_axis;    /* 0: one scale per value column (the method's grouping); 1: one scale
                        per key row, s_i = max_j |S_ij| / r ([LoReS] (1/4), the grouping
                        ablation).  Key-axis: Gated DeltaNet, 4/8-bit heads, RSQ_RTN,
                        RSQ_SR or RSQ_SR8; scales are [B][H][dk]; a CTA works on one head
                        at a time (a row maximum spans every column). */
    rsq_alloc_fn alloc;      /* allocator hook (above); NULL with release NULL: cudaMalloc */
    rsq_release_fn release;  /* its release; set both or neither (else RSQ_E_INVAL) */
    void* alloc_user;        /* passed to both */
} rsq_config;

typedef struct rsq_ctx rsq_ctx;

/* A stored state (device, caller-owned; format above). */
typedef struct {
    void* codes;     /* device [batch][row_bytes] */
    float* scales;   /* device [batch][heads][dv] (may be NULL when every head is 32-bit) */
} rsq_state;

/* Gated DeltaNet step inputs (device).  q, k: [B][H][dk]; v: [B][H][dv], in
 * in_dtype; alpha (decay gate in (0,1)), beta (write strength): float [B][H]. */
typedef struct {
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;
    const float* beta;
} rsq_gdn_inputs;

/* Mamba-2 step inputs (device).  x: [B][H][dv]; Bm, Cm: [B][ngroups][dk], in
 * in_dtype; dt: float [B][H]; A, D: float [H]; decay: float [B][H] or NULL.
 * When decay is non-NULL it replaces exp(dt*A) (a caller that already holds
 * the decay, or a test that needs a decay value fixed bit for bit). */
typedef struct {
    const void* x;
    const void* Bm;
    const void* Cm;
    const float* dt;
    const float* A;
    const float* D;
    const float* decay;
} rsq_mamba2_inputs;

/* GLA / KDA step inputs (device).  q, k: [B][H][dk], v: [B][H][dv] in
 * in_dtype; alpha: float [B][H][dk], the decay of each key channel; beta:
 * float [B][H] (KDA; ignored and may be NULL for GLA).
 *   GLA:  S_ij = alpha_i S^_ij + k_i v_j
 *   KDA:  u_j = sum_i alpha_i S^_ij k_i,  w_j = beta (v_j - u_j),
 *         S_ij = alpha_i S^_ij + k_i w_j
 * with S^ the dequantized previous state; readout o_j = sum_i S_ij q_i. */
typedef struct {
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;
    const float* beta;
} rsq_diag_inputs;

/* Create a context for one layer configuration.  Validates the configuration
 * (RSQ_E_INVAL / RSQ_E_UNSUPPORTED, nothing allocated), then allocates a
 * 4-byte device flag word on the current device, through cfg->alloc when set
 * (RSQ_E_NOMEM / RSQ_E_CUDA on failure).  *out receives the context; release
 * it with rsq_destroy. */
rsq_status rsq_create(const rsq_config* cfg, rsq_ctx** out);

/* Release a context (NULL is a no-op).  Not stream-ordered: call it only after
 * every stream that used the context has finished with it. */
void rsq_destroy(rsq_ctx* ctx);

/* Bytes of the caller-owned state buffers: codes (batch * row_bytes) and
 * scales (batch * heads * dv * 4). */
rsq_status rsq_state_bytes(const rsq_ctx* ctx, size_t* code_bytes, size_t* scale_bytes);

/* Per-head byte offset of head h inside a batch row of the code buffer. */
rsq_status rsq_head_offset(const rsq_ctx* ctx, int h, size_t* offset);

/* One decode step for every (request, head) of the layer.
 *
 * Per head, with the stored codes c and scales s of state_in:
 *  GDN ([LRB] abstract, [LoReS] Table 1), state S_t = alpha (I - beta k k^T) S_{t-1} + beta k v^T:
 *     u_j = s_j * sum_i c_ij k_i                 (= (S^_{t-1}^T k)_j, S^ = c*s)
 *     w_j = beta * fma(-alpha, u_j, v_j)
 *     S_ij = fma(c_ij, alpha*s_j, k_i*w_j)
 *     out_j = sum_i S_ij q_i                     (readout from the full-precision S_t)
 *  Mamba-2, state S_t = exp(dt A) S_{t-1} + dt B x^T:
 *     a = decay ? decay : expf(dt*A);  S_ij = fma(c_ij, a*s_j, B_i*(dt*x_j))
 *     out_j = fma(D, x_j, sum_i S_ij C_i)
 *  then per column ([LoReS] (1/4), (3/4); noisy dynamic scale [FEED]):
 *     m_j = max_i |S_ij|;  s'_j = m_j / r;  inv_j = r / m_j rounded toward zero
 *     (inv_j = 0 when m_j = 0);
 *     RTN: c'_ij = nearest integer (ties to even) of the exact S_ij * inv_j
 *     SR8: t = fma(S_ij, inv_j, 2^15 + o + u_ij/256) in binary32 (t lies in
 *          [2^15, 2^16), where rounding to the ulp 2^-8 adds the half of
 *          u + 1/2), c'_ij = floor(t) - 2^15 - o, o = 128 (8-bit) / 8 (4-bit);
 *          u_ij is an 8-bit uniform from Philox4x32-10 (Salmon et al., SC'11)
 *          with key = seed and counter { (i mod dk/4) | (j/4) << 16, h, b,
 *          step }; element (i, j) takes byte j mod 4 (lowest first) of word
 *          i div (dk/4).
 *     SR : t = fma(S_ij, inv_j, o + u_ij/65536) in binary32, c'_ij = floor(t) - o,
 *          o = 128 (8-bit) / 136 (4-bit); u_ij is a 16-bit uniform from
 *          Philox4x32-10 with counter { (i mod dk/2) | (j/4) << 16, h, b, step };
 *          element (i, j) takes 16-bit chunk 4*[i >= dk/2] + (j mod 4) (word
 *          chunk/2, low half first).
 *  32-bit heads skip the quantizer and store S_t; their update is
 *     GDN: u_j = sum_i S_ij k_i, S_ij = fma(alpha, S_ij, k_i*w_j);
 *     Mamba-2: S_ij = fma(a, S_ij, B_i*(dt*x_j)).
 *  A column whose maximum is not finite keeps that scale (inf or NaN), gets
 *  codes 0 and raises the context's non-finite flag (rsq_check_flags).
 *
 * Arguments: state_in / state_out: device states of this context's format;
 *   state_out may equal state_in (in-place update; any other overlap is
 *   invalid).  inputs: host pointer to rsq_gdn_inputs, rsq_mamba2_inputs or
 *   rsq_diag_inputs (GLA, KDA) -- the context's family -- holding device
 *   pointers.  out: device float
 *   [B][H][dv].  step: decode-step index (stochastic-rounding counter; keep it
 *   across checkpoints for reproducible runs).
 * Errors: RSQ_E_INVAL for null/misaligned pointers; RSQ_E_CUDA if the launch
 *   fails.  No memory is written when an argument check fails. */
rsq_status rsq_decode_step(const rsq_ctx* ctx, const rsq_state* state_in,
                           const rsq_state* state_out, const void* inputs, float* out,
                           uint32_t step, void* stream);

/* Quantize a full-precision state (device float [B][H][dk][dv], row-major per
 * head) into state_out with the same per-column scale and rounding as
 * rsq_decode_step (RTN or SR with counter step).  32-bit heads are copied.
 * Used to initialise and to load checkpoints. */
rsq_status rsq_quantize(const rsq_ctx* ctx, const float* S, const rsq_state* state_out,
                        uint32_t step, void* stream);

/* Dequantize state_in into device float [B][H][dk][dv]: S^_ij = c_ij * s_j
 * (32-bit heads: the stored value). */
rsq_status rsq_dequantize(const rsq_ctx* ctx, const rsq_state* state_in, float* S_out,
                          void* stream);

/* Per-head sums for the relative state drift ||deq(Q) - F||_F / ||F||_F of a
 * quantized trajectory Q against a full-precision trajectory F of the same
 * shape (q_ctx: 4/8-bit heads; f_ctx: 32-bit heads).  sums: device double
 * [B][H][2] receives { sum (S^_ij - F_ij)^2, sum F_ij^2 } per head. */
rsq_status rsq_state_drift(const rsq_ctx* q_ctx, const rsq_state* q_state,
                           const rsq_ctx* f_ctx, const rsq_state* f_state, double* sums,
                           void* stream);

/* Decode step with the copy scale ([LoReS] (4/4), animation details; the
 * ablation of [FEED]): identical to rsq_decode_step except that each column's
 * new scale is copy_absmax[b][h][j] / r, the maximum of |S_t| of an
 * unquantized copy of the state (e.g. a full-precision trajectory run on the
 * same inputs, read with rsq_column_absmax), instead of the maximum of the
 * column itself; codes beyond it clip to +-r.  This removes the feedback of
 * earlier quantization errors into the scale.  copy_absmax: device float
 * [B][H][dv].  A column whose own values are non-finite is still flagged and
 * stored as zero codes.  RSQ_E_UNSUPPORTED for a full-precision context. */
rsq_status rsq_decode_step_copy_scale(const rsq_ctx* ctx, const rsq_state* state_in,
                                      const rsq_state* state_out, const void* inputs,
                                      const float* copy_absmax, float* out, uint32_t step,
                                      void* stream);

/* Column maxima max_i |S^_ij| of a stored state (dequantized values; the
 * stored values for 32-bit heads), NaN-propagating.  absmax: device float
 * [B][H][dv]. */
rsq_status rsq_column_absmax(const rsq_ctx* ctx, const rsq_state* state, float* absmax, void* stream);

/* Pure-write window of a Gated DeltaNet context with rsq_config.window = W > 0
 * ([PW]).  The full state is the stored low-bit history H plus the W most
 * recent pure writes a b^T: a = k propagated through every later transition
 * a <- alpha (a - beta k (k.a)), b = beta v.  Each vector is FP8 E4M3 (round to
 * nearest even, saturating) with one float scale max|x| / 448.  Device
 * buffers, caller-owned, 16-byte aligned; an all-zero window is empty:
 *   a        uint8 [B][H][W][dk]          codes of the a vectors
 *   a_scale  float [B][H][W]
 *   b        uint8 [B][H][dv/16][W][16]   codes of the b vectors, in 16-column
 *                                          blocks like the state
 *   b_scale  float [B][H][W] */
typedef struct {
    void* a;
    float* a_scale;
    void* b;
    float* b_scale;
} rsq_window;

/* Bytes of the window buffers: a codes, b codes, and each scale array. */
rsq_status rsq_window_bytes(const rsq_ctx* ctx, size_t* a_bytes, size_t* b_bytes,
                            size_t* scale_bytes);

/* Decode step of a context with a pure-write window.  Step t uses slot
 * p = t mod W: its write (from step t - W) is propagated, merged into H, and
 * the slot takes the new write (k, beta v).  H follows the GDN transition
 * without the new write, is read out together with the window
 * (o_j = sum_i H_ij q_i + sum_w b_w,j (a_w . q), window dots in 8 contiguous
 * chunks combined by the XOR butterfly) and requantized as usual.  win_in and
 * win_out must not share buffers (every column unit of a head reads the a
 * vectors); states may be updated in place.  RSQ_E_INVAL for a context
 * without a window. */
rsq_status rsq_decode_step_window(const rsq_ctx* ctx, const rsq_state* state_in,
                                  const rsq_state* state_out, const rsq_window* win_in,
                                  const rsq_window* win_out, const void* inputs, float* out,
                                  uint32_t step, void* stream);

/* Synchronize `stream`, then report (and clear) the context's non-finite
 * flag: *seen = 1 if any decode step since the last check met a non-finite
 * column.  Returns RSQ_E_NONFINITE when *seen = 1. */
rsq_status rsq_check_flags(const rsq_ctx* ctx, int* seen, void* stream);

/* Failure-detection hook for tests (no counterpart in the method's pages).
 * Sets the limit of this context's decode kernels' bounded barrier waits to
 * `wait_iters` polls (0: the default, 2^22).  With withhold = 1 the second
 * warp of every two-warp block (dk = 256) skips its arrivals on the block's
 * exchange barrier, so that both warps' waits on it run out; and the
 * key-axis kernel (key_axis = 1) never fills the first stage of its ring, so
 * that its first stage wait runs out while the second stage's copies are in
 * flight.  A kernel whose wait runs out sets the
 * context's timeout flag, waits (bounded) for the copies it still has in
 * flight towards its shared memory, and ends; that step's outputs are
 * incomplete and rsq_check_flags returns RSQ_E_CUDA.  withhold = 0 and
 * wait_iters = 0 restore normal operation.  For tests of the failure path:
 * call it while no step of the context is in flight, from one thread.
 * RSQ_E_INVAL for a null context or withhold not 0 or 1. */
rsq_status rsq_debug_waits(rsq_ctx* ctx, uint32_t wait_iters, int withhold);

/* Decay-based mixed precision ([LoReS] (2/4)): host-only.  score: host
 * double [heads] (a decay statistic, e.g. the mean gate alpha; larger = slower
 * decay).  The n_high heads with the largest score get high_bits, the others
 * low_bits; ties go to the lower head index.  bits_out: host int8 [heads]. */
rsq_status rsq_allocate_bits(const double* score, int heads, int n_high, int high_bits,
                             int low_bits, int8_t* bits_out);

/* Number of partial sums R of the key-axis reduction order for a given dk
 * (host-only): 8 for dk <= 128, 16 for dk = 256. */
int rsq_reduction_partials(int dk);

/* Decode step that allocates nothing (no counterpart in the method's pages).
 *
 * Same computation, arguments and results as rsq_decode_step, but without a
 * context: the configuration is passed directly and nothing is allocated.
 * rsq_create allocates a 4-byte device flag word (cudaMalloc, or the
 * config's allocator hook).  Some callers cannot allocate device memory once
 * they are running: serving runtimes that reserve nearly all GPU memory for
 * their own pools at start-up (a later cudaMalloc could fail or fragment what
 * the pool manages) and embedded hosts with a fixed memory budget.  They use
 * this entry point instead.  cfg->alloc, release and alloc_user are ignored.
 *
 * Its scratch (the decode kernel's flag word) lives in a statically allocated
 * device array of 64 words (256 bytes) that every GPU loading the library
 * holds until the process exits; a call needing more scratch than that is
 * rejected with RSQ_E_UNSUPPORTED.  All calls share the array.  The kernels
 * only set bits in its flag word and nothing reads or clears it, so a
 * non-finite column or a timed-out wait is not reported on this path (use a
 * context and rsq_check_flags for that), and overlapping calls may set bits
 * concurrently without harm.  The first call on a device looks up the
 * array's device address for that device, and the first call with a given
 * kernel sets its shared-memory attribute and queries its occupancy; make
 * those first calls before any stream capture.  The remembered address
 * belongs to the device's current context: after cudaDeviceReset it is
 * stale.  Errors as rsq_create plus rsq_decode_step. */
rsq_status rsq_decode_step_noalloc(const rsq_config* cfg, const rsq_state* state_in,
                                   const rsq_state* state_out, const void* inputs, float* out,
                                   uint32_t step, void* stream);

/* End-to-end pipeline over host buffers (no counterpart in the method's pages:
 * the serving-side plumbing of the decode step).
 *
 * rsq_host_input_layout: one step's inputs packed in one host buffer, the
 *   arrays of the family's input struct in its field order, each starting at
 *   a 16-byte aligned offset: GDN q, k, v, alpha, beta; GLA / KDA q, k, v,
 *   alpha (float [B][H][dk]), beta (GLA: 0 bytes); Mamba-2 x, Bm, Cm, dt, A, D
 *   (the decay is computed on the device).  Array shapes and types as in the
 *   input structs above.  offsets[6], sizes[6]: host arrays filled with each
 *   field's byte offset and byte count (unused entries 0); *total: the buffer
 *   size.  Host-only.
 * rsq_pipe_create: three non-blocking streams (input copy, compute, output
 *   copy), events and device staging for 3 steps in flight, on the current
 *   device, which must be the context's (else RSQ_E_INVAL; RSQ_E_NOMEM /
 *   RSQ_E_CUDA on failure).  The pipe borrows ctx: destroy the pipe first.
 *   rsq_pipe_step also returns RSQ_E_INVAL when called on another device.
 * rsq_pipe_step: one decode step.  Copies host_inputs (the packed layout;
 *   page-locked memory for the copies to overlap) to the device, runs
 *   rsq_decode_step (rsq_decode_step_window with win_in / win_out for a window
 *   context, else both NULL) on the compute stream, and copies the output
 *   [B][H][dv] to host_out.  Returns once the work is queued; when the pipe
 *   already has 3 steps in flight it first waits for the oldest to finish, so
 *   the host buffers of step n may be reused once step n + 3 has been issued
 *   (or after rsq_pipe_sync).  The states are read and written on the compute
 *   stream, in step order; a caller using them on another stream orders it
 *   against rsq_pipe_streams' compute stream.  Errors as rsq_decode_step.
 * rsq_pipe_sync: wait for every queued step.
 * rsq_pipe_streams: the pipe's three streams (cudaStream_t), e.g. to time it
 *   with events.  rsq_pipe_destroy waits for the pipe's work, then frees it
 *   (NULL is a no-op). */
typedef struct rsq_pipe rsq_pipe;
rsq_status rsq_host_input_layout(const rsq_ctx* ctx, size_t* offsets, size_t* sizes, size_t* total);
rsq_status rsq_pipe_create(const rsq_ctx* ctx, rsq_pipe** out);
void rsq_pipe_destroy(rsq_pipe* pipe);
rsq_status rsq_pipe_step(rsq_pipe* pipe, const rsq_state* state_in, const rsq_state* state_out,
                         const rsq_window* win_in, const rsq_window* win_out, const void* host_inputs,
                         float* host_out, uint32_t step);
rsq_status rsq_pipe_sync(rsq_pipe* pipe);
rsq_status rsq_pipe_streams(const rsq_pipe* pipe, void** copy_in, void** compute, void** copy_out);

const char* rsq_status_string(rsq_status s);
const char* rsq_last_error(void);
const char* rsq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RSQ_H */
