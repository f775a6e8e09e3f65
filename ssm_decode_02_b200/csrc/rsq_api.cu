// rsq_api.cu -- the C ABI declared in include/rsq.h: validation, context
// bookkeeping (per-head bit widths and offsets, launch geometry) and launches.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "rsq_internal.h"
#include "rsq_tile.cuh"

struct rsq_ctx {
    rsq_config cfg;
    int8_t bits[RSQ_MAX_HEADS];
    uint32_t head_off[RSQ_MAX_HEADS];
    long long row_bytes;
    bool f32state;
    int ub, ncb, units;   // 16-column blocks per unit, units per head, units per step
    int bpw;              // blocks each warp of the decode kernel takes per unit (1 or 2)
    int grid;        // persistent decode grid
    int ka_grid;     // persistent grid of the key-axis kernel (key-axis scales)
    int device;
    unsigned* flag;  // device word: rsq::kFlag* bits
    uint32_t wait_iters;  // limit of the kernels' bounded barrier waits (0: the default)
    int withhold;         // failure-detection tests: withhold an exchange-barrier arrival
};

namespace {

// The context's flag word goes back to whoever allocated it.
void release_flag(rsq_ctx* ctx) {
    if (!ctx->flag) return;
    if (ctx->cfg.release)
        ctx->cfg.release(ctx->flag, ctx->cfg.alloc_user);
    else
        cudaFree(ctx->flag);
    ctx->flag = nullptr;
}

thread_local char g_err[512] = "";

rsq_status fail(rsq_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

rsq_status cuda_fail(int err, const char* what) {
    return fail(RSQ_E_CUDA, "%s: %s", what, cudaGetErrorString(static_cast<cudaError_t>(err)));
}

constexpr int kCopyScaleBit = rsq::kRndCopy;  // kernel rule bit of the copy scale (beside the rsq_rounding bits)
// Kernel family of a configuration (Gated DeltaNet with a window has its own kernels).
int kernel_family(const rsq_config& c) {
    if (c.family != RSQ_GDN || c.window <= 0) return c.family;
    return rsq::kFamGdnPw + (c.window == 4 ? 0 : (c.window == 8 ? 1 : 2));
}
bool family_ok(int f) { return f == RSQ_GDN || f == RSQ_MAMBA2 || f == RSQ_GLA || f == RSQ_KDA; }
bool rounding_ok(int r) {
    return r == RSQ_RTN || r == RSQ_SR || r == RSQ_BDR || r == RSQ_SR_BDR || r == RSQ_SR8 || r == RSQ_SR8_BDR;
}
// nearest or stochastic rounding without the directional correction
bool plain_rounding(int r) { return r == RSQ_RTN || r == RSQ_SR || r == RSQ_SR8; }
// base-rounding bits of the kernels (stochastic, 8-bit uniforms)
int base_rule(int r) { return r & (rsq::kRndSr | rsq::kRndU8); }
// 16-column blocks per work unit (at most): four, except stochastic rounding
// at dk = 256, whose two-warp blocks run faster as 128-thread CTAs at three
// per SM (168 registers, no spills) than as 256-thread CTAs at two.
// Blocks per work unit.  At d_k = 256 stochastic rounding takes two (three
// 128-thread CTAs per SM at 168 registers, no spills) and BDR one: with two
// blocks per unit its instances spilled 400-700 bytes per thread, with four
// they take 255 registers and run one CTA per SM.
int unit_blocks(const rsq_config& c) {
    if (c.dk <= 128) return 4;
    if (c.rounding & RSQ_BDR) return 1;
    return (c.rounding & RSQ_SR) ? 2 : 4;
}

bool dk_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128 || d == 256; }
bool dv_ok(int d) { return d == 16 || d == 32 || d == 64 || d == 128 || d == 256; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Resident CTAs per SM of a decode kernel instance, after allowing its dynamic
// shared memory.  Nonzero cudaError_t on failure.
int instance_occupancy(const rsq_config& c, int ub, int bpw, bool f32state, int* per_sm, const void** func_out) {
    int threads = 0;
    size_t smem = 0;
    const void* func = nullptr;
    if (rsq::decode_kernel_info(kernel_family(c), c.dk, ub, bpw, f32state, c.rounding, &threads, &smem, &func) != 0)
        return -1;
    int err = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (!err) err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, func, threads, smem);
    if (!err && *per_sm < 1) err = cudaErrorInvalidConfiguration;
    if (func_out) *func_out = func;
    return err;
}

// Decode kernel geometry of a configuration: one block per warp, or two (64-
// thread CTAs, d_k = 128 units of four blocks) when the step has at least four
// units per resident CTA of that geometry -- there a warp's per-unit work
// serving two blocks pays off, while small steps keep more CTAs busy with one.
rsq_status choose_geometry(const rsq_config& c, int ub, bool f32state, long long units, int sms, int* bpw,
                           int* per_sm) {
    int err = instance_occupancy(c, ub, 1, f32state, per_sm, nullptr);
    if (err == -1) return fail(RSQ_E_UNSUPPORTED, "create: no kernel for dk=%d dv=%d", c.dk, c.dv);
    if (err) return cuda_fail(err, "create: launch geometry");
    *bpw = 1;
    if (!f32state && c.dk == 128 && ub == 4 && c.window == 0 && c.key_axis == 0) {
        int per_sm2 = 0;
        err = instance_occupancy(c, ub, 2, false, &per_sm2, nullptr);
        if (err == -1) return RSQ_OK;  // no two-block instance for this rule
        if (err) return cuda_fail(err, "create: launch geometry");
        if (units >= 4LL * sms * per_sm2) {
            *bpw = 2;
            *per_sm = per_sm2;
        }
    }
    return RSQ_OK;
}

template <class P>
void fill_heads(const rsq_ctx* c, P& p) {
    for (int h = 0; h < c->cfg.heads; ++h) {
        p.head_off[h] = c->head_off[h];
        p.head_bits[h] = static_cast<uint8_t>(c->bits[h]);
    }
}

rsq_status check_state(const rsq_ctx* c, const rsq_state* s, const char* name) {
    if (!s || !s->codes) return fail(RSQ_E_INVAL, "%s: null state or codes", name);
    if (!aligned16(s->codes)) return fail(RSQ_E_INVAL, "%s: codes not 16-byte aligned", name);
    if (!c->f32state) {
        if (!s->scales) return fail(RSQ_E_INVAL, "%s: null scales", name);
        if (!aligned16(s->scales)) return fail(RSQ_E_INVAL, "%s: scales not 16-byte aligned", name);
    }
    return RSQ_OK;
}

}  // namespace

extern "C" {

rsq_status rsq_debug_waits(rsq_ctx* ctx, uint32_t wait_iters, int withhold) {
    if (!ctx) return fail(RSQ_E_INVAL, "debug_waits: null context");
    if (withhold != 0 && withhold != 1) return fail(RSQ_E_INVAL, "debug_waits: withhold must be 0 or 1");
    ctx->wait_iters = wait_iters;
    ctx->withhold = withhold;
    return RSQ_OK;
}

const char* rsq_last_error(void) { return g_err; }

const char* rsq_version(void) { return "rsq 0.1 (sm_100a)"; }

const char* rsq_status_string(rsq_status s) {
    switch (s) {
        case RSQ_OK: return "ok";
        case RSQ_E_INVAL: return "invalid argument";
        case RSQ_E_UNSUPPORTED: return "unsupported configuration";
        case RSQ_E_CUDA: return "CUDA error";
        case RSQ_E_NOMEM: return "out of memory";
        case RSQ_E_NONFINITE: return "non-finite state column seen";
    }
    return "unknown status";
}

int rsq_reduction_partials(int dk) {
    // one partial per row group of a warp tile (rsq_tile.cuh); at dk = 256 two
    // warps share a block, each with 8 row groups of its own
    return dk > 128 ? 2 * rsq::kR : rsq::kR;
}

rsq_status rsq_allocate_bits(const double* score, int heads, int n_high, int high_bits,
                             int low_bits, int8_t* bits_out) {
    if (!score || !bits_out) return fail(RSQ_E_INVAL, "allocate_bits: null pointer");
    if (heads < 1 || heads > RSQ_MAX_HEADS) return fail(RSQ_E_INVAL, "allocate_bits: heads out of range");
    if (n_high < 0 || n_high > heads) return fail(RSQ_E_INVAL, "allocate_bits: n_high out of range");
    auto ok_bits = [](int b) { return b == 4 || b == 8; };
    if (!ok_bits(high_bits) || !ok_bits(low_bits)) return fail(RSQ_E_INVAL, "allocate_bits: bits must be 4 or 8");
    std::vector<int> order(static_cast<size_t>(heads));
    for (int h = 0; h < heads; ++h) order[h] = h;
    // slowest decay first; equal scores keep head order
    std::stable_sort(order.begin(), order.end(),
                     [&](int a, int b) { return score[a] > score[b]; });
    for (int h = 0; h < heads; ++h) bits_out[h] = static_cast<int8_t>(low_bits);
    for (int t = 0; t < n_high; ++t) bits_out[order[t]] = static_cast<int8_t>(high_bits);
    return RSQ_OK;
}

rsq_status rsq_create(const rsq_config* cfg, rsq_ctx** out) {
    if (!cfg || !out) return fail(RSQ_E_INVAL, "create: null argument");
    *out = nullptr;
    const rsq_config& c = *cfg;
    if (!family_ok(c.family)) return fail(RSQ_E_INVAL, "create: bad family %d", c.family);
    if (c.batch < 1) return fail(RSQ_E_INVAL, "create: batch must be >= 1");
    if (c.heads < 1 || c.heads > RSQ_MAX_HEADS) return fail(RSQ_E_INVAL, "create: heads must be in [1, %d]", RSQ_MAX_HEADS);
    if (!dk_ok(c.dk) || !dv_ok(c.dv))
        return fail(RSQ_E_UNSUPPORTED, "create: dk and dv must be one of 16, 32, 64, 128, 256 (got %d, %d)", c.dk, c.dv);
    if (!rounding_ok(c.rounding)) return fail(RSQ_E_INVAL, "create: bad rounding %d", c.rounding);
    if (c.in_dtype != RSQ_F32 && c.in_dtype != RSQ_BF16) return fail(RSQ_E_INVAL, "create: bad in_dtype %d", c.in_dtype);
    if (c.family == RSQ_MAMBA2 && (c.ngroups < 1 || c.heads % c.ngroups != 0))
        return fail(RSQ_E_INVAL, "create: ngroups must divide heads");
    if (c.window != 0 && c.window != 4 && c.window != 8 && c.window != 16)
        return fail(RSQ_E_INVAL, "create: window must be 0, 4, 8 or 16 (got %d)", c.window);
    if (c.window && c.family != RSQ_GDN)
        return fail(RSQ_E_UNSUPPORTED, "create: the pure-write window is defined for Gated DeltaNet");
    if (c.window && !plain_rounding(c.rounding))
        return fail(RSQ_E_UNSUPPORTED, "create: the pure-write window takes nearest or stochastic rounding");
    if (c.key_axis != 0 && c.key_axis != 1) return fail(RSQ_E_INVAL, "create: key_axis must be 0 or 1");
    if ((c.alloc == nullptr) != (c.release == nullptr))
        return fail(RSQ_E_INVAL, "create: set both alloc and release, or neither");
    if (c.key_axis && (c.family != RSQ_GDN || c.window || !plain_rounding(c.rounding)))
        return fail(RSQ_E_UNSUPPORTED, "create: key-axis scales: Gated DeltaNet, no window, nearest or stochastic rounding");
    if ((c.window || c.key_axis) && c.dk > 128)
        return fail(RSQ_E_UNSUPPORTED, "create: the pure-write window and key-axis scales are built for dk <= 128");

    rsq_ctx* ctx = new (std::nothrow) rsq_ctx();
    if (!ctx) return fail(RSQ_E_NOMEM, "create: host allocation failed");
    ctx->cfg = c;
    ctx->cfg.head_bits = nullptr;
    int n32 = 0;
    for (int h = 0; h < c.heads; ++h) {
        const int b = c.head_bits ? c.head_bits[h] : 8;
        if (b != 4 && b != 8 && b != 32) {
            delete ctx;
            return fail(RSQ_E_INVAL, "create: head %d has %d bits (4, 8 or 32)", h, b);
        }
        n32 += (b == 32);
        ctx->bits[h] = static_cast<int8_t>(b);
    }
    if (n32 != 0 && n32 != c.heads) {
        delete ctx;
        return fail(RSQ_E_UNSUPPORTED, "create: 32-bit heads cannot be mixed with 4/8-bit heads");
    }
    if (n32 && c.key_axis) {
        delete ctx;
        return fail(RSQ_E_UNSUPPORTED, "create: key-axis scales need 4/8-bit heads");
    }
    ctx->f32state = (n32 == c.heads);
    long long off = 0;
    for (int h = 0; h < c.heads; ++h) {
        ctx->head_off[h] = static_cast<uint32_t>(off);
        off += static_cast<long long>(c.dk) * c.dv * ctx->bits[h] / 8;
    }
    ctx->row_bytes = off;
    ctx->ub = std::min(c.dv / rsq::kBlockCols, unit_blocks(c));
    ctx->ncb = c.dv / (rsq::kBlockCols * ctx->ub);
    const long long units = static_cast<long long>(c.batch) * c.heads * ctx->ncb;
    if (units > (1LL << 30)) {
        delete ctx;
        return fail(RSQ_E_UNSUPPORTED, "create: too many work units");
    }
    ctx->units = static_cast<int>(units);

    // launch geometry: persistent grid of every resident CTA
    int err = cudaGetDevice(&ctx->device);
    int sms = 0, per_sm = 0;
    if (!err) err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, ctx->device);
    if (err) {
        delete ctx;
        return cuda_fail(err, "create");
    }
    const rsq_status gs = choose_geometry(c, ctx->ub, ctx->f32state, units, sms, &ctx->bpw, &per_sm);
    if (gs) {
        delete ctx;
        return gs;
    }
    if (!ctx->f32state) {
        // the copy-scale instance of the same rule (rsq_decode_step_copy_scale)
        int t2 = 0;
        size_t sm2 = 0;
        const void* f2 = nullptr;
        if (rsq::decode_kernel_info(kernel_family(c), c.dk, ctx->ub, ctx->bpw, false, c.rounding | kCopyScaleBit, &t2,
                                    &sm2, &f2) == 0)
            err = cudaFuncSetAttribute(f2, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(sm2));
    }
    if (!err) {
        if (c.alloc) {
            ctx->flag = static_cast<unsigned*>(c.alloc(sizeof(unsigned), c.alloc_user));
            if (!ctx->flag || (reinterpret_cast<uintptr_t>(ctx->flag) & 15u)) {
                if (ctx->flag) c.release(ctx->flag, c.alloc_user);
                delete ctx;
                return fail(RSQ_E_NOMEM, "create: the allocator hook returned no 16-byte aligned memory");
            }
        } else {
            err = cudaMalloc(&ctx->flag, sizeof(unsigned));
        }
    }
    if (!err) err = cudaMemset(ctx->flag, 0, sizeof(unsigned));
    if (err) {
        release_flag(ctx);
        delete ctx;
        if (err == cudaErrorMemoryAllocation) return fail(RSQ_E_NOMEM, "create: flag allocation failed");
        return cuda_fail(err, "create");
    }
    ctx->grid = static_cast<int>(std::min<long long>(units, static_cast<long long>(sms) * per_sm));
    if (c.key_axis) {
        // the key-axis kernel: one head at a time per CTA, every resident CTA
        int threads = 0, per_sm_ka = 0;
        size_t smem = 0;
        const void* func = nullptr;
        int e = rsq::decode_ka_info(c.dk, c.dv, base_rule(c.rounding), &threads, &smem, &func);
        if (e == 0) e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e == 0) e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm_ka, func, threads, smem);
        if (e == 0 && per_sm_ka < 1) e = cudaErrorInvalidConfiguration;
        if (e) {
            release_flag(ctx);
            delete ctx;
            return e == -1 ? fail(RSQ_E_UNSUPPORTED, "create: no key-axis kernel for dk=%d", c.dk)
                           : cuda_fail(e, "create: key-axis launch geometry");
        }
        ctx->ka_grid = static_cast<int>(std::min<long long>(static_cast<long long>(c.batch) * c.heads,
                                                            static_cast<long long>(sms) * per_sm_ka));
    }
    *out = ctx;
    return RSQ_OK;
}

void rsq_destroy(rsq_ctx* ctx) {
    if (!ctx) return;
    release_flag(ctx);
    delete ctx;
}

rsq_status rsq_state_bytes(const rsq_ctx* ctx, size_t* code_bytes, size_t* scale_bytes) {
    if (!ctx || !code_bytes || !scale_bytes) return fail(RSQ_E_INVAL, "state_bytes: null argument");
    *code_bytes = static_cast<size_t>(ctx->row_bytes) * ctx->cfg.batch;
    *scale_bytes = static_cast<size_t>(ctx->cfg.batch) * ctx->cfg.heads *
                   (ctx->cfg.key_axis ? ctx->cfg.dk : ctx->cfg.dv) * sizeof(float);
    return RSQ_OK;
}

rsq_status rsq_head_offset(const rsq_ctx* ctx, int h, size_t* offset) {
    if (!ctx || !offset) return fail(RSQ_E_INVAL, "head_offset: null argument");
    if (h < 0 || h >= ctx->cfg.heads) return fail(RSQ_E_INVAL, "head_offset: head out of range");
    *offset = ctx->head_off[h];
    return RSQ_OK;
}

namespace {
rsq_status decode_step_impl(const rsq_ctx* ctx, const rsq_state* state_in, const rsq_state* state_out,
                            const void* inputs, const float* copy_absmax, const rsq_window* win_in,
                            const rsq_window* win_out, float* out, uint32_t step, void* stream);
}

rsq_status rsq_decode_step(const rsq_ctx* ctx, const rsq_state* state_in, const rsq_state* state_out,
                           const void* inputs, float* out, uint32_t step, void* stream) {
    return decode_step_impl(ctx, state_in, state_out, inputs, nullptr, nullptr, nullptr, out, step, stream);
}

rsq_status rsq_window_bytes(const rsq_ctx* ctx, size_t* a_bytes, size_t* b_bytes, size_t* scale_bytes) {
    if (!ctx || !a_bytes || !b_bytes || !scale_bytes) return fail(RSQ_E_INVAL, "window_bytes: null argument");
    const rsq_config& c = ctx->cfg;
    const size_t bhw = static_cast<size_t>(c.batch) * c.heads * c.window;
    *a_bytes = bhw * c.dk;
    *b_bytes = bhw * c.dv;
    *scale_bytes = bhw * sizeof(float);
    return RSQ_OK;
}

rsq_status rsq_decode_step_window(const rsq_ctx* ctx, const rsq_state* state_in, const rsq_state* state_out,
                                  const rsq_window* win_in, const rsq_window* win_out, const void* inputs,
                                  float* out, uint32_t step, void* stream) {
    if (!ctx) return fail(RSQ_E_INVAL, "decode_step_window: null context");
    if (!win_in || !win_out) return fail(RSQ_E_INVAL, "decode_step_window: null window");
    const rsq_window* ws[2] = {win_in, win_out};
    for (const rsq_window* wv : ws)
        if (!wv->a || !wv->a_scale || !wv->b || !wv->b_scale || !aligned16(wv->a) || !aligned16(wv->a_scale) ||
            !aligned16(wv->b) || !aligned16(wv->b_scale))
            return fail(RSQ_E_INVAL, "decode_step_window: window buffer null or not 16-byte aligned");
    if (win_in->a == win_out->a || win_in->b == win_out->b || win_in->a_scale == win_out->a_scale ||
        win_in->b_scale == win_out->b_scale)
        return fail(RSQ_E_INVAL, "decode_step_window: win_in and win_out must be distinct buffers");
    return decode_step_impl(ctx, state_in, state_out, inputs, nullptr, win_in, win_out, out, step, stream);
}

rsq_status rsq_decode_step_copy_scale(const rsq_ctx* ctx, const rsq_state* state_in,
                                      const rsq_state* state_out, const void* inputs,
                                      const float* copy_absmax, float* out, uint32_t step,
                                      void* stream) {
    if (!ctx) return fail(RSQ_E_INVAL, "decode_step_copy_scale: null context");
    if (!copy_absmax || !aligned16(copy_absmax))
        return fail(RSQ_E_INVAL, "decode_step_copy_scale: copy_absmax null or not 16-byte aligned");
    if (ctx->f32state)
        return fail(RSQ_E_UNSUPPORTED, "decode_step_copy_scale: a full-precision state has no scale");
    if (ctx->cfg.window) return fail(RSQ_E_UNSUPPORTED, "decode_step_copy_scale: not with a pure-write window");
    return decode_step_impl(ctx, state_in, state_out, inputs, copy_absmax, nullptr, nullptr, out, step, stream);
}

rsq_status rsq_column_absmax(const rsq_ctx* ctx, const rsq_state* state, float* absmax, void* stream) {
    if (!ctx) return fail(RSQ_E_INVAL, "column_absmax: null context");
    if (!absmax || !aligned16(absmax)) return fail(RSQ_E_INVAL, "column_absmax: absmax null or not 16-byte aligned");
    rsq_status s = check_state(ctx, state, "column_absmax(state)");
    if (s) return s;
    const rsq_config& c = ctx->cfg;
    rsq::DequantParams p;
    std::memset(&p, 0, sizeof(p));
    p.B = c.batch; p.H = c.heads; p.dk = c.dk; p.dv = c.dv; p.ncb = ctx->ncb;
    p.row_bytes = ctx->row_bytes;
    p.codes = static_cast<const uint8_t*>(state->codes);
    p.scales = state->scales;
    p.absmax = absmax;
    p.key_axis = c.key_axis;
    fill_heads(ctx, p);
    const int err = rsq::launch_dequantize(c.dk, p, stream);
    if (err) return cuda_fail(err, "column_absmax launch");
    return RSQ_OK;
}

namespace {
rsq_status decode_step_impl(const rsq_ctx* ctx, const rsq_state* state_in, const rsq_state* state_out,
                            const void* inputs, const float* copy_absmax, const rsq_window* win_in,
                            const rsq_window* win_out, float* out, uint32_t step, void* stream) {
    if (!ctx) return fail(RSQ_E_INVAL, "decode_step: null context");
    if ((ctx->cfg.window > 0) != (win_in != nullptr))
        return fail(RSQ_E_INVAL, ctx->cfg.window ? "decode_step: this context has a pure-write window: use rsq_decode_step_window"
                                                 : "decode_step_window: this context has no window");
    rsq_status s = check_state(ctx, state_in, "decode_step(state_in)");
    if (s) return s;
    if ((s = check_state(ctx, state_out, "decode_step(state_out)"))) return s;
    if (!inputs) return fail(RSQ_E_INVAL, "decode_step: null inputs");
    if (!out || !aligned16(out)) return fail(RSQ_E_INVAL, "decode_step: out null or not 16-byte aligned");
    const rsq_config& c = ctx->cfg;
    rsq::DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    p.B = c.batch; p.H = c.heads; p.dk = c.dk; p.dv = c.dv; p.ncb = ctx->ncb; p.units = ctx->units;
    p.in_bf16 = (c.in_dtype == RSQ_BF16);
    p.rnd = base_rule(c.rounding);
    p.row_bytes = ctx->row_bytes;
    p.codes_in = static_cast<const uint8_t*>(state_in->codes);
    p.codes_out = static_cast<uint8_t*>(state_out->codes);
    p.scales_in = state_in->scales;
    p.scales_out = state_out->scales;
    p.out = out;
    p.copy_absmax = copy_absmax;
    if (win_in) {
        p.W = c.window;
        p.win_a_in = static_cast<const uint8_t*>(win_in->a);
        p.win_as_in = win_in->a_scale;
        p.win_b_in = static_cast<const uint8_t*>(win_in->b);
        p.win_bs_in = win_in->b_scale;
        p.win_a_out = static_cast<uint8_t*>(win_out->a);
        p.win_as_out = win_out->a_scale;
        p.win_b_out = static_cast<uint8_t*>(win_out->b);
        p.win_bs_out = win_out->b_scale;
    }
    p.flag = ctx->flag;
    p.step = step;
    p.key0 = static_cast<uint32_t>(c.seed);
    p.key1 = static_cast<uint32_t>(c.seed >> 32);
    p.rk = rsq::philox_round_keys(p.key0, p.key1);
    p.wait_iters = ctx->wait_iters ? ctx->wait_iters : rsq::kWaitIters;
    p.withhold = ctx->withhold;
    if (c.family == RSQ_GDN) {
        const rsq_gdn_inputs* in = static_cast<const rsq_gdn_inputs*>(inputs);
        if (!in->q || !in->k || !in->v || !in->alpha || !in->beta)
            return fail(RSQ_E_INVAL, "decode_step: null GDN input");
        if (!aligned16(in->q) || !aligned16(in->k) || !aligned16(in->v))
            return fail(RSQ_E_INVAL, "decode_step: q/k/v not 16-byte aligned");
        p.vA = in->q; p.vB = in->k; p.vC = in->v; p.g0 = in->alpha; p.g1 = in->beta;
        p.ngroups = 1; p.heads_per_group = c.heads;
    } else if (c.family == RSQ_GLA || c.family == RSQ_KDA) {
        const rsq_diag_inputs* in = static_cast<const rsq_diag_inputs*>(inputs);
        if (!in->q || !in->k || !in->v || !in->alpha || (c.family == RSQ_KDA && !in->beta))
            return fail(RSQ_E_INVAL, "decode_step: null GLA/KDA input");
        if (!aligned16(in->q) || !aligned16(in->k) || !aligned16(in->v) || !aligned16(in->alpha))
            return fail(RSQ_E_INVAL, "decode_step: q/k/v/alpha not 16-byte aligned");
        p.vA = in->q; p.vB = in->k; p.vC = in->v; p.vD = in->alpha;
        p.g0 = nullptr; p.g1 = (c.family == RSQ_KDA) ? in->beta : nullptr;
        p.ngroups = 1; p.heads_per_group = c.heads;
    } else {
        const rsq_mamba2_inputs* in = static_cast<const rsq_mamba2_inputs*>(inputs);
        if (!in->x || !in->Bm || !in->Cm || !in->dt || !in->A || !in->D)
            return fail(RSQ_E_INVAL, "decode_step: null Mamba-2 input");
        if (!aligned16(in->x) || !aligned16(in->Bm) || !aligned16(in->Cm))
            return fail(RSQ_E_INVAL, "decode_step: x/B/C not 16-byte aligned");
        p.vA = in->Cm; p.vB = in->Bm; p.vC = in->x; p.g0 = in->dt; p.g1 = in->decay;
        p.A = in->A; p.D = in->D;
        p.ngroups = c.ngroups; p.heads_per_group = c.heads / c.ngroups;
    }
    fill_heads(ctx, p);
    p.grid = ctx->grid;
    p.gcb = ctx->grid % ctx->ncb;
    const int ghu = ctx->grid / ctx->ncb;
    p.gh = ghu % c.heads;
    p.gb = ghu / c.heads;
    if (c.key_axis) {
        if (copy_absmax) return fail(RSQ_E_UNSUPPORTED, "decode_step_copy_scale: not with key-axis scales");
        p.grid = ctx->ka_grid;
        const int e = rsq::launch_decode_ka(c.dk, p, stream);
        if (e) return cuda_fail(e, "decode_step launch");
        return RSQ_OK;
    }
    const int err = rsq::launch_decode(kernel_family(c), c.dk, ctx->ub, ctx->bpw, ctx->f32state,
                                       c.rounding | (copy_absmax ? kCopyScaleBit : 0), p,
                                       stream);
    if (err) return cuda_fail(err, "decode_step launch");
    return RSQ_OK;
}

}  // namespace

rsq_status rsq_quantize(const rsq_ctx* ctx, const float* S, const rsq_state* state_out, uint32_t step,
                        void* stream) {
    if (!ctx) return fail(RSQ_E_INVAL, "quantize: null context");
    if (!S || !aligned16(S)) return fail(RSQ_E_INVAL, "quantize: S null or not 16-byte aligned");
    rsq_status s = check_state(ctx, state_out, "quantize(state_out)");
    if (s) return s;
    const rsq_config& c = ctx->cfg;
    rsq::QuantParams p;
    std::memset(&p, 0, sizeof(p));
    p.B = c.batch; p.H = c.heads; p.dk = c.dk; p.dv = c.dv; p.ncb = ctx->ncb; p.units = ctx->units;
    p.rnd = base_rule(c.rounding);
    p.row_bytes = ctx->row_bytes;
    p.S = S;
    p.codes = static_cast<uint8_t*>(state_out->codes);
    p.scales = state_out->scales;
    p.flag = ctx->flag;
    p.step = step;
    p.key0 = static_cast<uint32_t>(c.seed);
    p.key1 = static_cast<uint32_t>(c.seed >> 32);
    p.rk = rsq::philox_round_keys(p.key0, p.key1);
    fill_heads(ctx, p);
    const int err = c.key_axis ? rsq::launch_quantize_ka(c.dk, p, stream) : rsq::launch_quantize(c.dk, p, stream);
    if (err) return cuda_fail(err, "quantize launch");
    return RSQ_OK;
}

rsq_status rsq_dequantize(const rsq_ctx* ctx, const rsq_state* state_in, float* S_out, void* stream) {
    if (!ctx) return fail(RSQ_E_INVAL, "dequantize: null context");
    if (!S_out || !aligned16(S_out)) return fail(RSQ_E_INVAL, "dequantize: S_out null or not 16-byte aligned");
    rsq_status s = check_state(ctx, state_in, "dequantize(state_in)");
    if (s) return s;
    const rsq_config& c = ctx->cfg;
    rsq::DequantParams p;
    std::memset(&p, 0, sizeof(p));
    p.B = c.batch; p.H = c.heads; p.dk = c.dk; p.dv = c.dv; p.ncb = ctx->ncb;
    p.row_bytes = ctx->row_bytes;
    p.codes = static_cast<const uint8_t*>(state_in->codes);
    p.scales = state_in->scales;
    p.S = S_out;
    p.key_axis = c.key_axis;
    fill_heads(ctx, p);
    const int err = rsq::launch_dequantize(c.dk, p, stream);
    if (err) return cuda_fail(err, "dequantize launch");
    return RSQ_OK;
}

rsq_status rsq_state_drift(const rsq_ctx* q_ctx, const rsq_state* q_state, const rsq_ctx* f_ctx,
                           const rsq_state* f_state, double* sums, void* stream) {
    if (!q_ctx || !f_ctx || !sums) return fail(RSQ_E_INVAL, "state_drift: null argument");
    if (q_ctx->f32state || !f_ctx->f32state)
        return fail(RSQ_E_INVAL, "state_drift: need a quantized and a full-precision context");
    if (q_ctx->cfg.key_axis)
        return fail(RSQ_E_UNSUPPORTED, "state_drift: key-axis scales (use rsq_dequantize)");
    const rsq_config& a = q_ctx->cfg;
    const rsq_config& b = f_ctx->cfg;
    if (a.batch != b.batch || a.heads != b.heads || a.dk != b.dk || a.dv != b.dv)
        return fail(RSQ_E_INVAL, "state_drift: shapes differ");
    rsq_status s = check_state(q_ctx, q_state, "state_drift(q)");
    if (s) return s;
    if ((s = check_state(f_ctx, f_state, "state_drift(f)"))) return s;
    if (reinterpret_cast<uintptr_t>(sums) & 7u) return fail(RSQ_E_INVAL, "state_drift: sums not 8-byte aligned");
    rsq::DriftParams p;
    std::memset(&p, 0, sizeof(p));
    p.B = a.batch; p.H = a.heads; p.dk = a.dk; p.dv = a.dv; p.ncb = q_ctx->ncb;
    p.q_row_bytes = q_ctx->row_bytes;
    p.f_row_bytes = f_ctx->row_bytes;
    p.q_codes = static_cast<const uint8_t*>(q_state->codes);
    p.q_scales = q_state->scales;
    p.f_codes = static_cast<const uint8_t*>(f_state->codes);
    p.sums = sums;
    for (int h = 0; h < a.heads; ++h) {
        p.q_head_off[h] = q_ctx->head_off[h];
        p.q_head_bits[h] = static_cast<uint8_t>(q_ctx->bits[h]);
    }
    const int err = rsq::launch_drift(p, stream);
    if (err) return cuda_fail(err, "state_drift launch");
    return RSQ_OK;
}

rsq_status rsq_check_flags(const rsq_ctx* ctx, int* seen, void* stream) {
    if (!ctx || !seen) return fail(RSQ_E_INVAL, "check_flags: null argument");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned h = 0;
    int err = cudaStreamSynchronize(st);
    if (!err) err = cudaMemcpyAsync(&h, ctx->flag, sizeof(unsigned), cudaMemcpyDeviceToHost, st);
    if (!err) err = cudaMemsetAsync(ctx->flag, 0, sizeof(unsigned), st);
    if (!err) err = cudaStreamSynchronize(st);
    if (err) return cuda_fail(err, "check_flags");
    *seen = (h & rsq::kFlagNonFinite) ? 1 : 0;
    if (h & rsq::kFlagTimeout) return fail(RSQ_E_CUDA, "check_flags: a kernel barrier wait timed out");
    if (*seen) return fail(RSQ_E_NONFINITE, "check_flags: non-finite state column seen");
    return RSQ_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode step without any allocation.
//
// rsq_create allocates the context's 4-byte device flag word with cudaMalloc
// (or the configuration's allocator hook).  Some callers cannot allocate
// device memory after start-up: serving runtimes that reserve nearly all of
// the GPU's memory for their own pools when they start (a later cudaMalloc
// could fail, or fragment what the pool manages) and embedded hosts that run
// under a fixed memory budget.  This entry point keeps the flag word in a
// small statically allocated device array instead, so those callers can still
// run a decode step.
// ---------------------------------------------------------------------------
namespace {

constexpr int kNoallocScratchWords = 64;   // 256 bytes on every device that loads the library
constexpr int kNoallocWordsNeeded = 1;     // the decode kernel's flag word
constexpr int kNoallocMaxDevices = 64;
constexpr int kNoallocMaxKernels = 16;     // launch geometries remembered per device

// In host code this name is only a stand-in for the device array; its device
// address comes from cudaGetSymbolAddress (per device) below.
static __device__ __align__(256) unsigned g_noalloc_scratch[kNoallocScratchWords];

std::mutex g_noalloc_mu;
unsigned* g_noalloc_ptr[kNoallocMaxDevices] = {};

// Per device: the kernels already prepared (dynamic shared memory attribute
// set) and their resident CTAs per SM, so later calls make no attribute or
// occupancy query.
struct NoallocGeometry {
    const void* func;
    int per_sm;
};
NoallocGeometry g_noalloc_geom[kNoallocMaxDevices][kNoallocMaxKernels] = {};
int g_noalloc_sms[kNoallocMaxDevices] = {};

// Device address of the scratch array for the current device (resolved once
// per device, with that device current).
rsq_status noalloc_scratch(int device, unsigned** out) {
    if (device < 0 || device >= kNoallocMaxDevices)
        return fail(RSQ_E_UNSUPPORTED, "decode_step_noalloc: device index %d out of range", device);
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[device]) {
        void* ptr = nullptr;
        const int err = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (err) return cuda_fail(err, "decode_step_noalloc: cudaGetSymbolAddress");
        g_noalloc_ptr[device] = static_cast<unsigned*>(ptr);
    }
    *out = g_noalloc_ptr[device];
    return RSQ_OK;
}

// SM count and resident CTAs per SM of `func` on `device` (current), set up
// and queried on the first call for that kernel, remembered afterwards.
rsq_status noalloc_geometry(int device, const void* func, int threads, size_t smem, int* sms, int* per_sm) {
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    int err = 0;
    if (!g_noalloc_sms[device]) err = cudaDeviceGetAttribute(&g_noalloc_sms[device], cudaDevAttrMultiProcessorCount, device);
    if (err) return cuda_fail(err, "decode_step_noalloc: SM count");
    *sms = g_noalloc_sms[device];
    NoallocGeometry* slot = nullptr;
    for (auto& e : g_noalloc_geom[device]) {
        if (e.func == func) {
            *per_sm = e.per_sm;
            return RSQ_OK;
        }
        if (!e.func && !slot) slot = &e;
    }
    int n = 0;
    err = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (!err) err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem);
    if (!err && n < 1) err = cudaErrorInvalidConfiguration;
    if (err) return cuda_fail(err, "decode_step_noalloc: launch geometry");
    if (slot) *slot = NoallocGeometry{func, n};  // a full table only means the query repeats
    *per_sm = n;
    return RSQ_OK;
}

}  // namespace

extern "C" rsq_status rsq_decode_step_noalloc(const rsq_config* cfg, const rsq_state* state_in,
                                              const rsq_state* state_out, const void* inputs,
                                              float* out, uint32_t step, void* stream) {
    if (!cfg) return fail(RSQ_E_INVAL, "decode_step_noalloc: null config");
    const rsq_config& c = *cfg;
    if (!family_ok(c.family))
        return fail(RSQ_E_INVAL, "decode_step_noalloc: bad family %d", c.family);
    if (c.batch < 1) return fail(RSQ_E_INVAL, "decode_step_noalloc: batch must be >= 1");
    if (c.heads < 1 || c.heads > RSQ_MAX_HEADS)
        return fail(RSQ_E_INVAL, "decode_step_noalloc: heads must be in [1, %d]", RSQ_MAX_HEADS);
    if (!dk_ok(c.dk) || !dv_ok(c.dv))
        return fail(RSQ_E_UNSUPPORTED, "decode_step_noalloc: unsupported dk=%d dv=%d", c.dk, c.dv);
    if (!rounding_ok(c.rounding))
        return fail(RSQ_E_INVAL, "decode_step_noalloc: bad rounding %d", c.rounding);
    if (c.in_dtype != RSQ_F32 && c.in_dtype != RSQ_BF16)
        return fail(RSQ_E_INVAL, "decode_step_noalloc: bad in_dtype %d", c.in_dtype);
    if (c.family == RSQ_MAMBA2 && (c.ngroups < 1 || c.heads % c.ngroups != 0))
        return fail(RSQ_E_INVAL, "decode_step_noalloc: ngroups must divide heads");
    if (c.window != 0 || c.key_axis != 0)
        return fail(RSQ_E_UNSUPPORTED, "decode_step_noalloc: no pure-write window or key-axis scales here");
    if (kNoallocWordsNeeded > kNoallocScratchWords)
        return fail(RSQ_E_UNSUPPORTED, "decode_step_noalloc: needs %d scratch words, the static array holds %d",
                    kNoallocWordsNeeded, kNoallocScratchWords);

    // the context lives on the stack: bit widths, offsets and launch geometry
    rsq_ctx ctx;
    std::memset(&ctx, 0, sizeof(ctx));
    ctx.cfg = c;
    ctx.cfg.head_bits = nullptr;
    int n32 = 0;
    for (int h = 0; h < c.heads; ++h) {
        const int b = c.head_bits ? c.head_bits[h] : 8;
        if (b != 4 && b != 8 && b != 32)
            return fail(RSQ_E_INVAL, "decode_step_noalloc: head %d has %d bits (4, 8 or 32)", h, b);
        n32 += (b == 32);
        ctx.bits[h] = static_cast<int8_t>(b);
    }
    if (n32 != 0 && n32 != c.heads)
        return fail(RSQ_E_UNSUPPORTED, "decode_step_noalloc: 32-bit heads cannot be mixed with 4/8-bit heads");
    ctx.f32state = (n32 == c.heads);
    long long off = 0;
    for (int h = 0; h < c.heads; ++h) {
        ctx.head_off[h] = static_cast<uint32_t>(off);
        off += static_cast<long long>(c.dk) * c.dv * ctx.bits[h] / 8;
    }
    ctx.row_bytes = off;
    ctx.ub = std::min(c.dv / rsq::kBlockCols, unit_blocks(c));
    ctx.ncb = c.dv / (rsq::kBlockCols * ctx.ub);
    const long long units = static_cast<long long>(c.batch) * c.heads * ctx.ncb;
    if (units > (1LL << 30)) return fail(RSQ_E_UNSUPPORTED, "decode_step_noalloc: too many work units");
    ctx.units = static_cast<int>(units);

    int threads = 0;
    size_t smem = 0;
    const void* func = nullptr;
    ctx.bpw = 1;  // one block per warp (results do not depend on the geometry)
    if (rsq::decode_kernel_info(kernel_family(c), c.dk, ctx.ub, ctx.bpw, ctx.f32state, c.rounding, &threads, &smem,
                                &func) != 0)
        return fail(RSQ_E_UNSUPPORTED, "decode_step_noalloc: no kernel for dk=%d dv=%d", c.dk, c.dv);
    int err = cudaGetDevice(&ctx.device);
    if (err) return cuda_fail(err, "decode_step_noalloc: cudaGetDevice");
    unsigned* scratch = nullptr;
    rsq_status s = noalloc_scratch(ctx.device, &scratch);
    if (s) return s;
    int sms = 0, per_sm = 0;
    s = noalloc_geometry(ctx.device, func, threads, smem, &sms, &per_sm);
    if (s) return s;
    ctx.grid = static_cast<int>(std::min<long long>(units, static_cast<long long>(sms) * per_sm));

    // the kernels only set bits in the flag word and nothing reads it on this
    // path, so it is never cleared (every call shares the array)
    ctx.flag = scratch;
    return rsq_decode_step(&ctx, state_in, state_out, inputs, out, step, stream);
}

// ---------------------------------------------------------------------------
// Host-buffer pipeline (rsq_pipe): one call per step copies the step's packed
// inputs host -> device, runs the decode step and copies the output back, on
// three streams ordered by events, so step t's input copy, step t-1's kernel
// and step t-2's output copy overlap.  Device staging is owned by the pipe.
// ---------------------------------------------------------------------------
namespace {

constexpr int kPipeDepth = 3;   // steps in flight (staging and output buffers)
constexpr int kHostFields = 6;  // largest input struct (Mamba-2 without decay)

size_t round16(size_t n) { return (n + 15) / 16 * 16; }

// Byte sizes of the host input fields of a context, in its input struct's
// field order (unused entries 0).
void host_field_sizes(const rsq_config& c, size_t sizes[kHostFields]) {
    const size_t esz = (c.in_dtype == RSQ_BF16) ? 2 : 4;
    const size_t bh = static_cast<size_t>(c.batch) * c.heads;
    for (int f = 0; f < kHostFields; ++f) sizes[f] = 0;
    if (c.family == RSQ_MAMBA2) {
        const size_t bg = static_cast<size_t>(c.batch) * c.ngroups;
        sizes[0] = bh * c.dv * esz;  // x
        sizes[1] = bg * c.dk * esz;  // B
        sizes[2] = bg * c.dk * esz;  // C
        sizes[3] = bh * 4;           // dt
        sizes[4] = static_cast<size_t>(c.heads) * 4;  // A
        sizes[5] = static_cast<size_t>(c.heads) * 4;  // D
        return;
    }
    sizes[0] = bh * c.dk * esz;  // q
    sizes[1] = bh * c.dk * esz;  // k
    sizes[2] = bh * c.dv * esz;  // v
    sizes[3] = (c.family == RSQ_GDN) ? bh * 4 : bh * c.dk * 4;  // alpha: gate / decay per key channel
    sizes[4] = (c.family == RSQ_GLA) ? 0 : bh * 4;              // beta
}

}  // namespace

struct rsq_pipe {
    const rsq_ctx* ctx;
    size_t off[kHostFields], size[kHostFields];
    size_t in_bytes, out_bytes;
    uint8_t* stage[kPipeDepth];
    float* out_dev[kPipeDepth];
    cudaStream_t s_in, s_cmp, s_out;
    cudaEvent_t copied[kPipeDepth], done[kPipeDepth], read[kPipeDepth];
    unsigned long long issued;
};

rsq_status rsq_host_input_layout(const rsq_ctx* ctx, size_t* offsets, size_t* sizes, size_t* total) {
    if (!ctx || !offsets || !sizes || !total) return fail(RSQ_E_INVAL, "host_input_layout: null argument");
    host_field_sizes(ctx->cfg, sizes);
    size_t off = 0;
    for (int f = 0; f < kHostFields; ++f) {
        offsets[f] = off;
        off += round16(sizes[f]);
    }
    *total = off;
    return RSQ_OK;
}

void rsq_pipe_destroy(rsq_pipe* pipe) {
    if (!pipe) return;
    if (pipe->s_out) cudaStreamSynchronize(pipe->s_out);
    if (pipe->s_cmp) cudaStreamSynchronize(pipe->s_cmp);
    if (pipe->s_in) cudaStreamSynchronize(pipe->s_in);
    for (int i = 0; i < kPipeDepth; ++i) {
        if (pipe->stage[i]) cudaFree(pipe->stage[i]);
        if (pipe->out_dev[i]) cudaFree(pipe->out_dev[i]);
        if (pipe->copied[i]) cudaEventDestroy(pipe->copied[i]);
        if (pipe->done[i]) cudaEventDestroy(pipe->done[i]);
        if (pipe->read[i]) cudaEventDestroy(pipe->read[i]);
    }
    if (pipe->s_in) cudaStreamDestroy(pipe->s_in);
    if (pipe->s_cmp) cudaStreamDestroy(pipe->s_cmp);
    if (pipe->s_out) cudaStreamDestroy(pipe->s_out);
    delete pipe;
}

rsq_status rsq_pipe_create(const rsq_ctx* ctx, rsq_pipe** out) {
    if (!ctx || !out) return fail(RSQ_E_INVAL, "pipe_create: null argument");
    *out = nullptr;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != ctx->device)
        return fail(RSQ_E_INVAL, "pipe_create: the current device is not the context's device");
    rsq_pipe* p = new (std::nothrow) rsq_pipe();
    if (!p) return fail(RSQ_E_NOMEM, "pipe_create: host allocation failed");
    p->ctx = ctx;
    size_t total = 0;
    rsq_host_input_layout(ctx, p->off, p->size, &total);
    p->in_bytes = total;
    p->out_bytes = static_cast<size_t>(ctx->cfg.batch) * ctx->cfg.heads * ctx->cfg.dv * sizeof(float);
    int err = cudaStreamCreateWithFlags(&p->s_in, cudaStreamNonBlocking);
    if (!err) err = cudaStreamCreateWithFlags(&p->s_cmp, cudaStreamNonBlocking);
    if (!err) err = cudaStreamCreateWithFlags(&p->s_out, cudaStreamNonBlocking);
    for (int i = 0; i < kPipeDepth && !err; ++i) {
        err = cudaMalloc(&p->stage[i], p->in_bytes);
        if (!err) err = cudaMalloc(&p->out_dev[i], p->out_bytes);
        if (!err) err = cudaEventCreateWithFlags(&p->copied[i], cudaEventDisableTiming);
        if (!err) err = cudaEventCreateWithFlags(&p->done[i], cudaEventDisableTiming);
        if (!err) err = cudaEventCreateWithFlags(&p->read[i], cudaEventDisableTiming);
    }
    if (err) {
        rsq_pipe_destroy(p);
        if (err == cudaErrorMemoryAllocation) return fail(RSQ_E_NOMEM, "pipe_create: device allocation failed");
        return cuda_fail(err, "pipe_create");
    }
    *out = p;
    return RSQ_OK;
}

rsq_status rsq_pipe_step(rsq_pipe* pipe, const rsq_state* state_in, const rsq_state* state_out,
                         const rsq_window* win_in, const rsq_window* win_out, const void* host_inputs,
                         float* host_out, uint32_t step) {
    if (!pipe || !host_inputs || !host_out) return fail(RSQ_E_INVAL, "pipe_step: null argument");
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev != pipe->ctx->device)
        return fail(RSQ_E_INVAL, "pipe_step: the current device is not the context's device");
    const int i = static_cast<int>(pipe->issued % kPipeDepth);
    // the step that used slot i (kPipeDepth steps ago) has finished its output
    // copy, hence also its kernel and its input copy: the slot's buffers and
    // that step's host buffers are free again
    int err = 0;
    if (pipe->issued >= kPipeDepth) err = cudaEventSynchronize(pipe->read[i]);
    if (!err) err = cudaMemcpyAsync(pipe->stage[i], host_inputs, pipe->in_bytes, cudaMemcpyHostToDevice, pipe->s_in);
    if (!err) err = cudaEventRecord(pipe->copied[i], pipe->s_in);
    if (!err) err = cudaStreamWaitEvent(pipe->s_cmp, pipe->copied[i], 0);
    if (err) return cuda_fail(err, "pipe_step: input copy");
    const uint8_t* b = pipe->stage[i];
    const size_t* o = pipe->off;
    const rsq_config& c = pipe->ctx->cfg;
    rsq_gdn_inputs gi;
    rsq_diag_inputs di;
    rsq_mamba2_inputs mi;
    const void* inputs;
    if (c.family == RSQ_GDN) {
        gi = {b + o[0], b + o[1], b + o[2], reinterpret_cast<const float*>(b + o[3]),
              reinterpret_cast<const float*>(b + o[4])};
        inputs = &gi;
    } else if (c.family == RSQ_MAMBA2) {
        mi = {b + o[0], b + o[1], b + o[2], reinterpret_cast<const float*>(b + o[3]),
              reinterpret_cast<const float*>(b + o[4]), reinterpret_cast<const float*>(b + o[5]), nullptr};
        inputs = &mi;
    } else {
        di = {b + o[0], b + o[1], b + o[2], reinterpret_cast<const float*>(b + o[3]),
              c.family == RSQ_KDA ? reinterpret_cast<const float*>(b + o[4]) : nullptr};
        inputs = &di;
    }
    rsq_status s = decode_step_impl(pipe->ctx, state_in, state_out, inputs, nullptr, win_in, win_out,
                                    pipe->out_dev[i], step, pipe->s_cmp);
    if (s) return s;
    err = cudaEventRecord(pipe->done[i], pipe->s_cmp);
    if (!err) err = cudaStreamWaitEvent(pipe->s_out, pipe->done[i], 0);
    if (!err) err = cudaMemcpyAsync(host_out, pipe->out_dev[i], pipe->out_bytes, cudaMemcpyDeviceToHost, pipe->s_out);
    if (!err) err = cudaEventRecord(pipe->read[i], pipe->s_out);
    if (err) return cuda_fail(err, "pipe_step: output copy");
    ++pipe->issued;
    return RSQ_OK;
}

rsq_status rsq_pipe_sync(rsq_pipe* pipe) {
    if (!pipe) return fail(RSQ_E_INVAL, "pipe_sync: null pipe");
    int err = cudaStreamSynchronize(pipe->s_in);
    if (!err) err = cudaStreamSynchronize(pipe->s_cmp);
    if (!err) err = cudaStreamSynchronize(pipe->s_out);
    return err ? cuda_fail(err, "pipe_sync") : RSQ_OK;
}

rsq_status rsq_pipe_streams(const rsq_pipe* pipe, void** copy_in, void** compute, void** copy_out) {
    if (!pipe || !copy_in || !compute || !copy_out) return fail(RSQ_E_INVAL, "pipe_streams: null argument");
    *copy_in = pipe->s_in;
    *compute = pipe->s_cmp;
    *copy_out = pipe->s_out;
    return RSQ_OK;
}
