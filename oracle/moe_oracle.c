/*
 * moe_oracle.c -- plain CPU oracle for the MoE expert-epilogue ops.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, __graft_entry__.smoke() and the
 * CPU-baseline / reference legs of bench.py load this library.  The CUDA path
 * neither links nor calls it, and the two share no code, header or table.
 *
 * Each function is the plain definition of one op, one element at a time, in
 * the precision the pages fix: inputs are widened to fp32, the documented
 * formula is evaluated in fp32 in the order it reads, and the result is
 * rounded once (round-to-nearest-even) to the storage dtype.  Row sums whose
 * order the pages leave open (the probability gradients) are accumulated in
 * float64, together with the sum of the absolute terms, so that the tests can
 * bound any fp32 summation order against them.
 *
 * Sources (API reference pages, cited by page title and documented symbol):
 *   [OPT]  nemo_automodel.components.moe.optimized_ops
 *   [SWI]  nemo_automodel.components.moe.swiglu_triton
 *   [BI]   core.inference.moe.batch_invariant
 *   [RES]  core.fusions.fused_moe_residual_add
 *
 * Parity pins: every function here is pinned by the not-gpu tests in
 * tests/test_oracle_pins.py (library cross-checks, closed forms, float64
 * finite differences, brute force on tiny inputs).
 *
 * Build: gcc -O2 -std=c99 -ffp-contract=off -fno-fast-math -shared -fPIC -lm
 * (no FMA contraction: every product and sum is rounded on its own, as an
 * unfused fp32 evaluation of the formula would be).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

enum { ORC_BF16 = 0, ORC_F16 = 1, ORC_F32 = 2 };
enum { ORC_SQRELU = 0, ORC_SQRELU_CLAMP = 1, ORC_SWIGLU = 2 };
enum { ORC_ERR_COUNT = 1, ORC_ERR_MAP = 2, ORC_ERR_INVERSE = 4 };

/* ---------------------------------------------------------------- dtypes */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* bf16 = the top 16 bits of an fp32.  Round to nearest, ties to even: add
 * 0x7FFF plus the lowest kept bit, then truncate.  A carry out of the
 * significand bumps the exponent, which also yields +-inf on overflow.  NaN
 * keeps its sign and becomes the quiet NaN 0x7FC0. */
uint16_t orc_bf16_from_f32(float f)
{
    uint32_t u = bits_from_f32(f);
    if ((u & 0x7fffffffu) > 0x7f800000u)
        return (uint16_t)(((u >> 16) & 0x8000u) | 0x7fc0u);
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

float orc_f32_from_bf16(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits.
 * Round to nearest even, with gradual underflow and overflow to inf. */
uint16_t orc_f16_from_f32(float f)
{
    uint32_t u = bits_from_f32(f);
    uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
    uint32_t a = u & 0x7fffffffu;
    if (a > 0x7f800000u) return (uint16_t)(sign | 0x7e00u);   /* NaN */
    if (a == 0x7f800000u) return (uint16_t)(sign | 0x7c00u);  /* inf */
    int e = (int)(a >> 23) - 127;                               /* unbiased */
    if (e > 15) return (uint16_t)(sign | 0x7c00u);              /* >= 2^16 */
    if (e < -25) return sign;                                   /* < 2^-25: to zero */
    uint32_t mant = (a & 0x7fffffu) | 0x800000u;                /* 24-bit significand */
    if (e >= -14) {                                             /* normal binary16 */
        uint32_t q = mant >> 13, rem = mant & 0x1fffu;
        if (rem > 0x1000u || (rem == 0x1000u && (q & 1u))) q++;
        int he = e + 15;
        if (q == 0x800u) { q = 0x400u; he++; }                  /* significand carry */
        if (he >= 31) return (uint16_t)(sign | 0x7c00u);
        return (uint16_t)(sign | ((uint32_t)he << 10) | (q & 0x3ffu));
    }
    /* subnormal binary16: the value is q * 2^-24 with q = f / 2^-24 rounded */
    int shift = -(e + 1);                                       /* 14 .. 24 */
    uint32_t q = mant >> shift;
    uint32_t rem = mant & ((1u << shift) - 1u), half = 1u << (shift - 1);
    if (rem > half || (rem == half && (q & 1u))) q++;
    return (uint16_t)(sign | q);                                /* q == 0x400 is the smallest normal */
}

float orc_f32_from_f16(uint16_t h)
{
    uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
    uint32_t e = ((uint32_t)h >> 10) & 0x1fu, m = (uint32_t)h & 0x3ffu;
    if (e == 0) {                                 /* zero or subnormal: m * 2^-24 */
        float v = (float)m * 5.9604644775390625e-08f;
        return sign ? -v : v;
    }
    if (e == 31) return f32_from_bits(sign | 0x7f800000u | (m << 13));
    return f32_from_bits(sign | ((e - 15u + 127u) << 23) | (m << 13));
}

static float load_as_f32(const void *p, int dt, int64_t i)
{
    if (dt == ORC_BF16) return orc_f32_from_bf16(((const uint16_t *)p)[i]);
    if (dt == ORC_F16) return orc_f32_from_f16(((const uint16_t *)p)[i]);
    return ((const float *)p)[i];
}

/* Round an fp32 value once to the storage dtype and store it. */
static void store_rounded(void *p, int dt, int64_t i, float v)
{
    if (dt == ORC_BF16) ((uint16_t *)p)[i] = orc_bf16_from_f32(v);
    else if (dt == ORC_F16) ((uint16_t *)p)[i] = orc_f16_from_f32(v);
    else ((float *)p)[i] = v;
}

/* Round-trip through the storage dtype: what materialising a tensor does. */
static float round_to_dtype(float v, int dt)
{
    if (dt == ORC_BF16) return orc_f32_from_bf16(orc_bf16_from_f32(v));
    if (dt == ORC_F16) return orc_f32_from_f16(orc_f16_from_f32(v));
    return v;
}

/* ------------------------------------------------------- scalar functions */

/* logistic sigmoid, 1 / (1 + e^-z), in fp32 */
static float sigmoid_f32(float z) { return 1.0f / (1.0f + expf(-z)); }

/* torch.clamp(v, max=hi): NaN stays NaN (the comparison is false). */
static float clamp_max_f32(float v, float hi) { return (v > hi) ? hi : v; }

/* torch.clamp(v, lo, hi): NaN stays NaN. */
static float clamp_f32(float v, float lo, float hi)
{
    return (v < lo) ? lo : ((v > hi) ? hi : v);
}

/* ---------------------------------------------------- clamped SwiGLU [SWI] */

/* [SWI] module docstring and forward kernel: for every row r and column
 * j < inter, with gate g = x[r, j] and up u = x[r, inter + j],
 *     y[r, j] = silu(clamp(g, max=L)) * clamp(u, -L, L) * probs[r]
 * in fp32, rounded once to x's dtype (bf16, fp16 or fp32: the page's
 * _SUPPORTED_DTYPES).  silu(z) = z * sigmoid(z). */
void orc_swiglu_clamped_fwd_dt(const void *x, const float *probs, void *y, int64_t rows,
                               int64_t inter, int64_t ld_x, int64_t ld_y, float limit, int dt)
{
    for (int64_t r = 0; r < rows; ++r) {
        float p = probs[r];
        for (int64_t j = 0; j < inter; ++j) {
            float g = load_as_f32(x, dt, r * ld_x + j);
            float u = load_as_f32(x, dt, r * ld_x + inter + j);
            float gc = clamp_max_f32(g, limit);
            float uc = clamp_f32(u, -limit, limit);
            float s = gc * sigmoid_f32(gc);
            float v = s * uc;
            v = v * p;
            store_rounded(y, dt, r * ld_y + j, v);
        }
    }
}

void orc_swiglu_clamped_fwd(const uint16_t *x, const float *probs, uint16_t *y,
                            int64_t rows, int64_t inter, int64_t ld_x, int64_t ld_y,
                            float limit)
{
    orc_swiglu_clamped_fwd_dt(x, probs, y, rows, inter, ld_x, ld_y, limit, ORC_BF16);
}

/* [SWI] backward kernel: the chain rule of the forward above.
 *   a      = dy * p                         (gradient of silu(gc) * uc)
 *   d_gate = (a * uc) * silu'(gc) where g <= L, else 0
 *   d_up   = a * silu(gc)         where -L <= u <= L, else 0
 * with silu'(z) = sigmoid(z) * (1 + z * (1 - sigmoid(z))).  The masks are
 * torch.clamp's: inclusive ranges tested on the input values.  d_gate goes to
 * grad_x[r, j] and d_up to grad_x[r, inter + j], each rounded once to x's
 * dtype.  grad_probs[r] = sum_j dy * (silu(gc) * uc), each term in fp32, summed
 * here in float64; grad_probs_abs[r] is the float64 sum of the absolute terms. */
void orc_swiglu_clamped_bwd_dt(const void *x, const float *probs, const void *grad_y,
                               void *grad_x, double *grad_probs, double *grad_probs_abs,
                               int64_t rows, int64_t inter, int64_t ld_x, int64_t ld_gy,
                               int64_t ld_gx, float limit, int dt)
{
    for (int64_t r = 0; r < rows; ++r) {
        float p = probs[r];
        double acc = 0.0, acc_abs = 0.0;
        for (int64_t j = 0; j < inter; ++j) {
            float g = load_as_f32(x, dt, r * ld_x + j);
            float u = load_as_f32(x, dt, r * ld_x + inter + j);
            float dy = load_as_f32(grad_y, dt, r * ld_gy + j);
            float gc = clamp_max_f32(g, limit);
            float uc = clamp_f32(u, -limit, limit);
            float sg = sigmoid_f32(gc);
            float s = gc * sg;
            float a = dy * p;
            float dsilu = sg * (1.0f + gc * (1.0f - sg));
            float d_gate = (a * uc) * dsilu;
            float d_up = a * s;
            int gate_in = (g <= limit);
            int up_in = (u >= -limit) && (u <= limit);
            store_rounded(grad_x, dt, r * ld_gx + j, gate_in ? d_gate : 0.0f);
            store_rounded(grad_x, dt, r * ld_gx + inter + j, up_in ? d_up : 0.0f);
            float t = dy * (s * uc);
            acc += (double)t;
            acc_abs += fabs((double)t);
        }
        grad_probs[r] = acc;
        grad_probs_abs[r] = acc_abs;
    }
}

void orc_swiglu_clamped_bwd(const uint16_t *x, const float *probs, const uint16_t *grad_y,
                            uint16_t *grad_x, double *grad_probs, double *grad_probs_abs,
                            int64_t rows, int64_t inter, int64_t ld_x, int64_t ld_gy,
                            int64_t ld_gx, float limit)
{
    orc_swiglu_clamped_bwd_dt(x, probs, grad_y, grad_x, grad_probs, grad_probs_abs, rows, inter,
                              ld_x, ld_gy, ld_gx, limit, ORC_BF16);
}

/* float64 twin of the forward, unrounded, for finite-difference checks of the
 * backward: y = silu(min(g, L)) * clamp(u, -L, L) * p elementwise. */
void orc_swiglu_clamped_fwd_f64(const double *g, const double *u, const double *p,
                                double *y, int64_t n, double limit)
{
    for (int64_t i = 0; i < n; ++i) {
        double gc = (g[i] > limit) ? limit : g[i];
        double uc = (u[i] < -limit) ? -limit : ((u[i] > limit) ? limit : u[i]);
        double s = gc / (1.0 + exp(-gc));
        y[i] = s * uc * p[i];
    }
}

/* ------------------------------------------------ router-weight multiply [OPT] */

/* [OPT] _rw_fwd_core: out = (x.float() * probs.float()).to(out_dtype), one
 * fp32 multiply per element and one rounding.  probs has dtype p_dt (widened
 * exactly to fp32). */
void orc_router_weight_fwd_p(const void *x, int x_dt, const void *probs, int p_dt, void *out,
                             int out_dt, int64_t rows, int64_t hidden)
{
    for (int64_t r = 0; r < rows; ++r) {
        float p = load_as_f32(probs, p_dt, r);
        for (int64_t h = 0; h < hidden; ++h) {
            float v = load_as_f32(x, x_dt, r * hidden + h) * p;
            store_rounded(out, out_dt, r * hidden + h, v);
        }
    }
}

void orc_router_weight_fwd(const void *x, int x_dt, const float *probs, void *out,
                           int out_dt, int64_t rows, int64_t hidden)
{
    orc_router_weight_fwd_p(x, x_dt, probs, ORC_F32, out, out_dt, rows, hidden);
}

/* [OPT] _rw_bwd_x_core and _rw_bwd_probs_core:
 *   grad_x = (g_f32 * probs_f32).to(x.dtype)
 *   grad_probs = (g_f32 * x_f32).sum(-1)   (fp32 terms, summed here in float64;
 *                                           the caller rounds to probs.dtype)
 * x == NULL means the forward did not save x (save_x false): the probability
 * gradient is not computed. */
void orc_router_weight_bwd_p(const void *grad_out, int g_dt, const void *x, int x_dt,
                             const void *probs, int p_dt, void *grad_x, double *grad_probs,
                             double *grad_probs_abs, int64_t rows, int64_t hidden)
{
    for (int64_t r = 0; r < rows; ++r) {
        float p = load_as_f32(probs, p_dt, r);
        double acc = 0.0, acc_abs = 0.0;
        for (int64_t h = 0; h < hidden; ++h) {
            float g = load_as_f32(grad_out, g_dt, r * hidden + h);
            store_rounded(grad_x, x_dt, r * hidden + h, g * p);
            if (x) {
                float t = g * load_as_f32(x, x_dt, r * hidden + h);
                acc += (double)t;
                acc_abs += fabs((double)t);
            }
        }
        if (x) {
            grad_probs[r] = acc;
            grad_probs_abs[r] = acc_abs;
        }
    }
}

void orc_router_weight_bwd(const void *grad_out, int g_dt, const void *x, int x_dt,
                           const float *probs, void *grad_x, double *grad_probs,
                           double *grad_probs_abs, int64_t rows, int64_t hidden)
{
    orc_router_weight_bwd_p(grad_out, g_dt, x, x_dt, probs, ORC_F32, grad_x, grad_probs,
                            grad_probs_abs, rows, hidden);
}

/* ------------------------------------ batch-invariant permuted activation [BI] */

/* [BI] _squared_relu_with_probs_kernel / _swiglu_with_probs_kernel.
 * Rows r < n_used are live.  map[r] >= 0 is the flat index of the row's
 * routing probability; map[r] < 0 marks an alignment padding row, which is
 * zero-filled when zero_padding is set and otherwise left untouched.  Rows at
 * or past n_used are never read or written.
 *   SQRELU:        sq = bf16(relu(x)^2); out = bf16(f32(sq) * p)
 *   SQRELU_CLAMP:  z = s * tanh(x / s); out = bf16(relu(z)^2 * p), all fp32
 *   SWIGLU:        out = bf16(silu(gate) * up * p), gate = first half of the
 *                  2*width input row, up = second half.
 * Bad metadata is reported, not trusted: an n_used outside [0, max_rows] is
 * clamped (ORC_ERR_COUNT); a map entry >= num_probs skips its row
 * (ORC_ERR_MAP).  Returns the error bits. */
int orc_act_with_probs_permuted(int act, const uint16_t *x, uint16_t *out,
                                const int32_t *permutation_map, int32_t n_used,
                                const float *probs, int64_t num_probs, int64_t max_rows,
                                int64_t width, float clamp_scale, int zero_padding)
{
    int err = 0;
    int64_t n = n_used;
    if (n < 0) { n = 0; err |= ORC_ERR_COUNT; }
    if (n > max_rows) { n = max_rows; err |= ORC_ERR_COUNT; }
    int64_t in_w = (act == ORC_SWIGLU) ? 2 * width : width;
    for (int64_t r = 0; r < n; ++r) {
        int32_t m = permutation_map[r];
        if (m < 0) {
            if (zero_padding)
                for (int64_t j = 0; j < width; ++j) out[r * width + j] = 0;
            continue;
        }
        if ((int64_t)m >= num_probs) { err |= ORC_ERR_MAP; continue; }
        float p = probs[m];
        for (int64_t j = 0; j < width; ++j) {
            float v;
            if (act == ORC_SQRELU) {
                float xv = orc_f32_from_bf16(x[r * in_w + j]);
                float rl = (xv < 0.0f) ? 0.0f : xv;            /* relu, NaN kept */
                float sq = round_to_dtype(rl * rl, ORC_BF16);   /* the bf16 square */
                v = sq * p;
            } else if (act == ORC_SQRELU_CLAMP) {
                float xv = orc_f32_from_bf16(x[r * in_w + j]);
                float z = clamp_scale * tanhf(xv / clamp_scale);
                float rl = (z < 0.0f) ? 0.0f : z;
                v = (rl * rl) * p;
            } else {
                float g = orc_f32_from_bf16(x[r * in_w + j]);
                float u = orc_f32_from_bf16(x[r * in_w + width + j]);
                float s = g * sigmoid_f32(g);
                v = (s * u) * p;
            }
            out[r * width + j] = orc_bf16_from_f32(v);
        }
    }
    return err;
}

/* ------------------------------------------- fixed-order unpermute [BI] */

/* [BI] _unpermute_tokens_in_expert_order_kernel: for each token t below
 * valid_tokens, out[t, :] = sum over local experts e = 0, 1, ..., E-1 in
 * increasing order of expert_output[inverse_map[t, e], :], accumulated in fp32
 * from +0, then rounded once to out's dtype.  inverse_map[t, e] < 0 means the
 * token was not routed to local expert e.  Tokens at or past valid_tokens are
 * left untouched.  A valid_tokens outside [0, tokens] is clamped
 * (ORC_ERR_COUNT); an entry >= max_rows is skipped (ORC_ERR_INVERSE). */
int orc_unpermute_ordered(const void *expert_output, int in_dt, int64_t max_rows,
                          const int32_t *inverse_map, int32_t valid_tokens, void *out,
                          int out_dt, int64_t tokens, int64_t hidden,
                          int32_t num_local_experts)
{
    int err = 0;
    int64_t n = valid_tokens;
    if (n < 0) { n = 0; err |= ORC_ERR_COUNT; }
    if (n > tokens) { n = tokens; err |= ORC_ERR_COUNT; }
    for (int64_t t = 0; t < n; ++t)
        for (int64_t h = 0; h < hidden; ++h) {
            float acc = 0.0f;
            for (int32_t e = 0; e < num_local_experts; ++e) {
                int32_t row = inverse_map[t * num_local_experts + e];
                if (row < 0) continue;
                if ((int64_t)row >= max_rows) { err |= ORC_ERR_INVERSE; continue; }
                acc = acc + load_as_f32(expert_output, in_dt, (int64_t)row * hidden + h);
            }
            store_rounded(out, out_dt, t * hidden + h, acc);
        }
    return err;
}

/* --------------------------------------------------- residual add [RES] */

/* [RES] module docstring: out = residual + (expert_output + shared_expert_output),
 * where the expert sum is rounded to the activation dtype before the residual
 * is added -- i.e. exactly the two unfused adds, each computed in fp32 and
 * rounded to the dtype. */
void orc_residual_add(const void *expert_output, const void *shared_expert_output,
                      const void *residual, void *out, int64_t numel, int dt)
{
    for (int64_t i = 0; i < numel; ++i) {
        float e = load_as_f32(expert_output, dt, i);
        float s = load_as_f32(shared_expert_output, dt, i);
        float r = load_as_f32(residual, dt, i);
        float t = round_to_dtype(e + s, dt);
        store_rounded(out, dt, i, r + t);
    }
}

/* ------------------------------------- device-bounded weighted SwiGLU [BI] */

/* [BI] _weighted_silu_mul_bounded_kernel, weighted_silu_mul_bounded: y is
 * [rows, 2*half_n] (gate | up), out is [rows, half_n], weights [rows].  Every
 * output element e = r * half_n + j below bound_elems gets
 *     out[r, j] = bf16( silu(gate) * up * weights[r] )     (fp32, one rounding)
 * and elements at or past the bound are neither read nor written.  A bound
 * outside [0, rows*half_n] is clamped (ORC_ERR_COUNT).  Returns the error bits. */
int orc_weighted_silu_mul_bounded(const uint16_t *y, const float *weights, uint16_t *out,
                                  int64_t bound_elems, int64_t rows, int64_t half_n)
{
    int err = 0;
    int64_t n = bound_elems;
    if (n < 0) { n = 0; err |= ORC_ERR_COUNT; }
    if (n > rows * half_n) { n = rows * half_n; err |= ORC_ERR_COUNT; }
    for (int64_t e = 0; e < n; ++e) {
        int64_t r = e / half_n, j = e % half_n;
        float g = orc_f32_from_bf16(y[r * 2 * half_n + j]);
        float u = orc_f32_from_bf16(y[r * 2 * half_n + half_n + j]);
        float s = g * sigmoid_f32(g);
        float v = (s * u) * weights[r];
        out[r * half_n + j] = orc_bf16_from_f32(v);
    }
    return err;
}

/* ------------------------------------------- fused epilogue chain [OPT][BI][RES] */

/* The epilogue chain as three materialised steps, each exactly as above:
 *   1. router-weight multiply per expert-output row ([OPT] _rw_fwd_core with the
 *      permuted probabilities): w[row, :] = round_dt(eo[row, :] * row_probs[row])
 *   2. fixed-order unpermute ([BI]): routed[t, :] = round_dt(sum over e ascending
 *      of w[inverse_map[t, e], :]), fp32 from +0
 *   3. residual add ([RES]): out[t, :] = round_dt(residual + round_dt(routed + shared))
 * for tokens t < valid_tokens; other tokens untouched.  `scratch` is a
 * caller-provided [max_rows, hidden] buffer of dtype dt for step 1 and
 * `routed` a [tokens, hidden] one for step 2.  Returns the unpermute's error bits. */
int orc_epilogue_chain(const void *expert_output, const float *row_probs, int64_t max_rows,
                       const int32_t *inverse_map, int32_t valid_tokens,
                       const void *shared_expert_output, const void *residual, void *out,
                       int64_t tokens, int64_t hidden, int32_t num_local_experts, int dt,
                       void *scratch, void *routed)
{
    orc_router_weight_fwd(expert_output, dt, row_probs, scratch, dt, max_rows, hidden);
    int err = orc_unpermute_ordered(scratch, dt, max_rows, inverse_map, valid_tokens, routed, dt,
                                    tokens, hidden, num_local_experts);
    int64_t n = valid_tokens < 0 ? 0 : (valid_tokens > tokens ? tokens : valid_tokens);
    orc_residual_add(routed, shared_expert_output, residual, out, n * hidden, dt);
    return err;
}

/* ------------------------------------- rank-order reduce-scatter [BI] */

/* [BI] ordered_reduce_scatter_v, _ordered_reduce_scatter_v_kernel ("reduce peer
 * rows with an explicit rank-order FP32 sum"): each of `world` ranks holds a
 * [capacity_rows, hidden] buffer (dtype in_dt) of partial results for the
 * tokens of every rank; rank q's tokens are the rows starting at
 * rank_token_offset[q].  Rank `rank` receives its local_tokens rows:
 *     out[t, h] = out_dt( ((x_0 + x_1) + x_2) + ... + x_{world-1} ),
 *     x_q = f32(inputs[q][rank_token_offset[rank] + t, h]),
 * each add in fp32 in rank order, one rounding at the end.  Only the first
 * ep_tokens rows of the buffers hold data (the page's ep_max_tokens); an
 * ep_tokens outside [0, capacity_rows] is clamped, and an output row whose
 * source row falls outside the data is neither read nor written; both set
 * ORC_ERR_COUNT.  Returns the error bits. */
int orc_ordered_reduce_scatter_v(const void *const *inputs, int32_t world, int32_t rank,
                                 const int32_t *rank_token_offset, int32_t ep_tokens,
                                 int64_t capacity_rows, int64_t local_tokens, int64_t hidden,
                                 int in_dt, void *out, int out_dt)
{
    int err = 0;
    int64_t rows = ep_tokens;
    if (rows < 0) { rows = 0; err |= ORC_ERR_COUNT; }
    if (rows > capacity_rows) { rows = capacity_rows; err |= ORC_ERR_COUNT; }
    const int64_t first = rank_token_offset[rank];
    for (int64_t t = 0; t < local_tokens; ++t) {
        const int64_t g = first + t;
        if (g < 0 || g >= rows) { err |= ORC_ERR_COUNT; continue; }
        for (int64_t h = 0; h < hidden; ++h) {
            float acc = load_as_f32(inputs[0], in_dt, g * hidden + h);
            for (int32_t q = 1; q < world; ++q)
                acc = acc + load_as_f32(inputs[q], in_dt, g * hidden + h);
            store_rounded(out, out_dt, t * hidden + h, acc);
        }
    }
    return err;
}

/* --------------- EP combine: unpermute, then rank-order reduce-scatter [BI] */

/* [BI] _unpermute_tokens_in_expert_order_kernel followed by
 * ordered_reduce_scatter_v, materialised as the pages run them: every rank q
 * unpermutes its own expert outputs (expert_outputs[q], rows of its
 * num_local_experts experts, inverse_maps[q] over the capacity_rows token rows
 * of all ranks) for the first ep_tokens tokens into a block of partial sums of
 * dtype partial_dt; rank `rank` then sums its token rows over the ranks'
 * blocks in rank order and rounds once to out_dt.  `partials` is a
 * caller-provided buffer of world * capacity_rows * hidden elements of
 * partial_dt (the symmetric buffers).  Returns the error bits of both steps. */
int orc_unpermute_reduce_scatter(const void *const *expert_outputs, int eo_dt, int64_t max_rows,
                                 const int32_t *const *inverse_maps, int32_t num_local_experts,
                                 int64_t capacity_rows, int32_t ep_tokens, int32_t world,
                                 int32_t rank, const int32_t *rank_token_offset, int partial_dt,
                                 void *partials, void *out, int out_dt, int64_t local_tokens,
                                 int64_t hidden)
{
    int err = 0;
    const int64_t esize = partial_dt == ORC_F32 ? 4 : 2;
    const void *blocks[64];
    if (world < 1 || world > 64) return ORC_ERR_COUNT;
    for (int32_t q = 0; q < world; ++q) {
        void *block = (char *)partials + (int64_t)q * capacity_rows * hidden * esize;
        err |= orc_unpermute_ordered(expert_outputs[q], eo_dt, max_rows, inverse_maps[q],
                                     ep_tokens, block, partial_dt, capacity_rows, hidden,
                                     num_local_experts);
        blocks[q] = block;
    }
    err |= orc_ordered_reduce_scatter_v(blocks, world, rank, rank_token_offset, ep_tokens,
                                        capacity_rows, local_tokens, hidden, partial_dt, out,
                                        out_dt);
    return err;
}
