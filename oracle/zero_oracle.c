/*
 * CPU oracle for the ZeRO optimizer step: per-element arithmetic.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; only the test suite, the smoke check and the bench's
 * CPU-baseline leg load it.  It shares no source, header or table with the
 * CUDA path.
 *
 * Plain, slow, single-threaded loops.  Every floating-point operation is one
 * IEEE-754 binary32 (or binary64 where stated) operation rounded to nearest
 * even; compile with -O2 -ffp-contract=off and no fast-math so that no
 * multiply-add is contracted and no subnormal is flushed.
 *
 * Sources (three web pages on ZeRO):
 *   [T]  "ZERO训练技术" (wqh011128.github.io)
 *   [M]  "ZeRO：从优化器状态到残差状态的显存优化" (xuesongtap.github.io)
 *   [Q]  mstx.cn post 475, a ZeRO interview write-up
 * The pages fix the precisions (16-bit params and grads, fp32 master, m, v:
 * [M] section 1 table; [Q] section 二) but print no equation for the reduction
 * or for Adam.  The readings taken are stated at each function.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static float f32_of_bits(uint32_t u) {
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

static uint32_t bits_of_f32(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return u;
}

/* ---------------------------------------------------------------- bf16 ---- */

/* bf16 -> fp32 is exact: a bf16 is the upper half of a binary32 pattern. */
float zo_bf16_to_f32(uint16_t h) { return f32_of_bits((uint32_t)h << 16); }

/* The real value of a bf16 pattern for distance comparisons; the two
 * infinity patterns stand for +-2^128, the point one ulp beyond the largest
 * finite bf16, so that IEEE overflow rounding falls out of the same rule. */
static double bf16_value_ext(uint16_t h) {
  if ((h & 0x7FFFu) == 0x7F80u) return (h & 0x8000u) ? -ldexp(1.0, 128) : ldexp(1.0, 128);
  return (double)zo_bf16_to_f32(h);
}

/*
 * fp32 -> bf16, round to nearest, ties to even (IEEE-754 roundTiesToEven
 * applied to an 8-bit significand): take the two bf16 neighbours of x (the
 * truncation toward zero and the next pattern away from zero), keep the
 * nearer, and on a tie keep the one whose last significand bit is 0.
 * NaN maps to a quiet NaN with the sign and the upper payload bits kept.
 * Used for the averaged gradient and for the cast of the master weights to
 * the 16-bit parameter copy ([M] section 1 table; [T] section "ZeRO-1").
 */
uint16_t zo_bf16_rne(float x) {
  uint32_t u = bits_of_f32(x);
  if (isnan(x)) return (uint16_t)((u >> 16) | 0x0040u);
  uint16_t toward_zero = (uint16_t)(u >> 16);
  if ((u & 0xFFFFu) == 0u) return toward_zero;          /* exactly representable */
  uint16_t away = (uint16_t)(toward_zero + 1u);          /* same sign, larger magnitude */
  double xd = (double)x;                                 /* exact */
  double d_tz = fabs(xd - bf16_value_ext(toward_zero));  /* exact: both within 2^-133..2^128 */
  double d_aw = fabs(bf16_value_ext(away) - xd);
  if (d_tz < d_aw) return toward_zero;
  if (d_aw < d_tz) return away;
  return (toward_zero & 1u) ? away : toward_zero;
}

void zo_bf16_rne_array(int64_t n, const float* x, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = zo_bf16_rne(x[i]);
}

void zo_bf16_to_f32_array(int64_t n, const uint16_t* h, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = zo_bf16_to_f32(h[i]);
}

/* ------------------------------------------------------------ reduction ---- */

/*
 * The "reduce" half of reduce-scatter / all-reduce ([T] section "ZeRO-2",
 * part "reduce-scatter 是什么"; [Q] section 四.3): for every element i, the
 * average over the N data-parallel ranks of rank-local gradient i.
 *
 * Reading (the pages say "sum or average" only): the sum runs in fixed rank
 * order 0..N-1 into a binary32 accumulator that starts at +0; the mean is
 * that sum times the binary32 reciprocal of N (exact for power-of-two N);
 * the averaged gradient is stored as bf16 (round to nearest even), since the
 * pages account gradients at 2 bytes per element everywhere.
 *
 * rank_grads[r] points at element 0 of rank r's slice; n elements each.
 */
void zo_reduce_mean(int32_t n_ranks, int64_t n, const uint16_t* const* rank_grads, uint16_t* out) {
  const float inv_n = (float)(1.0 / (double)n_ranks);
  for (int64_t i = 0; i < n; ++i) {
    float acc = 0.0f;
    for (int32_t r = 0; r < n_ranks; ++r) acc = acc + zo_bf16_to_f32(rank_grads[r][i]);
    out[i] = zo_bf16_rne(acc * inv_n);
  }
}

/* Same sum in fp32 without the mean and the bf16 rounding, for the tests that
 * bound the accumulation error against the exact sum. */
void zo_rank_sum_f32(int32_t n_ranks, int64_t n, const uint16_t* const* rank_grads, float* out) {
  for (int64_t i = 0; i < n; ++i) {
    float acc = 0.0f;
    for (int32_t r = 0; r < n_ranks; ++r) acc = acc + zo_bf16_to_f32(rank_grads[r][i]);
    out[i] = acc;
  }
}

/* ----------------------------------------------------------------- Adam ---- */

/*
 * Host scalars of Adam step t (t >= 1).  The hyper-parameters arrive as
 * binary64 numbers (as a user writes them); every scalar the per-element
 * update uses is computed in binary64 and rounded once to binary32:
 *   out[0] = beta1            out[1] = beta2
 *   out[2] = 1 - beta1        out[3] = 1 - beta2
 *   out[4] = bc1 = 1 - beta1^t
 *   out[5] = bc2 = 1 - beta2^t
 *   out[6] = decay = 1 - lr * weight_decay
 *   out[7] = lr               out[8] = eps
 * beta^t is t successive binary64 multiplications of beta.
 */
void zo_adam_scalars(double lr, double beta1, double beta2, double eps, double weight_decay,
                     int64_t t, float* out) {
  double p1 = 1.0, p2 = 1.0;
  for (int64_t k = 0; k < t; ++k) {
    p1 = p1 * beta1;
    p2 = p2 * beta2;
  }
  out[0] = (float)beta1;
  out[1] = (float)beta2;
  out[2] = (float)(1.0 - beta1);
  out[3] = (float)(1.0 - beta2);
  out[4] = (float)(1.0 - p1);
  out[5] = (float)(1.0 - p2);
  out[6] = (float)(1.0 - lr * weight_decay);
  out[7] = (float)lr;
  out[8] = (float)eps;
}

/*
 * Mixed-precision Adam on one rank's owned elements ([T] section "ZeRO-1",
 * part "3. 更新"; [M] section 1 table for the state set: fp32 master weight,
 * fp32 first moment m, fp32 second moment v, 16-bit parameter copy).
 *
 * The pages name Adam but print no equation.  Reading: Adam with bias
 * correction (Kingma & Ba 2015, Algorithm 1) with decoupled weight decay
 * (Loshchilov & Hutter, AdamW), eps added after the square root of the
 * bias-corrected second moment.  Per element, each line one binary32 op
 * rounded to nearest even, in this order (scalars from zo_adam_scalars):
 *   p  = p * decay
 *   m  = beta1*m + (1-beta1)*g        (both products rounded before the sum)
 *   v  = beta2*v + (1-beta2)*(g*g)
 *   mh = m / bc1 ;  vh = v / bc2
 *   p  = p - lr * (mh / (sqrt(vh) + eps))
 *   out = bf16(p)
 * g is the averaged bf16 gradient; master, m, v are updated in place.
 */
void zo_adam(int64_t n, const uint16_t* g, float* master, float* m, float* v, uint16_t* p_out,
             double lr, double beta1, double beta2, double eps, double weight_decay, int64_t t) {
  float s[9];
  zo_adam_scalars(lr, beta1, beta2, eps, weight_decay, t, s);
  const float b1 = s[0], b2 = s[1], omb1 = s[2], omb2 = s[3], bc1 = s[4], bc2 = s[5];
  const float decay = s[6], lr_f = s[7], eps_f = s[8];
  for (int64_t i = 0; i < n; ++i) {
    const float gi = zo_bf16_to_f32(g[i]);
    float p = master[i];
    p = p * decay;
    float a = b1 * m[i];
    float b = omb1 * gi;
    const float mi = a + b;
    const float gg = gi * gi;
    a = b2 * v[i];
    b = omb2 * gg;
    const float vi = a + b;
    const float mh = mi / bc1;
    const float vh = vi / bc2;
    const float den = sqrtf(vh) + eps_f;
    const float ratio = mh / den;
    const float upd = lr_f * ratio;
    p = p - upd;
    master[i] = p;
    m[i] = mi;
    v[i] = vi;
    if (p_out) p_out[i] = zo_bf16_rne(p);
  }
}

/*
 * The same Adam update with the averaged gradient scaled first by a
 * global-norm clipping coefficient: g_used = fp32(g) * coef (one binary32
 * rounding) when coef < 1, g_used = fp32(g) otherwise (coef >= 1 means the
 * norm is within the limit and nothing is scaled).  Not on the pages: the
 * optional clipping of a mixed-precision step; see the oracle's clip_coef
 * for the coefficient.
 */
void zo_adam_coef(int64_t n, const uint16_t* g, float coef, float* master, float* m, float* v,
                  uint16_t* p_out, double lr, double beta1, double beta2, double eps,
                  double weight_decay, int64_t t) {
  float s[9];
  zo_adam_scalars(lr, beta1, beta2, eps, weight_decay, t, s);
  const float b1 = s[0], b2 = s[1], omb1 = s[2], omb2 = s[3], bc1 = s[4], bc2 = s[5];
  const float decay = s[6], lr_f = s[7], eps_f = s[8];
  for (int64_t i = 0; i < n; ++i) {
    float gi = zo_bf16_to_f32(g[i]);
    if (coef < 1.0f) gi = gi * coef;
    float p = master[i];
    p = p * decay;
    float a = b1 * m[i];
    float b = omb1 * gi;
    const float mi = a + b;
    const float gg = gi * gi;
    a = b2 * v[i];
    b = omb2 * gg;
    const float vi = a + b;
    const float mh = mi / bc1;
    const float vh = vi / bc2;
    const float den = sqrtf(vh) + eps_f;
    const float ratio = mh / den;
    const float upd = lr_f * ratio;
    p = p - upd;
    master[i] = p;
    m[i] = mi;
    v[i] = vi;
    if (p_out) p_out[i] = zo_bf16_rne(p);
  }
}

/* ----------------------------------------------- gradient norm / overflow ---- */

/* Sum of squares of the averaged bf16 gradient, in binary64, index order.
 * (Not on the pages: a norm / overflow report, never a skip or a clip.) */
double zo_sumsq(int64_t n, const uint16_t* g) {
  double s = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    const double x = (double)zo_bf16_to_f32(g[i]);
    s = s + x * x;
  }
  return s;
}

int64_t zo_count_nonfinite(int64_t n, const uint16_t* g) {
  int64_t c = 0;
  for (int64_t i = 0; i < n; ++i)
    if (!isfinite(zo_bf16_to_f32(g[i]))) ++c;
  return c;
}
