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

/* -------------------------------------------------------------- binary16 ---- */

/* IEEE-754 binary16 -> fp32 (exact): sign, 5-bit exponent (bias 15), 10-bit
 * fraction; exponent 0 holds zeros and subnormals (fraction x 2^-24), 31 holds
 * infinities and NaNs. */
float zo_f16_to_f32(uint16_t h) {
  const int sign = (h >> 15) & 1, e = (h >> 10) & 0x1F, f = h & 0x3FF;
  float mag;
  if (e == 0) mag = (float)ldexp((double)f, -24);
  else if (e == 31) mag = f ? NAN : INFINITY;
  else mag = (float)ldexp((double)(1024 + f), e - 25);
  return sign ? -mag : mag;
}

/*
 * fp32 -> binary16, round to nearest, ties to even (IEEE-754
 * roundTiesToEven with an 11-bit significand, exponent range -14..15,
 * subnormals spaced 2^-24): x / q with q the spacing of x's binade (2^(e-10),
 * at least 2^-24) is exact in binary64; it is rounded to an integer k with
 * ties to the even one, and k*q is encoded (k = 2048 carries into the next
 * binade, k = 1024 from the subnormal range is the smallest normal).
 * Magnitudes at or above 65520 (halfway past the largest finite 65504) round to
 * infinity.  NaN maps to a quiet NaN with the sign kept.
 */
uint16_t zo_f16_rne(float x) {
  const uint16_t sign = signbit(x) ? 0x8000u : 0u;
  if (isnan(x)) return (uint16_t)(sign | 0x7E00u);
  const double a = fabs((double)x);
  if (a >= 65520.0) return (uint16_t)(sign | 0x7C00u);
  if (a == 0.0) return sign;
  int e = (int)floor(log2(a));
  if (ldexp(1.0, e) > a) --e;           /* guard log2 rounding at binade edges */
  else if (ldexp(1.0, e + 1) <= a) ++e;
  if (e < -14) e = -14;                  /* subnormal spacing */
  const double n = ldexp(a, 10 - e);     /* a / q, exact */
  double k = floor(n);
  const double frac = n - k;
  if (frac > 0.5 || (frac == 0.5 && fmod(k, 2.0) != 0.0)) k += 1.0;
  int ki = (int)k;
  int be;                                /* biased exponent */
  if (ki >= 2048) {                      /* carried into the next binade */
    ki >>= 1;
    ++e;
  }
  if (ki < 1024) {                       /* subnormal (e == -14) */
    return (uint16_t)(sign | (uint16_t)ki);
  }
  be = e + 15;
  if (be >= 31) return (uint16_t)(sign | 0x7C00u);
  return (uint16_t)(sign | (uint16_t)(be << 10) | (uint16_t)(ki - 1024));
}

void zo_f16_rne_array(int64_t n, const float* x, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = zo_f16_rne(x[i]);
}

void zo_f16_to_f32_array(int64_t n, const uint16_t* h, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = zo_f16_to_f32(h[i]);
}

/* 16-bit storage formats of gradients and parameters. */
enum { ZO_BF16 = 0, ZO_F16 = 1 };

static float fmt_to_f32(int fmt, uint16_t h) { return fmt == ZO_F16 ? zo_f16_to_f32(h) : zo_bf16_to_f32(h); }
static uint16_t fmt_rne(int fmt, float x) { return fmt == ZO_F16 ? zo_f16_rne(x) : zo_bf16_rne(x); }

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
static float rank_sum(int fmt, int32_t n_ranks, const uint16_t* const* rank_grads, int64_t i) {
  float acc = 0.0f;
  for (int32_t r = 0; r < n_ranks; ++r) acc = acc + fmt_to_f32(fmt, rank_grads[r][i]);
  return acc;
}

/* The averaged gradient in either 16-bit format (zo_reduce_mean is this
 * function with ZO_BF16): the mean rounded once to the format.  Under a loss
 * scale the ranks' gradients are S times the true ones and the mean is
 * formed and rounded while still scaled, so that an overflow shows as Inf
 * (mixed-precision convention; the pages only name fp16 as a communication
 * type, [M] section 3.3). */
void zo_reduce_mean_fmt(int fmt, int32_t n_ranks, int64_t n, const uint16_t* const* rank_grads, uint16_t* out) {
  const float inv_n = (float)(1.0 / (double)n_ranks);
  for (int64_t i = 0; i < n; ++i) out[i] = fmt_rne(fmt, rank_sum(fmt, n_ranks, rank_grads, i) * inv_n);
}

void zo_reduce_mean(int32_t n_ranks, int64_t n, const uint16_t* const* rank_grads, uint16_t* out) {
  zo_reduce_mean_fmt(ZO_BF16, n_ranks, n, rank_grads, out);
}

/* Same sum in fp32 without the mean and the bf16 rounding, for the tests that
 * bound the accumulation error against the exact sum. */
void zo_rank_sum_f32(int32_t n_ranks, int64_t n, const uint16_t* const* rank_grads, float* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = rank_sum(ZO_BF16, n_ranks, rank_grads, i);
}

/* ----------------------------------------------------------------- Adam ---- */

/*
 * Host scalars of Adam step t (t >= 1), for the owner's update below ([T]
 * sections "ZeRO-1" to "ZeRO-3", part "3. 更新").  The hyper-parameters arrive as
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
 * fp32 first moment m, fp32 second moment v, 16-bit parameter copy).  This is
 * the oracle's only update loop; zo_adam and zo_adam_coef below call it.
 *
 * The pages name Adam but print no equation.  Reading: Adam with bias
 * correction (Kingma & Ba 2015, Algorithm 1) with decoupled weight decay
 * (Loshchilov & Hutter, AdamW), eps added after the square root of the
 * bias-corrected second moment.  Per element, each line one binary32 op
 * rounded to nearest even, in this order (scalars from zo_adam_scalars):
 *   g  = fp32(g16) [* inv_scale when inv_scale != 1] [* coef when coef < 1]
 *   p  = p * decay
 *   m  = beta1*m + (1-beta1)*g        (both products rounded before the sum)
 *   v  = beta2*v + (1-beta2)*(g*g)
 *   mh = m / bc1 ;  vh = v / bc2
 *   p  = p - lr * (mh / (sqrt(vh) + eps))
 *   out = 16-bit(p)
 * g16 is the averaged gradient in storage format `fmt`; master, m, v are
 * updated in place.  The two optional factors are the usual mixed-precision
 * conventions, not on the pages beyond their mention of fp16 as the
 * communication type: the ranks' gradients are S times the true ones under a
 * loss scale S (inv_scale = fp32(1/S)), and a global-norm clipping
 * coefficient scales the gradient when below 1 (see the oracle's clip_coef).
 */
void zo_adam_ex(int fmt, int64_t n, const uint16_t* g, float inv_scale, float coef, float* master, float* m,
                float* v, uint16_t* p_out, double lr, double beta1, double beta2, double eps,
                double weight_decay, int64_t t) {
  float s[9];
  zo_adam_scalars(lr, beta1, beta2, eps, weight_decay, t, s);
  const float b1 = s[0], b2 = s[1], omb1 = s[2], omb2 = s[3], bc1 = s[4], bc2 = s[5];
  const float decay = s[6], lr_f = s[7], eps_f = s[8];
  for (int64_t i = 0; i < n; ++i) {
    float gi = fmt_to_f32(fmt, g[i]);
    if (inv_scale != 1.0f) gi = gi * inv_scale;
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
    if (p_out) p_out[i] = fmt_rne(fmt, p);
  }
}

/* The bf16 update without a loss scale or a clipping coefficient. */
void zo_adam(int64_t n, const uint16_t* g, float* master, float* m, float* v, uint16_t* p_out,
             double lr, double beta1, double beta2, double eps, double weight_decay, int64_t t) {
  zo_adam_ex(ZO_BF16, n, g, 1.0f, 1.0f, master, m, v, p_out, lr, beta1, beta2, eps, weight_decay, t);
}

/* The bf16 update with the averaged gradient scaled first by a global-norm
 * clipping coefficient (when coef < 1; coef >= 1 scales nothing). */
void zo_adam_coef(int64_t n, const uint16_t* g, float coef, float* master, float* m, float* v,
                  uint16_t* p_out, double lr, double beta1, double beta2, double eps,
                  double weight_decay, int64_t t) {
  zo_adam_ex(ZO_BF16, n, g, 1.0f, coef, master, m, v, p_out, lr, beta1, beta2, eps, weight_decay, t);
}

/* zo_sumsq and zo_count_nonfinite below for either 16-bit format (not on the
 * pages: the norm and the overflow count of the optional clip and skip). */
double zo_sumsq_fmt(int fmt, int64_t n, const uint16_t* g) {
  double acc = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    const double x = (double)fmt_to_f32(fmt, g[i]);
    acc = acc + x * x;
  }
  return acc;
}

int64_t zo_count_nonfinite_fmt(int fmt, int64_t n, const uint16_t* g) {
  int64_t c = 0;
  for (int64_t i = 0; i < n; ++i)
    if (!isfinite(fmt_to_f32(fmt, g[i]))) ++c;
  return c;
}

/* ----------------------------------------------- gradient norm / overflow ---- */

/* Sum of squares of the averaged bf16 gradient, in binary64, index order.
 * (Not on the pages: the reported norm, which the optional global-norm clip
 * and the overflow skip of the step flows also use.) */
double zo_sumsq(int64_t n, const uint16_t* g) {
  double s = 0.0;
  for (int64_t i = 0; i < n; ++i) {
    const double x = (double)zo_bf16_to_f32(g[i]);
    s = s + x * x;
  }
  return s;
}

/* Number of infinite or NaN elements of the averaged bf16 gradient (not on
 * the pages: the overflow report and the optional skip's test). */
int64_t zo_count_nonfinite(int64_t n, const uint16_t* g) {
  int64_t c = 0;
  for (int64_t i = 0; i < n; ++i)
    if (!isfinite(zo_bf16_to_f32(g[i]))) ++c;
  return c;
}
