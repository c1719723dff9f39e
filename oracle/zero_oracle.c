/*
 * CPU oracle for the ZeRO partitioned mixed-precision Adam step -- TEST
 * INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file; only the tests, the smoke check and the bench's CPU-baseline leg
 * use it.  It shares no code with the CUDA library.
 *
 * Plain scalar C99, one element at a time, every floating-point operation a
 * separate IEEE-754 binary32 operation rounded to nearest-even.  It must be
 * compiled with -ffp-contract=off and without -ffast-math so that no
 * multiply-add is fused and no operation is reordered.
 *
 * Sources (three web pages about ZeRO, arXiv 1910.02054):
 *  - "ZeRO" concept page (papers.lqhl.me), section "为什么需要它" (why it is
 *    needed): mixed-precision Adam keeps low-precision parameters, an fp32
 *    master weight, the first moment and the second moment.
 *  - same page, table "三个阶段" (three stages), ZeRO-2 row: gradients are
 *    reduce-scattered so that each rank keeps the part it is responsible for.
 *  - mind-map page "ZeRO 真正在做什么：长期分开存，计算时临时拼齐", glossary
 *    entry "reduce-scatter": results of several GPUs are combined, then split
 *    so that each card keeps only its own part.
 *  The pages name Adam but print no formula; the per-element update below is
 *  textbook Adam (Kingma & Ba): bias correction on, epsilon outside the
 *  square root, no weight decay, written as
 *     m = b1*m + (1-b1)*g ;  v = b2*v + ((1-b2)*g)*g
 *     w = w - (lr/(1-b1^t)) * ( m / (sqrt(v)/sqrt(1-b2^t) + eps) )
 *  where the division by sqrt(1-b2^t) is taken as a multiplication by the
 *  host-precomputed 1/sqrt(1-b2^t).  Two optional extensions: decoupled
 *  weight decay (AdamW, Loshchilov & Hutter), w is first multiplied by
 *  (1 - lr*wd); and a global-norm clip coefficient c <= 1 applied to the
 *  gradient, g = (g_sum*s)*c.  With wd = 0 and c = 1 both multiplications are
 *  exact (by 1), so the plain Adam result is unchanged bit for bit.  The
 *  hyperparameters come in double, as
 *  optimizer settings usually do; b1, b2, eps and the gradient scale are
 *  used rounded to float, and 1-b1, 1-b2 are formed in double before their
 *  own rounding.  The pages do not fix the summation order
 *  of the reduction; the reading used here is the sequential sum over ranks
 *  r = 0, 1, ..., Nd-1 starting from rank 0's value.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

/* bf16 -> fp32 is exact: the bf16 bits are the top 16 bits of the fp32. */
static float bf16_bits_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* fp32 -> bf16, round to nearest, ties to even, on the bit pattern.
 * NaN keeps its sign and its top payload bits and is made quiet. */
uint16_t oracle_bf16_rne(float x)
{
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u)          /* NaN */
        return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;                 /* ties go to even */
    uint32_t rounded = u + 0x7fffu + lsb;          /* no overflow past inf */
    return (uint16_t)(rounded >> 16);
}

float oracle_bf16_to_float(uint16_t b) { return bf16_bits_to_float(b); }

/* Vector forms of the two conversions above (tests call these on big
 * samples of bit patterns). */
void oracle_bf16_rne_array(const float *x, uint16_t *out, uint64_t n)
{
    for (uint64_t i = 0; i < n; ++i) out[i] = oracle_bf16_rne(x[i]);
}

/* Host scalars of one Adam step t >= 1.  The hyperparameters are given in
 * double; every constant the per-element update uses is computed in double
 * and rounded once to float:
 *   sc[0] grad_scale   sc[1] b1        sc[2] b2        sc[3] eps
 *   sc[4] 1-b1         sc[5] 1-b2      sc[6] lr/(1-b1^t)
 *   sc[7] 1/sqrt(1-b2^t)               sc[8] 1-lr*wd (AdamW decay)
 * b1^t and b2^t are C99 pow() in double. */
void oracle_adam_scalars(double lr, double beta1, double beta2, double eps,
                         double grad_scale, double weight_decay, uint64_t t,
                         float sc[9])
{
    double bc1 = 1.0 - pow(beta1, (double)t);
    double bc2 = 1.0 - pow(beta2, (double)t);
    sc[0] = (float)grad_scale;
    sc[1] = (float)beta1;
    sc[2] = (float)beta2;
    sc[3] = (float)eps;
    sc[4] = (float)(1.0 - beta1);
    sc[5] = (float)(1.0 - beta2);
    sc[6] = (float)(lr / bc1);
    sc[7] = (float)(1.0 / sqrt(bc2));
    sc[8] = (float)(1.0 - lr * weight_decay);
}

/* The reduce step for one element: the fp32 sum of the Nd ranks' bf16
 * gradients, in rank order, starting from rank 0's value (so that the sign of
 * an all-zero sum is that of rank 0's zero). */
static float reduce_in_rank_order(const uint16_t *grads, uint64_t rank_stride,
                                  uint32_t nd, uint64_t e)
{
    float s = bf16_bits_to_float(grads[e]);
    for (uint32_t r = 1; r < nd; ++r) {
        float x = bf16_bits_to_float(grads[(uint64_t)r * rank_stride + e]);
        s = s + x;
    }
    return s;
}

/* One Adam update of one element, exactly in the order stated above. */
static void adam_element(float g_sum, const float sc[9], float clip_coef,
                         float *w, float *m, float *v)
{
    const float grad_scale = sc[0], beta1 = sc[1], beta2 = sc[2], eps = sc[3];
    const float omb1 = sc[4], omb2 = sc[5], step = sc[6], ibc2 = sc[7];
    const float decay = sc[8];
    float g_scaled = g_sum * grad_scale;
    float g = g_scaled * clip_coef;

    float m_old = beta1 * (*m);
    float m_new_part = omb1 * g;
    float m_new = m_old + m_new_part;

    float v_old = beta2 * (*v);
    float v_g = omb2 * g;
    float v_new_part = v_g * g;
    float v_new = v_old + v_new_part;

    float root = sqrtf(v_new);
    float root_hat = root * ibc2;
    float denom = root_hat + eps;
    float ratio = m_new / denom;
    float delta = step * ratio;
    float w_decayed = (*w) * decay;
    float w_new = w_decayed - delta;

    *m = m_new;
    *v = v_new;
    *w = w_new;
}

/*
 * The elementwise core used by every oracle step driver: for n elements laid
 * out contiguously (element e of rank r's gradient at grads[r*rank_stride+e]),
 *   reduce in rank order -> optional reduced_out[e]
 *   -> norm_sq += (double)g_sum^2, nonfinite += !isfinite(g_sum)
 *   -> Adam (with optional AdamW decay and clip coefficient) on w[e], m[e],
 *   v[e] -> p_out[e] = bf16(w[e]).
 * reduced_out, p_out, norm_sq and nonfinite may be NULL.
 */
void oracle_update(uint64_t n, uint32_t nd, const uint16_t *grads,
                   uint64_t rank_stride, float *w, float *m, float *v,
                   uint16_t *p_out, float *reduced_out, double grad_scale,
                   double lr, double beta1, double beta2, double eps,
                   double weight_decay, float clip_coef, uint64_t t,
                   double *norm_sq, int64_t *nonfinite)
{
    float sc[9];
    oracle_adam_scalars(lr, beta1, beta2, eps, grad_scale, weight_decay, t, sc);
    double acc = 0.0;
    int64_t bad = 0;
    for (uint64_t e = 0; e < n; ++e) {
        float g_sum = reduce_in_rank_order(grads, rank_stride, nd, e);
        if (reduced_out) reduced_out[e] = g_sum;
        acc += (double)g_sum * (double)g_sum;
        if (!isfinite(g_sum)) ++bad;
        adam_element(g_sum, sc, clip_coef, &w[e], &m[e], &v[e]);
        if (p_out) p_out[e] = oracle_bf16_rne(w[e]);
    }
    if (norm_sq) *norm_sq += acc;
    if (nonfinite) *nonfinite += bad;
}

/* Only the reduce step, for tests that pin the summation on its own. */
void oracle_reduce(uint64_t n, uint32_t nd, const uint16_t *grads,
                   uint64_t rank_stride, float *out)
{
    for (uint64_t e = 0; e < n; ++e)
        out[e] = reduce_in_rank_order(grads, rank_stride, nd, e);
}
