/*
 * msda_oracle.c -- plain fp64 CPU oracle for multi-scale deformable attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package smoke check and the
 * bench's CPU-baseline leg may load this.  It shares no code, header, table or
 * helper with the CUDA library; the two are built separately and neither
 * includes or links the other.
 *
 * Everything is a direct transcription of the defining sums, in double
 * precision, one output element at a time, with no blocking, fusion or
 * reordering.  Inputs arrive already widened to double (exactly: they were
 * stored as float32 or bfloat16).
 *
 * Sources (web pages on the operator, cited by page and section):
 *   [discosf]  discosf.com/news/5175395 -- tutorial.  §2.1 bilinear sampling is
 *              differentiable in the coordinates; §2.2 the multi-scale formula
 *              and "out-of-range sampling points are masked to zero".
 *   [cf-1]     cf-1.com/news/4799680 -- DETR to Deformable DETR.  §3.1 the
 *              formula with sum_l sum_k A = 1; §3.2 softmax over (levels x
 *              points), locations = reference + offsets / (W, H) with
 *              normalizer (spatial_shapes[:,1], spatial_shapes[:,0]); §3.3 the
 *              flattened multi-level value with spatial_shapes and
 *              level_start_index; §5.3 the grid_sample reduction
 *              (grid = 2*loc - 1, bilinear, zeros, align_corners=False).
 *   [csdn]     x-humanoid.csdn.net MSDA explainer -- §3 implementation notes
 *              1-3: normalized coordinates, align_corners=False (pixels are
 *              cell centres), softmax over all L*K points.
 *
 * Readings where the pages are silent:
 *   - pixel coordinate of a normalized location: x = loc_x * W - 0.5,
 *     y = loc_y * H - 0.5 (what grid_sample with align_corners=False does to
 *     grid = 2*loc - 1, [cf-1] §5.3, [csdn] §3 note 2);
 *   - a sample is taken only when -1 < x < W and -1 < y < H; otherwise it
 *     contributes nothing and has zero gradients; inside that range each of the
 *     four corners outside the map contributes zero ([discosf] §2.2);
 *   - the derivative at an integer coordinate is the one of the cell
 *     floor(x) (one-sided), which is what the definition with floor gives;
 *   - the backward pass is the exact derivative of the forward sum (the pages
 *     only state that it exists, [discosf] §2.1).
 *
 * Layouts (row-major, C order):
 *   value        [B, S, M, D]           S = sum_l H_l * W_l
 *   shapes       [L, 2]  (H, W)         int64
 *   start        [L]                    int64
 *   loc          [B, Q, M, L, K, 2]     (x, y) normalized
 *   attn         [B, Q, M, L, K]
 *   out          [B, Q, M, D]
 *   ref          [B, Q, 2]              (x, y) normalized
 *   off          [B, Q, M, L, K, 2]     level pixels
 *   logits       [B, Q, M, L*K]
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

typedef struct {
    int64_t B, S, Q, M, D, L, K;
} oracle_dims;

/* One bilinear sample: the four corners and their weights ([discosf] §2.1). */
typedef struct {
    int valid;           /* -1 < x < W and -1 < y < H */
    int64_t x0, y0;
    double fx, fy;
    int64_t cx[4], cy[4];
    int inb[4];          /* corner lies inside the H x W map */
    double w[4];
} bilinear;

static bilinear bilinear_at_pixel(double x, double y, int64_t H, int64_t W);

/* A normalized location: pixel coordinate x = lx * W - 0.5, y = ly * H - 0.5. */
static bilinear bilinear_setup(double lx, double ly, int64_t H, int64_t W)
{
    return bilinear_at_pixel(lx * (double)W - 0.5, ly * (double)H - 0.5, H, W);
}

/* A pixel coordinate (pixel centres at integers). */
static bilinear bilinear_at_pixel(double x, double y, int64_t H, int64_t W)
{
    bilinear s;
    memset(&s, 0, sizeof s);
    s.valid = (x > -1.0) && (x < (double)W) && (y > -1.0) && (y < (double)H);
    if (!s.valid)
        return s;
    double fx0 = floor(x), fy0 = floor(y);
    s.x0 = (int64_t)fx0;
    s.y0 = (int64_t)fy0;
    s.fx = x - fx0;
    s.fy = y - fy0;
    /* corner order: (y0,x0) (y0,x0+1) (y0+1,x0) (y0+1,x0+1) */
    for (int c = 0; c < 4; ++c) {
        s.cx[c] = s.x0 + (c & 1);
        s.cy[c] = s.y0 + (c >> 1);
        s.inb[c] = s.cx[c] >= 0 && s.cx[c] < W && s.cy[c] >= 0 && s.cy[c] < H;
    }
    s.w[0] = (1.0 - s.fy) * (1.0 - s.fx);
    s.w[1] = (1.0 - s.fy) * s.fx;
    s.w[2] = s.fy * (1.0 - s.fx);
    s.w[3] = s.fy * s.fx;
    return s;
}

static int64_t value_row(const oracle_dims *d, int64_t b, int64_t start_l, int64_t W,
                         int64_t cy, int64_t cx, int64_t m)
{
    int64_t key = start_l + cy * W + cx;
    return ((b * d->S + key) * d->M + m) * d->D;
}

/*
 * Forward: out[b,q,m,:] = sum_l sum_k A[b,q,m,l,k] * x^l_m(loc[b,q,m,l,k])
 * ([discosf] §2.2, [cf-1] §3.1; the W_m / W'_m projections are outside the
 * operator, as in the argument list of [cf-1] §5.3).
 */
void msda_oracle_forward(const oracle_dims *d, const double *value, const int64_t *shapes,
                         const int64_t *start, const double *loc, const double *attn,
                         double *out)
{
    for (int64_t b = 0; b < d->B; ++b)
    for (int64_t q = 0; q < d->Q; ++q)
    for (int64_t m = 0; m < d->M; ++m) {
        double *o = out + ((b * d->Q + q) * d->M + m) * d->D;
        for (int64_t c = 0; c < d->D; ++c)
            o[c] = 0.0;
        for (int64_t l = 0; l < d->L; ++l) {
            int64_t H = shapes[2 * l], W = shapes[2 * l + 1];
            for (int64_t k = 0; k < d->K; ++k) {
                int64_t p = (((b * d->Q + q) * d->M + m) * d->L + l) * d->K + k;
                bilinear s = bilinear_setup(loc[2 * p], loc[2 * p + 1], H, W);
                if (!s.valid)
                    continue;
                double a = attn[p];
                for (int c = 0; c < 4; ++c) {
                    if (!s.inb[c])
                        continue;
                    const double *v = value + value_row(d, b, start[l], W, s.cy[c], s.cx[c], m);
                    for (int64_t ch = 0; ch < d->D; ++ch)
                        o[ch] += a * s.w[c] * v[ch];
                }
            }
        }
    }
}

/*
 * Backward: exact derivative of the forward sum.  With s = sum_c w_c v_c the
 * bilinear sample and g = grad_out[b,q,m,:]:
 *   grad_attn              = <g, s>
 *   ds/dx                  = (1-fy)(v01 - v00) + fy (v11 - v10)
 *   ds/dy                  = (1-fx)(v10 - v00) + fx (v11 - v01)
 *   grad_loc_x             = W * A * <g, ds/dx>      (x = loc_x * W - 0.5)
 *   grad_loc_y             = H * A * <g, ds/dy>
 *   grad_value[corner c]  += A * w_c * g              (in-map corners only)
 * Out-of-map corners enter ds/dx and ds/dy as v = 0.  grad_value is
 * overwritten (zeroed first).
 */
void msda_oracle_backward(const oracle_dims *d, const double *value, const int64_t *shapes,
                          const int64_t *start, const double *loc, const double *attn,
                          const double *grad_out, double *grad_value, double *grad_loc,
                          double *grad_attn)
{
    int64_t nval = d->B * d->S * d->M * d->D;
    for (int64_t i = 0; i < nval; ++i)
        grad_value[i] = 0.0;
    for (int64_t b = 0; b < d->B; ++b)
    for (int64_t q = 0; q < d->Q; ++q)
    for (int64_t m = 0; m < d->M; ++m) {
        const double *g = grad_out + ((b * d->Q + q) * d->M + m) * d->D;
        for (int64_t l = 0; l < d->L; ++l) {
            int64_t H = shapes[2 * l], W = shapes[2 * l + 1];
            for (int64_t k = 0; k < d->K; ++k) {
                int64_t p = (((b * d->Q + q) * d->M + m) * d->L + l) * d->K + k;
                bilinear s = bilinear_setup(loc[2 * p], loc[2 * p + 1], H, W);
                grad_attn[p] = 0.0;
                grad_loc[2 * p] = 0.0;
                grad_loc[2 * p + 1] = 0.0;
                if (!s.valid)
                    continue;
                double a = attn[p];
                const double *v[4];
                for (int c = 0; c < 4; ++c)
                    v[c] = s.inb[c] ? value + value_row(d, b, start[l], W, s.cy[c], s.cx[c], m) : 0;
                double ga = 0.0, gx = 0.0, gy = 0.0;
                for (int64_t ch = 0; ch < d->D; ++ch) {
                    double v00 = v[0] ? v[0][ch] : 0.0;
                    double v01 = v[1] ? v[1][ch] : 0.0;
                    double v10 = v[2] ? v[2][ch] : 0.0;
                    double v11 = v[3] ? v[3][ch] : 0.0;
                    double samp = s.w[0] * v00 + s.w[1] * v01 + s.w[2] * v10 + s.w[3] * v11;
                    double dx = (1.0 - s.fy) * (v01 - v00) + s.fy * (v11 - v10);
                    double dy = (1.0 - s.fx) * (v10 - v00) + s.fx * (v11 - v01);
                    ga += g[ch] * samp;
                    gx += g[ch] * dx;
                    gy += g[ch] * dy;
                }
                grad_attn[p] = ga;
                grad_loc[2 * p] = (double)W * a * gx;
                grad_loc[2 * p + 1] = (double)H * a * gy;
                for (int c = 0; c < 4; ++c) {
                    if (!s.inb[c])
                        continue;
                    double *gv = grad_value + value_row(d, b, start[l], W, s.cy[c], s.cx[c], m);
                    for (int64_t ch = 0; ch < d->D; ++ch)
                        gv[ch] += a * s.w[c] * g[ch];
                }
            }
        }
    }
}

/*
 * Sampling locations from reference points and raw offsets ([cf-1] §3.2):
 *   loc = ref + off / (W_l, H_l)
 * The offsets are raw linear-layer outputs in level-l pixels (no sigmoid);
 * one reference point per query is used for every level (the level map phi_l
 * of a normalized point is the identity in normalized units, [discosf] §2.2).
 */
void msda_oracle_sampling_locations(const oracle_dims *d, const int64_t *shapes,
                                    const double *ref, const double *off, double *loc)
{
    for (int64_t b = 0; b < d->B; ++b)
    for (int64_t q = 0; q < d->Q; ++q)
    for (int64_t m = 0; m < d->M; ++m)
    for (int64_t l = 0; l < d->L; ++l)
    for (int64_t k = 0; k < d->K; ++k) {
        int64_t p = (((b * d->Q + q) * d->M + m) * d->L + l) * d->K + k;
        const double *r = ref + 2 * (b * d->Q + q);
        loc[2 * p] = r[0] + off[2 * p] / (double)shapes[2 * l + 1];
        loc[2 * p + 1] = r[1] + off[2 * p + 1] / (double)shapes[2 * l];
    }
}

/*
 * Attention weights: softmax over the L*K logits of each (b, q, m)
 * ([cf-1] §3.1-3.2, [csdn] §3 note 3).  The maximum is subtracted before
 * exponentiation; exp is the C library's double exp.
 */
void msda_oracle_softmax(const oracle_dims *d, const double *logits, double *attn)
{
    int64_t n = d->L * d->K;
    for (int64_t r = 0; r < d->B * d->Q * d->M; ++r) {
        const double *z = logits + r * n;
        double *a = attn + r * n;
        double mx = z[0];
        for (int64_t j = 1; j < n; ++j)
            if (z[j] > mx)
                mx = z[j];
        double sum = 0.0;
        for (int64_t j = 0; j < n; ++j) {
            a[j] = exp(z[j] - mx);
            sum += a[j];
        }
        for (int64_t j = 0; j < n; ++j)
            a[j] /= sum;
    }
}

/*
 * Chain rule from the core gradients to the fused inputs:
 *   grad_off_x = grad_loc_x / W_l, grad_off_y = grad_loc_y / H_l
 *   grad_ref[b,q,:] = sum over (m, l, k) of grad_loc        (ref is shared)
 *   grad_logit_j = A_j * (gA_j - sum_i A_i gA_i)            (softmax Jacobian)
 * grad_ref may be NULL.
 */
void msda_oracle_fused_chain(const oracle_dims *d, const int64_t *shapes, const double *attn,
                             const double *grad_loc, const double *grad_attn,
                             double *grad_off, double *grad_ref, double *grad_logits)
{
    int64_t n = d->L * d->K;
    if (grad_ref)
        for (int64_t i = 0; i < d->B * d->Q * 2; ++i)
            grad_ref[i] = 0.0;
    for (int64_t b = 0; b < d->B; ++b)
    for (int64_t q = 0; q < d->Q; ++q)
    for (int64_t m = 0; m < d->M; ++m) {
        int64_t r = (b * d->Q + q) * d->M + m;
        double dot = 0.0;
        for (int64_t j = 0; j < n; ++j)
            dot += attn[r * n + j] * grad_attn[r * n + j];
        for (int64_t j = 0; j < n; ++j)
            grad_logits[r * n + j] = attn[r * n + j] * (grad_attn[r * n + j] - dot);
        for (int64_t l = 0; l < d->L; ++l)
        for (int64_t k = 0; k < d->K; ++k) {
            int64_t p = r * n + l * d->K + k;
            grad_off[2 * p] = grad_loc[2 * p] / (double)shapes[2 * l + 1];
            grad_off[2 * p + 1] = grad_loc[2 * p + 1] / (double)shapes[2 * l];
            if (grad_ref) {
                grad_ref[2 * (b * d->Q + q)] += grad_loc[2 * p];
                grad_ref[2 * (b * d->Q + q) + 1] += grad_loc[2 * p + 1];
            }
        }
    }
}

/*
 * INT8 value storage ([csdn] §4, "quantization and low-precision inference":
 * store the operator's data as INT8 to cut memory traffic; the page gives no
 * scheme).  Reading taken (listed with the others): symmetric quantisation
 * with one scale per (batch, head), in float32 as a quantising kernel would
 * compute it:
 *   amax  = max over s, d of |value[b, s, m, d]|
 *   scale = amax / 127, or 1 when amax == 0
 *   q     = value / scale rounded half to even, clipped to [-127, 127]
 * The operator then samples the dequantized tensor q * scale (exact in
 * double), so the core sums above are unchanged.  value: [B, S, M, D] float32
 * (finite); q: [B, S, M, D]; scale: [B, M].
 */
void msda_oracle_quantize_value_s8(const oracle_dims *d, const float *value, int8_t *q, float *scale)
{
    for (int64_t b = 0; b < d->B; ++b)
        for (int64_t m = 0; m < d->M; ++m) {
            float amax = 0.0f;
            for (int64_t s = 0; s < d->S; ++s)
                for (int64_t c = 0; c < d->D; ++c) {
                    const float a = fabsf(value[((b * d->S + s) * d->M + m) * d->D + c]);
                    if (a > amax)
                        amax = a;
                }
            const float sc = amax > 0.0f ? amax / 127.0f : 1.0f;
            scale[b * d->M + m] = sc;
            for (int64_t s = 0; s < d->S; ++s)
                for (int64_t c = 0; c < d->D; ++c) {
                    const int64_t i = ((b * d->S + s) * d->M + m) * d->D + c;
                    float r = nearbyintf(value[i] / sc); /* default mode: half to even */
                    if (r > 127.0f)
                        r = 127.0f;
                    if (r < -127.0f)
                        r = -127.0f;
                    q[i] = (int8_t)r;
                }
        }
}

/*
 * FP8 value storage, the other low-precision format of the same note
 * ([csdn] §4).  Format: the E4M3 encoding of the OCP 8-bit floating-point
 * specification (v1.0): bit 7 the sign, bits 6..3 a biased exponent (bias 7),
 * bits 2..0 a mantissa; exponent field e > 0 encodes (1 + m/8) * 2^(e - 7),
 * e = 0 encodes the subnormals (m/8) * 2^-6; S.1111.111 is NaN and there is no
 * infinity, so the largest finite magnitude is S.1111.110 = 1.75 * 2^8 = 448.
 * Reading taken (listed with the others): the INT8 scheme above with 448 in
 * place of 127 -- scale = amax / 448 (1 when amax == 0), x = value / scale in
 * float32, the code the E4M3 value nearest to x (ties to the even mantissa),
 * magnitudes above 448 clipped to 448 ("satfinite"); the sign of x is kept
 * when x rounds to zero.
 */

/* The E4M3 code of the float x (finite), from the definition above: the
 * representable magnitudes around |x| are multiples of the quantum 2^(E-3)
 * of |x|'s binade E (E >= -6; the subnormals share the quantum 2^-9). */
unsigned char msda_oracle_e4m3_encode(float x)
{
    const unsigned char sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (a >= 448.0)
        return (unsigned char)(sign | 0x7E);
    int E = -6;                               /* binade: 2^E <= a < 2^(E+1) */
    if (a >= ldexp(1.0, -6)) {
        (void)frexp(a, &E);                   /* a = f * 2^E, f in [0.5, 1) */
        E -= 1;
    }
    const double quantum = ldexp(1.0, E - 3);
    double r = nearbyint(a / quantum);        /* a / quantum is exact; half to even */
    /* r counts quanta of binade E: subnormals 0..8, normals 8..16 (16 carries
     * into the next binade, whose mantissa is then 0) */
    if (a < ldexp(1.0, -6)) {                 /* subnormal range */
        if (r >= 8.0)
            return (unsigned char)(sign | (1 << 3));      /* rounds up to 2^-6 */
        return (unsigned char)(sign | (unsigned)r);
    }
    if (r >= 16.0) {
        E += 1;
        r = 8.0;
    }
    if (E > 8 || (E == 8 && r > 14.0))        /* beyond 448: clip */
        return (unsigned char)(sign | 0x7E);
    return (unsigned char)(sign | ((unsigned)(E + 7) << 3) | (unsigned)(r - 8.0));
}

/* The value of an E4M3 code (NaN codes return NaN). */
double msda_oracle_e4m3_decode(unsigned char c)
{
    const int e = (c >> 3) & 15, m = c & 7;
    const double sgn = (c & 0x80) ? -1.0 : 1.0;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        return sgn * ldexp((double)m, -9);
    return sgn * ldexp(8.0 + m, e - 10);
}

void msda_oracle_quantize_value_e4m3(const oracle_dims *d, const float *value, unsigned char *q,
                                     float *scale)
{
    for (int64_t b = 0; b < d->B; ++b)
        for (int64_t m = 0; m < d->M; ++m) {
            float amax = 0.0f;
            for (int64_t s = 0; s < d->S; ++s)
                for (int64_t c = 0; c < d->D; ++c) {
                    const float a = fabsf(value[((b * d->S + s) * d->M + m) * d->D + c]);
                    if (a > amax)
                        amax = a;
                }
            const float sc = amax > 0.0f ? amax / 448.0f : 1.0f;
            scale[b * d->M + m] = sc;
            for (int64_t s = 0; s < d->S; ++s)
                for (int64_t c = 0; c < d->D; ++c) {
                    const int64_t i = ((b * d->S + s) * d->M + m) * d->D + c;
                    q[i] = msda_oracle_e4m3_encode(value[i] / sc);
                }
        }
}

/*
 * DCNv3 core ([discosf] §4.2): for output pixel p0 = (i, j) of image n and
 * group g,
 *   y[n,i,j,g,:] = sum_k m[n,i,j,g,k] * x_g(p0 + p_k + dp[n,i,j,g,k])
 * where x_g bilinearly samples group g of the channels-last input
 * x[N, H, W, G, C] at a pixel coordinate (pixel centres at integers, corners
 * outside the map contribute zero, a sample is taken only when -1 < px < W
 * and -1 < py < H).  The grid p0 + p_k is the convolution's: point k = r*kw + c
 * of a kh x kw kernel sits at
 *   px = j*stride_w - pad_w + c*dil_w,  py = i*stride_h - pad_h + r*dil_h,
 * and the offset dp = (dx, dy) is added in pixels.  The shared projection w_g
 * of the formula is a linear layer outside the core, like the attention's
 * projections.  Readings (listed with the others): the page gives the
 * formula only; the conv grid, the pixel-centre convention, (x, y) offset
 * order and taking m as given (no normalisation inside the core) are the
 * plainest completions.
 * Layouts: x [N,H,W,G,C]; offset [N,Ho,Wo,G,K,2]; mask [N,Ho,Wo,G,K];
 * y [N,Ho,Wo,G,C]; K = kh*kw.
 */
typedef struct {
    int64_t N, H, W, G, C, Ho, Wo, kh, kw, stride_h, stride_w, pad_h, pad_w, dil_h, dil_w;
} dcn_dims;

static bilinear dcn_sample(const dcn_dims *d, int64_t i, int64_t j, int64_t k, const double *dp)
{
    const int64_t r = k / d->kw, c = k % d->kw;
    const double px = (double)(j * d->stride_w - d->pad_w + c * d->dil_w) + dp[0];
    const double py = (double)(i * d->stride_h - d->pad_h + r * d->dil_h) + dp[1];
    return bilinear_at_pixel(px, py, d->H, d->W);
}

static int64_t dcn_row(const dcn_dims *d, int64_t n, int64_t cy, int64_t cx, int64_t g)
{
    return (((n * d->H + cy) * d->W + cx) * d->G + g) * d->C;
}

void msda_oracle_dcn_forward(const dcn_dims *d, const double *x, const double *offset,
                             const double *mask, double *y)
{
    const int64_t K = d->kh * d->kw;
    for (int64_t n = 0; n < d->N; ++n)
    for (int64_t i = 0; i < d->Ho; ++i)
    for (int64_t j = 0; j < d->Wo; ++j)
    for (int64_t g = 0; g < d->G; ++g) {
        const int64_t row = ((n * d->Ho + i) * d->Wo + j) * d->G + g;
        double *o = y + row * d->C;
        for (int64_t ch = 0; ch < d->C; ++ch)
            o[ch] = 0.0;
        for (int64_t k = 0; k < K; ++k) {
            const int64_t p = row * K + k;
            bilinear s = dcn_sample(d, i, j, k, offset + 2 * p);
            if (!s.valid)
                continue;
            for (int c = 0; c < 4; ++c) {
                if (!s.inb[c])
                    continue;
                const double *v = x + dcn_row(d, n, s.cy[c], s.cx[c], g);
                for (int64_t ch = 0; ch < d->C; ++ch)
                    o[ch] += mask[p] * s.w[c] * v[ch];
            }
        }
    }
}

/*
 * DCNv3 core backward: exact derivative of the forward sum.  With s the
 * bilinear sample and g = grad_y[n,i,j,g,:]:
 *   grad_mask      = <g, s>
 *   grad_offset_x  = m * <g, ds/dpx>,  grad_offset_y = m * <g, ds/dpy>
 *                    (the offsets are in pixels: no scale factor)
 *   grad_x[corner c] += m * w_c * g   (in-map corners; grad_x zeroed first)
 */
void msda_oracle_dcn_backward(const dcn_dims *d, const double *x, const double *offset,
                              const double *mask, const double *grad_y, double *grad_x,
                              double *grad_offset, double *grad_mask)
{
    const int64_t K = d->kh * d->kw;
    const int64_t nx = d->N * d->H * d->W * d->G * d->C;
    for (int64_t t = 0; t < nx; ++t)
        grad_x[t] = 0.0;
    for (int64_t n = 0; n < d->N; ++n)
    for (int64_t i = 0; i < d->Ho; ++i)
    for (int64_t j = 0; j < d->Wo; ++j)
    for (int64_t g = 0; g < d->G; ++g) {
        const int64_t row = ((n * d->Ho + i) * d->Wo + j) * d->G + g;
        const double *gy = grad_y + row * d->C;
        for (int64_t k = 0; k < K; ++k) {
            const int64_t p = row * K + k;
            bilinear s = dcn_sample(d, i, j, k, offset + 2 * p);
            grad_mask[p] = 0.0;
            grad_offset[2 * p] = 0.0;
            grad_offset[2 * p + 1] = 0.0;
            if (!s.valid)
                continue;
            const double *v[4];
            for (int c = 0; c < 4; ++c)
                v[c] = s.inb[c] ? x + dcn_row(d, n, s.cy[c], s.cx[c], g) : 0;
            double gm = 0.0, gx = 0.0, gyy = 0.0;
            for (int64_t ch = 0; ch < d->C; ++ch) {
                const double v00 = v[0] ? v[0][ch] : 0.0, v01 = v[1] ? v[1][ch] : 0.0;
                const double v10 = v[2] ? v[2][ch] : 0.0, v11 = v[3] ? v[3][ch] : 0.0;
                const double samp = s.w[0] * v00 + s.w[1] * v01 + s.w[2] * v10 + s.w[3] * v11;
                const double dx = (1.0 - s.fy) * (v01 - v00) + s.fy * (v11 - v10);
                const double dy = (1.0 - s.fx) * (v10 - v00) + s.fx * (v11 - v01);
                gm += gy[ch] * samp;
                gx += gy[ch] * dx;
                gyy += gy[ch] * dy;
            }
            grad_mask[p] = gm;
            grad_offset[2 * p] = mask[p] * gx;
            grad_offset[2 * p + 1] = mask[p] * gyy;
            for (int c = 0; c < 4; ++c) {
                if (!s.inb[c])
                    continue;
                double *gxr = grad_x + dcn_row(d, n, s.cy[c], s.cx[c], g);
                for (int64_t ch = 0; ch < d->C; ++ch)
                    gxr[ch] += mask[p] * s.w[c] * gy[ch];
            }
        }
    }
}

/*
 * Dense layer of the module around the operator: the value projection W'_m
 * and the output projection W_m of the formula ([discosf] §2.2, §3.1) and the
 * query head that predicts the sampling offsets and attention logits
 * ([cf-1] §3.2; [discosf] §3.1).  nn.Linear's convention:
 *   y[r, n] = sum_k x[r, k] * w[n, k] + b[n]      (b may be NULL)
 * x [rows, K], w [N, K], y [rows, N].
 */
void msda_oracle_linear(int64_t rows, int64_t K, int64_t N, const double *x, const double *w,
                        const double *b, double *y)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t n = 0; n < N; ++n) {
            double s = b ? b[n] : 0.0;
            for (int64_t k = 0; k < K; ++k)
                s += x[r * K + k] * w[n * K + k];
            y[r * N + n] = s;
        }
}

/*
 * Its exact derivative for an upstream gradient gy [rows, N]:
 *   gx[r, k] = sum_n gy[r, n] * w[n, k]
 *   gw[n, k] = sum_r gy[r, n] * x[r, k]
 *   gb[n]    = sum_r gy[r, n]
 */
void msda_oracle_linear_backward(int64_t rows, int64_t K, int64_t N, const double *x, const double *w,
                                 const double *gy, double *gx, double *gw, double *gb)
{
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t n = 0; n < N; ++n)
                s += gy[r * N + n] * w[n * K + k];
            gx[r * K + k] = s;
        }
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            double s = 0.0;
            for (int64_t r = 0; r < rows; ++r)
                s += gy[r * N + n] * x[r * K + k];
            gw[n * K + k] = s;
        }
        double s = 0.0;
        for (int64_t r = 0; r < rows; ++r)
            s += gy[r * N + n];
        gb[n] = s;
    }
}
