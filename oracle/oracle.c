/*
 * oracle.c -- plain, slow, fp64 CPU oracle for the generalized-causal GQA
 * self-attention with the generalized 2D RoPE (HunyuanImage-3.0).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this file's library.  It shares no
 * code, header, table or constant with the CUDA path, and it never reads a
 * value produced by the CUDA path.
 *
 * Sources (page title, section / API item):
 *   - "HunyuanImage-3.0" model-coverage page, Cache Contract: the sequence is
 *     prefix (ending in <timestep>) + <img> * (h*w) + suffix, right-padded.
 *   - nemo_automodel ... hunyuan_image3.model, build_joint_attention_mask:
 *     boolean [batch,1,seq,seq] mask indexed [b,1,query,key]: causal text,
 *     bidirectional image span, padded keys masked out.
 *   - HunyuanImage 3.0 Technical Report summary, 3.1.2 Generalized Causal
 *     Attention and 3.1.3 Position Embedding.
 *   - Paper review (xllm-io), 3.3 generalized causal attention and 3.4
 *     generalized 2D RoPE: 1D RoPE [cos n t0, cos n t1, ..., sin n t0, ...];
 *     2D [cos x t0, cos y t1, ..., sin x t0, sin y t1, ...]; text on the
 *     diagonal x = y = n; image positions reshaped to h x w between the text
 *     segments; exact reduction to 1D RoPE with no image.
 *   - nemo_automodel ... hunyuan_image3.layers, HunyuanImage3Attention:
 *     fused KV-head-grouped QKV (query head h uses kv head h / q_per_kv);
 *     cos/sin tables are fp32 [batch, seq, head_dim].
 *   - ... layers, UNetDown.forward: image tokens in row-major (height, width)
 *     order.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *   - padded query rows (q >= L) are ordinary rows that see keys [0, L-1];
 *   - a row with no visible key (only when L == 0) has O = 0, LSE = -inf and
 *     zero gradients;
 *   - theta_j = base^(-2j/D), j < D/2; channel pair (j, j + D/2) is rotated by
 *     angle_j (half-split layout);
 *   - image token i (row r = i / w, column c = i % w) sits at x = I0 + c,
 *     y = I0 + r; even j use x, odd j use y; every other token (text, suffix,
 *     padding) sits at x = y = n, its sequence index;
 *   - scores are scale * <R q, R k>, with scale passed in (1/sqrt(D));
 *   - optional per-head QK RMSNorm (HunyuanImage3Attention: RoPE is applied
 *     before the per-head QK RMSNorm; HunyuanRMSNorm normalizes over the
 *     last axis with eps, default 1e-5, and multiplies by its weight): with
 *     weights wq, wk the scores use y = w * x / sqrt(mean(x^2) + eps) of the
 *     rotated rows x = R q, R k.  In fp64 here; the dtype casts of the
 *     reference layer are rounding, covered by the parity tolerances.
 *
 * Parity pins: every function here is pinned by the CPU tests (hand-written
 * masks, closed-form pair counts, the 1D-RoPE library routine, relative
 * position invariance, a library attention routine, finite differences).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------------ */
/* Sample geometry                                                          */
/* ------------------------------------------------------------------------ */

/* One sample: text and images in order, then suffix text.  Image i spans
 * [I0_i, I1_i) (I1_i = I0_i + h_i * w_i, row-major, width w_i); L is the
 * sample's length; padding is [L, S).  The single-image layout of the Cache
 * Contract is prefix P, one image, suffix s: I0 = P, I1 = P + h*w,
 * L = I1 + s. */
#define OMAX_IMG 64
typedef struct {
    int64_t I0, I1, w;
} oimage;
typedef struct {
    int64_t L;
    int n;
    oimage img[OMAX_IMG];
} osample;

/* Flat batch geometry: sample b holds n_img[b] images, entries
 * first_b .. first_b + n_img[b] - 1 of text_before / img_h / img_w (first_b
 * the running sum of n_img); image j is preceded by text_before[j] text
 * tokens; after the last image come suffix[b] text tokens. */
typedef struct {
    int B;
    const int32_t *n_img, *text_before, *img_h, *img_w, *suffix;
} ogeom;

static int make_sample(const ogeom* g, int b, osample* s) {
    int64_t first = 0;
    for (int i = 0; i < b; ++i) first += g->n_img[i];
    int n = g->n_img[b];
    if (n < 0 || n > OMAX_IMG || g->suffix[b] < 0) return -1;
    int64_t pos = 0;
    s->n = n;
    for (int j = 0; j < n; ++j) {
        int64_t t = g->text_before[first + j], h = g->img_h[first + j], w = g->img_w[first + j];
        if (t < 0 || h <= 0 || w <= 0) return -1;
        s->img[j].I0 = pos + t;
        s->img[j].I1 = s->img[j].I0 + h * w;
        s->img[j].w = w;
        pos = s->img[j].I1;
    }
    s->L = pos + g->suffix[b];
    return 0;
}

static int image_of(const osample* s, int64_t n) {
    for (int j = 0; j < s->n; ++j)
        if (s->img[j].I0 <= n && n < s->img[j].I1) return j;
    return -1;
}

/* The literal mask rule (build_joint_attention_mask; 3.1.2; 3.3), with the
 * multi-image rule of 3.1.2 (in a training sequence with several generated
 * images, an image already in context is masked from the tokens after it;
 * read here as: every image but the sample's last is hidden from all tokens
 * after its span, the last image follows the one-image rule):
 *   key k visible from query q  <=>  k < L  and  ( q, k in the same image  or
 *                                   ( k <= q  and  k not in a context image ) ),
 * a context image being one of images 0 .. n-2 (any k <= q outside q's own
 * image lies before q's image, so it is hidden exactly when its image is a
 * context image). */
static int visible(const osample* s, int64_t q, int64_t k) {
    if (k >= s->L) return 0;
    int iq = image_of(s, q), ik = image_of(s, k);
    if (iq >= 0 && iq == ik) return 1;
    if (k > q) return 0;
    if (ik >= 0 && ik < s->n - 1) return 0;
    return 1;
}

/* mask: uint8 [B, S, S] indexed [b, q, k]. */
int oracle_mask(int B, int S, const int32_t* n_img, const int32_t* text_before, const int32_t* img_h,
                const int32_t* img_w, const int32_t* suffix, uint8_t* mask) {
    ogeom g = {B, n_img, text_before, img_h, img_w, suffix};
    osample s;
    for (int b = 0; b < B; ++b) {
        if (make_sample(&g, b, &s) || s.L > S) return -1;
        for (int64_t q = 0; q < S; ++q)
            for (int64_t k = 0; k < S; ++k)
                mask[((int64_t)b * S + q) * S + k] = (uint8_t)visible(&s, q, k);
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Generalized 2D RoPE (3.4 of the paper review)                             */
/* ------------------------------------------------------------------------ */

/* 2D position (x, y) of token n of sample s: a token of image j at row r,
 * column c of its grid sits at (I0_j + c, I0_j + r); any other token at
 * (n, n).  (With several images the pages also shift the positions after a
 * generated image, 3.1.3, by an amount they do not give: not modelled.) */
static void position(const osample* s, int64_t n, double* x, double* y) {
    int j = image_of(s, n);
    if (j >= 0) {
        int64_t i = n - s->img[j].I0;
        int64_t r = i / s->img[j].w, c = i % s->img[j].w;
        *x = (double)(s->img[j].I0 + c);
        *y = (double)(s->img[j].I0 + r);
    } else {
        *x = (double)n;
        *y = (double)n;
    }
}

/* angle_j of token n: (j even ? x : y) * base^(-2j/D). */
static double angle(const osample* s, int64_t n, int j, int D, double base) {
    double x, y;
    position(s, n, &x, &y);
    double theta = pow(base, -2.0 * (double)j / (double)D);
    return ((j % 2 == 0) ? x : y) * theta;
}

/* positions: int64 [B, S] x and y. */
int oracle_positions(int B, int S, const int32_t* n_img, const int32_t* text_before, const int32_t* img_h,
                     const int32_t* img_w, const int32_t* suffix, int64_t* xs, int64_t* ys) {
    ogeom g = {B, n_img, text_before, img_h, img_w, suffix};
    osample s;
    for (int b = 0; b < B; ++b) {
        if (make_sample(&g, b, &s) || s.L > S) return -1;
        for (int64_t n = 0; n < S; ++n) {
            double x, y;
            position(&s, n, &x, &y);
            xs[(int64_t)b * S + n] = (int64_t)x;
            ys[(int64_t)b * S + n] = (int64_t)y;
        }
    }
    return 0;
}

/* cos, sin fp64 [B, S, D]: entry j and j + D/2 both hold angle_j. */
int oracle_rope_tables(int B, int S, int D, const int32_t* n_img, const int32_t* text_before,
                       const int32_t* img_h, const int32_t* img_w, const int32_t* suffix, double base,
                       double* cos_t, double* sin_t) {
    if (D % 2) return -1;
    ogeom g = {B, n_img, text_before, img_h, img_w, suffix};
    osample s;
    for (int b = 0; b < B; ++b) {
        if (make_sample(&g, b, &s) || s.L > S) return -1;
        for (int64_t n = 0; n < S; ++n)
            for (int j = 0; j < D / 2; ++j) {
                double a = angle(&s, n, j, D, base);
                int64_t o = ((int64_t)b * S + n) * D;
                cos_t[o + j] = cos(a);
                cos_t[o + j + D / 2] = cos(a);
                sin_t[o + j] = sin(a);
                sin_t[o + j + D / 2] = sin(a);
            }
    }
    return 0;
}

/* R(n) v: (Rv)_j = v_j cos a_j - v_{j+D/2} sin a_j,
 *         (Rv)_{j+D/2} = v_{j+D/2} cos a_j + v_j sin a_j.
 * (v * cos + rotate_half(v) * sin, rotate_half(v) = [-v_hi, v_lo].) */
static void rotate(const osample* s, int64_t n, int D, double base, const double* v, double* out) {
    for (int j = 0; j < D / 2; ++j) {
        double a = angle(s, n, j, D, base);
        double c = cos(a), sn = sin(a);
        double lo = v[j], hi = v[j + D / 2];
        out[j] = lo * c - hi * sn;
        out[j + D / 2] = hi * c + lo * sn;
    }
}

/* R(n)^T v, the inverse rotation (R is orthogonal). */
static void rotate_t(const osample* s, int64_t n, int D, double base, const double* v, double* out) {
    for (int j = 0; j < D / 2; ++j) {
        double a = angle(s, n, j, D, base);
        double c = cos(a), sn = sin(a);
        double lo = v[j], hi = v[j + D / 2];
        out[j] = lo * c + hi * sn;
        out[j + D / 2] = hi * c - lo * sn;
    }
}

/* Apply R (inverse = 0) or R^T (inverse = 1) to x [B, S, H, D] in place of y. */
int oracle_rope_apply(int B, int S, int H, int D, const int32_t* n_img, const int32_t* text_before,
                      const int32_t* img_h, const int32_t* img_w, const int32_t* suffix, double base,
                      int inverse, const double* x, double* y) {
    if (D % 2) return -1;
    ogeom g = {B, n_img, text_before, img_h, img_w, suffix};
    osample s;
    for (int b = 0; b < B; ++b) {
        if (make_sample(&g, b, &s) || s.L > S) return -1;
        for (int64_t n = 0; n < S; ++n)
            for (int h = 0; h < H; ++h) {
                int64_t o = (((int64_t)b * S + n) * H + h) * D;
                if (inverse) rotate_t(&s, n, D, base, x + o, y + o);
                else rotate(&s, n, D, base, x + o, y + o);
            }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Attention: naive S x S scores with the explicit mask, fp64 softmax.        */
/* ------------------------------------------------------------------------ */

typedef struct {
    int B, S, Hq, Hkv, D;
    const osample* samples;     /* [B], built from the flat geometry */
    const double *q, *k, *v, *dout;
    double scale, base;
    int rotate_inputs;          /* 1: apply R to q, k here; 0: inputs already rotated */
    const int32_t* rows;        /* query rows to compute, or NULL for all */
    int n_rows;
    const uint8_t* group_sel;   /* [B * Hkv] 1 = compute this (b, kv head) group; NULL = all */
    const double *wq, *wk;      /* QK RMSNorm weights [D] each, or NULL: no norm */
    double eps;
    double *o, *lse;            /* fwd outputs */
    double *dq, *dk_h, *dv_h;   /* bwd outputs; dk_h, dv_h per q head [B,S,Hq,D] */
    double *dwq_h, *dwk_h;      /* bwd, with the norm: weight gradients per (b, q head) [B*Hq][D] */
    int n_tasks;
    int next_task;
    pthread_mutex_t lock;
} job_t;

static double dot(const double* a, const double* b, int D) {
    double s = 0.0;
    for (int d = 0; d < D; ++d) s += a[d] * b[d];
    return s;
}

/* HunyuanRMSNorm of one head vector: y = w * x / sqrt(mean(x^2) + eps).
 * Returns r = 1 / sqrt(mean(x^2) + eps). */
static double rms_norm(const double* x, const double* w, int D, double eps, double* y) {
    double ss = 0.0;
    for (int d = 0; d < D; ++d) ss += x[d] * x[d];
    double r = 1.0 / sqrt(ss / D + eps);
    for (int d = 0; d < D; ++d) y[d] = w[d] * x[d] * r;
    return r;
}

/* Vector-Jacobian product of rms_norm at x (r from rms_norm): with
 * xh = r x and a = w * gy, gx = r (a - xh <a, xh> / D); gw += gy * xh. */
static void rms_norm_vjp(const double* x, const double* w, int D, double r, const double* gy,
                         double* gx, double* gw) {
    double ax = 0.0;
    for (int d = 0; d < D; ++d) ax += w[d] * gy[d] * x[d] * r;
    for (int d = 0; d < D; ++d) gx[d] = r * (w[d] * gy[d] - x[d] * r * ax / D);
    if (gw)
        for (int d = 0; d < D; ++d) gw[d] += gy[d] * x[d] * r;
}

/* Rotated copy of head h of tensor x [B,S,H,D] for sample b: out [S, D]. */
static void gather_head(const job_t* J, const double* x, int H, int b, int h, int rot, double* out) {
    const osample* sp = &J->samples[b];
    for (int64_t n = 0; n < J->S; ++n) {
        const double* src = x + (((int64_t)b * J->S + n) * H + h) * J->D;
        if (rot) rotate(sp, n, J->D, J->base, src, out + n * J->D);
        else memcpy(out + n * J->D, src, sizeof(double) * J->D);
    }
}

/* Forward for one (b, h): o [B,S,Hq,D], lse [B,Hq,S] (natural log of the sum
 * of exp(scaled score)). */
static void fwd_task(job_t* J, int b, int h) {
    const int S = J->S, D = J->D, g = J->Hq / J->Hkv;
    const osample* sp = &J->samples[b];
    double* qr = malloc(sizeof(double) * (size_t)S * D);
    double* kr = malloc(sizeof(double) * (size_t)S * D);
    double* vv = malloc(sizeof(double) * (size_t)S * D);
    double* sc = malloc(sizeof(double) * (size_t)S);
    gather_head(J, J->q, J->Hq, b, h, J->rotate_inputs, qr);
    gather_head(J, J->k, J->Hkv, b, h / g, J->rotate_inputs, kr);
    gather_head(J, J->v, J->Hkv, b, h / g, 0, vv);
    if (J->wq)
        for (int64_t n = 0; n < S; ++n) {
            rms_norm(qr + n * D, J->wq, D, J->eps, qr + n * D);
            rms_norm(kr + n * D, J->wk, D, J->eps, kr + n * D);
        }
    int nr = J->rows ? J->n_rows : S;
    for (int ri = 0; ri < nr; ++ri) {
        int64_t q = J->rows ? J->rows[ri] : ri;
        double m = -INFINITY;
        for (int64_t k = 0; k < S; ++k) {
            sc[k] = visible(sp, q, k) ? J->scale * dot(qr + q * D, kr + k * D, D) : -INFINITY;
            if (sc[k] > m) m = sc[k];
        }
        double* orow = J->o + (((int64_t)b * S + q) * J->Hq + h) * D;
        double* lrow = J->lse + ((int64_t)b * J->Hq + h) * S + q;
        for (int d = 0; d < D; ++d) orow[d] = 0.0;
        if (m == -INFINITY) { *lrow = -INFINITY; continue; }
        double l = 0.0;
        for (int64_t k = 0; k < S; ++k) {
            if (sc[k] == -INFINITY) continue;
            double p = exp(sc[k] - m);
            l += p;
            for (int d = 0; d < D; ++d) orow[d] += p * vv[k * D + d];
        }
        for (int d = 0; d < D; ++d) orow[d] /= l;
        *lrow = m + log(l);
    }
    free(qr); free(kr); free(vv); free(sc);
}

/* Backward for one (b, h).  Recomputes the forward in fp64, then
 *   dP = dO V^T,  Dq = dO . O,  dS = P (dP - Dq),
 *   dQr = scale dS Kr,  dKr += scale dS^T Qr,  dV += P^T dO,
 * and returns dQ = R^T dQr; dk_h/dv_h hold this head's R^T dKr and dV
 * contributions (summed over the heads of a group by the caller).  With the
 * QK RMSNorm, Qr and Kr are the normalized rotated rows and the gradients
 * pass through the norm's vector-Jacobian product before R^T; the weight
 * gradients of this head go to dwq_h / dwk_h. */
static void bwd_task(job_t* J, int b, int h) {
    const int S = J->S, D = J->D, g = J->Hq / J->Hkv;
    const osample* sp = &J->samples[b];
    size_t SD = (size_t)S * D;
    double* qr = malloc(sizeof(double) * SD);
    double* kr = malloc(sizeof(double) * SD);
    double* vv = malloc(sizeof(double) * SD);
    double* dkr = calloc(SD, sizeof(double));
    double* dvv = calloc(SD, sizeof(double));
    double* dqr = malloc(sizeof(double) * D);
    double* orow = malloc(sizeof(double) * D);
    double* sc = malloc(sizeof(double) * (size_t)S);
    gather_head(J, J->q, J->Hq, b, h, J->rotate_inputs, qr);
    gather_head(J, J->k, J->Hkv, b, h / g, J->rotate_inputs, kr);
    gather_head(J, J->v, J->Hkv, b, h / g, 0, vv);
    /* with the norm: keep the rotated rows (qx, kx) and normalize qr, kr */
    double *qx = NULL, *kx = NULL, *rq = NULL, *rk = NULL, *gx = NULL;
    double *dwq = NULL, *dwk = NULL;
    if (J->wq) {
        qx = malloc(sizeof(double) * SD);
        kx = malloc(sizeof(double) * SD);
        rq = malloc(sizeof(double) * (size_t)S);
        rk = malloc(sizeof(double) * (size_t)S);
        gx = malloc(sizeof(double) * D);
        memcpy(qx, qr, sizeof(double) * SD);
        memcpy(kx, kr, sizeof(double) * SD);
        for (int64_t n = 0; n < S; ++n) {
            rq[n] = rms_norm(qx + n * D, J->wq, D, J->eps, qr + n * D);
            rk[n] = rms_norm(kx + n * D, J->wk, D, J->eps, kr + n * D);
        }
        dwq = J->dwq_h + ((size_t)b * J->Hq + h) * D;
        dwk = J->dwk_h + ((size_t)b * J->Hq + h) * D;
    }
    int nr = J->rows ? J->n_rows : S;
    for (int ri = 0; ri < nr; ++ri) {
        int64_t q = J->rows ? J->rows[ri] : ri;
        const double* dorow = J->dout + (((int64_t)b * S + q) * J->Hq + h) * D;
        double* dqout = J->dq + (((int64_t)b * S + q) * J->Hq + h) * D;
        double m = -INFINITY;
        for (int64_t k = 0; k < S; ++k) {
            sc[k] = visible(sp, q, k) ? J->scale * dot(qr + q * D, kr + k * D, D) : -INFINITY;
            if (sc[k] > m) m = sc[k];
        }
        if (m == -INFINITY) { for (int d = 0; d < D; ++d) dqout[d] = 0.0; continue; }
        double l = 0.0;
        for (int d = 0; d < D; ++d) orow[d] = 0.0;
        for (int64_t k = 0; k < S; ++k) {
            if (sc[k] == -INFINITY) { sc[k] = 0.0; continue; }
            sc[k] = exp(sc[k] - m);          /* unnormalised P */
            l += sc[k];
            for (int d = 0; d < D; ++d) orow[d] += sc[k] * vv[k * D + d];
        }
        for (int d = 0; d < D; ++d) orow[d] /= l;
        double Dq = dot(dorow, orow, D);
        for (int d = 0; d < D; ++d) dqr[d] = 0.0;
        for (int64_t k = 0; k < S; ++k) {
            if (sc[k] == 0.0) continue;
            double p = sc[k] / l;
            double dp = dot(dorow, vv + k * D, D);
            double ds = p * (dp - Dq);
            for (int d = 0; d < D; ++d) {
                dqr[d] += J->scale * ds * kr[k * D + d];
                dkr[k * D + d] += J->scale * ds * qr[q * D + d];
                dvv[k * D + d] += p * dorow[d];
            }
        }
        if (J->wq) {
            rms_norm_vjp(qx + q * D, J->wq, D, rq[q], dqr, gx, dwq);
            memcpy(dqr, gx, sizeof(double) * D);
        }
        if (J->rotate_inputs) rotate_t(sp, q, D, J->base, dqr, dqout);
        else memcpy(dqout, dqr, sizeof(double) * D);
    }
    for (int64_t k = 0; k < S; ++k) {
        double* dko = J->dk_h + (((int64_t)b * S + k) * J->Hq + h) * D;
        double* dvo = J->dv_h + (((int64_t)b * S + k) * J->Hq + h) * D;
        if (J->wq) {
            rms_norm_vjp(kx + k * D, J->wk, D, rk[k], dkr + k * D, gx, dwk);
            memcpy(dkr + k * D, gx, sizeof(double) * D);
        }
        if (J->rotate_inputs) rotate_t(sp, k, D, J->base, dkr + k * D, dko);
        else memcpy(dko, dkr + k * D, sizeof(double) * D);
        memcpy(dvo, dvv + k * D, sizeof(double) * D);
    }
    free(qr); free(kr); free(vv); free(dkr); free(dvv); free(dqr); free(orow); free(sc);
    free(qx); free(kx); free(rq); free(rk); free(gx);
}

static int task_selected(const job_t* J, int t) {
    int b = t / J->Hq, h = t % J->Hq, g = J->Hq / J->Hkv;
    return J->group_sel == NULL || J->group_sel[b * J->Hkv + h / g];
}

typedef struct { job_t* J; int is_bwd; } worker_arg;

static void* worker(void* p) {
    worker_arg* a = (worker_arg*)p;
    job_t* J = a->J;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int t = J->next_task++;
        pthread_mutex_unlock(&J->lock);
        if (t >= J->n_tasks) break;
        if (!task_selected(J, t)) continue;
        if (a->is_bwd) bwd_task(J, t / J->Hq, t % J->Hq);
        else fwd_task(J, t / J->Hq, t % J->Hq);
    }
    return NULL;
}

static int run_job(job_t* J, int is_bwd, int nthreads) {
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 1024) nthreads = 1024;
    J->n_tasks = J->B * J->Hq;
    J->next_task = 0;
    pthread_mutex_init(&J->lock, NULL);
    pthread_t* th = malloc(sizeof(pthread_t) * nthreads);
    worker_arg a = {J, is_bwd};
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &a);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J->lock);
    return nthreads;
}

/* Builds J->samples from the flat geometry; -1 on bad geometry. */
static int load_geom(job_t* J, osample* buf, const ogeom* g, int S, int Hq, int Hkv, int D) {
    if (g->B < 0 || S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv || D <= 0 || D % 2) return -1;
    for (int b = 0; b < g->B; ++b)
        if (make_sample(g, b, &buf[b]) || buf[b].L > S) return -1;
    J->samples = buf;
    return 0;
}

/* Forward.  q [B,S,Hq,D], k, v [B,S,Hkv,D] (fp64, exact copies of the bf16
 * inputs); o [B,S,Hq,D]; lse [B,Hq,S].  rows/n_rows restrict the query rows;
 * group_sel [B*Hkv] restricts the (b, kv head) groups; wq, wk [D] (both or
 * neither) turn on the QK RMSNorm with epsilon eps.  Returns the number of
 * threads used, or -1 on bad arguments. */
int oracle_attn_fwd(int B, int S, int Hq, int Hkv, int D, const int32_t* n_img, const int32_t* text_before,
                    const int32_t* img_h, const int32_t* img_w, const int32_t* suffix,
                    const double* q, const double* k, const double* v, double scale,
                    double base, int rotate_inputs, const int32_t* rows, int n_rows,
                    const uint8_t* group_sel, const double* wq, const double* wk, double eps,
                    double* o, double* lse, int nthreads) {
    if ((wq == NULL) != (wk == NULL) || (wq && !(eps >= 0.0))) return -1;
    job_t J;
    memset(&J, 0, sizeof(J));
    ogeom g = {B, n_img, text_before, img_h, img_w, suffix};
    osample* smp = malloc(sizeof(osample) * (B > 0 ? B : 1));
    if (load_geom(&J, smp, &g, S, Hq, Hkv, D)) { free(smp); return -1; }
    J.B = B; J.S = S; J.Hq = Hq; J.Hkv = Hkv; J.D = D;
    J.q = q; J.k = k; J.v = v; J.scale = scale; J.base = base;
    J.rotate_inputs = rotate_inputs; J.rows = rows; J.n_rows = n_rows;
    J.group_sel = group_sel; J.o = o; J.lse = lse;
    J.wq = wq; J.wk = wk; J.eps = eps;
    int used = run_job(&J, 0, nthreads);
    free(smp);
    return used;
}

/* Backward.  dq [B,S,Hq,D]; dk, dv [B,S,Hkv,D].  group_sel as above (dq of
 * unselected groups and their dk/dv are left untouched).  rows/n_rows
 * restrict the query rows: dq is written for those rows only and dk, dv hold
 * the contributions of those rows only (a partial sum over queries).  With
 * the QK RMSNorm (wq, wk non-NULL) dwq, dwk [D] receive the weight
 * gradients, summed over the selected groups and rows. */
int oracle_attn_bwd(int B, int S, int Hq, int Hkv, int D, const int32_t* n_img, const int32_t* text_before,
                    const int32_t* img_h, const int32_t* img_w, const int32_t* suffix,
                    const double* q, const double* k, const double* v, const double* dout,
                    double scale, double base, int rotate_inputs, const int32_t* rows, int n_rows,
                    const uint8_t* group_sel, const double* wq, const double* wk, double eps,
                    double* dq, double* dk, double* dv, double* dwq, double* dwk, int nthreads) {
    if ((wq == NULL) != (wk == NULL) || (wq && (!(eps >= 0.0) || !dwq || !dwk))) return -1;
    size_t n = (size_t)B * S * Hq * D;
    job_t J;
    memset(&J, 0, sizeof(J));
    ogeom geom = {B, n_img, text_before, img_h, img_w, suffix};
    osample* smp = malloc(sizeof(osample) * (B > 0 ? B : 1));
    if (load_geom(&J, smp, &geom, S, Hq, Hkv, D)) { free(smp); return -1; }
    J.B = B; J.S = S; J.Hq = Hq; J.Hkv = Hkv; J.D = D;
    J.q = q; J.k = k; J.v = v; J.dout = dout; J.scale = scale; J.base = base;
    J.rotate_inputs = rotate_inputs; J.rows = rows; J.n_rows = n_rows;
    J.group_sel = group_sel; J.dq = dq;
    J.dk_h = calloc(n ? n : 1, sizeof(double));
    J.dv_h = calloc(n ? n : 1, sizeof(double));
    J.wq = wq; J.wk = wk; J.eps = eps;
    size_t nw = (size_t)B * Hq * D;
    if (wq) {
        J.dwq_h = calloc(nw ? nw : 1, sizeof(double));
        J.dwk_h = calloc(nw ? nw : 1, sizeof(double));
    }
    int used = run_job(&J, 1, nthreads);
    if (wq) {
        /* weight gradients: sum of the per-(b, head) partials, in a fixed order */
        for (int d = 0; d < D; ++d) { dwq[d] = 0.0; dwk[d] = 0.0; }
        for (size_t t = 0; t < (size_t)B * Hq; ++t)
            for (int d = 0; d < D; ++d) {
                dwq[d] += J.dwq_h[t * D + d];
                dwk[d] += J.dwk_h[t * D + d];
            }
        free(J.dwq_h);
        free(J.dwk_h);
    }
    int g = Hq / Hkv;
    for (int b = 0; b < B; ++b)
        for (int hk = 0; hk < Hkv; ++hk) {
            if (group_sel && !group_sel[b * Hkv + hk]) continue;
            for (int64_t s = 0; s < S; ++s)
                for (int d = 0; d < D; ++d) {
                    double ak = 0.0, av = 0.0;
                    for (int i = 0; i < g; ++i) {
                        int64_t o = (((int64_t)b * S + s) * Hq + hk * g + i) * D + d;
                        ak += J.dk_h[o];
                        av += J.dv_h[o];
                    }
                    dk[(((int64_t)b * S + s) * Hkv + hk) * D + d] = ak;
                    dv[(((int64_t)b * S + s) * Hkv + hk) * D + d] = av;
                }
        }
    free(J.dk_h);
    free(J.dv_h);
    free(smp);
    return used;
}
