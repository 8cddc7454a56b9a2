/*
 * CPU oracle for the RotateAttention INT4 attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check
 * and the benchmark's CPU-baseline leg may load this library.  It is a plain,
 * slow, obviously-correct restatement of what the method computes; it shares
 * no code, header, table or constant generator with the CUDA library.
 *
 * Source: "RotateAttention: RoPE-Aware Rotation and Range Rectification for
 * INT4 Quantized Attention in Video Generation" (arXiv 2607.02584), as
 * summarised on its review page:
 *   - 3D RoPE splits head_dim into frame / height / width segments
 *     (core claim; axiom ledger; Fig. 2 caption);
 *   - RoPE-aware rotation: block-diagonal 2x2 orthogonal blocks, either on
 *     adjacent dims (Interleaved, mergeable into RoPE) or pairing a dim with
 *     its counterpart in the other half of its segment (Half)
 *     (Fig. 3 caption; "What carries the argument");
 *   - blocks initialised to the 2x2 Hadamard H2 (free-parameter ledger);
 *   - INT4 FlashAttention with online softmax (abstract);
 *   - range-optimised P quantisation: P = exp(QK^T - max) in [0,1] mapped to
 *     [-8,7] with fixed scale 15 and zero-point -8 (Sec. 4.2; ledger);
 *   - the V column-sum term that corrects the zero-point in P.V.
 * Where the pages are silent the plainest reading is taken; each such reading
 * is marked READING below.
 *
 * Precision: every step that decides an integer (a Q/K/V code, a P code)
 * is taken in IEEE fp32 with no FMA contraction (build with
 * -ffp-contract=off; the one fused multiply-add, in the P exponent, is an
 * explicit fmaf), because that is the precision the CUDA path decides in;
 * the P code itself is then exact for its fp32 exponent; integer products are
 * exact (int32/int64); the running accumulators of the online softmax are
 * float64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef _Float16 f16;

/* The oracle's own description of one problem. */
typedef struct {
    int B, H, d;          /* batch, heads, head_dim (128) */
    int F, Hh, W;         /* latent video grid, frame-major */
    int n_text;           /* text tokens appended after the video tokens */
    int split[3];         /* RoPE segment sizes (frame, height, width) */
    double theta;         /* RoPE base */
    int rot;              /* 0 = no rotation, 1 = Interleaved, 2 = Half, 3 = Full */
    int v_rot;            /* 1: Hadamard on V (INT4 path), undone on O */
    const double *blocks; /* rot 4/5: d/2 caller 2x2 blocks {r00, r01, r10, r11} */
} orc_problem;

enum { ORC_ROT_NONE = 0, ORC_ROT_INTERLEAVED = 1, ORC_ROT_HALF = 2, ORC_ROT_FULL = 3,
       ORC_ROT_BLOCKS_INTERLEAVED = 4, ORC_ROT_BLOCKS_HALF = 5 };
enum { QK_BLOCK = 64, KV_TILE = 128 };

int orc_seq_len(const orc_problem *p) { return p->F * p->Hh * p->W + p->n_text; }

/* Padded length: a whole number of 128-token tiles. */
int orc_seq_pad(const orc_problem *p) { return (orc_seq_len(p) + KV_TILE - 1) / KV_TILE * KV_TILE; }

/* Token n -> axis positions (frame, row, column).  Video tokens are laid out
 * frame-major (f slowest, w fastest); appended text tokens sit at position 0
 * on every axis, i.e. RoPE leaves them unchanged.  READING: the pages give
 * neither the token order nor the text-token convention. */
void orc_token_pos(const orc_problem *p, int n, int pos[3])
{
    int nv = p->F * p->Hh * p->W;
    if (n >= nv) { pos[0] = pos[1] = pos[2] = 0; return; }
    pos[0] = n / (p->Hh * p->W);
    pos[1] = (n / p->W) % p->Hh;
    pos[2] = n % p->W;
}

/* RoPE angle for axis segment s, axis position pos, pair j (dims o_s+2j and
 * o_s+2j+1 of the segment): pos * theta^(-2j/d_s), in float64. */
double orc_rope_angle(const orc_problem *p, int s, int pos, int j)
{
    double w = pow(p->theta, -(double)(2 * j) / (double)p->split[s]);
    return (double)pos * w;
}

/* The fp32 coefficients the prologue uses, each rounded once from float64:
 * (cos a, sin a) for RoPE alone, and (alpha, beta) for RoPE followed by the
 * 2x2 Hadamard H2 on the same adjacent pair (the Interleaved rotation merged
 * into RoPE): H2 * [[c,-s],[s,c]] = [[alpha, beta],[beta, -alpha]] with
 * alpha = (c+s)/sqrt2, beta = (c-s)/sqrt2. */
void orc_rope_coef(const orc_problem *p, int s, int pos, int j,
                   float *c, float *sn, float *alpha, float *beta)
{
    double a = orc_rope_angle(p, s, pos, j);
    double ca = cos(a), sa = sin(a);
    *c = (float)ca;
    *sn = (float)sa;
    *alpha = (float)((ca + sa) * M_SQRT1_2);
    *beta = (float)((ca - sa) * M_SQRT1_2);
}

/* RoPE (no rotation) of one token in fp32: each adjacent pair (x0, x1) of a
 * segment becomes (c x0 - s x1, s x0 + c x1). */
static void rope_row(const orc_problem *p, int n, const f16 *x, float *y)
{
    int pos[3];
    orc_token_pos(p, n, pos);
    int o = 0;
    for (int s = 0; s < 3; ++s) {
        for (int j = 0; j < p->split[s] / 2; ++j) {
            float c, sn, al, be;
            orc_rope_coef(p, s, pos[s], j, &c, &sn, &al, &be);
            float x0 = (float)x[o + 2 * j], x1 = (float)x[o + 2 * j + 1];
            float a0 = c * x0, a1 = sn * x1;
            float b0 = sn * x0, b1 = c * x1;
            y[o + 2 * j] = a0 - a1;
            y[o + 2 * j + 1] = b0 + b1;
        }
        o += p->split[s];
    }
}

/* RoPE then the RoPE-aware rotation of one token (Q or K), fp32.
 *  - none:        z = RoPE(x)
 *  - Interleaved: H2 after RoPE on each adjacent pair, with the merged
 *                 (alpha, beta) coefficients: z0 = alpha x0 + beta x1,
 *                 z1 = beta x0 - alpha x1
 *  - Half:        z = RoPE(x), then in each segment dim i and dim i + d_s/2
 *                 (a, b) -> ((a+b)/sqrt2, (a-b)/sqrt2).
 * READING: rotation after RoPE (either order leaves QK^T unchanged); H2 is
 * the default block (free-parameter ledger). */
/* Normalised Walsh-Hadamard transform z = y H / sqrt(d), H in Sylvester
 * order (READING for the unspecified "Full" rotation and for the Hadamard the
 * pages fuse into V), as the fast transform in fp32: for h = 1, 2, ..., d/2
 * every pair (k, k + h) with k & h == 0 becomes (a + b, a - b); then one
 * multiply by fp32(1/sqrt(d)).  y is overwritten. */
static void hadamard_fp32(float *y, float *z, int d)
{
    for (int h = 1; h < d; h <<= 1)
        for (int i = 0; i < d; i += 2 * h)
            for (int k = i; k < i + h; ++k) {
                float a = y[k], b = y[k + h];
                y[k] = a + b;
                y[k + h] = a - b;
            }
    const float r = (float)(1.0 / sqrt((double)(d)));
    for (int c = 0; c < d; ++c) z[c] = y[c] * r;
}

/* The same transform in float64 (for undoing the V Hadamard on O: H is
 * symmetric and orthogonal, so H^T = H). */
static void hadamard_f64(double *y, int d)
{
    for (int w = 1; w < d; w *= 2)
        for (int i = 0; i < d; i += 2 * w)
            for (int k = i; k < i + w; ++k) {
                double u = y[k], t = y[k + w];
                y[k] = u + t;
                y[k + w] = u - t;
            }
    const double r = 1.0 / sqrt((double)d);
    for (int c = 0; c < d; ++c) y[c] *= r;
}

void orc_rotate_row(const orc_problem *p, int n, const f16 *x, float *z)
{
    if (p->rot == ORC_ROT_BLOCKS_INTERLEAVED) {
        /* caller's orthogonal block R_p on the adjacent pair p = o_s / 2 + j,
         * merged with the RoPE rotation: M = R Rot(a) in float64, rounded once */
        int pos[3];
        orc_token_pos(p, n, pos);
        int o = 0;
        for (int s = 0; s < 3; ++s) {
            for (int j = 0; j < p->split[s] / 2; ++j) {
                double a = orc_rope_angle(p, s, pos[s], j);
                double ca = cos(a), sa = sin(a);
                const double *R = p->blocks + 4 * (o / 2 + j);
                float m00 = (float)(R[0] * ca + R[1] * sa), m01 = (float)(R[1] * ca - R[0] * sa);
                float m10 = (float)(R[2] * ca + R[3] * sa), m11 = (float)(R[3] * ca - R[2] * sa);
                float x0 = (float)x[o + 2 * j], x1 = (float)x[o + 2 * j + 1];
                float t0 = m00 * x0, t1 = m01 * x1, t2 = m10 * x0, t3 = m11 * x1;
                z[o + 2 * j] = t0 + t1;
                z[o + 2 * j + 1] = t2 + t3;
            }
            o += p->split[s];
        }
        return;
    }
    if (p->rot == ORC_ROT_INTERLEAVED) {
        int pos[3];
        orc_token_pos(p, n, pos);
        int o = 0;
        for (int s = 0; s < 3; ++s) {
            for (int j = 0; j < p->split[s] / 2; ++j) {
                float c, sn, al, be;
                orc_rope_coef(p, s, pos[s], j, &c, &sn, &al, &be);
                float x0 = (float)x[o + 2 * j], x1 = (float)x[o + 2 * j + 1];
                float a0 = al * x0, a1 = be * x1;
                float b0 = be * x0, b1 = al * x1;
                z[o + 2 * j] = a0 + a1;
                z[o + 2 * j + 1] = b0 - b1;
            }
            o += p->split[s];
        }
        return;
    }
    float y[512];
    rope_row(p, n, x, y);
    if (p->rot == ORC_ROT_NONE) {
        memcpy(z, y, sizeof(float) * p->d);
        return;
    }
    if (p->rot == ORC_ROT_FULL) {   /* the dense comparison of Figs. 4-5 */
        hadamard_fp32(y, z, p->d);
        return;
    }
    if (p->rot == ORC_ROT_BLOCKS_HALF) {
        /* caller's orthogonal block R_p on (o_s + i, o_s + i + d_s/2) after RoPE,
         * p = o_s / 2 + i (learned rotations, Sec. 4.1); R rounded to fp32 */
        int o = 0;
        for (int s = 0; s < 3; ++s) {
            int h = p->split[s] / 2;
            for (int i = 0; i < h; ++i) {
                const double *R = p->blocks + 4 * (o / 2 + i);
                float r00 = (float)R[0], r01 = (float)R[1], r10 = (float)R[2], r11 = (float)R[3];
                float ya = y[o + i], yb = y[o + i + h];
                float t0 = r00 * ya, t1 = r01 * yb, t2 = r10 * ya, t3 = r11 * yb;
                z[o + i] = t0 + t1;
                z[o + i + h] = t2 + t3;
            }
            o += p->split[s];
        }
        return;
    }
    const float r = (float)M_SQRT1_2;
    int o = 0;
    for (int s = 0; s < 3; ++s) {
        int h = p->split[s] / 2;
        for (int i = 0; i < h; ++i) {
            float a = y[o + i], b = y[o + i + h];
            float sum = a + b, dif = a - b;
            z[o + i] = sum * r;
            z[o + i + h] = dif * r;
        }
        o += p->split[s];
    }
}

/* RoPE only, rounded to fp16 (RNE): the FP16 path's Q/K after RoPE. */
void orc_rope_fp16_head(const orc_problem *p, const f16 *x, f16 *y)
{
    int N = orc_seq_len(p), d = p->d;
    #pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) {
        float t[512];
        rope_row(p, n, x + (size_t)n * d, t);
        for (int c = 0; c < d; ++c) y[(size_t)n * d + c] = (f16)t[c];
    }
}

/* Symmetric INT4 code of v with scale s: clamp(rne(v / s), -7, 7), 0 if s == 0. */
static int8_t int4_code(float v, float s)
{
    if (s == 0.0f) return 0;
    float q = nearbyintf(v / s);
    if (q > 7.0f) q = 7.0f;
    if (q < -7.0f) q = -7.0f;
    return (int8_t)q;
}

/* Q or K of one head: RoPE + rotation, then per 64-token block one scale
 * amax/7 over all 64 x d values and codes rne(z/scale) in [-7, 7].
 * codes: [N_pad][d], padded tokens 0; scales: [N_pad/64], padded blocks 0.
 * READING: the 64-token block matches the FlashAttention block size used by
 * block-wise attention quantisation; V is handled by orc_quantize_v_head. */
void orc_quantize_qk_head(const orc_problem *p, const f16 *x, int8_t *codes, float *scales)
{
    int N = orc_seq_len(p), Np = orc_seq_pad(p), d = p->d;
    float *z = (float *)malloc(sizeof(float) * (size_t)N * d);
    #pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) orc_rotate_row(p, n, x + (size_t)n * d, z + (size_t)n * d);
    memset(codes, 0, (size_t)Np * d);
    for (int g = 0; g < Np / QK_BLOCK; ++g) {
        int n0 = g * QK_BLOCK, n1 = n0 + QK_BLOCK < N ? n0 + QK_BLOCK : N;
        float amax = 0.0f;
        for (int n = n0; n < n1; ++n)
            for (int c = 0; c < d; ++c) {
                float a = fabsf(z[(size_t)n * d + c]);
                if (a > amax) amax = a;
            }
        float s = amax / 7.0f;
        scales[g] = s;
        for (int n = n0; n < n1; ++n)
            for (int c = 0; c < d; ++c)
                codes[(size_t)n * d + c] = int4_code(z[(size_t)n * d + c], s);
    }
    free(z);
}

/* V of one head: one symmetric INT4 scale per channel over all N tokens
 * (amax_c / 7), codes in [-7, 7], and the per-64-token-block column sums of
 * the codes used by the zero-point correction.  By default no transform is
 * applied to V (v_rot = 0):
 * the paper's Hadamard on V is fused offline into the model weights.
 * codes: [N_pad][d]; sv: [d]; colsum: [N_pad/64][d].
 * READING: the pages fix no granularity for V; per-channel over the whole
 * sequence keeps the scale constant along the P.V contraction. */
void orc_quantize_v_head(const orc_problem *p, const f16 *v, int8_t *codes, float *sv, int32_t *colsum)
{
    int N = orc_seq_len(p), Np = orc_seq_pad(p), d = p->d;
    /* V as fp32; with v_rot every row times H / sqrt(d) first (the stand-in
     * for the Hadamard the pages fuse into V offline) */
    float *vf = (float *)malloc(sizeof(float) * (size_t)N * d);
    for (int n = 0; n < N; ++n) {
        float y[512];
        for (int c = 0; c < d; ++c) y[c] = (float)v[(size_t)n * d + c];
        if (p->v_rot) hadamard_fp32(y, vf + (size_t)n * d, d);
        else memcpy(vf + (size_t)n * d, y, sizeof(float) * d);
    }
    for (int c = 0; c < d; ++c) {
        float amax = 0.0f;
        for (int n = 0; n < N; ++n) {
            float a = fabsf(vf[(size_t)n * d + c]);
            if (a > amax) amax = a;
        }
        sv[c] = amax / 7.0f;
    }
    memset(codes, 0, (size_t)Np * d);
    memset(colsum, 0, sizeof(int32_t) * (size_t)(Np / QK_BLOCK) * d);
    for (int n = 0; n < N; ++n)
        for (int c = 0; c < d; ++c) {
            int8_t q = int4_code(vf[(size_t)n * d + c], sv[c]);
            codes[(size_t)n * d + c] = q;
            colsum[(size_t)(n / QK_BLOCK) * d + c] += q;
        }
    free(vf);
}

/* Range-optimised P code: P in [0,1] -> rne(15 P) - 8 in [-8, 7]
 * (fixed scale 15, zero-point -8; Sec. 4.2). */
int orc_p_code(float P) { return (int)nearbyintf(15.0f * P) - 8; }

/* Symmetric INT4 code of P in [0,1] (the map the range-optimised one
 * replaces; abstract: symmetric quantisation of the non-negative P leaves
 * half of the codes unused): scale max|P| / 7 = 1/7, code = rne(7 P) in [0, 7],
 * no zero-point. */
int orc_p_code_sym(float P) { return (int)nearbyintf(7.0f * P); }

/* The P weight w = code + zero-point of the quantised path, taken from the
 * exponent in log2 units: w = rne(levels * 2^x) with P = 2^x, levels = 15
 * for the range-optimised map (code = w - 8) and 7 for the symmetric one
 * (code = w).  READING: the pages fix no precision for P = exp(s - m); the
 * code is decided for the fp32 exponent x, exactly: levels * 2^x is
 * evaluated in float64 (exact to ~1e-16 relative, far below the distance of
 * any 2^x with fp32 x from a half-integer, except x = -1 where
 * 15 * 2^-1 = 7.5 exactly and the round-half-to-even rint gives 8). */
int orc_p_weight(float x, int levels) { return (int)rint((double)levels * exp2((double)x)); }

/* READING (several correct results): a P code is decided on hardware from an
 * approximate 2^x with relative error at most ORC_EX2_REL (measured on the
 * GPU and bounded there by a test).  Where levels * 2^x lies within that
 * relative distance of a half-integer, either neighbouring weight is a
 * correct fp32 decision: orc_p_weight_amb returns the exact weight and sets
 * *amb; the alternative is the other neighbour of that half-integer. */
#define ORC_EX2_REL 9.5367431640625e-07   /* 2^-20 */
int orc_p_weight_amb(float x, int levels, int *amb)
{
    double v = (double)levels * exp2((double)x);
    double h = floor(v) + 0.5;               /* nearest half-integer above floor */
    double dist = fabs(v - h);
    if (fabs(v - (h - 1.0)) < dist) dist = fabs(v - (h - 1.0));
    *amb = dist <= v * ORC_EX2_REL;
    return (int)rint(v);
}

/* The other weight of an ambiguous key: the neighbour across the half-integer
 * next to levels * 2^x. */
static int p_weight_other(float x, int levels, int w)
{
    double v = (double)levels * exp2((double)x);
    return v >= (double)w ? w + 1 : w - 1;
}

/* One query row i of the INT4 attention (one head), T_kv = `tile` keys per
 * step of the online softmax (128 for the method as built).
 *
 * Per tile j (keys [n0, n1)):
 *   S[n]  = sum_c q_code[i,c] k_code[n,c]                         (int32)
 *   s[n]  = S[n] * s_Q[i/64] * s_K[n/64] / sqrt d, taken in log2 units:
 *           t[n] = S[n] * c_b with c_b = (s_Q[i/64] log2(e) / sqrt d) s_K[b] (fp32)
 *   m_j   = max(m_{j-1}, max_n t[n])                               (fp32)
 *   P[n]  = exp(s[n] - s_max) = 2^x[n], x[n] = S[n] c_b - m_j      (fp32, one rounding)
 *   code[n] = rne(15 P) - 8, decided exactly for that x            (float64)
 *   PV[c] = sum_n code[n] v_code[n,c] + 8 colsum_j[c]              (int64)
 *   L     = sum_n (code[n] + 8)                                    (int64)
 *   acc   = acc * 2^(m_{j-1} - m_j) + PV;  l = l * 2^(..) + L     (float64)
 * O[i,c] = acc[c] * s_V[c] / l, rounded to fp16; the common 1/15 cancels.
 * READINGS: the standard 1/sqrt(d) softmax scale applies to the dequantised
 * logits; the normaliser uses the dequantised codes (keeps O a convex
 * combination of dequantised V rows); P is quantised against the running max.
 *
 * quant_p = 1: the range-optimised code above.  quant_p = 2: the symmetric
 * code rne(7 P) instead, with no zero-point term and L = sum code.
 * quant_p = 0 replaces the P code by the exact P (float64, natural-log
 * units, s = fl(fl(S fl(s_Q s_K)) / sqrt d)) and drops the zero-point, for
 * checking the loop against two-pass softmax attention.
 * Optional outputs: o64 [d] (float64 before the fp16 rounding); for tile
 * index dbg_tile >= 0, dbg_S [tile] and dbg_P [tile] (S and P codes of that
 * tile, -128 where the key is past N); amb [max_amb] and n_amb: the keys
 * whose P code is ambiguous (orc_p_weight_amb).  flip [n_flip]: ambiguous
 * keys to decide the other way (to form the other correct results).
 * colsum: [N_pad/64][d] per-64-block column sums of the V codes. */
void orc_attention_row(const orc_problem *p, int i, int tile, int quant_p,
                       const int8_t *qc, const float *qs, const int8_t *kc, const float *ks,
                       const int8_t *vc, const float *sv, const int32_t *colsum,
                       f16 *o, double *o64, int dbg_tile, int32_t *dbg_S, int8_t *dbg_P,
                       int32_t *amb, int max_amb, int32_t *n_amb, const int32_t *flip, int n_flip)
{
    int N = orc_seq_len(p), d = p->d;
    const float inv_sqrt_d = (float)(1.0 / sqrt((double)d));
    /* quantised P: log2 units in fp32, the precision the CUDA path decides
     * in: K = fl(fl(log2 e) / fl(sqrt d)), per 64-key block b the factor
     * c_b = fl(fl(s_Q[i/64] K) s_K[b]), the dequantised logit t = fl(S c_b)
     * (s log2 e), the running max m of t, the exponent x = fl(S c_b - m)
     * rounded once (a fused multiply-add), and w = rne(levels 2^x) exactly
     * (orc_p_weight).  With P = 2^x this is P = exp(s - m). */
    const float log2e_f = (float)M_LOG2E, sqrt_d_f = (float)sqrt((double)d);
    const float K_log2 = log2e_f / sqrt_d_f;
    const float kq = qs[i / QK_BLOCK] * K_log2;
    float m = -INFINITY;
    double *acc = (double *)calloc((size_t)d, sizeof(double));
    double l = 0.0;
    int32_t *S = (int32_t *)malloc(sizeof(int32_t) * (size_t)tile);
    float *sl = (float *)malloc(sizeof(float) * (size_t)tile);
    double *pv = (double *)malloc(sizeof(double) * (size_t)d);
    const int8_t *qrow = qc + (size_t)i * d;
    for (int j = 0, n0 = 0; n0 < N; ++j, n0 += tile) {
        int n1 = n0 + tile < N ? n0 + tile : N;
        float tmax = -INFINITY;
        for (int n = n0; n < n1; ++n) {
            int32_t acc_s = 0;
            for (int c = 0; c < d; ++c) acc_s += (int32_t)qrow[c] * (int32_t)kc[(size_t)n * d + c];
            S[n - n0] = acc_s;
            float s;
            if (quant_p) {
                s = (float)acc_s * (kq * ks[n / QK_BLOCK]);   /* log2 units */
            } else {
                float sc = qs[i / QK_BLOCK] * ks[n / QK_BLOCK];
                float t = (float)acc_s * sc;
                s = t * inv_sqrt_d;
            }
            sl[n - n0] = s;
            if (s > tmax) tmax = s;
        }
        float m_new = m > tmax ? m : tmax;
        double L = 0.0;
        for (int c = 0; c < d; ++c) pv[c] = 0.0;
        if (quant_p) {
            int64_t pvi[512] = {0};
            int64_t Li = 0;
            const int zp = quant_p == 2 ? 0 : 8;
            const int levels = quant_p == 2 ? 7 : 15;
            for (int n = n0; n < n1; ++n) {
                float x = fmaf((float)S[n - n0], kq * ks[n / QK_BLOCK], -m_new);
                int is_amb = 0;
                int w = orc_p_weight_amb(x, levels, &is_amb);
                if (is_amb) {
                    if (n_amb && *n_amb < max_amb && amb) amb[*n_amb] = n;
                    if (n_amb) ++*n_amb;
                    for (int f = 0; f < n_flip; ++f)
                        if (flip[f] == n) w = p_weight_other(x, levels, w);
                }
                int code = w - (quant_p == 2 ? 0 : 8);
                Li += code + zp;
                for (int c = 0; c < d; ++c) pvi[c] += (int64_t)code * vc[(size_t)n * d + c];
                if (j == dbg_tile && dbg_P) dbg_P[n - n0] = (int8_t)code;
            }
            /* zero-point correction: + 8 * sum over the tile's keys of the V codes */
            if (zp)
                for (int g = n0 / QK_BLOCK; g * QK_BLOCK < n1; ++g)
                    for (int c = 0; c < d; ++c) pvi[c] += 8 * (int64_t)colsum[(size_t)g * d + c];
            for (int c = 0; c < d; ++c) pv[c] = (double)pvi[c];
            L = (double)Li;
        } else {
            for (int n = n0; n < n1; ++n) {
                double P = exp((double)sl[n - n0] - (double)m_new);
                L += P;
                for (int c = 0; c < d; ++c) pv[c] += P * (double)vc[(size_t)n * d + c];
            }
        }
        if (j == dbg_tile) {
            for (int n = 0; n < tile; ++n) {
                if (dbg_S) dbg_S[n] = n0 + n < n1 ? S[n] : 0;
                if (dbg_P && n0 + n >= n1) dbg_P[n] = -128;
            }
        }
        double alpha = (j == 0) ? 0.0 : quant_p ? exp2((double)m - (double)m_new) : exp((double)m - (double)m_new);
        for (int c = 0; c < d; ++c) acc[c] = acc[c] * alpha + pv[c];
        l = l * alpha + L;
        m = m_new;
    }
    double orow[512];
    for (int c = 0; c < d; ++c) orow[c] = acc[c] * (double)sv[c] / l;
    if (p->v_rot) hadamard_f64(orow, d);   /* O = O' H^T undoes V' = V H */
    for (int c = 0; c < d; ++c) {
        double val = orow[c];
        if (o64) o64[c] = val;
        if (o) o[c] = (f16)val;
    }
    free(acc); free(S); free(sl); free(pv);
}

/* Rows `rows[0..nrows)` of one head; out: [nrows][d] fp16, out64 optional.
 * amb_count [nrows] and amb_keys [nrows][max_amb] (optional): the ambiguous
 * keys of each row (see orc_p_weight_amb), their number and the first
 * max_amb of them. */
void orc_attention_rows(const orc_problem *p, const int64_t *rows, int nrows, int tile, int quant_p,
                        const int8_t *qc, const float *qs, const int8_t *kc, const float *ks,
                        const int8_t *vc, const float *sv, const int32_t *colsum,
                        f16 *out, double *out64, int32_t *amb_count, int32_t *amb_keys, int max_amb)
{
    int d = p->d;
    #pragma omp parallel for schedule(dynamic, 4)
    for (int r = 0; r < nrows; ++r) {
        int32_t cnt = 0;
        orc_attention_row(p, (int)rows[r], tile, quant_p, qc, qs, kc, ks, vc, sv, colsum,
                          out ? out + (size_t)r * d : NULL, out64 ? out64 + (size_t)r * d : NULL,
                          -1, NULL, NULL, amb_keys ? amb_keys + (size_t)r * max_amb : NULL, max_amb,
                          &cnt, NULL, 0);
        if (amb_count) amb_count[r] = cnt;
    }
}

/* Float64 softmax attention of one head on given (already position-encoded)
 * fp32 or fp16-valued rows: O[i] = sum_n softmax_n(q_i.k_n / sqrt d) v_n.
 * Used for the unquantised diagnostic and as the FP16 path's oracle. */
void orc_softmax_attention_rows(const orc_problem *p, const int64_t *rows, int nrows,
                                const double *q, const double *k, const double *v, double *out)
{
    int N = orc_seq_len(p), d = p->d;
    double scale = 1.0 / sqrt((double)d);
    #pragma omp parallel for schedule(dynamic, 4)
    for (int r = 0; r < nrows; ++r) {
        const double *qi = q + (size_t)rows[r] * d;
        double *s = (double *)malloc(sizeof(double) * (size_t)N);
        double mx = -INFINITY;
        for (int n = 0; n < N; ++n) {
            double t = 0.0;
            for (int c = 0; c < d; ++c) t += qi[c] * k[(size_t)n * d + c];
            s[n] = t * scale;
            if (s[n] > mx) mx = s[n];
        }
        double den = 0.0;
        for (int n = 0; n < N; ++n) { s[n] = exp(s[n] - mx); den += s[n]; }
        double *o = out + (size_t)r * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        for (int n = 0; n < N; ++n)
            for (int c = 0; c < d; ++c) o[c] += s[n] * v[(size_t)n * d + c];
        for (int c = 0; c < d; ++c) o[c] /= den;
        free(s);
    }
}

/* Rotated fp32 rows of one head (RoPE + rotation, before quantisation). */
void orc_rotate_head(const orc_problem *p, const f16 *x, float *z)
{
    int N = orc_seq_len(p), d = p->d;
    #pragma omp parallel for schedule(static)
    for (int n = 0; n < N; ++n) orc_rotate_row(p, n, x + (size_t)n * d, z + (size_t)n * d);
}
