/*
 * sage_oracle.c -- CPU oracle for the SageAttention quantized attention
 * forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the plain, slow, obviously-correct
 * reference that the CUDA path is checked against.  Only the tests, the
 * package's smoke check and the benchmark's CPU-baseline leg load it; the
 * product path never does, and this file shares no code, header, table or
 * constant generator with the CUDA sources.
 *
 * What the method computes, and where the web pages say it:
 *   - "sageattention" package page (skillfed.io), "Quickstart": the call is
 *     sageattn(q, k, v, tensor_layout="HND", is_causal=False, smooth_k=True);
 *     "What it is": per-block quantization of queries and keys plus
 *     smoothing; head dims 64/96/128, Nq != Nkv, group-query attention.
 *   - closerAI ComfyUI blog, part 2 ("keeping precision"): INT8 for QK^T,
 *     FP8 for PV, smoothing to reduce quantisation error, quantisation at
 *     several granularities; part 4: SageAttention2's per-thread
 *     quantisation, finer than per block.
 *   - "SageAttention2: Technical report" (ai-digest.ru), section 1: Q and K
 *     quantised at warp / thread granularity; section 2 ("smoothing Q and
 *     V"): the channel mean of Q and V is subtracted before quantisation.
 *   - The flash-style tiled pass (online softmax with running max and sum,
 *     exp2, P quantised to FP8, FP32 accumulation) is the FlashAttention
 *     comparison all pages make (e.g. the pwwt.cn guide, section 3.2).
 *
 * The pages fix no block size, rounding rule or scale convention.  The
 * readings taken here are:
 *   - Q is quantised with one INT8 scale per query token (per-thread
 *     granularity where one thread owns one query row); K with one scale per
 *     block of 32 keys; the online softmax walks KV tiles of 128 keys.
 *   - INT8 codes are symmetric in [-127, 127]: scale = amax/127,
 *     code = rint(x * (127/amax)) with round-half-even, computed in IEEE
 *     fp32 without FMA contraction.  A block with amax < 2^-64 gets scale 0
 *     and all-zero codes.
 *   - The 4-bit variant (SageAttention2 technical report, section 1: Q and
 *     K in INT4 at warp level; section 3: 8 bits for the sensitive layers,
 *     4 bits elsewhere) uses the same blocks with codes in [-7, 7]:
 *     scale = amax/7, code = rint(x * (7/amax)).
 *   - Means are exact fixed-point means: sum of rint(x * 2^24) in int64,
 *     divided in fp64 by n * 2^24 and rounded to fp32.  This makes the mean
 *     independent of summation order.  Q's smoothing mean is taken per block
 *     of 128 tokens.
 *   - V is FP8 e4m3 per channel over all tokens: scale = amax/448, code =
 *     e4m3_rn_satfinite(x * (448/amax)).
 *   - Online softmax, the plain definition: per KV tile the row's running
 *     max m becomes max(m, tile max); when it grows, O and l are multiplied
 *     by 2^(m_old - m_new); every visible key contributes
 *     p = 448 * 2^(s - m) to l unquantised and, quantised to e4m3, to
 *     O += e4m3(p) * v.  p <= 448, e4m3's largest finite value.
 *   - Causal masking is top-left aligned (key j is visible to query i when
 *     j <= i), as in scaled_dot_product_attention.
 *   - Query head h reads kv head h / (Hq / Hkv).
 *
 * Floating point: the quantisation steps whose result is an integer code
 * (INT8 of Q and K, FP8 of V) are taken in fp32, the precision of the CUDA
 * path.  The logits s = S * q_scale * k_scale * sm_scale * log2(e) and
 * everything after them are fp64.  Build with -ffp-contract=off and no
 * -ffast-math so that every fp32 operation here is one IEEE-rounded op.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <float.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define QMBLK 128  /* query smoothing-mean block (tokens)  */
#define KBLK 32    /* key quantisation block (tokens)     */
#define KVT 128    /* keys per online-softmax tile        */
#define QTILE 128  /* query rows per output tile          */

typedef struct {
    int B, Hq, Hkv, Nq, Nkv, D;
    int layout;      /* 0 = HND [B,H,N,D], 1 = NHD [B,N,H,D]; contiguous */
    int dtype;       /* 0 = fp16, 1 = bf16 */
    int is_causal, smooth_k, smooth_q, smooth_v;
    float sm_scale;  /* already resolved (> 0) */
    int qk_bits;     /* 8: INT8 codes of Q and K in [-127, 127]; 4: INT4 codes in [-7, 7] */
} oracle_params;

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------------
 * Number formats, written from their definitions.
 * ------------------------------------------------------------------- */

/* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 mantissa bits. */
double oracle_f16_to_double(uint16_t h) {
    int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
    double v;
    if (e == 31) v = m ? NAN : INFINITY;
    else if (e == 0) v = ldexp((double)m, -24);
    else v = ldexp((double)(1024 + m), e - 25);
    return s ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static double in_to_double(const oracle_params *p, uint16_t bits) {
    return p->dtype == 0 ? oracle_f16_to_double(bits) : oracle_bf16_to_double(bits);
}

/* Round a double to a binary format with `mbits` mantissa bits, exponent
 * bias `bias`, max biased exponent `emax_field` (all-ones is inf/NaN),
 * round-half-even, overflow to infinity. */
static uint16_t round_to_16(double x, int mbits, int ebits) {
    int bias = (1 << (ebits - 1)) - 1;
    uint16_t s = signbit(x) ? (uint16_t)(1u << 15) : 0;
    double a = fabs(x);
    uint16_t inf = (uint16_t)(((1u << ebits) - 1) << mbits);
    if (isnan(x)) return s | inf | 1;
    if (isinf(a)) return s | inf;
    double min_normal = ldexp(1.0, 1 - bias);
    if (a < min_normal) {
        /* subnormal grid: multiples of 2^(1 - bias - mbits) */
        double q = nearbyint(ldexp(a, bias - 1 + mbits));
        return s | (uint16_t)q;   /* q == 2^mbits lands on the smallest normal */
    }
    int E;
    double f = frexp(a, &E);      /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1;
    double q = nearbyint((2.0 * f - 1.0) * ldexp(1.0, mbits));
    if (q == ldexp(1.0, mbits)) { e += 1; q = 0.0; }
    if (e + bias >= (1 << ebits) - 1) return s | inf;
    return s | (uint16_t)(((e + bias) << mbits) | (int)q);
}

uint16_t oracle_double_to_f16(double x) { return round_to_16(x, 10, 5); }
uint16_t oracle_double_to_bf16(double x) { return round_to_16(x, 7, 8); }

/* OCP 8-bit floating point, E4M3 variant: 1 sign, 4 exponent (bias 7),
 * 3 mantissa bits, no infinities, S.1111.111 is NaN, largest finite 448,
 * subnormals m * 2^-9.  Encoding rounds half to even and saturates finite
 * values to +-448 ("satfinite"). */
double oracle_e4m3_decode(uint8_t c) {
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp((double)(8 + m), e - 10);
    return s ? -v : v;
}

uint8_t oracle_e4m3_encode(double x) {
    if (isnan(x)) return 0x7F;
    uint8_t s = signbit(x) ? 0x80 : 0;
    double a = fabs(x);
    if (a >= 448.0) return s | 0x7E;
    if (a < 0.015625) {                 /* below 2^-6: the subnormal grid */
        double q = nearbyint(a * 512.0);/* 0..8; 8 is the smallest normal */
        return s | (uint8_t)q;
    }
    int E;
    double f = frexp(a, &E);
    int e = E - 1;                      /* a = (2f) * 2^e, e in [-6, 8] */
    double q = nearbyint((2.0 * f - 1.0) * 8.0);
    if (q == 8.0) { e += 1; q = 0.0; }
    return s | (uint8_t)(((e + 7) << 3) | (int)q);
}

void oracle_e4m3_encode_array(const double *x, uint8_t *out, int64_t n) {
    for (int64_t i = 0; i < n; i++) out[i] = oracle_e4m3_encode(x[i]);
}

void oracle_e4m3_encode_f32_array(const float *x, uint8_t *out, int64_t n) {
    for (int64_t i = 0; i < n; i++) out[i] = oracle_e4m3_encode((double)x[i]);
}

/* ---------------------------------------------------------------------
 * Indexing of the caller's tensors (contiguous, in the given layout).
 * ------------------------------------------------------------------- */
static int64_t idx(const oracle_params *p, int H, int N, int b, int h, int n, int c) {
    if (p->layout == 0) return (((int64_t)b * H + h) * N + n) * p->D + c;
    return (((int64_t)b * N + n) * H + h) * p->D + c;
}

/* Exact fixed-point mean of n values: sum of rint(x * 2^24) in int64,
 * divided in fp64 by n * 2^24, rounded to fp32. */
static float fixed_point_mean(const double *x, int64_t n) {
    int64_t acc = 0;
    for (int64_t i = 0; i < n; i++) acc += (int64_t)nearbyint(x[i] * 16777216.0);
    return (float)((double)acc / ((double)n * 16777216.0));
}

/* Symmetric integer quantisation of one block (fp32 arithmetic): codes in
 * [-qmax, qmax], qmax = 127 (INT8) or 7 (INT4). */
static float quantise_int_block(const float *x, int64_t n, int8_t *codes, float qmax) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; i++) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    if (!(amax >= 0x1p-64f)) {
        for (int64_t i = 0; i < n; i++) codes[i] = 0;
        return 0.0f;
    }
    float scale = amax / qmax;
    float inv = qmax / amax;
    for (int64_t i = 0; i < n; i++) {
        float t = x[i] * inv;
        float r = nearbyintf(t);
        if (r > qmax) r = qmax;
        if (r < -qmax) r = -qmax;
        codes[i] = (int8_t)r;
    }
    return scale;
}

/* ---------------------------------------------------------------------
 * Smoothing and quantisation of Q, K, V for every (batch, head).
 *
 * Outputs (natural layouts, independent of the input layout):
 *   mean_k  f32 [B][Hkv][D]          (zeros when smooth_k == 0)
 *   kp      f32 [B][Hkv][Nkv][D]     K' = K - mean_k (fp32)
 *   k8      i8  [B][Hkv][Nkv][D];  k_scale f32 [B][Hkv][ceil(Nkv/32)]
 *   mq      f32 [B][Hq][ceil(Nq/128)][D]   (zeros when smooth_q == 0)
 *   q8      i8  [B][Hq][Nq][D];    q_scale f32 [B][Hq][Nq]  (one per token)
 *   mean_v  f32 [B][Hkv][D]          (zeros when smooth_v == 0)
 *   v8      u8  [B][Hkv][Nkv][D];  v_scale f32 [B][Hkv][D]
 *   qp      f32 [B][Hq][Nq][D]       Q' = Q - mq (fp32); may be NULL
 *   vp      f32 [B][Hkv][Nkv][D]     V' = V - mean_v (fp32); may be NULL
 * ------------------------------------------------------------------- */
void oracle_prepass(const oracle_params *p, const uint16_t *q, const uint16_t *k,
                    const uint16_t *v, float *mean_k, float *kp, int8_t *k8,
                    float *k_scale, float *mq, int8_t *q8, float *q_scale,
                    float *mean_v, uint8_t *v8, float *v_scale, float *qp, float *vp_out) {
    const int D = p->D, Nq = p->Nq, Nkv = p->Nkv;
    const int nmb = (Nq + QMBLK - 1) / QMBLK, nkb = (Nkv + KBLK - 1) / KBLK;

    const float qmax = p->qk_bits == 4 ? 7.0f : 127.0f;

    /* K: mean over all tokens, K' = K - mean, per-32-token INT8 blocks. */
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < p->B; b++)
        for (int h = 0; h < p->Hkv; h++) {
            double *col = (double *)malloc(sizeof(double) * (size_t)Nkv);
            float *mk = mean_k + ((int64_t)b * p->Hkv + h) * D;
            float *kph = kp + ((int64_t)b * p->Hkv + h) * Nkv * D;
            for (int c = 0; c < D; c++) {
                for (int j = 0; j < Nkv; j++) col[j] = in_to_double(p, k[idx(p, p->Hkv, Nkv, b, h, j, c)]);
                mk[c] = p->smooth_k ? fixed_point_mean(col, Nkv) : 0.0f;
                for (int j = 0; j < Nkv; j++) kph[(int64_t)j * D + c] = (float)col[j] - mk[c];
            }
            for (int kb = 0; kb < nkb; kb++) {
                int j0 = kb * KBLK, n = (Nkv - j0 < KBLK) ? Nkv - j0 : KBLK;
                k_scale[((int64_t)b * p->Hkv + h) * nkb + kb] = quantise_int_block(
                    kph + (int64_t)j0 * D, (int64_t)n * D,
                    k8 + (((int64_t)b * p->Hkv + h) * Nkv + j0) * D, qmax);
            }
            free(col);
        }

    /* Q: optional per-128-token block mean, Q' = Q - mq, one INT8 scale per
     * token (the token's D channels form its quantisation block). */
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < p->B; b++)
        for (int h = 0; h < p->Hq; h++) {
            float *blk = (float *)malloc(sizeof(float) * QMBLK * (size_t)D);
            double *col = (double *)malloc(sizeof(double) * QMBLK);
            for (int mb = 0; mb < nmb; mb++) {
                int i0 = mb * QMBLK, n = (Nq - i0 < QMBLK) ? Nq - i0 : QMBLK;
                float *mqb = mq + (((int64_t)b * p->Hq + h) * nmb + mb) * D;
                for (int c = 0; c < D; c++) {
                    for (int r = 0; r < n; r++) col[r] = in_to_double(p, q[idx(p, p->Hq, Nq, b, h, i0 + r, c)]);
                    mqb[c] = p->smooth_q ? fixed_point_mean(col, n) : 0.0f;
                    for (int r = 0; r < n; r++) blk[(int64_t)r * D + c] = (float)col[r] - mqb[c];
                }
                for (int r = 0; r < n; r++) {
                    const int64_t row = ((int64_t)b * p->Hq + h) * Nq + i0 + r;
                    q_scale[row] = quantise_int_block(blk + (int64_t)r * D, D, q8 + row * D, qmax);
                    if (qp) memcpy(qp + row * D, blk + (int64_t)r * D, sizeof(float) * (size_t)D);
                }
            }
            free(blk);
            free(col);
        }

    /* V: optional channel mean, V' = V - mean_v, per-channel FP8 e4m3. */
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < p->B; b++)
        for (int h = 0; h < p->Hkv; h++) {
            double *col = (double *)malloc(sizeof(double) * (size_t)Nkv);
            float *vp = (float *)malloc(sizeof(float) * (size_t)Nkv);
            for (int c = 0; c < D; c++) {
                for (int j = 0; j < Nkv; j++) col[j] = in_to_double(p, v[idx(p, p->Hkv, Nkv, b, h, j, c)]);
                float mv = p->smooth_v ? fixed_point_mean(col, Nkv) : 0.0f;
                mean_v[((int64_t)b * p->Hkv + h) * D + c] = mv;
                float amax = 0.0f;
                for (int j = 0; j < Nkv; j++) {
                    vp[j] = (float)col[j] - mv;
                    if (fabsf(vp[j]) > amax) amax = fabsf(vp[j]);
                    if (vp_out) vp_out[(((int64_t)b * p->Hkv + h) * Nkv + j) * D + c] = vp[j];
                }
                uint8_t *v8h = v8 + ((int64_t)b * p->Hkv + h) * Nkv * D;
                if (!(amax >= 0x1p-64f)) {
                    v_scale[((int64_t)b * p->Hkv + h) * D + c] = 0.0f;
                    for (int j = 0; j < Nkv; j++) v8h[(int64_t)j * D + c] = 0;
                    continue;
                }
                v_scale[((int64_t)b * p->Hkv + h) * D + c] = amax / 448.0f;
                float inv = 448.0f / amax;
                for (int j = 0; j < Nkv; j++) {
                    float t = vp[j] * inv;
                    v8h[(int64_t)j * D + c] = oracle_e4m3_encode((double)t);
                }
            }
            free(col);
            free(vp);
        }
}

/* Q-smoothing correction for one query block: dS[j] = sum_c mq[c] K'[j][c]
 * in fp64 (the term that restores Q K'^T from Q' K'^T). */
void oracle_delta_s(const oracle_params *p, const float *mq_blk, const float *kp_head,
                    double *dS) {
    for (int j = 0; j < p->Nkv; j++) {
        double acc = 0.0;
        for (int c = 0; c < p->D; c++) acc += (double)mq_blk[c] * (double)kp_head[(int64_t)j * p->D + c];
        dS[j] = acc;
    }
}

/* ---------------------------------------------------------------------
 * The tiled quantised attention, step by step, for selected query tiles.
 *
 * tiles: n_tiles triples (b, h, qt); out: [n_tiles][128][D] fp64 outputs
 * (rows >= Nq are left untouched).  Per row i and 128-key tile:
 *   S_j  = q8_i . k8_j in int64 (exact);
 *   s_j  = S_j * q_scale_i * k_scale_blk(j) * sm_scale * log2(e)
 *          (+ dS_j * sm_scale * log2(e) with smoothed Q), in fp64 from the
 *          fp32 scales;
 *   m    = max(m, max_j s_j); when m grows, O and l *= 2^(m_old - m_new);
 *   p_j  = 448 * 2^(s_j - m);  l += p_j;  O += e4m3(p_j) * v8_j;
 * and finally o = O * v_scale / l (+ mean_v).
 *
 * exact_mask (for the error decomposition; 0 in every parity use):
 *   bit 0: P enters O unquantised (O += p_j * v)
 *   bit 1: V unquantised (v = V' in fp32, and no v_scale)
 *   bit 2: Q K^T unquantised (s_j from Q' . K' in fp64; needs qp)
 * With all three set the result is exact softmax attention of (Q, K', V)
 * up to the fp32 rounding of the smoothed inputs.
 *
 * unc (optional, same shape as out): how far an implementation may lie from
 * `out` because the FP8 code of P is not unique when p is computed in fp32
 * with a hardware exp2.  Such an implementation forms the exponent from fp32
 * scales and logits (a few IEEE roundings, each at most 2^-24 relative:
 * the scale product, the logit, the running max, its shift by log2(448),
 * the subtraction; and, with smoothed Q, an fp32 dot product of D terms for
 * dS), then a hardware exp2 of relative error at most EXP2_REL.  The first-
 * order bound on the exponent's error, doubled, gives a relative band on p;
 * wherever p lies within that band of an e4m3 rounding midpoint both
 * neighbouring codes are valid, and unc accumulates, per output channel,
 * the effect of taking the other code: |step| * |v8| * v_scale / l.
 * ------------------------------------------------------------------- */
#define EXP2_REL 0x1p-21   /* hardware exp2 allowance (measured on the GPU by a test) */
#define U32 0x1p-24        /* fp32 unit roundoff */

void oracle_attention_tiles(const oracle_params *p, const int8_t *q8, const float *q_scale,
                            const int8_t *k8, const float *k_scale, const uint8_t *v8,
                            const float *v_scale, const float *mean_v, const float *mq,
                            const float *kp, const float *qp, const float *vp, int exact_mask,
                            int n_tiles, const int *tiles, double *out, double *unc) {
    const int D = p->D, Nq = p->Nq, Nkv = p->Nkv;
    const int nmb = (Nq + QMBLK - 1) / QMBLK, nkb = (Nkv + KBLK - 1) / KBLK;
    const int nkt = (Nkv + KVT - 1) / KVT;
    const double scl = (double)p->sm_scale * 1.44269504088896340736;  /* sm_scale * log2(e) */
    const double LN2 = 0.69314718055994530942;
    const int keep_p = exact_mask & 1, keep_v = exact_mask & 2, keep_qk = exact_mask & 4;
    double vdec[256];
    for (int c = 0; c < 256; c++) vdec[c] = oracle_e4m3_decode((uint8_t)c);

#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int t = 0; t < n_tiles; t++)
        for (int r = 0; r < QTILE; r++) {
            const int b = tiles[3 * t], h = tiles[3 * t + 1], qt = tiles[3 * t + 2];
            const int i = qt * QTILE + r;
            if (i >= Nq) continue;
            const int hk = h / (p->Hq / p->Hkv);
            const int64_t qrow_i = ((int64_t)b * p->Hq + h) * Nq + i;
            const double qs = (double)q_scale[qrow_i];
            const int8_t *qrow = q8 + qrow_i * D;
            const float *qprow = qp ? qp + qrow_i * D : NULL;
            const int8_t *kh = k8 + ((int64_t)b * p->Hkv + hk) * Nkv * D;
            const float *kph = kp + ((int64_t)b * p->Hkv + hk) * Nkv * D;
            const uint8_t *vh = v8 + ((int64_t)b * p->Hkv + hk) * Nkv * D;
            const float *vph = vp ? vp + ((int64_t)b * p->Hkv + hk) * Nkv * D : NULL;
            const float *ksh = k_scale + ((int64_t)b * p->Hkv + hk) * nkb;
            double *O = (double *)calloc((size_t)D, sizeof(double));
            double *U = (double *)calloc((size_t)D, sizeof(double));
            double *dS = NULL, *dmag = NULL;
            const float *mqb = NULL;
            if (p->smooth_q) {
                mqb = mq + (((int64_t)b * p->Hq + h) * nmb + i / QMBLK) * D;
                dS = (double *)malloc(sizeof(double) * (size_t)Nkv);
                dmag = (double *)malloc(sizeof(double) * (size_t)Nkv);
                oracle_delta_s(p, mqb, kph, dS);
                for (int j = 0; j < Nkv; j++) {
                    double a = 0.0;
                    for (int c = 0; c < D; c++) a += fabs((double)mqb[c] * (double)kph[(int64_t)j * D + c]);
                    dmag[j] = a;
                }
            }
            double m = -INFINITY, l = 0.0;
            double s[KVT], mag[KVT];
            int valid[KVT];
            for (int kt = 0; kt < nkt; kt++) {
                /* logits of the tile's visible keys */
                double tile_max = -INFINITY;
                int any = 0;
                for (int jj = 0; jj < KVT; jj++) {
                    const int j = kt * KVT + jj;
                    valid[jj] = j < Nkv && (!p->is_causal || j <= i);
                    if (!valid[jj]) continue;
                    any = 1;
                    double x;
                    if (keep_qk) {
                        double acc = 0.0;
                        for (int c = 0; c < D; c++) acc += (double)qprow[c] * (double)kph[(int64_t)j * D + c];
                        x = acc * scl;
                    } else {
                        int64_t acc = 0;
                        for (int c = 0; c < D; c++) acc += (int64_t)qrow[c] * (int64_t)kh[(int64_t)j * D + c];
                        x = (double)acc * qs * (double)ksh[j / KBLK] * scl;
                    }
                    mag[jj] = fabs(x);
                    if (p->smooth_q) {
                        x += dS[j] * scl;
                        mag[jj] += fabs(dS[j] * scl) + (double)(D + 2) * dmag[j] * scl;
                    }
                    s[jj] = x;
                    if (x > tile_max) tile_max = x;
                }
                if (!any) continue;
                if (tile_max > m) {
                    if (m != -INFINITY) {
                        const double alpha = exp2(m - tile_max);
                        l *= alpha;
                        for (int cc = 0; cc < D; cc++) {
                            O[cc] *= alpha;
                            U[cc] *= alpha;
                        }
                    }
                    m = tile_max;
                }
                for (int jj = 0; jj < KVT; jj++) {
                    if (!valid[jj]) continue;
                    const int j = kt * KVT + jj;
                    const double pj = 448.0 * exp2(s[jj] - m);
                    l += pj;
                    double pq = pj;
                    uint8_t code = 0;
                    if (!keep_p) {
                        code = oracle_e4m3_encode(pj);
                        pq = vdec[code];
                    }
                    for (int cc = 0; cc < D; cc++) {
                        const double vv = keep_v ? (double)vph[(int64_t)j * D + cc] : vdec[vh[(int64_t)j * D + cc]];
                        O[cc] += pq * vv;
                    }
                    if (unc && !keep_p) {
                        const double band =
                            2.0 * LN2 * U32 * (5.0 * mag[jj] + 7.0 * fabs(m) + 27.0) + EXP2_REL;
                        const double lo = vdec[oracle_e4m3_encode(pj * (1.0 - band))];
                        const double hi = vdec[oracle_e4m3_encode(pj * (1.0 + band))];
                        const double step = fmax(hi - pq, pq - lo);
                        if (step > 0)
                            for (int cc = 0; cc < D; cc++) {
                                const double vv = keep_v ? (double)vph[(int64_t)j * D + cc] : vdec[vh[(int64_t)j * D + cc]];
                                U[cc] += step * fabs(vv);
                            }
                    }
                }
            }
            double *o = out + ((int64_t)t * QTILE + r) * D;
            const float *vs = v_scale + ((int64_t)b * p->Hkv + hk) * D;
            const float *mv = mean_v + ((int64_t)b * p->Hkv + hk) * D;
            for (int cc = 0; cc < D; cc++) {
                const double sc = keep_v ? 1.0 : (double)vs[cc];
                o[cc] = O[cc] * sc / l;
                if (p->smooth_v) o[cc] += (double)mv[cc];
                if (unc) unc[((int64_t)t * QTILE + r) * D + cc] = U[cc] * sc / l;
            }
            free(O);
            free(U);
            free(dS);
            free(dmag);
        }
}

/* ---------------------------------------------------------------------
 * Exact attention in fp64 from the unquantised inputs:
 * o_i = sum_j softmax_j(sm_scale * q_i . k_j) v_j over visible keys.
 * Same tile selection and output shape as oracle_attention_tiles.
 * ------------------------------------------------------------------- */
void oracle_exact_attention_tiles(const oracle_params *p, const uint16_t *q, const uint16_t *k,
                                  const uint16_t *v, int n_tiles, const int *tiles, double *out) {
    const int D = p->D, Nq = p->Nq, Nkv = p->Nkv;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int t = 0; t < n_tiles; t++)
        for (int r = 0; r < QTILE; r++) {
            const int b = tiles[3 * t], h = tiles[3 * t + 1], qt = tiles[3 * t + 2];
            const int i = qt * QTILE + r;
            if (i >= Nq) continue;
            const int hk = h / (p->Hq / p->Hkv);
            double *qi = (double *)malloc(sizeof(double) * (size_t)D);
            double *s = (double *)malloc(sizeof(double) * (size_t)Nkv);
            for (int c = 0; c < D; c++) qi[c] = in_to_double(p, q[idx(p, p->Hq, Nq, b, h, i, c)]);
            double m = -INFINITY;
            for (int j = 0; j < Nkv; j++) {
                if (p->is_causal && j > i) { s[j] = -INFINITY; continue; }
                double acc = 0.0;
                for (int c = 0; c < D; c++) acc += qi[c] * in_to_double(p, k[idx(p, p->Hkv, Nkv, b, hk, j, c)]);
                s[j] = acc * (double)p->sm_scale;
                if (s[j] > m) m = s[j];
            }
            double l = 0.0;
            double *o = out + ((int64_t)t * QTILE + r) * D;
            for (int c = 0; c < D; c++) o[c] = 0.0;
            for (int j = 0; j < Nkv; j++) {
                if (s[j] == -INFINITY) continue;
                double e = exp(s[j] - m);
                l += e;
                for (int c = 0; c < D; c++) o[c] += e * in_to_double(p, v[idx(p, p->Hkv, Nkv, b, hk, j, c)]);
            }
            for (int c = 0; c < D; c++) o[c] /= l;
            free(qi);
            free(s);
        }
}

/* Round fp64 outputs to the 16-bit output dtype (round-half-even). */
void oracle_round_output(const oracle_params *p, const double *x, uint16_t *bits, int64_t n) {
    for (int64_t i = 0; i < n; i++)
        bits[i] = p->dtype == 0 ? oracle_double_to_f16(x[i]) : oracle_double_to_bf16(x[i]);
}
