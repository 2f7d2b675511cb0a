/*
 * CPU oracle for the quantized projection GEMM of a diffusion-LLM denoising step.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file; only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline
 * leg use it.  It shares no code, header, table or constant with the CUDA path.
 *
 * What it computes, and where that is defined:
 *
 *  - Weights are GGUF K-quant super-blocks of QK_K = 256 weights.  The pages
 *    (mojo-dllm Architecture page, "Source map", quant/kquants.mojo row, and
 *    "Memory") name the Q4_K and Q6_K formats and make the scalar decoders the
 *    test oracle; the heatdrop repository card ("Key highlights") names the gguf
 *    package's dequantization as the external correctness reference.  The byte
 *    layouts themselves are not on the pages; they are the GGUF block formats
 *    (144-byte Q4_K, 210-byte Q6_K), restated below in our own words.  Q5_K
 *    (176 bytes) and Q8_0 (34-byte blocks of 32), the other formats the same row
 *    lists, are decoded too: the oracle side of the next formats.
 *  - Activations are quantized to int8 with one f32 scale per 256 elements
 *    (Architecture page, "Source map", kernels/qgemm.mojo row).  The pages do
 *    not fix the rounding; the reading used here is: amax over the block,
 *    iscale = 127/amax in f32, q = round-half-even(x*iscale) clamped to
 *    [-127, 127], scale = amax/127 in f32; an all-zero block has scale 0.
 *  - The GEMM result is out[m][n] = sum_k w[n][k] * a[m][k] where
 *    w = d*sc_j*q - dmin*m_j (Q4_K) or d*sc_j*(q-32) (Q6_K) and
 *    a = scale[m][sb] * qa.  It is formed the way the method runs it: integer
 *    sub-block dots, integer per-super-block combinations, and one fp64
 *    combine per super-block, rounded to f32 once at the end.
 *  - Bidirectional attention over the canvas (the next step the GPU path will
 *    take on; no kernel yet), in fp64, with grouped key/value heads.
 *  - The steps either side of the quantizer in a forward pass (Architecture page,
 *    "A forward pass", steps 2 and 4): RMSNorm of a projection input, and the
 *    SwiGLU gate SiLU(g) * u between the gate/up and down projections.  Both are
 *    formed in fp64 and rounded to f32 once; the fused library kernels quantize
 *    that f32 exactly like oracle_quantize_act.
 *
 * Parity status: every function here is pinned by tests (gguf package decode,
 * brute-force fp64 dequantize-then-matmul, closed forms and invariants).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define QK 256
#define Q4K_BYTES 144
#define Q5K_BYTES 176
#define Q6K_BYTES 210
#define Q80_BYTES 34     /* one Q8_0 block: 32 weights */

/* Bytes of one 256-weight span of a row, for each supported GGML type id:
 * 8 = Q8_0 (eight 34-byte blocks), 12 = Q4_K, 13 = Q5_K, 14 = Q6_K. */
static int span_bytes(int qtype)
{
    switch (qtype) {
    case 8: return 8 * Q80_BYTES;
    case 12: return Q4K_BYTES;
    case 13: return Q5K_BYTES;
    case 14: return Q6K_BYTES;
    default: return 0;
    }
}

/* IEEE 754 binary16 -> double, from the format definition: 1 sign bit,
 * 5 exponent bits (bias 15), 10 fraction bits; exponent 0 is subnormal,
 * exponent 31 is inf/nan.  Exact for every input. */
double oracle_f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int f = h & 1023;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);              /* f * 2^-14 * 2^-10 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);  /* (1 + f/1024) * 2^(e-15) */
    return sign ? -v : v;
}

static uint16_t rd16(const uint8_t *p) { return (uint16_t)(p[0] | (p[1] << 8)); }

/*
 * Q4_K super-block (144 bytes, 256 weights in 8 sub-blocks of 32):
 *   [0,2)  d     f16 super-block scale
 *   [2,4)  dmin  f16 super-block scale of the mins
 *   [4,16) 12 bytes holding eight 6-bit scales sc_j and eight 6-bit mins m_j:
 *          j < 4 : sc_j = b[j] & 63,          m_j = b[j+4] & 63
 *          j >= 4: sc_j = (b[j+4] & 15) | ((b[j-4] >> 6) << 4)
 *                  m_j  = (b[j+4] >> 4) | ((b[j]   >> 6) << 4)
 *   [16,144) 128 bytes of 4-bit quants: four 32-byte chunks; chunk c gives
 *          sub-block 2c its low nibbles and sub-block 2c+1 its high nibbles,
 *          both in byte order.
 *   weight value: d * sc_j * q - dmin * m_j.
 */
/* The eight 6-bit scales and mins of a Q4_K or Q5_K block, from its 12 packed bytes. */
static void scales_mins_6bit(const uint8_t *b, uint8_t sc[8], uint8_t mn[8])
{
    for (int j = 0; j < 8; j++) {
        if (j < 4) {
            sc[j] = b[j] & 63;
            mn[j] = b[j + 4] & 63;
        } else {
            sc[j] = (uint8_t)((b[j + 4] & 15) | ((b[j - 4] >> 6) << 4));
            mn[j] = (uint8_t)((b[j + 4] >> 4) | ((b[j] >> 6) << 4));
        }
    }
}

void oracle_q4k_decode(const uint8_t *blk, double *d, double *dmin,
                       uint8_t sc[8], uint8_t mn[8], uint8_t q[256])
{
    const uint8_t *qs = blk + 16;
    *d = oracle_f16_to_f64(rd16(blk));
    *dmin = oracle_f16_to_f64(rd16(blk + 2));
    scales_mins_6bit(blk + 4, sc, mn);
    for (int c = 0; c < 4; c++)
        for (int l = 0; l < 32; l++) {
            q[64 * c + l] = qs[32 * c + l] & 15;
            q[64 * c + 32 + l] = qs[32 * c + l] >> 4;
        }
}

/*
 * Q5_K super-block (176 bytes, 256 weights in 8 sub-blocks of 32): the Q4_K block
 * with a fifth bit per quant.  This is the GGUF definition; the pages list Q5_K among
 * the formats (Architecture page, "Source map", quant/kquants.mojo row).
 *   [0,2)    d     f16
 *   [2,4)    dmin  f16
 *   [4,16)   the eight 6-bit scales and mins, packed as in Q4_K
 *   [16,48)  qh: 32 bytes; bit j of qh[l] is the fifth bit of element l of sub-block j
 *   [48,176) qs: 128 bytes of low nibbles, in four 32-byte chunks as in Q4_K
 *            (chunk c: sub-block 2c in the low nibbles, 2c+1 in the high nibbles)
 *   q in [0, 31]; weight value: d * sc_j * q - dmin * m_j.
 */
void oracle_q5k_decode(const uint8_t *blk, double *d, double *dmin,
                       uint8_t sc[8], uint8_t mn[8], uint8_t q[256])
{
    const uint8_t *qh = blk + 16;
    const uint8_t *qs = blk + 48;
    *d = oracle_f16_to_f64(rd16(blk));
    *dmin = oracle_f16_to_f64(rd16(blk + 2));
    scales_mins_6bit(blk + 4, sc, mn);
    for (int c = 0; c < 4; c++)
        for (int l = 0; l < 32; l++) {
            int j0 = 2 * c, j1 = 2 * c + 1;
            q[32 * j0 + l] = (uint8_t)((qs[32 * c + l] & 15) | (((qh[l] >> j0) & 1) << 4));
            q[32 * j1 + l] = (uint8_t)((qs[32 * c + l] >> 4) | (((qh[l] >> j1) & 1) << 4));
        }
}

/*
 * Q8_0 block (34 bytes, 32 weights): d (f16) then 32 signed 8-bit quants;
 * weight value: d * q.  GGUF definition; the pages list Q8_0 among the formats
 * (Architecture page, "Source map", quant/kquants.mojo row).  A 256-weight span of a
 * row is eight consecutive blocks.
 */
void oracle_q80_decode(const uint8_t *blk, double *d, int8_t q[32])
{
    *d = oracle_f16_to_f64(rd16(blk));
    for (int i = 0; i < 32; i++) q[i] = (int8_t)blk[2 + i];
}

/*
 * Q6_K super-block (210 bytes, 256 weights in 16 sub-blocks of 16):
 *   [0,128)   ql: low 4 bits of the quants
 *   [128,192) qh: high 2 bits of the quants
 *   [192,208) 16 signed 8-bit sub-block scales
 *   [208,210) d f16
 *   The block is two halves h of 128 weights.  Inside a half, weight
 *   e = 32*g + l (g in 0..3, l in 0..31) takes its low 4 bits from byte
 *   ql[64h + l + 32*(g & 1)] (low nibble for g < 2, high nibble for g >= 2)
 *   and its high 2 bits from (qh[32h + l] >> 2g) & 3.  q is in [0, 63].
 *   weight value: d * scale[i / 16] * (q - 32) for global index i.
 */
void oracle_q6k_decode(const uint8_t *blk, double *d, int8_t sc[16], uint8_t q[256])
{
    const uint8_t *ql = blk;
    const uint8_t *qh = blk + 128;
    for (int i = 0; i < 16; i++)
        sc[i] = (int8_t)blk[192 + i];
    *d = oracle_f16_to_f64(rd16(blk + 208));
    for (int h = 0; h < 2; h++)
        for (int g = 0; g < 4; g++)
            for (int l = 0; l < 32; l++) {
                uint8_t lb = ql[64 * h + l + 32 * (g & 1)];
                int lo = (g < 2) ? (lb & 15) : (lb >> 4);
                int hi = (qh[32 * h + l] >> (2 * g)) & 3;
                q[128 * h + 32 * g + l] = (uint8_t)(lo | (hi << 4));
            }
}

/* Dequantize a row-major matrix of blocks ([N][K/256] super-blocks, or [N][K/32]
 * Q8_0 blocks) to fp64 [N][K].  qtype: 8 = Q8_0, 12 = Q4_K, 13 = Q5_K, 14 = Q6_K (the
 * GGML type ids). */
int oracle_dequant(int qtype, const uint8_t *w, int64_t N, int64_t K, double *out)
{
    if (K % QK || !span_bytes(qtype)) return -1;
    int64_t nsb = K / QK;
    int bb = span_bytes(qtype);
    for (int64_t n = 0; n < N; n++)
        for (int64_t s = 0; s < nsb; s++) {
            const uint8_t *blk = w + (n * nsb + s) * bb;
            double *o = out + n * K + s * QK;
            uint8_t q[256];
            if (qtype == 12) {
                double d, dmin;
                uint8_t sc[8], mn[8];
                oracle_q4k_decode(blk, &d, &dmin, sc, mn, q);
                for (int i = 0; i < QK; i++)
                    o[i] = d * sc[i / 32] * q[i] - dmin * mn[i / 32];
            } else if (qtype == 13) {
                double d, dmin;
                uint8_t sc[8], mn[8];
                oracle_q5k_decode(blk, &d, &dmin, sc, mn, q);
                for (int i = 0; i < QK; i++)
                    o[i] = d * sc[i / 32] * q[i] - dmin * mn[i / 32];
            } else if (qtype == 14) {
                double d;
                int8_t sc[16];
                oracle_q6k_decode(blk, &d, sc, q);
                for (int i = 0; i < QK; i++)
                    o[i] = d * sc[i / 16] * ((int)q[i] - 32);
            } else {
                for (int b = 0; b < 8; b++) {
                    double d;
                    int8_t q8[32];
                    oracle_q80_decode(blk + b * Q80_BYTES, &d, q8);
                    for (int i = 0; i < 32; i++) o[32 * b + i] = d * q8[i];
                }
            }
        }
    return 0;
}

/*
 * Activation quantization: int8 with one f32 scale per 256 elements
 * (Architecture page, "Source map", kernels/qgemm.mojo row).  Reading taken
 * for what the page leaves open: symmetric [-127,127]; iscale = 127/amax and
 * scale = amax/127, both single IEEE f32 divisions; q = round-half-even of the
 * single f32 product x*iscale; a block whose amax is 0 gets scale 0 and q 0.
 * Also returns the per-32 sums of q (the Q4_K sub-block width), needed by
 * the min term.  x is [M][ldx] f32 (ldx >= K); q is [M][K]; scale is
 * [M][K/256]; asum32 is [M][K/32].
 */
int oracle_quantize_act(const float *x, int64_t M, int64_t K, int64_t ldx,
                        int8_t *q, float *scale, int32_t *asum32)
{
    if (K % QK || ldx < K) return -1;
    int64_t nsb = K / QK;
    for (int64_t m = 0; m < M; m++)
        for (int64_t s = 0; s < nsb; s++) {
            const float *xb = x + m * ldx + s * QK;
            int8_t *qb = q + m * K + s * QK;
            float amax = 0.0f;
            for (int i = 0; i < QK; i++) {
                float a = fabsf(xb[i]);
                if (a > amax) amax = a;
            }
            if (amax == 0.0f) {
                scale[m * nsb + s] = 0.0f;
                for (int i = 0; i < QK; i++) qb[i] = 0;
            } else {
                float iscale = 127.0f / amax;
                for (int i = 0; i < QK; i++) {
                    float v = xb[i] * iscale;
                    long r = lrintf(v);             /* current mode: nearest-even */
                    if (r > 127) r = 127;
                    if (r < -127) r = -127;
                    qb[i] = (int8_t)r;
                }
                scale[m * nsb + s] = amax / 127.0f;
            }
            for (int j = 0; j < QK / 32; j++) {
                int32_t t = 0;
                for (int i = 0; i < 32; i++) t += qb[32 * j + i];
                asum32[m * (K / 32) + s * 8 + j] = t;
            }
        }
    return 0;
}

/*
 * RMSNorm (Architecture page, "A forward pass", steps 2 and 4: every layer
 * normalises its attention input and its FFN input, and the final hidden state is
 * normalised before the output projection).  The page names the step but gives no
 * formula or precision.  Reading taken, the usual RMSNorm of both model families:
 * y = x * r * gamma with r = 1 / sqrt(mean over the row of x^2 + eps).  It is
 * evaluated in fp64 and rounded to f32 once, because the f32 activation quantizer
 * consumes y:
 *     ss = sum over the K elements of x_k * x_k   (each square exact in fp64)
 *     r  = 1 / sqrt(ss / K + eps)
 *     y  = f32((x * r) * gamma)
 * ss_scale multiplies ss before use.  It is 1 for the definition.  Tests pass
 * 1 +- delta to bracket the effect of any other summation order: r and y are
 * monotone in ss, because every later step is one correctly rounded operation.
 * x is [M][ldx] (ldx >= K), gamma is [K], y is [M][K].
 */
int oracle_rmsnorm(const float *x, int64_t M, int64_t K, int64_t ldx,
                   const float *gamma, float eps, double ss_scale, float *y)
{
    if (K <= 0 || ldx < K || !(eps >= 0.0f)) return -1;
    for (int64_t m = 0; m < M; m++) {
        const float *xr = x + m * ldx;
        double ss = 0.0;
        for (int64_t k = 0; k < K; k++) ss += (double)xr[k] * (double)xr[k];
        ss *= ss_scale;
        double r = 1.0 / sqrt(ss / (double)K + (double)eps);
        for (int64_t k = 0; k < K; k++)
            y[m * K + k] = (float)(((double)xr[k] * r) * (double)gamma[k]);
    }
    return 0;
}

/*
 * Gated FFN activation (Architecture page, "A forward pass", step 2: the FFN
 * applies SiLU between the gate/up projections and the down projection).  Reading
 * taken, the SwiGLU of both model families: h = SiLU(g) * u with
 * SiLU(g) = g / (1 + e^-g).  Evaluated in fp64 and rounded to f32 once:
 *     h = f32((g / (1 + exp(-g))) * u * h_scale)
 * h_scale is 1 for the definition.  Tests pass 1 +- delta to bracket the last-place
 * differences of another exp.  gate and up are [M][ld] (ld >= K), h is [M][K].
 */
int oracle_swiglu(const float *gate, const float *up, int64_t M, int64_t K, int64_t ld,
                  double h_scale, float *h)
{
    if (K <= 0 || ld < K) return -1;
    for (int64_t m = 0; m < M; m++)
        for (int64_t k = 0; k < K; k++) {
            double g = gate[m * ld + k], u = up[m * ld + k];
            double silu = g / (1.0 + exp(-g));
            h[m * K + k] = (float)(silu * u * h_scale);
        }
    return 0;
}

/* Decoded form of one weight row: all super-blocks, kept as integers. */
typedef struct {
    double *d, *dmin;     /* [nsb] (Q8_0: unused) */
    double *dsub;         /* [nsb][8]: Q8_0 block scales (other types: unused) */
    int32_t *sc, *mn;     /* [nsb][nsub] (mn unused for Q6_K and Q8_0; sc = 1 for Q8_0) */
    int32_t *q;           /* [K]: Q4_K q in [0,15]; Q5_K q in [0,31]; Q6_K (q - 32) in
                             [-32,31]; Q8_0 q in [-128,127] */
} row_t;

static int subblocks(int qtype) { return qtype == 14 ? 16 : 8; }

static void decode_row(int qtype, const uint8_t *wrow, int64_t nsb, row_t *r)
{
    for (int64_t s = 0; s < nsb; s++) {
        uint8_t q[256];
        if (qtype == 12 || qtype == 13) {
            uint8_t sc[8], mn[8];
            if (qtype == 12)
                oracle_q4k_decode(wrow + s * Q4K_BYTES, &r->d[s], &r->dmin[s], sc, mn, q);
            else
                oracle_q5k_decode(wrow + s * Q5K_BYTES, &r->d[s], &r->dmin[s], sc, mn, q);
            for (int j = 0; j < 8; j++) {
                r->sc[s * 8 + j] = sc[j];
                r->mn[s * 8 + j] = mn[j];
            }
            for (int i = 0; i < QK; i++) r->q[s * QK + i] = q[i];
        } else if (qtype == 8) {
            r->d[s] = r->dmin[s] = 0.0;
            for (int b = 0; b < 8; b++) {
                int8_t q8[32];
                oracle_q80_decode(wrow + s * 8 * Q80_BYTES + b * Q80_BYTES, &r->dsub[s * 8 + b], q8);
                r->sc[s * 8 + b] = 1;
                r->mn[s * 8 + b] = 0;
                for (int i = 0; i < 32; i++) r->q[s * QK + 32 * b + i] = q8[i];
            }
        } else {
            int8_t sc[16];
            oracle_q6k_decode(wrow + s * Q6K_BYTES, &r->d[s], sc, q);
            r->dmin[s] = 0.0;
            for (int j = 0; j < 16; j++) r->sc[s * 16 + j] = sc[j];
            for (int i = 0; i < QK; i++) r->q[s * QK + i] = (int32_t)q[i] - 32;
        }
    }
}

/*
 * One output element, the way the method forms it: for every super-block sb
 *   Q4_K:  dot_j  = sum_{i in sub-block j} q_i * a_i        (int32, 32 terms)
 *          asum_j = sum_{i in sub-block j} a_i               (int32)
 *          S      = sum_j sc_j * dot_j,  Smin = sum_j m_j * asum_j   (int64)
 *          acc   += da * (d * S - dmin * Smin)               (fp64)
 *   Q5_K:  as Q4_K, with q in [0,31]
 *   Q6_K:  dot_j  = sum_{i in sub-block j} (q_i - 32) * a_i  (16 terms)
 *          S      = sum_j sc_j * dot_j;  acc += da * d * S
 *   Q8_0:  dot_b  = sum_{i in block b} q_i * a_i (32 terms);  acc += da * sum_b d_b * dot_b
 * T accumulates sum_sb |da| * (|d| * sum_j |sc_j dot_j| + |dmin| * sum_j |m_j asum_j|),
 * the scale of the rounding error any f32 evaluation order can make.
 */
static void one_output(int qtype, const row_t *r, int64_t nsb, const int8_t *a,
                       const float *da, double *acc_out, double *T_out)
{
    int nsub = subblocks(qtype);
    int sub = QK / nsub;
    int has_min = qtype == 12 || qtype == 13;
    double acc = 0.0, T = 0.0;
    for (int64_t s = 0; s < nsb; s++) {
        int64_t S = 0, Smin = 0;
        double Sabs = 0.0, Mabs = 0.0, part8 = 0.0, abs8 = 0.0;
        for (int j = 0; j < nsub; j++) {
            int32_t dot = 0, asum = 0;
            for (int i = 0; i < sub; i++) {
                int64_t k = s * QK + (int64_t)j * sub + i;
                dot += r->q[k] * (int32_t)a[k];
                asum += a[k];
            }
            if (qtype == 8) {
                part8 += r->dsub[s * 8 + j] * (double)dot;
                abs8 += fabs(r->dsub[s * 8 + j] * (double)dot);
                continue;
            }
            int64_t t = (int64_t)r->sc[s * nsub + j] * dot;
            S += t;
            Sabs += fabs((double)t);
            if (has_min) {
                int64_t u = (int64_t)r->mn[s * nsub + j] * asum;
                Smin += u;
                Mabs += fabs((double)u);
            }
        }
        double das = (double)da[s];
        if (qtype == 8) {
            acc += das * part8;
            T += fabs(das) * abs8;
            continue;
        }
        acc += das * (r->d[s] * (double)S - r->dmin[s] * (double)Smin);
        T += fabs(das) * (fabs(r->d[s]) * Sabs + fabs(r->dmin[s]) * Mabs);
    }
    *acc_out = acc;
    *T_out = T;
}

/*
 * out[i][n - n0] for output rows i and weight rows n in [n0, n1):
 *   rows == NULL: i ranges over all M canvas rows (i = m);
 *   otherwise i ranges over n_rows and uses canvas row rows[i]
 *   (Architecture page, "A forward pass", step 4: the output projection
 *   runs on the requested rows only; duplicates allowed).
 * out is f32 [n_out][ldo], out64 / T (nullable) are fp64 with the same shape.
 * w is row-major [N][K/256] GGUF blocks; q is [M][K]; scale is [M][K/256].
 * Returns -1 on a bad argument or an out-of-range row.
 */
int oracle_qgemm(int qtype, const uint8_t *w, int64_t N, int64_t K,
                 const int8_t *q, const float *scale, int64_t M,
                 const int32_t *rows, int64_t n_rows, int64_t n0, int64_t n1,
                 float *out, double *out64, double *T, int64_t ldo, int nthreads)
{
    if (!span_bytes(qtype) || K % QK || n0 < 0 || n1 > N || n0 > n1) return -1;
    int64_t nsb = K / QK;
    int64_t n_out = rows ? n_rows : M;
    if (ldo < n1 - n0) return -1;
    if (rows)
        for (int64_t i = 0; i < n_rows; i++)
            if (rows[i] < 0 || rows[i] >= M) return -1;
    int bb = span_bytes(qtype);
    int nsub = subblocks(qtype);
    if (nthreads <= 0) nthreads = 1;
    (void)nthreads;
#pragma omp parallel num_threads(nthreads)
    {
        row_t r;
        r.d = malloc(sizeof(double) * nsb);
        r.dmin = malloc(sizeof(double) * nsb);
        r.dsub = malloc(sizeof(double) * nsb * 8);
        r.sc = malloc(sizeof(int32_t) * nsb * nsub);
        r.mn = malloc(sizeof(int32_t) * nsb * nsub);
        r.q = malloc(sizeof(int32_t) * K);
#pragma omp for schedule(dynamic, 1)
        for (int64_t n = n0; n < n1; n++) {
            decode_row(qtype, w + n * nsb * bb, nsb, &r);
            for (int64_t i = 0; i < n_out; i++) {
                int64_t m = rows ? rows[i] : i;
                double acc, t;
                one_output(qtype, &r, nsb, q + m * K, scale + m * nsb, &acc, &t);
                out[i * ldo + (n - n0)] = (float)acc;
                if (out64) out64[i * ldo + (n - n0)] = acc;
                if (T) T[i * ldo + (n - n0)] = t;
            }
        }
        free(r.d); free(r.dmin); free(r.dsub); free(r.sc); free(r.mn); free(r.q);
    }
    return 0;
}

/*
 * Integer intermediates, for bit-exact comparison:
 *   dots[m][n][j]  per-sub-block dot products (Q4_K / Q5_K: K/32 of sum q*a;
 *                  Q6_K: K/16 of sum (q-32)*a; Q8_0: K/32 of sum q*a per block)
 *   S[m][n][sb], Smin[m][n][sb]  the per-super-block integer combinations
 *                  (Smin is 0 for Q6_K and Q8_0; for Q8_0, whose blocks carry their
 *                  own f16 scales, S is the plain sum of its eight dots).
 *   Any pointer may be NULL.
 */
int oracle_sb_ints(int qtype, const uint8_t *w, int64_t N, int64_t K,
                   const int8_t *q, int64_t M, int32_t *dots, int64_t *S, int64_t *Smin)
{
    if (!span_bytes(qtype) || K % QK) return -1;
    int64_t nsb = K / QK;
    int nsub = subblocks(qtype);
    int sub = QK / nsub;
    int bb = span_bytes(qtype);
    row_t r;
    r.d = malloc(sizeof(double) * nsb);
    r.dmin = malloc(sizeof(double) * nsb);
    r.dsub = malloc(sizeof(double) * nsb * 8);
    r.sc = malloc(sizeof(int32_t) * nsb * nsub);
    r.mn = malloc(sizeof(int32_t) * nsb * nsub);
    r.q = malloc(sizeof(int32_t) * K);
    for (int64_t n = 0; n < N; n++) {
        decode_row(qtype, w + n * nsb * bb, nsb, &r);
        for (int64_t m = 0; m < M; m++) {
            const int8_t *a = q + m * K;
            for (int64_t s = 0; s < nsb; s++) {
                int64_t Ss = 0, Sm = 0;
                for (int j = 0; j < nsub; j++) {
                    int32_t dot = 0, asum = 0;
                    for (int i = 0; i < sub; i++) {
                        int64_t k = s * QK + (int64_t)j * sub + i;
                        dot += r.q[k] * (int32_t)a[k];
                        asum += a[k];
                    }
                    if (dots) dots[(m * N + n) * (nsb * nsub) + s * nsub + j] = dot;
                    Ss += (int64_t)r.sc[s * nsub + j] * dot;
                    if (qtype == 12 || qtype == 13) Sm += (int64_t)r.mn[s * nsub + j] * asum;
                }
                if (S) S[(m * N + n) * nsb + s] = Ss;
                if (Smin) Smin[(m * N + n) * nsb + s] = Sm;
            }
        }
    }
    free(r.d); free(r.dmin); free(r.dsub); free(r.sc); free(r.mn); free(r.q);
    return 0;
}

/*
 * Bidirectional attention over the canvas (Architecture page, "A forward pass",
 * step 2: attention runs over all L positions with no mask; heatdrop card, "Key
 * highlights": the GPU path runs it as an online-softmax attention on f16 tensor
 * cores).  For query row i and head h, whose key/value head is g = h / (H / Hkv):
 *     o[i][h] = sum_j softmax_j( q[i][h] . k[j][g] / sqrt(dh) ) v[j][g]
 * over every key row j, evaluated in fp64 (the largest logit is subtracted before
 * exp, which leaves softmax unchanged).  q is [Lq][H][dh], k and v are [Lk][Hkv][dh]
 * (f32), o is [Lq][H][dh] (fp64).  Lq < Lk covers the last layer, where only the
 * requested rows continue but attend to the whole canvas.  H must be a multiple of Hkv.
 */
int oracle_attention(const float *q, const float *k, const float *v, int64_t Lq, int64_t Lk,
                     int64_t H, int64_t Hkv, int64_t dh, double *o, int nthreads)
{
    if (Lq <= 0 || Lk <= 0 || H <= 0 || Hkv <= 0 || dh <= 0 || H % Hkv) return -1;
    int64_t group = H / Hkv;
    double scale = 1.0 / sqrt((double)dh);
    if (nthreads <= 0) nthreads = 1;
    (void)nthreads;
#pragma omp parallel num_threads(nthreads)
    {
        double *logit = malloc(sizeof(double) * Lk);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < Lq * H; t++) {
            int64_t i = t / H, h = t % H, g = h / group;
            const float *qi = q + (i * H + h) * dh;
            double mx = -INFINITY;
            for (int64_t j = 0; j < Lk; j++) {
                const float *kj = k + (j * Hkv + g) * dh;
                double dot = 0.0;
                for (int64_t c = 0; c < dh; c++) dot += (double)qi[c] * (double)kj[c];
                logit[j] = dot * scale;
                if (logit[j] > mx) mx = logit[j];
            }
            double den = 0.0;
            for (int64_t j = 0; j < Lk; j++) {
                logit[j] = exp(logit[j] - mx);
                den += logit[j];
            }
            double *oi = o + (i * H + h) * dh;
            for (int64_t c = 0; c < dh; c++) oi[c] = 0.0;
            for (int64_t j = 0; j < Lk; j++) {
                const float *vj = v + (j * Hkv + g) * dh;
                double w = logit[j] / den;
                for (int64_t c = 0; c < dh; c++) oi[c] += w * (double)vj[c];
            }
        }
        free(logit);
    }
    return 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
