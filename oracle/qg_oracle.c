/*
 * qg_oracle.c -- plain, single-threaded CPU oracle for the block-quantized dequant GEMV
 *                y[N,B] = dequant(W[N,K]) . x[K,B].
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this library.  It shares no code, header, table or constant with the
 * CUDA library: it is written directly from the format definitions below and is deliberately
 * slow and literal (no blocking, no fusion, no reordering of the sums).
 *
 * Sources it follows (page title, then section):
 *   [T4 dossier] "HARDWARE GROUND TRUTH: 2x NVIDIA Tesla T4 (Kaggle)", section
 *       "QUANTIZATION MIX": the Q4_K superblock {half d; half dmin; uint8 scales[12];
 *       uint8 qs[128]} of 256 weights in 144 bytes, and the dequantization w = d*(sc*q4) - dmin*m;
 *       section "PHYSICS & CONTRACT": fp32 accumulation for every reduction.
 *   [T4 GEMV prompt] the same dossier's second prompt, section "SPEC": the op
 *       y = dequant(W[N,K]) @ x[K] with a tensor-type flag, diffed against a float reference.
 *   [DP4A issue] "DP4A Q4K/Q6K GEMV profile is catastrophic through the Gated DeltaNet
 *       recurrence ... #3513", Description: the accuracy yardstick is an exact f64 dequantized dot.
 *   GGML's block formats, which the pages name but do not spell out: the Q4_K 6-bit scale/min
 *       packing ("get_scale_min_k4" layout), the Q4_K nibble order, and Q8_0 = {half d; int8 qs[32]}
 *       with w = d*q.  The same dossier's quant mix also lists Q5_K and Q6_K (GGML's K-quants with a
 *       fifth bit per weight, and with 6-bit weights and 16 int8 group scales); their layouts are
 *       written out at orc_q5k_quant and orc_q6k_quant below.  The dossier's second prompt
 *       ("SPEC", "OUTPUT") also names IQ4_XS, GGML's 4-bit format whose indices select values of
 *       a fixed 16-entry non-linear codebook; its layout is written out at orc_iq4xs_index.
 *
 * Definition computed (exact up to the final fp64 summation):
 *   w[n,k]  = the fp32 dequantized weight, computed exactly in fp64 and rounded ONCE to fp32
 *             (round-to-nearest-even).  For Q4_K, d*sc*q and dmin*m have at most 21 and 17
 *             significant bits, and their difference spans at most 50 bits, so the fp64 value is
 *             exact and the single cast is the correctly rounded fp32 weight.  Q5_K is the same
 *             with 5-bit q (d*sc*q at most 22 bits).  Q6_K: d*sc*(q-32) has at most 25 significant
 *             bits, exact in fp64, rounded once.  For Q8_0, d*q is exact in fp32.  IQ4_XS:
 *             d*(ls-32)*v has at most 11 + 5 + 7 = 23 significant bits, exact in fp32.
 *   y[n,b]  = sum_k w[n,k] * x[k,b]    in fp64, k ascending (each product is exact in fp64);
 *   A[n,b]  = sum_k |w[n,k] * x[k,b]|  in fp64, the scale of the error bound
 *             |y_gpu - y| <= 1e-5 * A + 1e-6.
 *
 * Layouts: W is row-major, row n is K/256 consecutive superblocks (144 B Q4_K, 176 B Q5_K,
 * 210 B Q6_K, 136 B IQ4_XS) or K/32 consecutive 34-byte Q8_0 blocks; x is fp16 bits, x[k*B + b]; y and A are
 * y[n*B + b].
 *
 * Build with -ffp-contract=off so that no product is fused into a sum.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Format flags: GGML's type ids for the block formats. */
#define ORC_Q8_0 8
#define ORC_Q4_K 12
#define ORC_Q5_K 13
#define ORC_Q6_K 14
#define ORC_IQ4_XS 23

#define ORC_OK 0
#define ORC_EINVAL 1

/* ---------------------------------------------------------------------------------------------
 * IEEE-754 binary16 -> double, from the definition: 1 sign bit, 5 exponent bits (bias 15),
 * 10 fraction bits; exponent 0 encodes zero and subnormals f * 2^-24; exponent 31 encodes
 * infinity (f == 0) and NaN (f != 0).
 * ------------------------------------------------------------------------------------------- */
double orc_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 31;
    int f = h & 1023;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);
    } else if (e == 31) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(1024 + f), e - 25);
    }
    return sign ? -v : v;
}

/* ---------------------------------------------------------------------------------------------
 * Q4_K scale table (GGML "get_scale_min_k4" layout).  The 12 bytes hold eight 6-bit scales sc_j
 * and eight 6-bit mins m_j:
 *   j < 4 : sc_j = low 6 bits of byte j,   m_j = low 6 bits of byte j+4;
 *   j >= 4: sc_j = low nibble of byte j+4, with bits 4-5 taken from the top two bits of byte j-4;
 *           m_j  = high nibble of byte j+4, with bits 4-5 taken from the top two bits of byte j.
 * ------------------------------------------------------------------------------------------- */
void orc_q4k_scale_min(const uint8_t *scales, int j, int *sc, int *m)
{
    if (j < 4) {
        *sc = scales[j] & 63;
        *m = scales[j + 4] & 63;
    } else {
        int lo_sc = scales[j + 4] & 15;
        int lo_m = scales[j + 4] >> 4;
        int hi_sc = scales[j - 4] >> 6;
        int hi_m = scales[j] >> 6;
        *sc = lo_sc + 16 * hi_sc;
        *m = lo_m + 16 * hi_m;
    }
}

/* Q4_K nibble order: weight i of a superblock lies in 64-weight chunk c = i / 64; with
 * r = i % 64, byte qs[32c + r % 32] holds it in its low nibble when r < 32 and in its high
 * nibble when r >= 32.  Weight i belongs to 32-weight sub-block j = i / 32. */
static int orc_q4k_quant(const uint8_t *qs, int i)
{
    int c = i / 64;
    int r = i % 64;
    uint8_t byte = qs[32 * c + (r % 32)];
    return (r < 32) ? (byte & 15) : (byte >> 4);
}

/* One Q4_K superblock (144 bytes) -> 256 fp32 weights. */
static void orc_dequant_q4k_block(const uint8_t *blk, float *w)
{
    double d = orc_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
    double dmin = orc_half_to_double((uint16_t)(blk[2] | (blk[3] << 8)));
    const uint8_t *scales = blk + 4;
    const uint8_t *qs = blk + 16;
    for (int i = 0; i < 256; ++i) {
        int sc, m;
        orc_q4k_scale_min(scales, i / 32, &sc, &m);
        int q = orc_q4k_quant(qs, i);
        double exact = d * (double)sc * (double)q - dmin * (double)m;
        w[i] = (float)exact;
    }
}

/* Q5_K: the Q4_K superblock with a fifth bit per weight.  176 bytes: fp16 d (0-1), fp16 dmin
 * (2-3), the Q4_K scale table (4-15), qh[32] (16-47), qs[128] (48-175).  The low four bits of
 * weight i are its Q4_K nibble in qs; with c = i / 64 and r = i % 64, its fifth bit is bit 2c
 * (r < 32) or bit 2c + 1 (r >= 32) of qh[r % 32].  w = d * sc_j * q - dmin * m_j, q in 0..31
 * (d*sc*q has at most 22 significant bits: exact in fp64, rounded once to fp32). */
static int orc_q5k_quant(const uint8_t *qh, const uint8_t *qs, int i)
{
    int c = i / 64;
    int r = i % 64;
    int bit = (qh[r % 32] >> (2 * c + (r >= 32 ? 1 : 0))) & 1;
    return orc_q4k_quant(qs, i) + 16 * bit;
}

static void orc_dequant_q5k_block(const uint8_t *blk, float *w)
{
    double d = orc_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
    double dmin = orc_half_to_double((uint16_t)(blk[2] | (blk[3] << 8)));
    const uint8_t *scales = blk + 4;
    const uint8_t *qh = blk + 16;
    const uint8_t *qs = blk + 48;
    for (int i = 0; i < 256; ++i) {
        int sc, m;
        orc_q4k_scale_min(scales, i / 32, &sc, &m);
        int q = orc_q5k_quant(qh, qs, i);
        double exact = d * (double)sc * (double)q - dmin * (double)m;
        w[i] = (float)exact;
    }
}

/* Q6_K: 256 weights in 210 bytes: ql[128] (0-127), qh[64] (128-191), int8 scales[16]
 * (192-207), fp16 d (208-209).  The superblock is two halves of 128 weights; in half n, with
 * r = i % 128, k = r / 32 and l = r % 32, weight i takes
 *   its low four bits from ql[64n + l + 32 (k % 2)]: the low nibble for k < 2, the high for k >= 2,
 *   its high two bits from bits 2k, 2k+1 of qh[32n + l],
 * and w = d * scales[i / 16] * (q - 32), q in 0..63 (a signed 6-bit value; the product has up to
 * 25 significant bits: exact in fp64, rounded once to fp32). */
static int orc_q6k_quant(const uint8_t *ql, const uint8_t *qh, int i)
{
    int n = i / 128;
    int r = i % 128;
    int k = r / 32;
    int l = r % 32;
    uint8_t lb = ql[64 * n + l + 32 * (k % 2)];
    int low = (k < 2) ? (lb & 15) : (lb >> 4);
    int high = (qh[32 * n + l] >> (2 * k)) & 3;
    return low + 16 * high - 32;
}

static void orc_dequant_q6k_block(const uint8_t *blk, float *w)
{
    const uint8_t *ql = blk;
    const uint8_t *qh = blk + 128;
    const int8_t *scales = (const int8_t *)(blk + 192);
    double d = orc_half_to_double((uint16_t)(blk[208] | (blk[209] << 8)));
    for (int i = 0; i < 256; ++i) {
        int q = orc_q6k_quant(ql, qh, i);
        double exact = d * (double)scales[i / 16] * (double)q;
        w[i] = (float)exact;
    }
}

/* IQ4_XS: 256 weights in 136 bytes: fp16 d (0-1), a little-endian uint16 scales_h (2-3),
 * scales_l[4] (4-7), qs[128] (8-135).  Sub-block j (32 weights, j = 0..7) has the 6-bit scale
 *   ls_j = (nibble j % 2 of scales_l[j / 2]: the low nibble for even j, the high for odd j)
 *          + 16 * (bits 2j, 2j+1 of scales_h),
 * and weight i of sub-block j = i / 32, with r = i % 32, has the 4-bit index held by
 * qs[16j + r % 16]: its low nibble for r < 16, its high nibble for r >= 16.  The index selects
 * one of sixteen fixed integer levels (the codebook below, spaced more finely near zero), and
 *   w = d * (ls_j - 32) * codebook[index],
 * at most 23 significant bits: exact in fp32. */
static const int orc_iq4_levels[16] = {-127, -104, -83, -65, -49, -35, -22, -10,
                                       1,    13,   25,  38,  53,  69,  89,  113};

static int orc_iq4xs_scale(const uint8_t *blk, int j)
{
    int scales_h = blk[2] | (blk[3] << 8);
    int low = (blk[4 + j / 2] >> (4 * (j % 2))) & 15;
    int high = (scales_h >> (2 * j)) & 3;
    return low + 16 * high;
}

static int orc_iq4xs_index(const uint8_t *qs, int i)
{
    int j = i / 32;
    int r = i % 32;
    uint8_t byte = qs[16 * j + (r % 16)];
    return (r < 16) ? (byte & 15) : (byte >> 4);
}

static void orc_dequant_iq4xs_block(const uint8_t *blk, float *w)
{
    double d = orc_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
    const uint8_t *qs = blk + 8;
    for (int i = 0; i < 256; ++i) {
        int ls = orc_iq4xs_scale(blk, i / 32);
        int v = orc_iq4_levels[orc_iq4xs_index(qs, i)];
        double exact = d * (double)(ls - 32) * (double)v;
        w[i] = (float)exact;
    }
}

/* One Q8_0 block (34 bytes) -> 32 fp32 weights, w = d * q. */
static void orc_dequant_q8_0_block(const uint8_t *blk, float *w)
{
    double d = orc_half_to_double((uint16_t)(blk[0] | (blk[1] << 8)));
    for (int i = 0; i < 32; ++i) {
        int q = (int)(int8_t)blk[2 + i];
        w[i] = (float)(d * (double)q);
    }
}

static int orc_block_geometry(int fmt, int64_t K, int64_t *block_w, int64_t *block_b)
{
    if (fmt == ORC_Q4_K) {
        *block_w = 256;
        *block_b = 144;
    } else if (fmt == ORC_Q8_0) {
        *block_w = 32;
        *block_b = 34;
    } else if (fmt == ORC_Q5_K) {
        *block_w = 256;
        *block_b = 176;
    } else if (fmt == ORC_Q6_K) {
        *block_w = 256;
        *block_b = 210;
    } else if (fmt == ORC_IQ4_XS) {
        *block_w = 256;
        *block_b = 136;
    } else {
        return ORC_EINVAL;
    }
    if (K <= 0 || K % *block_w != 0) return ORC_EINVAL;
    return ORC_OK;
}

/* Bytes of an N x K tensor in the given format (0 if the arguments are invalid). */
int64_t orc_weight_bytes(int fmt, int64_t N, int64_t K)
{
    int64_t bw, bb;
    if (N < 0 || orc_block_geometry(fmt, K, &bw, &bb) != ORC_OK) return 0;
    return N * (K / bw) * bb;
}

/* Dequantize row n of W into w[K]. */
static void orc_dequant_row(int fmt, const uint8_t *W, int64_t n, int64_t K, float *w)
{
    int64_t bw, bb;
    orc_block_geometry(fmt, K, &bw, &bb);
    int64_t nblk = K / bw;
    const uint8_t *row = W + n * nblk * bb;
    for (int64_t t = 0; t < nblk; ++t) {
        if (fmt == ORC_Q4_K)
            orc_dequant_q4k_block(row + t * bb, w + t * bw);
        else if (fmt == ORC_Q5_K)
            orc_dequant_q5k_block(row + t * bb, w + t * bw);
        else if (fmt == ORC_Q6_K)
            orc_dequant_q6k_block(row + t * bb, w + t * bw);
        else if (fmt == ORC_IQ4_XS)
            orc_dequant_iq4xs_block(row + t * bb, w + t * bw);
        else
            orc_dequant_q8_0_block(row + t * bb, w + t * bw);
    }
}

/* Full dequantization: out[n*K + k] = w[n,k] (fp32). */
int orc_dequant(int fmt, const uint8_t *W, int64_t N, int64_t K, float *out)
{
    int64_t bw, bb;
    if (!W || !out || N < 0 || orc_block_geometry(fmt, K, &bw, &bb) != ORC_OK) return ORC_EINVAL;
    for (int64_t n = 0; n < N; ++n) orc_dequant_row(fmt, W, n, K, out + n * K);
    return ORC_OK;
}

/* y and A for the listed rows: y[r*B + b], A[r*B + b] for r = 0..nrows-1 refer to row rows[r]. */
int orc_gemv_rows(int fmt, const uint8_t *W, int64_t N, int64_t K, const uint16_t *x, int B,
                  const int64_t *rows, int64_t nrows, double *y, double *A)
{
    int64_t bw, bb;
    if (!W || !x || !rows || !y || !A || N < 0 || B < 1) return ORC_EINVAL;
    if (orc_block_geometry(fmt, K, &bw, &bb) != ORC_OK) return ORC_EINVAL;
    float *w = (float *)malloc((size_t)K * sizeof(float));
    double *xd = (double *)malloc((size_t)K * (size_t)B * sizeof(double));
    if (!w || !xd) {
        free(w);
        free(xd);
        return ORC_EINVAL;
    }
    for (int64_t i = 0; i < K * B; ++i) xd[i] = orc_half_to_double(x[i]);
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t n = rows[r];
        if (n < 0 || n >= N) {
            free(w);
            free(xd);
            return ORC_EINVAL;
        }
        orc_dequant_row(fmt, W, n, K, w);
        for (int b = 0; b < B; ++b) {
            double acc = 0.0, mag = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = (double)w[k] * xd[k * B + b];
                acc += p;
                mag += fabs(p);
            }
            y[r * B + b] = acc;
            A[r * B + b] = mag;
        }
    }
    free(w);
    free(xd);
    return ORC_OK;
}

/* All rows: y[n*B + b], A[n*B + b]. */
int orc_gemv(int fmt, const uint8_t *W, int64_t N, int64_t K, const uint16_t *x, int B,
             double *y, double *A)
{
    if (N < 0) return ORC_EINVAL;
    int64_t *rows = (int64_t *)malloc((size_t)(N > 0 ? N : 1) * sizeof(int64_t));
    if (!rows) return ORC_EINVAL;
    for (int64_t n = 0; n < N; ++n) rows[n] = n;
    int rc = orc_gemv_rows(fmt, W, N, K, x, B, rows, N, y, A);
    free(rows);
    return rc;
}

/* Field view of Q4_K superblocks (for checking a packer): for superblock s,
 * d[s], dmin[s] (fp16 bits), sc[8s + j], m[8s + j], q[256s + i]. */
int orc_unpack_q4k(const uint8_t *W, int64_t nsb, uint16_t *d, uint16_t *dmin, uint8_t *sc,
                   uint8_t *m, uint8_t *q)
{
    if (!W || !d || !dmin || !sc || !m || !q || nsb < 0) return ORC_EINVAL;
    for (int64_t s = 0; s < nsb; ++s) {
        const uint8_t *blk = W + s * 144;
        d[s] = (uint16_t)(blk[0] | (blk[1] << 8));
        dmin[s] = (uint16_t)(blk[2] | (blk[3] << 8));
        for (int j = 0; j < 8; ++j) {
            int a, b;
            orc_q4k_scale_min(blk + 4, j, &a, &b);
            sc[8 * s + j] = (uint8_t)a;
            m[8 * s + j] = (uint8_t)b;
        }
        for (int i = 0; i < 256; ++i) q[256 * s + i] = (uint8_t)orc_q4k_quant(blk + 16, i);
    }
    return ORC_OK;
}

/* Field view of Q8_0 blocks: d[t] (fp16 bits), q[32t + i]. */
int orc_unpack_q8_0(const uint8_t *W, int64_t nblk, uint16_t *d, int8_t *q)
{
    if (!W || !d || !q || nblk < 0) return ORC_EINVAL;
    for (int64_t t = 0; t < nblk; ++t) {
        const uint8_t *blk = W + t * 34;
        d[t] = (uint16_t)(blk[0] | (blk[1] << 8));
        for (int i = 0; i < 32; ++i) q[32 * t + i] = (int8_t)blk[2 + i];
    }
    return ORC_OK;
}

/* Field view of Q5_K superblocks: as orc_unpack_q4k, with q[256s + i] in 0..31. */
int orc_unpack_q5k(const uint8_t *W, int64_t nsb, uint16_t *d, uint16_t *dmin, uint8_t *sc,
                   uint8_t *m, uint8_t *q)
{
    if (!W || !d || !dmin || !sc || !m || !q || nsb < 0) return ORC_EINVAL;
    for (int64_t s = 0; s < nsb; ++s) {
        const uint8_t *blk = W + s * 176;
        d[s] = (uint16_t)(blk[0] | (blk[1] << 8));
        dmin[s] = (uint16_t)(blk[2] | (blk[3] << 8));
        for (int j = 0; j < 8; ++j) {
            int a, b;
            orc_q4k_scale_min(blk + 4, j, &a, &b);
            sc[8 * s + j] = (uint8_t)a;
            m[8 * s + j] = (uint8_t)b;
        }
        for (int i = 0; i < 256; ++i) q[256 * s + i] = (uint8_t)orc_q5k_quant(blk + 16, blk + 48, i);
    }
    return ORC_OK;
}

/* Field view of Q6_K superblocks: d[s] (fp16 bits), scales[16s + t] (int8), q[256s + i] in
 * -32..31 (the stored 6-bit value minus 32). */
int orc_unpack_q6k(const uint8_t *W, int64_t nsb, uint16_t *d, int8_t *scales, int8_t *q)
{
    if (!W || !d || !scales || !q || nsb < 0) return ORC_EINVAL;
    for (int64_t s = 0; s < nsb; ++s) {
        const uint8_t *blk = W + s * 210;
        d[s] = (uint16_t)(blk[208] | (blk[209] << 8));
        for (int t = 0; t < 16; ++t) scales[16 * s + t] = (int8_t)blk[192 + t];
        for (int i = 0; i < 256; ++i) q[256 * s + i] = (int8_t)orc_q6k_quant(blk, blk + 128, i);
    }
    return ORC_OK;
}

/* Field view of IQ4_XS superblocks: d[s] (fp16 bits), ls[8s + j] (6-bit sub-block scales, the
 * stored value: the multiplier is ls - 32), idx[256s + i] (codebook indices 0..15). */
int orc_unpack_iq4xs(const uint8_t *W, int64_t nsb, uint16_t *d, uint8_t *ls, uint8_t *idx)
{
    if (!W || !d || !ls || !idx || nsb < 0) return ORC_EINVAL;
    for (int64_t s = 0; s < nsb; ++s) {
        const uint8_t *blk = W + s * 136;
        d[s] = (uint16_t)(blk[0] | (blk[1] << 8));
        for (int j = 0; j < 8; ++j) ls[8 * s + j] = (uint8_t)orc_iq4xs_scale(blk, j);
        for (int i = 0; i < 256; ++i) idx[256 * s + i] = (uint8_t)orc_iq4xs_index(blk + 8, i);
    }
    return ORC_OK;
}

/* The codebook level of index v (0..15), for checking it against the format's printed table. */
int orc_iq4_level(int v) { return (v >= 0 && v < 16) ? orc_iq4_levels[v] : 0; }
