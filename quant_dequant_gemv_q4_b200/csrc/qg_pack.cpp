// qg_pack.cpp -- host-side format helpers of libqg: tensor sizes and the bit packer
// (fields -> GGML bytes).  The packer places bits only; it does not choose scales.
//
// Q4_K superblock {fp16 d; fp16 dmin; u8 scales[12]; u8 qs[128]} ("HARDWARE GROUND TRUTH: 2x
// NVIDIA Tesla T4 (Kaggle)", "QUANTIZATION MIX").  Scale table, GGML get_scale_min_k4 layout:
//   scales[j]   (j<4): bits 0-5 sc_j, bits 6-7 = bits 4-5 of sc_{j+4}
//   scales[j+4] (j<4): bits 0-5 m_j,  bits 6-7 = bits 4-5 of m_{j+4}
//   scales[j+8] (j<4): bits 0-3 = bits 0-3 of sc_{j+4}, bits 4-7 = bits 0-3 of m_{j+4}
// Nibbles: qs[32c + l] = q[64c + l] | q[64c + 32 + l] << 4.
// Q5_K superblock {fp16 d; fp16 dmin; u8 scales[12]; u8 qh[32]; u8 qs[128]}: the Q4_K fields plus
// the fifth bit of q[64c + l] at bit 2c of qh[l] and of q[64c + 32 + l] at bit 2c + 1.
// Q6_K superblock {u8 ql[128]; u8 qh[64]; i8 scales[16]; fp16 d}: in half h (weights 128h ..
// 128h + 127), weight 128h + 32t + l (t = 0..3, l = 0..31) keeps its low nibble in
// ql[64h + 32(t % 2) + l] (bits 0-3 for t < 2, bits 4-7 for t >= 2) and its high two bits at bits
// 2t, 2t + 1 of qh[32h + l].
// Q8_0 block {fp16 d; i8 qs[32]}.
// IQ4_XS superblock {fp16 d; u16 scales_h; u8 scales_l[4]; u8 qs[128]}: the 6-bit scale of
// sub-block j keeps bits 0-3 in nibble j % 2 of scales_l[j / 2] and bits 4-5 at bits 2j, 2j + 1 of
// scales_h; qs[16j + l] = idx[32j + l] | idx[32j + 16 + l] << 4.
#include <cstdint>
#include <cstring>

#include "../../include/qg.h"

namespace {

bool is_kquant(int fmt) { return fmt == QG_FMT_Q4_K || fmt == QG_FMT_Q5_K || fmt == QG_FMT_Q6_K; }

void put_half(uint8_t *p, uint16_t v)
{
    p[0] = (uint8_t)(v & 0xFF);
    p[1] = (uint8_t)(v >> 8);
}

// d, dmin and the scale table of a Q4_K / Q5_K superblock (bytes 0..15); false if out of range
bool pack_q4k_header(uint8_t *blk, uint16_t d, uint16_t dmin, const uint8_t *S, const uint8_t *M)
{
    for (int j = 0; j < 8; ++j)
        if (S[j] > 63 || M[j] > 63) return false;
    put_half(blk, d);
    put_half(blk + 2, dmin);
    for (int j = 0; j < 4; ++j) {
        blk[4 + j] = (uint8_t)(S[j] | ((S[j + 4] >> 4) << 6));
        blk[8 + j] = (uint8_t)(M[j] | ((M[j + 4] >> 4) << 6));
        blk[12 + j] = (uint8_t)((S[j + 4] & 15) | ((M[j + 4] & 15) << 4));
    }
    return true;
}

// the low nibbles of 256 weights into qs[128]
void pack_nibbles(uint8_t *qs, const uint8_t *Q)
{
    for (int c = 0; c < 4; ++c)
        for (int l = 0; l < 32; ++l)
            qs[32 * c + l] = (uint8_t)((Q[64 * c + l] & 15) | ((Q[64 * c + 32 + l] & 15) << 4));
}

}  // namespace

extern "C" {

size_t qg_weight_bytes(int fmt, int64_t N, int64_t K)
{
    if (N < 0 || K < 1) return 0;
    if (fmt == QG_FMT_Q4_K) return (K % 256) ? 0 : (size_t)N * (size_t)(K / 256) * 144u;
    if (fmt == QG_FMT_Q5_K) return (K % 256) ? 0 : (size_t)N * (size_t)(K / 256) * 176u;
    if (fmt == QG_FMT_Q6_K) return (K % 256) ? 0 : (size_t)N * (size_t)(K / 256) * 210u;
    if (fmt == QG_FMT_Q8_0) return (K % 32) ? 0 : (size_t)N * (size_t)(K / 32) * 34u;
    if (fmt == QG_FMT_IQ4_XS) return (K % 256) ? 0 : (size_t)N * (size_t)(K / 256) * 136u;
    return 0;
}

int qg_pack_reference(int fmt, int64_t N, int64_t K, const uint16_t *d, const uint16_t *dmin,
                      const uint8_t *sc, const uint8_t *m, const void *q, void *out)
{
    if (!is_kquant(fmt) && fmt != QG_FMT_Q8_0 && fmt != QG_FMT_IQ4_XS) return QG_ERR_FMT;
    if (qg_weight_bytes(fmt, N, K) == 0 && N != 0) return QG_ERR_SHAPE;
    if (N < 0) return QG_ERR_SHAPE;
    if (N == 0) return QG_OK;
    if (!d || !q || !out) return QG_ERR_NULL;
    uint8_t *o = static_cast<uint8_t *>(out);
    if (fmt == QG_FMT_Q4_K || fmt == QG_FMT_Q5_K) {
        if (!dmin || !sc || !m) return QG_ERR_NULL;
        const bool five = (fmt == QG_FMT_Q5_K);
        const int SB = five ? 176 : 144;
        const uint8_t qmax = five ? 31 : 15;
        const uint8_t *qq = static_cast<const uint8_t *>(q);
        const int64_t nsb = N * (K / 256);
        for (int64_t s = 0; s < nsb; ++s) {
            uint8_t *blk = o + s * SB;
            const uint8_t *Q = qq + 256 * s;
            for (int i = 0; i < 256; ++i)
                if (Q[i] > qmax) return QG_ERR_RANGE;
            if (!pack_q4k_header(blk, d[s], dmin[s], sc + 8 * s, m + 8 * s)) return QG_ERR_RANGE;
            if (five) {
                uint8_t *qh = blk + 16;
                std::memset(qh, 0, 32);
                for (int i = 0; i < 256; ++i) {
                    const int c = i / 64, r = i % 64;
                    qh[r % 32] |= (uint8_t)(((Q[i] >> 4) & 1) << (2 * c + (r >= 32 ? 1 : 0)));
                }
                pack_nibbles(blk + 48, Q);
            } else {
                pack_nibbles(blk + 16, Q);
            }
        }
    } else if (fmt == QG_FMT_Q6_K) {
        if (!sc) return QG_ERR_NULL;
        const uint8_t *qq = static_cast<const uint8_t *>(q);
        const int64_t nsb = N * (K / 256);
        for (int64_t s = 0; s < nsb; ++s) {
            uint8_t *blk = o + s * 210;
            const uint8_t *Q = qq + 256 * s;
            for (int i = 0; i < 256; ++i)
                if (Q[i] > 63) return QG_ERR_RANGE;
            std::memset(blk, 0, 192);
            for (int i = 0; i < 256; ++i) {
                const int h = i / 128, r = i % 128, t = r / 32, l = r % 32;
                uint8_t &lb = blk[64 * h + 32 * (t % 2) + l];
                lb |= (uint8_t)((Q[i] & 15) << (t < 2 ? 0 : 4));
                blk[128 + 32 * h + l] |= (uint8_t)((Q[i] >> 4) << (2 * t));
            }
            std::memcpy(blk + 192, sc + 16 * s, 16);
            put_half(blk + 208, d[s]);
        }
    } else if (fmt == QG_FMT_IQ4_XS) {
        if (!sc) return QG_ERR_NULL;
        const uint8_t *qq = static_cast<const uint8_t *>(q);
        const int64_t nsb = N * (K / 256);
        for (int64_t s = 0; s < nsb; ++s) {
            uint8_t *blk = o + s * 136;
            const uint8_t *Q = qq + 256 * s;
            const uint8_t *L = sc + 8 * s;
            for (int i = 0; i < 256; ++i)
                if (Q[i] > 15) return QG_ERR_RANGE;
            uint16_t scales_h = 0;
            std::memset(blk + 4, 0, 4);
            for (int j = 0; j < 8; ++j) {
                if (L[j] > 63) return QG_ERR_RANGE;
                blk[4 + j / 2] |= (uint8_t)((L[j] & 15) << (4 * (j % 2)));
                scales_h |= (uint16_t)((L[j] >> 4) << (2 * j));
            }
            put_half(blk, d[s]);
            put_half(blk + 2, scales_h);
            for (int j = 0; j < 8; ++j)
                for (int l = 0; l < 16; ++l)
                    blk[8 + 16 * j + l] = (uint8_t)(Q[32 * j + l] | (Q[32 * j + 16 + l] << 4));
        }
    } else {
        const int8_t *qq = static_cast<const int8_t *>(q);
        const int64_t nblk = N * (K / 32);
        for (int64_t t = 0; t < nblk; ++t) {
            uint8_t *blk = o + t * 34;
            const int8_t *Q = qq + 32 * t;
            for (int i = 0; i < 32; ++i)
                if (Q[i] == -128) return QG_ERR_RANGE;
            put_half(blk, d[t]);
            std::memcpy(blk + 2, Q, 32);
        }
    }
    return QG_OK;
}

}  // extern "C"
