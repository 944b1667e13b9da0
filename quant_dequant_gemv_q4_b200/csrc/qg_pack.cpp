// qg_pack.cpp -- host-side format helpers of libqg: tensor sizes and the bit packer
// (fields -> GGML bytes).  The packer places bits only; it does not choose scales.
//
// Q4_K superblock {fp16 d; fp16 dmin; u8 scales[12]; u8 qs[128]} ("HARDWARE GROUND TRUTH: 2x
// NVIDIA Tesla T4 (Kaggle)", "QUANTIZATION MIX").  Scale table, GGML get_scale_min_k4 layout:
//   scales[j]   (j<4): bits 0-5 sc_j, bits 6-7 = bits 4-5 of sc_{j+4}
//   scales[j+4] (j<4): bits 0-5 m_j,  bits 6-7 = bits 4-5 of m_{j+4}
//   scales[j+8] (j<4): bits 0-3 = bits 0-3 of sc_{j+4}, bits 4-7 = bits 0-3 of m_{j+4}
// Nibbles: qs[32c + l] = q[64c + l] | q[64c + 32 + l] << 4.
// Q8_0 block {fp16 d; i8 qs[32]}.
#include <cstdint>
#include <cstring>

#include "../../include/qg.h"

extern "C" {

size_t qg_weight_bytes(int fmt, int64_t N, int64_t K)
{
    if (N < 0 || K < 1) return 0;
    if (fmt == QG_FMT_Q4_K) return (K % 256) ? 0 : (size_t)N * (size_t)(K / 256) * 144u;
    if (fmt == QG_FMT_Q8_0) return (K % 32) ? 0 : (size_t)N * (size_t)(K / 32) * 34u;
    return 0;
}

int qg_pack_reference(int fmt, int64_t N, int64_t K, const uint16_t *d, const uint16_t *dmin,
                      const uint8_t *sc, const uint8_t *m, const void *q, void *out)
{
    if (fmt != QG_FMT_Q4_K && fmt != QG_FMT_Q8_0) return QG_ERR_FMT;
    if (qg_weight_bytes(fmt, N, K) == 0 && N != 0) return QG_ERR_SHAPE;
    if (N < 0) return QG_ERR_SHAPE;
    if (N == 0) return QG_OK;
    if (!d || !q || !out) return QG_ERR_NULL;
    uint8_t *o = static_cast<uint8_t *>(out);
    if (fmt == QG_FMT_Q4_K) {
        if (!dmin || !sc || !m) return QG_ERR_NULL;
        const uint8_t *qq = static_cast<const uint8_t *>(q);
        const int64_t nsb = N * (K / 256);
        for (int64_t s = 0; s < nsb; ++s) {
            uint8_t *blk = o + s * 144;
            const uint8_t *S = sc + 8 * s, *M = m + 8 * s;
            const uint8_t *Q = qq + 256 * s;
            for (int j = 0; j < 8; ++j)
                if (S[j] > 63 || M[j] > 63) return QG_ERR_RANGE;
            for (int i = 0; i < 256; ++i)
                if (Q[i] > 15) return QG_ERR_RANGE;
            blk[0] = (uint8_t)(d[s] & 0xFF);
            blk[1] = (uint8_t)(d[s] >> 8);
            blk[2] = (uint8_t)(dmin[s] & 0xFF);
            blk[3] = (uint8_t)(dmin[s] >> 8);
            for (int j = 0; j < 4; ++j) {
                blk[4 + j] = (uint8_t)(S[j] | ((S[j + 4] >> 4) << 6));
                blk[8 + j] = (uint8_t)(M[j] | ((M[j + 4] >> 4) << 6));
                blk[12 + j] = (uint8_t)((S[j + 4] & 15) | ((M[j + 4] & 15) << 4));
            }
            for (int c = 0; c < 4; ++c)
                for (int l = 0; l < 32; ++l)
                    blk[16 + 32 * c + l] = (uint8_t)(Q[64 * c + l] | (Q[64 * c + 32 + l] << 4));
        }
    } else {
        const int8_t *qq = static_cast<const int8_t *>(q);
        const int64_t nblk = N * (K / 32);
        for (int64_t t = 0; t < nblk; ++t) {
            uint8_t *blk = o + t * 34;
            const int8_t *Q = qq + 32 * t;
            for (int i = 0; i < 32; ++i)
                if (Q[i] == -128) return QG_ERR_RANGE;
            blk[0] = (uint8_t)(d[t] & 0xFF);
            blk[1] = (uint8_t)(d[t] >> 8);
            std::memcpy(blk + 2, Q, 32);
        }
    }
    return QG_OK;
}

}  // extern "C"
