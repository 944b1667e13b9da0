// qg_rows.cuh -- the default streaming GEMV kernel of libqg (sm_100a): one row per lane.
//
// Operation (HARDWARE GROUND TRUTH: 2x NVIDIA Tesla T4 (Kaggle), second prompt, "SPEC"):
//   y[n,b] = sum_k dequant(W)[n,k] * x[k,b] with the format chosen by a flag, fp32 accumulation
//   ("PHYSICS & CONTRACT"), Q4_K w = d*sc*q - dmin*m ("QUANTIZATION MIX"), Q8_0 w = d*q; the
//   dossier's mix also holds Q5_K (5-bit q) and Q6_K (w = d*sc*(q - 32), 16-weight scale groups).
//
// Mapping.  CTA c of K slice s owns a band of consecutive rows [R0, R1) and the slice's units.
// Its warps take (row group, K part) pairs: a row group is 32 consecutive rows of the band, a K
// part every P-th of the slice's 256-weight units.  Lane l of a warp owns row 32g + l of its
// group and decodes that row's whole unit per step, so the scale/min table is decoded once per
// 256 weights with SWAR masks and every x read is a broadcast (all lanes read the same unit of
// x).  One 2-D TMA tensor copy (cp.async.bulk.tensor.2d) per step brings 32 rows x one unit (144 B
// Q4_K, 176 B Q5_K, 272 B Q8_0: odd multiples of 16 B, so 8 consecutive lanes reading 16 B from
// 8 rows hit 8 different bank groups) into the warp's double-buffered ring; Q6_K rows (210 B per
// unit) take one bulk copy per lane.  When all warps are done, the K parts of each row are added
// in shared memory in part order and the band's rows are written once: no atomics (with S > 1
// slices, each slice writes partial rows and the band's last CTA adds them in slice order).
//
// Arithmetic (factored form).  With D_j = d*sc_j and M_j = dmin*m_j (both exact in fp32),
//   sum_i w_i x_i = sum_j [ D_j * sum_{i in j} q_i x_i  -  M_j * sum_{i in j} x_i ].
// The inner sums use fp16 "subnormal nibbles": (word & 0x000F000F) read as two fp16 values is
// exactly (q_a * 2^-24, q_b * 2^-24) (a nibble at bits 4-7 of a half gives q * 2^-20), one logic
// instruction per two weights; fma.rn.f32.f16 multiplies such a half by the fp16 x exactly and
// adds it to an fp32 accumulator.  The x sums per sub-block are computed once per CTA.  Q8_0
// converts its int8 pairs to exact fp16 integers (1152 + q, minus 1152) and uses the same FMA.
#pragma once

#include <cuda.h>

#include "qg_device.cuh"

namespace qg {

// Per-format geometry of a step (32 rows x one 256-weight unit):
//   kUnitBytes  bytes of a unit in W
//   kLaneBytes  ring bytes per lane (row): the unit itself, or for Q6_K a 16-byte aligned window
//               around it (see rows_issue_lanes)
//   kGroups     x-sum groups per unit (sub-blocks of 32 weights; Q6_K: scale groups of 16)
//   kHiOff      the weights of a byte's high nibble sit kHiOff after those of its low nibble
//   kPerLane    false: one 2-D tensor copy per step; true: one bulk copy per lane
//   kWinBytes   per-lane copies: bytes of the 16-byte aligned window copied around a unit
template <int FMT> struct RowsFmt;
template <> struct RowsFmt<kFmtQ4_K> {
    static constexpr int kUnitBytes = 144, kLaneBytes = 144, kGroups = 8, kHiOff = 32;
    static constexpr bool kPerLane = false;
    static constexpr int kWinBytes = 0;
};
template <> struct RowsFmt<kFmtQ8_0> {
    static constexpr int kUnitBytes = 272, kLaneBytes = 272, kGroups = 8, kHiOff = 32;
    static constexpr bool kPerLane = false;
    static constexpr int kWinBytes = 0;
};
template <> struct RowsFmt<kFmtQ5_K> {
    static constexpr int kUnitBytes = 176, kLaneBytes = 176, kGroups = 8, kHiOff = 32;
    static constexpr bool kPerLane = false;
    static constexpr int kWinBytes = 0;
};
// Q6_K: a 210-byte unit starts 0..14 bytes (even) past a 16-byte boundary: a 224-byte window,
// in a 240-byte slot (the consumer's funnel shifts read one word past the window)
template <> struct RowsFmt<kFmtQ6_K> {
    static constexpr int kUnitBytes = 210, kLaneBytes = 240, kGroups = 16, kHiOff = 64;
    static constexpr bool kPerLane = true;
    static constexpr int kWinBytes = 224;
};
// IQ4_XS: a 136-byte unit starts 0 or 8 bytes past a 16-byte boundary: a 144-byte window.  A
// byte of qs holds weights r and r + 16 of its 32-weight sub-block.
template <> struct RowsFmt<kFmtIQ4_XS> {
    static constexpr int kUnitBytes = 136, kLaneBytes = 144, kGroups = 8, kHiOff = 16;
    static constexpr bool kPerLane = true;
    static constexpr int kWinBytes = 144;
};

// First of the four weights whose x the staging stores at chunk c, word i of a unit: the weights
// of the low nibbles of qs word i of chunk c (Q4_K, Q5_K, Q8_0: 64c + 4i; Q6_K, whose chunk
// c = 2h + p is ql[64h + 32p .. 64h + 32p + 31]: 128h + 32p + 4i; IQ4_XS, whose chunk c is the
// 32 qs bytes of sub-blocks 2c and 2c + 1: 32 (2c + i / 4) + 4 (i % 4)).
template <int FMT>
__device__ __forceinline__ int rows_x_lo(int c, int i)
{
    return (FMT == kFmtQ6_K)     ? 128 * (c >> 1) + 32 * (c & 1) + 4 * i
           : (FMT == kFmtIQ4_XS) ? 64 * c + 32 * (i >> 2) + 4 * (i & 3)
                                 : 64 * c + 4 * i;
}

// warps per CTA: as many as the shared-memory budget allows next to x
template <int FMT, int BP> struct RowsWarps {
    static constexpr int value = (FMT == kFmtQ4_K || FMT == kFmtQ5_K || FMT == kFmtIQ4_XS)
                                     ? (BP >= 8 ? 12 : 16)
                                 : (FMT == kFmtQ6_K)                  ? (BP >= 4 ? 8 : 12)
                                                                      : (BP >= 4 ? 6 : 8);
};

constexpr int kRowsStages = 2;  // ring stages per warp (double buffering)
// Ring stages issued before the wait for the previous kernel; the rest are issued once the whole
// CTA's x is staged (after the barrier), or, for Q8_0, once this warp's own x has arrived.  A
// deeper prefetch at entry queues more weight data on the SM's return path ahead of x, and x then
// arrives later (measured: 1 of 2 stages early is 0.6-0.9 us faster per call than 2 of 2, and
// than any order that issues the second stage before x is in).  Refills issued by the warps whose
// x came in first likewise delay the x of the others: waiting for the barrier saves 0.3-0.45 us
// per call on the Q4_K, Q5_K and IQ4_XS FFN and attention shapes, while Q8_0 (272-byte units)
// measured 0.2 us faster with each warp refilling as soon as its own x is in.
constexpr int kPreStages = 1;
template <int FMT> struct RowsRefillAfterBarrier {
    static constexpr bool value = FMT != kFmtQ8_0;
};

struct RowsArgs {
    const uint16_t *x;  // fp16 bits [K][B]
    float *out;         // y [N][B] when S == 1, else per-slice partial rows [S][N][B]
    float *y;           // y [N][B] (the split-K result when S > 1)
    unsigned *cnt;      // S > 1: arrival counter per row band, zero between calls
    int *err;           // device error word
    int64_t N;
    int B;
    int UPR;         // units per row
    int US;          // units per slice (last slice may be shorter)
    int S;           // slices
    int Gs;          // CTAs per slice (row bands)
    int red_floats;  // floats of the per-CTA partial-row buffer
    int act;  // gate/up pair (MATS == 2): 1 writes h = silu(gate) * up
    const float *res;  // MATS == 1: y = W x + res (fp32 [N][B], may alias y), or nullptr
    const uint8_t *w[2];  // per-lane copies (Q6_K): the weight tensors (16-byte aligned)
    int64_t wend;         // per-lane copies: the tensor's byte size rounded down to 16
    int wtail;            // per-lane copies: 1 if the byte size is not a multiple of 16
    int tmap;             // a per-lane format whose rows are 16-byte multiples (IQ4_XS with an even
                          // number of superblocks per row): the weight maps are valid, one 2-D copy
                          // per step as for the other formats
};

// silu(v) * u, the FFN activation of the gate/up pair (silu(v) = v / (1 + e^-v))
__device__ __forceinline__ float silu_mul(float v, float u) { return v / (1.0f + expf(-v)) * u; }

// acc += lo(q)*lo(x) + hi(q)*hi(x), halves of q and x as fp16, products exact, sums fp32
__device__ __forceinline__ void mfma2(float &acc, uint32_t q, uint32_t x)
{
    asm("{\n\t.reg .f16 a0, a1, b0, b1;\n\t"
        "mov.b32 {a0, a1}, %1;\n\t"
        "mov.b32 {b0, b1}, %2;\n\t"
        "fma.rn.f32.f16 %0, a0, b0, %0;\n\t"
        "fma.rn.f32.f16 %0, a1, b1, %0;\n\t}"
        : "+f"(acc)
        : "r"(q), "r"(x));
}

// fp16x2 a - b on raw bits (both operands exact small integers here, so the result is exact)
__device__ __forceinline__ uint32_t hsub2_bits(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// x staging.  For unit j of the slice, column b, 64-weight chunk c and word i, one 16-byte chunk
// holds the 8 halves
//   x[e], x[e+2], x[e+1], x[e+3], x[32+e], x[32+e+2], x[32+e+1], x[32+e+3]   (e = 256j + 64c + 4i)
// i.e. the weights of qs word i of chunk c in the order its nibble pairs come out.  All lanes of
// a warp read the same chunk (a broadcast).  Offset in halves:
template <int BP>
__device__ __forceinline__ int rows_x_off(int US, int j, int c, int i, int b)
{
    (void)US;
    return (((j * 4 + c) * 8 + i) * BP + b) * 8;
}
// x sums per group (G groups per unit: 32-weight sub-blocks, or Q6_K's 16-weight scale groups):
// xsum[(j * G + g) * BP + b]
template <int BP, int G = 8>
__device__ __forceinline__ int rows_xsum_off(int US, int j, int sub, int b)
{
    (void)US;
    return (j * G + sub) * BP + b;
}

template <int BP, int FMT = kFmtQ4_K>
__device__ __forceinline__ void rows_stage_x(const RowsArgs &a, int s, int US_s, __half *xs,
                                             float *xsum)
{
    constexpr int HI = RowsFmt<FMT>::kHiOff;
    constexpr int G = RowsFmt<FMT>::kGroups;
    const int US = a.US;
    const int64_t kbase = (int64_t)s * US * 256;
    const uint16_t *xsl = a.x + kbase * a.B;
    // thread t stages word i = t % 8 of chunk (j, c) for column b; the 8 words of one chunk are 8
    // consecutive lanes, which then add their halves into the chunk's two sub-block sums
    const int nchunk = 32 * BP * US;  // a multiple of 32: every lane of a warp takes part
    const bool vec = (BP == 1) && ((reinterpret_cast<uintptr_t>(xsl) & 7) == 0);
    // x[e0 .. e0+3], x[e0+HI .. e0+HI+3] of chunk t in natural order (zero past the slice)
    auto load = [&](int t, uint32_t (&h)[8]) {
        const int i = t & 7;
        const int jcb = t >> 3;
        const int b = jcb % BP;
        const int jc = jcb / BP;
        const int c = jc & 3, j = jc >> 2;
        if (j < US_s && b < a.B) {
            const int e0 = j * 256 + rows_x_lo<FMT>(c, i);
            if (vec) {
                const uint2 lo = *reinterpret_cast<const uint2 *>(xsl + e0);
                const uint2 hi = *reinterpret_cast<const uint2 *>(xsl + e0 + HI);
                h[0] = lo.x & 0xFFFFu; h[1] = lo.x >> 16; h[2] = lo.y & 0xFFFFu; h[3] = lo.y >> 16;
                h[4] = hi.x & 0xFFFFu; h[5] = hi.x >> 16; h[6] = hi.y & 0xFFFFu; h[7] = hi.y >> 16;
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    h[q] = xsl[(int64_t)(e0 + q) * a.B + b];
                    h[4 + q] = xsl[(int64_t)(e0 + HI + q) * a.B + b];
                }
            }
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) h[q] = 0;
        }
    };
    // chunk t into shared memory, and its group sums (all 32 lanes of the warp together)
    auto store = [&](int t, const uint32_t (&h)[8]) {
        const int i = t & 7;
        const int jcb = t >> 3;
        const int b = jcb % BP;
        const int jc = jcb / BP;
        const int c = jc & 3, j = jc >> 2;
        uint4 v;
        if (FMT == kFmtIQ4_XS) {  // pair order (e, e+16), (e+1, e+17), (e+2, e+18), (e+3, e+19)
            v.x = h[0] | (h[4] << 16);
            v.y = h[1] | (h[5] << 16);
            v.z = h[2] | (h[6] << 16);
            v.w = h[3] | (h[7] << 16);
        } else {  // group order (e, e+2, e+1, e+3)
            v.x = h[0] | (h[2] << 16);
            v.y = h[1] | (h[3] << 16);
            v.z = h[4] | (h[6] << 16);
            v.w = h[5] | (h[7] << 16);
        }
        *reinterpret_cast<uint4 *>(xs + rows_x_off<BP>(US, j, c, i, b)) = v;
        // sub-block sums of the chunk: low half (sub-block 2c) and high half (2c+1), fp32, the
        // same xor-butterfly order on every lane
        float lo = (__half2float(__ushort_as_half((unsigned short)h[0])) +
                    __half2float(__ushort_as_half((unsigned short)h[1]))) +
                   (__half2float(__ushort_as_half((unsigned short)h[2])) +
                    __half2float(__ushort_as_half((unsigned short)h[3])));
        float hi = (__half2float(__ushort_as_half((unsigned short)h[4])) +
                    __half2float(__ushort_as_half((unsigned short)h[5]))) +
                   (__half2float(__ushort_as_half((unsigned short)h[6])) +
                    __half2float(__ushort_as_half((unsigned short)h[7])));
        if (FMT == kFmtIQ4_XS) {
            // all eight halves lie in sub-block 2c + i / 4: the four words of each sub-block
            float t = lo + hi;
#pragma unroll
            for (int off = 1; off < 4; off <<= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
            if ((i & 3) == 0) xsum[rows_xsum_off<BP, G>(US, j, 2 * c + (i >> 2), b)] = t;
        } else if (G == 8) {
            // 32-weight sub-blocks 2c (low nibbles) and 2c + 1: all 8 words of the chunk
#pragma unroll
            for (int off = 1; off < 8; off <<= 1) {
                lo += __shfl_xor_sync(0xffffffffu, lo, off);
                hi += __shfl_xor_sync(0xffffffffu, hi, off);
            }
            if (i == 0) {
                xsum[rows_xsum_off<BP, G>(US, j, 2 * c, b)] = lo;
                xsum[rows_xsum_off<BP, G>(US, j, 2 * c + 1, b)] = hi;
            }
        } else {
            // Q6_K: 16-weight groups, words 0-3 and 4-7 of the chunk; the low nibbles of chunk
            // c = 2h + p are group 8h + 2p (+1 for words 4-7), the high nibbles 4 groups later
#pragma unroll
            for (int off = 1; off < 4; off <<= 1) {
                lo += __shfl_xor_sync(0xffffffffu, lo, off);
                hi += __shfl_xor_sync(0xffffffffu, hi, off);
            }
            if ((i & 3) == 0) {
                const int g = 8 * (c >> 1) + 2 * (c & 1) + (i >> 2);
                xsum[rows_xsum_off<BP, G>(US, j, g, b)] = lo;
                xsum[rows_xsum_off<BP, G>(US, j, g + 4, b)] = hi;
            }
        }
    };
    // two chunks per pass where a thread has two: both loads go out before either is used, so
    // the pass waits for one round trip to L2 rather than two (the condition is uniform per warp:
    // nchunk and blockDim.x are multiples of 32)
    const int nthr = blockDim.x;
    int t = threadIdx.x;
    for (; t + nthr < nchunk; t += 2 * nthr) {
        uint32_t ha[8], hb[8];
        load(t, ha);
        load(t + nthr, hb);
        store(t, ha);
        store(t + nthr, hb);
    }
    for (; t < nchunk; t += nthr) {
        uint32_t h[8];
        load(t, h);
        store(t, h);
    }
}

// One Q4_K superblock against x (unit j of the slice): v[b] = sum over its 256 weights of w*x.
template <int BP>
__device__ __forceinline__ void rows_q4k(const uint8_t *u, const __half *xs, const float *xsum,
                                         int US, int j, float (&v)[BP])
{
    const uint4 hdr = *reinterpret_cast<const uint4 *>(u);
    // GGML get_scale_min_k4 table, all eight (sc, m) at once (byte k of each word = sub-block k or
    // k+4): sc0..3 / m0..3 are the low 6 bits of bytes 0..3 / 4..7; sc4..7 / m4..7 take their low
    // nibbles from bytes 8..11 and bits 4-5 from the top bits of bytes 0..3 / 4..7.
    const uint32_t SC_lo = hdr.y & 0x3F3F3F3Fu;
    const uint32_t MM_lo = hdr.z & 0x3F3F3F3Fu;
    const uint32_t SC_hi = (hdr.w & 0x0F0F0F0Fu) | ((hdr.y >> 2) & 0x30303030u);
    const uint32_t MM_hi = ((hdr.w >> 4) & 0x0F0F0F0Fu) | ((hdr.z >> 2) & 0x30303030u);
    __half2 dd;
    *reinterpret_cast<uint32_t *>(&dd) = hdr.x;
    const float2 dm = __half22float2(dd);  // (d, dmin), exact
    // low-nibble sums carry 2^-24, high-nibble sums 2^-20
    const float2 dscale = f2(dm.x * 16777216.0f, dm.x * 1048576.0f);
#pragma unroll
    for (int b = 0; b < BP; ++b) v[b] = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t scw = c < 2 ? SC_lo : SC_hi;
        const uint32_t mmw = c < 2 ? MM_lo : MM_hi;
        const uint32_t sel = 0x7650u + 2u * (c & 1);
        const float2 sc = __fadd2_rn(f2(__uint_as_float(__byte_perm(scw, 0x4B000000u, sel)),
                                        __uint_as_float(__byte_perm(scw, 0x4B000000u, sel + 1))),
                                     f2(-8388608.0f, -8388608.0f));
        const float2 mm = __fadd2_rn(f2(__uint_as_float(__byte_perm(mmw, 0x4B000000u, sel)),
                                        __uint_as_float(__byte_perm(mmw, 0x4B000000u, sel + 1))),
                                     f2(-8388608.0f, -8388608.0f));
        const float2 D = __fmul2_rn(dscale, sc);          // scaled d*sc for sub-blocks 2c, 2c+1
        const float2 M = __fmul2_rn(f2(dm.y, dm.y), mm);  // dmin*m for sub-blocks 2c, 2c+1
        const uint4 q0 = *reinterpret_cast<const uint4 *>(u + 16 + 32 * c);
        const uint4 q1 = *reinterpret_cast<const uint4 *>(u + 32 + 32 * c);
        const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        float l0[BP], l1[BP], h0[BP], h1[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) l0[b] = l1[b] = h0[b] = h1[b] = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w = qw[i], wb = w >> 8;
            const uint32_t qa = w & 0x000F000Fu, qb = wb & 0x000F000Fu;  // low nibbles
            const uint32_t qc = w & 0x00F000F0u, qd = wb & 0x00F000F0u;  // high nibbles
#pragma unroll
            for (int b = 0; b < BP; ++b) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(xs + rows_x_off<BP>(US, j, c, i, b));
                mfma2(l0[b], qa, xv.x);
                mfma2(l1[b], qb, xv.y);
                mfma2(h0[b], qc, xv.z);
                mfma2(h1[b], qd, xv.w);
            }
        }
#pragma unroll
        for (int b = 0; b < BP; ++b) {
            const float Xlo = xsum[rows_xsum_off<BP>(US, j, 2 * c, b)];
            const float Xhi = xsum[rows_xsum_off<BP>(US, j, 2 * c + 1, b)];
            float t = v[b];
            t = fmaf(D.x, l0[b] + l1[b], t);
            t = fmaf(D.y, h0[b] + h1[b], t);
            t = fmaf(-M.x, Xlo, t);
            t = fmaf(-M.y, Xhi, t);
            v[b] = t;
        }
    }
}

// One Q8_0 unit (eight 34-byte blocks) against x (unit j of the slice).  Chunk c = blocks 2c and
// 2c+1 = bytes [68c, 68c+68), read through the 16-byte chunks covering it.
template <int BP>
__device__ __forceinline__ void rows_q8_0(const uint8_t *u, const __half *xs, int US, int j,
                                          float (&v)[BP])
{
#pragma unroll
    for (int b = 0; b < BP; ++b) v[b] = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int base16 = (68 * c) >> 4;       // first 16-byte chunk
        const int woff = ((68 * c) & 15) >> 2;  // word offset of byte 68c inside it
        uint32_t win[20];
#pragma unroll
        for (int k = 0; k < 5; ++k) {
            const uint4 q = *reinterpret_cast<const uint4 *>(u + 16 * (base16 + k));
            win[4 * k] = q.x;
            win[4 * k + 1] = q.y;
            win[4 * k + 2] = q.z;
            win[4 * k + 3] = q.w;
        }
        uint32_t wd[17];
#pragma unroll
        for (int k = 0; k < 17; ++k) wd[k] = win[woff + k];
        const float dA = __half2float(__ushort_as_half((unsigned short)(wd[0] & 0xFFFFu)));
        const float dB = __half2float(__ushort_as_half((unsigned short)(wd[8] >> 16)));
        float a0[BP], a1[BP], b0[BP], b1[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) a0[b] = a1[b] = b0[b] = b1[b] = 0.0f;
        const uint32_t off2 = 0x64806480u;  // fp16 (1152, 1152): 1024 + the 128 bias
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t la = __funnelshift_r(wd[i], wd[i + 1], 16) ^ 0x80808080u;  // block 2c
            const uint32_t lb = wd[9 + i] ^ 0x80808080u;                               // block 2c+1
            // (1024 + q + 128) as fp16 pairs (bytes 0,2 and 1,3 under a 0x64 high byte), minus 1152
            const uint32_t qa = hsub2_bits(__byte_perm(la, 0x64646464u, 0x7250), off2);  // e, e+2
            const uint32_t qb = hsub2_bits(__byte_perm(la, 0x64646464u, 0x7351), off2);  // e+1, e+3
            const uint32_t qc = hsub2_bits(__byte_perm(lb, 0x64646464u, 0x7250), off2);
            const uint32_t qd = hsub2_bits(__byte_perm(lb, 0x64646464u, 0x7351), off2);
#pragma unroll
            for (int b = 0; b < BP; ++b) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(xs + rows_x_off<BP>(US, j, c, i, b));
                mfma2(a0[b], qa, xv.x);
                mfma2(a1[b], qb, xv.y);
                mfma2(b0[b], qc, xv.z);
                mfma2(b1[b], qd, xv.w);
            }
        }
#pragma unroll
        for (int b = 0; b < BP; ++b) v[b] = fmaf(dB, b0[b] + b1[b], fmaf(dA, a0[b] + a1[b], v[b]));
    }
}

// One Q5_K superblock against x (unit j of the slice).  The Q4_K arithmetic with 5-bit q: per qs
// word, the low nibbles and the fifth bits of their weights are merged byte-wise into
// wl = (q & 15) | h << 4 (the qh bit of sub-block 2c is bit 2c of each qh byte, moved to bit 4),
// the high nibbles likewise into wh; bits 5-7 of each byte are then masked off, so each half of
// (wl & 0x001F001F) is the fp16 subnormal q * 2^-24 of a whole 5-bit q.
template <int BP>
__device__ __forceinline__ void rows_q5k(const uint8_t *u, const __half *xs, const float *xsum,
                                         int US, int j, float (&v)[BP])
{
    const uint4 hdr = *reinterpret_cast<const uint4 *>(u);
    const uint32_t SC_lo = hdr.y & 0x3F3F3F3Fu;
    const uint32_t MM_lo = hdr.z & 0x3F3F3F3Fu;
    const uint32_t SC_hi = (hdr.w & 0x0F0F0F0Fu) | ((hdr.y >> 2) & 0x30303030u);
    const uint32_t MM_hi = ((hdr.w >> 4) & 0x0F0F0F0Fu) | ((hdr.z >> 2) & 0x30303030u);
    __half2 dd;
    *reinterpret_cast<uint32_t *>(&dd) = hdr.x;
    const float2 dm = __half22float2(dd);  // (d, dmin), exact
    const float ds = dm.x * 16777216.0f;   // every q*x sum carries 2^-24
    const uint4 h0 = *reinterpret_cast<const uint4 *>(u + 16);
    const uint4 h1 = *reinterpret_cast<const uint4 *>(u + 32);
    const uint32_t hq[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};  // qh bytes 4i..4i+3
#pragma unroll
    for (int b = 0; b < BP; ++b) v[b] = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const uint32_t scw = c < 2 ? SC_lo : SC_hi;
        const uint32_t mmw = c < 2 ? MM_lo : MM_hi;
        const uint32_t sel = 0x7650u + 2u * (c & 1);
        const float2 sc = __fadd2_rn(f2(__uint_as_float(__byte_perm(scw, 0x4B000000u, sel)),
                                        __uint_as_float(__byte_perm(scw, 0x4B000000u, sel + 1))),
                                     f2(-8388608.0f, -8388608.0f));
        const float2 mm = __fadd2_rn(f2(__uint_as_float(__byte_perm(mmw, 0x4B000000u, sel)),
                                        __uint_as_float(__byte_perm(mmw, 0x4B000000u, sel + 1))),
                                     f2(-8388608.0f, -8388608.0f));
        const float2 D = __fmul2_rn(f2(ds, ds), sc);      // scaled d*sc for sub-blocks 2c, 2c+1
        const float2 M = __fmul2_rn(f2(dm.y, dm.y), mm);  // dmin*m for sub-blocks 2c, 2c+1
        const uint4 q0 = *reinterpret_cast<const uint4 *>(u + 48 + 32 * c);
        const uint4 q1 = *reinterpret_cast<const uint4 *>(u + 64 + 32 * c);
        const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        float l0[BP], l1[BP], h0a[BP], h1a[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) l0[b] = l1[b] = h0a[b] = h1a[b] = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w = qw[i], hw = hq[i];
            // bit 2c (low nibbles' fifth bit) and bit 2c + 1 (high nibbles') of each byte -> bit 4
            const uint32_t t1 = (c == 0) ? hw << 4 : (c == 1) ? hw << 2 : (c == 2) ? hw : hw >> 2;
            const uint32_t t2 = (c == 0) ? hw << 3 : (c == 1) ? hw << 1 : (c == 2) ? hw >> 1 : hw >> 3;
            const uint32_t wl = (w & 0x0F0F0F0Fu) | (t1 & 0xF0F0F0F0u);
            const uint32_t wh = ((w >> 4) & 0x0F0F0F0Fu) | (t2 & 0xF0F0F0F0u);
            const uint32_t qa = wl & 0x001F001Fu, qb = (wl >> 8) & 0x001F001Fu;  // low: e,e+2 / e+1,e+3
            const uint32_t qc = wh & 0x001F001Fu, qd = (wh >> 8) & 0x001F001Fu;  // high
#pragma unroll
            for (int b = 0; b < BP; ++b) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(xs + rows_x_off<BP>(US, j, c, i, b));
                mfma2(l0[b], qa, xv.x);
                mfma2(l1[b], qb, xv.y);
                mfma2(h0a[b], qc, xv.z);
                mfma2(h1a[b], qd, xv.w);
            }
        }
#pragma unroll
        for (int b = 0; b < BP; ++b) {
            const float Xlo = xsum[rows_xsum_off<BP>(US, j, 2 * c, b)];
            const float Xhi = xsum[rows_xsum_off<BP>(US, j, 2 * c + 1, b)];
            float t = v[b];
            t = fmaf(D.x, l0[b] + l1[b], t);
            t = fmaf(D.y, h0a[b] + h1a[b], t);
            t = fmaf(-M.x, Xlo, t);
            t = fmaf(-M.y, Xhi, t);
            v[b] = t;
        }
    }
}

// One Q6_K superblock against x (unit j of the slice), from the lane's ring window: the
// superblock starts `o` bytes (even, 0..14) into the 16-byte aligned window `win`, so its word k
// is the funnel shift of window words o/4 + k and o/4 + k + 1 by 8 * (o % 4) bits.  When `tail` is
// set (the tensor's last superblock, whose window was cut at the tensor's last 16-byte boundary)
// the scales and d are read from `gblk`, the superblock in global memory.
// Arithmetic: per 16-weight group t, sum (q - 32) x = sum q x - 32 X_t, q in 0..63 built like
// Q5_K's: the low nibble of a ql byte and its two qh bits (bits 2p, 2p+1 of the qh byte for the
// low nibbles of chunk c = 2h + p, bits 2p + 4, 2p + 5 for the high nibbles) merged into one byte.
template <int BP>
__device__ __forceinline__ void rows_q6k(const uint32_t *win, int o, bool tail, const uint8_t *gblk,
                                         const __half *xs, const float *xsum, int US, int j,
                                         float (&v)[BP])
{
    const uint32_t *wp = win + (o >> 2);
    const uint32_t sh = (o & 2) ? 16u : 0u;
    auto word = [&](int k) { return __funnelshift_r(wp[k], wp[k + 1], sh); };
    uint32_t scw[4], dw;
    if (!tail) {
#pragma unroll
        for (int k = 0; k < 4; ++k) scw[k] = word(48 + k);
        dw = word(52);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            scw[k] = (uint32_t)gblk[192 + 4 * k] | ((uint32_t)gblk[193 + 4 * k] << 8) |
                     ((uint32_t)gblk[194 + 4 * k] << 16) | ((uint32_t)gblk[195 + 4 * k] << 24);
        dw = (uint32_t)gblk[208] | ((uint32_t)gblk[209] << 8);
    }
    const float ds = __half2float(__ushort_as_half((unsigned short)(dw & 0xFFFFu))) * 16777216.0f;
#pragma unroll
    for (int b = 0; b < BP; ++b) v[b] = 0.0f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t hq[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) hq[i] = word(32 + 8 * h + i);
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            const int c = 2 * h + p;
            uint32_t qw[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) qw[i] = word(16 * h + 8 * p + i);
#pragma unroll
            for (int hp = 0; hp < 2; ++hp) {
                const int tlo = 8 * h + 2 * p + hp, thi = tlo + 4;  // scale groups
                const float Dlo = ds * (float)(int8_t)(scw[tlo >> 2] >> (8 * (tlo & 3)));
                const float Dhi = ds * (float)(int8_t)(scw[thi >> 2] >> (8 * (thi & 3)));
                float l0[BP], l1[BP], h0a[BP], h1a[BP];
#pragma unroll
                for (int b = 0; b < BP; ++b) l0[b] = l1[b] = h0a[b] = h1a[b] = 0.0f;
#pragma unroll
                for (int i = 4 * hp; i < 4 * hp + 4; ++i) {
                    const uint32_t w = qw[i], hw = hq[i];
                    const uint32_t t1 = p ? hw << 2 : hw << 4;  // bits 2p, 2p+1 -> bits 4, 5
                    const uint32_t t2 = p ? hw >> 2 : hw;       // bits 2p+4, 2p+5 -> bits 4, 5
                    const uint32_t wl = (w & 0x0F0F0F0Fu) | (t1 & 0xF0F0F0F0u);
                    const uint32_t wh = ((w >> 4) & 0x0F0F0F0Fu) | (t2 & 0xF0F0F0F0u);
                    const uint32_t qa = wl & 0x003F003Fu, qb = (wl >> 8) & 0x003F003Fu;
                    const uint32_t qc = wh & 0x003F003Fu, qd = (wh >> 8) & 0x003F003Fu;
#pragma unroll
                    for (int b = 0; b < BP; ++b) {
                        const uint4 xv =
                            *reinterpret_cast<const uint4 *>(xs + rows_x_off<BP>(US, j, c, i, b));
                        mfma2(l0[b], qa, xv.x);
                        mfma2(l1[b], qb, xv.y);
                        mfma2(h0a[b], qc, xv.z);
                        mfma2(h1a[b], qd, xv.w);
                    }
                }
                // d*sc_t * (sum q x - 32 X_t): the q x sums carry 2^-24, so 32 X_t is scaled by
                // 2^-19 to match
#pragma unroll
                for (int b = 0; b < BP; ++b) {
                    const float Xlo = xsum[rows_xsum_off<BP, 16>(US, j, tlo, b)];
                    const float Xhi = xsum[rows_xsum_off<BP, 16>(US, j, thi, b)];
                    float t = v[b];
                    t = fmaf(Dlo, fmaf(-1.9073486328125e-06f, Xlo, l0[b] + l1[b]), t);
                    t = fmaf(Dhi, fmaf(-1.9073486328125e-06f, Xhi, h0a[b] + h1a[b]), t);
                    v[b] = t;
                }
            }
        }
    }
}

// IQ4_XS codebook lookup of the eight 4-bit indices of a qs word: lo = the biased levels
// (level + 128, one byte each) of nibbles 0..3, hi = of nibbles 4..7, in nibble order.  A nibble's
// low three bits pick one of the eight bytes of (kIq4Lut0, kIq4Lut1) and of (kIq4Lut2, kIq4Lut3);
// its bit 3 then picks which of the two results to keep.
__device__ __forceinline__ void iq4_lookup(uint32_t w, uint32_t &lo, uint32_t &hi)
{
    const uint32_t s = w & 0x77777777u;
    const uint32_t pick = ((w >> 1) & 0x44444444u) | 0x32103210u;  // nibble k: k % 4 + 4 * bit 3
    lo = __byte_perm(__byte_perm(kIq4Lut0, kIq4Lut1, s), __byte_perm(kIq4Lut2, kIq4Lut3, s), pick);
    hi = __byte_perm(__byte_perm(kIq4Lut0, kIq4Lut1, s >> 16), __byte_perm(kIq4Lut2, kIq4Lut3, s >> 16),
                     pick >> 16);
}

// One IQ4_XS superblock against x (unit j of the slice), from the lane's ring window: the
// superblock starts `o` bytes (0 or 8) into the 16-byte aligned window `win`, so its word k is
// window word o/4 + k.  When `tail` is set (the tensor's last superblock, whose window was cut at
// the tensor's last 16-byte boundary) its last two words are read from `gblk` in global memory.
// Arithmetic: each biased level u = level + 128 (1..241) becomes the fp16 subnormal u * 2^-24
// (the byte under a zero byte), fma.rn.f32.f16 forms u * x exactly, and per sub-block
//   sum level * x = 2^24 * sum (u * 2^-24) x - 128 X_j,
// scaled by d * (ls_j - 32) (exact in fp32).
template <int BP>
__device__ __forceinline__ void rows_iq4xs(const uint32_t *win, int o, bool tail, const uint8_t *gblk,
                                           const __half *xs, const float *xsum, int US, int j,
                                           float (&v)[BP])
{
    const uint32_t *wp = win + (o >> 2);
    const uint32_t w0 = wp[0];   // d (bits 0-15), scales_h (bits 16-31)
    const uint32_t sl = wp[1];   // scales_l[0..3]
    const uint32_t sh = w0 >> 16;
    const float ds = __half2float(__ushort_as_half((unsigned short)(w0 & 0xFFFFu))) * 16777216.0f;
    auto word = [&](int k) {
        return (tail && k >= 32) ? *reinterpret_cast<const uint32_t *>(gblk + 4 * k) : wp[k];
    };
#pragma unroll
    for (int b = 0; b < BP; ++b) v[b] = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        // sub-blocks 2c and 2c + 1: scales_l byte c (both nibbles), scales_h bits 4c .. 4c+3
        const int lsA = (int)(((sl >> (8 * c)) & 15u) | (((sh >> (4 * c)) & 3u) << 4));
        const int lsB = (int)(((sl >> (8 * c + 4)) & 15u) | (((sh >> (4 * c + 2)) & 3u) << 4));
        const float DA = ds * (float)(lsA - 32), DB = ds * (float)(lsB - 32);
        float a0[BP], a1[BP], b0[BP], b1[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) a0[b] = a1[b] = b0[b] = b1[b] = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t lo, hi;
            iq4_lookup(word(2 + 8 * c + i), lo, hi);
            const uint32_t p0 = __byte_perm(lo, 0u, 0x4140), p1 = __byte_perm(lo, 0u, 0x4342);
            const uint32_t p2 = __byte_perm(hi, 0u, 0x4140), p3 = __byte_perm(hi, 0u, 0x4342);
#pragma unroll
            for (int b = 0; b < BP; ++b) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(xs + rows_x_off<BP>(US, j, c, i, b));
                if (i < 4) {
                    mfma2(a0[b], p0, xv.x);
                    mfma2(a1[b], p1, xv.y);
                    mfma2(a0[b], p2, xv.z);
                    mfma2(a1[b], p3, xv.w);
                } else {
                    mfma2(b0[b], p0, xv.x);
                    mfma2(b1[b], p1, xv.y);
                    mfma2(b0[b], p2, xv.z);
                    mfma2(b1[b], p3, xv.w);
                }
            }
        }
        // the u x sums carry 2^-24, so 128 X is scaled by 2^-17 to match
#pragma unroll
        for (int b = 0; b < BP; ++b) {
            const float XA = xsum[rows_xsum_off<BP>(US, j, 2 * c, b)];
            const float XB = xsum[rows_xsum_off<BP>(US, j, 2 * c + 1, b)];
            float t = v[b];
            t = fmaf(DA, fmaf(-7.62939453125e-06f, XA, a0[b] + a1[b]), t);
            t = fmaf(DB, fmaf(-7.62939453125e-06f, XB, b0[b] + b1[b]), t);
            v[b] = t;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Pair layout of a band: G row groups of 32 rows, P K parts; pair q = g * P + p.
// Pair layout of a band: Gm row groups of 32 rows per matrix, G = mats * Gm groups (matrix-major),
// P K parts; pair q = g * P + p.
struct BandShape {
    int Gm, G, P;
};
template <int MATS>
__device__ __forceinline__ BandShape band_shape(int rows, int US_s, int NW)
{
    BandShape b;
    b.Gm = (rows + 31) / 32;
    b.G = MATS * b.Gm;
    b.P = max(1, min(NW / max(b.G, 1), US_s));
    return b;
}

// The band's finished rows: sum the K parts of every matrix in part order from the partial rows
// red[pair][32][BP] and write y (one slice: y itself, through the pair's activation) or this
// slice's partial rows part[s][MATS][N][B].
template <int BP, int MATS>
__device__ __forceinline__ void band_finish(const RowsArgs &a, const BandShape &bs, const float *red,
                                            int s, int64_t R0, int rows)
{
    const int64_t NB = a.N * a.B;
    for (int t = threadIdx.x; t < rows * a.B; t += blockDim.x) {
        const int rr = t / a.B, b = t - rr * a.B;
        const int g = rr >> 5, l = rr & 31;
        float v[MATS];
#pragma unroll
        for (int m = 0; m < MATS; ++m) {
            float sum = 0.0f;
            for (int p = 0; p < bs.P; ++p)
                sum += red[((size_t)((m * bs.Gm + g) * bs.P + p) * 32 + l) * BP + b];
            v[m] = sum;
        }
        const int64_t idx = R0 * a.B + t;
        if (a.S == 1) {
            if (MATS == 2) a.out[idx] = a.act ? silu_mul(v[0], v[MATS - 1]) : v[0];
            else a.out[idx] = a.res ? v[0] + a.res[idx] : v[0];
        } else {
#pragma unroll
            for (int m = 0; m < MATS; ++m) a.out[((int64_t)s * MATS + m) * NB + idx] = v[m];
        }
    }
}

// sum_{s < S} p[s * stride], added in slice order; the loads go out eight at a time, so the last
// CTA of a band waits for ceil(S / 8) round trips to L2 rather than S.
__device__ __forceinline__ float slice_sum(const float *p, int64_t stride, int S)
{
    float sum = 0.0f;
    for (int s0 = 0; s0 < S; s0 += 8) {
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = (s0 + j < S) ? __ldcg(p + (int64_t)(s0 + j) * stride) : 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if (s0 + j < S) sum += v[j];
    }
    return sum;
}

// Split-K across CTAs without a second kernel.  CTA (slice s, band) has written its band's
// partial rows to out = part[s][mats][N][B]; each makes its writes visible and bumps the band's
// counter, and the last of the S CTAs to arrive adds the S slices in slice order (so y does not
// depend on arrival order), writes y and resets the counter for the next call.  Every CTA
// arrives, also after a copy timeout, so the counters always return to zero.
// `flag` is one int of shared memory that nothing else uses any more (the kernels pass their x
// sums, which are dead once the steps are done), so the kernels need no static shared memory.
template <int MATS>
__device__ __forceinline__ void splitk_fixup(const RowsArgs &a, int band, int64_t R0, int rows,
                                             int *flag)
{
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned prev = atomicAdd(a.cnt + band, 1u);
        const int last = (prev == (unsigned)(a.S - 1)) ? 1 : 0;
        *flag = last;
        if (last) a.cnt[band] = 0u;  // all S arrivals of this call are in
    }
    __syncthreads();
    if (!*flag) return;
    __threadfence();
    const int64_t NB = a.N * a.B;
    for (int t = threadIdx.x; t < rows * a.B; t += blockDim.x) {
        const int64_t idx = R0 * a.B + t;
        float v[MATS];
#pragma unroll
        for (int m = 0; m < MATS; ++m) v[m] = slice_sum(a.out + (int64_t)m * NB + idx, (int64_t)MATS * NB, a.S);
        if (MATS == 2) a.y[idx] = a.act ? silu_mul(v[0], v[MATS - 1]) : v[0];
        else a.y[idx] = a.res ? v[0] + a.res[idx] : v[0];
    }
}

// The weight tensor maps of a launch: one per matrix (a kernel parameter, in the parameter space
// the TMA reads descriptors from).
template <int MATS> struct WeightMaps {
    CUtensorMap m[MATS];
};

// MATS = 1: y = W x.  MATS = 2: the gate/up pair, the second matrix through maps.m[1] (the band's
// row groups of both matrices, matrix-major), combined by band_finish / splitk_fixup.
template <int FMT, int BP, int MATS>
__global__ void __launch_bounds__(RowsWarps<FMT, BP>::value * 32, 1)
    rows_gemv_kernel(const RowsArgs a, const __grid_constant__ WeightMaps<MATS> maps)
{
    constexpr int NW = RowsWarps<FMT, BP>::value;
    constexpr int NS = kRowsStages;
    constexpr int UB = RowsFmt<FMT>::kUnitBytes;
    constexpr int LB = RowsFmt<FMT>::kLaneBytes;
    constexpr bool PER_LANE = RowsFmt<FMT>::kPerLane;
    constexpr int BOX = 32 * LB;  // ring bytes of one step: 32 rows x one unit (or its window)
    // one bulk copy per lane, or (a per-lane format whose rows are 16-byte multiples) 2-D copies
    const bool lane_copy = PER_LANE && !a.tmap;
    static_assert(BOX % 128 == 0, "tensor-copy destinations in shared memory must be 128-byte aligned");
    static_assert(LB % 16 == 0, "bulk-copy destinations must be 16-byte aligned");

    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *ring = smem;
    __half *xs = reinterpret_cast<__half *>(smem + NW * NS * BOX);
    float *xsum = reinterpret_cast<float *>(xs + (size_t)a.US * 256 * BP);
    float *red = xsum + a.US * RowsFmt<FMT>::kGroups * BP;  // [pair][32][BP] partial rows
    uint64_t *bars = reinterpret_cast<uint64_t *>(red + a.red_floats);

    const int s = blockIdx.x / a.Gs;
    const int cta = blockIdx.x % a.Gs;
    const int US_s = min(a.US, a.UPR - s * a.US);
    const int64_t R0 = ((int64_t)cta * a.N) / a.Gs, R1 = ((int64_t)(cta + 1) * a.N) / a.Gs;
    const int rows = (int)(R1 - R0);
    const BandShape bs = band_shape<MATS>(rows, US_s, NW);
    const int npairs = bs.G * bs.P;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ucol0 = s * a.US;  // first unit column of this slice

    // this warp's pairs: warp, warp + NW, ...; steps run over the units of each pair in turn.
    // K part p of a row group takes the units p, p + P, p + 2P, ... of the slice, so the P warps
    // of a group stream adjacent units of the same 32 rows at about the same time (measured
    // faster than contiguous ranges of units per part: DRAM sees longer runs of each row).
    const int du = bs.P;
    auto pair_units = [&](int q, int &ua, int &ub) {
        ua = q % bs.P;
        ub = US_s;
    };
    int nsteps = 0;
    for (int q = warp; q < npairs; q += NW) {
        int ua, ub;
        pair_units(q, ua, ub);
        nsteps += (ub - ua + du - 1) / du;
    }
    uint8_t *myring = ring + warp * NS * BOX;
    const uint32_t bar0 = smem_u32(bars + warp * NS);
    // issue cursor (lane 0): pair iq, unit iu, ring slot islot
    int iq = warp, iu = 0, iub = 0, islot = 0;
    int ig_row = 0, ig_map = 0;  // the pair's first row in its matrix, and its matrix
    auto cursor_pair = [&]() {
        pair_units(iq, iu, iub);
        const int g = iq / bs.P;  // group g of matrix 0, or group g - Gm of matrix 1
        const bool second = (MATS > 1) && g >= bs.Gm;
        ig_row = (int)R0 + 32 * (second ? g - bs.Gm : g);
        ig_map = second ? MATS - 1 : 0;
    };
    if (iq < npairs) cursor_pair();
    auto advance = [&]() {
        islot = (islot + 1 == NS) ? 0 : islot + 1;
        iu += du;
        if (iu >= iub) {
            iq += NW;
            if (iq < npairs) cursor_pair();
        }
    };
    // one 2-D tensor copy of the step's 32 rows x one unit (lane 0 alone).  The box starts at the
    // unit's first byte rounded down to 16 (the unit itself for the formats whose units are
    // 16-byte multiples; IQ4_XS units sit 0 or 8 bytes past it, inside a 144-byte box).
    auto issue = [&]() {
        const uint32_t bar = bar0 + 8 * islot;
        mbar_arrive_expect_tx(bar, BOX);
        const int xw = (int)((((int64_t)(ucol0 + iu) * UB) & ~(int64_t)15) >> 2);
        tma_load_2d(smem_u32(myring + islot * BOX), &maps.m[ig_map], xw, ig_row, bar);
        advance();
    };
    // per-lane copies (all 32 lanes): rows whose unit is not 16-byte aligned in W (Q6_K, IQ4_XS)
    // cannot be described by a tensor map, so each lane copies the 16-byte aligned window
    // [off & ~15, (off & ~15) + kWinBytes) around its row's unit at byte off; windows never reach past the
    // tensor's last 16-byte boundary (the last unit of the tensor may come up short: its tail is
    // read from global memory by the consumer).  Lanes past the last row copy nothing.
    auto issue_lanes = [&]() {
        const uint32_t bar = bar0 + 8 * islot;
        const int64_t row = (int64_t)ig_row + lane;
        uint32_t nb = 0;
        const uint8_t *src = nullptr;
        if (row < a.N) {
            const int64_t ad = ((row * a.UPR + ucol0 + iu) * UB) & ~(int64_t)15;
            const int64_t room = a.wend - ad;
            constexpr int WIN = RowsFmt<FMT>::kWinBytes;
            nb = (uint32_t)(room < WIN ? room : WIN);
            src = a.w[ig_map] + ad;
        }
        const uint32_t tot = __reduce_add_sync(0xffffffffu, nb);
        if (lane == 0) mbar_arrive_expect_tx(bar, tot);
        __syncwarp();
        if (nb) bulk_g2s_plain(smem_u32(myring + islot * BOX + lane * LB), src, nb, bar);
        advance();
    };

    // 1. weight prefetch (independent of the previous kernel on the stream): the first steps
    //    into the ring
    if (nsteps > 0 && lane == 0) {
        if (!lane_copy) {
#pragma unroll
            for (int m = 0; m < MATS; ++m)
                asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.m[m])) : "memory");
        }
        for (int i = 0; i < NS; ++i) mbar_init(bar0 + 8 * i, 1);
        mbar_init_fence();
        if (!lane_copy)
            for (int i = 0; i < kPreStages && i < nsteps; ++i) issue();
    }
    if (lane_copy && nsteps > 0) {
        __syncwarp();
        for (int i = 0; i < kPreStages && i < nsteps; ++i) issue_lanes();
    }
    // 2. programmatic dependent launch: let the next kernel start prefetching, then wait for the
    //    previous kernel's results before reading x or writing y
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // 3. x for this slice -> shared memory (fp16 in consumer order) and per-sub-block sums,
    //    then the rest of the ring: after the CTA's barrier, or (Q8_0) as soon as this warp's own
    //    x loads have returned
    constexpr bool REFILL_LATE = RowsRefillAfterBarrier<FMT>::value;
    rows_stage_x<BP, FMT>(a, s, US_s, xs, xsum);
    if (REFILL_LATE) __syncthreads();
    if (lane_copy) {
        for (int i = kPreStages; i < NS && i < nsteps; ++i) issue_lanes();
    } else if (lane == 0) {
        for (int i = kPreStages; i < NS && i < nsteps; ++i) issue();
    }
    if (!REFILL_LATE) __syncthreads();

    int step = 0, cslot = 0;
    uint32_t cphase = 0;  // consumer: ring slot and its phase parity
    bool failed = false;
    for (int q = warp; q < npairs && !failed; q += NW) {
        int ua, ub;
        pair_units(q, ua, ub);
        float acc[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) acc[b] = 0.0f;
        for (int j = ua; j < ub; j += du, ++step) {
            const bool ok = mbar_wait_bounded(bar0 + 8 * cslot, cphase);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) {
                    atomicExch(a.err, kErrCopyTimeout);
                    // wait (bounded) for the copies still in flight before the CTA exits
                    int r_slot = cslot;
                    uint32_t r_phase = cphase;
                    for (int r = step + 1; r < nsteps && r < step + NS; ++r) {
                        if (++r_slot == NS) { r_slot = 0; r_phase ^= 1u; }
                        (void)mbar_wait_bounded(bar0 + 8 * r_slot, r_phase);
                    }
                }
                failed = true;
                break;
            }
            const uint8_t *u = myring + cslot * BOX + lane * LB;
            float v[BP];
            if (FMT == kFmtQ4_K) {
                rows_q4k<BP>(u, xs, xsum, a.US, j, v);
            } else if (FMT == kFmtQ5_K) {
                rows_q5k<BP>(u, xs, xsum, a.US, j, v);
            } else if (FMT == kFmtQ6_K || FMT == kFmtIQ4_XS) {
                // this lane's row and unit: where its superblock sits in the window
                const int g = q / bs.P;
                const bool second = (MATS > 1) && g >= bs.Gm;
                const int64_t row = R0 + 32 * (second ? g - bs.Gm : g) + lane;
                const int64_t m = row * a.UPR + ucol0 + j;  // superblock index in the tensor
                const int o = (int)((m * UB) & 15);
                const bool tail = a.wtail && row == a.N - 1 && ucol0 + j == a.UPR - 1;
                const uint8_t *gblk = a.w[second ? MATS - 1 : 0] + m * UB;
                if (FMT == kFmtQ6_K)
                    rows_q6k<BP>(reinterpret_cast<const uint32_t *>(u), o, tail, gblk, xs, xsum, a.US, j, v);
                else
                    rows_iq4xs<BP>(reinterpret_cast<const uint32_t *>(u), o, tail, gblk, xs, xsum, a.US, j, v);
            } else {
                rows_q8_0<BP>(u, xs, a.US, j, v);
            }
#pragma unroll
            for (int b = 0; b < BP; ++b) acc[b] += v[b];
            __syncwarp();
            if (step + NS < nsteps) {
                if (lane_copy) {
                    fence_proxy_async_smem();
                    issue_lanes();
                } else if (lane == 0) {
                    fence_proxy_async_smem();
                    issue();
                }
            }
            if (++cslot == NS) { cslot = 0; cphase ^= 1u; }
        }
        if (bs.P == 1 && MATS == 1) {
            // a single K part of a single matrix: the row is complete, write it
            const int rr = (q / bs.P) * 32 + lane;
            if (rr < rows) {
                const int64_t row0 = (R0 + rr) * a.B;
                float *dst = a.out + (int64_t)s * a.N * a.B + row0;
                if (a.S == 1 && a.res) {
                    for (int b = 0; b < a.B; ++b) dst[b] = acc[b] + a.res[row0 + b];
                } else {
                    for (int b = 0; b < a.B; ++b) dst[b] = acc[b];
                }
            }
        } else {
            float *r = red + ((size_t)q * 32 + lane) * BP;
#pragma unroll
            for (int b = 0; b < BP; ++b) r[b] = acc[b];
        }
    }
    const bool any_failed = __syncthreads_or(failed ? 1 : 0);
    // 4. rows of the band: sum the K parts (and combine the pair) in part order, write once
    if (!any_failed && (bs.P > 1 || MATS > 1)) band_finish<BP, MATS>(a, bs, red, s, R0, rows);
    // 5. K slices: the last CTA of the band adds them up
    if (a.S > 1) splitk_fixup<MATS>(a, cta, R0, rows, reinterpret_cast<int *>(xsum));
}

}  // namespace qg
