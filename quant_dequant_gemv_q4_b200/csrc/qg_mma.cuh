// qg_mma.cuh -- the tensor-core streaming GEMV of libqg (sm_100a) for the K-quants (Q4_K, Q5_K,
// Q6_K), Q8_0 and IQ4_XS, B = 1..16 columns (two 8-column n-tiles past 8).
//
// Operation (HARDWARE GROUND TRUTH: 2x NVIDIA Tesla T4 (Kaggle), second prompt, "SPEC"):
//   y[n,b] = sum_k dequant(W)[n,k] * x[k,b], fp32 accumulation ("PHYSICS & CONTRACT"), Q4_K
//   w = d*sc*q - dmin*m ("QUANTIZATION MIX").
//
// Why tensor cores here.  With B columns, the CUDA-core kernel spends one fp32 FMA per weight and
// column, so at B = 8 the FMA pipe, not HBM, bounds it.  mma.sync.m16n8k16 (f16 x f16 -> f32)
// multiplies a 16-row x 16-weight tile of integer codes by a 16 x 8 tile of x in one
// instruction: the 8 columns of the instruction are the B <= 8 columns of x, so B = 1..8 cost the
// same tensor work, and the weights are unpacked once for all columns.  Products are exact
// (small integers, or integers times a power of two, times fp16 x) and the sums are fp32, so the
// arithmetic is the factored form of the CUDA-core kernel (Q4_K / Q5_K shown; Q6_K, Q8_0 and
// IQ4_XS have their own scales and no min, see their step functions):
//   sum_i w_i x_i = d * sum_j sc_j sum_{i in j} q_i x_i  -  sum_j M_j * sum_{i in j} x_i,
//   M_j = dmin*m_j (exact in fp32), j = 32-weight sub-block.
//
// Mapping.  The grid, row bands, (row group, K part) pairs and the per-warp ring of 2-D TMA
// boxes (32 rows x one 144-byte superblock) are those of the CUDA-core kernel (qg_rows.cuh).  Per
// step a warp multiplies its 32 rows as two 16-row tiles:
//   A fragment (rows g and g+8 of a tile, lane = 4g + t): word 2t+h of the 32-byte chunk c of the
//     row; its low nibbles of bytes 0 and 2 (sub-block 2c) are masked as the fp16 subnormal pair
//     q 2^-24 and multiplied (one f16x2 multiply) into normal fp16 numbers; its high nibbles
//     (sub-block 2c+1) stay in place as q 2^-20 and are multiplied likewise; word >> 8 gives
//     bytes 1 and 3.  So one 32-bit word feeds four A registers through four LOP3 (ALU pipe), one
//     multiply-high (the shift) and four f16x2 multiplies (FMA pipe).  Normal operands keep the
//     tensor core's full accumulation precision (on subnormal codes its sums keep only about 12
//     bits below the largest product, which measured up to 0.95 of the error bound with massive
//     activations).  The multiplier is a power of two (Q4_K, Q6_K) or the sub-block scale times
//     a power of two (Q5_K), see mma_q4k_step / mma_q5k_step.
//   B fragment: x in the matching order, staged once per CTA (mma_stage_x).
//   C fragment: rows g, g+8 x columns 2t, 2t+1, scaled by the sub-block's d sc_j (Q4_K), or the
//     superblock's d (Q5_K), of its row and added to the warp's accumulators.
// The scales come from a per-warp table: lane l decodes row l's header (as in the CUDA-core
// kernel), writes its row's entries, and folds -M_j * sum(x over j) into its own per-row sum.
// Q5_K keeps this skeleton; its fifth-bit plane is merged into the A words byte-wise
// (q5k_a_codes).  Q6_K (mma_q6k_step) has signed 8-bit scales whose products with the 6-bit codes
// do not fit fp16 exactly: its codes enter as q 2^-10 and each 16-weight k-tile's C fragments are
// scaled by its own group's d sc_t 2^10.
#pragma once

#include "qg_codes.cuh"
#include "qg_rows.cuh"

namespace qg {

// warps per CTA of the tensor-core kernel (shared memory: ring + x fragments + tables; at 16
// columns, registers)
template <int BP> struct MmaWarps {
    static constexpr int value = BP >= 16 ? 8 : BP >= 8 ? 12 : 16;
};

// Formats of the tensor-core kernel: Q4_K, Q5_K (the Q4_K superblock with a fifth-bit plane
// qh[32] before qs), Q6_K, and below IQ4_XS and Q8_0.  kQs: offset of qs in the superblock.
template <int FMT> struct MmaFmt;
template <> struct MmaFmt<kFmtQ4_K> {
    static constexpr int kUnitBytes = 144, kQs = 16;
};
template <> struct MmaFmt<kFmtQ5_K> {
    static constexpr int kUnitBytes = 176, kQs = 48;
};
template <> struct MmaFmt<kFmtQ6_K> {  // rows arrive in 240-byte per-lane windows (qg_rows.cuh)
    static constexpr int kUnitBytes = 240, kQs = 0;
};
// IQ4_XS with an even number of 136-byte units per row: a 144-byte box per row, the 16-byte
// aligned window around the unit, which starts 0 or 8 bytes into it (the same for every row of a
// step); qs at byte 8 of the unit
template <> struct MmaFmt<kFmtIQ4_XS> {
    static constexpr int kUnitBytes = 144, kQs = 8;
};
// Q8_0 with K % 256 == 0: a unit is 8 blocks of {fp16 d; i8 qs[32]}, 272 bytes (as in the
// CUDA-core kernel); block b's qs start at byte 34 b + 2
template <> struct MmaFmt<kFmtQ8_0> {
    static constexpr int kUnitBytes = 272, kQs = 2;
};

// n-tiles of 8 columns per mma (16 columns: two, sharing the unpacked A fragment)
template <int BP> struct MmaNT {
    static constexpr int value = BP > 8 ? 2 : 1;
};
// floats of a warp's table: D_j [8][32], reused for the epilogue's [32][BP] rows
template <int BP> struct MmaTab {
    static constexpr int value = 32 * BP > 256 ? 32 * BP : 256;
};
// Q6_K: 16 scale groups per superblock (D_t [16][32]); its per-lane copy windows (240 B a row)
// leave shared memory for 8 warps
template <int FMT, int BP> struct MmaTabF {
    static constexpr int value = (FMT == kFmtQ6_K && MmaTab<BP>::value < 512) ? 512 : MmaTab<BP>::value;
};
template <int FMT, int BP> struct MmaWarpsF {
    // Q8_0: 272-byte units make each warp's ring twice Q4_K's, so fewer warps fit next to x
    static constexpr int value = (FMT == kFmtQ6_K) ? 8 : (FMT == kFmtQ8_0) ? (BP >= 8 ? 6 : 8)
                                                                          : MmaWarps<BP>::value;
};

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// x fragments.  For unit j of the slice, chunk c, nibble half lh (0 low, 1 high), k-step h,
// column col < BP and t = lane % 4, one uint2 holds
//   { (x[e], x[e+2]), (x[e+1], x[e+3]) },  e = 256j + 64c + 32lh + 8t + 4h,
// the weights that word 2t+h of chunk c contributes in that nibble half, in the order the masks
// produce them.  Index (in uint2):
__device__ __forceinline__ int mma_xf_idx(int j, int c, int lh, int h, int col, int t, int BP)
{
    return ((((j * 4 + c) * 2 + lh) * 2 + h) * BP + col) * 4 + t;
}
// Columns are stored XOR-swizzled per block, col ^ mma_xf_swz(c, lh, h): the staging lanes that
// differ only in (h, lh, chunk) then write different banks (with BP >= 4 a block spans a multiple
// of 32 words, so unswizzled they would all hit one bank).
__device__ __forceinline__ int mma_xf_swz(int c, int lh, int h, int BP)
{
    return BP >= 4 ? ((h + 2 * lh + 4 * (c & 1)) & (BP - 1)) : 0;
}

// Sums over the 8 lanes of a sub-block group (lanes 8i .. 8i+7 of the warp, th = lane % 8) of
// the per-column values s[0..BP): a transposing butterfly.  At xor distance 4, 2, 1 each lane keeps
// half of its columns (the upper half when its bit of th is set), sends the other half to its
// partner and adds what it receives, so 8 columns take 4 + 2 + 1 shuffles instead of 3 per column.
// Once a lane holds a single column the remaining levels are plain butterfly adds.  On return lane
// th holds the sums of columns [c0, c0 + n) with n = max(BP / 8, 1) and
// c0 = (th * BP / 8) for BP >= 8, th >> (3 - log2 BP) otherwise (then lanes whose low 3 - log2 BP
// bits of th are zero hold the only copy needed).
template <int N, int M>
__device__ __forceinline__ void xsum_butterfly(float *s, int th)
{
    if constexpr (M > 0) {
        if constexpr (N >= 2) {
            constexpr int H = N / 2;
            const bool up = (th & M) != 0;
#pragma unroll
            for (int i = 0; i < H; ++i) {
                const float send = up ? s[i] : s[i + H];
                const float keep = up ? s[i + H] : s[i];
                s[i] = keep + __shfl_xor_sync(0xffffffffu, send, M);
            }
            xsum_butterfly<H, M / 2>(s, th);
        } else {
            s[0] += __shfl_xor_sync(0xffffffffu, s[0], M);
            xsum_butterfly<1, M / 2>(s, th);
        }
    }
}

// Thread g stages the 4 x rows of group g = ((j*4 + c)*2 + lh)*8 + 2t + h (rows e..e+3 for the
// K-quants, all B columns), writes their BP fragments, and the 8 groups of one sub-block (8
// consecutive lanes) add up its x sums.  A thread loads the rows of up to NB groups before it
// processes any, so their L2 round trips overlap.  A row's BP halves are BP / 2 words (word m:
// columns 2m, 2m + 1), and a fragment register takes two halves of one column from two rows with
// one byte permute.
// Q6_K keeps the same fragment slots with its own weight order: chunk c = 2hf + p is
// ql[64hf + 32p ..], k-tile h covers its words 4h .. 4h+3 (one 16-weight scale group), so
//   e = 256j + 128(c >> 1) + 32(c & 1) + 64lh + 16h + 4t,
// and the x sums are per 16-weight group 8(c >> 1) + 2(c & 1) + h + 4lh.  IQ4_XS: k-tile h of chunk
// c is sub-block 2c + h (qs words 4h .. 4h+3 of the chunk; a qs byte holds weights r and r + 16 of
// its sub-block; k-half lh takes qs bytes 2lh, 2lh + 1 of the thread's word, whose weights pair
// as (r, r + 16)), so the four x rows are e, e + 1, e + 16, e + 17 with e = 256j + 32(2c + h) +
// 4t + 2lh, and it needs no x sums (its codes are the signed levels themselves).
template <int BP, int FMT = kFmtQ4_K>
__device__ __forceinline__ void mma_stage_x(const RowsArgs &a, int s, int US_s, uint2 *xf,
                                            float *xsum)
{
    constexpr int W = (BP + 1) / 2;           // words of one x row (BP halves, BP >= 2; BP = 1: 1)
    constexpr int NB = BP >= 16 ? 2 : 4;      // groups whose loads are in flight together
    const int B = a.B;
    const uint16_t *xsl = a.x + (int64_t)s * a.US * 256 * B;
    const int ngroups = a.US * 64;  // a multiple of 32: every lane of a warp takes part
    auto first_row = [&](int gi) {
        const int th = gi & 7, t = th >> 1, h = th & 1;
        const int lh = (gi >> 3) & 1, c = (gi >> 4) & 3, j = gi >> 6;
        return (FMT == kFmtQ6_K) ? j * 256 + 128 * (c >> 1) + 32 * (c & 1) + 64 * lh + 16 * h + 4 * t
               : (FMT == kFmtIQ4_XS) ? j * 256 + 32 * (2 * c + h) + 4 * t + 2 * lh
               : (FMT == kFmtQ8_0)   ? j * 256 + 32 * (2 * c + lh) + 16 * h + 4 * t
                                     : j * 256 + 64 * c + 32 * lh + 8 * t + 4 * h;
    };
    // x row r (0..3) of a group: e + r; IQ4_XS e + (r & 1) + 16 (r >> 1); Q8_0 e, e+2, e+1, e+3
    // (its fragment registers pair consecutive weights)
    auto row_off = [](int r) {
        return (FMT == kFmtIQ4_XS) ? (r & 1) + 16 * (r >> 1) : (FMT == kFmtQ8_0) ? ((r & 1) << 1) | (r >> 1) : r;
    };
    for (int g0 = threadIdx.x; g0 < ngroups; g0 += NB * blockDim.x) {
        uint32_t rw[NB][4][W];  // raw x rows: [group][row][word], zero when absent
#pragma unroll
        for (int u = 0; u < NB; ++u) {
            const int gi = g0 + u * blockDim.x;
            const int j = gi >> 6;
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int m = 0; m < W; ++m) rw[u][r][m] = 0u;
            if (gi < ngroups && j < US_s) {
                const int e = first_row(gi);
                const uint16_t *src = xsl + (int64_t)e * B;
                const uintptr_t addr = reinterpret_cast<uintptr_t>(src);
                if (FMT != kFmtIQ4_XS && B == BP && BP >= 2 && (addr & 15) == 0) {
                    // 4 rows x BP halves = 2 BP words, contiguous: BP / 2 16-byte loads (Q8_0: the
                    // rows' slots in the order e, e+2, e+1, e+3)
#pragma unroll
                    for (int q = 0; q < BP / 2; ++q) {
                        const uint4 v = reinterpret_cast<const uint4 *>(src)[q];
                        const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int r = (4 * q + k) / W;
                            rw[u][(FMT == kFmtQ8_0) ? row_off(r) : r][(4 * q + k) % W] = vv[k];
                        }
                    }
                } else if (FMT == kFmtIQ4_XS && B == BP && BP >= 4 && (addr & 15) == 0) {
                    // two runs of 2 rows (e, e + 1 and e + 16, e + 17): BP / 4 16-byte loads each
#pragma unroll
                    for (int run = 0; run < 2; ++run)
#pragma unroll
                        for (int q = 0; q < BP / 4; ++q) {
                            const uint4 v = reinterpret_cast<const uint4 *>(src + 16 * run * B)[q];
                            const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                rw[u][2 * run + (4 * q + k) / W][(4 * q + k) % W] = vv[k];
                        }
                } else if (FMT == kFmtIQ4_XS && B == BP && BP == 2 && (addr & 7) == 0) {
#pragma unroll
                    for (int run = 0; run < 2; ++run) {
                        const uint2 v = *reinterpret_cast<const uint2 *>(src + 16 * run * B);
                        rw[u][2 * run][0] = v.x;
                        rw[u][2 * run + 1][0] = v.y;
                    }
                } else if (FMT != kFmtIQ4_XS && FMT != kFmtQ8_0 && B == 1 && BP == 1 && (addr & 7) == 0) {
                    const uint2 v = *reinterpret_cast<const uint2 *>(src);
                    rw[u][0][0] = v.x & 0xFFFFu; rw[u][1][0] = v.x >> 16;
                    rw[u][2][0] = v.y & 0xFFFFu; rw[u][3][0] = v.y >> 16;
                } else {
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int col = 0; col < BP; ++col)
                            if (col < B)
                                rw[u][r][col >> 1] |= (uint32_t)src[row_off(r) * B + col] << (16 * (col & 1));
                }
            }
        }
#pragma unroll
        for (int u = 0; u < NB; ++u) {
            const int gi = g0 + u * blockDim.x;
            if (gi >= ngroups) break;  // uniform across the warp (ngroups and blockDim: multiples of 32)
            const int th = gi & 7, t = th >> 1, h = th & 1;
            const int lh = (gi >> 3) & 1, c = (gi >> 4) & 3, j = gi >> 6;
            if (FMT != kFmtIQ4_XS && FMT != kFmtQ8_0) {  // (neither has an offset or a min)
                // column sums of the 4 rows in fp32: (x0 + x1) + (x2 + x3)
                float sc[BP];
#pragma unroll
                for (int m = 0; m < W; ++m) {
                    float2 f[4];
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        __half2 hh;
                        *reinterpret_cast<uint32_t *>(&hh) = rw[u][r][m];
                        f[r] = __half22float2(hh);
                    }
                    const float2 sm = __fadd2_rn(__fadd2_rn(f[0], f[1]), __fadd2_rn(f[2], f[3]));
                    sc[2 * m] = sm.x;
                    if (2 * m + 1 < BP) sc[2 * m + 1] = sm.y;
                }
                if (FMT == kFmtQ6_K) {
                    // the 4 lanes t = 0..3 of (c, lh, h) (th = 2t + h): xor over th bits 1 and 2
#pragma unroll
                    for (int col = 0; col < BP; ++col) {
                        float sum = sc[col];
                        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
                        sum += __shfl_xor_sync(0xffffffffu, sum, 4);
                        if (t == 0)
                            xsum[rows_xsum_off<BP, 16>(a.US, j, 8 * (c >> 1) + 2 * (c & 1) + h + 4 * lh, col)] = sum;
                    }
                } else {
                    xsum_butterfly<BP, 4>(sc, th);
                    if (BP >= 8) {
#pragma unroll
                        for (int i = 0; i < (BP >= 8 ? BP / 8 : 1); ++i)
                            xsum[rows_xsum_off<BP>(a.US, j, 2 * c + lh, th * (BP / 8) + i)] = sc[i];
                    } else {
                        constexpr int SH = BP == 4 ? 1 : BP == 2 ? 2 : 3;  // 3 - log2 BP
                        if ((th & ((1 << SH) - 1)) == 0)
                            xsum[rows_xsum_off<BP>(a.US, j, 2 * c + lh, th >> SH)] = sc[0];
                    }
                }
            }
            // fragments: (x[r0][col], x[r2][col]), (x[r1][col], x[r3][col])
            const int swz = mma_xf_swz(c, lh, h, BP);
#pragma unroll
            for (int col = 0; col < BP; ++col) {
                const uint32_t sel = (col & 1) ? 0x7632u : 0x5410u;
                xf[mma_xf_idx(j, c, lh, h, col ^ swz, t, BP)] =
                    make_uint2(__byte_perm(rw[u][0][col >> 1], rw[u][2][col >> 1], sel),
                               __byte_perm(rw[u][1][col >> 1], rw[u][3][col >> 1], sel));
            }
        }
    }
}

// One step: 32 rows (two 16-row tiles) x one superblock (unit j of the slice) at u0 (row stride
// 144 B; Q5_K 176 B).  acc: C-fragment accumulators of the warp's rows; accM: this lane's row
// (row = lane), the min term.  Rows are placed in the warp's table dtab at position
// (row % 8) * 4 + row / 8, so that rows g, g+8, g+16, g+24 are one run.
//
// Q4_K (mma_q4k_step): the codes enter the MMA as the normal fp16 numbers q * 2^-10 (low nibbles
// masked as q * 2^-24 and multiplied by 2^14, high nibbles left in place as q * 2^-20 and
// multiplied by 2^10).  A C fragment sums one sub-block's half of a chunk for one tile (two MMAs)
// and is scaled by d * sc_j * 2^10 of its row (dtab: [8 sub-blocks][32 positions] floats).
//
// Q5_K (mma_q5k_step): the sub-block scales are folded into the A operand.  A code q of sub-block
// j enters as q * sc_j * 2^-14 (the masked subnormal q * 2^-24 times the fp16 pair sc_j * 2^10;
// dtab holds those pairs, [4 chunks][32 positions] x (low, high)); q * sc_j <= 31 * 63 < 2^11, so
// the product is exact and normal (or zero).  The C fragments then sum a whole superblock and are
// scaled once per step by d * 2^14 of their row:
//   sum_i w_i x_i = d * 2^14 * sum_i (q_i sc_j(i) 2^-14) x_i  -  sum_j dmin m_j X_j.
// Measured on B200: folding saves Q5_K about 1.5 us per 17408 x 5120 call at B = 8 (its A words
// cost more instructions, which folding offsets), while for Q4_K the longer MMA accumulation
// chains cost more than the saved scaling instructions (0.5 us slower at B = 8).
// Q5_K: the A codes of one qs word w and its qh word hw (bytes l..l+3 of chunk c): the low nibbles
// with their fifth bit (bit 2c of each qh byte) and the high nibbles with theirs (bit 2c + 1), each
// merged into a byte as q = nibble | bit << 4, masked as subnormals q * 2^-24: lo0 / hi0 = bytes 0
// and 2, lo1 / hi1 = bytes 1 and 3.
template <int C>
__device__ __forceinline__ void q5k_a_codes(uint32_t w, uint32_t hw, uint32_t &lo0, uint32_t &lo1,
                                            uint32_t &hi0, uint32_t &hi1)
{
    const uint32_t t1 = (C == 0) ? hw << 4 : (C == 1) ? hw << 2 : (C == 2) ? hw : hw >> 2;
    const uint32_t t2 = (C == 0) ? hw << 3 : (C == 1) ? hw << 1 : (C == 2) ? hw >> 1 : hw >> 3;
    const uint32_t wl = (w & 0x0F0F0F0Fu) | (t1 & 0xF0F0F0F0u);
    const uint32_t wh = ((w >> 4) & 0x0F0F0F0Fu) | (t2 & 0xF0F0F0F0u);
    lo0 = wl & 0x001F001Fu;
    lo1 = __umulhi(wl, 1u << 24) & 0x001F001Fu;  // >> 8 on the FMA pipe
    hi0 = wh & 0x001F001Fu;
    hi1 = __umulhi(wh, 1u << 24) & 0x001F001Fu;
}

// Row of a 16-row tile that fragment row g (lane >> 2) of mma.m16n8k16 stands for, in the Q4_K /
// Q5_K steps: 2 (g mod 4) + g / 4.  Each half-warp's 8-byte A loads then read rows {0, 2, 4, 6}
// or {1, 3, 5, 7}, which start 16 or 24 banks apart at the 144- and 176-byte row strides of the
// ring (36 and 44 words), so the loads are free of bank conflicts; rows g = 0..3 in order would
// start 4 (Q4_K) or 12 (Q5_K) banks apart and collide two-way.  Rows are independent outputs,
// so the map only decides where each C fragment row lands.
template <int FMT>
__device__ __forceinline__ int mma_frag_row(int g)
{
    return (FMT == kFmtQ6_K) ? g : 2 * (g & 3) + (g >> 2);
}

template <int BP>
__device__ __forceinline__ void mma_q4k_step(const uint8_t *u0, const uint2 *xf, const float *xsum,
                                             int US, int j, float *dtab,
                                             float (&acc)[2][MmaNT<BP>::value][4], float (&accM)[BP],
                                             int lane)
{
    constexpr int FMT = kFmtQ4_K;
    constexpr int UB = MmaFmt<FMT>::kUnitBytes;
    constexpr int QS = MmaFmt<FMT>::kQs;
    const int g = lane >> 2, t = lane & 3;
    const int pr = mma_frag_row<FMT>(g);  // the tile row of fragment row g
    {
        // header of row `lane`: the GGML get_scale_min_k4 table decoded with 32-bit masks (byte k
        // of each word = sub-block k or k+4), d and dmin exact in fp32
        const uint4 hdr = *reinterpret_cast<const uint4 *>(u0 + lane * UB);
        const uint32_t SC_lo = hdr.y & 0x3F3F3F3Fu;
        const uint32_t MM_lo = hdr.z & 0x3F3F3F3Fu;
        const uint32_t SC_hi = (hdr.w & 0x0F0F0F0Fu) | ((hdr.y >> 2) & 0x30303030u);
        const uint32_t MM_hi = ((hdr.w >> 4) & 0x0F0F0F0Fu) | ((hdr.z >> 2) & 0x30303030u);
        __half2 dd;
        *reinterpret_cast<uint32_t *>(&dd) = hdr.x;
        const float2 dm = __half22float2(dd);
        const float2 dscale = f2(dm.x, dm.x);
        const int pos = (lane & 7) * 4 + (lane >> 3);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint32_t scw = c < 2 ? SC_lo : SC_hi;
            const uint32_t mmw = c < 2 ? MM_lo : MM_hi;
            const uint32_t sel = 0x7650u + 2u * (c & 1);
            // 6-bit integers to float through the 2^23 mantissa: (2^23 + v) - 2^23
            const float2 sc = __fadd2_rn(f2(__uint_as_float(__byte_perm(scw, 0x4B000000u, sel)),
                                            __uint_as_float(__byte_perm(scw, 0x4B000000u, sel + 1))),
                                         f2(-8388608.0f, -8388608.0f));
            const float2 mm = __fadd2_rn(f2(__uint_as_float(__byte_perm(mmw, 0x4B000000u, sel)),
                                            __uint_as_float(__byte_perm(mmw, 0x4B000000u, sel + 1))),
                                         f2(-8388608.0f, -8388608.0f));
            const float2 D = __fmul2_rn(dscale, sc);
            const float2 M = __fmul2_rn(f2(dm.y, dm.y), mm);
            dtab[(2 * c) * 32 + pos] = D.x * 1024.0f;  // the codes are q 2^-10
            dtab[(2 * c + 1) * 32 + pos] = D.y * 1024.0f;
            // the min term: -M_j X_j
#pragma unroll
            for (int b = 0; b < BP; ++b) {
                accM[b] = fmaf(-M.x, xsum[rows_xsum_off<BP>(US, j, 2 * c, b)], accM[b]);
                accM[b] = fmaf(-M.y, xsum[rows_xsum_off<BP>(US, j, 2 * c + 1, b)], accM[b]);
            }
        }
    }
    __syncwarp();
    // n-tile nt covers columns 8nt .. 8nt+7 (one tile for BP <= 8); lane g supplies column 8nt + g
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint2 xb[MmaNT<BP>::value][2][2];
#pragma unroll
        for (int nt = 0; nt < MmaNT<BP>::value; ++nt)
#pragma unroll
            for (int lh = 0; lh < 2; ++lh)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int col = (BP > 8) ? 8 * nt + g : g % BP;
                    xb[nt][lh][h] = xf[mma_xf_idx(j, c, lh, h, col ^ mma_xf_swz(c, lh, h, BP), t, BP)];
                }
        const float4 Dlo = *reinterpret_cast<const float4 *>(dtab + (2 * c) * 32 + 4 * pr);
        const float4 Dhi = *reinterpret_cast<const float4 *>(dtab + (2 * c + 1) * 32 + 4 * pr);
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
            const uint8_t *rowA = u0 + (tile * 16 + pr) * UB + QS + 32 * c + 8 * t;
            const uint2 wA = *reinterpret_cast<const uint2 *>(rowA);           // row tile*16 + pr
            const uint2 wB = *reinterpret_cast<const uint2 *>(rowA + 8 * UB);  // row tile*16 + pr + 8
            float cl[MmaNT<BP>::value][4], ch[MmaNT<BP>::value][4];
#pragma unroll
            for (int nt = 0; nt < MmaNT<BP>::value; ++nt)
#pragma unroll
                for (int k = 0; k < 4; ++k) cl[nt][k] = ch[nt][k] = 0.0f;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t wa = h ? wA.y : wA.x, wb = h ? wB.y : wB.x;
                uint32_t l0, l1, l2, l3, h0, h1, h2, h3;
                {
                    // low nibbles masked as q 2^-24, high nibbles left in place as q 2^-20, then
                    // made the normal fp16 numbers q 2^-10 (word >> 8 as a multiply-high on the
                    // FMA pipe for bytes 1 and 3)
                    const uint32_t va = __umulhi(wa, 1u << 24), vb = __umulhi(wb, 1u << 24);
                    l0 = f16x2_mul(wa & 0x000F000Fu, kF16x2_2p14);  // low nibbles, bytes 0 and 2
                    l1 = f16x2_mul(wb & 0x000F000Fu, kF16x2_2p14);
                    l2 = f16x2_mul(va & 0x000F000Fu, kF16x2_2p14);  // low nibbles, bytes 1 and 3
                    l3 = f16x2_mul(vb & 0x000F000Fu, kF16x2_2p14);
                    h0 = f16x2_mul(wa & 0x00F000F0u, kF16x2_2p10);  // high nibbles, bytes 0 and 2
                    h1 = f16x2_mul(wb & 0x00F000F0u, kF16x2_2p10);
                    h2 = f16x2_mul(va & 0x00F000F0u, kF16x2_2p10);  // high nibbles, bytes 1 and 3
                    h3 = f16x2_mul(vb & 0x00F000F0u, kF16x2_2p10);
                }
#pragma unroll
                for (int nt = 0; nt < MmaNT<BP>::value; ++nt) {
                    mma_16816(cl[nt], l0, l1, l2, l3, xb[nt][0][h].x, xb[nt][0][h].y);
                    mma_16816(ch[nt], h0, h1, h2, h3, xb[nt][1][h].x, xb[nt][1][h].y);
                }
            }
            const float la = tile ? Dlo.z : Dlo.x, lb = tile ? Dlo.w : Dlo.y;
            const float ha = tile ? Dhi.z : Dhi.x, hb = tile ? Dhi.w : Dhi.y;
#pragma unroll
            for (int nt = 0; nt < MmaNT<BP>::value; ++nt) {
                acc[tile][nt][0] = fmaf(ha, ch[nt][0], fmaf(la, cl[nt][0], acc[tile][nt][0]));
                acc[tile][nt][2] = fmaf(hb, ch[nt][2], fmaf(lb, cl[nt][2], acc[tile][nt][2]));
                if (BP > 1) {
                    acc[tile][nt][1] = fmaf(ha, ch[nt][1], fmaf(la, cl[nt][1], acc[tile][nt][1]));
                    acc[tile][nt][3] = fmaf(hb, ch[nt][3], fmaf(lb, cl[nt][3], acc[tile][nt][3]));
                }
            }
        }
    }
}

template <int BP>
__device__ __forceinline__ void mma_q5k_step(const uint8_t *u0, const uint2 *xf, const float *xsum,
                                             int US, int j, float *dtab,
                                             float (&acc)[2][MmaNT<BP>::value][4], float (&accM)[BP],
                                             int lane)
{
    constexpr int FMT = kFmtQ5_K;
    constexpr int UB = MmaFmt<FMT>::kUnitBytes;
    constexpr int QS = MmaFmt<FMT>::kQs;
    constexpr int NT = MmaNT<BP>::value;
    constexpr int SPLIT = (NT == 1) ? 2 : 1;  // C fragments per (tile, n-tile): low / high codes
    const int g = lane >> 2, t = lane & 3;
    const int pr = mma_frag_row<FMT>(g);  // the tile row of fragment row g
    uint2 *mtab = reinterpret_cast<uint2 *>(dtab);
    float dsh;  // d * 2^14 of row `lane`
    {
        // header of row `lane`: the GGML get_scale_min_k4 table decoded with 32-bit masks (byte k
        // of each word = sub-block k or k+4), d and dmin exact in fp32
        const uint4 hdr = *reinterpret_cast<const uint4 *>(u0 + lane * UB);
        const uint32_t SC_lo = hdr.y & 0x3F3F3F3Fu;
        const uint32_t MM_lo = hdr.z & 0x3F3F3F3Fu;
        const uint32_t SC_hi = (hdr.w & 0x0F0F0F0Fu) | ((hdr.y >> 2) & 0x30303030u);
        const uint32_t MM_hi = ((hdr.w >> 4) & 0x0F0F0F0Fu) | ((hdr.z >> 2) & 0x30303030u);
        __half2 dd;
        *reinterpret_cast<uint32_t *>(&dd) = hdr.x;
        const float2 dm = __half22float2(dd);
        dsh = dm.x * 16384.0f;
        const int pos = (lane & 7) * 4 + (lane >> 3);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const uint32_t scw = c < 2 ? SC_lo : SC_hi;
            const uint32_t mmw = c < 2 ? MM_lo : MM_hi;
            const uint32_t sel = 0x7650u + 2u * (c & 1);
            // 6-bit integers to float through the 2^23 mantissa: (2^23 + v) - 2^23
            const float2 sc = __fadd2_rn(f2(__uint_as_float(__byte_perm(scw, 0x4B000000u, sel)),
                                            __uint_as_float(__byte_perm(scw, 0x4B000000u, sel + 1))),
                                         f2(-8388608.0f, -8388608.0f));
            const float2 mm = __fadd2_rn(f2(__uint_as_float(__byte_perm(mmw, 0x4B000000u, sel)),
                                            __uint_as_float(__byte_perm(mmw, 0x4B000000u, sel + 1))),
                                         f2(-8388608.0f, -8388608.0f));
            mtab[c * 32 + pos] = make_uint2(f16x2_dup(sc.x * 1024.0f), f16x2_dup(sc.y * 1024.0f));
            const float2 M = __fmul2_rn(f2(dm.y, dm.y), mm);
            // the min term: -M_j X_j
#pragma unroll
            for (int b = 0; b < BP; ++b) {
                accM[b] = fmaf(-M.x, xsum[rows_xsum_off<BP>(US, j, 2 * c, b)], accM[b]);
                accM[b] = fmaf(-M.y, xsum[rows_xsum_off<BP>(US, j, 2 * c + 1, b)], accM[b]);
            }
        }
    }
    __syncwarp();
    // the superblock's sums times d * 2^14 of their rows (rows pr and pr + 8 of each tile)
    float C[2][NT][SPLIT][4];
    auto zero_c = [&]() {
#pragma unroll
        for (int tile = 0; tile < 2; ++tile)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int sp = 0; sp < SPLIT; ++sp)
#pragma unroll
                    for (int k = 0; k < 4; ++k) C[tile][nt][sp][k] = 0.0f;
    };
    auto fold_c = [&]() {
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
            const float dA = __shfl_sync(0xffffffffu, dsh, tile * 16 + pr);
            const float dB = __shfl_sync(0xffffffffu, dsh, tile * 16 + pr + 8);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int sp = 0; sp < SPLIT; ++sp) {
                    acc[tile][nt][0] = fmaf(dA, C[tile][nt][sp][0], acc[tile][nt][0]);
                    acc[tile][nt][2] = fmaf(dB, C[tile][nt][sp][2], acc[tile][nt][2]);
                    if (BP > 1) {
                        acc[tile][nt][1] = fmaf(dA, C[tile][nt][sp][1], acc[tile][nt][1]);
                        acc[tile][nt][3] = fmaf(dB, C[tile][nt][sp][3], acc[tile][nt][3]);
                    }
                }
        }
    };
    // at 16 columns (two n-tiles sharing the A registers) the C fragments are folded per chunk,
    // which keeps them out of the registers live across the step
    constexpr bool kFoldPerChunk = (NT == 2);
    zero_c();
    // n-tile nt covers columns 8nt .. 8nt+7 (one tile for BP <= 8); lane g supplies column 8nt + g
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        if (kFoldPerChunk && c > 0) zero_c();
        uint2 xb[NT][2][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int lh = 0; lh < 2; ++lh)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int col = (BP > 8) ? 8 * nt + g : g % BP;
                    xb[nt][lh][h] = xf[mma_xf_idx(j, c, lh, h, col ^ mma_xf_swz(c, lh, h, BP), t, BP)];
                }
        // multipliers of rows pr, pr + 8 (tile 0) and pr + 16, pr + 24 (tile 1): (low, high) pairs
        const uint4 m0 = *reinterpret_cast<const uint4 *>(mtab + c * 32 + 4 * pr);
        const uint4 m1 = *reinterpret_cast<const uint4 *>(mtab + c * 32 + 4 * pr + 2);
        // the A words of both tiles: rows tile*16 + pr and tile*16 + pr + 8
        uint2 wA[2], wB[2], qhA[2], qhB[2];
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
            const uint8_t *rowA = u0 + (tile * 16 + pr) * UB + QS + 32 * c + 8 * t;
            wA[tile] = *reinterpret_cast<const uint2 *>(rowA);
            wB[tile] = *reinterpret_cast<const uint2 *>(rowA + 8 * UB);
            const uint8_t *qhp = u0 + (tile * 16 + pr) * UB + 16 + 8 * t;  // qh words 2t, 2t+1
            qhA[tile] = *reinterpret_cast<const uint2 *>(qhp);
            qhB[tile] = *reinterpret_cast<const uint2 *>(qhp + 8 * UB);
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            // A registers of both tiles, then their MMAs interleaved so that no MMA waits on the
            // one just issued
            uint32_t A[2][2][4];  // [tile][low / high codes][register]
#pragma unroll
            for (int tile = 0; tile < 2; ++tile) {
                const uint4 m = tile ? m1 : m0;
                const uint32_t wa = h ? wA[tile].y : wA[tile].x, wb = h ? wB[tile].y : wB[tile].x;
                uint32_t l0, l1, l2, l3, h0, h1, h2, h3;  // masked codes (subnormal fp16 pairs)
                const uint32_t ha = h ? qhA[tile].y : qhA[tile].x, hb = h ? qhB[tile].y : qhB[tile].x;
                switch (c) {  // c is a compile-time constant after unrolling
                case 0: q5k_a_codes<0>(wa, ha, l0, l2, h0, h2); q5k_a_codes<0>(wb, hb, l1, l3, h1, h3); break;
                case 1: q5k_a_codes<1>(wa, ha, l0, l2, h0, h2); q5k_a_codes<1>(wb, hb, l1, l3, h1, h3); break;
                case 2: q5k_a_codes<2>(wa, ha, l0, l2, h0, h2); q5k_a_codes<2>(wb, hb, l1, l3, h1, h3); break;
                default: q5k_a_codes<3>(wa, ha, l0, l2, h0, h2); q5k_a_codes<3>(wb, hb, l1, l3, h1, h3); break;
                }
                // times sc * 2^10: q sc 2^-14, exact and normal
                A[tile][0][0] = f16x2_mul(l0, m.x);
                A[tile][0][2] = f16x2_mul(l2, m.x);
                A[tile][0][1] = f16x2_mul(l1, m.z);
                A[tile][0][3] = f16x2_mul(l3, m.z);
                A[tile][1][0] = f16x2_mul(h0, m.y);
                A[tile][1][2] = f16x2_mul(h2, m.y);
                A[tile][1][1] = f16x2_mul(h1, m.w);
                A[tile][1][3] = f16x2_mul(h3, m.w);
            }
#pragma unroll
            for (int lh = 0; lh < 2; ++lh)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int tile = 0; tile < 2; ++tile)
                        mma_16816(C[tile][nt][lh * (SPLIT - 1)], A[tile][lh][0], A[tile][lh][1], A[tile][lh][2],
                                  A[tile][lh][3], xb[nt][lh][h].x, xb[nt][lh][h].y);
        }
        if (kFoldPerChunk) fold_c();
    }
    if (!kFoldPerChunk) fold_c();
}

// One IQ4_XS step: 32 rows (two 16-row tiles) x one superblock at u0 (row stride 144 B; the unit
// starts `o` = 0 or 8 bytes into each row's window).  Thread (g, t) takes qs word t + 4h of chunk c
// of rows g and g + 8 of a tile (sub-block 2c + h, weights 4t .. 4t+3 and 16 + 4t .. 16 + 4t+3),
// looks its eight indices up in the codebook (iq4_lookup: biased levels u = level + 128, a byte
// each, in nibble order), spreads two bytes under the exponent of 1024 (one byte permute per
// register: the fp16 pair 1024 + u) and takes 1152 out with one f16x2 add, leaving the levels as
// exact fp16 integers (-127..113, all normal).  The MMA of k-half lh takes qs bytes 2lh, 2lh + 1
// of the word, so a register holds the weights (r, r + 16) of one byte; x is staged in that order
// (mma_stage_x).  Both MMAs of (c, h) sum into one C fragment of sub-block 2c + h, scaled by
// d (ls - 32) of its row (dtab: [8 sub-blocks][32 positions]).
template <int BP>
__device__ __forceinline__ void mma_iq4xs_step(const uint8_t *u0, int o, const uint2 *xf, int j,
                                               float *dtab, float (&acc)[2][MmaNT<BP>::value][4],
                                               int lane)
{
    constexpr int FMT = kFmtIQ4_XS;
    constexpr int LB = MmaFmt<FMT>::kUnitBytes;
    constexpr int NT = MmaNT<BP>::value;
    const int g = lane >> 2, t = lane & 3;
    const int pr = mma_frag_row<FMT>(g);
    const uint8_t *unit = u0 + o;
    {
        // header of row `lane`: d (bytes 0-1), scales_h (2-3), scales_l (4-7)
        const uint32_t w0 = *reinterpret_cast<const uint32_t *>(unit + lane * LB);
        const uint32_t sl = *reinterpret_cast<const uint32_t *>(unit + lane * LB + 4);
        const uint32_t sh = w0 >> 16;
        const float d = __half2float(__ushort_as_half((unsigned short)(w0 & 0xFFFFu)));
        const int pos = (lane & 7) * 4 + (lane >> 3);
#pragma unroll
        for (int sb = 0; sb < 8; ++sb) {
            const int ls = (int)(((sl >> (4 * sb)) & 15u) | (((sh >> (2 * sb)) & 3u) << 4));
            dtab[sb * 32 + pos] = d * (float)(ls - 32);  // exact: an fp16 times a 6-bit integer
        }
    }
    __syncwarp();
    // two biased bytes of v (selector: bytes 0 and 2, or 1 and 3) -> the fp16 levels u - 128
    auto levels = [](uint32_t v, uint32_t sel) {  // sel 0x4140: bytes 0, 1; 0x4342: bytes 2, 3
        const uint32_t p = __byte_perm(v, 0x64646464u, sel);  // (1024 + u, 1024 + u')
        uint32_t r;
        asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(p), "r"(0xE480E480u));  // - (1152, 1152)
        return r;
    };
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint2 xb[NT][2][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int lh = 0; lh < 2; ++lh)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int col = (BP > 8) ? 8 * nt + g : g % BP;
                    xb[nt][lh][h] = xf[mma_xf_idx(j, c, lh, h, col ^ mma_xf_swz(c, lh, h, BP), t, BP)];
                }
        const float4 D0 = *reinterpret_cast<const float4 *>(dtab + (2 * c) * 32 + 4 * pr);
        const float4 D1 = *reinterpret_cast<const float4 *>(dtab + (2 * c + 1) * 32 + 4 * pr);
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
            const uint8_t *rowA = unit + (tile * 16 + pr) * LB + MmaFmt<FMT>::kQs + 32 * c + 4 * t;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t wa = *reinterpret_cast<const uint32_t *>(rowA + 16 * h);
                const uint32_t wb = *reinterpret_cast<const uint32_t *>(rowA + 16 * h + 8 * LB);
                uint32_t loA, hiA, loB, hiB;
                iq4_lookup(wa, loA, hiA);
                iq4_lookup(wb, loB, hiB);
                float cs[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int k = 0; k < 4; ++k) cs[nt][k] = 0.0f;
                // lo = levels of qs bytes 0, 1 (low, high nibble each), hi = of bytes 2, 3: the
                // pairs (byte b low, byte b high) are weights (4t + b, 4t + b + 16)
                {
                    const uint32_t a0 = levels(loA, 0x4140u), a1 = levels(loB, 0x4140u);
                    const uint32_t a2 = levels(loA, 0x4342u), a3 = levels(loB, 0x4342u);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_16816(cs[nt], a0, a1, a2, a3, xb[nt][0][h].x, xb[nt][0][h].y);
                }
                {
                    const uint32_t a0 = levels(hiA, 0x4140u), a1 = levels(hiB, 0x4140u);
                    const uint32_t a2 = levels(hiA, 0x4342u), a3 = levels(hiB, 0x4342u);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_16816(cs[nt], a0, a1, a2, a3, xb[nt][1][h].x, xb[nt][1][h].y);
                }
                const float4 D = h ? D1 : D0;
                const float da = tile ? D.z : D.x, db = tile ? D.w : D.y;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    acc[tile][nt][0] = fmaf(da, cs[nt][0], acc[tile][nt][0]);
                    acc[tile][nt][2] = fmaf(db, cs[nt][2], acc[tile][nt][2]);
                    if (BP > 1) {
                        acc[tile][nt][1] = fmaf(da, cs[nt][1], acc[tile][nt][1]);
                        acc[tile][nt][3] = fmaf(db, cs[nt][3], acc[tile][nt][3]);
                    }
                }
            }
        }
    }
}

// One Q8_0 step: 32 rows (two 16-row tiles) x one 272-byte unit (8 blocks of 32 weights) at u0.
// k-tile (block 2c + lh, half h) of a row holds qs bytes 16h .. 16h+15 of the block; thread (g, t)
// takes the 4 bytes 16h + 4t .. +3 (weights e .. e+3, e = 32 (2c + lh) + 16h + 4t) of rows g and
// g + 8: one 32-bit load (odd blocks start 4-byte aligned; even ones 2 bytes past, read as a funnel
// shift of two words), an XOR with 0x80 per byte (q + 128, as unsigned bytes), one byte permute per
// register under the exponent of 1024 (the fp16 pair 1024 + q + 128) and one f16x2 add of -1152:
// the int8 codes as exact fp16 integers.  A register pairs consecutive weights (e, e+1) or
// (e+2, e+3); x is staged in that order.  Both k-tiles of a block sum into one C fragment, scaled by
// the block's d of its row (dtab: [8 blocks][32 positions]).
template <int BP>
__device__ __forceinline__ void mma_q8_step(const uint8_t *u0, const uint2 *xf, int j, float *dtab,
                                            float (&acc)[2][MmaNT<BP>::value][4], int lane)
{
    constexpr int FMT = kFmtQ8_0;
    constexpr int LB = MmaFmt<FMT>::kUnitBytes;
    constexpr int NT = MmaNT<BP>::value;
    const int g = lane >> 2, t = lane & 3;
    const int pr = mma_frag_row<FMT>(g);
    {
        // the 8 block scales of row `lane`
        const uint8_t *row = u0 + lane * LB;
        const int pos = (lane & 7) * 4 + (lane >> 3);
#pragma unroll
        for (int b = 0; b < 8; ++b)
            dtab[b * 32 + pos] = __half2float(*reinterpret_cast<const __half *>(row + 34 * b));
    }
    __syncwarp();
    auto code_word = [&](const uint8_t *row, int blk, int h) {
        const int off = 34 * blk + MmaFmt<FMT>::kQs + 16 * h + 4 * t;  // 4-byte aligned iff blk odd
        uint32_t w;
        if (blk & 1) {
            w = *reinterpret_cast<const uint32_t *>(row + off);
        } else {
            const uint32_t *p = reinterpret_cast<const uint32_t *>(row + off - 2);
            w = __funnelshift_r(p[0], p[1], 16);
        }
        return w ^ 0x80808080u;  // q + 128 per byte
    };
    auto codes = [](uint32_t v, uint32_t sel) {  // sel 0x4140: bytes 0, 1; 0x4342: bytes 2, 3
        const uint32_t p = __byte_perm(v, 0x64646464u, sel);  // (1024 + q + 128, ...)
        uint32_t r;
        asm("add.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(p), "r"(0xE480E480u));  // - (1152, 1152)
        return r;
    };
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint2 xb[NT][2][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int lh = 0; lh < 2; ++lh)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int col = (BP > 8) ? 8 * nt + g : g % BP;
                    xb[nt][lh][h] = xf[mma_xf_idx(j, c, lh, h, col ^ mma_xf_swz(c, lh, h, BP), t, BP)];
                }
        const float4 D0 = *reinterpret_cast<const float4 *>(dtab + (2 * c) * 32 + 4 * pr);
        const float4 D1 = *reinterpret_cast<const float4 *>(dtab + (2 * c + 1) * 32 + 4 * pr);
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
            const uint8_t *rowA = u0 + (tile * 16 + pr) * LB;
            const uint8_t *rowB = rowA + 8 * LB;
#pragma unroll
            for (int lh = 0; lh < 2; ++lh) {
                const int blk = 2 * c + lh;
                float cs[NT][4];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int k = 0; k < 4; ++k) cs[nt][k] = 0.0f;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t vA = code_word(rowA, blk, h), vB = code_word(rowB, blk, h);
                    const uint32_t a0 = codes(vA, 0x4140u), a1 = codes(vB, 0x4140u);
                    const uint32_t a2 = codes(vA, 0x4342u), a3 = codes(vB, 0x4342u);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
                        mma_16816(cs[nt], a0, a1, a2, a3, xb[nt][lh][h].x, xb[nt][lh][h].y);
                }
                const float4 D = lh ? D1 : D0;
                const float da = tile ? D.z : D.x, db = tile ? D.w : D.y;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    acc[tile][nt][0] = fmaf(da, cs[nt][0], acc[tile][nt][0]);
                    acc[tile][nt][2] = fmaf(db, cs[nt][2], acc[tile][nt][2]);
                    if (BP > 1) {
                        acc[tile][nt][1] = fmaf(da, cs[nt][1], acc[tile][nt][1]);
                        acc[tile][nt][3] = fmaf(db, cs[nt][3], acc[tile][nt][3]);
                    }
                }
            }
        }
    }
}

// One Q6_K step: 32 rows x one superblock from the warp's per-lane windows at u0 (window of row
// r at u0 + 240 r; its superblock starts o_r = (m_r * 210) mod 16 bytes in, m_r its superblock
// index in the tensor).  Chunk c = 2hf + p is ql[64hf + 32p ..]; its k-tile kk (words 4kk .. 4kk+3)
// is one 16-weight scale group for the low nibbles (group 8hf + 2p + kk) and one for the high
// nibbles (4 groups later), so each k-tile's C fragments are scaled by one D_t per row.  A words:
// thread (g, t) takes ql word 16hf + 8p + 4kk + t and qh word 32 + 8hf + 4kk + t of rows g and
// g + 8 of the tile; their two high bits (bits 2p, 2p+1 for the low nibbles, 2p+4, 2p+5 for the
// high ones) are merged byte-wise next to the nibbles and the 6-bit values q enter the MMA as the
// normal fp16 numbers q 2^-10 (the D_t table holds d sc_t 2^10).  The offset is applied per group
// through the x sums: sum (q - 32) x = sum q x - 32 X_t.
template <int BP>
__device__ __forceinline__ void mma_q6k_step(const uint8_t *u0, const uint2 *xf, const float *xsum,
                                             int US, int j, float *dtab,
                                             float (&acc)[2][MmaNT<BP>::value][4], float (&accM)[BP],
                                             int lane, const RowsArgs &a, int64_t row0, int unit,
                                             const uint8_t *wbase)
{
    constexpr int LB = MmaFmt<kFmtQ6_K>::kUnitBytes;
    const int g = lane >> 2, t = lane & 3;
    {
        // header of row `lane`: 16 int8 scales (bytes 192..207) and d (208..209)
        const int64_t row = row0 + lane;
        const int64_t m = row * a.UPR + unit;
        const int o = (int)((m * 210) & 15);
        const uint32_t *wp = reinterpret_cast<const uint32_t *>(u0 + lane * LB) + (o >> 2);
        const uint32_t sh = (o & 2) ? 16u : 0u;
        uint32_t scw[4], dw;
        if (!(a.wtail && row == a.N - 1 && unit == a.UPR - 1)) {
#pragma unroll
            for (int k = 0; k < 4; ++k) scw[k] = __funnelshift_r(wp[48 + k], wp[49 + k], sh);
            dw = __funnelshift_r(wp[52], wp[53], sh);
        } else {
            // the tensor's last superblock: its copy window stopped at the last 16-byte boundary
            const uint8_t *gb = wbase + m * 210;
#pragma unroll
            for (int k = 0; k < 4; ++k)
                scw[k] = (uint32_t)gb[192 + 4 * k] | ((uint32_t)gb[193 + 4 * k] << 8) |
                         ((uint32_t)gb[194 + 4 * k] << 16) | ((uint32_t)gb[195 + 4 * k] << 24);
            dw = (uint32_t)gb[208] | ((uint32_t)gb[209] << 8);
        }
        const float ds = __half2float(__ushort_as_half((unsigned short)(dw & 0xFFFFu)));
        const int pos = (lane & 7) * 4 + (lane >> 3);
#pragma unroll
        for (int tg = 0; tg < 16; ++tg) {
            const float D = ds * (float)(int8_t)(scw[tg >> 2] >> (8 * (tg & 3)));
            dtab[tg * 32 + pos] = D * 1024.0f;  // the codes are q 2^-10
            // sum (q - 32) x = sum q x - 32 X_t
#pragma unroll
            for (int b = 0; b < BP; ++b)
                accM[b] = fmaf(D * -32.0f, xsum[rows_xsum_off<BP, 16>(US, j, tg, b)], accM[b]);
        }
    }
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int hf = c >> 1, p = c & 1;
        uint2 xb[MmaNT<BP>::value][2][2];
#pragma unroll
        for (int nt = 0; nt < MmaNT<BP>::value; ++nt)
#pragma unroll
            for (int lh = 0; lh < 2; ++lh)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int col = (BP > 8) ? 8 * nt + g : g % BP;
                    xb[nt][lh][h] = xf[mma_xf_idx(j, c, lh, h, col ^ mma_xf_swz(c, lh, h, BP), t, BP)];
                }
#pragma unroll
        for (int tile = 0; tile < 2; ++tile) {
            // the two rows of this thread in the tile, their windows and misalignments
            const int rA = tile * 16 + g, rB = rA + 8;
            const int64_t mA = (row0 + rA) * a.UPR + unit, mB = (row0 + rB) * a.UPR + unit;
            const int oA = (int)((mA * 210) & 15), oB = (int)((mB * 210) & 15);
            const uint32_t *wa_p = reinterpret_cast<const uint32_t *>(u0 + rA * LB) + (oA >> 2);
            const uint32_t *wb_p = reinterpret_cast<const uint32_t *>(u0 + rB * LB) + (oB >> 2);
            const uint32_t sA = (oA & 2) ? 16u : 0u, sB = (oB & 2) ? 16u : 0u;
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                const int ql = 16 * hf + 8 * p + 4 * kk + t, qh = 32 + 8 * hf + 4 * kk + t;
                const uint32_t wa = __funnelshift_r(wa_p[ql], wa_p[ql + 1], sA);
                const uint32_t ha = __funnelshift_r(wa_p[qh], wa_p[qh + 1], sA);
                const uint32_t wb = __funnelshift_r(wb_p[ql], wb_p[ql + 1], sB);
                const uint32_t hb = __funnelshift_r(wb_p[qh], wb_p[qh + 1], sB);
                // bits 2p, 2p+1 (low nibbles) and 2p+4, 2p+5 (high nibbles) of each qh byte -> bits 4, 5
                const uint32_t t1a = p ? ha << 2 : ha << 4, t2a = p ? ha >> 2 : ha;
                const uint32_t t1b = p ? hb << 2 : hb << 4, t2b = p ? hb >> 2 : hb;
                const uint32_t wla = (wa & 0x0F0F0F0Fu) | (t1a & 0xF0F0F0F0u);
                const uint32_t wha = ((wa >> 4) & 0x0F0F0F0Fu) | (t2a & 0xF0F0F0F0u);
                const uint32_t wlb = (wb & 0x0F0F0F0Fu) | (t1b & 0xF0F0F0F0u);
                const uint32_t whb = ((wb >> 4) & 0x0F0F0F0Fu) | (t2b & 0xF0F0F0F0u);
                // the 6-bit codes masked as subnormals q 2^-24 (bytes 1 and 3 through a
                // multiply-high by 2^24), then made the normal fp16 numbers q 2^-10 (qg_codes.cuh)
                constexpr uint32_t M6 = 0x003F003Fu;
                const uint32_t l0 = f16x2_mul(wla & M6, kF16x2_2p14), l1 = f16x2_mul(wlb & M6, kF16x2_2p14);
                const uint32_t l2 = f16x2_mul(__umulhi(wla, 1u << 24) & M6, kF16x2_2p14);
                const uint32_t l3 = f16x2_mul(__umulhi(wlb, 1u << 24) & M6, kF16x2_2p14);
                const uint32_t h0 = f16x2_mul(wha & M6, kF16x2_2p14), h1 = f16x2_mul(whb & M6, kF16x2_2p14);
                const uint32_t h2 = f16x2_mul(__umulhi(wha, 1u << 24) & M6, kF16x2_2p14);
                const uint32_t h3 = f16x2_mul(__umulhi(whb, 1u << 24) & M6, kF16x2_2p14);
                const int tlo = 8 * hf + 2 * p + kk;
                const float4 Dlo = *reinterpret_cast<const float4 *>(dtab + tlo * 32 + 4 * g);
                const float4 Dhi = *reinterpret_cast<const float4 *>(dtab + (tlo + 4) * 32 + 4 * g);
                const float la = tile ? Dlo.z : Dlo.x, lb = tile ? Dlo.w : Dlo.y;
                const float ha_s = tile ? Dhi.z : Dhi.x, hb_s = tile ? Dhi.w : Dhi.y;
#pragma unroll
                for (int nt = 0; nt < MmaNT<BP>::value; ++nt) {
                    float cl[4] = {0.0f, 0.0f, 0.0f, 0.0f}, ch[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                    mma_16816(cl, l0, l1, l2, l3, xb[nt][0][kk].x, xb[nt][0][kk].y);
                    mma_16816(ch, h0, h1, h2, h3, xb[nt][1][kk].x, xb[nt][1][kk].y);
                    acc[tile][nt][0] = fmaf(ha_s, ch[0], fmaf(la, cl[0], acc[tile][nt][0]));
                    acc[tile][nt][2] = fmaf(hb_s, ch[2], fmaf(lb, cl[2], acc[tile][nt][2]));
                    if (BP > 1) {
                        acc[tile][nt][1] = fmaf(ha_s, ch[1], fmaf(la, cl[1], acc[tile][nt][1]));
                        acc[tile][nt][3] = fmaf(hb_s, ch[3], fmaf(lb, cl[3], acc[tile][nt][3]));
                    }
                }
            }
        }
    }
}

// Shared memory of the tensor-core kernel, in order: ring [NW][2][32 x 144 B], x fragments
// [US][16][BP][4] uint2, x sums [US][8][BP], per-warp tables [NW][256] floats, partial rows
// [red_floats], mbarriers [NW][2].
template <int BP, int MATS, int FMT = kFmtQ4_K>
__global__ void __launch_bounds__(MmaWarpsF<FMT, BP>::value * 32, 1)
    mma_gemv_kernel(const RowsArgs a, const __grid_constant__ WeightMaps<MATS> maps)
{
    constexpr int NW = MmaWarpsF<FMT, BP>::value;
    constexpr int TAB = MmaTabF<FMT, BP>::value;
    constexpr bool PER_LANE = (FMT == kFmtQ6_K);    // per-lane copy windows (rows kernel, Q6_K)
    constexpr int UB = PER_LANE ? 210 : (FMT == kFmtIQ4_XS) ? 136 : MmaFmt<FMT>::kUnitBytes;  // in W
    constexpr int LB = MmaFmt<FMT>::kUnitBytes;     // ring bytes per row
    constexpr int GR = PER_LANE ? 16 : 8;           // x-sum groups per unit
    constexpr int BOX = 32 * LB;
    constexpr int INNER = UB / 4;
    static_assert(BOX % 128 == 0, "tensor-copy destinations in shared memory must be 128-byte aligned");

    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *ring = smem;
    uint2 *xf = reinterpret_cast<uint2 *>(smem + NW * kRowsStages * BOX);
    float *xsum = reinterpret_cast<float *>(xf + (size_t)a.US * 16 * BP * 4);
    float *tabs = xsum + a.US * GR * BP;
    float *red = tabs + NW * TAB;
    uint64_t *bars = reinterpret_cast<uint64_t *>(red + a.red_floats);

    const int s = blockIdx.x / a.Gs;
    const int cta = blockIdx.x % a.Gs;
    const int US_s = min(a.US, a.UPR - s * a.US);
    const int64_t R0 = ((int64_t)cta * a.N) / a.Gs, R1 = ((int64_t)(cta + 1) * a.N) / a.Gs;
    const int rows = (int)(R1 - R0);
    const BandShape bs = band_shape<MATS>(rows, US_s, NW);
    const int npairs = bs.G * bs.P;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ucol0 = s * a.US;
    float *dtab = tabs + warp * TAB;

    // K part p of a row group takes units p, p + P, ... (as in rows_gemv_kernel)
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
    uint8_t *myring = ring + warp * kRowsStages * BOX;
    const uint32_t bar0 = smem_u32(bars + warp * kRowsStages);
    int iq = warp, iu = 0, iub = 0;
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
        iu += du;
        if (iu >= iub) {
            iq += NW;
            if (iq < npairs) cursor_pair();
        }
    };
    auto issue = [&](int i) {
        const uint32_t bar = bar0 + 8 * (i % kRowsStages);
        mbar_arrive_expect_tx(bar, BOX);
        // IQ4_XS: the box starts at the unit's byte offset rounded down to 16 bytes
        const int bx = (FMT == kFmtIQ4_XS) ? (int)(((int64_t)(ucol0 + iu) * UB & ~(int64_t)15) >> 2)
                                           : (ucol0 + iu) * INNER;
        tma_load_2d(smem_u32(myring + (i % kRowsStages) * BOX), &maps.m[ig_map], bx, ig_row, bar);
        advance();
    };
    // Q6_K: per-lane bulk copies of the 16-byte aligned window around each row's unit (all 32
    // lanes; the same windows as rows_gemv_kernel)
    auto issue_lanes = [&](int i) {
        const uint32_t bar = bar0 + 8 * (i % kRowsStages);
        const int64_t row = (int64_t)ig_row + lane;
        uint32_t nb = 0;
        const uint8_t *src = nullptr;
        if (row < a.N) {
            const int64_t ad = ((row * a.UPR + ucol0 + iu) * UB) & ~(int64_t)15;
            const int64_t room = a.wend - ad;
            nb = (uint32_t)(room < (LB - 16) ? room : (LB - 16));
            src = a.w[ig_map] + ad;
        }
        const uint32_t tot = __reduce_add_sync(0xffffffffu, nb);
        if (lane == 0) mbar_arrive_expect_tx(bar, tot);
        __syncwarp();
        if (nb) bulk_g2s_plain(smem_u32(myring + (i % kRowsStages) * BOX + lane * LB), src, nb, bar);
        advance();
    };

    // 1. weight prefetch (independent of the previous kernel on the stream)
    if (nsteps > 0 && lane == 0) {
        if (!PER_LANE) {
#pragma unroll
            for (int m = 0; m < MATS; ++m)
                asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.m[m])) : "memory");
        }
        for (int i = 0; i < kRowsStages; ++i) mbar_init(bar0 + 8 * i, 1);
        mbar_init_fence();
        if (!PER_LANE)
            for (int i = 0; i < kPreStages && i < nsteps; ++i) issue(i);
    }
    if (PER_LANE && nsteps > 0) {
        __syncwarp();
        for (int i = 0; i < kPreStages && i < nsteps; ++i) issue_lanes(i);
    }
    // 2. programmatic dependent launch: let the next kernel start prefetching, then wait for the
    //    previous kernel's results before reading x or writing y
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // 3. x fragments and sub-block sums of this slice
    mma_stage_x<BP, FMT>(a, s, US_s, xf, xsum);
    // the rest of the ring, once this warp's x loads have returned (issuing it after the CTA's
    // barrier instead, as rows_gemv_kernel does, measured no better here: B = 8 unchanged,
    // Q5_K at B = 16 0.7 us slower)
    if (PER_LANE) {
        for (int i = kPreStages; i < kRowsStages && i < nsteps; ++i) issue_lanes(i);
    } else if (lane == 0) {
        for (int i = kPreStages; i < kRowsStages && i < nsteps; ++i) issue(i);
    }
    __syncthreads();

    int step = 0;
    bool failed = false;
    for (int q = warp; q < npairs && !failed; q += NW) {
        int ua, ub;
        pair_units(q, ua, ub);
        float acc[2][MmaNT<BP>::value][4];
#pragma unroll
        for (int tile = 0; tile < 2; ++tile)
#pragma unroll
            for (int nt = 0; nt < MmaNT<BP>::value; ++nt)
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[tile][nt][k] = 0.0f;
        float accM[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) accM[b] = 0.0f;
        for (int j = ua; j < ub; j += du, ++step) {
            const bool ok = mbar_wait_bounded(bar0 + 8 * (step % kRowsStages),
                                              (uint32_t)((step / kRowsStages) & 1));
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) {
                    atomicExch(a.err, kErrCopyTimeout);
                    for (int r = step + 1; r < nsteps && r < step + kRowsStages; ++r)
                        (void)mbar_wait_bounded(bar0 + 8 * (r % kRowsStages), (uint32_t)((r / kRowsStages) & 1));
                }
                failed = true;
                break;
            }
            if (FMT == kFmtQ6_K) {
                const int gq = q / bs.P;
                const bool second = (MATS > 1) && gq >= bs.Gm;
                const int64_t row0 = R0 + 32 * (second ? gq - bs.Gm : gq);
                mma_q6k_step<BP>(myring + (step % kRowsStages) * BOX, xf, xsum, a.US, j, dtab, acc, accM,
                                 lane, a, row0, ucol0 + j, a.w[second ? MATS - 1 : 0]);
            } else {
                if (FMT == kFmtQ8_0)
                    mma_q8_step<BP>(myring + (step % kRowsStages) * BOX, xf, j, dtab, acc, lane);
                else if (FMT == kFmtIQ4_XS)
                    mma_iq4xs_step<BP>(myring + (step % kRowsStages) * BOX, (int)(((int64_t)(ucol0 + j) * UB) & 15),
                                       xf, j, dtab, acc, lane);
                else if (FMT == kFmtQ5_K)
                    mma_q5k_step<BP>(myring + (step % kRowsStages) * BOX, xf, xsum, a.US, j, dtab, acc, accM, lane);
                else
                    mma_q4k_step<BP>(myring + (step % kRowsStages) * BOX, xf, xsum, a.US, j, dtab, acc, accM, lane);
            }
            __syncwarp();
            if (step + kRowsStages < nsteps) {
                if (PER_LANE) {
                    fence_proxy_async_smem();
                    issue_lanes(step + kRowsStages);
                } else if (lane == 0) {
                    fence_proxy_async_smem();
                    issue(step + kRowsStages);
                }
            }
        }
        if (failed) break;
        // C fragments -> rows (row = lane) through the warp's table, plus the lane's min term
        {
            const int pr = mma_frag_row<FMT>(lane >> 2), t = lane & 3;
#pragma unroll
            for (int tile = 0; tile < 2; ++tile)
#pragma unroll
                for (int nt = 0; nt < MmaNT<BP>::value; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int col = 8 * nt + 2 * t + (i & 1);
                        if (col < BP) dtab[(tile * 16 + pr + 8 * (i >> 1)) * BP + col] = acc[tile][nt][i];
                    }
        }
        __syncwarp();
        float v[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) v[b] = dtab[lane * BP + b] + accM[b];
        __syncwarp();
        if (bs.P == 1 && MATS == 1) {
            const int rr = (q / bs.P) * 32 + lane;
            if (rr < rows) {
                const int64_t row0 = (R0 + rr) * a.B;
                float *dst = a.out + (int64_t)s * a.N * a.B + row0;
                if (a.S == 1 && a.res) {
                    for (int b = 0; b < a.B; ++b) dst[b] = v[b] + a.res[row0 + b];
                } else {
                    for (int b = 0; b < a.B; ++b) dst[b] = v[b];
                }
            }
        } else {
            float *r = red + ((size_t)q * 32 + lane) * BP;
#pragma unroll
            for (int b = 0; b < BP; ++b) r[b] = v[b];
        }
    }
    const bool any_failed = __syncthreads_or(failed ? 1 : 0);
    // 4. rows of the band: sum the K parts (and combine the pair) in part order, write once
    if (!any_failed && (bs.P > 1 || MATS > 1)) band_finish<BP, MATS>(a, bs, red, s, R0, rows);
    // 5. K slices: the last CTA of the band adds them up
    if (a.S > 1) splitk_fixup<MATS>(a, cta, R0, rows, reinterpret_cast<int *>(xsum));
}

}  // namespace qg
