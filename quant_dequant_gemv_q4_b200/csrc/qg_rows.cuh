// qg_rows.cuh -- the default streaming GEMV kernel of libqg (sm_100a): one row per lane.
//
// Operation (HARDWARE GROUND TRUTH: 2x NVIDIA Tesla T4 (Kaggle), second prompt, "SPEC"):
//   y[n,b] = sum_k dequant(W)[n,k] * x[k,b] with the format chosen by a flag, fp32 accumulation
//   ("PHYSICS & CONTRACT"), Q4_K w = d*sc*q - dmin*m ("QUANTIZATION MIX"), Q8_0 w = d*q.
//
// Mapping.  An "item" is 32 consecutive rows x one 256-weight unit column (a Q4_K superblock or
// eight Q8_0 blocks per row).  One 2-D TMA tensor copy (cp.async.bulk.tensor.2d) brings an item
// into a warp's ring: 32 rows x 144 B (Q4_K) or 32 x 272 B (Q8_0); both row strides are odd
// multiples of 16 B, so the 8 lanes of a quarter-warp reading 16 B from 8 different rows hit 8
// different bank groups.  Lane l owns row 32*g + l of the item's row group g, decodes the whole
// unit of that row (all 8 sub-blocks) and keeps that row's running sum in registers: there is no
// cross-lane reduction, and the scale/min table is decoded once per 256 weights with SWAR masks.
//
// Arithmetic (factored form).  With D_j = d*sc_j and M_j = dmin*m_j (both exact in fp32),
//   sum_i w_i x_i = sum_j [ D_j * sum_{i in j} q_i x_i  -  M_j * sum_{i in j} x_i ].
// The inner sums use fp16 "subnormal nibbles": (word & 0x000F000F) read as two fp16 values is
// exactly (q_a * 2^-24, q_b * 2^-24) (a nibble at bits 4-7 of a half gives q * 2^-20), one logic
// instruction per two weights; fma.rn.f32.f16 multiplies such a half by the fp16 x exactly and
// adds it to an fp32 accumulator.  The x sums per sub-block are computed once per CTA.  Q8_0
// converts its int8 pairs to exact fp16 integers (1152 + q, minus 1152) and uses the same FMA.
//
// Work split: items are numbered group-major within a K slice and dealt to the slice's warps as
// equal contiguous ranges (so every SM streams the same number of bytes +-1 item).  A row group
// cut between warps is finished by whichever contributing warp arrives last at an arrival counter;
// it sums the partial rows of all contributors in warp order (deterministic, no waiting).
#pragma once

#include <cuda.h>

#include "qg_device.cuh"

namespace qg {

template <int FMT> struct RowsFmt;
template <> struct RowsFmt<kFmtQ4_K> {
    static constexpr int kUnitBytes = 144;
    static constexpr int kBoxInner = 36;  // u32 elements per row of a box
};
template <> struct RowsFmt<kFmtQ8_0> {
    static constexpr int kUnitBytes = 272;
    static constexpr int kBoxInner = 68;
};

// warps per CTA: as many as the shared-memory budget allows next to x
template <int FMT, int BP> struct RowsWarps {
    static constexpr int value = (FMT == kFmtQ4_K) ? (BP >= 8 ? 12 : 16) : (BP >= 4 ? 6 : 8);
};

constexpr int kRowsStages = 2;  // ring stages per warp (double buffering)

struct RowsArgs {
    const uint16_t *x;  // fp16 bits [K][B]
    float *out;         // y [N][B] when S == 1, else per-slice partial rows [S][N][B]
    float *slots;       // [nwarps][2][32][BP] partial rows of row groups cut between warps
    unsigned *cnt;      // [nwarps] arrival counters (zero between calls)
    int *err;
    int64_t N;
    int B;
    int UPR;  // units per row
    int US;   // units per slice
    int S;    // slices
    int Gs;   // CTAs per slice
};

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}

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

// x staging.  Per unit j of the slice and column b: 4 chunks c x 8 words i x 8 halves:
//   x[e], x[e+2], x[e+1], x[e+3], x[32+e], x[32+e+2], x[32+e+1], x[32+e+3]   (e = 64c + 4i)
// i.e. the weights of qs word i of chunk c in the order its nibble pairs come out.
// Offset of that 16-byte chunk, in halves:
template <int BP>
__device__ __forceinline__ int rows_x_off(int j, int c, int i, int b)
{
    return (((j * 4 + c) * 8 + i) * BP + b) * 8;
}

template <int BP>
__device__ __forceinline__ void rows_stage_x(const RowsArgs &a, int s, int US_s, __half *xs,
                                             float *xsum)
{
    const int64_t kbase = (int64_t)s * a.US * 256;
    const uint16_t *xsl = a.x + kbase * a.B;
    const int nchunk = US_s * 32 * BP;  // 16-byte chunks of staged x
    for (int t = threadIdx.x; t < nchunk; t += blockDim.x) {
        const int b = t % BP;
        const int ji = t / BP;  // (j*4 + c)*8 + i
        const int i = ji & 7, jc = ji >> 3;
        const int e0 = (jc >> 2) * 256 + (jc & 3) * 64 + 4 * i;  // k_local of e
        uint32_t h[8];  // x[e0 .. e0+3], x[e0+32 .. e0+35] in natural order
        if (b < a.B) {
            if (BP == 1 && (reinterpret_cast<uintptr_t>(xsl) & 7) == 0) {
                const uint2 lo = *reinterpret_cast<const uint2 *>(xsl + e0);
                const uint2 hi = *reinterpret_cast<const uint2 *>(xsl + e0 + 32);
                h[0] = lo.x & 0xFFFFu; h[1] = lo.x >> 16; h[2] = lo.y & 0xFFFFu; h[3] = lo.y >> 16;
                h[4] = hi.x & 0xFFFFu; h[5] = hi.x >> 16; h[6] = hi.y & 0xFFFFu; h[7] = hi.y >> 16;
            } else {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    h[q] = xsl[(int64_t)(e0 + q) * a.B + b];
                    h[4 + q] = xsl[(int64_t)(e0 + 32 + q) * a.B + b];
                }
            }
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) h[q] = 0;
        }
        // order (e, e+2, e+1, e+3): halves 0,2,1,3 of each group of four
        uint4 v;
        v.x = h[0] | (h[2] << 16);
        v.y = h[1] | (h[3] << 16);
        v.z = h[4] | (h[6] << 16);
        v.w = h[5] | (h[7] << 16);
        *reinterpret_cast<uint4 *>(xs + (int64_t)t * 8) = v;
    }
    __syncthreads();
    // xsum[(j*8 + sub)*BP + b] = sum of the 32 x of sub-block `sub` of unit j, from shared memory,
    // in a fixed order (sub-block 2c+h = halves 4h..4h+3 of the 8 words of chunk c)
    const int nsum = US_s * 8 * BP;
    for (int t = threadIdx.x; t < nsum; t += blockDim.x) {
        const int b = t % BP;
        const int js = t / BP;
        const int sub = js & 7, j = js >> 3;
        const int c = sub >> 1, hsel = sub & 1;
        float acc = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint2 v = *reinterpret_cast<const uint2 *>(xs + rows_x_off<BP>(j, c, i, b) + 4 * hsel);
            const float2 p = __half22float2(*reinterpret_cast<const __half2 *>(&v.x));
            const float2 q = __half22float2(*reinterpret_cast<const __half2 *>(&v.y));
            acc += (p.x + p.y) + (q.x + q.y);
        }
        xsum[t] = acc;
    }
}

// One Q4_K superblock of this lane's row against x (unit j of the slice).
template <int BP>
__device__ __forceinline__ void rows_q4k(const uint8_t *u, const __half *xs, const float *xsum, int j,
                                         float (&acc)[BP])
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
        const float2 D = __fmul2_rn(dscale, sc);           // scaled d*sc for sub-blocks 2c, 2c+1
        const float2 M = __fmul2_rn(f2(dm.y, dm.y), mm);   // dmin*m for sub-blocks 2c, 2c+1
        const uint4 q0 = *reinterpret_cast<const uint4 *>(u + 16 + 32 * c);
        const uint4 q1 = *reinterpret_cast<const uint4 *>(u + 32 + 32 * c);
        const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        float l0[BP], l1[BP], h0[BP], h1[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) l0[b] = l1[b] = h0[b] = h1[b] = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w = qw[i], wb = w >> 8;
            const uint32_t qa = w & 0x000F000Fu, qb = wb & 0x000F000Fu;   // low nibbles
            const uint32_t qc = w & 0x00F000F0u, qd = wb & 0x00F000F0u;   // high nibbles
#pragma unroll
            for (int b = 0; b < BP; ++b) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(xs + rows_x_off<BP>(j, c, i, b));
                mfma2(l0[b], qa, xv.x);
                mfma2(l1[b], qb, xv.y);
                mfma2(h0[b], qc, xv.z);
                mfma2(h1[b], qd, xv.w);
            }
        }
#pragma unroll
        for (int b = 0; b < BP; ++b) {
            const float Xlo = xsum[(j * 8 + 2 * c) * BP + b];
            const float Xhi = xsum[(j * 8 + 2 * c + 1) * BP + b];
            float t = acc[b];
            t = fmaf(D.x, l0[b] + l1[b], t);
            t = fmaf(D.y, h0[b] + h1[b], t);
            t = fmaf(-M.x, Xlo, t);
            t = fmaf(-M.y, Xhi, t);
            acc[b] = t;
        }
    }
}

// One Q8_0 unit (eight 34-byte blocks) of this lane's row against x (unit j of the slice).
// Chunk c = blocks 2c, 2c+1 = bytes [68c, 68c+68), read through the 16-byte chunks covering it.
template <int BP>
__device__ __forceinline__ void rows_q8_0(const uint8_t *u, const __half *xs, int j, float (&acc)[BP])
{
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int base16 = (68 * c) >> 4;          // first 16-byte chunk
        const int woff = ((68 * c) & 15) >> 2;     // word offset of byte 68c inside it
        uint32_t win[20];
#pragma unroll
        for (int k = 0; k < 5; ++k) {
            const uint4 v = *reinterpret_cast<const uint4 *>(u + 16 * (base16 + k));
            win[4 * k] = v.x;
            win[4 * k + 1] = v.y;
            win[4 * k + 2] = v.z;
            win[4 * k + 3] = v.w;
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
            // (1024 + q + 128) as fp16 pairs: bytes (0, 2) and (1, 3) under a 0x64 high byte
            const uint32_t qa = hsub2_bits(__byte_perm(la, 0x64646464u, 0x7250), off2);  // weights e, e+2
            const uint32_t qb = hsub2_bits(__byte_perm(la, 0x64646464u, 0x7351), off2);  // e+1, e+3
            const uint32_t qc = hsub2_bits(__byte_perm(lb, 0x64646464u, 0x7250), off2);
            const uint32_t qd = hsub2_bits(__byte_perm(lb, 0x64646464u, 0x7351), off2);
#pragma unroll
            for (int b = 0; b < BP; ++b) {
                const uint4 xv = *reinterpret_cast<const uint4 *>(xs + rows_x_off<BP>(j, c, i, b));
                mfma2(a0[b], qa, xv.x);
                mfma2(a1[b], qb, xv.y);
                mfma2(b0[b], qc, xv.z);
                mfma2(b1[b], qd, xv.w);
            }
        }
#pragma unroll
        for (int b = 0; b < BP; ++b) acc[b] = fmaf(dB, b0[b] + b1[b], fmaf(dA, a0[b] + a1[b], acc[b]));
    }
}

template <int BP>
__device__ __forceinline__ void rows_finish(const RowsArgs &a, int s, int64_t group, const float (&acc)[BP],
                                            bool complete, int64_t group0, int64_t w, int64_t Ws,
                                            int64_t Is, int US_s, int nwarps_slice)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = group * 32 + lane;
    float *dst = a.out + ((int64_t)s * a.N + row) * a.B;
    if (complete) {
        if (row < a.N)
            for (int b = 0; b < a.B; ++b) dst[b] = acc[b];
        return;
    }
    const int64_t base = (int64_t)s * nwarps_slice;
    const int side = (group == group0) ? 0 : 1;
    float *mine = a.slots + (((base + w) * 2 + side) * 32 + lane) * BP;
    for (int b = 0; b < BP; ++b) __stcg(mine + b, acc[b]);
    const int64_t wlo = warp_of_item(group * US_s, Ws, Is);
    const int64_t whi = warp_of_item((group + 1) * US_s - 1, Ws, Is);
    const unsigned n = (unsigned)(whi - wlo + 1);
    __syncwarp();
    unsigned last = 0;
    if (lane == 0) {
        __threadfence();
        last = (atomicInc(a.cnt + base + wlo, n - 1) == n - 1) ? 1u : 0u;
    }
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    __threadfence();
    float sum[BP];
    for (int b = 0; b < BP; ++b) sum[b] = 0.0f;
    for (int64_t w2 = wlo; w2 <= whi; ++w2) {
        const int64_t g0 = ((w2 * Is) / Ws) / US_s;  // first row group of warp w2
        const int side2 = (group == g0) ? 0 : 1;
        const float *p = a.slots + (((base + w2) * 2 + side2) * 32 + lane) * BP;
        for (int b = 0; b < BP; ++b) sum[b] += __ldcg(p + b);
    }
    if (row < a.N)
        for (int b = 0; b < a.B; ++b) dst[b] = sum[b];
}

template <int FMT, int BP>
__global__ void __launch_bounds__(RowsWarps<FMT, BP>::value * 32, 1)
    rows_gemv_kernel(const RowsArgs a, const __grid_constant__ CUtensorMap tmap)
{
    constexpr int NW = RowsWarps<FMT, BP>::value;
    constexpr int UB = RowsFmt<FMT>::kUnitBytes;
    constexpr int BOX = 32 * UB;  // bytes of one item

    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *ring = smem;
    __half *xs = reinterpret_cast<__half *>(smem + NW * kRowsStages * BOX);
    float *xsum = reinterpret_cast<float *>(xs + (size_t)a.US * 256 * BP);
    uint64_t *bars = reinterpret_cast<uint64_t *>(xsum + a.US * 8 * BP);

    const int s = blockIdx.x / a.Gs;
    const int cta = blockIdx.x % a.Gs;
    const int US_s = min(a.US, a.UPR - s * a.US);
    const int64_t ngroups = (a.N + 31) / 32;
    const int64_t Is = ngroups * US_s;
    const int nwarps_slice = a.Gs * NW;
    const int64_t Ws = min((int64_t)nwarps_slice, Is);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t w = (int64_t)cta * NW + warp;
    const bool active = w < Ws;
    int64_t t0 = 0, t1 = 0;
    if (active) {
        t0 = (w * Is) / Ws;
        t1 = ((w + 1) * Is) / Ws;
    }
    const int n = (int)(t1 - t0);
    uint8_t *myring = ring + warp * kRowsStages * BOX;
    const uint32_t bar0 = smem_u32(bars + warp * kRowsStages);
    const int x_unit0 = s * a.US;  // first unit column of this slice

    // item t -> (group, unit) ; issue with the next-to-issue position tracked incrementally
    int64_t ig = 0;
    int ij = 0;
    auto issue = [&](int i) {
        const uint32_t bar = bar0 + 8 * (i % kRowsStages);
        mbar_arrive_expect_tx(bar, BOX);
        tma_load_2d(smem_u32(myring + (i % kRowsStages) * BOX), &tmap,
                    (x_unit0 + ij) * RowsFmt<FMT>::kBoxInner, (int)(ig * 32), bar,
                    evict_first_policy());
        if (++ij == US_s) {
            ij = 0;
            ++ig;
        }
    };

    // 1. weight prefetch (independent of the previous kernel on the stream)
    if (active && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap)) : "memory");
        for (int i = 0; i < kRowsStages; ++i) mbar_init(bar0 + 8 * i, 1);
        mbar_init_fence();
        ig = t0 / US_s;
        ij = (int)(t0 - ig * US_s);
        for (int i = 0; i < kRowsStages && i < n; ++i) issue(i);
    }
    // 2. programmatic dependent launch: let the next kernel start prefetching, then wait for
    //    the previous kernel's results before reading x or writing y / the workspace
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // 3. x for this slice -> shared memory (fp16 in consumer order) and per-sub-block sums
    rows_stage_x<BP>(a, s, US_s, xs, xsum);
    __syncthreads();
    if (!active) return;

    const int64_t group0 = t0 / US_s;
    int64_t group = group0;
    int j = (int)(t0 - group0 * US_s);
    bool started_here = (j == 0);
    float acc[BP];
#pragma unroll
    for (int b = 0; b < BP; ++b) acc[b] = 0.0f;

    for (int i = 0; i < n; ++i) {
        const bool ok = mbar_wait_bounded(bar0 + 8 * (i % kRowsStages), (uint32_t)((i / kRowsStages) & 1));
        if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0) {
                atomicExch(a.err, kErrCopyTimeout);
                for (int r = i + 1; r < n && r < i + kRowsStages; ++r)
                    (void)mbar_wait_bounded(bar0 + 8 * (r % kRowsStages), (uint32_t)((r / kRowsStages) & 1));
            }
            __syncwarp();
            return;
        }
        const uint8_t *u = myring + (i % kRowsStages) * BOX + lane * UB;
        if (FMT == kFmtQ4_K)
            rows_q4k<BP>(u, xs, xsum, j, acc);
        else
            rows_q8_0<BP>(u, xs, j, acc);
        __syncwarp();
        if (lane == 0 && i + kRowsStages < n) {
            fence_proxy_async_smem();
            issue(i + kRowsStages);
        }
        if (++j == US_s) {
            rows_finish<BP>(a, s, group, acc, started_here, group0, w, Ws, Is, US_s, nwarps_slice);
#pragma unroll
            for (int b = 0; b < BP; ++b) acc[b] = 0.0f;
            ++group;
            j = 0;
            started_here = true;
        }
    }
    if (j > 0) rows_finish<BP>(a, s, group, acc, false, group0, w, Ws, Is, US_s, nwarps_slice);
}

}  // namespace qg
