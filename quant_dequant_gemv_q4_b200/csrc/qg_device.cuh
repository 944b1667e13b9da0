// qg_device.cuh -- device code of libqg shared by the kernels (PTX wrappers: mbarriers, bulk
// copies, timers), plus the kernels that are not the default streaming ones: the four-lanes-per-
// unit kernel of QG_VARIANT_DIRECT (stream_gemv_kernel) and its split-K second pass, the dequant
// dumps, the plain per-row kernel of QG_VARIANT_GENERIC, the host-x copy of qg_gemv_host, and
// bandwidth probes (sm_100a).  The default kernels are in qg_rows.cuh (CUDA cores) and qg_mma.cuh
// (tensor cores).
//
// Operation (HARDWARE GROUND TRUTH: 2x NVIDIA Tesla T4 (Kaggle), second prompt, "SPEC"):
//   y[n,b] = sum_k dequant(W)[n,k] * x[k,b], format chosen per call by a flag; fp32 accumulation
//   ("PHYSICS & CONTRACT"); Q4_K w = d*sc*q - dmin*m ("QUANTIZATION MIX"); Q8_0 w = d*q; Q5_K and
//   Q6_K (the same mix) in the dumps and the per-row kernel.
//
// Work decomposition of stream_gemv_kernel (Q4_K and Q8_0).  A "unit" is 256 consecutive weights of one row:
// one Q4_K superblock (144 B) or eight Q8_0 blocks (272 B).  Both are 16-byte multiples, so any
// run of whole units of a row is a legal bulk-copy source.  The K axis may be cut into S slices
// (only when x for the whole of K would not fit in shared memory); slice s of row n is a
// "virtual row" of US_s units.  Items (virtual-row units) of one slice are numbered row-major and
// dealt to the slice's warps as equal contiguous ranges, so every warp streams the same number of
// bytes (+-1 unit) whatever N and K are.  A warp's range starts and ends mid-row in general: rows
// that lie wholly inside one warp are written directly; a row cut between warps is finished by
// whichever contributing warp arrives last at that row's arrival counter, which sums the
// contributors' partials in warp order, so the result does not depend on arrival order.
//
// Memory path.  Each warp owns a ring of NSTAGE shared-memory stages; lane 0 fills them with
// cp.async.bulk (TMA bulk copies, completion counted in bytes on an mbarrier) several chunks ahead
// of the 32 lanes that decode.  x for the CTA's slice is converted to fp32 once and kept resident
// in shared memory, in a lane-interleaved order that makes every 16-byte x load conflict-free.
// Four lanes decode one unit, each lane 64 weights (Q4_K: the 32 bytes qs[32c..32c+31], i.e. the
// whole sub-blocks 2c and 2c+1; Q8_0: blocks 2c and 2c+1), so the per-unit scale/min decoding is
// done once per sub-block, never redundantly.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qg {

constexpr int kFmtQ8_0 = 8;
constexpr int kFmtQ4_K = 12;
constexpr int kFmtQ5_K = 13;
constexpr int kFmtQ6_K = 14;
constexpr int kFmtIQ4_XS = 23;

// IQ4_XS codebook: the sixteen integer levels of the format, each stored biased by +128 as one
// unsigned byte (levels -127 .. 113 -> 1 .. 241), four per word in index order.
constexpr uint32_t kIq4Lut0 = 0x3F2D1801u;  // levels of indices 0..3:   -127 -104  -83  -65
constexpr uint32_t kIq4Lut1 = 0x766A5D4Fu;  // indices 4..7:              -49  -35  -22  -10
constexpr uint32_t kIq4Lut2 = 0xA6998D81u;  // indices 8..11:               1   13   25   38
constexpr uint32_t kIq4Lut3 = 0xF1D9C5B5u;  // indices 12..15:             53   69   89  113

constexpr int kVarDirect = 1;
constexpr int kVarFactored = 2;

constexpr int kWarps = 16;   // warps per CTA of the streaming kernel
constexpr int kStages = 3;   // ring stages per warp
constexpr unsigned kWaitNs = 2000000000u;  // give up on a bulk copy after 2 s

// Device error codes (written to the workspace error word).
constexpr int kErrCopyTimeout = 1;

template <int FMT> struct UnitFmt;
template <> struct UnitFmt<kFmtQ4_K> {
    static constexpr int kBytes = 144;  // one superblock
    static constexpr int kChunk = 16;   // units per bulk-copy chunk (2304 B)
};
template <> struct UnitFmt<kFmtQ8_0> {
    static constexpr int kBytes = 272;  // eight 34-byte blocks
    static constexpr int kChunk = 8;    // units per chunk (2176 B)
};

struct StreamArgs {
    const uint8_t *W;
    const uint16_t *x;  // fp16 bits [K][B]
    float *out;         // y [N][B] when S == 1, else per-slice partial rows [S][N][B]
    float *slots;       // [S*Gs*kWarps][2][BP] partial sums of rows cut between warps
    unsigned *cnt;      // [S*Gs*kWarps] arrival counters (zero between calls)
    int *err;           // device error word
    int64_t N;
    int B;              // real columns (BP >= B is the padded width)
    int UPR;            // units per row (K / 256)
    int US;             // units per slice (last slice may be shorter)
    int S;              // slices
    int Gs;             // CTAs per slice
    int xs_floats;      // floats of staged x per CTA
};

// ------------------------------------------------------------------------------------------------
// PTX wrappers
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// try_wait with a suspend-time hint: a waiting warp sleeps (issuing nothing) until the phase
// completes or about kSuspendNs pass, instead of returning at once and spinning.
constexpr uint32_t kSuspendNs = 1000000u;

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of an mbarrier, giving up after kWaitNs of wall time.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > kWaitNs) return false;
    }
    return true;
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Global -> shared bulk copy; bytes and both addresses are 16-byte multiples.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar,
                                         uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

// The same without a cache hint.
__device__ __forceinline__ void bulk_g2s_plain(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ uint64_t evict_first_policy()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// ------------------------------------------------------------------------------------------------
// Q4_K decoding shared by the dump and the GEMV.
//
// Header word 0 = {d, dmin} (fp16 pair); words 1..3 = scales[0..11].  Lane c of a unit owns the
// 64-weight chunk c, i.e. sub-blocks j0 = 2c and j1 = 2c+1 (the low and high nibbles of
// qs[32c .. 32c+31]).  GGML's scale table (get_scale_min_k4): for j < 4, sc_j = scales[j] & 63,
// m_j = scales[j+4] & 63; for j >= 4, sc_j = (scales[j+4] & 15) | (scales[j-4] >> 6) << 4 and
// m_j = (scales[j+4] >> 4) | (scales[j] >> 6) << 4.  j0 and j1 are adjacent bytes of a word, so
// both are read through one 16-bit window.
// ------------------------------------------------------------------------------------------------
struct Q4kLaneScales {
    float D0, D1;  // d*sc for sub-blocks 2c, 2c+1 (exact in fp32)
    float M0, M1;  // dmin*m for sub-blocks 2c, 2c+1 (exact in fp32)
};

__device__ __forceinline__ Q4kLaneScales q4k_lane_scales(uint4 hdr, int c)
{
    const int sh = 16 * (c & 1);
    const uint32_t y = hdr.y >> sh, z = hdr.z >> sh, w = hdr.w >> sh;
    const bool upper = c >= 2;
    const uint32_t SC = upper ? ((w & 0x0F0Fu) | ((y >> 2) & 0x3030u)) : (y & 0x3F3Fu);
    const uint32_t MM = upper ? (((w >> 4) & 0x0F0Fu) | ((z >> 2) & 0x3030u)) : (z & 0x3F3Fu);
    // small integers -> fp32 through the 2^23 exponent trick (exact)
    const float2 sc = __fadd2_rn(f2(__uint_as_float(0x4B000000u | (SC & 0xFFu)),
                                    __uint_as_float(0x4B000000u | (SC >> 8))),
                                 f2(-8388608.0f, -8388608.0f));
    const float2 mm = __fadd2_rn(f2(__uint_as_float(0x4B000000u | (MM & 0xFFu)),
                                    __uint_as_float(0x4B000000u | (MM >> 8))),
                                 f2(-8388608.0f, -8388608.0f));
    __half2 dd;
    *reinterpret_cast<uint32_t *>(&dd) = hdr.x;
    const float2 ddf = __half22float2(dd);  // (d, dmin), exact
    Q4kLaneScales r;
    const float2 D = __fmul2_rn(f2(ddf.x, ddf.x), sc);
    const float2 M = __fmul2_rn(f2(ddf.y, ddf.y), mm);
    r.D0 = D.x;
    r.D1 = D.y;
    r.M0 = M.x;
    r.M1 = M.y;
    return r;
}

// Nibble extraction.  A qs word holds bytes l..l+3 of the lane's 32; window 0 is the word, window
// 1 the word >> 16, so bytes l, l+1 sit at bits 0-15 of window 0 and bytes l+2, l+3 at bits 0-15
// of window 1.  Within a window the low nibble of its byte 0 is at bits 0-3 ("k=0"), the high
// nibble at 4-7 (k=1), the low nibble of byte 1 at 8-11 (k=2), the high one at 12-15 (k=3).  The
// pair (window 0, window 1) at one k therefore holds weights (e, e+2): the x layout in shared
// memory stores each group of 4 weights as (e, e+2, e+1, e+3) so that pairs line up.
//
// Direct form: f = (bits & mask_k) | 0x4B000000 is the float 2^23 + q*16^k; with A_k = D/16^k and
// C_k = -A_k*2^23, fma(A_k, f, C_k) = D*q exactly (the result needs at most 21 bits), and one
// fp32 subtraction of M gives RN(D*q - M), the correctly rounded weight.
struct Q4kDirectConsts {
    float2 A0, C0, A2, C2;  // low nibbles (sub-block 2c): k = 0 and k = 2
    float2 A1, C1, A3, C3;  // high nibbles (sub-block 2c+1): k = 1 and k = 3
    float2 M0, M1;          // -dmin*m pairs
};

__device__ __forceinline__ Q4kDirectConsts q4k_direct_consts(const Q4kLaneScales &s)
{
    Q4kDirectConsts k;
    k.A0 = f2(s.D0, s.D0);
    k.C0 = f2(-s.D0 * 8388608.0f, -s.D0 * 8388608.0f);
    k.A2 = f2(s.D0 * 0.00390625f, s.D0 * 0.00390625f);
    k.C2 = f2(-s.D0 * 32768.0f, -s.D0 * 32768.0f);
    k.A1 = f2(s.D1 * 0.0625f, s.D1 * 0.0625f);
    k.C1 = f2(-s.D1 * 524288.0f, -s.D1 * 524288.0f);
    k.A3 = f2(s.D1 * 0.000244140625f, s.D1 * 0.000244140625f);
    k.C3 = f2(-s.D1 * 2048.0f, -s.D1 * 2048.0f);
    k.M0 = f2(-s.M0, -s.M0);
    k.M1 = f2(-s.M1, -s.M1);
    return k;
}

// Correctly rounded weights of one qs word: lo = sub-block 2c weights (e, e+2), (e+1, e+3) with
// e = 4i; hi = sub-block 2c+1 weights (32+e, 34+e), (33+e, 35+e).
struct Q4kWordWeights {
    float2 loA, loB, hiA, hiB;
};

__device__ __forceinline__ Q4kWordWeights q4k_direct_word(uint32_t word, const Q4kDirectConsts &k)
{
    const uint32_t w0 = word, w1 = word >> 16;
    const float2 fa = f2(__uint_as_float((w0 & 0x000Fu) | 0x4B000000u),
                         __uint_as_float((w1 & 0x000Fu) | 0x4B000000u));
    const float2 fb = f2(__uint_as_float((w0 & 0x0F00u) | 0x4B000000u),
                         __uint_as_float((w1 & 0x0F00u) | 0x4B000000u));
    const float2 fc = f2(__uint_as_float((w0 & 0x00F0u) | 0x4B000000u),
                         __uint_as_float((w1 & 0x00F0u) | 0x4B000000u));
    const float2 fd = f2(__uint_as_float((w0 & 0xF000u) | 0x4B000000u),
                         __uint_as_float((w1 & 0xF000u) | 0x4B000000u));
    Q4kWordWeights r;
    r.loA = __fadd2_rn(__ffma2_rn(k.A0, fa, k.C0), k.M0);
    r.loB = __fadd2_rn(__ffma2_rn(k.A2, fb, k.C2), k.M0);
    r.hiA = __fadd2_rn(__ffma2_rn(k.A1, fc, k.C1), k.M1);
    r.hiB = __fadd2_rn(__ffma2_rn(k.A3, fd, k.C3), k.M1);
    return r;
}

// Factored form: f = bits & mask_k alone is the fp32 subnormal q * 16^k * 2^-149 (bits 0-15 only).
// x is staged pre-scaled by 2^(64-4k) for the k its weight is read at, so every product is
// q * x * 2^-85 exactly, whatever k: one accumulator per sub-block, no per-weight offset.
constexpr float kFactoredUnscale = 3.8685626227668134e+25f;  // 2^85

// ------------------------------------------------------------------------------------------------
// x staging: slice-local x -> fp32 shared memory in the consumer's order.
//   position p = ((((j >> 1) * 16*BP + iota) * 2 + (j & 1)) * 4 + c) * 4 + el
// for unit j of the slice, lane chunk c (weights 64c..64c+63 of the unit), 16-byte chunk iota =
// g*BP + b (g = group of 4 weights, b = column) and el in the group order (e, e+2, e+1, e+3).  A
// quarter-warp (two consecutive units x four lanes) reads eight different 16-byte bank slots.
// ------------------------------------------------------------------------------------------------
template <int BP>
__device__ __forceinline__ int xs_index(int j, int c, int iota)
{
    return ((((j >> 1) * 16 * BP + iota) * 2 + (j & 1)) * 4 + c) * 4;
}

// Shared-memory position of x[k_local][b] (k_local = 256 j + 64 c + e within the slice).
template <int BP>
__device__ __forceinline__ int xs_pos(int k_local, int b)
{
    const int j = k_local >> 8, r = k_local & 255;
    const int c = r >> 6, e = r & 63;
    const int e4 = e & 3;
    const int el = ((e4 & 1) << 1) | (e4 >> 1);  // group order (e, e+2, e+1, e+3)
    return xs_index<BP>(j, c, (e >> 2) * BP + b) + el;
}

// Scale applied to x in the factored form: 2^(64 - 4k) for the nibble position k its weight is
// read at (k = 2 * (byte & 1) + high-nibble, byte = the weight's byte within its qs word).
__device__ __forceinline__ float factored_x_scale(int k_local)
{
    const int e = k_local & 63;
    const int kk = 2 * (e & 1) + (e >> 5);
    return __uint_as_float((uint32_t)(127 + 64 - 4 * kk) << 23);
}

template <int FMT, int BP, int VAR>
__device__ __forceinline__ void stage_x(const StreamArgs &a, int s, int US_s, float *xs, float *xsum)
{
    const int64_t kbase = (int64_t)s * a.US * 256;
    const int KS = US_s * 256;
    const int nfl = a.xs_floats;
    // zero the padding (columns b >= B and the odd unit of the last pair) first
    if (a.B != BP || (US_s & 1)) {
        for (int p = threadIdx.x; p < nfl; p += blockDim.x) xs[p] = 0.0f;
        __syncthreads();
    }
    const uint16_t *xsl = a.x + kbase * a.B;
    const int nh = KS * a.B;  // halves of this slice, a multiple of 8
    if ((reinterpret_cast<uintptr_t>(xsl) & 15) == 0) {
        // 16-byte loads: two per thread in flight
        const int nv = nh >> 3;
        for (int v0 = threadIdx.x; v0 < nv; v0 += 2 * blockDim.x) {
            uint4 q[2];
            const int v1 = v0 + blockDim.x;
            q[0] = reinterpret_cast<const uint4 *>(xsl)[v0];
            if (v1 < nv) q[1] = reinterpret_cast<const uint4 *>(xsl)[v1];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int v = u ? v1 : v0;
                if (v >= nv) break;
                const uint32_t w4[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    const int flat = 8 * v + h;
                    const int kl = flat / a.B, b = flat - kl * a.B;
                    float f = __half2float(__ushort_as_half(
                        (unsigned short)((h & 1) ? (w4[h >> 1] >> 16) : (w4[h >> 1] & 0xFFFFu))));
                    if (VAR == kVarFactored) f *= factored_x_scale(kl);
                    xs[xs_pos<BP>(kl, b)] = f;
                }
            }
        }
    } else {
        for (int flat = threadIdx.x; flat < nh; flat += blockDim.x) {
            const int kl = flat / a.B, b = flat - kl * a.B;
            float f = __half2float(__ushort_as_half(xsl[flat]));
            if (VAR == kVarFactored) f *= factored_x_scale(kl);
            xs[xs_pos<BP>(kl, b)] = f;
        }
    }
    if (VAR == kVarFactored) {
        // xsum[((j*4 + c)*2 + h)*BP + b] = sum of the 32 unscaled x of sub-block 2c+h of unit j
        const int nsum = US_s * 8 * BP;
        for (int t = threadIdx.x; t < nsum; t += blockDim.x) {
            const int b = t % BP;
            const int hc = t / BP;  // (j*4 + c)*2 + h
            float acc = 0.0f;
            if (b < a.B) {
                const uint16_t *xp = xsl + (int64_t)(32 * hc) * a.B + b;
#pragma unroll 8
                for (int i = 0; i < 32; ++i) acc += __half2float(__ushort_as_half(xp[i * a.B]));
            }
            xsum[t] = acc;
        }
    }
}

// ------------------------------------------------------------------------------------------------
// Per-lane contribution of one unit: v[b] = sum over the lane's 64 weights of w * x[., b].
// ------------------------------------------------------------------------------------------------
template <int BP, int VAR>
__device__ __forceinline__ void q4k_unit(const uint8_t *u, int c, const float *xs, const float *xsum,
                                         int j, float (&v)[BP])
{
    const uint4 hdr = *reinterpret_cast<const uint4 *>(u);
    const uint4 q0 = *reinterpret_cast<const uint4 *>(u + 16 + 32 * c);
    const uint4 q1 = *reinterpret_cast<const uint4 *>(u + 32 + 32 * c);
    const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    const Q4kLaneScales sc = q4k_lane_scales(hdr, c);
    const float *xb = xs + xs_index<BP>(j, c, 0);
    if (VAR == kVarDirect) {
        const Q4kDirectConsts kc = q4k_direct_consts(sc);
        float2 acc[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) acc[b] = f2(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const Q4kWordWeights w = q4k_direct_word(qw[i], kc);
#pragma unroll
            for (int b = 0; b < BP; ++b) {
                const float4 xl = *reinterpret_cast<const float4 *>(xb + (i * BP + b) * 32);
                const float4 xh = *reinterpret_cast<const float4 *>(xb + ((8 + i) * BP + b) * 32);
                acc[b] = __ffma2_rn(w.loA, f2(xl.x, xl.y), acc[b]);
                acc[b] = __ffma2_rn(w.loB, f2(xl.z, xl.w), acc[b]);
                acc[b] = __ffma2_rn(w.hiA, f2(xh.x, xh.y), acc[b]);
                acc[b] = __ffma2_rn(w.hiB, f2(xh.z, xh.w), acc[b]);
            }
        }
#pragma unroll
        for (int b = 0; b < BP; ++b) v[b] = acc[b].x + acc[b].y;
    } else {
        float2 slo[BP], shi[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) {
            slo[b] = f2(0.0f, 0.0f);
            shi[b] = f2(0.0f, 0.0f);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t w0 = qw[i], w1 = qw[i] >> 16;
            const float2 fa = f2(__uint_as_float(w0 & 0x000Fu), __uint_as_float(w1 & 0x000Fu));
            const float2 fb = f2(__uint_as_float(w0 & 0x0F00u), __uint_as_float(w1 & 0x0F00u));
            const float2 fc = f2(__uint_as_float(w0 & 0x00F0u), __uint_as_float(w1 & 0x00F0u));
            const float2 fd = f2(__uint_as_float(w0 & 0xF000u), __uint_as_float(w1 & 0xF000u));
#pragma unroll
            for (int b = 0; b < BP; ++b) {
                const float4 xl = *reinterpret_cast<const float4 *>(xb + (i * BP + b) * 32);
                const float4 xh = *reinterpret_cast<const float4 *>(xb + ((8 + i) * BP + b) * 32);
                slo[b] = __ffma2_rn(fa, f2(xl.x, xl.y), slo[b]);
                slo[b] = __ffma2_rn(fb, f2(xl.z, xl.w), slo[b]);
                shi[b] = __ffma2_rn(fc, f2(xh.x, xh.y), shi[b]);
                shi[b] = __ffma2_rn(fd, f2(xh.z, xh.w), shi[b]);
            }
        }
        const float D0 = sc.D0 * kFactoredUnscale, D1 = sc.D1 * kFactoredUnscale;
        const float *xsm = xsum + (j * 4 + c) * 2 * BP;
#pragma unroll
        for (int b = 0; b < BP; ++b) {
            float t = D0 * (slo[b].x + slo[b].y);
            t = fmaf(D1, shi[b].x + shi[b].y, t);
            t = fmaf(-sc.M0, xsm[b], t);
            t = fmaf(-sc.M1, xsm[BP + b], t);
            v[b] = t;
        }
    }
}

// Q8_0: lane c owns blocks 2c and 2c+1 of the unit (bytes 68c .. 68c+67, 4-byte aligned).
// int8 -> fp32 exactly: bias the byte to unsigned (xor 0x80), place it under the 2^23 exponent
// (2^23 + q + 128) and subtract 2^23 + 128.  The block scale d is applied once per block:
// sum_i (d*q_i)*x_i = d * sum_i q_i*x_i, whose error is bounded relative to sum|w*x|.
template <int BP>
__device__ __forceinline__ void q8_0_unit(const uint8_t *u, int c, const float *xs, int j,
                                          float (&v)[BP])
{
    const uint32_t *p = reinterpret_cast<const uint32_t *>(u + 68 * c);
    uint32_t wd[17];
#pragma unroll
    for (int i = 0; i < 17; ++i) wd[i] = p[i];
    const float dA = __half2float(__ushort_as_half((unsigned short)(wd[0] & 0xFFFFu)));
    const float dB = __half2float(__ushort_as_half((unsigned short)(wd[8] >> 16)));
    const float *xb = xs + xs_index<BP>(j, c, 0);
    float2 sA[BP], sB[BP];
#pragma unroll
    for (int b = 0; b < BP; ++b) {
        sA[b] = f2(0.0f, 0.0f);
        sB[b] = f2(0.0f, 0.0f);
    }
    const float2 off = f2(-8388736.0f, -8388736.0f);  // -(2^23 + 128)
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        // words 0..7: block 2c (bytes shifted by the 2-byte d); words 8..15: block 2c+1
        const uint32_t a = (i < 8) ? __funnelshift_r(wd[i], wd[i + 1], 16) : wd[i + 1];
        const uint32_t ub = a ^ 0x80808080u;
        const float2 qa = __fadd2_rn(f2(__uint_as_float(__byte_perm(ub, 0x4B000000u, 0x7650)),
                                        __uint_as_float(__byte_perm(ub, 0x4B000000u, 0x7652))),
                                     off);
        const float2 qb = __fadd2_rn(f2(__uint_as_float(__byte_perm(ub, 0x4B000000u, 0x7651)),
                                        __uint_as_float(__byte_perm(ub, 0x4B000000u, 0x7653))),
                                     off);
#pragma unroll
        for (int b = 0; b < BP; ++b) {
            const float4 xv = *reinterpret_cast<const float4 *>(xb + (i * BP + b) * 32);
            if (i < 8) {
                sA[b] = __ffma2_rn(qa, f2(xv.x, xv.y), sA[b]);
                sA[b] = __ffma2_rn(qb, f2(xv.z, xv.w), sA[b]);
            } else {
                sB[b] = __ffma2_rn(qa, f2(xv.x, xv.y), sB[b]);
                sB[b] = __ffma2_rn(qb, f2(xv.z, xv.w), sB[b]);
            }
        }
    }
#pragma unroll
    for (int b = 0; b < BP; ++b) v[b] = fmaf(dB, sB[b].x + sB[b].y, dA * (sA[b].x + sA[b].y));
}

// ------------------------------------------------------------------------------------------------
// Streaming GEMV kernel.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ int64_t warp_of_item(int64_t t, int64_t Ws, int64_t Is)
{
    // the warp w whose range [floor(w*Is/Ws), floor((w+1)*Is/Ws)) contains item t (Ws <= Is)
    return ((t + 1) * Ws - 1) / Is;
}

template <int BP>
__device__ void finish_row(const StreamArgs &a, int s, int64_t row, const float (&tot)[BP],
                           bool complete, int64_t row0, int64_t w, int64_t Ws, int64_t Is, int US_s)
{
    float *dst = a.out + ((int64_t)s * a.N + row) * a.B;
    if (complete) {
        for (int b = 0; b < a.B; ++b) dst[b] = tot[b];
        return;
    }
    const int64_t base = (int64_t)s * a.Gs * kWarps;
    const int side = (row == row0) ? 0 : 1;  // row0: the first row of this warp's range
    float *mine = a.slots + ((base + w) * 2 + side) * BP;
    for (int b = 0; b < BP; ++b) __stcg(mine + b, tot[b]);
    const int64_t wlo = warp_of_item(row * US_s, Ws, Is);
    const int64_t whi = warp_of_item((row + 1) * US_s - 1, Ws, Is);
    const unsigned n = (unsigned)(whi - wlo + 1);
    __threadfence();
    const unsigned old = atomicInc(a.cnt + base + wlo, n - 1);
    if (old != n - 1) return;
    __threadfence();
    float sum[BP];
    for (int b = 0; b < BP; ++b) sum[b] = 0.0f;
    for (int64_t w2 = wlo; w2 <= whi; ++w2) {
        const int64_t first_row = ((w2 * Is) / Ws) / US_s;
        const int side2 = (row == first_row) ? 0 : 1;
        const float *p = a.slots + ((base + w2) * 2 + side2) * BP;
        for (int b = 0; b < BP; ++b) sum[b] += __ldcg(p + b);
    }
    for (int b = 0; b < a.B; ++b) dst[b] = sum[b];
}

template <int FMT, int BP, int VAR>
__global__ void __launch_bounds__(kWarps * 32, 1) stream_gemv_kernel(const StreamArgs a)
{
    using UF = UnitFmt<FMT>;
    constexpr int UB = UF::kBytes;
    constexpr int CH = UF::kChunk;
    constexpr int CHB = CH * UB;

    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *ring = smem;
    float *xs = reinterpret_cast<float *>(smem + kWarps * kStages * CHB);
    float *xsum = xs + a.xs_floats;
    const int xsum_floats = (VAR == kVarFactored) ? a.US * 8 * BP : 0;
    uint64_t *bars = reinterpret_cast<uint64_t *>(xsum + xsum_floats);

    const int s = blockIdx.x / a.Gs;
    const int cta = blockIdx.x % a.Gs;
    const int US_s = min(a.US, a.UPR - s * a.US);
    const int64_t Is = a.N * US_s;
    const int64_t Ws = min((int64_t)a.Gs * kWarps, Is);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t w = (int64_t)cta * kWarps + warp;
    const bool active = w < Ws;

    int64_t t0 = 0, t1 = 0;
    if (active) {
        t0 = (w * Is) / Ws;
        t1 = ((w + 1) * Is) / Ws;
    }
    const int L = (int)(t1 - t0);  // units of this warp's range
    const int nch = (L + CH - 1) / CH;
    uint8_t *myring = ring + warp * kStages * CHB;
    const uint32_t bar0 = smem_u32(bars + warp * kStages);

    auto issue = [&](int i) {
        const int64_t ta = t0 + (int64_t)i * CH;
        const int64_t tb = min(ta + CH, t1);
        const uint32_t bar = bar0 + 8 * (i % kStages);
        const uint32_t dst0 = smem_u32(myring + (i % kStages) * CHB);
        const uint64_t policy = evict_first_policy();
        mbar_arrive_expect_tx(bar, (uint32_t)((tb - ta) * UB));
        if (a.S == 1) {
            bulk_g2s(dst0, a.W + ta * UB, (uint32_t)((tb - ta) * UB), bar, policy);
        } else {
            int64_t t = ta;
            while (t < tb) {
                const int64_t n = t / US_s, j = t - n * US_s;
                const int64_t e = min(tb, (n + 1) * US_s);
                const uint8_t *src = a.W + ((n * a.UPR) + (int64_t)s * a.US + j) * UB;
                bulk_g2s(dst0 + (uint32_t)((t - ta) * UB), src, (uint32_t)((e - t) * UB), bar, policy);
                t = e;
            }
        }
    };

    // 1. Weight prefetch: fill the ring.  W does not depend on the kernel before this one on the
    //    stream, so this may overlap that kernel's tail (programmatic dependent launch).
    if (active && lane == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(bar0 + 8 * i, 1);
        mbar_init_fence();
        for (int i = 0; i < kStages && i < nch; ++i) issue(i);
    }
    // 2. Let the next kernel on the stream begin its own prefetch as SMs free up, then wait for
    //    the previous kernel's results (x) before reading x or writing y / the workspace.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // 3. x for this slice -> shared memory (fp32, consumer order)
    stage_x<FMT, BP, VAR>(a, s, US_s, xs, xsum);
    __syncthreads();
    if (!active) return;
    __syncwarp();

    const int c = lane & 3;
    const int g = lane >> 2;  // unit of this lane within a pass of 8 units
    const int64_t row0 = t0 / US_s;
    int64_t row = row0;
    int j = (int)(t0 - row0 * US_s);  // position of the next pass's first unit within its row
    bool row_started_here = (j == 0);
    float acc[BP];
#pragma unroll
    for (int b = 0; b < BP; ++b) acc[b] = 0.0f;

    auto flush = [&](bool complete) {
        float tot[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) tot[b] = warp_sum(acc[b]);
        if (lane == 0) finish_row<BP>(a, s, row, tot, complete, row0, w, Ws, Is, US_s);
#pragma unroll
        for (int b = 0; b < BP; ++b) acc[b] = 0.0f;
    };

    for (int i = 0; i < nch; ++i) {
        const bool ok = mbar_wait_bounded(bar0 + 8 * (i % kStages), (uint32_t)((i / kStages) & 1));
        if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0) {
                atomicExch(a.err, kErrCopyTimeout);
                // let any copy still in flight into this warp's ring land before leaving
                for (int r = i + 1; r < nch && r < i + kStages; ++r)
                    (void)mbar_wait_bounded(bar0 + 8 * (r % kStages), (uint32_t)((r / kStages) & 1));
            }
            __syncwarp();
            return;
        }
        const uint8_t *stage = myring + (i % kStages) * CHB;
        const int nu = min(CH, L - i * CH);  // units in this chunk
        for (int p = 0; p < nu; p += 8) {
            const int pn = min(8, nu - p);  // units in this pass (8 except at the range's end)
            // the lane's unit position within its row, and how many rows past the current one
            int jj = j + g, rel = 0;
            while (jj >= US_s) {
                jj -= US_s;
                ++rel;
            }
            float v[BP];
#pragma unroll
            for (int b = 0; b < BP; ++b) v[b] = 0.0f;
            if (g < pn) {
                const uint8_t *u = stage + (p + g) * UB;
                if (FMT == kFmtQ4_K)
                    q4k_unit<BP, VAR>(u, c, xs, xsum, jj, v);
                else
                    q8_0_unit<BP>(u, c, xs, jj, v);
            }
            if (j + pn < US_s) {
                // the current row continues past this pass
#pragma unroll
                for (int b = 0; b < BP; ++b) acc[b] += v[b];
                j += pn;
            } else {
                // the current row ends inside this pass: hand contributions out row by row
                int k = 0, end = US_s - j;  // pass offset where row k ends
                while (true) {
                    if (rel == k) {
#pragma unroll
                        for (int b = 0; b < BP; ++b) acc[b] += v[b];
                    }
                    if (end > pn) {
                        j = pn - (end - US_s);
                        break;
                    }
                    flush(row_started_here);
                    ++row;
                    row_started_here = true;
                    ++k;
                    if (end == pn) {
                        j = 0;
                        break;
                    }
                    end += US_s;
                }
            }
        }
        __syncwarp();
        if (lane == 0 && i + kStages < nch) {
            fence_proxy_async_smem();
            issue(i + kStages);
        }
    }
    // the warp's range ends inside the current row: hand its partial to the row's last arriver
    if (j > 0) flush(false);
}

// Second pass of split-K: y[n][b] = sum over slices s = 0..S-1 (in that order) of part[s][n][b].
__global__ void splitk_sum_kernel(const float *part, float *y, int64_t NB, int S)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < NB;
         i += (int64_t)gridDim.x * blockDim.x) {
        float acc = part[i];
        for (int s = 1; s < S; ++s) acc += part[(int64_t)s * NB + i];
        y[i] = acc;
    }
}

// ------------------------------------------------------------------------------------------------
// Dump mode: the same decoding as the GEMV's direct form, written out as fp32 W[N][K].
// ------------------------------------------------------------------------------------------------
__global__ void dequant_q4k_kernel(const uint8_t *W, int64_t nsb, float *out)
{
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;  // (superblock, c)
    if (t >= nsb * 4) return;
    const int64_t sb = t >> 2;
    const int c = (int)(t & 3);
    const uint8_t *u = W + sb * 144;
    const uint4 hdr = *reinterpret_cast<const uint4 *>(u);
    const uint4 q0 = *reinterpret_cast<const uint4 *>(u + 16 + 32 * c);
    const uint4 q1 = *reinterpret_cast<const uint4 *>(u + 32 + 32 * c);
    const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    const Q4kDirectConsts kc = q4k_direct_consts(q4k_lane_scales(hdr, c));
    float *o = out + sb * 256 + 64 * c;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const Q4kWordWeights w = q4k_direct_word(qw[i], kc);
        // low nibbles: weights 4i+{0,2,1,3}; high nibbles: 32+4i+{0,2,1,3}
        o[4 * i + 0] = w.loA.x;
        o[4 * i + 2] = w.loA.y;
        o[4 * i + 1] = w.loB.x;
        o[4 * i + 3] = w.loB.y;
        o[32 + 4 * i + 0] = w.hiA.x;
        o[32 + 4 * i + 2] = w.hiA.y;
        o[32 + 4 * i + 1] = w.hiB.x;
        o[32 + 4 * i + 3] = w.hiB.y;
    }
}

__global__ void dequant_q8_0_kernel(const uint8_t *W, int64_t nblk, float *out)
{
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (t >= nblk) return;
    const uint8_t *u = W + t * 34;
    const float d = __half2float(__ushort_as_half((unsigned short)(u[0] | (u[1] << 8))));
    float *o = out + t * 32;
#pragma unroll 8
    for (int i = 0; i < 32; ++i) o[i] = d * (float)(int8_t)u[2 + i];
}

// ------------------------------------------------------------------------------------------------
// Q5_K and Q6_K, one weight at a time (the dump and the plain per-row kernel).  Byte loads only:
// Q6_K superblocks (210 B) are 2-byte aligned at best.
//   Q5_K {fp16 d; fp16 dmin; u8 scales[12]; u8 qh[32]; u8 qs[128]}: q = the Q4_K nibble of qs
//        plus 16 * bit (2c + (r >= 32)) of qh[r % 32] (c = i / 64, r = i % 64);
//        w = RN(d*sc_j*q - dmin*m_j), both products exact in fp32 (17 + 5 and 11 + 6 bits).
//   Q6_K {u8 ql[128]; u8 qh[64]; i8 scales[16]; fp16 d}: in half h = i / 128 with r = i % 128,
//        t = r / 32, l = r % 32: low nibble of ql[64h + 32(t % 2) + l] (t < 2) or its high nibble
//        (t >= 2), plus 16 * bits 2t..2t+1 of qh[32h + l]; w = RN(d*sc*(q - 32)), d*sc exact.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ float half_bits_to_float(const uint8_t *p)
{
    return __half2float(__ushort_as_half((unsigned short)(p[0] | (p[1] << 8))));
}

// GGML get_scale_min_k4: (sc_j, m_j) of sub-block j from the 12-byte table
__device__ __forceinline__ void kq_scale_min(const uint8_t *scales, int j, int &sc, int &m)
{
    if (j < 4) {
        sc = scales[j] & 63;
        m = scales[j + 4] & 63;
    } else {
        sc = (scales[j + 4] & 15) | ((scales[j - 4] >> 6) << 4);
        m = (scales[j + 4] >> 4) | ((scales[j] >> 6) << 4);
    }
}

__device__ __forceinline__ float q5k_weight(const uint8_t *blk, int i)
{
    int sc, m;
    kq_scale_min(blk + 4, i >> 5, sc, m);
    const int c = i >> 6, r = i & 63;
    const uint8_t qsb = blk[48 + 32 * c + (r & 31)];
    const int q = ((r < 32) ? (qsb & 15) : (qsb >> 4)) +
                  16 * ((blk[16 + (r & 31)] >> (2 * c + (r >> 5))) & 1);
    const float D = __fmul_rn(half_bits_to_float(blk), (float)sc);
    const float M = __fmul_rn(half_bits_to_float(blk + 2), (float)m);
    return __fsub_rn(__fmul_rn(D, (float)q), M);
}

__device__ __forceinline__ float q6k_weight(const uint8_t *blk, int i)
{
    const int h = i >> 7, r = i & 127, t = r >> 5, l = r & 31;
    const uint8_t lb = blk[64 * h + 32 * (t & 1) + l];
    const int q = ((t < 2) ? (lb & 15) : (lb >> 4)) + 16 * ((blk[128 + 32 * h + l] >> (2 * t)) & 3);
    const float D = __fmul_rn(half_bits_to_float(blk + 208), (float)(int8_t)blk[192 + (i >> 4)]);
    return __fmul_rn(D, (float)(q - 32));
}

// IQ4_XS {fp16 d; u16 scales_h; u8 scales_l[4]; u8 qs[128]}: sub-block j = i / 32 has the 6-bit
// ls_j = nibble (j % 2) of scales_l[j / 2] + 16 * bits 2j..2j+1 of scales_h; weight i's index is
// the low (r < 16) or high (r >= 16) nibble of qs[16j + r % 16], r = i % 32;
// w = d * (ls_j - 32) * level[index], exact in fp32 (d*(ls-32) has at most 16 significant bits,
// the level at most 7).
__device__ __forceinline__ int iq4_level(int v)
{
    const uint32_t w = (v < 8) ? ((v < 4) ? kIq4Lut0 : kIq4Lut1) : ((v < 12) ? kIq4Lut2 : kIq4Lut3);
    return (int)((w >> (8 * (v & 3))) & 0xFFu) - 128;
}

__device__ __forceinline__ float iq4xs_weight(const uint8_t *blk, int i)
{
    const int j = i >> 5, r = i & 31;
    const int sh = blk[2] | (blk[3] << 8);
    const int ls = ((blk[4 + (j >> 1)] >> (4 * (j & 1))) & 15) | (((sh >> (2 * j)) & 3) << 4);
    const uint8_t qb = blk[8 + 16 * j + (r & 15)];
    const int v = iq4_level((r < 16) ? (qb & 15) : (qb >> 4));
    return __fmul_rn(__fmul_rn(half_bits_to_float(blk), (float)(ls - 32)), (float)v);
}

template <int FMT> struct KqBlock {
    static constexpr int kBytes = (FMT == kFmtQ5_K) ? 176 : (FMT == kFmtQ6_K) ? 210 : 136;
};

template <int FMT>
__device__ __forceinline__ float kq_weight(const uint8_t *blk, int i)
{
    return (FMT == kFmtQ5_K) ? q5k_weight(blk, i) : (FMT == kFmtQ6_K) ? q6k_weight(blk, i)
                                                                        : iq4xs_weight(blk, i);
}

// dump: thread t writes the 16 weights of group t % 16 of superblock t / 16
template <int FMT>
__global__ void dequant_kq_kernel(const uint8_t *W, int64_t nsb, float *out)
{
    constexpr int SB = KqBlock<FMT>::kBytes;
    const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (t >= nsb * 16) return;
    const int64_t sb = t >> 4;
    const int g = (int)(t & 15);
    const uint8_t *blk = W + sb * SB;
    float *o = out + sb * 256 + 16 * g;
#pragma unroll 4
    for (int e = 0; e < 16; ++e) o[e] = kq_weight<FMT>(blk, 16 * g + e);
}

// ------------------------------------------------------------------------------------------------
// Plain per-row kernel (any K the format allows; no staging): one warp per row, lanes stride
// over blocks, correctly rounded weights as in the dump, fp32 partial sums, warp reduction.
// ------------------------------------------------------------------------------------------------
template <int FMT>
__global__ void rowwise_gemv_kernel(const uint8_t *W, int64_t N, int64_t K, const uint16_t *x, int B,
                                    float *y)
{
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t n = blockIdx.x * (int64_t)(blockDim.x >> 5) + (threadIdx.x >> 5); n < N;
         n += nwarps) {
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (FMT == kFmtQ4_K) {
            const int64_t nsb = K / 256;
            // lane -> (superblock, chunk c); 8 superblocks per warp step
            for (int64_t it = lane; it < nsb * 4; it += 32) {
                const int64_t sb = it >> 2;
                const int c = (int)(it & 3);
                const uint8_t *u = W + (n * nsb + sb) * 144;
                const uint4 hdr = *reinterpret_cast<const uint4 *>(u);
                const uint4 q0 = *reinterpret_cast<const uint4 *>(u + 16 + 32 * c);
                const uint4 q1 = *reinterpret_cast<const uint4 *>(u + 32 + 32 * c);
                const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
                const Q4kDirectConsts kc = q4k_direct_consts(q4k_lane_scales(hdr, c));
                const int64_t k0 = sb * 256 + 64 * c;
                for (int i = 0; i < 8; ++i) {
                    const Q4kWordWeights w = q4k_direct_word(qw[i], kc);
                    const float wl[4] = {w.loA.x, w.loB.x, w.loA.y, w.loB.y};  // weights 4i+0..3
                    const float wh[4] = {w.hiA.x, w.hiB.x, w.hiA.y, w.hiB.y};
                    for (int e = 0; e < 4; ++e) {
                        for (int b = 0; b < B; ++b) {
                            const float xl = __half2float(__ushort_as_half(x[(k0 + 4 * i + e) * B + b]));
                            const float xh =
                                __half2float(__ushort_as_half(x[(k0 + 32 + 4 * i + e) * B + b]));
                            acc[b] = fmaf(wl[e], xl, acc[b]);
                            acc[b] = fmaf(wh[e], xh, acc[b]);
                        }
                    }
                }
            }
        } else if (FMT == kFmtQ5_K || FMT == kFmtQ6_K || FMT == kFmtIQ4_XS) {
            constexpr int SB = KqBlock<FMT>::kBytes;
            const int64_t nsb = K / 256;
            // lane -> (superblock, 16-weight group)
            for (int64_t it = lane; it < nsb * 16; it += 32) {
                const int64_t sb = it >> 4;
                const int g = (int)(it & 15);
                const uint8_t *blk = W + (n * nsb + sb) * SB;
                const int64_t k0 = sb * 256 + 16 * g;
                for (int e = 0; e < 16; ++e) {
                    const float wv = kq_weight<FMT>(blk, 16 * g + e);
                    for (int b = 0; b < B; ++b)
                        acc[b] = fmaf(wv, __half2float(__ushort_as_half(x[(k0 + e) * B + b])), acc[b]);
                }
            }
        } else {
            const int64_t nblk = K / 32;
            for (int64_t t = lane; t < nblk; t += 32) {
                const uint8_t *u = W + (n * nblk + t) * 34;
                const float d = __half2float(__ushort_as_half((unsigned short)(u[0] | (u[1] << 8))));
                for (int i = 0; i < 32; ++i) {
                    const float wv = d * (float)(int8_t)u[2 + i];
                    for (int b = 0; b < B; ++b)
                        acc[b] = fmaf(wv, __half2float(__ushort_as_half(x[(t * 32 + i) * B + b])), acc[b]);
                }
            }
        }
        for (int b = 0; b < B; ++b) {
            const float tot = warp_sum(acc[b]);
            if (lane == 0) y[n * B + b] = tot;
        }
    }
}

// ------------------------------------------------------------------------------------------------
// x from page-locked host memory into device scratch (qg_gemv_host).  Each thread reads one
// 16-byte piece (or, unaligned, 8 halves one by one) of the host copy first, then waits for the
// previous kernel on the stream before it overwrites the scratch that kernel may still be
// reading; it lets the next kernel (the GEMV) launch at once, so the GEMV's weight prefetch
// overlaps the copy.  Reading the host copy before that wait is what the entry point's contract
// allows: x_host must not be written by device work queued before the call (a host-side caller
// fills it before making the call).
// ------------------------------------------------------------------------------------------------
__global__ void host_x_copy_kernel(const uint16_t *src, uint16_t *dst, int64_t n)
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t i0 = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) * 8;
    const bool aligned = ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0;
    uint16_t v[8];
    uint4 q = make_uint4(0u, 0u, 0u, 0u);
    const bool whole = aligned && i0 + 8 <= n;
    if (whole) {
        q = *reinterpret_cast<const uint4 *>(src + i0);
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = (i0 + k < n) ? src[i0 + k] : (uint16_t)0;
    }
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (whole) {
        *reinterpret_cast<uint4 *>(dst + i0) = q;
    } else {
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (i0 + k < n) dst[i0 + k] = v[k];
    }
}

// ------------------------------------------------------------------------------------------------
// Bandwidth probes.
// ------------------------------------------------------------------------------------------------
__global__ void hbm_copy_kernel(const uint4 *__restrict__ src, uint4 *__restrict__ dst, int64_t n16)
{
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n16;
         i += (int64_t)gridDim.x * blockDim.x)
        dst[i] = __ldcs(src + i);
}

__global__ void hbm_read_kernel(const uint4 *__restrict__ src, int64_t n16, uint32_t *out)
{
    uint32_t acc = 0;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n16;
         i += (int64_t)gridDim.x * blockDim.x) {
        const uint4 v = __ldcs(src + i);
        acc ^= v.x ^ v.y ^ v.z ^ v.w;
    }
    for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
    if ((threadIdx.x & 31) == 0) atomicXor(out + blockIdx.x, acc);
}

}  // namespace qg
