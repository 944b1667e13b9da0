// qg_umma.cuh -- the K-quant GEMV on the fifth-generation tensor cores (tcgen05, sm_100a).
//
// Operation (HARDWARE GROUND TRUTH: 2x NVIDIA Tesla T4 (Kaggle), second prompt, "SPEC"):
//   y[n,b] = sum_k dequant(W)[n,k] * x[k,b], Q4_K / Q5_K w = d*sc_j*q - dmin*m_j ("QUANTIZATION
//   MIX"), fp32 accumulation ("PHYSICS & CONTRACT"), B = 1..16 columns read against one pass over W.
//
// The arithmetic is the factored form of the CUDA-core kernel,
//   sum_i w_i x_i = sum_j [ d*sc_j * sum_{i in j} q_i x_i  -  dmin*m_j * sum_{i in j} x_i ],
// with the inner sums on the tensor cores.  Each code q enters the MMA as the normal fp16 number
// q 2^-10 (qg_codes.cuh: one LOP3 leaves the subnormal q 2^-24, one f16x2 multiply by a power of two
// normalises it), so every product with x is exact.  (Codes carried as fp16 subnormals, as the CUDA-core kernels do,
// lose accumulation precision in the tensor core: measured, the sums keep about 12 bits below the
// largest product then, 22 or more with normal operands.)
//
// Mapping.  A CTA owns a band of rows of one K slice, as in the CUDA-core kernel.  Its warps form
// warpgroups of four; a warpgroup takes (row tile, K part) pairs, a row tile being 128 rows: warp
// w % 4 of the group owns rows 32 (w % 4) .. +31 of the tile, which are also the tensor-memory
// lanes that warp may access.  Each warp streams its 32 rows x one 256-weight unit per step with a
// 2-D TMA copy into its own double-buffered ring (the CUDA-core kernel's ring).  Per 64-weight chunk
// c of a unit (sub-blocks 2c and 2c + 1), in one of two chunk slots:
//   1. every lane writes its row's 64 codes as 32 registers of fp16 pairs to tensor memory with
//      one tcgen05.st (32 columns: the A operand of four K = 16 steps, M = 128 rows) and its warp
//      arrives on the slot's "written" mbarrier (four arrivals complete it);
//   2. one thread of the warpgroup, one chunk later, waits for that barrier and issues four
//      tcgen05.mma kind::f16 (A from tensor memory, B = x from shared memory, D fp32 in tensor
//      memory): the two K-steps of sub-block 2c into one N = 16 accumulator tile, those of
//      sub-block 2c + 1 into a second, and commits them to the slot's "done" mbarrier;
//   3. before it writes the slot again, each warp waits for "done", reads its rows' accumulators
//      back (tcgen05.ld) and adds d*sc_j * D_j; the terms dmin*m_j * X_j (X_j from the staged x
//      sums) are applied at unpack time.
// No warp waits for the others of its group: only the issuing thread waits for the slot's four
// arrivals, and a warp waits only for MMAs issued a chunk before it needs their slot.
//
// B operand layout.  The MMA's N = 16 columns carry U = 16 / BP units of x times BP columns: the
// K-step t of unit j reads an N x 16 tile whose row n holds the x of unit U*(j/U) + n/BP, column
// n % BP, so x is stored once (no expansion at B = 1) and only the accumulator column
// (j % U) * BP + b of the tile is read back.  Tiles use the canonical no-swizzle K-major layout:
// 8-row x 16-byte core matrices, 128-byte aligned, k-halves 128 bytes apart (leading byte offset),
// 8-row groups 256 bytes apart (stride byte offset), K-step t of group g at 8192 g + 512 t.
#pragma once

#include <cuda.h>

#include "qg_codes.cuh"
#include "qg_device.cuh"
#include "qg_rows.cuh"

namespace qg {

// ------------------------------------------------------------------------------------------------
// tcgen05 wrappers (PTX ISA: tensor memory allocation, data movement, MMA, commit, fences)
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive 32-bit columns of this thread's lane
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
        "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
        "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// N consecutive 32-bit columns of this thread's lane (N = 1, 2, 4, 8, 16; taddr's column a
// multiple of N)
template <int N> struct TmemLd;
template <> struct TmemLd<1> {
    static __device__ __forceinline__ void run(uint32_t t, float *v)
    {
        uint32_t r0;
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r0) : "r"(t) : "memory");
        v[0] = __uint_as_float(r0);
    }
};
template <> struct TmemLd<2> {
    static __device__ __forceinline__ void run(uint32_t t, float *v)
    {
        uint32_t r0, r1;
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(t) : "memory");
        v[0] = __uint_as_float(r0);
        v[1] = __uint_as_float(r1);
    }
};
template <> struct TmemLd<4> {
    static __device__ __forceinline__ void run(uint32_t t, float *v)
    {
        uint32_t r[4];
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                     : "r"(t)
                     : "memory");
#pragma unroll
        for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
    }
};
template <> struct TmemLd<8> {
    static __device__ __forceinline__ void run(uint32_t t, float *v)
    {
        uint32_t r[8];
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                     : "r"(t)
                     : "memory");
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
    }
};
template <> struct TmemLd<16> {
    static __device__ __forceinline__ void run(uint32_t t, float *v)
    {
        uint32_t r[16];
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
            "%15}, [%16];"
            : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
              "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
            : "r"(t)
            : "memory");
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
    }
};

// D (+)= A * B: A (M = 128 x K = 16 f16) in tensor memory, B (K = 16 x N = 16 f16) in shared memory,
// D (fp32) in tensor memory; acc = 0 overwrites D
__device__ __forceinline__ void umma_f16_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a), "l"(bdesc), "r"(idesc), "r"(acc)
        : "memory");
}

// arrive (once) on the mbarrier when every MMA this thread issued so far has completed
__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// Shared-memory matrix descriptor: no swizzle, K-major canonical layout with 128-byte core
// matrices, leading byte offset 128 (the two 8-element k-halves), stride byte offset 256 (8-row
// groups), descriptor version 1.
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)(256u >> 4) << 32) |
           ((uint64_t)1 << 46);
}

// Instruction descriptor of kind::f16: D fp32, A and B fp16, both K-major, N = 16, M = 128.
constexpr uint32_t kUmmaIdesc = (1u << 4) | ((16u >> 3) << 17) | ((128u >> 4) << 24);

// one arrival (release) on an mbarrier of this CTA
__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// ------------------------------------------------------------------------------------------------
// Geometry
// ------------------------------------------------------------------------------------------------
template <int BP> struct UmmaWarps {
    // as many warpgroups as the shared memory allows next to x (x grows with BP)
    static constexpr int value = BP >= 16 ? 8 : BP >= 8 ? 12 : 16;
};
constexpr int kUmmaTmemCols = 512;   // 128 columns per warpgroup (two A slots, two D slots)
constexpr int kUmmaGroupBytes = 8192; // one B group: 16 K-steps x 16 rows x 16 k x 2 bytes

template <int FMT> struct UmmaFmt;
template <> struct UmmaFmt<kFmtQ4_K> { static constexpr int kUnitBytes = 144; };
template <> struct UmmaFmt<kFmtQ5_K> { static constexpr int kUnitBytes = 176; };

// ------------------------------------------------------------------------------------------------
// x staging.  Work item w = (((u * BP + b) * 4 + c) * 2 + s) * 2 + h) * 2 + hp covers the 8 weights
// 64c + 32s + 16h + 8hp + {0, 2, 1, 3, 4, 6, 5, 7} of unit u, column b: the elements 8hp .. 8hp + 7
// of K-step t = 4c + 2s + h in the order the A registers hold them.  The four items of sub-block
// 2c + s are adjacent lanes, which add their sums into X_j.  Units past the slice and columns past
// B are zero.
// ------------------------------------------------------------------------------------------------
template <int BP>
__device__ __forceinline__ void umma_stage_x(const RowsArgs &a, int s_idx, int US_s, int USP, uint8_t *xs,
                                             float *xsum)
{
    constexpr int U = 16 / BP;
    const int64_t kbase = (int64_t)s_idx * a.US * 256;
    const uint16_t *xsl = a.x + kbase * a.B;
    const int nitems = USP * BP * 32;  // a multiple of 32
    const bool vec = (BP == 1) && ((reinterpret_cast<uintptr_t>(xsl) & 15) == 0);
    auto load = [&](int w, uint32_t (&hv)[8]) {
        const int hp = w & 1, h = (w >> 1) & 1, s = (w >> 2) & 1, c = (w >> 3) & 3;
        const int rest = w >> 5;
        const int b = rest % BP, u = rest / BP;
        if (u < US_s && b < a.B) {
            const int e0 = u * 256 + 64 * c + 32 * s + 16 * h + 8 * hp;
            if (vec) {
                const uint4 v = *reinterpret_cast<const uint4 *>(xsl + e0);
                hv[0] = v.x & 0xFFFFu; hv[1] = v.x >> 16; hv[2] = v.y & 0xFFFFu; hv[3] = v.y >> 16;
                hv[4] = v.z & 0xFFFFu; hv[5] = v.z >> 16; hv[6] = v.w & 0xFFFFu; hv[7] = v.w >> 16;
            } else {
#pragma unroll
                for (int q = 0; q < 8; ++q) hv[q] = xsl[(int64_t)(e0 + q) * a.B + b];
            }
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) hv[q] = 0;
        }
    };
    auto store = [&](int w, const uint32_t (&hv)[8]) {
        const int hp = w & 1, h = (w >> 1) & 1, s = (w >> 2) & 1, c = (w >> 3) & 3;
        const int rest = w >> 5;
        const int b = rest % BP, u = rest / BP;
        const int t = 4 * c + 2 * s + h;
        const int n = (u % U) * BP + b;
        uint4 v;  // register order of the A operand: (e, e+2), (e+1, e+3), (e+4, e+6), (e+5, e+7)
        v.x = hv[0] | (hv[2] << 16);
        v.y = hv[1] | (hv[3] << 16);
        v.z = hv[4] | (hv[6] << 16);
        v.w = hv[5] | (hv[7] << 16);
        *reinterpret_cast<uint4 *>(xs + kUmmaGroupBytes * (u / U) + 512 * t + 256 * (n >> 3) + 128 * hp +
                                   16 * (n & 7)) = v;
        float sum = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) sum += __half2float(__ushort_as_half((unsigned short)hv[q]));
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        if ((w & 3) == 0 && u < US_s) xsum[(u * 8 + 2 * c + s) * BP + b] = sum;
    };
    const int nthr = blockDim.x;
    int w = threadIdx.x;
    for (; w + nthr < nitems; w += 2 * nthr) {
        uint32_t ha[8], hb[8];
        load(w, ha);
        load(w + nthr, hb);
        store(w, ha);
        store(w + nthr, hb);
    }
    for (; w < nitems; w += nthr) {
        uint32_t hv[8];
        load(w, hv);
        store(w, hv);
    }
}

// ------------------------------------------------------------------------------------------------
// The kernel
// ------------------------------------------------------------------------------------------------
template <int FMT, int BP, int MATS>
__global__ void __launch_bounds__(UmmaWarps<BP>::value * 32, 1)
    umma_gemv_kernel(const RowsArgs a, const __grid_constant__ WeightMaps<MATS> maps)
{
    constexpr int NW = UmmaWarps<BP>::value;
    constexpr int NWG = NW / 4;
    constexpr int NS = kRowsStages;
    constexpr int UB = UmmaFmt<FMT>::kUnitBytes;
    constexpr int BOX = 32 * UB;
    constexpr int INNER = UB / 4;
    constexpr int U = 16 / BP;
    static_assert(BOX % 128 == 0, "tensor-copy destinations in shared memory must be 128-byte aligned");
    static_assert(NW % 4 == 0 && NWG <= 4, "warpgroups of four warps, at most four per CTA");

    extern __shared__ __align__(128) uint8_t smem[];
    const int s = blockIdx.x / a.Gs;
    const int cta = blockIdx.x % a.Gs;
    const int US_s = min(a.US, a.UPR - s * a.US);
    const int USP = ((a.US + U - 1) / U) * U;  // staged units, a whole number of B groups
    uint8_t *ring = smem;
    uint8_t *xs = smem + NW * NS * BOX;  // B groups: 128-byte aligned core matrices (BOX is a 128 multiple)
    float *xsum = reinterpret_cast<float *>(xs + (size_t)USP * 512 * BP);
    float *red = xsum + a.US * 8 * BP;
    uint64_t *bars = reinterpret_cast<uint64_t *>(red + a.red_floats);  // ring bars, then MMA bars
    uint32_t *tslot = reinterpret_cast<uint32_t *>(bars + NW * NS + NWG * 4);

    const int64_t R0 = ((int64_t)cta * a.N) / a.Gs, R1 = ((int64_t)(cta + 1) * a.N) / a.Gs;
    const int rows = (int)(R1 - R0);
    const int T = (rows + 127) / 128;                 // row tiles per matrix
    const int P = max(1, min(NWG / max(MATS * T, 1), US_s));
    const int npairs = MATS * T * P;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wg = warp >> 2, quad = warp & 3;
    const int ucol0 = s * a.US;

    // the warp's steps: its warpgroup's pairs wg, wg + NWG, ..., each over units p, p + P, ...
    int nsteps = 0;
    for (int q = wg; q < npairs; q += NWG) nsteps += (US_s - q % P + P - 1) / P;
    // a pair's 32-row group of this warp: matrix, first row, and whether it has rows of the band
    auto pair_group = [&](int q, int &m, int &row0, bool &live) {
        const int tile = q / P;  // over MATS * T
        m = tile / T;
        const int g = 4 * (tile % T) + quad;  // 32-row group of the band in matrix m
        row0 = (int)R0 + 32 * g;
        live = 32 * g < rows;
    };

    uint8_t *myring = ring + warp * NS * BOX;
    const uint32_t bar0 = smem_u32(bars + warp * NS);
    const uint32_t fbar0 = smem_u32(bars + NW * NS + 4 * wg);      // A operand written (4 arrivals)
    const uint32_t dbar0 = smem_u32(bars + NW * NS + 4 * wg + 2);  // MMAs completed (commit)
    // issue cursor (lane 0): pair iq, unit iu, ring slot islot
    int iq = wg, iu = 0, islot = 0, im = 0, irow = 0;
    bool ilive = false;
    if (iq < npairs) { pair_group(iq, im, irow, ilive); iu = iq % P; }
    auto issue = [&](bool copy) {
        const uint32_t bar = bar0 + 8 * islot;
        if (copy && ilive) {
            mbar_arrive_expect_tx(bar, BOX);
            tma_load_2d(smem_u32(myring + islot * BOX), &maps.m[im], (ucol0 + iu) * INNER, irow, bar);
        }
        islot = (islot + 1 == NS) ? 0 : islot + 1;
        iu += P;
        if (iu >= US_s) {
            iq += NWG;
            if (iq < npairs) { pair_group(iq, im, irow, ilive); iu = iq % P; }
        }
    };

    // 1. tensor memory (warp 0), barriers, the first ring stage
    if (warp == 0) tmem_alloc(smem_u32(tslot), kUmmaTmemCols);
    if (nsteps > 0 && lane == 0) {
#pragma unroll
        for (int m = 0; m < MATS; ++m)
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.m[m])) : "memory");
        for (int i = 0; i < NS; ++i) mbar_init(bar0 + 8 * i, 1);
        if (quad == 0) {
            mbar_init(fbar0, 4);
            mbar_init(fbar0 + 8, 4);
            mbar_init(dbar0, 1);
            mbar_init(dbar0 + 8, 1);
        }
        mbar_init_fence();
        for (int i = 0; i < kPreStages && i < nsteps; ++i) issue(true);
    }
    // 2. programmatic dependent launch: wait for the previous kernel before reading x
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // 3. x of this slice as the MMA's B operand, and the x sums per sub-block
    umma_stage_x<BP>(a, s, US_s, USP, xs, xsum);
    if (lane == 0)
        for (int i = kPreStages; i < NS && i < nsteps; ++i) issue(true);
    fence_proxy_async_smem();  // the staged x is read by the tensor cores (async proxy)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tslot;
    const uint32_t lane_off = (uint32_t)(32 * quad) << 16;
    const uint32_t wg_col = tbase + 128u * wg;  // A slots at +0, +32; D slots at +64, +96
    const uint32_t xs_addr = smem_u32(xs);
    const bool issuer = (quad == 0) && (lane == 0);

    int step = 0, cslot = 0;
    uint32_t cphase = 0;  // ring consumer: slot and phase parity
    uint32_t dph = 0;     // "MMAs done" barrier parity, bit per chunk slot (every warp)
    uint32_t fph = 0;     // "A operand written" barrier parity, bit per chunk slot (the issuer)
    bool failed = false;
    // per chunk slot: a chunk whose MMAs are in flight and not yet added, its d*sc factors and the
    // accumulator column of its unit
    bool pend0 = false, pend1 = false;
    float e00 = 0.f, e01 = 0.f, e10 = 0.f, e11 = 0.f;
    int col0 = 0, col1 = 0;
    // the issuer's chunk written but not yet handed to the tensor cores: unit, chunk, slot
    bool prev = false;
    int prev_j = 0, prev_c = 0, prev_sl = 0;

    // On the first failure (a copy, or MMAs that never completed): record it, wait (bounded) for
    // this warp's copies still in flight, and copy nothing more.  The warp keeps stepping, so the
    // barriers' arrivals and phases stay matched.
    auto fail = [&]() {
        if (lane == 0 && !failed) {
            atomicExch(a.err, kErrCopyTimeout);
            int r_slot = cslot;
            uint32_t r_phase = cphase;
            for (int r = step + 1; r < nsteps && r < step + NS; ++r) {
                if (++r_slot == NS) { r_slot = 0; r_phase ^= 1u; }
                (void)mbar_wait_bounded(bar0 + 8 * r_slot, r_phase);
            }
        }
        failed = true;
    };
    // the MMAs of the chunk in slot sl have completed: add its two sub-block sums d*sc_j * D_j
    auto drain = [&](int sl, float (&acc)[BP]) {
        const bool ok = mbar_wait_bounded(dbar0 + 8 * sl, (dph >> sl) & 1u);
        if (!__all_sync(0xffffffffu, ok)) fail();
        dph ^= 1u << sl;
        tc_fence_after();
        float lo[BP], hi[BP];
        const uint32_t col = (uint32_t)(sl ? col1 : col0);
        TmemLd<BP>::run(lane_off + wg_col + 64u + 32u * sl + col, lo);
        TmemLd<BP>::run(lane_off + wg_col + 80u + 32u * sl + col, hi);
        tmem_wait_ld();
        const float f0 = sl ? e10 : e00, f1 = sl ? e11 : e01;
#pragma unroll
        for (int b = 0; b < BP; ++b) acc[b] = fmaf(f1, hi[b], fmaf(f0, lo[b], acc[b]));
        if (sl) pend1 = false; else pend0 = false;
    };
    // the issuer hands the previous chunk to the tensor cores once all four warps have written it:
    // sub-block 2c (K-steps 0, 1) into the slot's first accumulator tile, 2c + 1 into the second
    // (runs on the issuing lane alone; returns false if the wait gave up)
    auto issue_prev = [&]() -> bool {
        if (!prev) return true;
        const bool ok = mbar_wait_bounded(fbar0 + 8 * prev_sl, (fph >> prev_sl) & 1u);
        fph ^= 1u << prev_sl;
        tc_fence_after();
        const uint32_t bgrp = xs_addr + kUmmaGroupBytes * (prev_j / U);
#pragma unroll
        for (int sb = 0; sb < 2; ++sb)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                umma_f16_ts(wg_col + 64u + 32u * prev_sl + 16u * sb, wg_col + 32u * prev_sl + 8u * (2 * sb + h),
                            umma_desc(bgrp + 512u * (4 * prev_c + 2 * sb + h)), kUmmaIdesc, (uint32_t)h);
        umma_commit(dbar0 + 8 * prev_sl);
        prev = false;
        return ok;
    };
    // the issuing lane's hand-off, with its failure made warp-uniform
    auto hand_off = [&]() {
        bool bad = false;
        if (issuer) bad = !issue_prev();
        if (__any_sync(0xffffffffu, bad)) fail();
    };

    for (int q = wg; q < npairs; q += NWG) {
        int m, row0;
        bool live;
        pair_group(q, m, row0, live);
        (void)m;
        (void)row0;
        float acc[BP];
#pragma unroll
        for (int b = 0; b < BP; ++b) acc[b] = 0.0f;
        for (int j = q % P; j < US_s; j += P, ++step) {
            if (live && !failed) {
                const bool ok = mbar_wait_bounded(bar0 + 8 * cslot, cphase);
                if (!__all_sync(0xffffffffu, ok)) fail();
            }
            const uint8_t *u = myring + cslot * BOX + lane * UB;
            const uint4 hdr = *reinterpret_cast<const uint4 *>(u);
            const uint32_t SC_lo = hdr.y & 0x3F3F3F3Fu;
            const uint32_t MM_lo = hdr.z & 0x3F3F3F3Fu;
            const uint32_t SC_hi = (hdr.w & 0x0F0F0F0Fu) | ((hdr.y >> 2) & 0x30303030u);
            const uint32_t MM_hi = ((hdr.w >> 4) & 0x0F0F0F0Fu) | ((hdr.z >> 2) & 0x30303030u);
            __half2 dd;
            *reinterpret_cast<uint32_t *>(&dd) = hdr.x;
            const float2 dm = __half22float2(dd);  // (d, dmin), exact
            uint32_t hq[8];
            if (FMT == kFmtQ5_K) {
                const uint4 h0 = *reinterpret_cast<const uint4 *>(u + 16);
                const uint4 h1 = *reinterpret_cast<const uint4 *>(u + 32);
                hq[0] = h0.x; hq[1] = h0.y; hq[2] = h0.z; hq[3] = h0.w;
                hq[4] = h1.x; hq[5] = h1.y; hq[6] = h1.z; hq[7] = h1.w;
            }
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int sl = c & 1;  // compile-time under the unrolled loop
                if (sl ? pend1 : pend0) drain(sl, acc);
                const uint32_t scw = c < 2 ? SC_lo : SC_hi;
                const uint32_t mmw = c < 2 ? MM_lo : MM_hi;
                const int shb = 16 * (c & 1);
                const float dsc0 = dm.x * (float)((scw >> shb) & 0xFFu);
                const float dsc1 = dm.x * (float)((scw >> (shb + 8)) & 0xFFu);
                const float dmm0 = dm.y * (float)((mmw >> shb) & 0xFFu);
                const float dmm1 = dm.y * (float)((mmw >> (shb + 8)) & 0xFFu);
                const int qs0 = (FMT == kFmtQ4_K) ? 16 : 48;
                const uint4 q0 = *reinterpret_cast<const uint4 *>(u + qs0 + 32 * c);
                const uint4 q1 = *reinterpret_cast<const uint4 *>(u + qs0 + 16 + 32 * c);
                const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
                uint32_t r[32];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    // codes as the normal fp16 numbers q 2^-10 (qg_codes.cuh): every product with
                    // x is exact and the tensor core keeps its full accumulation precision
                    uint32_t a0, a1, a2, a3;
                    if (FMT == kFmtQ4_K) {
                        const uint32_t w = qw[i], v = __umulhi(w, 1u << 24);  // v = w >> 8
                        a0 = f16x2_mul(w & 0x000F000Fu, kF16x2_2p14);  // low nibbles of bytes 0, 2
                        a1 = f16x2_mul(v & 0x000F000Fu, kF16x2_2p14);  // low nibbles of bytes 1, 3
                        a2 = f16x2_mul(w & 0x00F000F0u, kF16x2_2p10);  // high nibbles of bytes 0, 2
                        a3 = f16x2_mul(v & 0x00F000F0u, kF16x2_2p10);  // high nibbles of bytes 1, 3
                    } else {
                        const uint32_t hw = hq[i];
                        const uint32_t t1 = (c == 0) ? hw << 4 : (c == 1) ? hw << 2 : (c == 2) ? hw : hw >> 2;
                        const uint32_t t2 = (c == 0) ? hw << 3 : (c == 1) ? hw << 1 : (c == 2) ? hw >> 1 : hw >> 3;
                        const uint32_t wl = (qw[i] & 0x0F0F0F0Fu) | (t1 & 0xF0F0F0F0u);
                        const uint32_t wh = ((qw[i] >> 4) & 0x0F0F0F0Fu) | (t2 & 0xF0F0F0F0u);
                        a0 = f16x2_mul(wl & 0x001F001Fu, kF16x2_2p14);
                        a1 = f16x2_mul(__umulhi(wl, 1u << 24) & 0x001F001Fu, kF16x2_2p14);
                        a2 = f16x2_mul(wh & 0x001F001Fu, kF16x2_2p14);
                        a3 = f16x2_mul(__umulhi(wh, 1u << 24) & 0x001F001Fu, kF16x2_2p14);
                    }
                    // K-step (s, h) with h = i / 4 holds columns 8 (2s + h) + 2 (i % 4) + {0, 1}: the
                    // weights (e, e+2) then (e+1, e+3) of the word
                    const int cl = 8 * (i >> 2) + 2 * (i & 3);
                    r[cl] = live ? a0 : 0u;
                    r[cl + 1] = live ? a1 : 0u;
                    r[16 + cl] = live ? a2 : 0u;
                    r[16 + cl + 1] = live ? a3 : 0u;
                }
                // the min terms now: sum w x = d sc D - dmin m X per sub-block
#pragma unroll
                for (int b = 0; b < BP; ++b) {
                    const float X0 = xsum[(j * 8 + 2 * c) * BP + b];
                    const float X1 = xsum[(j * 8 + 2 * c + 1) * BP + b];
                    acc[b] = fmaf(-dmm1, X1, fmaf(-dmm0, X0, acc[b]));
                }
                // the accumulators hold sums of (q 2^-10) x
                if (sl) { e10 = dsc0 * 1024.0f; e11 = dsc1 * 1024.0f; col1 = (j % U) * BP; }
                else    { e00 = dsc0 * 1024.0f; e01 = dsc1 * 1024.0f; col0 = (j % U) * BP; }
                tmem_st32(lane_off + wg_col + 32u * sl, r);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(fbar0 + 8 * sl);
                hand_off();
                if (issuer) { prev = true; prev_j = j; prev_c = c; prev_sl = sl; }
                if (sl) pend1 = true; else pend0 = true;
            }
            // the unit is in registers and tensor memory: refill its ring slot (after a failure the
            // cursor only moves on, so the consumer's slots and phases stay in step)
            __syncwarp();
            if (lane == 0 && step + NS < nsteps) {
                fence_proxy_async_smem();
                issue(!failed);
            }
            if (++cslot == NS) { cslot = 0; cphase ^= 1u; }
        }
        // the pair's last chunk to the tensor cores, then its last two chunks' sums
        hand_off();
        // older chunk first: the last chunk went to slot 1 (four chunks per unit)
        if (pend0) drain(0, acc);
        if (pend1) drain(1, acc);
        // this warp's 32 rows of the pair: partial rows of its (group, part)
        const int tile = q / P;
        const int g = (tile / T) * (4 * T) + 4 * (tile % T) + quad;  // group index over both matrices
        float *rp = red + ((size_t)(g * P + q % P) * 32 + lane) * BP;
#pragma unroll
        for (int b = 0; b < BP; ++b) rp[b] = acc[b];
    }
    tc_fence_before();
    const bool any_failed = __syncthreads_or(failed ? 1 : 0);
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tbase, kUmmaTmemCols);
    }
    // 4. rows of the band: sum the K parts in part order, write once (or this slice's partials)
    BandShape bs;
    bs.Gm = 4 * T;
    bs.G = MATS * bs.Gm;
    bs.P = P;
    if (!any_failed) band_finish<BP, MATS>(a, bs, red, s, R0, rows);
    // 5. K slices: the last CTA of the band adds them up
    if (a.S > 1) splitk_fixup<MATS>(a, cta, R0, rows, reinterpret_cast<int *>(xsum));
}

}  // namespace qg
