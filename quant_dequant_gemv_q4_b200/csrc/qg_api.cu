// qg_api.cu -- host side of libqg's C ABI: argument checks, launch planning, the per-stream
// workspace, kernel dispatch.  Declarations and contracts: include/qg.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <tuple>
#include <utility>

#include "../../include/qg.h"
#include "qg_device.cuh"
#include "qg_rows.cuh"
#include "qg_mma.cuh"
#include "qg_umma.cuh"

#include <cudaTypedefs.h>

namespace {

using namespace qg;

struct DeviceInfo {
    int sms = 0;
    int smem_optin = 0;
};

std::mutex g_mu;
std::map<int, DeviceInfo> g_dev;
constexpr size_t kCachePlans = 4096;  // bound of the launch-plan cache
std::set<std::pair<int, const void *>> g_attr_set;

thread_local int t_last_variant = 0;
thread_local int t_last_splits = 0;

int device_info(DeviceInfo *out, int *dev_out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QG_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_dev.find(dev);
    if (it == g_dev.end()) {
        DeviceInfo d;
        if (cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
                cudaSuccess)
            return QG_ERR_CUDA;
        it = g_dev.emplace(dev, d).first;
    }
    *out = it->second;
    *dev_out = dev;
    return QG_OK;
}

// Raise a kernel's dynamic shared-memory limit once per (device, kernel).
int ensure_smem_attr(int dev, const void *func, int bytes)
{
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (g_attr_set.count({dev, func})) return QG_OK;
    }
    // static and dynamic shared memory together must fit the per-block limit
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, func) != cudaSuccess) return QG_ERR_CUDA;
    const int dyn = bytes - (int)fa.sharedSizeBytes;
    if (dyn <= 0 ||
        cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn) != cudaSuccess)
        return QG_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_mu);
    g_attr_set.insert({dev, func});
    return QG_OK;
}

// ---------------------------------------------------------------------------------------------
// Workspace: one per (device, stream).  Layout: [err int | pad to 256] [cnt uint[nw]]
// [slots float[nw*2*8]] [part float[...]].  Counters are zeroed once at allocation; every
// completed call leaves them at zero again (each counter wraps after its last arrival).
// ---------------------------------------------------------------------------------------------
struct Workspace {
    uint8_t *base = nullptr;
    size_t bytes = 0;
    size_t nw = 0;       // warps covered by cnt
    size_t slot_f = 0;   // floats of split-row partial sums
    size_t part_f = 0;   // floats of the split-K partial buffer
};
std::map<std::pair<int, void *>, Workspace> g_ws;

struct WsView {
    int *err;
    unsigned *cnt;
    float *slots;
    float *part;
};

size_t ws_bytes_for(size_t nw, size_t slot_f, size_t part_f)
{
    const size_t cnt_b = ((nw * sizeof(unsigned) + 255) / 256) * 256;
    const size_t slot_b = ((slot_f * sizeof(float) + 255) / 256) * 256;
    return 256 + cnt_b + slot_b + part_f * sizeof(float) + 256;
}

WsView ws_view(const Workspace &w)
{
    WsView v;
    const size_t cnt_b = ((w.nw * sizeof(unsigned) + 255) / 256) * 256;
    const size_t slot_b = ((w.slot_f * sizeof(float) + 255) / 256) * 256;
    v.err = reinterpret_cast<int *>(w.base);
    v.cnt = reinterpret_cast<unsigned *>(w.base + 256);
    v.slots = reinterpret_cast<float *>(w.base + 256 + cnt_b);
    v.part = reinterpret_cast<float *>(w.base + 256 + cnt_b + slot_b);
    return v;
}

int get_workspace(int dev, void *stream, size_t nw, size_t slot_f, size_t part_f, WsView *out)
{
    std::lock_guard<std::mutex> lk(g_mu);
    Workspace &w = g_ws[{dev, stream}];
    if (w.base && w.nw >= nw && w.slot_f >= slot_f && w.part_f >= part_f) {
        *out = ws_view(w);
        return QG_OK;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cap) != cudaSuccess)
        return QG_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return QG_ERR_NOMEM;  // cannot grow while capturing
    const size_t new_nw = std::max(nw, w.nw);
    const size_t new_sf = std::max(slot_f, w.slot_f);
    const size_t new_pf = std::max(part_f, w.part_f);
    const size_t bytes = ws_bytes_for(new_nw, new_sf, new_pf);
    if (w.base) {
        // the old buffer may still be read by work queued on this stream
        if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return QG_ERR_CUDA;
        cudaFree(w.base);
        w.base = nullptr;
    }
    void *p = nullptr;
    if (cudaMalloc(&p, bytes) != cudaSuccess) {
        w = Workspace();
        return QG_ERR_NOMEM;
    }
    if (cudaMemset(p, 0, bytes) != cudaSuccess) {
        cudaFree(p);
        w = Workspace();
        return QG_ERR_CUDA;
    }
    w.base = static_cast<uint8_t *>(p);
    w.bytes = bytes;
    w.nw = new_nw;
    w.slot_f = new_sf;
    w.part_f = new_pf;
    *out = ws_view(w);
    return QG_OK;
}

// ---------------------------------------------------------------------------------------------
// Planning.
// ---------------------------------------------------------------------------------------------
// columns of x: 1..8 on every kernel, up to 16 on the tensor-core kernel (Q4_K, K % 256 == 0)
constexpr int kMaxB = 16;

int padded_cols(int B) { return B == 1 ? 1 : B == 2 ? 2 : B <= 4 ? 4 : B <= 8 ? 8 : 16; }

struct Plan {
    int BP, S, US, Gs, G, xs_floats;
    size_t smem;
};

Plan make_plan(int fmt, int var, int64_t N, int64_t K, int B, const DeviceInfo &di)
{
    Plan p;
    p.BP = padded_cols(B);
    const int UB = (fmt == kFmtQ4_K) ? UnitFmt<kFmtQ4_K>::kBytes : UnitFmt<kFmtQ8_0>::kBytes;
    const int CH = (fmt == kFmtQ4_K) ? UnitFmt<kFmtQ4_K>::kChunk : UnitFmt<kFmtQ8_0>::kChunk;
    const size_t ring = (size_t)kWarps * kStages * CH * UB;
    const size_t bars = (size_t)kWarps * kStages * 8;
    const bool factored = (fmt == kFmtQ4_K && var == kVarFactored);
    const size_t per_unit = (size_t)(256 * p.BP + (factored ? 8 * p.BP : 0)) * sizeof(float);
    const size_t avail = (size_t)di.smem_optin - ring - bars - 128;
    int64_t fit = (int64_t)(avail / per_unit);
    fit -= fit & 1;  // staged x is allocated in pairs of units
    if (fit < 2) fit = 2;
    const int64_t UPR = K / 256;
    int64_t S = (UPR + fit - 1) / fit;
    const int64_t US = (UPR + S - 1) / S;
    S = (UPR + US - 1) / US;
    p.S = (int)S;
    p.US = (int)US;
    p.xs_floats = (int)(((US + 1) / 2) * 2 * 256 * p.BP);
    const size_t xsum_f = factored ? (size_t)US * 8 * p.BP : 0;
    p.smem = ring + (size_t)p.xs_floats * sizeof(float) + xsum_f * sizeof(float) + bars;
    const int64_t items = N * US;
    const int64_t want = std::max<int64_t>(1, (items + kWarps * 8 - 1) / (kWarps * 8));
    const int64_t per_slice = std::max<int64_t>(1, di.sms / S);
    p.Gs = (int)std::min(per_slice, want);
    p.G = p.Gs * p.S;
    return p;
}

const void *stream_kernel_ptr(int fmt, int BP, int var)
{
#define QG_PICK(F, V)                                                           \
    switch (BP) {                                                              \
    case 1: return reinterpret_cast<const void *>(&stream_gemv_kernel<F, 1, V>); \
    case 2: return reinterpret_cast<const void *>(&stream_gemv_kernel<F, 2, V>); \
    case 4: return reinterpret_cast<const void *>(&stream_gemv_kernel<F, 4, V>); \
    default: return reinterpret_cast<const void *>(&stream_gemv_kernel<F, 8, V>); \
    }
    (void)var;
    if (fmt == kFmtQ8_0) {
        QG_PICK(kFmtQ8_0, kVarDirect)
    } else {
        QG_PICK(kFmtQ4_K, kVarDirect)
    }
#undef QG_PICK
}

// Plan of the row-band kernel.
struct RowsPlan {
    int BP, NW, S, US, Gs, G, red_floats;
    size_t smem;
    bool tensor;  // mma_gemv_kernel instead of rows_gemv_kernel
    bool umma;    // umma_gemv_kernel (tcgen05) instead of either
};

RowsPlan make_rows_plan(int fmt, int64_t N, int64_t K, int B, const DeviceInfo &di, bool tensor,
                        int mats = 1)
{
    RowsPlan best{};
    double best_util = -1.0;
    const int BP = padded_cols(B);
    int LB = 0, groups_per_unit = 8, NW = 0;
    switch (fmt) {
    case kFmtQ4_K:
        LB = RowsFmt<kFmtQ4_K>::kLaneBytes;
        NW = BP >= 8 ? RowsWarps<kFmtQ4_K, 8>::value : RowsWarps<kFmtQ4_K, 1>::value;
        break;
    case kFmtQ5_K:
        LB = RowsFmt<kFmtQ5_K>::kLaneBytes;
        NW = BP >= 8 ? RowsWarps<kFmtQ5_K, 8>::value : RowsWarps<kFmtQ5_K, 1>::value;
        break;
    case kFmtQ6_K:
        LB = RowsFmt<kFmtQ6_K>::kLaneBytes;
        groups_per_unit = RowsFmt<kFmtQ6_K>::kGroups;
        NW = BP >= 4 ? RowsWarps<kFmtQ6_K, 4>::value : RowsWarps<kFmtQ6_K, 1>::value;
        break;
    case kFmtIQ4_XS:
        LB = RowsFmt<kFmtIQ4_XS>::kLaneBytes;
        NW = BP >= 8 ? RowsWarps<kFmtIQ4_XS, 8>::value : RowsWarps<kFmtIQ4_XS, 1>::value;
        break;
    default:
        LB = RowsFmt<kFmtQ8_0>::kLaneBytes;
        NW = BP >= 4 ? RowsWarps<kFmtQ8_0, 4>::value : RowsWarps<kFmtQ8_0, 1>::value;
        break;
    }
    int tab_floats = 0;  // per-warp table of the tensor-core kernel
    if (tensor) {
        if (fmt == kFmtQ6_K) {
            LB = MmaFmt<kFmtQ6_K>::kUnitBytes;
            NW = MmaWarpsF<kFmtQ6_K, 1>::value;
            tab_floats = std::max(512, 32 * BP);
        } else if (fmt == kFmtQ8_0) {
            LB = MmaFmt<kFmtQ8_0>::kUnitBytes;
            NW = BP >= 8 ? MmaWarpsF<kFmtQ8_0, 8>::value : MmaWarpsF<kFmtQ8_0, 1>::value;
            tab_floats = std::max(256, 32 * BP);
        } else {
            LB = (fmt == kFmtQ5_K)     ? MmaFmt<kFmtQ5_K>::kUnitBytes
                 : (fmt == kFmtIQ4_XS) ? MmaFmt<kFmtIQ4_XS>::kUnitBytes
                                       : MmaFmt<kFmtQ4_K>::kUnitBytes;
            NW = BP >= 16 ? MmaWarps<16>::value : BP >= 8 ? MmaWarps<8>::value : MmaWarps<1>::value;
            tab_floats = std::max(256, 32 * BP);
        }
    }
    const size_t ring = (size_t)NW * kRowsStages * 32 * LB;
    const size_t tabs = (size_t)NW * tab_floats * sizeof(float);
    const size_t bars = (size_t)NW * kRowsStages * 8;

    const int64_t UPR = K / 256;
    // K slices.  Among the slicings whose shared memory fits (and, past one slice, whose slices
    // keep at least 5 units of a row, so that each row is still read in long runs), the least
    //   cost = max(steps of a CTA, NW * steps of its busiest warp) + [S > 1] * 16 * 144 / UB
    // in 32-row steps: a call took about 3.3 us + 0.11 us per step of a CTA, plus about 1.8 us
    // (16 Q4_K steps) for the cross-CTA sum of K slices, when measured over slicings of the FFN,
    // attention and SSM shapes at B = 1 and 8 (the warp term covers bands with too few (row
    // group, K part) pairs to keep every warp streaming).  Ties: fewer steps, then fewer slices.
    // The tensor-core kernel only takes slicings with at most one pair per warp.  If no slicing
    // qualifies, the one with the most busy lanes.
    const int UB = tensor ? (fmt == kFmtQ5_K ? 176 : fmt == kFmtQ6_K ? 210 : fmt == kFmtIQ4_XS ? 136
                             : fmt == kFmtQ8_0 ? 272 : 144)
                          : (fmt == kFmtQ6_K ? 210 : fmt == kFmtIQ4_XS ? 136 : LB);
    double best_cost = 1e300;
    int64_t best_steps = INT64_MAX;
    RowsPlan util_best{};
    // at most 64 slices, and no more slices than SMs (every slice gets at least one CTA per wave)
    const int64_t max_slices = std::min<int64_t>(std::min<int64_t>(UPR, 64), std::max(di.sms, 1));
    for (int64_t S0 = 1; S0 <= max_slices; ++S0) {
        const int64_t US = (UPR + S0 - 1) / S0;
        const int64_t S = (UPR + US - 1) / US;
        if (S != S0) continue;  // the same slicing as a smaller S0
        const int64_t Gs = std::max<int64_t>(1, std::min<int64_t>(di.sms / S, N));
        // partial rows: one (group, part) pair per warp, or, for the gate/up pair, every group of
        // both matrices when there are more groups than warps
        const int64_t band_rows = (N + Gs - 1) / Gs;
        const int64_t groups = (int64_t)mats * ((band_rows + 31) / 32);
        const int red = (int)((mats == 1 ? NW : std::max<int64_t>(NW, groups)) * 32 * BP);
        const size_t xbytes = (size_t)US * (512 + 4 * groups_per_unit) * BP;
        const size_t smem = ring + xbytes + tabs + (size_t)red * sizeof(float) + bars;
        if (smem > (size_t)di.smem_optin) continue;  // the kernels have no static shared memory
        const double util = ((double)N / (double)Gs) / (32.0 * (double)((N / Gs + 31) / 32 > 0 ? (N / Gs + 31) / 32 : 1));
        RowsPlan p;
        p.BP = BP;
        p.NW = NW;
        p.S = (int)S;
        p.US = (int)US;
        p.Gs = (int)Gs;
        p.G = (int)(Gs * S);
        p.red_floats = red;
        p.smem = smem;
        p.tensor = tensor;
        p.umma = false;
        if (util > best_util) {
            best_util = util;
            util_best = p;
        }
        if (S > 1 && US < 5) continue;
        const int64_t P = std::max<int64_t>(1, std::min<int64_t>(NW / std::max<int64_t>(groups, 1), US));
        if (tensor && groups * P > NW) continue;  // measured slower: tensor-core warps with two pairs
        const int64_t warp_steps = ((groups * P + NW - 1) / NW) * ((US + P - 1) / P);
        const int64_t steps = groups * US;
        const double cost = (double)std::max<int64_t>(steps, NW * warp_steps) + (S > 1 ? 16.0 * 144.0 / UB : 0.0);
        if (cost < best_cost || (cost == best_cost && steps < best_steps)) {
            best_cost = cost;
            best_steps = steps;
            best = p;
        }
    }
    if (best.smem == 0) best = util_best;
    return best;  // smem == 0 if nothing fits
}

// Plan of the tcgen05 kernel: the same bands and K slices as the row-band kernels, with warpgroups
// of four warps taking (128-row tile, K part) pairs.  Among the slicings whose shared memory fits
// (and, past one slice, keep at least 5 units of a row per slice), the least
//   cost = max(32-row steps of a CTA, warps x steps of its busiest warp) + [S > 1] * 16 * 144 / UB,
// the row-band kernels' model with a warp's step being its quarter of a warpgroup step.
RowsPlan make_umma_plan(int fmt, int64_t N, int64_t K, int B, const DeviceInfo &di, int mats = 1)
{
    RowsPlan best{};
    const int BP = padded_cols(B);
    const int NW = BP >= 16 ? UmmaWarps<16>::value : BP >= 8 ? UmmaWarps<8>::value : UmmaWarps<1>::value;
    const int NWG = NW / 4;
    const int UB = (fmt == kFmtQ5_K) ? UmmaFmt<kFmtQ5_K>::kUnitBytes : UmmaFmt<kFmtQ4_K>::kUnitBytes;
    const int U = 16 / BP;
    const size_t ring = (size_t)NW * kRowsStages * 32 * UB;
    const size_t bars = (size_t)(NW * kRowsStages + NWG * 4) * 8 + 16;
    const int64_t UPR = K / 256;
    const int64_t max_slices = std::min<int64_t>(std::min<int64_t>(UPR, 64), std::max(di.sms, 1));
    double best_cost = 1e300;
    int64_t best_steps = INT64_MAX;
    for (int64_t S0 = 1; S0 <= max_slices; ++S0) {
        const int64_t US = (UPR + S0 - 1) / S0;
        const int64_t S = (UPR + US - 1) / US;
        if (S != S0) continue;
        if (S > 1 && US < 5) continue;
        const int64_t Gs = std::max<int64_t>(1, std::min<int64_t>(di.sms / S, N));
        const int64_t band_rows = (N + Gs - 1) / Gs;
        const int64_t T = (band_rows + 127) / 128;
        const int64_t P = std::max<int64_t>(1, std::min<int64_t>(NWG / std::max<int64_t>(mats * T, 1), US));
        const int64_t pairs = mats * T * P;
        const int64_t USP = ((US + U - 1) / U) * U;
        // partial rows of every (32-row group, K part); a CTA with fewer rows than band_rows may
        // have fewer tiles and more parts, so take the largest tiles x parts over T' <= T
        int64_t tp = 0;
        for (int64_t T1 = 1; T1 <= T; ++T1)
            tp = std::max<int64_t>(tp, T1 * std::max<int64_t>(1, std::min<int64_t>(NWG / std::max<int64_t>(mats * T1, 1), US)));
        const int64_t red = mats * 4 * tp * 32 * BP;
        const size_t smem = ring + (size_t)USP * 512 * BP + (size_t)US * 8 * BP * 4 + (size_t)red * 4 + bars;
        if (smem > (size_t)di.smem_optin) continue;
        const int64_t warp_steps = ((pairs + NWG - 1) / NWG) * ((US + P - 1) / P);
        const int64_t steps = mats * 4 * T * US;
        const double cost = (double)std::max<int64_t>(steps, NW * warp_steps) + (S > 1 ? 16.0 * 144.0 / UB : 0.0);
        if (cost < best_cost || (cost == best_cost && steps < best_steps)) {
            best_cost = cost;
            best_steps = steps;
            best.BP = BP;
            best.NW = NW;
            best.S = (int)S;
            best.US = (int)US;
            best.Gs = (int)Gs;
            best.G = (int)(Gs * S);
            best.red_floats = (int)red;
            best.smem = smem;
            best.tensor = true;
            best.umma = true;
        }
    }
    return best;  // smem == 0 if nothing fits
}

// The plan of a call (a pure function of the device's SM count and shared memory, the kernel
// variant and the shape), cached: kind 0 = CUDA-core rows kernel, 1 = tensor-core kernel,
// 2 = tcgen05 kernel.
std::map<std::tuple<int, int, int, int, int64_t, int64_t, int, int>, RowsPlan> g_plans;

RowsPlan plan_cached(int kind, int fmt, int64_t N, int64_t K, int B, const DeviceInfo &di, int mats = 1)
{
    const auto key = std::make_tuple(di.sms, di.smem_optin, kind, fmt, N, K, B, mats);
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_plans.find(key);
        if (it != g_plans.end()) return it->second;
    }
    const RowsPlan p = (kind == 2) ? make_umma_plan(fmt, N, K, B, di, mats)
                                   : make_rows_plan(fmt, N, K, B, di, kind == 1, mats);
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_plans.size() >= kCachePlans) g_plans.clear();
    g_plans.emplace(key, p);
    return p;
}

const void *umma_kernel_ptr(int fmt, int BP, int mats)
{
#define QG_UMMA_SWITCH(F, M)                                                              \
    switch (BP) {                                                                         \
    case 1: return reinterpret_cast<const void *>(&umma_gemv_kernel<F, 1, M>);          \
    case 2: return reinterpret_cast<const void *>(&umma_gemv_kernel<F, 2, M>);          \
    case 4: return reinterpret_cast<const void *>(&umma_gemv_kernel<F, 4, M>);          \
    case 8: return reinterpret_cast<const void *>(&umma_gemv_kernel<F, 8, M>);          \
    default: return reinterpret_cast<const void *>(&umma_gemv_kernel<F, 16, M>);        \
    }
    if (fmt == kFmtQ5_K) {
        if (mats == 2) { QG_UMMA_SWITCH(kFmtQ5_K, 2) }
        QG_UMMA_SWITCH(kFmtQ5_K, 1)
    }
    if (mats == 2) { QG_UMMA_SWITCH(kFmtQ4_K, 2) }
    QG_UMMA_SWITCH(kFmtQ4_K, 1)
#undef QG_UMMA_SWITCH
}

const void *rows_kernel_ptr(int fmt, int BP, bool tensor, int mats)
{
#define QG_BP_SWITCH(KERNEL)                                                   \
    switch (BP) {                                                              \
    case 1: return reinterpret_cast<const void *>(&KERNEL(1));                 \
    case 2: return reinterpret_cast<const void *>(&KERNEL(2));                 \
    case 4: return reinterpret_cast<const void *>(&KERNEL(4));                 \
    default: return reinterpret_cast<const void *>(&KERNEL(8));                \
    }
#define QG_BP_SWITCH16(KERNEL)                                                 \
    switch (BP) {                                                              \
    case 1: return reinterpret_cast<const void *>(&KERNEL(1));                 \
    case 2: return reinterpret_cast<const void *>(&KERNEL(2));                 \
    case 4: return reinterpret_cast<const void *>(&KERNEL(4));                 \
    case 8: return reinterpret_cast<const void *>(&KERNEL(8));                 \
    default: return reinterpret_cast<const void *>(&KERNEL(16));               \
    }
#define QG_MMA1(bp) mma_gemv_kernel<bp, 1>
#define QG_MMA2(bp) mma_gemv_kernel<bp, 2>
#define QG_MMA5K1(bp) mma_gemv_kernel<bp, 1, kFmtQ5_K>
#define QG_MMA5K2(bp) mma_gemv_kernel<bp, 2, kFmtQ5_K>
#define QG_MMA6K1(bp) mma_gemv_kernel<bp, 1, kFmtQ6_K>
#define QG_MMA6K2(bp) mma_gemv_kernel<bp, 2, kFmtQ6_K>
#define QG_MMAIQ1(bp) mma_gemv_kernel<bp, 1, kFmtIQ4_XS>
#define QG_MMAIQ2(bp) mma_gemv_kernel<bp, 2, kFmtIQ4_XS>
#define QG_MMAQ81(bp) mma_gemv_kernel<bp, 1, kFmtQ8_0>
#define QG_MMAQ82(bp) mma_gemv_kernel<bp, 2, kFmtQ8_0>
#define QG_ROWS_Q4K1(bp) rows_gemv_kernel<kFmtQ4_K, bp, 1>
#define QG_ROWS_Q4K2(bp) rows_gemv_kernel<kFmtQ4_K, bp, 2>
#define QG_ROWS_Q801(bp) rows_gemv_kernel<kFmtQ8_0, bp, 1>
#define QG_ROWS_Q802(bp) rows_gemv_kernel<kFmtQ8_0, bp, 2>
#define QG_ROWS_Q5K1(bp) rows_gemv_kernel<kFmtQ5_K, bp, 1>
#define QG_ROWS_Q5K2(bp) rows_gemv_kernel<kFmtQ5_K, bp, 2>
#define QG_ROWS_Q6K1(bp) rows_gemv_kernel<kFmtQ6_K, bp, 1>
#define QG_ROWS_Q6K2(bp) rows_gemv_kernel<kFmtQ6_K, bp, 2>
#define QG_ROWS_IQ41(bp) rows_gemv_kernel<kFmtIQ4_XS, bp, 1>
#define QG_ROWS_IQ42(bp) rows_gemv_kernel<kFmtIQ4_XS, bp, 2>
    if (tensor && fmt == kFmtQ5_K) {
        if (mats == 2) { QG_BP_SWITCH16(QG_MMA5K2) }
        QG_BP_SWITCH16(QG_MMA5K1)
    }
    if (tensor && fmt == kFmtQ6_K) {
        if (mats == 2) { QG_BP_SWITCH16(QG_MMA6K2) }
        QG_BP_SWITCH16(QG_MMA6K1)
    }
    if (tensor && fmt == kFmtIQ4_XS) {
        if (mats == 2) { QG_BP_SWITCH16(QG_MMAIQ2) }
        QG_BP_SWITCH16(QG_MMAIQ1)
    }
    if (tensor && fmt == kFmtQ8_0) {
        if (mats == 2) { QG_BP_SWITCH16(QG_MMAQ82) }
        QG_BP_SWITCH16(QG_MMAQ81)
    }
    if (tensor) {
        if (mats == 2) { QG_BP_SWITCH16(QG_MMA2) }
        QG_BP_SWITCH16(QG_MMA1)
    }
    if (fmt == kFmtQ8_0) {
        if (mats == 2) { QG_BP_SWITCH(QG_ROWS_Q802) }
        QG_BP_SWITCH(QG_ROWS_Q801)
    }
    if (fmt == kFmtQ5_K) {
        if (mats == 2) { QG_BP_SWITCH(QG_ROWS_Q5K2) }
        QG_BP_SWITCH(QG_ROWS_Q5K1)
    }
    if (fmt == kFmtQ6_K) {
        if (mats == 2) { QG_BP_SWITCH(QG_ROWS_Q6K2) }
        QG_BP_SWITCH(QG_ROWS_Q6K1)
    }
    if (fmt == kFmtIQ4_XS) {
        if (mats == 2) { QG_BP_SWITCH(QG_ROWS_IQ42) }
        QG_BP_SWITCH(QG_ROWS_IQ41)
    }
    if (mats == 2) { QG_BP_SWITCH(QG_ROWS_Q4K2) }
    QG_BP_SWITCH(QG_ROWS_Q4K1)
#undef QG_ROWS_IQ42
#undef QG_ROWS_IQ41
#undef QG_ROWS_Q6K2
#undef QG_ROWS_Q6K1
#undef QG_ROWS_Q5K2
#undef QG_ROWS_Q5K1
#undef QG_ROWS_Q802
#undef QG_ROWS_Q801
#undef QG_ROWS_Q4K2
#undef QG_ROWS_Q4K1
#undef QG_MMAQ82
#undef QG_MMAQ81
#undef QG_MMAIQ2
#undef QG_MMAIQ1
#undef QG_MMA6K2
#undef QG_MMA6K1
#undef QG_MMA5K2
#undef QG_MMA5K1
#undef QG_MMA2
#undef QG_MMA1
#undef QG_BP_SWITCH16
#undef QG_BP_SWITCH
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link needed).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// 2-D view of W for the TMA: N rows of K/256 units in u32 elements; a box is 32 rows x one unit
// (IQ4_XS: x 144 bytes, the 16-byte aligned window around a 136-byte unit; its rows must be
// 16-byte multiples, an even number of units).
int make_weight_map(const void *W, int fmt, int64_t N, int64_t K, CUtensorMap *map)
{
    auto enc = tensor_map_encoder();
    if (!enc) return QG_ERR_CUDA;
    const int UB = (fmt == kFmtQ4_K)     ? RowsFmt<kFmtQ4_K>::kUnitBytes
                   : (fmt == kFmtQ5_K)   ? RowsFmt<kFmtQ5_K>::kUnitBytes
                   : (fmt == kFmtIQ4_XS) ? RowsFmt<kFmtIQ4_XS>::kUnitBytes
                                         : RowsFmt<kFmtQ8_0>::kUnitBytes;
    const int BB = (fmt == kFmtIQ4_XS) ? RowsFmt<kFmtIQ4_XS>::kWinBytes : UB;  // box bytes of a row
    if (((K / 256) * UB) % 16 != 0) return QG_ERR_SHAPE;
    const cuuint64_t dims[2] = {(cuuint64_t)(K / 256) * UB / 4, (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)(K / 256) * UB};
    const cuuint32_t box[2] = {(cuuint32_t)(BB / 4), 32};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(W), dims, strides,
                           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? QG_OK : QG_ERR_CUDA;
}

// Host work per call is part of a decode step's latency when calls are issued back to back, so
// the two pure functions of a call's shape are cached: the tensor map of a weight tensor (it
// encodes only the address, the format and the shape, so a map stays right for whatever tensor
// later occupies the same address with the same shape) and the launch plan.  Both caches are
// bounded: past kCacheMax entries they start over.
constexpr size_t kCacheMax = 4096;
std::map<std::tuple<const void *, int, int64_t, int64_t>, CUtensorMap> g_maps;

int weight_map_cached(const void *W, int fmt, int64_t N, int64_t K, CUtensorMap *map)
{
    const auto key = std::make_tuple(W, fmt, N, K);
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_maps.find(key);
        if (it != g_maps.end()) {
            *map = it->second;
            return QG_OK;
        }
    }
    const int rc = make_weight_map(W, fmt, N, K, map);
    if (rc != QG_OK) return rc;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_maps.size() >= kCacheMax) g_maps.clear();
    g_maps.emplace(key, *map);
    return QG_OK;
}

// Launch the row-band kernel (+ the split-K second pass when S > 1).  `err` is the device error
// word; `part` holds S*N*B floats when S > 1.
int launch_rows(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x, int B, float *y,
                cudaStream_t st, const DeviceInfo &di, int dev, const RowsPlan &p, int *err,
                unsigned *cnt, float *part, bool pdl, const void *W2 = nullptr, int act = 0,
                const float *res = nullptr)
{
    const void *fn = p.umma ? umma_kernel_ptr(fmt, p.BP, W2 ? 2 : 1) : rows_kernel_ptr(fmt, p.BP, p.tensor, W2 ? 2 : 1);
    int rc = ensure_smem_attr(dev, fn, di.smem_optin);
    if (rc != QG_OK) return rc;
    WeightMaps<2> maps;  // the first map alone is the WeightMaps<1> of a single matrix
    static_assert(offsetof(WeightMaps<2>, m) == 0 && sizeof(WeightMaps<1>) == sizeof(CUtensorMap),
                  "WeightMaps<1> is a prefix of WeightMaps<2>");
    std::memset(&maps, 0, sizeof(maps));
    // units not 16-byte aligned: no tensor map for Q6_K; IQ4_XS rows of an even number of units
    // are 16-byte multiples, and a 144-byte box around each unit is a legal copy
    const bool per_lane = (fmt == kFmtQ6_K) || (fmt == kFmtIQ4_XS && (K / 256) % 2 != 0);
    if (!per_lane) {
        if ((rc = weight_map_cached(W, fmt, N, K, &maps.m[0])) != QG_OK) return rc;
        if (W2 && (rc = weight_map_cached(W2, fmt, N, K, &maps.m[1])) != QG_OK) return rc;
    }
    RowsArgs a;
    const int64_t wbytes = (int64_t)qg_weight_bytes(fmt, N, K);
    a.w[0] = static_cast<const uint8_t *>(W);
    a.w[1] = static_cast<const uint8_t *>(W2 ? W2 : W);
    a.wend = wbytes & ~(int64_t)15;
    a.wtail = (wbytes & 15) ? 1 : 0;
    a.tmap = (fmt == kFmtIQ4_XS && !per_lane) ? 1 : 0;
    a.x = x;
    a.out = (p.S > 1) ? part : y;
    a.y = y;
    a.cnt = cnt;
    a.err = err;
    a.N = N;
    a.B = B;
    a.UPR = (int)(K / 256);
    a.US = p.US;
    a.S = p.S;
    a.Gs = p.Gs;
    a.red_floats = p.red_floats;
    a.act = act;
    a.res = res;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.G);
    cfg.blockDim = dim3(p.NW * 32);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *args[] = {&a, &maps};  // the kernel reads sizeof(WeightMaps<MATS>) bytes of it
    if (cudaLaunchKernelExC(&cfg, fn, args) != cudaSuccess) return QG_ERR_CUDA;
    return QG_OK;
}

int check_common(const void *W, int fmt, int64_t N, int64_t K)
{
    if (fmt != QG_FMT_Q4_K && fmt != QG_FMT_Q5_K && fmt != QG_FMT_Q6_K && fmt != QG_FMT_Q8_0 &&
        fmt != QG_FMT_IQ4_XS)
        return QG_ERR_FMT;
    const int64_t bw = (fmt == QG_FMT_Q8_0) ? 32 : 256;
    if (N < 0 || K < 1 || K % bw != 0) return QG_ERR_SHAPE;
    if (N > 0 && !W) return QG_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(W) % 16 != 0) return QG_ERR_ALIGN;
    return QG_OK;
}

int launch_rowwise(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x, int B, float *y,
                   cudaStream_t st, const DeviceInfo &di)
{
    const int threads = 256;
    const int64_t warps_needed = N;
    const int64_t blocks = std::min<int64_t>((warps_needed + 7) / 8, (int64_t)di.sms * 8);
    const uint8_t *w = static_cast<const uint8_t *>(W);
    switch (fmt) {
    case kFmtQ4_K: rowwise_gemv_kernel<kFmtQ4_K><<<(unsigned)blocks, threads, 0, st>>>(w, N, K, x, B, y); break;
    case kFmtQ5_K: rowwise_gemv_kernel<kFmtQ5_K><<<(unsigned)blocks, threads, 0, st>>>(w, N, K, x, B, y); break;
    case kFmtQ6_K: rowwise_gemv_kernel<kFmtQ6_K><<<(unsigned)blocks, threads, 0, st>>>(w, N, K, x, B, y); break;
    case kFmtIQ4_XS: rowwise_gemv_kernel<kFmtIQ4_XS><<<(unsigned)blocks, threads, 0, st>>>(w, N, K, x, B, y); break;
    default: rowwise_gemv_kernel<kFmtQ8_0><<<(unsigned)blocks, threads, 0, st>>>(w, N, K, x, B, y); break;
    }
    return cudaGetLastError() == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

// Formats with a tensor-core kernel: the K-quants, IQ4_XS with an even number of units per row
// (its rows are then 16-byte multiples, copied in tensor boxes), and Q8_0 with K % 256 == 0 (rows
// of whole 8-block units).
bool has_tensor_kernel(int fmt, int64_t K)
{
    return fmt == QG_FMT_Q4_K || fmt == QG_FMT_Q5_K || fmt == QG_FMT_Q6_K ||
           (fmt == QG_FMT_IQ4_XS && (K / 256) % 2 == 0) || (fmt == QG_FMT_Q8_0 && K % 256 == 0);
}

// The variant qg_gemv takes: the tensor-core kernel where the format has one and B is past the
// measured crossover (the CUDA-core kernel spends one FMA per weight and column, so its cost grows
// with B while the tensor-core kernel's does not), the CUDA-core row kernel otherwise, and the
// generic kernel for rows that are not whole 256-weight units.  Crossover on B200 (17408 x 5120 and
// 5120 x 17408): B = 2 for Q4_K, Q5_K and IQ4_XS (the CUDA-core kernels win only at B = 1); B = 3
// for Q6_K, whose CUDA-core kernel still wins at B = 2 (31.2 vs 34.7 us) and whose tensor-core
// step pays for the per-lane copy windows.
int auto_variant(int fmt, int64_t K, int B)
{
    if (K % 256 != 0) return QG_VARIANT_GENERIC;
    const int tc_min = (fmt == QG_FMT_Q6_K) ? 3 : 2;
    return (has_tensor_kernel(fmt, K) && B >= tc_min) ? QG_VARIANT_TENSOR : QG_VARIANT_FACTORED;
}

// The kernel variant a GEMV call runs (QG_VARIANT_AUTO resolved), or the argument error.
int resolve_variant(int fmt, int64_t K, int B, int variant, int *var_out)
{
    // the streaming kernels need rows of whole 256-weight units (16-byte multiples): always for
    // Q4_K, K % 256 == 0 for Q8_0
    const bool streamable = (K % 256 == 0);
    int var = variant;
    if (var == QG_VARIANT_AUTO) var = auto_variant(fmt, K, B);
    if (var != QG_VARIANT_GENERIC && !streamable) return QG_ERR_VARIANT;
    if (var == QG_VARIANT_TENSOR && !has_tensor_kernel(fmt, K)) return QG_ERR_VARIANT;
    // 9..16 columns: the tensor-core kernels only
    if (B > 8 && !has_tensor_kernel(fmt, K)) return QG_ERR_BATCH;
    if (var == QG_VARIANT_DIRECT && fmt != QG_FMT_Q4_K && fmt != QG_FMT_Q8_0) return QG_ERR_VARIANT;
    if (var == QG_VARIANT_TCGEN05 && fmt != QG_FMT_Q4_K && fmt != QG_FMT_Q5_K) return QG_ERR_VARIANT;
    if (B > 8 && var != QG_VARIANT_TENSOR && var != QG_VARIANT_TCGEN05) return QG_ERR_BATCH;
    *var_out = var;
    return QG_OK;
}

int gemv_impl(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x, int B, float *y,
              void *stream, int variant)
{
    int rc = check_common(W, fmt, N, K);
    if (rc != QG_OK) return rc;
    if (B < 1 || B > kMaxB) return QG_ERR_BATCH;
    if (variant < QG_VARIANT_AUTO || variant > QG_VARIANT_TCGEN05) return QG_ERR_VARIANT;
    if (N == 0) return QG_OK;
    if (!x || !y) return QG_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x) % 2 != 0 || reinterpret_cast<uintptr_t>(y) % 4 != 0)
        return QG_ERR_ALIGN;
    int var = 0;
    if ((rc = resolve_variant(fmt, K, B, variant, &var)) != QG_OK) return rc;
    DeviceInfo di;
    int dev = 0;
    if ((rc = device_info(&di, &dev)) != QG_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    if (var == QG_VARIANT_GENERIC) {
        rc = launch_rowwise(W, fmt, N, K, x, B, y, st, di);
        if (rc == QG_OK) {
            t_last_variant = QG_VARIANT_GENERIC;
            t_last_splits = 1;
        }
        return rc;
    }

    if (var == QG_VARIANT_FACTORED || var == QG_VARIANT_TENSOR || var == QG_VARIANT_TCGEN05) {
        const RowsPlan p = plan_cached(var == QG_VARIANT_TCGEN05 ? 2 : var == QG_VARIANT_TENSOR ? 1 : 0,
                                       fmt, N, K, B, di);
        if (p.smem == 0 || (size_t)di.smem_optin < p.smem) return QG_ERR_SHAPE;
        WsView ws;
        const size_t part_f = (p.S > 1) ? (size_t)p.S * (size_t)N * (size_t)B : 0;
        const size_t ncnt = (p.S > 1) ? (size_t)p.Gs : 0;
        if ((rc = get_workspace(dev, stream, ncnt, 0, part_f, &ws)) != QG_OK) return rc;
        if ((rc = launch_rows(W, fmt, N, K, x, B, y, st, di, dev, p, ws.err, ws.cnt, ws.part, true)) !=
            QG_OK)
            return rc;
        t_last_variant = var;
        t_last_splits = p.S;
        return QG_OK;
    }

    // QG_VARIANT_DIRECT: four lanes per unit, correctly rounded fp32 weights
    const int kvar = kVarDirect;
    const Plan p = make_plan(fmt, kvar, N, K, B, di);
    const void *fn = stream_kernel_ptr(fmt, p.BP, kvar);
    if ((size_t)di.smem_optin < p.smem) return QG_ERR_SHAPE;
    if ((rc = ensure_smem_attr(dev, fn, di.smem_optin)) != QG_OK) return rc;
    WsView ws;
    const size_t part_f = (p.S > 1) ? (size_t)p.S * (size_t)N * (size_t)B : 0;
    if ((rc = get_workspace(dev, stream, (size_t)p.G * kWarps, (size_t)p.G * kWarps * 2 * 8, part_f,
                            &ws)) != QG_OK)
        return rc;

    StreamArgs a;
    a.W = static_cast<const uint8_t *>(W);
    a.x = x;
    a.out = (p.S > 1) ? ws.part : y;
    a.slots = ws.slots;
    a.cnt = ws.cnt;
    a.err = ws.err;
    a.N = N;
    a.B = B;
    a.UPR = (int)(K / 256);
    a.US = p.US;
    a.S = p.S;
    a.Gs = p.Gs;
    a.xs_floats = p.xs_floats;
    // Programmatic dependent launch: the kernel prefetches weights, then waits for the previous
    // kernel on the stream (griddepcontrol.wait) before it reads x or writes y / the workspace.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.G);
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *args[] = {&a};
    if (cudaLaunchKernelExC(&cfg, fn, args) != cudaSuccess) return QG_ERR_CUDA;
    if (p.S > 1) {
        const int64_t NB = N * B;
        const int64_t blocks = std::min<int64_t>((NB + 255) / 256, (int64_t)di.sms * 4);
        splitk_sum_kernel<<<(unsigned)blocks, 256, 0, st>>>(ws.part, y, NB, p.S);
        if (cudaGetLastError() != cudaSuccess) return QG_ERR_CUDA;
    }
    t_last_variant = var;
    t_last_splits = p.S;
    return QG_OK;
}

// The FFN gate/up pair on one x, h = silu(Wg x) * (Wu x): the streaming kernels with both
// matrices in one launch (x staged once, the two rows of h's entry meet in shared memory).
int gate_up_impl(const void *Wg, const void *Wu, int fmt, int64_t N, int64_t K, const uint16_t *x,
                 int B, float *h, void *stream)
{
    int rc = check_common(Wg, fmt, N, K);
    if (rc != QG_OK) return rc;
    if ((rc = check_common(Wu, fmt, N, K)) != QG_OK) return rc;
    if (B < 1 || B > kMaxB) return QG_ERR_BATCH;
    if (N == 0) return QG_OK;
    if (!x || !h) return QG_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x) % 2 != 0 || reinterpret_cast<uintptr_t>(h) % 4 != 0)
        return QG_ERR_ALIGN;
    if (K % 256 != 0) return QG_ERR_SHAPE;  // rows of whole 256-weight units only
    const int var = auto_variant(fmt, K, B);
    // 9..16 columns: the tensor-core kernel; the Q6_K pair's partial rows and copy windows leave
    // no room for them
    if (B > 8 && (var != QG_VARIANT_TENSOR || fmt == QG_FMT_Q6_K)) return QG_ERR_BATCH;
    DeviceInfo di;
    int dev = 0;
    if ((rc = device_info(&di, &dev)) != QG_OK) return rc;
    const RowsPlan p = plan_cached(var == QG_VARIANT_TENSOR ? 1 : 0, fmt, N, K, B, di, 2);
    if (p.smem == 0 || (size_t)di.smem_optin < p.smem) return QG_ERR_SHAPE;
    WsView ws;
    const size_t part_f = (p.S > 1) ? (size_t)p.S * 2 * (size_t)N * (size_t)B : 0;
    const size_t ncnt = (p.S > 1) ? (size_t)p.Gs : 0;
    if ((rc = get_workspace(dev, stream, ncnt, 0, part_f, &ws)) != QG_OK) return rc;
    if ((rc = launch_rows(Wg, fmt, N, K, x, B, h, static_cast<cudaStream_t>(stream), di, dev, p, ws.err,
                          ws.cnt, ws.part, true, Wu, 1)) != QG_OK)
        return rc;
    t_last_variant = var;
    t_last_splits = p.S;
    return QG_OK;
}

// y = W x + r with the residual add in the streaming kernels' epilogue.
int residual_impl(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x, int B,
                  const float *r, float *y, void *stream)
{
    int rc = check_common(W, fmt, N, K);
    if (rc != QG_OK) return rc;
    if (B < 1 || B > kMaxB) return QG_ERR_BATCH;
    if (N == 0) return QG_OK;
    if (!x || !y || !r) return QG_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x) % 2 != 0 || reinterpret_cast<uintptr_t>(y) % 4 != 0 ||
        reinterpret_cast<uintptr_t>(r) % 4 != 0)
        return QG_ERR_ALIGN;
    if (K % 256 != 0) return QG_ERR_SHAPE;  // rows of whole 256-weight units only
    const int var = auto_variant(fmt, K, B);
    if (B > 8 && var != QG_VARIANT_TENSOR) return QG_ERR_BATCH;  // 9..16: the tensor-core kernel only
    DeviceInfo di;
    int dev = 0;
    if ((rc = device_info(&di, &dev)) != QG_OK) return rc;
    const RowsPlan p = plan_cached(var == QG_VARIANT_TENSOR ? 1 : 0, fmt, N, K, B, di);
    if (p.smem == 0 || (size_t)di.smem_optin < p.smem) return QG_ERR_SHAPE;
    WsView ws;
    const size_t part_f = (p.S > 1) ? (size_t)p.S * (size_t)N * (size_t)B : 0;
    const size_t ncnt = (p.S > 1) ? (size_t)p.Gs : 0;
    if ((rc = get_workspace(dev, stream, ncnt, 0, part_f, &ws)) != QG_OK) return rc;
    if ((rc = launch_rows(W, fmt, N, K, x, B, y, static_cast<cudaStream_t>(stream), di, dev, p, ws.err,
                          ws.cnt, ws.part, true, nullptr, 0, r)) != QG_OK)
        return rc;
    t_last_variant = var;
    t_last_splits = p.S;
    return QG_OK;
}

// The device address of page-locked host memory (registered or allocated with the CUDA
// runtime), or nullptr for pageable memory.
void *device_view_of_host(const void *p)
{
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        (void)cudaGetLastError();  // an unknown pointer: clear the error, treat it as pageable
        return nullptr;
    }
    if (at.type != cudaMemoryTypeHost || at.devicePointer == nullptr) return nullptr;
    return at.devicePointer;
}

// Device scratch for x and y of qg_gemv_host: one pair per (device, stream), grown on demand.
struct IoBuf {
    void *x = nullptr, *y = nullptr;
    size_t xb = 0, yb = 0;
};
std::map<std::pair<int, void *>, IoBuf> g_io;

int get_iobuf(int dev, void *stream, size_t xb, size_t yb, IoBuf *out)
{
    std::lock_guard<std::mutex> lk(g_mu);
    IoBuf &b = g_io[{dev, stream}];
    if (b.xb >= xb && b.yb >= yb && b.x && b.y) {
        *out = b;
        return QG_OK;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(static_cast<cudaStream_t>(stream), &cap) != cudaSuccess)
        return QG_ERR_CUDA;
    if (cap != cudaStreamCaptureStatusNone) return QG_ERR_NOMEM;  // cannot grow while capturing
    if (b.x || b.y) {
        // queued work on this stream may still use the old buffers
        if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QG_ERR_CUDA;
        cudaFree(b.x);
        cudaFree(b.y);
    }
    const size_t nx = std::max(xb, b.xb), ny = std::max(yb, b.yb);
    b = IoBuf();
    void *px = nullptr, *py = nullptr;
    if (cudaMalloc(&px, nx) != cudaSuccess) return QG_ERR_NOMEM;
    if (cudaMalloc(&py, ny) != cudaSuccess) {
        cudaFree(px);
        return QG_ERR_NOMEM;
    }
    b.x = px;
    b.y = py;
    b.xb = nx;
    b.yb = ny;
    *out = b;
    return QG_OK;
}

}  // namespace

extern "C" {

int qg_gemv_host(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x_host, int B,
                 float *y_host, void *stream)
{
    int rc = check_common(W, fmt, N, K);
    if (rc != QG_OK) return rc;
    if (B < 1 || B > kMaxB) return QG_ERR_BATCH;
    // 9..16 columns run on the tensor-core kernels only (rows of whole 256-weight units)
    if (B > 8 && (!has_tensor_kernel(fmt, K) || K % 256 != 0)) return QG_ERR_BATCH;
    if (N == 0) return QG_OK;
    if (!x_host || !y_host) return QG_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x_host) % 2 != 0 || reinterpret_cast<uintptr_t>(y_host) % 4 != 0)
        return QG_ERR_ALIGN;
    DeviceInfo di;
    int dev = 0;
    if ((rc = device_info(&di, &dev)) != QG_OK) return rc;
    const size_t xb = (size_t)K * (size_t)B * sizeof(uint16_t), yb = (size_t)N * (size_t)B * sizeof(float);
    IoBuf io;
    if ((rc = get_iobuf(dev, stream, xb, yb, &io)) != QG_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    // Page-locked host memory is readable and writable from the device: x is then read by a
    // small kernel chained to the GEMV (no separate copy operation on the stream) and y is
    // written by the GEMV straight into y_host.  Pageable memory takes stream copies.
    const void *xdev_host = device_view_of_host(x_host);
    void *ydev_host = device_view_of_host(y_host);
    if (xdev_host) {
        const int64_t n = K * B;
        const int64_t pieces = (n + 7) / 8;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)((pieces + 255) / 256));
        cfg.blockDim = dim3(256);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const uint16_t *src = static_cast<const uint16_t *>(xdev_host);
        uint16_t *dst = static_cast<uint16_t *>(io.x);
        if (cudaLaunchKernelEx(&cfg, host_x_copy_kernel, src, dst, n) != cudaSuccess) return QG_ERR_CUDA;
    } else if (cudaMemcpyAsync(io.x, x_host, xb, cudaMemcpyHostToDevice, st) != cudaSuccess) {
        return QG_ERR_CUDA;
    }
    float *ydst = ydev_host ? static_cast<float *>(ydev_host) : static_cast<float *>(io.y);
    rc = gemv_impl(W, fmt, N, K, static_cast<const uint16_t *>(io.x), B, ydst, stream, QG_VARIANT_AUTO);
    if (rc != QG_OK) return rc;
    if (!ydev_host && cudaMemcpyAsync(y_host, io.y, yb, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return QG_ERR_CUDA;
    return QG_OK;
}

int qg_gemv_residual(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x, int B,
                     const float *r, float *y, void *stream)
{
    return residual_impl(W, fmt, N, K, x, B, r, y, stream);
}

int qg_gemv_gate_up_silu(const void *Wg, const void *Wu, int fmt, int64_t N, int64_t K,
                         const uint16_t *x, int B, float *h, void *stream)
{
    return gate_up_impl(Wg, Wu, fmt, N, K, x, B, h, stream);
}

int qg_gemv(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x, int B, float *y,
            void *stream)
{
    return gemv_impl(W, fmt, N, K, x, B, y, stream, QG_VARIANT_AUTO);
}

int qg_gemv_variant(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x, int B,
                    float *y, void *stream, int variant)
{
    return gemv_impl(W, fmt, N, K, x, B, y, stream, variant);
}

int qg_dequant_f32(const void *W, int fmt, int64_t N, int64_t K, float *out, void *stream)
{
    int rc = check_common(W, fmt, N, K);
    if (rc != QG_OK) return rc;
    if (N == 0) return QG_OK;
    if (!out) return QG_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(out) % 4 != 0) return QG_ERR_ALIGN;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (fmt == QG_FMT_Q4_K) {
        const int64_t nsb = N * (K / 256);
        const int64_t threads = nsb * 4;
        dequant_q4k_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(
            static_cast<const uint8_t *>(W), nsb, out);
    } else if (fmt == QG_FMT_Q5_K || fmt == QG_FMT_Q6_K || fmt == QG_FMT_IQ4_XS) {
        const int64_t nsb = N * (K / 256);
        const int64_t threads = nsb * 16;
        const unsigned grid = (unsigned)((threads + 255) / 256);
        const uint8_t *w = static_cast<const uint8_t *>(W);
        if (fmt == QG_FMT_Q5_K)
            dequant_kq_kernel<kFmtQ5_K><<<grid, 256, 0, st>>>(w, nsb, out);
        else if (fmt == QG_FMT_Q6_K)
            dequant_kq_kernel<kFmtQ6_K><<<grid, 256, 0, st>>>(w, nsb, out);
        else
            dequant_kq_kernel<kFmtIQ4_XS><<<grid, 256, 0, st>>>(w, nsb, out);
    } else {
        const int64_t nblk = N * (K / 32);
        dequant_q8_0_kernel<<<(unsigned)((nblk + 255) / 256), 256, 0, st>>>(
            static_cast<const uint8_t *>(W), nblk, out);
    }
    return cudaGetLastError() == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

int qg_last_variant(void) { return t_last_variant; }

int qg_last_splits(void) { return t_last_splits; }

int qg_plan(int fmt, int64_t N, int64_t K, int B, int variant, int mats, int sms, int smem_optin,
            int64_t *out)
{
    if (!out) return QG_ERR_NULL;
    if (fmt != QG_FMT_Q4_K && fmt != QG_FMT_Q5_K && fmt != QG_FMT_Q6_K && fmt != QG_FMT_Q8_0 &&
        fmt != QG_FMT_IQ4_XS)
        return QG_ERR_FMT;
    const int64_t bw = (fmt == QG_FMT_Q8_0) ? 32 : 256;
    if (N < 1 || K < 1 || K % bw != 0 || (mats != 1 && mats != 2)) return QG_ERR_SHAPE;
    if (B < 1 || B > kMaxB) return QG_ERR_BATCH;
    if (variant < QG_VARIANT_AUTO || variant > QG_VARIANT_TCGEN05) return QG_ERR_VARIANT;
    int var = 0, rc = QG_OK;
    if (mats == 2) {
        // the gate/up pair: the variant qg_gemv would take, rows of whole units
        if (variant != QG_VARIANT_AUTO) return QG_ERR_VARIANT;
        if (K % 256 != 0) return QG_ERR_SHAPE;
        var = auto_variant(fmt, K, B);
        if (B > 8 && (var != QG_VARIANT_TENSOR || fmt == QG_FMT_Q6_K)) return QG_ERR_BATCH;
    } else if ((rc = resolve_variant(fmt, K, B, variant, &var)) != QG_OK) {
        return rc;
    }
    DeviceInfo di;
    if (sms > 0 && smem_optin > 0) {
        di.sms = sms;
        di.smem_optin = smem_optin;
    } else {
        int dev = 0;
        if ((rc = device_info(&di, &dev)) != QG_OK) return rc;
    }
    if (var == QG_VARIANT_GENERIC) {
        const int64_t blocks = std::min<int64_t>((N + 7) / 8, (int64_t)di.sms * 8);
        const int64_t o[6] = {var, 1, K / bw, blocks, 8, 0};
        std::memcpy(out, o, sizeof(o));
        return QG_OK;
    }
    if (var == QG_VARIANT_DIRECT) {
        const Plan p = make_plan(fmt, kVarDirect, N, K, B, di);
        if ((size_t)di.smem_optin < p.smem) return QG_ERR_SHAPE;
        const int64_t o[6] = {var, p.S, p.US, p.G, kWarps, (int64_t)p.smem};
        std::memcpy(out, o, sizeof(o));
        return QG_OK;
    }
    const RowsPlan p = (var == QG_VARIANT_TCGEN05) ? make_umma_plan(fmt, N, K, B, di, mats)
                                                   : make_rows_plan(fmt, N, K, B, di, var == QG_VARIANT_TENSOR, mats);
    if (p.smem == 0 || (size_t)di.smem_optin < p.smem) return QG_ERR_SHAPE;
    const int64_t o[6] = {var, p.S, p.US, p.G, p.NW, (int64_t)p.smem};
    std::memcpy(out, o, sizeof(o));
    return QG_OK;
}

int qg_device_error(void *stream, int *flag)
{
    if (!flag) return QG_ERR_NULL;
    *flag = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QG_ERR_CUDA;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    Workspace w;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_ws.find({dev, stream});
        if (it == g_ws.end()) return QG_OK;
        w = it->second;
    }
    if (cudaStreamSynchronize(st) != cudaSuccess) return QG_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, w.base, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return QG_ERR_CUDA;
    if (v != 0) {
        // a warp that gave up left its rows unfinished: clear the error word and the counters
        if (cudaMemset(w.base, 0, 256 + w.nw * sizeof(unsigned)) != cudaSuccess) return QG_ERR_CUDA;
    }
    *flag = v;
    return QG_OK;
}

int qg_hbm_copy(const void *src, void *dst, size_t bytes, void *stream)
{
    if (!src || !dst) return QG_ERR_NULL;
    if (bytes % 16 || reinterpret_cast<uintptr_t>(src) % 16 || reinterpret_cast<uintptr_t>(dst) % 16)
        return QG_ERR_ALIGN;
    DeviceInfo di;
    int dev = 0;
    int rc = device_info(&di, &dev);
    if (rc != QG_OK) return rc;
    hbm_copy_kernel<<<di.sms * 4, 512, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), (int64_t)(bytes / 16));
    return cudaGetLastError() == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

int qg_hbm_read(const void *src, size_t bytes, uint32_t *out, void *stream)
{
    if (!src || !out) return QG_ERR_NULL;
    if (bytes % 16 || reinterpret_cast<uintptr_t>(src) % 16) return QG_ERR_ALIGN;
    DeviceInfo di;
    int dev = 0;
    int rc = device_info(&di, &dev);
    if (rc != QG_OK) return rc;
    hbm_read_kernel<<<di.sms * 4, 512, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4 *>(src), (int64_t)(bytes / 16), out);
    return cudaGetLastError() == cudaSuccess ? QG_OK : QG_ERR_CUDA;
}

const char *qg_status_string(int status)
{
    switch (status) {
    case QG_OK: return "ok";
    case QG_ERR_NULL: return "a required pointer is NULL";
    case QG_ERR_FMT: return "unknown format flag";
    case QG_ERR_SHAPE: return "invalid shape (N < 0, K < 1 or K not a multiple of the block size)";
    case QG_ERR_BATCH: return "B must be in 1..8 (1..16 for Q4_K, Q5_K, Q6_K with K % 256 == 0)";
    case QG_ERR_ALIGN: return "misaligned pointer (W 16 B, x 2 B, y 4 B)";
    case QG_ERR_CUDA: return "CUDA runtime error";
    case QG_ERR_NOMEM: return "workspace allocation failed";
    case QG_ERR_RANGE: return "packer field out of range";
    case QG_ERR_VARIANT: return "kernel variant not available for this format/shape";
    case QG_ERR_SCRATCH: return "call needs more scratch than the fixed no-allocation array holds";
    default: return "unknown status";
    }
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Allocation-free entry point.  Some callers cannot let a library call cudaMalloc: a host
// framework or plugin interface that owns every device allocation through its own pool, or a
// decode loop that cannot afford the device-wide synchronization cudaMalloc may cause.
// qg_gemv_noalloc runs the same streaming kernel with its scratch (error word, arrival counters,
// split-K partial rows) in the fixed file-scope device array below instead of a cudaMalloc'd
// workspace.
// ---------------------------------------------------------------------------------------------
namespace {

// Every GPU that loads this library holds this array until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[QG_NOALLOC_SCRATCH_BYTES];

std::map<int, uint8_t *> g_noalloc_base;  // device address of the array, per device

// The array's name is only a host-side stand-in in host code: its device address is looked up
// once per device (with that device current) and cached.
int noalloc_scratch(int dev, uint8_t **out)
{
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_noalloc_base.find(dev);
    if (it != g_noalloc_base.end()) {
        *out = it->second;
        return QG_OK;
    }
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
        return QG_ERR_CUDA;
    g_noalloc_base.emplace(dev, static_cast<uint8_t *>(p));
    *out = static_cast<uint8_t *>(p);
    return QG_OK;
}

}  // namespace

// band counters reserved at the start of the fixed scratch array (a band per CTA of a slice, at
// most one per SM)
constexpr size_t kNoallocCounters = 1024;

extern "C" int qg_gemv_noalloc(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x,
                               int B, float *y, void *stream)
{
    int rc = check_common(W, fmt, N, K);
    if (rc != QG_OK) return rc;
    if (B < 1 || B > kMaxB) return QG_ERR_BATCH;
    if (N == 0) return QG_OK;
    if (!x || !y) return QG_ERR_NULL;
    if (reinterpret_cast<uintptr_t>(x) % 2 != 0 || reinterpret_cast<uintptr_t>(y) % 4 != 0)
        return QG_ERR_ALIGN;
    const int var = auto_variant(fmt, K, B);
    if (B > 8 && var != QG_VARIANT_TENSOR) return QG_ERR_BATCH;  // 9..16: the tensor-core kernel only
    DeviceInfo di;
    int dev = 0;
    if ((rc = device_info(&di, &dev)) != QG_OK) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (var == QG_VARIANT_GENERIC) {  // no scratch
        rc = launch_rowwise(W, fmt, N, K, x, B, y, st, di);
        if (rc == QG_OK) {
            t_last_variant = QG_VARIANT_GENERIC;
            t_last_splits = 1;
        }
        return rc;
    }

    const RowsPlan p = plan_cached(var == QG_VARIANT_TENSOR ? 1 : 0, fmt, N, K, B, di);
    if (p.smem == 0 || (size_t)di.smem_optin < p.smem) return QG_ERR_SHAPE;
    const size_t part_f = (p.S > 1) ? (size_t)p.S * (size_t)N * (size_t)B : 0;
    // one fixed layout for every call: the error word, kNoallocCounters band counters, then the
    // partial rows
    const size_t ncnt = kNoallocCounters;
    if ((size_t)p.Gs > kNoallocCounters) return QG_ERR_SCRATCH;
    if (ws_bytes_for(ncnt, 0, part_f) > QG_NOALLOC_SCRATCH_BYTES) return QG_ERR_SCRATCH;
    uint8_t *base = nullptr;
    if ((rc = noalloc_scratch(dev, &base)) != QG_OK) return rc;
    Workspace w;
    w.base = base;
    w.bytes = QG_NOALLOC_SCRATCH_BYTES;
    w.nw = ncnt;
    const WsView ws = ws_view(w);
    // Every element of the split-K partial rows is written before it is read, and the kernel
    // returns every band counter to zero (the array starts zeroed), so nothing has to be cleared
    // between calls.
    if ((rc = launch_rows(W, fmt, N, K, x, B, y, st, di, dev, p, ws.err, ws.cnt, ws.part, false)) !=
        QG_OK)
        return rc;
    t_last_variant = var;
    t_last_splits = p.S;
    return QG_OK;
}

// The fixed array's error word (and, after a timeout, its band counters): read with plain copies
// to and from the array's cached device address, so this allocates nothing either.
extern "C" int qg_noalloc_device_error(void *stream, int *flag)
{
    if (!flag) return QG_ERR_NULL;
    *flag = 0;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return QG_ERR_CUDA;
    uint8_t *base = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = g_noalloc_base.find(dev);
        if (it == g_noalloc_base.end()) return QG_OK;  // no call on this device yet
        base = it->second;
    }
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return QG_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, base, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return QG_ERR_CUDA;
    if (v != 0) {
        // a warp that gave up left its band unfinished: clear the error word and the counters
        if (cudaMemset(base, 0, ws_bytes_for(kNoallocCounters, 0, 0) - 256) != cudaSuccess)
            return QG_ERR_CUDA;
    }
    *flag = v;
    return QG_OK;
}
