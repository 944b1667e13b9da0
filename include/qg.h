/*
 * qg.h -- C ABI of libqg, a B200 (sm_100a) dequant GEMV over GGML block-quantized weights:
 *
 *     y[N,B] = dequant(W[N,K]) . x[K,B]      x fp16, accumulation fp32, y fp32, 1 <= B <= 16
 *
 * The operation is the mixed-quant GEMV of "HARDWARE GROUND TRUTH: 2x NVIDIA Tesla T4 (Kaggle)"
 * (second prompt, section "SPEC": y = dequant(W[N,K]) @ x[K], the format chosen by a tensor-type
 * flag passed to the kernel; section "HARD CONSTRAINTS": x broadcast through shared memory, wide
 * coalesced weight loads).  The Q4_K superblock and its dequantization w = d*(sc*q) - dmin*m are
 * from the same dossier's "QUANTIZATION MIX"; "PHYSICS & CONTRACT" fixes fp32 accumulation and
 * that each weight byte is read from DRAM at most once per token, which is what makes a batch of
 * B <= 8 columns (speculative / MTP verify) share one pass over W.  The pages' fp16 y is replaced
 * by fp32 y.
 *
 * Formats (GGML layouts; the pages name them but do not spell them out):
 *   QG_FMT_Q4_K: 256 weights in 144 bytes {fp16 d; fp16 dmin; u8 scales[12]; u8 qs[128]},
 *                w = d*sc_j*q - dmin*m_j with 6-bit (sc_j, m_j) of sub-block j = i/32 packed in
 *                scales[12] (get_scale_min_k4 layout) and q the 4-bit nibble of weight i:
 *                byte qs[32*(i/64) + i%32], low nibble if i%64 < 32 else high nibble.
 *   QG_FMT_Q5_K: 256 weights in 176 bytes {fp16 d; fp16 dmin; u8 scales[12]; u8 qh[32];
 *                u8 qs[128]}: the Q4_K superblock with a fifth bit per weight.  q in 0..31 is the
 *                Q4_K nibble plus 16 * (bit 2*(i/64) + (i%64 >= 32) of qh[i%32]);
 *                w = d*sc_j*q - dmin*m_j as Q4_K.
 *   QG_FMT_Q6_K: 256 weights in 210 bytes {u8 ql[128]; u8 qh[64]; i8 scales[16]; fp16 d}.  In half
 *                h = i/128, with r = i%128, t = r/32 and l = r%32, the low four bits of q are
 *                ql[64h + l + 32*(t%2)] (low nibble for t < 2, high nibble for t >= 2), the high two
 *                bits are bits 2t, 2t+1 of qh[32h + l]; w = d*scales[i/16]*(q - 32), q in 0..63.
 *                (The T4 dossier's "QUANTIZATION MIX" lists Q5_K and Q6_K next to Q4_K.)
 *   QG_FMT_Q8_0: 32 weights in 34 bytes {fp16 d; i8 qs[32]}, w = d*q.
 *   QG_FMT_IQ4_XS: 256 weights in 136 bytes {fp16 d; u16 scales_h; u8 scales_l[4]; u8 qs[128]}
 *                (named by the same dossier's second prompt, "SPEC").  Sub-block j = i/32 has the
 *                6-bit scale ls_j = nibble (j%2) of scales_l[j/2] + 16 * bits 2j..2j+1 of
 *                scales_h; weight i's 4-bit index is the low (r < 16) or high (r >= 16) nibble of
 *                qs[16j + r%16], r = i%32; w = d*(ls_j - 32)*level[index] with the format's
 *                non-linear levels {-127,-104,-83,-65,-49,-35,-22,-10,1,13,25,38,53,69,89,113}.
 *   The flag values are GGML's type ids.
 *
 * Layouts: W row-major, row n = K/256 consecutive superblocks (K-quants) or K/32 consecutive
 * blocks (Q8_0); x[k*B + b] (fp16 bits); y[n*B + b] (fp32).  A caller holding activations [B][K] passes
 * their transpose.
 *
 * Ownership: every pointer is the caller's; the library never frees caller memory.  The library
 * owns one small workspace per (device, stream handle) for split rows (partial sums, arrival
 * counters, an error word), allocated with cudaMalloc the first time a stream needs one of that
 * size and kept until process exit: it is not released when the stream is destroyed, and a new
 * stream that happens to get a destroyed stream's handle reuses that workspace (safe, since the
 * calls on one stream are ordered).  qg_gemv_host's x/y scratch follows the same rule.  Make the
 * first call on a stream outside CUDA-graph capture.
 *
 * Errors: every call returns a qg_status.  Argument errors are found on the host before anything
 * is enqueued.  Launch errors return QG_ERR_CUDA.  Faults of the asynchronous work surface at the
 * caller's next synchronization.  Device-side timeouts (a copy that never lands) are recorded in
 * the stream's error word, read with qg_device_error().  The library never aborts or prints.
 *
 * Determinism: for fixed inputs, device and library build, y is bitwise identical run to run
 * (every reduction, including across thread blocks, sums in a fixed order).
 *
 * Thread safety: calls on different streams may run concurrently.  Calls on one stream are
 * ordered by the stream.
 */
#ifndef QG_H
#define QG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Block formats (GGML type ids). */
enum { QG_FMT_Q8_0 = 8, QG_FMT_Q4_K = 12, QG_FMT_Q5_K = 13, QG_FMT_Q6_K = 14, QG_FMT_IQ4_XS = 23 };

/* Status codes. */
enum {
    QG_OK = 0,
    QG_ERR_NULL = 1,    /* a required pointer is NULL */
    QG_ERR_FMT = 2,     /* unknown format flag */
    QG_ERR_SHAPE = 3,   /* N < 0, K < 1, or K not a multiple of the block size */
    QG_ERR_BATCH = 4,   /* B outside 1..8 (1..16 for Q4_K, Q5_K, Q6_K and Q8_0 with K % 256 == 0,
                           and IQ4_XS with an even K / 256) */
    QG_ERR_ALIGN = 5,   /* W not 16-byte aligned, x not 2-byte aligned or y not 4-byte aligned */
    QG_ERR_CUDA = 6,    /* a CUDA runtime call failed (device query, launch, copy) */
    QG_ERR_NOMEM = 7,   /* the workspace could not be allocated */
    QG_ERR_RANGE = 8,   /* a packer field is out of range (sc, m > 63; q above 15 / 31 / 63 / 15
                           for Q4_K / Q5_K / Q6_K / IQ4_XS; Q8_0 q = -128) */
    QG_ERR_VARIANT = 9, /* unknown kernel variant, or a variant that does not take this format */
    QG_ERR_SCRATCH = 10 /* qg_gemv_noalloc: the call needs more scratch than its fixed array holds */
};

/* Kernel variants of the GEMV (qg_gemv_variant).  QG_VARIANT_AUTO is what qg_gemv uses: when
 * K % 256 == 0, TENSOR with B >= 2 for Q4_K, Q5_K, Q8_0 and IQ4_XS with an even K / 256, and with
 * B >= 3 for Q6_K, FACTORED otherwise; GENERIC when K % 256 != 0. */
enum {
    QG_VARIANT_AUTO = 0,
    /* Each weight is dequantized to the correctly rounded fp32 w = RN(d*sc*q - dmin*m) (Q4_K; the
     * dump's value) or w = d*q (Q8_0) and multiplied by x: the error is bounded relative to
     * sum|w*x| for any input.  Four lanes per 256-weight unit; slower.  Q4_K and Q8_0 only. */
    QG_VARIANT_DIRECT = 1,
    /* One lane per row.  Q4_K and Q5_K: the scale and min are applied per 32-weight sub-block,
     * y = sum_j (d*sc_j)*sum(q*x) - (dmin*m_j)*sum(x), with every q*x product exact; the error is
     * bounded relative to sum(|d*sc*q*x| + |dmin*m*x|), which exceeds sum|w*x| only when
     * d*sc*q and dmin*m nearly cancel.  Q6_K: per 16-weight group,
     * y = sum_t (d*sc_t)*(sum(q*x) - 32*sum(x)), the same kind of bound with 32*|d*sc*x| in place
     * of |dmin*m*x|.  Q8_0: the block scale d is applied per 32 weights (error relative to
     * sum|w*x|).  IQ4_XS: per 32-weight sub-block, y = sum_j d*(ls_j - 32)*(sum(u*x) - 128*sum(x))
     * with u = level + 128 (1..241), the same kind of bound with (|level| + 128)*|x| in place of
     * |level*x|.  Requires K % 256 == 0. */
    QG_VARIANT_FACTORED = 2,
    /* Any format and shape: one warp per row, plain loads, no shared-memory staging.  Used by
     * AUTO for Q8_0 tensors whose rows are not 16-byte multiples (K % 256 != 0).  IQ4_XS weights
     * are exact in fp32, so FACTORED's offset form (see below) and GENERIC differ only in their
     * summation. */
    QG_VARIANT_GENERIC = 3,
    /* The K-quants (Q4_K, Q5_K, Q6_K), Q8_0, and IQ4_XS with an even K / 256: the FACTORED
     * arithmetic with the code*x products on the tensor cores (mma.sync m16n8k16, f16 operands,
     * fp32 accumulation; the 8 columns of the instruction are the B columns of x), so B = 1..8
     * cost the same (up to 16 columns as two 8-column tiles).  The codes (IQ4_XS: the codebook
     * levels; Q8_0: the int8 values) enter the MMA as exact normal fp16 numbers (or zero), so every
     * product is exact.  Same error bound as FACTORED (Q8_0: relative to sum |w*x|).  Requires
     * K % 256 == 0; QG_ERR_VARIANT for IQ4_XS with an odd K / 256. */
    QG_VARIANT_TENSOR = 4,
    /* Q4_K and Q5_K: the FACTORED arithmetic with the q*x sums on the fifth-generation tensor
     * cores (tcgen05.mma kind::f16: the unpacked codes as the A operand in tensor memory, x as the
     * B operand in shared memory, fp32 accumulators in tensor memory, one accumulator column per
     * 32-weight sub-block), B = 1..16 for both formats.  Same error bound as FACTORED.  Requires
     * K % 256 == 0. */
    QG_VARIANT_TCGEN05 = 5
};

/* Bytes of an N x K tensor in format fmt; 0 if fmt is unknown, N < 0, K < 1 or K is not a
 * multiple of the block size (256 for the K-quants, 32 for Q8_0). */
size_t qg_weight_bytes(int fmt, int64_t N, int64_t K);

/* y = dequant(W) . x on the device.
 *   W      device, qg_weight_bytes(fmt, N, K) bytes, 16-byte aligned, read only
 *   fmt    QG_FMT_Q4_K, QG_FMT_Q5_K, QG_FMT_Q6_K, QG_FMT_IQ4_XS or QG_FMT_Q8_0
 *   N, K   rows and reduction length; N >= 0 (N == 0 does nothing); K >= 1, K % block == 0
 *   x      device, fp16 bits [K][B], 2-byte aligned, read only
 *   B      number of columns: 1..8; 1..16 for Q4_K, Q5_K and Q6_K with K % 256 == 0 (9..16 columns
 *          run on the tensor-core kernel, every weight still read once)
 *   y      device, fp32 [N][B], 4-byte aligned, fully overwritten (not accumulated)
 *   stream a cudaStream_t (NULL = the legacy default stream); the call is asynchronous
 * Returns QG_OK once the work is enqueued. */
int qg_gemv(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x, int B, float *y,
            void *stream);

/* qg_gemv for a caller whose activations live in host memory: enqueues on `stream` the copy of
 * x_host into library-owned device scratch, the GEMV (the default kernel variant) and the copy
 * of y back to y_host, so one call does what a host-side caller would otherwise do in three.
 *   W        device, as for qg_gemv (weights stay resident on the GPU)
 *   x_host   host, fp16 bits [K][B], 2-byte aligned; filled by the host before the call.  With
 *            a pinned buffer it may be read while the kernel queued just before the call on the
 *            stream is still finishing (the copy overlaps that kernel's tail), so x_host must not
 *            be written by device work queued on the stream before the call
 *   y_host   host, fp32 [N][B], 4-byte aligned; valid after the stream has been synchronized
 *   fmt, N, K, B, stream as for qg_gemv.
 * With page-locked (pinned) host buffers nothing is copied by a separate operation: a small
 * kernel reads x_host into the scratch (chained to the GEMV, whose weight prefetch overlaps it)
 * and the GEMV writes y straight into y_host.  Pageable buffers take two stream copies, which the
 * CUDA runtime stages (the call may then block the host).  The scratch (K*B*2 + N*B*4 bytes) is one
 * pair of buffers per (device, stream), allocated on first use and grown when a larger call
 * comes (never during stream capture: QG_ERR_NOMEM then); calls on one stream share it, in
 * stream order.  Errors as qg_gemv; argument errors are found before anything is enqueued. */
int qg_gemv_host(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x_host, int B,
                 float *y_host, void *stream);

/* The FFN gate/up pair on one x, fused with its activation:
 *     h[n,b] = silu(gate[n,b]) * up[n,b],  gate = dequant(Wg) . x,  up = dequant(Wu) . x,
 *     silu(v) = v / (1 + e^-v)
 * as "Qwen3.6 27B Single-B70 Maximum-Speed Requirements And Execution Plan", "Phase 3: Maximum
 * Useful Fusion" names it first among the fusion families (the gate+up projection pair and its
 * SiLU-mul epilogue).  One launch streams both weight tensors, stages x once and writes only h;
 * gate and up never reach HBM.
 *   Wg, Wu   device, two N x K tensors of format fmt (each qg_weight_bytes(fmt, N, K) bytes,
 *            16-byte aligned), read only
 *   x, B     as for qg_gemv; h: device, fp32 [N][B], 4-byte aligned, fully overwritten
 * The products and sums are those of qg_gemv's default kernels for (fmt, B); silu is evaluated in
 * fp32 with expf.  Errors as qg_gemv, plus QG_ERR_SHAPE when K % 256 != 0 (the fused path needs rows
 * of whole 256-weight units); B = 9..16 for Q4_K, Q5_K, Q8_0 and IQ4_XS with an even K / 256 only
 * (QG_ERR_BATCH otherwise). */
int qg_gemv_gate_up_silu(const void *Wg, const void *Wu, int fmt, int64_t N, int64_t K,
                         const uint16_t *x, int B, float *h, void *stream);

/* The output projection with the residual add fused into its epilogue:
 *     y[n,b] = (dequant(W) . x)[n,b] + r[n,b]
 * ("Qwen3.6 27B Single-B70 Maximum-Speed Requirements And Execution Plan", "Phase 3: Maximum
 * Useful Fusion": the output projection plus residual).  r is device fp32 [N][B], 4-byte aligned,
 * read only; it may be y itself (an in-place update of the residual stream: each element is read
 * once, by the thread that then writes it).  Arguments and errors otherwise as qg_gemv, plus
 * QG_ERR_SHAPE when K % 256 != 0.  The sum is the GEMV's fp32 result plus r, rounded once. */
int qg_gemv_residual(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x, int B,
                     const float *r, float *y, void *stream);

/* qg_gemv with an explicit kernel variant (QG_VARIANT_*); QG_ERR_VARIANT for an unknown variant,
 * for DIRECT / FACTORED / TENSOR when K % 256 != 0, for TENSOR with Q8_0, and for DIRECT with
 * Q5_K or Q6_K.  FACTORED and GENERIC take every format. */
int qg_gemv_variant(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x, int B,
                    float *y, void *stream, int variant);

/* Dump mode: out[n*K + k] = the fp32 dequantized weight w[n,k], correctly rounded from its exact
 * value, computed by the same device unpacking code the GEMV uses.
 *   W device as for qg_gemv; out device, fp32 [N][K], 4-byte aligned.  Asynchronous on stream. */
int qg_dequant_f32(const void *W, int fmt, int64_t N, int64_t K, float *out, void *stream);

/* Host-side bit packer (fields -> GGML bytes); it does not choose scales, it only places bits.
 *   Q4_K: d[N*K/256], dmin[N*K/256] fp16 bits; sc[N*K/32], m[N*K/32] 6-bit values (<= 63);
 *         q = uint8 [N*K] values 0..15, weight order.
 *   Q5_K: as Q4_K with q = uint8 [N*K] values 0..31.
 *   Q6_K: d[N*K/256] fp16 bits; sc = the int8 group scales [N*K/16] (two's-complement bytes);
 *         dmin and m are ignored; q = uint8 [N*K] stored values 0..63 (w = d*sc*(q - 32)).
 *   Q8_0: d[N*K/32] fp16 bits; dmin, sc, m are ignored; q = int8 [N*K] in -127..127.
 *   IQ4_XS: d[N*K/256] fp16 bits; sc = the stored 6-bit sub-block scales ls [N*K/32] (<= 63; the
 *         multiplier is ls - 32); dmin and m are ignored; q = uint8 [N*K] codebook indices 0..15.
 *   out   host, qg_weight_bytes(fmt, N, K) bytes.
 * All pointers are host pointers.  QG_ERR_RANGE if a field is out of range (out is then
 * unspecified). */
int qg_pack_reference(int fmt, int64_t N, int64_t K, const uint16_t *d, const uint16_t *dmin,
                      const uint8_t *sc, const uint8_t *m, const void *q, void *out);

/* Kernel variant launched by the last successful qg_gemv / qg_gemv_variant of the calling host
 * thread (a launch witness: QG_VARIANT_DIRECT, _FACTORED, _GENERIC, _TENSOR or _TCGEN05), 0 if none yet. */
int qg_last_variant(void);

/* Number of K slices the last GEMV of the calling thread used (1 = no split-K second pass). */
int qg_last_splits(void);

/* The launch plan a call would use, computed on the host; no GPU work and no allocation.
 * Arguments as qg_gemv_variant's (fmt, N >= 1, K, B, variant), plus:
 *   mats        1 for qg_gemv / qg_gemv_variant / qg_gemv_residual, 2 for qg_gemv_gate_up_silu
 *               (then variant must be QG_VARIANT_AUTO);
 *   sms, smem_optin
 *               the device's multiprocessor count and opt-in shared memory per block in bytes;
 *               if either is <= 0, the current device's (which needs a GPU: QG_ERR_CUDA
 *               without one);
 *   out         host array of 6 int64_t, written on success:
 *               {variant launched (QG_VARIANT_*, AUTO resolved), K slices S, 256-weight units
 *                per slice (K/32 blocks for QG_VARIANT_GENERIC), CTAs launched, warps per CTA,
 *                dynamic shared memory per CTA in bytes}.
 * The slice count of the streaming kernels is the slicing with the least modelled cost in 32-row
 * steps: max(steps of a CTA, warps x steps of its busiest warp), plus a fixed charge for the
 * cross-CTA sum when K is sliced; this call lets a caller or a test see the choice.
 * Returns QG_OK, or the argument error the call itself would return (QG_ERR_FMT, _SHAPE, _BATCH,
 * _VARIANT, _NULL for out == NULL), or QG_ERR_SHAPE if no plan fits the shared memory. */
int qg_plan(int fmt, int64_t N, int64_t K, int B, int variant, int mats, int sms, int smem_optin,
            int64_t *out);

/* Reads and clears the device error word of the workspace that (current device, stream) uses;
 * synchronizes the stream.  *flag = 0 if no device-side timeout happened, else a nonzero code. */
int qg_device_error(void *stream, int *flag);

/* Bandwidth probes (for measurement): dst[i] = src[i] over `bytes` bytes (16-byte multiple,
 * both 16-byte aligned), and a read-only pass that xor-folds `bytes` of src into out[i] for
 * i < 4 * (SM count) (out: device, zero-initialised by the caller, at least 4096 uint32).
 * Asynchronous on stream. */
int qg_hbm_copy(const void *src, void *dst, size_t bytes, void *stream);
int qg_hbm_read(const void *src, size_t bytes, uint32_t *out, void *stream);

/* Size of the fixed device array qg_gemv_noalloc uses as scratch (per GPU, held until exit). */
#define QG_NOALLOC_SCRATCH_BYTES (8u << 20)

/* qg_gemv without any allocation.  The pages have no counterpart of this entry point; it exists
 * for callers that cannot let a library call cudaMalloc: a host framework or plugin interface
 * that owns all device memory through its own pool, or a decode loop that cannot afford the
 * device-wide synchronization an allocation may cause.  The caller passes inputs and outputs
 * exactly as for qg_gemv (same arguments, layouts, preconditions and results, default kernel
 * variant); the kernel's scratch (an error word, one arrival counter per row band when K is
 * split, the split-K partial rows) lives in one file-scope device array of
 * QG_NOALLOC_SCRATCH_BYTES per GPU, which every GPU that loads the library holds until exit.
 *   - No device memory is allocated: no cudaMalloc/cudaFree, no allocating library routine.  The
 *     counters start at zero (the array is zero-initialized) and every call leaves them at zero
 *     again (the last CTA of a band resets its counter); the partial rows are written before they
 *     are read.  So nothing is cleared between calls.  (On the host, the library's caches of
 *     launch plans and weight tensor maps take a few hundred bytes of C++ heap the first time a
 *     shape or a weight address is seen, shared with the other entry points.)
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 *     that device current) and caches it; later calls reuse it.
 *   - Every call on every stream shares the one array: calls that overlap on the GPU race and give
 *     wrong results.  Serialize them (one stream, or events between streams).
 *   - QG_ERR_SCRATCH if the call needs more scratch than the array holds (this happens only when
 *     x for the whole of K does not fit in shared memory and N*B is large: the split-K partial
 *     rows need S*N*B*4 bytes); nothing is enqueued then.
 *   - qg_last_variant / qg_last_splits report its launch like qg_gemv's.
 *   - Device-side copy timeouts go to the array's error word: read them with
 *     qg_noalloc_device_error (qg_device_error reads the allocating entry points' workspaces). */
int qg_gemv_noalloc(const void *W, int fmt, int64_t N, int64_t K, const uint16_t *x, int B,
                    float *y, void *stream);

/* Reads and clears the error word of qg_gemv_noalloc's fixed array on the current device, after
 * synchronizing `stream` (the stream of the calls to check; NULL = the legacy default stream).
 * *flag = 0 if no device-side timeout happened (or no qg_gemv_noalloc call has run on this
 * device), else a nonzero code; a nonzero word also clears the array's band counters.  No
 * counterpart on the pages; it allocates nothing (plain copies to and from the array). */
int qg_noalloc_device_error(void *stream, int *flag);

/* Static text for a status code. */
const char *qg_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* QG_H */
