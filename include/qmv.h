/*
 * qmv.h -- C ABI of libqmv: weight-only block-quantized encoders and fused
 * dequantize-and-matvec kernels for LLM decode on NVIDIA B200 (sm_100a).
 *
 * The operations follow the pages' statement of the problem:
 *   [P1] "Stream D -- Quantization (FP4 + QAT-int4): feasibility, first
 *        result, and plan": sec. 1 (E2M1 / OCP MX FP4 weights, per-block 32
 *        along in-features, e8m0 scale 2^(floor(log2(max_abs)) - 2), two
 *        values per byte; int4/int8/int4km gather formats for routed
 *        experts) and sec. 2 (symmetric int4/int8 with an MSE-optimal clip).
 *   [P2] "Dense-path int4km coverage + flagship Qwen3.6-35B -- session
 *        findings & methods": sec. 1-3 (decode is weight-bandwidth bound; a
 *        fused int4km matvec for lm_head and attention q/o; gather over the
 *        selected experts only) and sec. 8 (FP4 dense matvec: fixed E2M1 grid
 *        times a per-K-block e8m0 scale; per-row 16-entry k-means codebook).
 *   [P3] "coreai-optimization (coreai-opt) reference -- quantization &
 *        palettization": per-block symmetric quantization, 1-D k-means
 *        palettes, fp16 scales, and the pitfall that layers whose dimension
 *        does not divide the block are silently skipped (here: rejected).
 *   [P5] "Compression (palettization & quantization)": "int8 k-means >
 *        whole-model int4" (the recommended recipe, 8-bit k-means with
 *        group 32).
 *
 * Conventions for every call below
 *  - All array pointers are DEVICE pointers owned by the caller, 16-byte
 *    aligned, row-major and densely packed.  Host pointers are marked
 *    "host".  The library keeps no pointer after a call returns and
 *    allocates no device memory in any call.
 *  - `stream` is a cudaStream_t passed as void* (NULL: the legacy default
 *    stream).  Calls only enqueue work on it; they never synchronize, except
 *    qmv_status_fetch.
 *  - Shapes: N output rows (out-features), K in-features with K % 32 == 0
 *    (one quantization block = 32 consecutive in-features of one row).
 *    B is the number of activation rows (decode tokens), 1 <= B <= 16.
 *  - fp16 arrays are IEEE binary16 bit patterns (uint16_t).
 *  - Packed 4-bit codes: element k of a row lives in byte k/2, low nibble
 *    for even k, high nibble for odd k (the little-endian reading of eight
 *    codes per 32-bit word).
 *  - Errors: argument checks run on the host before anything is enqueued
 *    and return QMV_ERR_ARG (null or misaligned pointer, bad format or clip
 *    list), QMV_ERR_SHAPE (N < 1, K < 32, K % 32 != 0, E < 1) or
 *    QMV_ERR_UNSUPPORTED (B or topk outside [1, 16]; for int8km, and for the
 *    int4km part of the mixed format, a shape whose activations do not fit
 *    the kernel's on-chip staging -- the other formats stage such
 *    activations one K-phase at a time); a failed launch returns
 *    QMV_ERR_CUDA.  Bad DATA is found on the device: the kernel sets
 *    a bit of a library-owned device status word (QMV_FLAG_*) and carries
 *    on; qmv_status_fetch reads and clears it.  No kernel traps.
 *  - The library-owned status word is per device; calls that run on several
 *    streams at once share it.
 */
#ifndef QMV_H
#define QMV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QMV_OK = 0,
  QMV_ERR_ARG = -1,
  QMV_ERR_SHAPE = -2,
  QMV_ERR_UNSUPPORTED = -3,
  QMV_ERR_DATA = -4,
  QMV_ERR_CUDA = -5
} qmv_status;

/* Weight formats. */
enum {
  QMV_FMT_FP4 = 0,    /* E2M1 codes + e8m0 scale byte per 32-block      */
  QMV_FMT_INT4 = 1,   /* symmetric int4 (nibble = q + 8) + fp16 scale   */
  QMV_FMT_INT4KM = 2, /* 4-bit index into a per-row 16-entry fp16 LUT   */
  QMV_FMT_INT8 = 3,   /* symmetric int8 (two's complement) + fp16 scale */
  QMV_FMT_INT4AFF = 4, /* affine int4 (q, zero point) + fp16 scale     */
  QMV_FMT_INT8KM = 5   /* 8-bit index into a 256-entry fp16 LUT per 32 rows */
};

/* Device status bits (qmv_status_fetch). */
#define QMV_FLAG_NONFINITE 0x1u      /* encode: a block held Inf/NaN (block written as zeros) */
#define QMV_FLAG_SCALE_OVERFLOW 0x2u /* encode: no clip gave a finite fp16 scale (block zeroed) */
#define QMV_FLAG_BAD_EXPERT 0x4u     /* gather: expert id outside [0, E) (that output row zeroed) */
#define QMV_FLAG_TIMEOUT 0x8u        /* a kernel's bounded wait on its own tensor-core work gave up (that launch's outputs are invalid) */

/* ---------------------------------------------------------------------
 * Encoders (offline conversion; [P1] sec. 1-2).
 * --------------------------------------------------------------------- */

/* FP4 E2M1 encode.  Per row and 32-block: amax = max|w|; e = floor(log2(
 * amax)) - 2 clamped to [-127, 127] (amax == 0 gives -127); scale byte =
 * e + 127; code = sign bit | E2M1 magnitude of |w| * 2^-e rounded to nearest,
 * ties to even, saturating at 6.  A negative weight that rounds to zero keeps
 * its sign (code 8).
 *   W       [N, K] float32 (in)
 *   codes   [N, K/2] uint8 (out, packed as above)
 *   scales  [N, K/32] uint8 e8m0 bytes (out)
 * A block with Inf/NaN: codes 0, scale byte 0, QMV_FLAG_NONFINITE. */
qmv_status qmv_encode_fp4(const float* W, int64_t N, int64_t K, uint8_t* codes,
                          uint8_t* scales, void* stream);

/* Symmetric int4 encode with MSE-searched clip.  Per block, for each clip
 * alpha in list order: s = fp16_rne(float(alpha * amax) / 7); q_i =
 * clamp(rint_even(w_i / s), -7, 7) (0 when s == 0); err = sum over i of
 * (double(w_i) - q_i * double(s))^2 accumulated in order i = 0..31; the first
 * alpha with the strictly smallest err wins.  A clip whose fp16 scale
 * overflows is skipped; a block with none left is zeroed with
 * QMV_FLAG_SCALE_OVERFLOW.
 *   clips   host float32 [n_clips], 1 <= n_clips <= 16 (e.g. 1.00 .. 0.50)
 *   codes   [N, K/2] uint8, nibble = q + 8 (out)
 *   scales  [N, K/32] fp16 (out) */
qmv_status qmv_encode_int4(const float* W, int64_t N, int64_t K, const float* clips,
                           int n_clips, uint8_t* codes, uint16_t* scales, void* stream);

/* Symmetric int8 encode: as qmv_encode_int4 with qmax = 127 and one
 * two's-complement byte per weight.  clips = {1.0f} is plain absmax.
 *   codes   [N, K] int8 (out);  scales [N, K/32] fp16 (out) */
qmv_status qmv_encode_int8(const float* W, int64_t N, int64_t K, const float* clips,
                           int n_clips, int8_t* codes, uint16_t* scales, void* stream);

/* Affine (asymmetric) int4 encode per block of 32 ([P3] "Quantization":
 * asymmetric scheme; "Theoretical size": an fp16 scale and an n_bits zero
 * point per group; [P1] sec. 1: the gather format int4aff).  Per block:
 * range [lo, hi] = [min(min w, 0), max(max w, 0)]; s = fp16_RNE((hi - lo) /
 * 15); z = clamp(rint(-lo / s), 0, 15); q = clamp(rint(w / s) + z, 0, 15),
 * float arithmetic with the stored s; Wdq = s * (q - z).  An all-zero block
 * has s = 0, q = z = 0; an fp16 overflow of s zeroes the block with
 * QMV_FLAG_SCALE_OVERFLOW; Inf/NaN zeroes it with QMV_FLAG_NONFINITE.
 *   codes  [N, K/2] uint8, q nibbles, element 2j in the low nibble (out)
 *   aux    [N, qmv_int4aff_aux_row_bytes(K)] uint8 (out): per row the fp16
 *          scales [K/32], then the zero points two per byte (block 2j in the
 *          low nibble; a last odd block leaves the high nibble 0). */
qmv_status qmv_encode_int4aff(const float* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* aux,
                              void* stream);

/* Bytes of one int4aff aux row: 2 * (K/32) + ceil(K/64). */
int64_t qmv_int4aff_aux_row_bytes(int64_t K);

/* int4km encode: per row a 16-entry fp16 palette by scalar 1-D k-means and
 * the packed 4-bit index of each weight ([P3] "Palettization": scalar
 * k-means, 2^n_bits centroids, per-channel grouping; [P2] sec. 8: per-row
 * 16-entry codebook).  Per row of K weights: sort ascending (-0 before +0);
 * centre k starts at sorted[floor((2k+1) K / 32)]; `iters` Lloyd steps (each
 * weight to the nearest centre by double distance, ties to the lower index;
 * a non-empty centre becomes float(double sum of its members in ascending
 * order / count), an empty one keeps its value); palette = fp16 RNE of the
 * centres; index = nearest palette entry (double distance, ties to the
 * lower index).  A row with Inf/NaN is written as zeros and sets
 * QMV_FLAG_NONFINITE.
 *   W      [N, K] float32 (device)
 *   K      multiple of 32, at most 16384
 *   iters  0 .. 1000 (the workloads use 20)
 *   lut    [N, 16] fp16 (out);  idx [N, K/2] uint8, element 2j in the low nibble (out)
 * Errors: QMV_ERR_ARG (pointers, iters), QMV_ERR_SHAPE (N, K % 32),
 * QMV_ERR_UNSUPPORTED (K > 16384). */
qmv_status qmv_encode_int4km(const float* W, int64_t N, int64_t K, int iters, uint16_t* lut, uint8_t* idx,
                             void* stream);

/* int8km encode: per group of 32 consecutive output rows a 256-entry fp16
 * palette by scalar 1-D k-means and one 8-bit index per weight ([P3]
 * "Palettization": per-grouped-channel LUTs, 2^n_bits centroids; [P5]
 * "int8 k-means > whole-model int4": 8-bit k-means, group size 32).  Per
 * group of n = rows * K weights (a last group of N % 32 rows is fitted on
 * the rows it has) the steps of qmv_encode_int4km with 256 centres: sort
 * ascending (-0 before +0); centre k starts at sorted[floor((2k+1) n / 512)];
 * `iters` Lloyd steps (nearest centre by double distance, ties to the lower
 * index; a non-empty centre becomes float(double sum of its members in
 * ascending order / count), an empty one keeps its value); palette = fp16
 * RNE of the centres; index = nearest palette entry (double distance, ties
 * to the lower index).  A group with Inf/NaN is written as zeros and sets
 * QMV_FLAG_NONFINITE.
 *   W          [N, K] float32 (device)
 *   K          multiple of 32, at most 16384
 *   iters      0 .. 1000 (the workloads use 20)
 *   lut        [ceil(N/32), 256] fp16 (out);  idx [N, K] uint8 (out)
 *   workspace  device buffer of at least qmv_int8km_encode_workspace_bytes
 *              (N, K) bytes, 16-byte aligned (sort scratch, overwritten)
 * Errors: QMV_ERR_ARG (pointers, iters, short workspace), QMV_ERR_SHAPE
 * (N, K % 32), QMV_ERR_UNSUPPORTED (K > 16384). */
qmv_status qmv_encode_int8km(const float* W, int64_t N, int64_t K, int iters, uint16_t* lut, uint8_t* idx,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of the workspace of qmv_encode_int8km: at most 160 groups in
 * flight, next_pow2(min(N, 32) * K) 4-byte keys each. */
int64_t qmv_int8km_encode_workspace_bytes(int64_t N, int64_t K);

/* ---------------------------------------------------------------------
 * Fused dequantize + matvec, y = x Wdq^T with fp32 accumulation
 * ([P2] sec. 1-3, 8).  x: [B, K] fp16; y: [B, N] float32 (overwritten).
 * Block-scaled formats apply the scale to each 32-block's exact partial sum.
 * --------------------------------------------------------------------- */

/* codes [N, K/2] uint8 E2M1; scales [N, K/32] uint8 e8m0. */
qmv_status qmv_matvec_fp4(const uint8_t* codes, const uint8_t* scales, const uint16_t* x,
                          int B, int64_t N, int64_t K, float* y, void* stream);

/* codes [N, K/2] uint8 (q + 8 nibbles); scales [N, K/32] fp16. */
qmv_status qmv_matvec_int4(const uint8_t* codes, const uint16_t* scales, const uint16_t* x,
                           int B, int64_t N, int64_t K, float* y, void* stream);

/* idx [N, K/2] uint8 (4-bit LUT indices); lut [N, 16] fp16 per-row palette. */
qmv_status qmv_matvec_int4km(const uint8_t* idx, const uint16_t* lut, const uint16_t* x,
                             int B, int64_t N, int64_t K, float* y, void* stream);

/* codes [N, K] int8; scales [N, K/32] fp16. */
qmv_status qmv_matvec_int8(const int8_t* codes, const uint16_t* scales, const uint16_t* x,
                           int B, int64_t N, int64_t K, float* y, void* stream);

/* codes [N, K/2] uint8 (q nibbles); aux [N, qmv_int4aff_aux_row_bytes(K)]
 * (fp16 scales, then zero-point nibbles), as qmv_encode_int4aff writes them;
 * y[b, n] = sum_k s(n, k/32) * (q[n, k] - z(n, k/32)) * x[b, k].  aux may
 * have any alignment; with aux 8-byte aligned and K % 512 == 0 the scales
 * and zero points are copied asynchronously, otherwise byte by byte (slower,
 * same result). */
qmv_status qmv_matvec_int4aff(const uint8_t* codes, const uint8_t* aux, const uint16_t* x,
                              int B, int64_t N, int64_t K, float* y, void* stream);

/* int8km matvec ([P3] "Palettization": per-grouped-channel LUTs, 2^n_bits
 * entries; [P5] "int8 k-means > whole-model int4": 8-bit k-means, group 32;
 * [P1] sec. 1: the gather format int8km):
 *   y[b, n] = sum_k x[b, k] * lut[n / 32][idx[n, k]]
 *   idx  [N, K] uint8 (16-byte aligned)
 *   lut  [ceil(N/32), 256] fp16 bits (2-byte aligned); rows 32g..32g+31
 *        share lut[g] (a last group may have fewer rows)
 * Other arguments and errors as qmv_matvec_fp4.  The LUTs come from the
 * caller (a k-means fit; no encoder in this library). */
qmv_status qmv_matvec_int8km(const uint8_t* idx, const uint16_t* lut, const uint16_t* x, int B,
                             int64_t N, int64_t K, float* y, void* stream);

/* ---------------------------------------------------------------------
 * Mixed int4km + int8 outlier columns ("Stream D", next steps: a mixed
 * int4 + int8-outlier matvec extending the int4km linear; the format is
 * the pages' open question, the reading taken here):
 *   the C input columns (C % 32 == 0, 0 <= C < K) with the largest
 *   max_n |W[n, k]| (Inf/NaN the largest; ties to the lower column) are
 *   symmetric int8 with per-block-32 fp16 scales along the outlier columns
 *   (clip 1.0); the other K - C columns, ascending, are an int4km matrix.
 *   y[b, n] = sum_{k main} x[b, k] lut[n][idx] + sum_{k outlier} x[b, k] q s
 * Arrays: cols int32 [C] (ascending), lut fp16 [N, 16], idx uint8
 * [N, (K-C)/2], ocodes int8 [N, C], oscales fp16 [N, C/32].  The encoder's
 * workspace is caller-owned device memory (16-byte aligned).
 * --------------------------------------------------------------------- */

/* Bytes of the workspace of qmv_encode_int4km_o8. */
int64_t qmv_int4km_o8_encode_workspace_bytes(int64_t N, int64_t K, int64_t C);

/* The C outlier columns of W fp32 [N, K] into cols (ascending).
 * workspace: at least 8 * K bytes. */
qmv_status qmv_outlier_columns(const float* W, int64_t N, int64_t K, int64_t C, int32_t* cols,
                               void* workspace, size_t workspace_bytes, void* stream);

/* Encode: the outlier columns (written to cols), the int4km fit of the main
 * columns (qmv_encode_int4km, `iters` Lloyd steps) and the int8 encode of
 * the outlier columns.  K - C <= 16384. */
qmv_status qmv_encode_int4km_o8(const float* W, int64_t N, int64_t K, int64_t C, int iters,
                                int32_t* cols, uint16_t* lut, uint8_t* idx, int8_t* ocodes,
                                uint16_t* oscales, void* workspace, size_t workspace_bytes,
                                void* stream);

/* y fp32 [B, N] for x fp16 [B, K]: the int4km kernel stages the main
 * columns of x and writes y; a second kernel adds the outlier columns
 * (two launches on `stream`, the second a dependent launch).  No
 * workspace. */
qmv_status qmv_matvec_int4km_o8(const uint8_t* idx, const uint16_t* lut, const int8_t* ocodes,
                                const uint16_t* oscales, const int32_t* cols, const uint16_t* x,
                                int B, int64_t N, int64_t K, int64_t C, float* y, void* stream);

/* ---------------------------------------------------------------------
 * Fused matvec + argmax (greedy next token from the lm_head; the pages'
 * fused head+argmax kernel: "coreai-optimization (coreai-opt) reference",
 * sec. "The LM head + embeddings").  For each activation row b computes
 * y[b, :] = x[b, :] Wdq^T exactly as qmv_matvec_* does, without writing y,
 * and returns
 *     idx[b] = the lowest n with y[b, n] = max_n y[b, n]     (int32, device)
 *     val[b] = y[b, idx[b]]                                   (float32, device)
 * Values are ordered as floats with -0 == +0 (a NaN with the sign bit clear
 * ranks above +Inf, one with it set below -Inf).
 *   fmt        QMV_FMT_*; codes / aux as for the format's qmv_matvec_* call.
 *   N          < 2^31.
 *   workspace  device buffer of at least qmv_argmax_workspace_bytes() bytes,
 *              16-byte aligned, zero-filled before its first use; every call
 *              leaves it zero-filled again.  One call at a time per
 *              workspace (calls on other streams need their own).
 * Errors as for qmv_matvec_*; QMV_ERR_ARG also for a short or misaligned
 * workspace or misaligned idx / val. */
qmv_status qmv_matvec_argmax(int fmt, const void* codes, const void* aux, const uint16_t* x, int B,
                             int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                             int32_t* idx, float* val, void* stream);

/* Bytes of workspace qmv_matvec_argmax needs on the current device. */
qmv_status qmv_argmax_workspace_bytes(size_t* bytes);

/* qmv_matvec_argmax with a library-owned scratch instead of a caller
 * workspace: a static device array (zero at load, left zero by every call),
 * located once per device; nothing is allocated.  One call at a time per
 * device (calls on several streams at once need qmv_matvec_argmax with
 * their own workspaces).  QMV_ERR_UNSUPPORTED when the device needs more
 * scratch than the array holds (more than 512 SMs); otherwise arguments and
 * errors as for qmv_matvec_argmax. */
qmv_status qmv_matvec_argmax_static(int fmt, const void* codes, const void* aux, const uint16_t* x, int B,
                                    int64_t N, int64_t K, int32_t* idx, float* val, void* stream);

/* ---------------------------------------------------------------------
 * Routed-expert gather matvec ([P1] sec. 1 gather formats; [P2] sec. 3:
 * only the selected experts' weights are read).  For token b and slot j,
 * e = expert_ids[b*topk + j] and
 *    y[b, j, :] = W_e x_b        (x_per_slot == 0, x [B, K])
 *    y[b, j, :] = W_e x_{b,j}    (x_per_slot == 1, x [B, topk, K]).
 * Each selected expert's weights are streamed once per call for all the
 * (b, j) that chose it.
 *   fmt          QMV_FMT_*; codes_stack / aux_stack are the per-format
 *                arrays of qmv_matvec_* stacked over experts: [E, N, ...]
 *   expert_ids   [B, topk] int32 (device)
 *   y            [B, topk, N] float32 (out)
 * An id outside [0, E) zeroes its output row and sets QMV_FLAG_BAD_EXPERT.
 * The (b, j) pairs that chose one expert are served together, in column
 * groups of up to 16 pairs per pass over that expert's weights. */
qmv_status qmv_gather_matvec(int fmt, const void* codes_stack, const void* aux_stack, int E,
                             int64_t N, int64_t K, const int32_t* expert_ids, int B, int topk,
                             const uint16_t* x, int x_per_slot, float* y, void* stream);

/* ---------------------------------------------------------------------
 * Test support and status
 * --------------------------------------------------------------------- */

/* Dequantize to float32 Wdq [N, K] with the same decode the matvec kernels
 * use (exact: every format's dequantized value is a float32). */
qmv_status qmv_dequant(int fmt, const void* codes, const void* aux, int64_t N, int64_t K,
                       float* Wdq, void* stream);

/* Synchronize `stream`, then read and clear the current device's status
 * word into *flags (host).  Returns QMV_ERR_DATA when any QMV_FLAG_* bit was
 * set, QMV_OK otherwise, QMV_ERR_CUDA if the stream reported an error. */
qmv_status qmv_status_fetch(void* stream, uint32_t* flags);

/* Overlap of consecutive matvec launches.  Every matvec / gather launch
 * lets the next one in its stream become resident during its last blocks
 * (programmatic dependent launch) and waits for the preceding work before
 * it reads activations or expert ids or writes outputs.  With
 * enable = 1, dense matvec launches made afterwards (any stream, any
 * thread) also start streaming their weight codes, scales and palettes
 * BEFORE that wait, so a kernel's pipeline fill hides under its
 * predecessor's tail.  Enable it only when no work still in flight on the
 * stream writes those weights (a decode loop over fixed weights); after an
 * encoder call on the same stream, synchronize or keep it off.  Default 0.
 * Returns QMV_ERR_ARG if enable is not 0 or 1. */
qmv_status qmv_set_weight_prefetch(int enable);

/* fp4 matvecs at 2..16 activation columns on the tcgen05 tensor cores.
 * With mode = 1, dense fp4 matvec launches made afterwards (any stream, any
 * thread) with 2 <= B <= 16, K a multiple of 512 no larger than 4608 (16
 * activation columns and two 16 KB code stages in shared memory), 16-byte
 * aligned codes, scales and x, and neither the fused argmax nor the
 * mixed format's accumulation, run the tensor-memory kernel: 128-row tiles,
 * codes streamed by TMA, each row's E2M1 weights times its block scales
 * decoded exactly to fp16 relative to the row's largest block exponent, the
 * MMA (M = 128, N = 16) accumulating in fp32 ("Dense-path int4km coverage",
 * sec. 8).  Blocks more than 2^36 below the row's largest scale are dropped
 * (their terms lie below fp32's resolution of the result).  Other launches
 * keep the mma.sync kernel.  mode = 0 uses the mma.sync kernel everywhere.
 * A bounded wait inside the kernel that gives up sets QMV_FLAG_TIMEOUT.
 * Returns QMV_ERR_ARG if mode is not 0 or 1. */
qmv_status qmv_set_fp4_tensor_cores(int mode);

/* Text of the last error of this host thread ("" if none). */
const char* qmv_last_error(void);

/* Library version, e.g. "0.1.0". */
const char* qmv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QMV_H */
