// qmv_internal.h -- declarations shared by the libqmv translation units:
// kernel parameter blocks, per-format geometry and the launchers the C ABI
// (qmv_abi.cu) calls after validating its arguments.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "qmv.h"

namespace qmv {

// ---- fused dequant-matvec / gather kernel -----------------------------------
constexpr int kWarps = 8;                  // warps per CTA (16 for one-CTA-per-SM launches)
constexpr int kThreads = 32 * kWarps;
constexpr int kTileRows = 16;              // rows per tile: one m16 step
constexpr int kMaxCols = 16;               // activation columns per pass
#ifndef QMV_STAGES
#define QMV_STAGES 3                       // per-warp ring depth (slices in flight + 1)
#endif
constexpr int kStages = QMV_STAGES;
#ifndef QMV_SLICE_BYTES
#define QMV_SLICE_BYTES 256                // bytes of codes per row in a warp's K-slice
#endif
#ifndef QMV_MIN_CTAS
#define QMV_MIN_CTAS 2                     // CTAs per SM the kernel's register budget targets
#endif
constexpr int kSliceBytes = QMV_SLICE_BYTES;
constexpr int kMinCtas = QMV_MIN_CTAS;
constexpr int kMaxCtasPerSM = 4;
constexpr int kMaxPairs = 256;             // B * topk upper bound (16 * 16)
constexpr int kSmemLimit = 227 * 1024;     // per-block opt-in maximum on sm_100
constexpr int kSmemPerSM = 228 * 1024;     // shared memory of one SM
constexpr int kZeroBytes = 1024;           // zero activations read by the batch-1 form's idle columns
constexpr int kStaticSmem = 5 * 1024;      // the kernel's static shared memory (group table), rounded up

// Aux (scale / palette) staging mode of a launch.
enum AuxMode : int {
  kAuxRows = 0,   // 8-byte asynchronous copies of each row's scale segment (8-byte granular rows)
  kAuxBlock = 1,  // plain byte loads of the slice's scales (any K % 32 == 0)
  kAuxLut = 2     // the tile's 16 x 16 fp16 palette, first chunk only
};

struct MvParams {
  const uint8_t* codes;   // codes of expert 0 (dense: the matrix)
  const uint8_t* aux;     // scales / palette of expert 0
  const uint16_t* x;      // activations, fp16 bits
  float* y;               // outputs
  const int32_t* ids;     // gather: expert ids [B * topk]
  uint32_t* status;       // library device status word
  int64_t N, K;
  int64_t code_row_bytes;  // bytes of codes per weight row
  int64_t aux_row_bytes;   // bytes of scales per row (palette: 32)
  int64_t expert_code_bytes, expert_aux_bytes;
  int64_t tiles;           // ceil(N / 16)
  int B;                   // dense: activation rows; gather: tokens
  int topk, E, x_per_slot, gather;
  int KC, nchunks;         // in-features per warp slice, slices per tile
  int gk;                  // K granule of split units (in-features)
  int min_part;            // split units: the least granules a warp's part of K keeps
  int one;                 // batch-1 block-column form (dense B == 1, K % 256 == 0)
  int off_zero;            // its zero activation region
  int off_xsum;            // its per-block activation sums (int4, int4aff)
  int64_t zplane;          // int4aff: byte offset of the zero points in an aux row
  int zoff;                // int4aff: byte offset of the slice's zero points in a staged aux row
  int off_tab;             // int8km: the replicated LUT table (64 KB, two buffers)
  int off_kmtab;           // int4km: lane palette copies (4 KB per four warps, 4 KB aligned at run time)
  int km_smem;             // int4km: rows g+8 look up their palette copy in shared memory
  int red_bufs;            // int8km: partial-sum buffers (2, or 1 where shared memory is short)
  int accum;               // y += result instead of y = result
  const int32_t* xcols;    // mixed format: the outlier columns (ascending); x rows hold all columns and
  int64_t ncols;           //   the kernel stages the K main ones (the others taken out)
  int64_t xstride;         //   elements per activation row
  int prefetch;            // dense: weights may be read before the preceding grid completes
  int RS;                  // shared-memory bytes per staged code row
  int AS;                  // shared-memory bytes per staged scale row (kAuxRows)
  int aux_mode;
  int stages, stage_bytes, aux_off;  // ring geometry; aux_off: scale region inside a stage
  int XS;                  // shared-memory bytes per staged activation row
  int64_t xphase;          // 0: all of K staged; else in-features staged per phase (a multiple of KC)
  int n_xrows;             // activation rows staged
  int off_red, off_x, off_stage;  // dynamic shared-memory offsets
  int smem_bytes;
  int ctas_per_sm;         // 1..2, by shared-memory footprint
  int warps;               // warps per CTA (8 or 16)
  int grid;                // CTAs of the launch
  int argmax;              // fused argmax: outputs go to am_* instead of y
  uint32_t* am_ticket;     // workspace: CTA counter, then [grid][kMaxCols] partial keys
  unsigned long long* am_part;
  int32_t* am_idx;
  float* am_val;
};

// Per-format constants (bits per weight, scale bytes per 32-block).
struct FmtInfo {
  int bits, scale_bytes, kc_max;
  bool lut;
  bool zp;  // per-block zero points after the scales (int4aff)
};
inline FmtInfo fmt_info(int fmt) {
  switch (fmt) {
    case QMV_FMT_FP4: return {4, 1, 2048, false, false};
    case QMV_FMT_INT4: return {4, 2, 2048, false, false};
    case QMV_FMT_INT4KM: return {4, 0, 2048, true, false};
    case QMV_FMT_INT4AFF: return {4, 2, 2048, false, true};
    default: return {8, 2, 1024, false, false};
  }
}
// Bytes of one int4aff aux row: fp16 scales, then zero points two per byte.
__host__ __device__ inline int64_t int4aff_aux_row_bytes(int64_t K) { return 2 * (K / 32) + (K / 32 + 1) / 2; }

// Fills the geometry and the launch shape of `p` (shapes and pointers
// already set) for a device with `num_sms` SMs.  Returns false when the
// activations plus a two-stage ring do not fit in shared memory.
bool plan_matvec(int fmt, MvParams& p, int num_sms);

// Workspace bytes of the fused argmax for a device with `num_sms` SMs: a
// 16-byte counter block and one partial key per (CTA, activation row).
inline size_t argmax_workspace_bytes(int num_sms) {
  return 16 + (size_t)num_sms * 2 * kMaxCols * sizeof(unsigned long long);
}

cudaError_t launch_matvec(int fmt, const MvParams& p, cudaStream_t stream);
// int8km (dense or gather; p.argmax for the fused argmax): geometry, launch.
bool plan_km8(MvParams& p, int num_sms);
// The mixed int4km + int8 outlier-column format: column choice (ws: 2K
// ints) and the column split of fp32 weights.
cudaError_t launch_outlier_columns(const float* W, int64_t N, int64_t K, int64_t C, int32_t* cols, int* ws,
                                   int num_sms, cudaStream_t stream);
cudaError_t launch_split_f32(const float* W, int64_t N, int64_t K, const int32_t* cols, int64_t C, float* Wmain,
                             float* Wout, int num_sms, cudaStream_t stream);
// y[b, n] += sum over the C outlier columns of x[b, cols[c]] * q[n, c] * s[n, c / 32]
// (dependent launch: everything is read after the wait for the int4km part).
cudaError_t launch_outlier_acc(const int8_t* q, const uint16_t* s, const int32_t* cols, const uint16_t* x, int B,
                               int64_t N, int64_t K, int64_t C, float* y, int num_sms, cudaStream_t stream);
cudaError_t launch_km8(const MvParams& p, cudaStream_t stream);
// int8km palette fit (256 entries per 32 rows) and its workspace: one slot
// of next_pow2(min(N, 32) * K) keys per CTA.
int64_t km8fit_workspace_bytes(int64_t N, int64_t K);
cudaError_t launch_encode_int8km(const float* W, int64_t N, int64_t K, int iters, uint16_t* lut, uint8_t* idx,
                                 void* workspace, uint32_t* status, int num_sms, cudaStream_t stream);
// fp4 at 1..16 activation columns on the tcgen05 tensor cores (dense only;
// the activations of all K staged per CTA): geometry, launch.
bool plan_fp4_tc(MvParams& p, int num_sms);
cudaError_t launch_fp4_tc(const MvParams& p, cudaStream_t stream);

// ---- encoders / dequant ------------------------------------------------------
struct ClipList {
  float v[16];
  int n;
};

cudaError_t launch_encode_fp4(const float* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* scales,
                              uint32_t* status, int num_sms, cudaStream_t stream);
cudaError_t launch_encode_int(int qmax, const float* W, int64_t N, int64_t K, const ClipList& clips,
                              uint8_t* codes, uint16_t* scales, uint32_t* status, int num_sms,
                              cudaStream_t stream);
cudaError_t launch_encode_int4aff(const float* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* aux,
                                  uint32_t* status, int num_sms, cudaStream_t stream);
cudaError_t launch_encode_int4km(const float* W, int64_t N, int64_t K, int iters, uint16_t* lut, uint8_t* idx,
                                 uint32_t* status, int num_sms, cudaStream_t stream);
cudaError_t launch_dequant(int fmt, const uint8_t* codes, const uint8_t* aux, int64_t N, int64_t K, float* Wdq,
                           int num_sms, cudaStream_t stream);

}  // namespace qmv
