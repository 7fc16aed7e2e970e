// qmv_abi.cu -- the extern "C" entry points of libqmv (declared in qmv.h):
// host-side argument validation, the per-device status word, last-error text
// and the kernel launches on the caller's stream.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "qmv_internal.h"

namespace {

thread_local char g_err[512] = "";
std::atomic<int> g_weight_prefetch{0};  // qmv_set_weight_prefetch
std::atomic<int> g_fp4_tc{0};           // qmv_set_fp4_tensor_cores

qmv_status fail(qmv_status code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

qmv_status cuda_fail(cudaError_t e, const char* what) {
  return fail(QMV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Device status word: one per device (a __device__ variable exists once per
// device that loads the module).  Kernels OR QMV_FLAG_* bits into it.
__device__ uint32_t g_status_word;

constexpr int kMaxDevices = 64;
// Filled on a device's first call; several host threads may make that first
// call at once, so the values are published with release stores after the
// set-up ran under g_setup_mutex, and read with acquire loads.
std::atomic<uint32_t*> g_status_ptr[kMaxDevices];
std::atomic<int> g_num_sms[kMaxDevices];
std::mutex g_setup_mutex;

// Per-device set-up (current device): the status word's device address and
// the SM count.  Runs on a device's first call.
qmv_status device_ctx(uint32_t** status, int* num_sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(QMV_ERR_UNSUPPORTED, "device %d out of range", dev);
  uint32_t* sp = g_status_ptr[dev].load(std::memory_order_acquire);
  if (!sp) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    sp = g_status_ptr[dev].load(std::memory_order_acquire);
    if (!sp) {
      void* ptr = nullptr;
      e = cudaGetSymbolAddress(&ptr, g_status_word);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
      int sms = 0;
      e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
      g_num_sms[dev].store(sms, std::memory_order_relaxed);
      sp = static_cast<uint32_t*>(ptr);
      g_status_ptr[dev].store(sp, std::memory_order_release);
    }
  }
  *status = sp;
  *num_sms = g_num_sms[dev].load(std::memory_order_relaxed);
  return QMV_OK;
}

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

qmv_status check_ptr(const void* p, const char* name) {
  if (!p) return fail(QMV_ERR_ARG, "%s is null", name);
  if (!aligned16(p)) return fail(QMV_ERR_ARG, "%s is not 16-byte aligned", name);
  return QMV_OK;
}

// formats whose aux is fp16 scales at every row start (int4aff rows may have
// an odd byte count and are read bytewise where they are not 8-byte granular)
bool has_fp16_scale_rows(int fmt) { return fmt == QMV_FMT_INT4 || fmt == QMV_FMT_INT8 || fmt == QMV_FMT_INT8KM; }

qmv_status check_shape(int64_t N, int64_t K) {
  if (N < 1) return fail(QMV_ERR_SHAPE, "N must be >= 1 (got %lld)", (long long)N);
  if (K < 32 || K % 32 != 0)
    return fail(QMV_ERR_SHAPE, "K must be a positive multiple of the 32-element block (got %lld)", (long long)K);
  if (K > (int64_t)1 << 30 || N > (int64_t)1 << 40) return fail(QMV_ERR_SHAPE, "shape too large");
  return QMV_OK;
}

#define QMV_TRY(x)                  \
  do {                              \
    const qmv_status _s = (x);      \
    if (_s != QMV_OK) return _s;    \
  } while (0)

qmv_status encode_int(int qmax, const float* W, int64_t N, int64_t K, const float* clips, int n_clips,
                      uint8_t* codes, uint16_t* scales, void* stream) {
  QMV_TRY(check_ptr(W, "W"));
  QMV_TRY(check_ptr(codes, "codes"));
  if (!scales || (reinterpret_cast<uintptr_t>(scales) & 1u)) return fail(QMV_ERR_ARG, "scales null or misaligned");
  QMV_TRY(check_shape(N, K));
  if (!clips || n_clips < 1 || n_clips > 16) return fail(QMV_ERR_ARG, "clip list must hold 1..16 values");
  qmv::ClipList cl{};
  for (int i = 0; i < n_clips; ++i) {
    if (!(clips[i] > 0.0f) || clips[i] != clips[i]) return fail(QMV_ERR_ARG, "clip %d is not a positive number", i);
    cl.v[i] = clips[i];
  }
  cl.n = n_clips;
  uint32_t* st;
  int sms;
  QMV_TRY(device_ctx(&st, &sms));
  cudaError_t e = qmv::launch_encode_int(qmax, W, N, K, cl, codes, scales, st, sms, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "encode launch");
  return QMV_OK;
}

// Scratch of qmv_matvec_argmax_static: room for 512 SMs (two CTAs each),
// zero at module load; every call leaves it zero.  Its address is looked up
// once per device.
constexpr size_t kStaticArgmaxBytes = 16 + 512 * 2 * qmv::kMaxCols * sizeof(unsigned long long);
__device__ __align__(256) unsigned char g_argmax_scratch[kStaticArgmaxBytes];
std::atomic<void*> g_argmax_scratch_ptr[kMaxDevices];

qmv_status static_argmax_scratch(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(QMV_ERR_UNSUPPORTED, "device %d out of range", dev);
  void* a = g_argmax_scratch_ptr[dev].load(std::memory_order_acquire);
  if (!a) {
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    a = g_argmax_scratch_ptr[dev].load(std::memory_order_acquire);
    if (!a) {
      e = cudaGetSymbolAddress(&a, g_argmax_scratch);
      if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(argmax scratch)");
      g_argmax_scratch_ptr[dev].store(a, std::memory_order_release);
    }
  }
  *ptr = a;
  return QMV_OK;
}

struct ArgmaxOut {
  void* ws;
  size_t ws_bytes;
  int32_t* idx;
  float* val;
};

qmv_status matvec_common(int fmt, const void* codes, const void* aux, const uint16_t* x, int B, int64_t N,
                         int64_t K, float* y, void* stream, bool gather, int E, const int32_t* ids, int topk,
                         int x_per_slot, const ArgmaxOut* am = nullptr, bool accum = false,
                         const int32_t* xcols = nullptr, int64_t ncols = 0, int64_t xstride = 0) {
  if (fmt < QMV_FMT_FP4 || fmt > QMV_FMT_INT8KM) return fail(QMV_ERR_ARG, "unknown format %d", fmt);
  QMV_TRY(check_ptr(codes, "codes"));
  if (!aux) return fail(QMV_ERR_ARG, "scales/lut is null");
  // the staged scale block copies handle any byte alignment; the palette and
  // row-aligned scale copies need 16-byte alignment
  if (fmt == QMV_FMT_INT4KM) QMV_TRY(check_ptr(aux, "lut"));
  if (has_fp16_scale_rows(fmt) && (reinterpret_cast<uintptr_t>(aux) & 1u))
    return fail(QMV_ERR_ARG, "fp16 scales misaligned");
  QMV_TRY(check_ptr(x, "x"));
  if (!am && (!y || (reinterpret_cast<uintptr_t>(y) & 3u))) return fail(QMV_ERR_ARG, "y null or misaligned");
  QMV_TRY(check_shape(N, K));
  if (B < 1 || B > 16) return fail(QMV_ERR_UNSUPPORTED, "B must be in [1, 16] (got %d)", B);
  qmv::MvParams p{};
  p.codes = static_cast<const uint8_t*>(codes);
  p.aux = static_cast<const uint8_t*>(aux);
  p.x = x;
  p.y = y;
  p.N = N;
  p.K = K;
  p.B = B;
  p.gather = gather ? 1 : 0;
  if (gather) {
    if (E < 1) return fail(QMV_ERR_SHAPE, "E must be >= 1");
    if (topk < 1 || topk > 16) return fail(QMV_ERR_UNSUPPORTED, "topk must be in [1, 16] (got %d)", topk);
    if (!ids || (reinterpret_cast<uintptr_t>(ids) & 3u)) return fail(QMV_ERR_ARG, "expert_ids null or misaligned");
    if (x_per_slot != 0 && x_per_slot != 1) return fail(QMV_ERR_ARG, "x_per_slot must be 0 or 1");
    p.ids = ids;
    p.E = E;
    p.topk = topk;
    p.x_per_slot = x_per_slot;
  } else {
    p.E = 1;
    p.topk = 1;
  }
  uint32_t* st;
  int sms;
  QMV_TRY(device_ctx(&st, &sms));
  const bool km8 = fmt == QMV_FMT_INT8KM;
  const bool tc = fmt == QMV_FMT_FP4 && !gather && !am && !accum && !xcols && B >= 2 &&
                  g_fp4_tc.load(std::memory_order_relaxed) && qmv::plan_fp4_tc(p, sms);
  if (!tc && !(km8 ? qmv::plan_km8(p, sms) : qmv::plan_matvec(fmt, p, sms)))
    return fail(QMV_ERR_UNSUPPORTED, "activations (%d rows x %lld) do not fit the on-chip staging", p.n_xrows,
                (long long)K);
  p.status = st;
  p.prefetch = (!gather && g_weight_prefetch.load(std::memory_order_relaxed)) ? 1 : 0;
  p.accum = accum ? 1 : 0;
  p.xcols = xcols;
  p.ncols = ncols;
  p.xstride = xstride;
  if (am) {
    if (N >= (int64_t(1) << 31)) return fail(QMV_ERR_SHAPE, "argmax needs N < 2^31");
    if (!am->ws || (reinterpret_cast<uintptr_t>(am->ws) & 15u)) return fail(QMV_ERR_ARG, "workspace null or not 16-byte aligned");
    if (am->ws_bytes < qmv::argmax_workspace_bytes(sms))
      return fail(QMV_ERR_ARG, "workspace has %zu bytes, needs %zu", am->ws_bytes, qmv::argmax_workspace_bytes(sms));
    if (!am->idx || (reinterpret_cast<uintptr_t>(am->idx) & 3u)) return fail(QMV_ERR_ARG, "idx null or misaligned");
    if (!am->val || (reinterpret_cast<uintptr_t>(am->val) & 3u)) return fail(QMV_ERR_ARG, "val null or misaligned");
    p.argmax = 1;
    p.am_ticket = static_cast<uint32_t*>(am->ws);
    p.am_part = reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(am->ws) + 16);
    p.am_idx = am->idx;
    p.am_val = am->val;
  }
  cudaError_t e = tc    ? qmv::launch_fp4_tc(p, (cudaStream_t)stream)
                  : km8 ? qmv::launch_km8(p, (cudaStream_t)stream)
                        : qmv::launch_matvec(fmt, p, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "matvec launch");
  return QMV_OK;
}

}  // namespace

extern "C" {

qmv_status qmv_encode_fp4(const float* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* scales, void* stream) {
  QMV_TRY(check_ptr(W, "W"));
  QMV_TRY(check_ptr(codes, "codes"));
  if (!scales) return fail(QMV_ERR_ARG, "scales is null");
  QMV_TRY(check_shape(N, K));
  uint32_t* st;
  int sms;
  QMV_TRY(device_ctx(&st, &sms));
  cudaError_t e = qmv::launch_encode_fp4(W, N, K, codes, scales, st, sms, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "encode_fp4 launch");
  return QMV_OK;
}

qmv_status qmv_encode_int4(const float* W, int64_t N, int64_t K, const float* clips, int n_clips,
                           uint8_t* codes, uint16_t* scales, void* stream) {
  return encode_int(7, W, N, K, clips, n_clips, codes, scales, stream);
}

qmv_status qmv_encode_int8(const float* W, int64_t N, int64_t K, const float* clips, int n_clips,
                           int8_t* codes, uint16_t* scales, void* stream) {
  return encode_int(127, W, N, K, clips, n_clips, reinterpret_cast<uint8_t*>(codes), scales, stream);
}

qmv_status qmv_encode_int4km(const float* W, int64_t N, int64_t K, int iters, uint16_t* lut, uint8_t* idx,
                             void* stream) {
  QMV_TRY(check_ptr(W, "W"));
  QMV_TRY(check_ptr(idx, "idx"));
  if (!lut || (reinterpret_cast<uintptr_t>(lut) & 1u)) return fail(QMV_ERR_ARG, "lut null or misaligned");
  if (iters < 0 || iters > 1000) return fail(QMV_ERR_ARG, "iters must be in [0, 1000] (got %d)", iters);
  QMV_TRY(check_shape(N, K));
  if (K > 16384) return fail(QMV_ERR_UNSUPPORTED, "K must be <= 16384 for the palette fit (got %lld)", (long long)K);
  uint32_t* st;
  int sms;
  QMV_TRY(device_ctx(&st, &sms));
  cudaError_t e = qmv::launch_encode_int4km(W, N, K, iters, lut, idx, st, sms, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "encode_int4km launch");
  return QMV_OK;
}

qmv_status qmv_encode_int4aff(const float* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* aux, void* stream) {
  QMV_TRY(check_ptr(W, "W"));
  QMV_TRY(check_ptr(codes, "codes"));
  if (!aux) return fail(QMV_ERR_ARG, "aux is null");
  QMV_TRY(check_shape(N, K));
  uint32_t* st;
  int sms;
  QMV_TRY(device_ctx(&st, &sms));
  cudaError_t e = qmv::launch_encode_int4aff(W, N, K, codes, aux, st, sms, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "encode_int4aff launch");
  return QMV_OK;
}

int64_t qmv_int4aff_aux_row_bytes(int64_t K) { return K >= 32 ? qmv::int4aff_aux_row_bytes(K) : 0; }

qmv_status qmv_matvec_fp4(const uint8_t* codes, const uint8_t* scales, const uint16_t* x, int B, int64_t N,
                          int64_t K, float* y, void* stream) {
  return matvec_common(QMV_FMT_FP4, codes, scales, x, B, N, K, y, stream, false, 0, nullptr, 0, 0);
}

qmv_status qmv_matvec_int4(const uint8_t* codes, const uint16_t* scales, const uint16_t* x, int B, int64_t N,
                           int64_t K, float* y, void* stream) {
  return matvec_common(QMV_FMT_INT4, codes, scales, x, B, N, K, y, stream, false, 0, nullptr, 0, 0);
}

qmv_status qmv_matvec_int4km(const uint8_t* idx, const uint16_t* lut, const uint16_t* x, int B, int64_t N,
                             int64_t K, float* y, void* stream) {
  return matvec_common(QMV_FMT_INT4KM, idx, lut, x, B, N, K, y, stream, false, 0, nullptr, 0, 0);
}

qmv_status qmv_matvec_int8(const int8_t* codes, const uint16_t* scales, const uint16_t* x, int B, int64_t N,
                           int64_t K, float* y, void* stream) {
  return matvec_common(QMV_FMT_INT8, codes, scales, x, B, N, K, y, stream, false, 0, nullptr, 0, 0);
}

qmv_status qmv_matvec_int4aff(const uint8_t* codes, const uint8_t* aux, const uint16_t* x, int B, int64_t N,
                              int64_t K, float* y, void* stream) {
  return matvec_common(QMV_FMT_INT4AFF, codes, aux, x, B, N, K, y, stream, false, 0, nullptr, 0, 0);
}

qmv_status qmv_matvec_int8km(const uint8_t* idx, const uint16_t* lut, const uint16_t* x, int B, int64_t N,
                             int64_t K, float* y, void* stream) {
  return matvec_common(QMV_FMT_INT8KM, idx, lut, x, B, N, K, y, stream, false, 0, nullptr, 0, 0);
}

// ---- mixed int4km + int8 outlier columns ----

static int64_t round256(int64_t v) { return (v + 255) / 256 * 256; }

static qmv_status check_mixed_shape(int64_t N, int64_t K, int64_t C) {
  QMV_TRY(check_shape(N, K));
  if (C < 0 || C % 32 != 0 || C >= K)
    return fail(QMV_ERR_SHAPE, "C must be a multiple of 32 in [0, K) (got %lld)", (long long)C);
  return QMV_OK;
}

int64_t qmv_int4km_o8_encode_workspace_bytes(int64_t N, int64_t K, int64_t C) {
  return round256(4 * N * (K - C)) + round256(4 * N * C) + round256(8 * K);
}

qmv_status qmv_outlier_columns(const float* W, int64_t N, int64_t K, int64_t C, int32_t* cols, void* workspace,
                               size_t workspace_bytes, void* stream) {
  QMV_TRY(check_ptr(W, "W"));
  QMV_TRY(check_mixed_shape(N, K, C));
  if (C > 0 && (!cols || (reinterpret_cast<uintptr_t>(cols) & 3u))) return fail(QMV_ERR_ARG, "cols null or misaligned");
  QMV_TRY(check_ptr(workspace, "workspace"));
  if (workspace_bytes < (size_t)(8 * K)) return fail(QMV_ERR_ARG, "workspace has %zu bytes, needs %lld",
                                                     workspace_bytes, (long long)(8 * K));
  uint32_t* st;
  int sms;
  QMV_TRY(device_ctx(&st, &sms));
  if (C == 0) return QMV_OK;
  cudaError_t e = qmv::launch_outlier_columns(W, N, K, C, cols, static_cast<int*>(workspace), sms, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "outlier_columns launch");
  return QMV_OK;
}

int64_t qmv_int8km_encode_workspace_bytes(int64_t N, int64_t K) {
  if (N < 1 || K < 32 || K > 16384) return 0;
  return qmv::km8fit_workspace_bytes(N, K);
}

qmv_status qmv_encode_int8km(const float* W, int64_t N, int64_t K, int iters, uint16_t* lut, uint8_t* idx,
                             void* workspace, size_t workspace_bytes, void* stream) {
  QMV_TRY(check_ptr(W, "W"));
  QMV_TRY(check_ptr(idx, "idx"));
  if (!lut || (reinterpret_cast<uintptr_t>(lut) & 1u)) return fail(QMV_ERR_ARG, "lut null or misaligned");
  QMV_TRY(check_shape(N, K));
  if (iters < 0 || iters > 1000) return fail(QMV_ERR_ARG, "iters must be in [0, 1000] (got %d)", iters);
  if (K > 16384) return fail(QMV_ERR_UNSUPPORTED, "K must be <= 16384 for the int8km palette fit");
  QMV_TRY(check_ptr(workspace, "workspace"));
  const int64_t need = qmv::km8fit_workspace_bytes(N, K);
  if ((int64_t)workspace_bytes < need)
    return fail(QMV_ERR_ARG, "workspace has %zu bytes, needs %lld", workspace_bytes, (long long)need);
  uint32_t* st;
  int sms;
  QMV_TRY(device_ctx(&st, &sms));
  cudaError_t e = qmv::launch_encode_int8km(W, N, K, iters, lut, idx, workspace, st, sms, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "encode_int8km launch");
  return QMV_OK;
}

qmv_status qmv_encode_int4km_o8(const float* W, int64_t N, int64_t K, int64_t C, int iters, int32_t* cols,
                                uint16_t* lut, uint8_t* idx, int8_t* ocodes, uint16_t* oscales, void* workspace,
                                size_t workspace_bytes, void* stream) {
  QMV_TRY(check_ptr(W, "W"));
  QMV_TRY(check_mixed_shape(N, K, C));
  QMV_TRY(check_ptr(idx, "idx"));
  if (!lut || (reinterpret_cast<uintptr_t>(lut) & 1u)) return fail(QMV_ERR_ARG, "lut null or misaligned");
  if (C > 0) {
    if (!cols || (reinterpret_cast<uintptr_t>(cols) & 3u)) return fail(QMV_ERR_ARG, "cols null or misaligned");
    QMV_TRY(check_ptr(ocodes, "ocodes"));
    if (!oscales || (reinterpret_cast<uintptr_t>(oscales) & 1u)) return fail(QMV_ERR_ARG, "oscales null or misaligned");
  }
  if (iters < 0 || iters > 1000) return fail(QMV_ERR_ARG, "iters must be in [0, 1000] (got %d)", iters);
  if (K - C > 16384) return fail(QMV_ERR_UNSUPPORTED, "K - C must be <= 16384 for the palette fit");
  QMV_TRY(check_ptr(workspace, "workspace"));
  const int64_t need = qmv_int4km_o8_encode_workspace_bytes(N, K, C);
  if ((int64_t)workspace_bytes < need)
    return fail(QMV_ERR_ARG, "workspace has %zu bytes, needs %lld", workspace_bytes, (long long)need);
  uint32_t* st;
  int sms;
  QMV_TRY(device_ctx(&st, &sms));
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* Wmain = reinterpret_cast<float*>(ws);
  float* Wout = reinterpret_cast<float*>(ws + round256(4 * N * (K - C)));
  int* keys = reinterpret_cast<int*>(ws + round256(4 * N * (K - C)) + round256(4 * N * C));
  cudaError_t e = cudaSuccess;
  if (C > 0) {
    e = qmv::launch_outlier_columns(W, N, K, C, cols, keys, sms, s);
    if (e == cudaSuccess) e = qmv::launch_split_f32(W, N, K, cols, C, Wmain, Wout, sms, s);
  }
  if (e == cudaSuccess) e = qmv::launch_encode_int4km(C > 0 ? Wmain : W, N, K - C, iters, lut, idx, st, sms, s);
  if (e == cudaSuccess && C > 0) {
    qmv::ClipList cl{};
    cl.v[0] = 1.0f;
    cl.n = 1;
    e = qmv::launch_encode_int(127, Wout, N, C, cl, reinterpret_cast<uint8_t*>(ocodes), oscales, st, sms, s);
  }
  if (e != cudaSuccess) return cuda_fail(e, "encode_int4km_o8 launch");
  return QMV_OK;
}

qmv_status qmv_matvec_int4km_o8(const uint8_t* idx, const uint16_t* lut, const int8_t* ocodes, const uint16_t* oscales,
                                const int32_t* cols, const uint16_t* x, int B, int64_t N, int64_t K, int64_t C,
                                float* y, void* stream) {
  QMV_TRY(check_mixed_shape(N, K, C));
  QMV_TRY(check_ptr(x, "x"));
  if (B < 1 || B > 16) return fail(QMV_ERR_UNSUPPORTED, "B must be in [1, 16] (got %d)", B);
  if (C > 0) {
    if (!cols || (reinterpret_cast<uintptr_t>(cols) & 3u)) return fail(QMV_ERR_ARG, "cols null or misaligned");
    QMV_TRY(check_ptr(ocodes, "ocodes"));
    if (!oscales || (reinterpret_cast<uintptr_t>(oscales) & 1u)) return fail(QMV_ERR_ARG, "oscales null or misaligned");
  }
  // the int4km kernel stages the main columns of x and writes y; the outlier
  // kernel adds the int8 columns
  QMV_TRY(matvec_common(QMV_FMT_INT4KM, idx, lut, x, B, N, K - C, y, stream, false, 0, nullptr, 0, 0, nullptr, false,
                        C > 0 ? cols : nullptr, C, K));
  if (C > 0) {
    uint32_t* st;
    int sms;
    QMV_TRY(device_ctx(&st, &sms));
    cudaError_t e = qmv::launch_outlier_acc(ocodes, oscales, cols, x, B, N, K, C, y, sms, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "outlier columns launch");
  }
  return QMV_OK;
}

qmv_status qmv_matvec_argmax(int fmt, const void* codes, const void* aux, const uint16_t* x, int B, int64_t N,
                             int64_t K, void* workspace, size_t workspace_bytes, int32_t* idx, float* val,
                             void* stream) {
  const ArgmaxOut am{workspace, workspace_bytes, idx, val};
  return matvec_common(fmt, codes, aux, x, B, N, K, nullptr, stream, false, 0, nullptr, 0, 0, &am);
}

qmv_status qmv_matvec_argmax_static(int fmt, const void* codes, const void* aux, const uint16_t* x, int B,
                                    int64_t N, int64_t K, int32_t* idx, float* val, void* stream) {
  void* ws = nullptr;
  QMV_TRY(static_argmax_scratch(&ws));
  uint32_t* st;
  int sms;
  QMV_TRY(device_ctx(&st, &sms));
  if (qmv::argmax_workspace_bytes(sms) > kStaticArgmaxBytes)
    return fail(QMV_ERR_UNSUPPORTED, "device needs %zu bytes of argmax scratch, the library holds %zu",
                qmv::argmax_workspace_bytes(sms), kStaticArgmaxBytes);
  const ArgmaxOut am{ws, kStaticArgmaxBytes, idx, val};
  return matvec_common(fmt, codes, aux, x, B, N, K, nullptr, stream, false, 0, nullptr, 0, 0, &am);
}

qmv_status qmv_argmax_workspace_bytes(size_t* bytes) {
  if (!bytes) return fail(QMV_ERR_ARG, "bytes is null");
  uint32_t* st;
  int sms;
  QMV_TRY(device_ctx(&st, &sms));
  *bytes = qmv::argmax_workspace_bytes(sms);
  return QMV_OK;
}

qmv_status qmv_gather_matvec(int fmt, const void* codes_stack, const void* aux_stack, int E, int64_t N, int64_t K,
                             const int32_t* expert_ids, int B, int topk, const uint16_t* x, int x_per_slot,
                             float* y, void* stream) {
  if (B < 1 || B > 16) return fail(QMV_ERR_UNSUPPORTED, "B must be in [1, 16] (got %d)", B);
  return matvec_common(fmt, codes_stack, aux_stack, x, B, N, K, y, stream, true, E, expert_ids, topk, x_per_slot);
}

qmv_status qmv_dequant(int fmt, const void* codes, const void* aux, int64_t N, int64_t K, float* Wdq, void* stream) {
  if (fmt < QMV_FMT_FP4 || fmt > QMV_FMT_INT8KM) return fail(QMV_ERR_ARG, "unknown format %d", fmt);
  QMV_TRY(check_ptr(codes, "codes"));
  if (!aux) return fail(QMV_ERR_ARG, "aux is null");
  if (fmt == QMV_FMT_INT4KM) QMV_TRY(check_ptr(aux, "lut"));
  if (has_fp16_scale_rows(fmt) && (reinterpret_cast<uintptr_t>(aux) & 1u))
    return fail(QMV_ERR_ARG, "fp16 scales misaligned");
  QMV_TRY(check_ptr(Wdq, "Wdq"));
  QMV_TRY(check_shape(N, K));
  uint32_t* st;
  int sms;
  QMV_TRY(device_ctx(&st, &sms));
  cudaError_t e = qmv::launch_dequant(fmt, static_cast<const uint8_t*>(codes), static_cast<const uint8_t*>(aux), N, K,
                                      Wdq, sms, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "dequant launch");
  return QMV_OK;
}

qmv_status qmv_status_fetch(void* stream, uint32_t* flags) {
  if (!flags) return fail(QMV_ERR_ARG, "flags is null");
  *flags = 0;
  uint32_t* st;
  int sms;
  QMV_TRY(device_ctx(&st, &sms));
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  uint32_t v = 0;
  e = cudaMemcpyFromSymbol(&v, g_status_word, sizeof(v));
  if (e != cudaSuccess) return cuda_fail(e, "read status");
  const uint32_t zero = 0;
  e = cudaMemcpyToSymbol(g_status_word, &zero, sizeof(zero));
  if (e != cudaSuccess) return cuda_fail(e, "clear status");
  *flags = v;
  if (v) return fail(QMV_ERR_DATA, "device status flags 0x%x", v);
  return QMV_OK;
}

const char* qmv_last_error(void) { return g_err; }

qmv_status qmv_set_weight_prefetch(int enable) {
  if (enable != 0 && enable != 1) return fail(QMV_ERR_ARG, "enable must be 0 or 1 (got %d)", enable);
  g_weight_prefetch.store(enable, std::memory_order_relaxed);
  return QMV_OK;
}

qmv_status qmv_set_fp4_tensor_cores(int mode) {
  if (mode != 0 && mode != 1) return fail(QMV_ERR_ARG, "mode must be 0 or 1 (got %d)", mode);
  g_fp4_tc.store(mode, std::memory_order_relaxed);
  return QMV_OK;
}

const char* qmv_version(void) { return "0.1.0"; }

}  // extern "C"
