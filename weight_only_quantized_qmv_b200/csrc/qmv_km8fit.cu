// qmv_km8fit.cu -- int8km encoder: a 256-entry fp16 palette per group of 32
// output rows by scalar 1-D k-means, plus one 8-bit palette index per
// weight, on the GPU.
//
// What it computes ("coreai-optimization (coreai-opt) reference --
// quantization & palettization", sec. "Palettization": scalar k-means,
// 2^n_bits centroids, per-grouped-channel LUTs; "Compression (palettization
// & quantization)", "int8 k-means > whole-model int4": 8-bit k-means with
// group size 32), with the readings the pages leave open fixed as for
// int4km, per group of 32 consecutive rows (n = rows * K weights; a last
// group of fewer rows is fitted on the rows it has):
//   1. sort ascending, -0 before +0;
//   2. centre k starts at sorted[floor((2k+1) n / 512)];
//   3. `iters` Lloyd steps: each weight goes to the nearest centre (double
//      distance, ties to the lower index); each non-empty centre becomes
//      float(double sum of its members added in ascending order / count);
//      an empty centre keeps its value;
//   4. palette = fp16 round-to-nearest-even of the centres;
//   5. index = nearest palette entry (double distance, ties to lower index).
// A group holding Inf/NaN is written as zeros and sets QMV_FLAG_NONFINITE.
//
// Design: one CTA per group (persistent over groups).  The group's n keys
// are sorted in a caller workspace slot (L2-resident) by a keys-only
// bitonic sort whose strides below 8192 run in shared memory.  On the
// sorted values the weights nearest to one centre form a contiguous run, so
// a Lloyd step sorts the 256 centres, finds each boundary between centres
// adjacent in value by a binary search that evaluates the assignment rule
// itself, and one thread per centre adds its run in ascending order in
// double -- the order of the per-weight accumulation, so every rounding
// matches.  The indices come from a binary search of each weight over the
// sorted palette with the same rule.  (The runs equal the rule's assignment
// when no two centres tie in computed double distance other than by equal
// values; for the weights of one group that needs a dynamic range beyond
// 2^50.)
#include <atomic>
#include <cuda_fp16.h>

#include "qmv_device.cuh"
#include "qmv_internal.h"

namespace qmv {

namespace {

constexpr int kFitThreads = 512;
constexpr int kFitChunk = 8192;  // keys per shared-memory bitonic phase
constexpr int kFitCentres = 256;
constexpr int kFitGroup = 32;   // rows per palette
constexpr int kFitMaxCtas = 160;

// float -> uint32 whose unsigned order is the float order with -0 < +0
__device__ __forceinline__ uint32_t fit_key(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float fit_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

struct FitShared {
  uint32_t chunk[kFitChunk];
  unsigned long long ord[kFitCentres];  // (key of the centre's value, index)
  double cen[kFitCentres];              // centres by index
  double dval[kFitCentres];             // distinct centre values, ascending
  int didx[kFitCentres];                // lowest index holding each
  int bnd[kFitCentres + 1];             // run starts in the sorted keys
  int first[kFitCentres];
  int nd;
};

// One bitonic compare-exchange pass over pairs (i, i + stride), i enumerated
// from t; direction by the global index gi of the pair's first element.
__device__ __forceinline__ void bitonic_pair(uint32_t* a, int t, int stride, int64_t base, int64_t size) {
  const int i = 2 * t - (t & (stride - 1)), j = i + stride;
  const uint32_t ki = a[i], kj = a[j];
  const bool up = ((base + i) & size) == 0;
  if ((ki > kj) == up) {
    a[i] = kj;
    a[j] = ki;
  }
}

// Shared-memory phase: strides stride0 .. 1 of sizes size0 .. min(C, P) for
// every chunk of C keys of S (size0 = 2: the chunk's whole sort).
__device__ void bitonic_local(FitShared& sh, uint32_t* S, int64_t P, int C, int64_t size_first, bool whole) {
  for (int64_t base = 0; base < P; base += C) {
    for (int i = threadIdx.x; i < C; i += kFitThreads) sh.chunk[i] = S[base + i];
    __syncthreads();
    if (whole) {
      for (int size = 2; size <= C; size <<= 1)
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
          for (int t = threadIdx.x; t < C / 2; t += kFitThreads) bitonic_pair(sh.chunk, t, stride, base, size);
          __syncthreads();
        }
    } else {
      for (int stride = C >> 1; stride > 0; stride >>= 1) {
        for (int t = threadIdx.x; t < C / 2; t += kFitThreads) bitonic_pair(sh.chunk, t, stride, base, size_first);
        __syncthreads();
      }
    }
    for (int i = threadIdx.x; i < C; i += kFitThreads) S[base + i] = sh.chunk[i];
    __syncthreads();
  }
}

// Sorts the centres cen[] (threads 0..255 hold one each) and builds the
// distinct ascending list dval / didx (nd entries; equal values, -0 and +0
// included, keep the lowest index).
__device__ void distinct_centres(FitShared& sh) {
  const int tid = threadIdx.x;
  if (tid < kFitCentres)
    sh.ord[tid] = ((unsigned long long)fit_key((float)sh.cen[tid]) << 32) | (unsigned long long)tid;
  __syncthreads();
  for (int size = 2; size <= kFitCentres; size <<= 1)
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (tid < kFitCentres / 2) {
        const int i = 2 * tid - (tid & (stride - 1)), j = i + stride;
        const unsigned long long a = sh.ord[i], b = sh.ord[j];
        const bool up = (i & size) == 0;
        if ((a > b) == up) {
          sh.ord[i] = b;
          sh.ord[j] = a;
        }
      }
      __syncthreads();
    }
  if (tid < kFitCentres) {
    const float v = fit_value((uint32_t)(sh.ord[tid] >> 32));
    sh.first[tid] = (tid == 0 || fit_value((uint32_t)(sh.ord[tid - 1] >> 32)) != v) ? 1 : 0;
  }
  __syncthreads();
  if (tid < kFitCentres && sh.first[tid]) {
    int rank = 0;
    for (int k = 0; k < tid; ++k) rank += sh.first[k];
    const float v = fit_value((uint32_t)(sh.ord[tid] >> 32));
    int lo = (int)(sh.ord[tid] & 0xFFFFu);
    for (int k = tid + 1; k < kFitCentres && !sh.first[k]; ++k) lo = min(lo, (int)(sh.ord[k] & 0xFFFFu));
    sh.dval[rank] = (double)v;
    sh.didx[rank] = lo;
  }
  if (tid == 0) {
    int nd = 0;
    for (int k = 0; k < kFitCentres; ++k) nd += sh.first[k];
    sh.nd = nd;
  }
  __syncthreads();
}

// Does centre (c, ic) take value v from its lower neighbour (u, iu)?  The
// assignment rule: smaller double distance, ties to the lower index.
__device__ __forceinline__ bool takes(double v, double c, int ic, double u, int iu) {
  const double dc = fabs(v - c), du = fabs(v - u);
  return dc < du || (dc == du && ic < iu);
}

}  // namespace

__global__ void __launch_bounds__(kFitThreads, 1)
    km8fit_kernel(const float* __restrict__ W, int64_t N, int64_t K, int iters, uint16_t* __restrict__ lut,
                  uint8_t* __restrict__ idx, uint32_t* __restrict__ ws, int64_t slot_keys, uint32_t* status) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  FitShared& sh = *reinterpret_cast<FitShared*>(smem_raw);
  const int tid = threadIdx.x;
  uint32_t* S = ws + (int64_t)blockIdx.x * slot_keys;
  const int64_t G = (N + kFitGroup - 1) / kFitGroup;
  for (int64_t g = blockIdx.x; g < G; g += gridDim.x) {
    const int64_t r0 = g * kFitGroup;
    const int64_t rows = min((int64_t)kFitGroup, N - r0);
    const int64_t n = rows * K;
    int64_t P = 1;
    while (P < n) P <<= 1;
    const float* w = W + r0 * K;
    // keys (padding sorts last) and the finiteness check
    bool finite = true;
    for (int64_t i = tid; i < P; i += kFitThreads) {
      uint32_t k = 0xffffffffu;
      if (i < n) {
        const float v = w[i];
        finite = finite && isfinite(v);
        k = fit_key(v);
      }
      S[i] = k;
    }
    if (!__syncthreads_and(finite)) {
      for (int64_t i = tid; i < n; i += kFitThreads) idx[r0 * K + i] = 0;
      if (tid < kFitCentres) lut[g * kFitCentres + tid] = 0;
      if (tid == 0) atomicOr(status, QMV_FLAG_NONFINITE);
      __syncthreads();
      continue;
    }
    // bitonic sort, ascending: chunks in shared memory, strides >= C in place
    const int C = (int)min(P, (int64_t)kFitChunk);
    bitonic_local(sh, S, P, C, 0, true);
    for (int64_t size = 2 * (int64_t)C; size <= P; size <<= 1) {
      for (int64_t stride = size >> 1; stride >= C; stride >>= 1) {
        for (int64_t t = tid; t < P / 2; t += kFitThreads) {
          const int64_t i = 2 * t - (t & (stride - 1)), j = i + stride;
          const uint32_t ki = S[i], kj = S[j];
          const bool up = (i & size) == 0;
          if ((ki > kj) == up) {
            S[i] = kj;
            S[j] = ki;
          }
        }
        __syncthreads();
      }
      bitonic_local(sh, S, P, C, size, false);
    }
    // initial centres at the (k + 1/2)/256 quantiles
    if (tid < kFitCentres) sh.cen[tid] = (double)fit_value(S[((2 * (int64_t)tid + 1) * n) / (2 * kFitCentres)]);
    __syncthreads();
    for (int it = 0; it < iters; ++it) {
      distinct_centres(sh);
      const int nd = sh.nd;
      if (tid < nd) {
        int b = 0;
        if (tid > 0) {
          // first sorted position the centre takes from its lower neighbour
          const double c = sh.dval[tid], u = sh.dval[tid - 1];
          const int ic = sh.didx[tid], iu = sh.didx[tid - 1];
          int64_t a = 0, e = n;
          while (a < e) {
            const int64_t mid = (a + e) >> 1;
            if (takes((double)fit_value(S[mid]), c, ic, u, iu))
              e = mid;
            else
              a = mid + 1;
          }
          b = (int)a;
        }
        sh.bnd[tid] = b;
      }
      if (tid == 0) sh.bnd[nd] = (int)n;
      __syncthreads();
      if (tid < nd) {
        const int lo = sh.bnd[tid], hi = max(sh.bnd[tid + 1], lo);
        if (hi > lo) {
          double sum = 0.0;
#pragma unroll 8
          for (int i = lo; i < hi; ++i) sum += (double)fit_value(S[i]);
          sh.cen[sh.didx[tid]] = (double)__double2float_rn(sum / (double)(hi - lo));
        }
      }
      __syncthreads();
    }
    // palette, then each weight's nearest palette entry
    if (tid < kFitCentres) {
      const __half hv = __float2half_rn((float)sh.cen[tid]);
      lut[g * kFitCentres + tid] = __half_as_ushort(hv);
      sh.cen[tid] = (double)__half2float(hv);
    }
    __syncthreads();
    distinct_centres(sh);
    const int nd = sh.nd;
    for (int64_t i = tid; i < n; i += kFitThreads) {
      const double v = (double)w[i];
      // p = distinct palette values below v
      int a = 0, e = nd;
      while (a < e) {
        const int mid = (a + e) >> 1;
        if (sh.dval[mid] < v)
          a = mid + 1;
        else
          e = mid;
      }
      int best;
      if (a == 0)
        best = 0;
      else if (a == nd)
        best = nd - 1;
      else
        best = takes(v, sh.dval[a], sh.didx[a], sh.dval[a - 1], sh.didx[a - 1]) ? a : a - 1;
      idx[r0 * K + i] = (uint8_t)sh.didx[best];
    }
    __syncthreads();
  }
}

int64_t km8fit_slot_keys(int64_t N, int64_t K) {
  const int64_t n = (N < kFitGroup ? N : kFitGroup) * K;
  int64_t P = 1;
  while (P < n) P <<= 1;
  return P;
}

int64_t km8fit_workspace_bytes(int64_t N, int64_t K) {
  const int64_t G = (N + kFitGroup - 1) / kFitGroup;
  const int64_t ctas = G < kFitMaxCtas ? G : kFitMaxCtas;
  return ctas * km8fit_slot_keys(N, K) * 4;
}

cudaError_t launch_encode_int8km(const float* W, int64_t N, int64_t K, int iters, uint16_t* lut, uint8_t* idx,
                                 void* workspace, uint32_t* status, int num_sms, cudaStream_t stream) {
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(km8fit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sizeof(FitShared));
    if (err != cudaSuccess) return err;
    attr_set[dev].store(true, std::memory_order_release);
  }
  const int64_t G = (N + kFitGroup - 1) / kFitGroup;
  int64_t grid = G < num_sms ? G : num_sms;
  if (grid > kFitMaxCtas) grid = kFitMaxCtas;
  km8fit_kernel<<<(unsigned)grid, kFitThreads, sizeof(FitShared), stream>>>(
      W, N, K, iters, lut, idx, static_cast<uint32_t*>(workspace), km8fit_slot_keys(N, K), status);
  return cudaGetLastError();
}

}  // namespace qmv
