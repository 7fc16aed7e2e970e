// qmv_kmeans.cu -- int4km encoder: per-row 16-entry fp16 palette by scalar
// 1-D k-means, plus packed 4-bit palette indices, on the GPU.
//
// What it computes (the pages' palettization: "coreai-optimization
// (coreai-opt) reference -- quantization & palettization", sec.
// "Palettization": scalar k-means, 2^n_bits centroids, per-channel grouping;
// "Dense-path int4km coverage + flagship Qwen3.6-35B -- session findings &
// methods", sec. 8: a per-output-row 16-entry codebook), with the readings
// the pages leave open fixed as follows, per row of K weights:
//   1. sort ascending, -0 before +0;
//   2. centre k starts at sorted[floor((2k+1) K / 32)];
//   3. `iters` Lloyd steps: each weight goes to the nearest centre (double
//      distance, ties to the lower index); each non-empty centre becomes
//      float(double sum of its members added in ascending order / count); an
//      empty centre keeps its value;
//   4. palette = fp16 round-to-nearest-even of the centres;
//   5. index = nearest palette entry (double distance, ties to lower index).
// A row holding Inf/NaN is written as zeros and sets QMV_FLAG_NONFINITE.
//
// Design: one warp per row.  The row is sorted as (key, position) pairs in
// shared memory by a warp bitonic sort.  On the sorted row the weights
// nearest to one centre form a contiguous run, so a Lloyd step needs only
// the run boundaries: each of the (at most 15) boundaries between centres
// adjacent in value is found by a binary search that evaluates the
// assignment rule itself (double distances, lower index on ties).  One lane
// per centre then adds its run in ascending order in double, which is the
// order of the per-weight accumulation, so every rounding matches.  The
// final indices are scattered back to the weights' positions.  (The runs
// equal the rule's assignment when no two centres tie in computed double
// distance at a weight other than by equal values; for weights of one row
// that needs a dynamic range beyond 2^50.)
#include <atomic>

#include "qmv_device.cuh"

namespace qmv {

namespace {

// float -> uint32 whose unsigned order is the float order with -0 < +0
__device__ __forceinline__ uint32_t fkey(float v) {
  const uint32_t u = __float_as_uint(v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float fkey_value(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

struct KmShared {
  uint32_t* key;   // [P] sorted keys
  uint16_t* pos;   // [P] original positions
  uint8_t* ib;     // [K] palette index per original position
  int* bnd;        // [17] run starts, in value order of the centres
  int* who;        // [16] centre index of each run
};

// Runs of the sorted row for centres c (lane j < 16 holds c_j; all lanes get
// the results): writes bnd[0..nd] and who[0..nd-1]; returns nd (distinct
// centres).  Lane j returns its run [lo, hi) in *lo / *hi (empty when a lower
// index holds the same value).
__device__ int km_runs(const KmShared& sh, int K, double cj, int lane, int* lo, int* hi) {
  double c[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) c[k] = __shfl_sync(0xffffffffu, cj, k);
  int nd = 0;
  int rank = 0, shadow = 0, pred = -1;
  if (lane < 16) {
    double best = 0.0;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (k < lane && c[k] == cj) shadow = 1;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      // distinct values below cj, counted once (the lowest index of each value)
      bool first = true;
#pragma unroll
      for (int m = 0; m < 16; ++m)
        if (m < k && c[m] == c[k]) first = false;
      if (first && c[k] < cj) {
        ++rank;
        if (pred < 0 || c[k] > best) {
          best = c[k];
          pred = k;
        }
      }
    }
  }
  // number of distinct centres
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    bool first = true;
#pragma unroll
    for (int m = 0; m < 16; ++m)
      if (m < k && c[m] == c[k]) first = false;
    nd += first ? 1 : 0;
  }
  if (lane < 16 && !shadow) {
    int l = 0;
    if (pred >= 0) {
      // first sorted position where centre `lane` beats its lower neighbour
      const double cu = c[pred];
      int a = 0, b = K;
      while (a < b) {
        const int mid = (a + b) >> 1;
        const double v = (double)fkey_value(sh.key[mid]);
        const double dj = fabs(v - cj), du = fabs(v - cu);
        const bool mine = dj < du || (dj == du && lane < pred);
        if (mine)
          b = mid;
        else
          a = mid + 1;
      }
      l = a;
    }
    sh.bnd[rank] = l;
    sh.who[rank] = lane;
  }
  if (lane == 0) sh.bnd[nd] = K;
  __syncwarp();
  if (lane < 16) {
    if (shadow) {
      *lo = *hi = 0;
    } else {
      *lo = sh.bnd[rank];
      *hi = sh.bnd[rank + 1];
      if (*hi < *lo) *hi = *lo;
    }
  }
  return nd;
}

}  // namespace

__global__ void __launch_bounds__(256) km_kernel(const float* __restrict__ W, int64_t N, int K, int P, int iters,
                                                  uint16_t* __restrict__ lut, uint8_t* __restrict__ idx,
                                                  uint32_t* status, int warps, int per_warp) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp >= warps) return;
  uint8_t* base = smem + (size_t)warp * per_warp;
  KmShared sh;
  sh.key = reinterpret_cast<uint32_t*>(base);
  sh.pos = reinterpret_cast<uint16_t*>(base + 4 * P);
  sh.ib = base + 6 * P;
  sh.bnd = reinterpret_cast<int*>(base + ((6 * P + K + 15) & ~15));
  sh.who = sh.bnd + 17;

  for (int64_t row = (int64_t)blockIdx.x * warps + warp; row < N; row += (int64_t)gridDim.x * warps) {
    const float* w = W + row * K;
    bool finite = true;
    for (int i = lane; i < P; i += 32) {
      if (i < K) {
        const float v = w[i];
        finite = finite && isfinite(v);
        sh.key[i] = fkey(v);
        sh.pos[i] = (uint16_t)i;
      } else {
        sh.key[i] = 0xffffffffu;  // padding sorts last
        sh.pos[i] = 0xffffu;
      }
    }
    if (__any_sync(0xffffffffu, !finite)) {
      for (int i = lane; i < K / 2; i += 32) idx[row * (K / 2) + i] = 0;
      if (lane < 16) lut[row * 16 + lane] = 0;
      if (lane == 0) atomicOr(status, QMV_FLAG_NONFINITE);
      __syncwarp();
      continue;
    }
    __syncwarp();
    // bitonic sort, ascending
    for (int size = 2; size <= P; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int t = lane; t < P / 2; t += 32) {
          const int i = 2 * t - (t & (stride - 1)), j = i + stride;
          const uint32_t ki = sh.key[i], kj = sh.key[j];
          const bool up = (i & size) == 0;
          if ((ki > kj) == up) {
            sh.key[i] = kj;
            sh.key[j] = ki;
            const uint16_t pi = sh.pos[i];
            sh.pos[i] = sh.pos[j];
            sh.pos[j] = pi;
          }
        }
        __syncwarp();
      }
    }
    // initial centres at the (k + 1/2)/16 quantiles
    double cj = 0.0;
    if (lane < 16) cj = (double)fkey_value(sh.key[((2 * lane + 1) * K) / 32]);
    for (int it = 0; it < iters; ++it) {
      int lo = 0, hi = 0;
      km_runs(sh, K, cj, lane, &lo, &hi);
      if (lane < 16 && hi > lo) {
        double sum = 0.0;
        for (int i = lo; i < hi; ++i) sum += (double)fkey_value(sh.key[i]);
        cj = (double)__double2float_rn(sum / (double)(hi - lo));
      }
      __syncwarp();
    }
    // palette, then each weight's nearest palette entry
    double cl = 0.0;
    if (lane < 16) {
      const __half h = __float2half_rn((float)cj);
      lut[row * 16 + lane] = __half_as_ushort(h);
      cl = (double)__half2float(h);
    }
    int lo = 0, hi = 0;
    const int nd = km_runs(sh, K, cl, lane, &lo, &hi);
    for (int i = lane; i < K; i += 32) {
      int r = 0;
      for (int q = 1; q < nd; ++q) r += (i >= sh.bnd[q]) ? 1 : 0;
      sh.ib[sh.pos[i]] = (uint8_t)sh.who[r];
    }
    __syncwarp();
    for (int i = lane; i < K / 2; i += 32)
      idx[row * (K / 2) + i] = (uint8_t)(sh.ib[2 * i] | (sh.ib[2 * i + 1] << 4));
    __syncwarp();
  }
}

int km_per_warp_bytes(int K) {
  int P = 1;
  while (P < K) P <<= 1;
  return ((6 * P + K + 15) & ~15) + 33 * 4 + 12;  // keys, positions, indices, runs
}

cudaError_t launch_encode_int4km(const float* W, int64_t N, int64_t K, int iters, uint16_t* lut, uint8_t* idx,
                                 uint32_t* status, int num_sms, cudaStream_t stream) {
  int P = 1;
  while (P < K) P <<= 1;
  const int per_warp = (km_per_warp_bytes((int)K) + 15) & ~15;
  int warps = (int)((200 * 1024) / per_warp);
  if (warps > 8) warps = 8;
  if (warps < 1) return cudaErrorInvalidValue;
  const size_t smem = (size_t)warps * per_warp;
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(km_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024 + 16 * 1024);
    if (err != cudaSuccess) return err;
    attr_set[dev].store(true, std::memory_order_release);
  }
  const int64_t want = (N + warps - 1) / warps;
  const int64_t cap = (int64_t)num_sms * 8;
  const int grid = (int)(want < cap ? want : cap);
  km_kernel<<<grid, 32 * warps, smem, stream>>>(W, N, (int)K, P, iters, lut, idx, status, warps, per_warp);
  return cudaGetLastError();
}

}  // namespace qmv
