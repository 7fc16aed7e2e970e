// qmv_mixed.cu -- the mixed int4km + int8 outlier-column format: the choice
// of outlier columns, the column splits of weights and activations, and
// the launchers that compose the int4km and int8 kernels ("Stream D", next
// steps: a mixed int4 + int8-outlier matvec extending the int4km linear).
//
// Format (the pages leave it open; the reading taken): the C input columns
// (C % 32 == 0, C < K) with the largest max |w| (Inf/NaN the largest, ties
// to the lower column) are stored as symmetric int8 with per-block-32 fp16
// scales along the outlier columns; the remaining K - C columns, in
// ascending order, form an int4km matrix.  y = x_main Wmain^T + x_out Wout^T.
#include <cstdint>
#include <cuda_fp16.h>

#include "qmv_internal.h"

namespace qmv {

// |w| as an order-preserving integer for non-negative floats; NaN counts as +Inf
__device__ __forceinline__ int abs_key(float w) {
  const float a = fabsf(w);
  return isnan(a) ? 0x7f800000 : __float_as_int(a);
}

__global__ void colmax_zero_kernel(int* m, int64_t K) {
  for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < K; k += (int64_t)gridDim.x * blockDim.x)
    m[k] = 0;
}

// column maxima of |W| over row stripes (atomic max of the integer keys)
__global__ void colmax_kernel(const float* __restrict__ W, int64_t N, int64_t K, int64_t rows_per_block, int* m) {
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const int64_t r0 = (int64_t)blockIdx.y * rows_per_block;
  const int64_t r1 = min(N, r0 + rows_per_block);
  int best = 0;
  for (int64_t n = r0; n < r1; ++n) best = max(best, abs_key(W[n * K + k]));
  atomicMax(&m[k], best);
}

// flag[k] = 1 when fewer than C columns outrank k (a larger maximum, or an
// equal one at a lower column)
__global__ void colrank_kernel(const int* __restrict__ m, int64_t K, int64_t C, int* flag) {
  __shared__ int tile[1024];
  const int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int mk = k < K ? m[k] : 0;
  int64_t rank = 0;
  for (int64_t j0 = 0; j0 < K; j0 += 1024) {
    __syncthreads();
    if (j0 + threadIdx.x < K) tile[threadIdx.x] = m[j0 + threadIdx.x];
    __syncthreads();
    const int jn = (int)min((int64_t)1024, K - j0);
    for (int j = 0; j < jn; ++j) {
      const int mj = tile[j];
      rank += (mj > mk || (mj == mk && j0 + j < k)) ? 1 : 0;
    }
  }
  if (k < K) flag[k] = rank < C ? 1 : 0;
}

// one CTA of 1024 threads: the flagged columns, ascending
__global__ void colcompact_kernel(const int* __restrict__ flag, int64_t K, int32_t* cols) {
  __shared__ int warp_sum[32];
  __shared__ int64_t base;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) base = 0;
  __syncthreads();
  for (int64_t k0 = 0; k0 < K; k0 += 1024) {
    const int64_t k = k0 + tid;
    const int f = k < K ? flag[k] : 0;
    int v = f;  // inclusive scan in the warp
#pragma unroll
    for (int o = 1; o < 32; o *= 2) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane == 31) warp_sum[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int s = warp_sum[lane];
#pragma unroll
      for (int o = 1; o < 32; o *= 2) {
        const int u = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += u;
      }
      warp_sum[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    const int64_t pos = base + (warp > 0 ? warp_sum[warp - 1] : 0) + v - f;
    if (f) cols[pos] = (int32_t)k;
    __syncthreads();
    if (tid == 0) base += warp_sum[31];
    __syncthreads();
  }
}

// position of column k among the main columns, or -(1 + its outlier index)
__device__ __forceinline__ int64_t split_pos(const int32_t* __restrict__ cols, int64_t C, int64_t k) {
  int64_t lo = 0, hi = C;  // lo = number of outlier columns below k
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    if (cols[mid] < k) lo = mid + 1;
    else hi = mid;
  }
  if (lo < C && cols[lo] == k) return -(1 + lo);
  return k - lo;
}

template <typename T>
__global__ void split_kernel(const T* __restrict__ src, int64_t R, int64_t K, const int32_t* __restrict__ cols,
                             int64_t C, T* __restrict__ main_out, T* __restrict__ out_out) {
  const int64_t total = R * K, M = K - C;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / K, k = i - r * K;
    const int64_t pos = split_pos(cols, C, k);
    if (pos >= 0) main_out[r * M + pos] = src[i];
    else out_out[r * C + (-pos - 1)] = src[i];
  }
}

static int grid_for_n(int64_t n, int threads, int num_sms) {
  const int64_t b = (n + threads - 1) / threads;
  const int64_t cap = (int64_t)num_sms * 16;
  return (int)(b < 1 ? 1 : (b < cap ? b : cap));
}

cudaError_t launch_outlier_columns(const float* W, int64_t N, int64_t K, int64_t C, int32_t* cols, int* ws,
                                   int num_sms, cudaStream_t stream) {
  int* m = ws;
  int* flag = ws + K;
  colmax_zero_kernel<<<grid_for_n(K, 256, num_sms), 256, 0, stream>>>(m, K);
  const int64_t stripes = (int64_t)num_sms * 8;
  const int64_t rpb = (N + stripes - 1) / stripes;
  colmax_kernel<<<dim3((unsigned)((K + 255) / 256), (unsigned)((N + rpb - 1) / rpb)), 256, 0, stream>>>(W, N, K, rpb, m);
  colrank_kernel<<<(unsigned)((K + 1023) / 1024), 1024, 0, stream>>>(m, K, C, flag);
  colcompact_kernel<<<1, 1024, 0, stream>>>(flag, K, cols);
  return cudaGetLastError();
}

cudaError_t launch_split_f32(const float* W, int64_t N, int64_t K, const int32_t* cols, int64_t C, float* Wmain,
                             float* Wout, int num_sms, cudaStream_t stream) {
  split_kernel<float><<<grid_for_n(N * K, 256, num_sms), 256, 0, stream>>>(W, N, K, cols, C, Wmain, Wout);
  return cudaGetLastError();
}

cudaError_t launch_split_f16(const uint16_t* x, int64_t B, int64_t K, const int32_t* cols, int64_t C,
                             uint16_t* xmain, uint16_t* xout, int num_sms, cudaStream_t stream) {
  split_kernel<uint16_t><<<grid_for_n(B * K, 256, num_sms), 256, 0, stream>>>(x, B, K, cols, C, xmain, xout);
  return cudaGetLastError();
}

}  // namespace qmv
