// qmv_mixed.cu -- the mixed int4km + int8 outlier-column format: the choice
// of outlier columns, the column split of the weights for encoding, and the
// kernel that adds the outlier columns to the int4km kernel's output
// ("Stream D", next steps: a mixed int4 + int8-outlier matvec extending the
// int4km linear).  The int4km kernel itself stages the main columns of the
// activations (MvParams::xcols).
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

// y[b, n] += sum_c x[b, cols[c]] * q[n, c] * s[n, c / 32].  A thread takes
// one 32-column block of one row (GS threads per row, GS = the block count
// rounded up to a power of two): the exact products add in fp32, take the
// block's scale, and the row's threads combine their sums by a fixed
// shuffle tree.  The outlier activations of the B rows are staged as fp32
// in shared memory.  Dependent launch: it waits for the kernel that writes
// y (the int4km part) before reading anything.
constexpr int kAccThreads = 256;
constexpr int kAccMaxC = 512;  // outlier columns per launch (<= 16 blocks, <= 33 KB of staged activations)

// BT: a bound on the batch (1, 2, 4, 8 or 16), B <= BT; GS: threads per row
template <int BT, int GS>
__global__ void __launch_bounds__(kAccThreads) outlier_acc_kernel(const int8_t* __restrict__ q,
                                                                  const uint16_t* __restrict__ sc,
                                                                  const int32_t* __restrict__ cols,
                                                                  const uint16_t* __restrict__ x, int B, int64_t N,
                                                                  int64_t K, int64_t C, int64_t c0, int64_t cn,
                                                                  float* __restrict__ y) {
  // staged activations [B][cn / 32 blocks][33]: a block's 32 values plus one
  // pad word, so the GS threads of a row (one block each) read distinct banks
  extern __shared__ float xs[];
  const int64_t cst = (cn / 32) * 33;
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // y (and the step's inputs) complete
  for (int64_t i = threadIdx.x; i < (int64_t)B * cn; i += kAccThreads) {
    const int64_t b = i / cn, c = i - b * cn;
    int64_t col = cols[c0 + c];
    col = col < 0 ? 0 : (col >= K ? K - 1 : col);  // a malformed column list stays inside the row
    xs[b * cst + (c >> 5) * 33 + (c & 31)] = __half2float(__ushort_as_half(x[b * K + col]));
  }
  __syncthreads();
  const int blk = (int)(threadIdx.x % GS);
  // a grid-stride loop over the rows: the staged activations serve them all
  for (int64_t t0 = (int64_t)blockIdx.x * kAccThreads; t0 < N * GS; t0 += (int64_t)gridDim.x * kAccThreads) {
  const int64_t n = (t0 + threadIdx.x) / GS;
  float acc[BT];
#pragma unroll
  for (int b = 0; b < BT; ++b) acc[b] = 0.0f;
  if (n < N && 32 * blk < cn) {
    const int8_t* qr = q + n * C + c0 + 32 * blk;
#pragma unroll
    for (int v = 0; v < 2; ++v) {
      const uint4 w = *reinterpret_cast<const uint4*>(qr + 16 * v);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float qi = (float)(int8_t)(ws[i / 4] >> (8 * (i % 4)));
        const int c = 33 * blk + 16 * v + i;
#pragma unroll
        for (int b = 0; b < BT; ++b)
          if (b < B) acc[b] = fmaf(qi, xs[b * cst + c], acc[b]);
      }
    }
    const float s = __half2float(__ushort_as_half(sc[n * (C / 32) + (c0 / 32) + blk]));
#pragma unroll
    for (int b = 0; b < BT; ++b) acc[b] *= s;
  }
  // the row's GS threads are consecutive lanes: a fixed tree
#pragma unroll
  for (int o = 1; o < GS; o *= 2)
#pragma unroll
    for (int b = 0; b < BT; ++b) acc[b] += __shfl_xor_sync(0xffffffffu, acc[b], o);
  if (n < N && blk == 0) {
#pragma unroll
    for (int b = 0; b < BT; ++b)
      if (b < B) y[(int64_t)b * N + n] += acc[b];
  }
  }
}

template <int BT, int GS>
static cudaError_t launch_acc_t(const int8_t* q, const uint16_t* s, const int32_t* cols, const uint16_t* x, int B,
                                int64_t N, int64_t K, int64_t C, int64_t c0, int64_t cn, float* y, int num_sms,
                                cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  const int64_t want = (N * GS + kAccThreads - 1) / kAccThreads, cap = (int64_t)num_sms * 8;
  cfg.gridDim = dim3((unsigned)(want < cap ? want : cap));
  cfg.blockDim = dim3(kAccThreads);
  cfg.dynamicSmemBytes = (size_t)(4 * B * (cn / 32) * 33);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, outlier_acc_kernel<BT, GS>, q, s, cols, x, B, N, K, C, c0, cn, y);
}

template <int BT>
static cudaError_t launch_acc_b(const int8_t* q, const uint16_t* s, const int32_t* cols, const uint16_t* x, int B,
                                int64_t N, int64_t K, int64_t C, int64_t c0, int64_t cn, float* y, int num_sms,
                                cudaStream_t stream) {
  const int64_t nb = cn / 32;  // 1..16 blocks
  if (nb <= 1) return launch_acc_t<BT, 1>(q, s, cols, x, B, N, K, C, c0, cn, y, num_sms, stream);
  if (nb <= 2) return launch_acc_t<BT, 2>(q, s, cols, x, B, N, K, C, c0, cn, y, num_sms, stream);
  if (nb <= 4) return launch_acc_t<BT, 4>(q, s, cols, x, B, N, K, C, c0, cn, y, num_sms, stream);
  if (nb <= 8) return launch_acc_t<BT, 8>(q, s, cols, x, B, N, K, C, c0, cn, y, num_sms, stream);
  return launch_acc_t<BT, 16>(q, s, cols, x, B, N, K, C, c0, cn, y, num_sms, stream);
}

cudaError_t launch_outlier_acc(const int8_t* q, const uint16_t* s, const int32_t* cols, const uint16_t* x, int B,
                               int64_t N, int64_t K, int64_t C, float* y, int num_sms, cudaStream_t stream) {
  for (int64_t c0 = 0; c0 < C; c0 += kAccMaxC) {
    const int64_t cn = C - c0 < kAccMaxC ? C - c0 : kAccMaxC;
    const cudaError_t e =
        B <= 1 ? launch_acc_b<1>(q, s, cols, x, B, N, K, C, c0, cn, y, num_sms, stream)
        : B <= 2 ? launch_acc_b<2>(q, s, cols, x, B, N, K, C, c0, cn, y, num_sms, stream)
        : B <= 4 ? launch_acc_b<4>(q, s, cols, x, B, N, K, C, c0, cn, y, num_sms, stream)
        : B <= 8 ? launch_acc_b<8>(q, s, cols, x, B, N, K, C, c0, cn, y, num_sms, stream)
                 : launch_acc_b<16>(q, s, cols, x, B, N, K, C, c0, cn, y, num_sms, stream);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
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


}  // namespace qmv
