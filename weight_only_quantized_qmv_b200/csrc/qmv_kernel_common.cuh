// qmv_kernel_common.cuh -- pieces shared by the matvec kernels (the block-
// quantized / palette kernel and the int8km kernel): small memory helpers,
// the column-group table of the gather over routed experts, the programmatic
// dependent launch controls and the fused-argmax epilogue.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

#include "qmv_device.cuh"
#include "qmv_internal.h"

namespace qmv {

__device__ __forceinline__ uint32_t lds_u8(uint32_t a) { return *sptr<uint8_t>(a); }
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) { return *sptr<uint16_t>(a); }
__device__ __forceinline__ void sts_u8(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u8 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void sts_u16(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"((unsigned short)v) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void sts_f32x2(uint32_t a, float u, float v) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(u), "f"(v) : "memory");
}
__device__ __forceinline__ uint4 ldg_nc_128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ uint8_t ldg_u8(const uint8_t* p) {
  uint32_t v;
  asm volatile("ld.global.nc.u8 %0, [%1];" : "=r"(v) : "l"(p));
  return (uint8_t)v;
}

__device__ __forceinline__ uint32_t ldg_u16(const uint16_t* p) {
  unsigned short v;
  asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
  return v;
}

// Paired fp32 arithmetic (two lanes of a 64-bit register, each element
// rounded as its scalar operation would be).
__device__ __forceinline__ uint64_t pack_f32x2(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ float2 unpack_f32x2(uint64_t v) {
  uint32_t lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
  return make_float2(__uint_as_float(lo), __uint_as_float(hi));
}
// per element: d = fma(a, b, c), round to nearest
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// per element: d = a - b, round to nearest
__device__ __forceinline__ uint64_t sub_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// The column of main in-feature j when the C columns in cols (ascending)
// are taken out: j + m, m = #{i : cols[i] - i <= j} (cols[i] - i, the main
// columns below outlier i, is non-decreasing).  The result is clamped to the
// row (width) so a malformed column list cannot address outside it.
__device__ __forceinline__ int64_t main_column(const int32_t* __restrict__ cols, int64_t C, int64_t j,
                                               int64_t width) {
  int64_t lo = 0, hi = C;
  while (lo < hi) {
    const int64_t mid = (lo + hi) >> 1;
    if ((int64_t)__ldg(cols + mid) - mid <= j) lo = mid + 1;
    else hi = mid;
  }
  const int64_t k = j + lo;
  return k < width ? k : width - 1;
}

// Programmatic dependent launch: let the next grid in the stream start, and
// wait for the preceding one to complete (its writes visible).
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void grid_wait_preceding() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Column groups: the activation rows served by one pass over one expert's
// weights (dense: one group of all B rows).
// ---------------------------------------------------------------------------
struct GroupTable {
  int ngroups;
  int expert[kMaxPairs];
  int start[kMaxPairs];
  int count[kMaxPairs];
  int16_t sorted[kMaxPairs];  // (token, slot) pair indices ordered by expert
};
// a kernel's static shared memory: the group table, the ids, a counter, the
// argmax keys
static_assert(sizeof(GroupTable) + kMaxPairs * sizeof(int) + kMaxCols * 8 + 32 <= kStaticSmem,
              "static shared memory reserve");

// Whole CTA (at least kMaxPairs threads), ends with a barrier: fills `gt`
// with groups of at most CAP pairs of one expert each (valid ids only, in
// expert order, stable), zeroes the output rows of pairs whose expert id is
// out of range (raising QMV_FLAG_BAD_EXPERT), and clears the argmax keys.
template <int CAP>
__device__ void setup_groups(const MvParams& p, GroupTable& gt, int* s_ids, int& s_nvalid,
                             unsigned long long* s_best, int tid) {
  const int P = p.gather ? p.B * p.topk : p.B;
  if (tid == 0) s_nvalid = 0;
  if (tid < kMaxCols) s_best[tid] = 0ull;
  if (p.gather && tid < P) s_ids[tid] = p.ids[tid];
  __syncthreads();
  if (!p.gather) {
    if (tid == 0) {
      gt.ngroups = 1;
      gt.expert[0] = 0;
      gt.start[0] = 0;
      gt.count[0] = p.B;
    }
    if (tid < P) gt.sorted[tid] = (int16_t)tid;
  } else if (tid < P) {
    const int e = s_ids[tid];
    if (e >= 0 && e < p.E) {
      int rank = 0;  // stable rank of this pair among valid pairs ordered by expert id
      for (int j = 0; j < P; ++j) {
        const int f = s_ids[j];
        rank += (f >= 0 && f < p.E && (f < e || (f == e && j < tid))) ? 1 : 0;
      }
      gt.sorted[rank] = (int16_t)tid;
      atomicAdd(&s_nvalid, 1);
    }
  }
  __syncthreads();
  if (p.gather) {
    if (tid == 0) {
      int ng = 0;
      for (int i = 0; i < s_nvalid; ++i) {
        const int e = s_ids[gt.sorted[i]];
        if (ng == 0 || gt.expert[ng - 1] != e || gt.count[ng - 1] == CAP) {
          gt.expert[ng] = e;
          gt.start[ng] = i;
          gt.count[ng] = 0;
          ++ng;
        }
        gt.count[ng - 1]++;
      }
      gt.ngroups = ng;
    }
    // a pair with an out-of-range expert id gets a zero output row (one CTA per pair)
    for (int q = 0; q < P; ++q) {
      const int e = s_ids[q];
      if ((e < 0 || e >= p.E) && (q % (int)gridDim.x) == (int)blockIdx.x) {
        if (tid == 0) atomicOr(p.status, QMV_FLAG_BAD_EXPERT);
        for (int64_t n = tid; n < p.N; n += blockDim.x) p.y[(int64_t)q * p.N + n] = 0.0f;
      }
    }
  }
  __syncthreads();  // the group table
}

// ---------------------------------------------------------------------------
// Fused argmax
// ---------------------------------------------------------------------------

// An output y[b, n] as a 64-bit key whose unsigned order is (value as a float
// with -0 == +0, then lower n first).
__device__ __forceinline__ unsigned long long argmax_key(float v, int64_t n) {
  const uint32_t u = __float_as_uint(v + 0.0f);  // -0 -> +0
  const uint32_t k = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return ((unsigned long long)k << 32) | (unsigned long long)(~(uint32_t)n);
}
__device__ __forceinline__ float argmax_key_value(unsigned long long key) {
  const uint32_t k = (uint32_t)(key >> 32);
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Whole CTA of KT threads, after the last output: each thread holds NS
// running maxima (best) of fixed activation rows (bcol, -1 if none); lanes
// of a warp with equal lane % 4 hold the same rows.  They combine per warp,
// then per CTA in s_best; the CTA's partials go to the workspace and the
// last CTA to finish (ticket) takes the maximum over all CTAs for each row,
// writes idx / val, and leaves the workspace zero-filled.
template <int NS, int KT>
__device__ void argmax_finish(const unsigned long long (&best)[NS], const int (&bcol)[NS], unsigned long long* s_best,
                              int& s_last, const MvParams& p, int tid, int lane) {
#pragma unroll
  for (int i = 0; i < NS; ++i) {
    unsigned long long k = best[i];
    int c = bcol[i];
#pragma unroll
    for (int m = 4; m < 32; m *= 2) {
      const unsigned long long k2 = __shfl_xor_sync(0xffffffffu, k, m);
      const int c2 = __shfl_xor_sync(0xffffffffu, c, m);
      k = k2 > k ? k2 : k;
      c = c2 > c ? c2 : c;
    }
    if (lane < 4 && c >= 0) atomicMax(&s_best[c], k);
  }
  __syncthreads();
  if (tid < p.B) p.am_part[(int64_t)blockIdx.x * kMaxCols + tid] = s_best[tid];
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(p.am_ticket, 1u) == gridDim.x - 1;
  __syncthreads();
  if (s_last) {
    // all threads: thread tid folds entries (CTA c, row tid % 16) -- the
    // stride is a multiple of 16 -- and the rows meet in s_best (which
    // already holds this CTA's own partials)
    __threadfence();
    const int b = tid & (kMaxCols - 1);
    const int nent = (int)gridDim.x * kMaxCols;
    unsigned long long mine = 0ull;
#pragma unroll 4
    for (int e = tid; e < nent; e += KT) {
      const unsigned long long k = __ldcg(p.am_part + e);
      mine = k > mine ? k : mine;
      p.am_part[e] = 0ull;  // the workspace is left zero-filled
    }
    if (b < p.B) atomicMax(&s_best[b], mine);
    __syncthreads();
    if (tid < p.B) {
      const unsigned long long v = s_best[tid];
      p.am_idx[tid] = (int32_t)(~(uint32_t)v);
      p.am_val[tid] = argmax_key_value(v);
    }
    if (tid == 0) *p.am_ticket = 0u;
  }
}

}  // namespace qmv
