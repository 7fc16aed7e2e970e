// qmv_km8.cu -- fused lookup + matvec for int8km (8-bit k-means palettes):
// y[b, n] = sum_k x[b, k] * LUT[n / 32][idx[n, k]], one 256-entry fp16 LUT per
// group of 32 output rows ("coreai-optimization (coreai-opt) reference",
// "Palettization": per-grouped-channel LUTs of 2^n_bits entries;
// "Compression (palettization & quantization)", "int8 k-means > whole-model
// int4": 8-bit k-means with group 32; "Stream D", sec. 1: int8km among the
// gather formats).  Dense and routed-expert gather, optional fused argmax.
//
// Design (sm_100a):
//  * A CTA works on one 32-row group at a time (a "unit"), so one LUT serves
//    all of its warps.  K is cut into 8 parts of whole 64-wide chunks; warp w
//    takes row tile w % 2 (16 rows) and 1 (16 warps) or 2 (8 warps) of the
//    parts, and the 8 partial sums meet in shared memory in part order, so a
//    result does not depend on the CTA size.
//  * The unit's LUT is written to shared memory with each entry repeated in
//    all 32 banks (word e * 32 + lane), so the lookup of lane l reads bank l:
//    one conflict-free 32-bit load per weight whatever the indices.
//  * Index bytes go from global memory straight to registers (one 16-byte
//    load per row and chunk, one chunk ahead); the next unit's index rows are
//    prefetched into L2 (128-byte lines, spread over the CTA's threads)
//    while this one is computed.
//  * The looked-up fp16 values form the m16n8k16 A fragments directly: lane
//    (g, t) owns in-features 16t..16t+15 of a chunk, word s of its bytes is
//    the A operand of MMA step s, so the activations stay in natural order.
#include <cstdint>
#include <cuda_fp16.h>

#include "qmv_device.cuh"
#include "qmv_internal.h"
#include "qmv_kernel_common.cuh"

namespace qmv {

__device__ __forceinline__ uint4 ldg_stream_128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
// L2 prefetch of the line holding p
__device__ __forceinline__ void prefetch_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// Lookup of byte J of w in the replicated table (tab_l = table + 4 * lane):
// the entry's fp16 value in both halves of the returned word.
template <int J>
__device__ __forceinline__ uint32_t km8_lookup(uint32_t w, uint32_t tab_l) {
  const uint32_t c = (J == 3) ? (w >> 24) : prmt(w, 0u, 0x4440u + J);
  return lds32(tab_l + (c << 7));
}
// the A operand pair (byte J, byte J + 1) of w: low half from J
template <int J>
__device__ __forceinline__ uint32_t km8_pair(uint32_t w, uint32_t tab_l) {
  return prmt(km8_lookup<J>(w, tab_l), km8_lookup<J + 1>(w, tab_l), 0x5410u);
}

// NT: activation n-tiles of 8 columns (1 or 2).  WARPS: 8 (two CTAs per SM)
// or 16 (one CTA per SM, when the staged activations are large).
template <int NT, int WARPS, bool AM>
__global__ void __launch_bounds__(32 * WARPS, WARPS == 8 ? 2 : 1) km8_kernel(const __grid_constant__ MvParams p) {
  constexpr int kT = 32 * WARPS;
  constexpr int KP = 8;                 // K parts per unit
  constexpr int PPW = KP / (WARPS / 2);  // parts per warp
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ GroupTable gt;
  __shared__ int s_ids[kMaxPairs];
  __shared__ int s_nvalid;
  __shared__ unsigned long long s_best[kMaxCols];
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t sbase = smem_addr(smem);
  const uint32_t tab = sbase + p.off_tab;  // [256][32] words
  const uint32_t tab_l = tab + 4u * (uint32_t)lane;
  const uint32_t xbase = sbase + p.off_x;
  float* red = reinterpret_cast<float*>(smem + p.off_red);  // [KP][2 tiles][NT][4][32]
  const int64_t K = p.K;
  const int64_t G = p.tiles;  // row groups of 32

  grid_launch_dependents();
  if (!p.prefetch) grid_wait_preceding();
  setup_groups<8 * NT>(p, gt, s_ids, s_nvalid, s_best, tid);
  const int ngroups = gt.ngroups;
  const int64_t total = (int64_t)ngroups * G;

  // a unit's index rows: expert e, rows [32 rg, min(32 rg + 32, N))
  auto unit_codes = [&](int64_t u, int64_t& rg, int& grp, const uint8_t*& base, int& nrows) {
    if (ngroups == 1) {
      grp = 0;
      rg = u;
    } else {
      grp = (int)(u / G);
      rg = u - (int64_t)grp * G;
    }
    base = p.codes + (int64_t)gt.expert[grp] * p.expert_code_bytes + rg * 32 * K;
    nrows = (int)min((int64_t)32, p.N - rg * 32);
  };
  auto prefetch_unit = [&](int64_t u) {  // whole CTA; at most 256 KB
    int64_t rg;
    int grp, nrows;
    const uint8_t* base;
    unit_codes(u, rg, grp, base, nrows);
    const int64_t bytes = min((int64_t)nrows * K, (int64_t)1 << 18);
    for (int64_t off = 128 * (int64_t)tid; off < bytes; off += 128 * kT) prefetch_l2(base + off);
  };
  if ((int64_t)blockIdx.x < total) prefetch_unit(blockIdx.x);  // weights only

  if (p.prefetch) grid_wait_preceding();
  // activations in natural order, each row zero-padded to whole 64-wide chunks
  {
    const int64_t per_row = p.XS / 16;  // 16-byte pieces of a staged row
    const int64_t k16 = K / 8;          // pieces holding activations
    const int64_t n16 = (int64_t)p.n_xrows * per_row;
    for (int64_t i = tid; i < n16; i += kT) {
      const int64_t r = i / per_row, j = i - r * per_row;
      const uint4 v = j < k16 ? ldg_nc_128(p.x + r * K + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
      sts128(xbase + (uint32_t)(r * p.XS + 16 * j), v);
    }
  }

  const int tile = warp & 1;
  const int64_t nch = (K + 63) / 64;

  unsigned long long best[NT];
  int bcol[NT];
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    best[i] = 0ull;
    bcol[i] = -1;
  }

  for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
    int64_t rg;
    int grp, nrows;
    const uint8_t* ubase;
    unit_codes(u, rg, grp, ubase, nrows);
    const int ncols = gt.count[grp], gstart = gt.start[grp];

    // ---- the unit's LUT, replicated across the banks ----
    __syncthreads();  // the previous unit's lookups and partial sums are done (and the staged activations)
    {
      constexpr int EPW = 256 / WARPS;  // entries per warp
      const uint16_t* lut = reinterpret_cast<const uint16_t*>(p.aux + (int64_t)gt.expert[grp] * p.expert_aux_bytes) +
                            rg * 256;
      uint32_t v = 0u;
      if (lane < EPW) {
        const uint32_t h = lut[warp * EPW + lane];
        v = h | (h << 16);
      }
#pragma unroll
      for (int j = 0; j < EPW / 4; ++j) {
        // rows 4j .. 4j+3 of this warp's entries, 8 lanes x 16 bytes per row
        const int r = 4 * j + (lane >> 3);
        const uint32_t w = __shfl_sync(0xffffffffu, v, r);
        sts128(tab + (uint32_t)(warp * EPW + r) * 128u + 16u * (uint32_t)(lane & 7), make_uint4(w, w, w, w));
      }
    }
    if (u + (int64_t)gridDim.x < total) prefetch_unit(u + gridDim.x);
    __syncthreads();

    // ---- this warp's rows and K part ----
    const int rgi = tile * 16 + g;  // row g of the tile within the unit
    const uint8_t* row_g = ubase + (int64_t)min(rgi, nrows - 1) * K + 16 * t;
    const uint8_t* row_h = ubase + (int64_t)min(rgi + 8, nrows - 1) * K + 16 * t;
    uint32_t xa[NT];
    bool xon[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int col = 8 * n + g;
      xon[n] = col < ncols;
      int xrow = 0;
      if (xon[n]) {
        const int pair = gt.sorted[gstart + col];
        xrow = p.gather ? (p.x_per_slot ? pair : pair / p.topk) : pair;
      }
      xa[n] = xbase + (uint32_t)xrow * p.XS + 32u * (uint32_t)t;
    }
    // this warp's parts are contiguous in K: chunks [cA, cB), one chunk ahead
    const int kp0 = (warp >> 1) * PPW;
    const int64_t cA = kp0 * nch / KP, cB = (kp0 + PPW) * nch / KP;
    uint4 cg = make_uint4(0u, 0u, 0u, 0u), ch = cg;
    if (cA < cB && 64 * cA + 16 * t < K) {
      cg = ldg_stream_128(row_g + 64 * cA);
      ch = ldg_stream_128(row_h + 64 * cA);
    }
#pragma unroll 1
    for (int part = 0; part < PPW; ++part) {
      const int kp = kp0 + part;
      const int64_t c0 = kp * nch / KP, c1 = (kp + 1) * nch / KP;
      float acc[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[n][q] = 0.0f;

      for (int64_t c = c0; c < c1; ++c) {
        uint4 ng = make_uint4(0u, 0u, 0u, 0u), nh = ng;
        if (c + 1 < cB && 64 * (c + 1) + 16 * t < K) {
          ng = ldg_stream_128(row_g + 64 * (c + 1));
          nh = ldg_stream_128(row_h + 64 * (c + 1));
        }
        const bool live = 64 * c + 16 * t < K;  // in-features past K (a last half chunk) stay zero
        uint4 xr0[NT], xr1[NT];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          xr0[n] = make_uint4(0u, 0u, 0u, 0u);
          xr1[n] = xr0[n];
          if (xon[n]) {
            xr0[n] = lds128(xa[n] + 128u * (uint32_t)c);
            xr1[n] = lds128(xa[n] + 128u * (uint32_t)c + 16u);
          }
        }
        const uint32_t wg[4] = {cg.x, cg.y, cg.z, cg.w}, wh[4] = {ch.x, ch.y, ch.z, ch.w};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          uint32_t a0 = 0u, a1 = 0u, a2 = 0u, a3 = 0u;
          if (live) {
            a0 = km8_pair<0>(wg[s], tab_l);
            a2 = km8_pair<2>(wg[s], tab_l);
            a1 = km8_pair<0>(wh[s], tab_l);
            a3 = km8_pair<2>(wh[s], tab_l);
          }
#pragma unroll
          for (int n = 0; n < NT; ++n) {
            const uint32_t b0 = s == 0 ? xr0[n].x : s == 1 ? xr0[n].z : s == 2 ? xr1[n].x : xr1[n].z;
            const uint32_t b1 = s == 0 ? xr0[n].y : s == 1 ? xr0[n].w : s == 2 ? xr1[n].y : xr1[n].w;
            mma16816(acc[n], a0, a1, a2, a3, b0, b1);
          }
        }
        cg = ng;
        ch = nh;
      }
      // this part's partial sums
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) red[(((kp * 2 + tile) * NT + n) * 4 + q) * 32 + lane] = acc[n][q];
    }

    // ---- the K parts meet in shared memory, in order ----
    __syncthreads();
    if (tid < 256) {
      // thread: tile tid / 128, accumulator q, lane ln; its column of n-tile n is 8n + 2(ln % 4) + q % 2
      const int tl = tid >> 7, q = (tid >> 5) & 3, ln = tid & 31;
      const int row = tl * 16 + (ln >> 2) + 8 * (q >> 1);
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        float v = 0.0f;
#pragma unroll
        for (int k = 0; k < KP; ++k) v += red[(((2 * k + tl) * NT + n) * 4 + q) * 32 + ln];  // part order
        const int col = 8 * n + 2 * (ln & 3) + (q & 1);
        if (col < ncols && row < nrows) {
          const int pair = gt.sorted[gstart + col];
          const int64_t nrow = rg * 32 + row;
          if constexpr (AM) {
            const unsigned long long key = argmax_key(v, nrow);
            best[n] = key > best[n] ? key : best[n];
            bcol[n] = pair;
          } else {
            p.y[(int64_t)pair * p.N + nrow] = v;
          }
        }
      }
    }
  }

  if constexpr (AM) argmax_finish<NT, kT>(best, bcol, s_best, s_last, p, tid, lane);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

static int64_t round_up8(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

bool plan_km8(MvParams& p, int num_sms) {
  p.code_row_bytes = p.K;
  p.aux_row_bytes = 0;
  p.tiles = (p.N + 31) / 32;  // row groups
  p.expert_code_bytes = p.N * p.K;
  p.expert_aux_bytes = p.tiles * 512;
  // staged activation rows: natural order, whole 64-wide chunks, the row
  // stride at 16 mod 128 bytes so the 16-byte reads of 8 lanes (two rows,
  // four in-feature quarters) fall in distinct banks
  p.XS = (int)(round_up8(2 * round_up8(p.K, 64), 128) + 16);
  p.n_xrows = p.gather ? (p.x_per_slot ? p.B * p.topk : p.B) : p.B;
  const int nt = p.B > 8 ? 2 : 1;
  const int64_t units = (p.gather ? (int64_t)p.B * p.topk : 1) * p.tiles;
  const int64_t dyn_limit = (int64_t)kSmemLimit - kStaticSmem;
  const int cand[2][2] = {{8, 2}, {16, 1}};
  for (int ci = 0; ci < 2; ++ci) {
    const int warps = cand[ci][0], ctas = cand[ci][1];
    p.warps = warps;
    p.off_tab = 0;  // 32 KB
    p.off_red = 256 * 128;
    p.off_x = (int)round_up8(p.off_red + (int64_t)8 * 2 * nt * 4 * 32 * 4, 128);  // 8 parts x 2 tiles
    const int64_t bytes = p.off_x + (int64_t)p.n_xrows * p.XS;
    if (bytes <= dyn_limit && ctas * (bytes + kStaticSmem + 1024) <= kSmemPerSM) {
      p.smem_bytes = (int)bytes;
      p.ctas_per_sm = ctas;
      const int64_t slots = (int64_t)num_sms * ctas;
      p.grid = (int)(units < slots ? units : slots);
      return true;
    }
  }
  return false;
}

template <int NT, int WARPS, bool AM>
static cudaError_t launch_km8_t(const MvParams& p, cudaStream_t stream) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && !attr_set[dev]) {
    err = cudaFuncSetAttribute(km8_kernel<NT, WARPS, AM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemLimit - kStaticSmem);
    if (err != cudaSuccess) return err;
    attr_set[dev] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.grid);
  cfg.blockDim = dim3(32 * WARPS);
  cfg.dynamicSmemBytes = (size_t)p.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, km8_kernel<NT, WARPS, AM>, p);
}

template <bool AM>
static cudaError_t launch_km8_a(const MvParams& p, cudaStream_t stream) {
  const bool wide = p.warps == 16;
  if (p.B > 8) return wide ? launch_km8_t<2, 16, AM>(p, stream) : launch_km8_t<2, 8, AM>(p, stream);
  return wide ? launch_km8_t<1, 16, AM>(p, stream) : launch_km8_t<1, 8, AM>(p, stream);
}

cudaError_t launch_km8(const MvParams& p, cudaStream_t stream) {
  return p.argmax ? launch_km8_a<true>(p, stream) : launch_km8_a<false>(p, stream);
}

}  // namespace qmv
