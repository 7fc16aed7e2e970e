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
//    all 32 banks, so the lookup of lane l reads bank l: one conflict-free
//    32-bit load per weight whatever the indices.  Two table buffers: the
//    next unit's LUT is written while this one is read.
//  * Index bytes go from global memory straight to registers (16-byte loads,
//    one chunk ahead, across unit boundaries).  Explicit L2 prefetches of
//    the next units' rows (line or bulk) measured slower and are not used.
//  * The looked-up fp16 values form the m16n8k16 A fragments directly: lane
//    (g, t) owns in-features 16t..16t+15 of a chunk, word s of its bytes is
//    the A operand of MMA step s, so the activations stay in natural order.
#include <atomic>
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

// The LUT table: 256 rows of 256 bytes at the start of the dynamic shared
// memory; row c holds entry c of buffer 0 in words 0..31 and of buffer 1 in
// words 32..63 (each word: the fp16 value in both halves).  A lookup's byte
// offset c * 256 + buffer * 128 + lane * 4 is one byte permute of the index
// byte and lb = buffer * 128 + lane * 4, and the table's base is a constant,
// so a lookup is one permute and one conflict-free 32-bit shared load.
extern __shared__ __align__(1024) uint8_t km8_smem[];

template <int J>
__device__ __forceinline__ uint32_t km8_lookup(uint32_t w, uint32_t lb, uint32_t tb) {
  const uint32_t off = prmt(w, lb, 0x5504u + 16u * J);  // bytes: lb.0, w.J, 0, 0
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(tb + off));  // tb: the table's shared address
  return v;
}
// the A operand pair (byte J, byte J + 1) of w: low half from J
template <int J>
__device__ __forceinline__ uint32_t km8_pair(uint32_t w, uint32_t lb, uint32_t tb) {
  return prmt(km8_lookup<J>(w, lb, tb), km8_lookup<J + 1>(w, lb, tb), 0x5410u);
}

// One 64-wide chunk of a warp's rows g, g+8 (index words cg, ch of this
// lane's 16 in-features) against the staged activations xa[n] + 128 c.
// PARTIAL: the chunk ends at K after 32 in-features; lanes t >= 2 hold no
// weights and contribute exact zeros.
template <int NT, bool PARTIAL>
__device__ __forceinline__ void km8_chunk(float (&acc)[NT][4], const uint4& cg, const uint4& ch, const uint32_t (&xa)[NT],
                                          const bool (&xon)[NT], int64_t c, uint32_t lb, uint32_t tb, int t) {
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
    uint32_t a0 = km8_pair<0>(wg[s], lb, tb), a2 = km8_pair<2>(wg[s], lb, tb);
    uint32_t a1 = km8_pair<0>(wh[s], lb, tb), a3 = km8_pair<2>(wh[s], lb, tb);
    if (PARTIAL && t >= 2) a0 = a1 = a2 = a3 = 0u;
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const uint32_t b0 = s == 0 ? xr0[n].x : s == 1 ? xr0[n].z : s == 2 ? xr1[n].x : xr1[n].z;
      const uint32_t b1 = s == 0 ? xr0[n].y : s == 1 ? xr0[n].w : s == 2 ? xr1[n].y : xr1[n].w;
      mma16816(acc[n], a0, a1, a2, a3, b0, b1);
    }
  }
}

// NT: activation n-tiles of 8 columns (1 or 2).  WARPS: 8 (two CTAs per SM)
// or 16 (one CTA per SM, when the staged activations are large).  Dense
// batch 1 runs km8b1_kernel below, unless its fp32 activation row does not
// fit (then this kernel, with B = 1 as one column).
//
// Per unit, with one barrier: the next unit's LUT entries are requested at
// the start (registers) and written to the other table buffer at the end;
// the partial sums alternate between two buffers (one buffer and a second
// barrier where shared memory is short); a warp's index loads run one chunk
// ahead straight across unit boundaries.
template <int NT, int WARPS, bool AM>
__global__ void __launch_bounds__(32 * WARPS, WARPS == 8 ? 2 : 1) km8_kernel(const __grid_constant__ MvParams p) {
  constexpr int kT = 32 * WARPS;
  constexpr int KP = 8;                  // K parts per unit
  constexpr int PPW = KP / (WARPS / 2);  // parts per warp
  constexpr int NTX = NT;
  constexpr int EPW = 256 / WARPS;       // LUT entries per warp in a table build
  constexpr int kRedFloats = KP * 2 * NTX * 4 * 32;  // one partial-sum buffer
  __shared__ GroupTable gt;
  __shared__ int s_ids[kMaxPairs];
  __shared__ int s_nvalid;
  __shared__ unsigned long long s_best[kMaxCols];
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t sbase = smem_addr(km8_smem);  // the LUT table: [256][2 buffers][32] words
  const uint32_t xbase = sbase + p.off_x;
  // partial sums, two buffers of [KP][2 tiles][NT][4][32]
  float* red0 = reinterpret_cast<float*>(km8_smem + p.off_red);
  const int64_t K = p.K;
  const int64_t G = p.tiles;  // row groups of 32

  grid_launch_dependents();
  if (!p.prefetch) grid_wait_preceding();
  setup_groups<8 * NTX>(p, gt, s_ids, s_nvalid, s_best, tid);
  const int ngroups = gt.ngroups;
  const int64_t total = (int64_t)ngroups * G;
  const int64_t grid = gridDim.x;

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
  // this thread's LUT entry of unit u (lanes < EPW), in the table's word format
  auto lut_entry = [&](int64_t u) -> uint32_t {
    int64_t rg;
    int grp, nrows;
    const uint8_t* base;
    unit_codes(u, rg, grp, base, nrows);
    const uint16_t* lut =
        reinterpret_cast<const uint16_t*>(p.aux + (int64_t)gt.expert[grp] * p.expert_aux_bytes) + rg * 256;
    uint32_t v = 0u;
    if (lane < EPW) {
      const uint32_t h = lut[warp * EPW + lane];
      v = h | (h << 16);
    }
    return v;
  };
  // whole CTA: the entries (from lut_entry) into table buffer b
  auto write_table = [&](uint32_t v, int b) {
#pragma unroll
    for (int j = 0; j < EPW / 4; ++j) {
      // rows 4j .. 4j+3 of this warp's entries, 8 lanes x 16 bytes per row
      const int r = 4 * j + (lane >> 3);
      const uint32_t w = __shfl_sync(0xffffffffu, v, r);
      sts128(sbase + (uint32_t)(warp * EPW + r) * 256u + 128u * (uint32_t)b + 16u * (uint32_t)(lane & 7),
             make_uint4(w, w, w, w));
    }
  };
  const int tile = warp & 1;
  const int nch = (int)((K + 63) / 64);
  const int kp0 = (warp >> 1) * PPW;
  const int cA = kp0 * nch / KP, cB = (kp0 + PPW) * nch / KP;  // this warp's chunks, every unit
  const int rgi = tile * 16 + g;  // row g of this warp's tile within a unit

  // the first chunk of this warp in unit u (zero where past K)
  auto first_chunk = [&](int64_t u, uint4& cg, uint4& ch) {
    cg = make_uint4(0u, 0u, 0u, 0u);
    ch = cg;
    if (u < total && cA < cB && 64 * (int64_t)cA + 16 * t < K) {
      int64_t rg;
      int grp, nrows;
      const uint8_t* base;
      unit_codes(u, rg, grp, base, nrows);
      cg = ldg_stream_128(base + (int64_t)min(rgi, nrows - 1) * K + 64 * cA + 16 * t);
      ch = ldg_stream_128(base + (int64_t)min(rgi + 8, nrows - 1) * K + 64 * cA + 16 * t);
    }
  };
  // weights only before the wait (early weight reads): the first index chunk and LUT entries
  uint4 cg, ch;
  first_chunk(blockIdx.x, cg, ch);
  const uint32_t lut0 = (int64_t)blockIdx.x < total ? lut_entry(blockIdx.x) : 0u;

  if (p.prefetch) grid_wait_preceding();
  {
    // activations in natural order, each row zero-padded to whole 64-wide chunks
    const int64_t per_row = p.XS / 16;  // 16-byte pieces of a staged row
    const int64_t k16 = K / 8;          // pieces holding activations
    const int64_t n16 = (int64_t)p.n_xrows * per_row;
    for (int64_t i = tid; i < n16; i += kT) {
      const int64_t r = i / per_row, j = i - r * per_row;
      const uint4 v = j < k16 ? ldg_nc_128(p.x + r * K + 8 * j) : make_uint4(0u, 0u, 0u, 0u);
      sts128(xbase + (uint32_t)(r * p.XS + 16 * j), v);
    }
  }
  if ((int64_t)blockIdx.x < total) write_table(lut0, 0);
  __syncthreads();  // the first table and the activations

  unsigned long long best[NTX];
  int bcol[NTX];
#pragma unroll
  for (int i = 0; i < NTX; ++i) {
    best[i] = 0ull;
    bcol[i] = -1;
  }

  int buf = 0;
  for (int64_t u = blockIdx.x; u < total; u += grid, buf ^= 1) {
    int64_t rg;
    int grp, nrows;
    const uint8_t* ubase;
    unit_codes(u, rg, grp, ubase, nrows);
    const int ncols = gt.count[grp], gstart = gt.start[grp];
    const bool has_next = u + grid < total;
    float* red = red0 + (p.red_bufs == 2 ? buf : 0) * kRedFloats;
    if (p.red_bufs == 1) __syncthreads();  // one partial-sum buffer: the previous unit's sums have been read

    // the next unit's LUT entries, written to the other buffer after this unit's lookups
    const uint32_t lutv = has_next ? lut_entry(u + grid) : 0u;

    const uint8_t* row_g = ubase + (int64_t)min(rgi, nrows - 1) * K + 16 * t;
    const uint8_t* row_h = ubase + (int64_t)min(rgi + 8, nrows - 1) * K + 16 * t;
    const uint32_t lb = 128u * (uint32_t)buf + 4u * (uint32_t)lane;
    uint32_t xa[NTX];
    bool xon[NTX];
#pragma unroll
    for (int n = 0; n < NTX; ++n) {
      const int col = 8 * n + g;
      xon[n] = col < ncols;
      int xrow = 0;
      if (xon[n]) {
        const int pair = gt.sorted[gstart + col];
        xrow = p.gather ? (p.x_per_slot ? pair : pair / p.topk) : pair;
      }
      xa[n] = xbase + (uint32_t)xrow * p.XS + 32u * (uint32_t)t;
    }

#pragma unroll 1
    for (int part = 0; part < PPW; ++part) {
      const int kp = kp0 + part;
      const int c0 = kp * nch / KP, c1 = (kp + 1) * nch / KP;
      float acc[NTX][4];
#pragma unroll
      for (int n = 0; n < NTX; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[n][q] = 0.0f;
      for (int c = c0; c < c1; ++c) {
        // the next chunk: this unit's, or the next unit's first
        uint4 ng, nh;
        if (c + 1 < cB) {
          ng = make_uint4(0u, 0u, 0u, 0u);
          nh = ng;
          if (64 * (int64_t)(c + 1) + 16 * t < K) {
            ng = ldg_stream_128(row_g + 64 * (int64_t)(c + 1));
            nh = ldg_stream_128(row_h + 64 * (int64_t)(c + 1));
          }
        } else {
          first_chunk(u + grid, ng, nh);
        }
        if (64 * (int64_t)c + 64 <= K)
          km8_chunk<NTX, false>(acc, cg, ch, xa, xon, c, lb, sbase, t);
        else
          km8_chunk<NTX, true>(acc, cg, ch, xa, xon, c, lb, sbase, t);
        cg = ng;
        ch = nh;
      }
#pragma unroll
      for (int n = 0; n < NTX; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) red[(((kp * 2 + tile) * NTX + n) * 4 + q) * 32 + lane] = acc[n][q];
    }
    if (cA >= cB) first_chunk(u + grid, cg, ch);  // (no chunks: nothing was loaded ahead)

    // The next unit's LUT into the other buffer (its last reader, the
    // previous unit, passed the previous barrier), then one barrier: this
    // unit's partial sums and the next table are complete.
    if (has_next) write_table(lutv, buf ^ 1);
    __syncthreads();

    // ---- the K parts meet, in order (read while the next unit runs) ----
    if (tid < 256) {
      // thread: tile tid / 128, accumulator q, lane ln; its column of n-tile n is 8n + 2(ln % 4) + q % 2
      const int tl = tid >> 7, q = (tid >> 5) & 3, ln = tid & 31;
      const int row = tl * 16 + (ln >> 2) + 8 * (q >> 1);
#pragma unroll
      for (int n = 0; n < NTX; ++n) {
        float v = 0.0f;
#pragma unroll
        for (int k = 0; k < KP; ++k) v += red[(((2 * k + tl) * NTX + n) * 4 + q) * 32 + ln];  // part order
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

  if constexpr (AM) argmax_finish<NTX, kT>(best, bcol, s_best, s_last, p, tid, lane);
}

// ---------------------------------------------------------------------------
// Dense batch 1: its own kernel, without tensor cores, laid out so that one
// staged activation load serves eight rows.  512-wide chunks: lane l owns
// in-features 512c + 16l .. +15 of every row (one 16-byte index load per
// row), warp w takes rows 8 (w % 4) .. +7 of the unit and K part w / 4 (two
// parts of whole chunks), and the activations are staged as fp32 with piece
// j (in-features 4j .. 4j+3 of a lane's 16) of lane l at byte
// 2048c + 512j + 16l, so a warp's 16-byte activation loads are
// conflict-free.  Each pair of weights takes two permutes, two shared loads
// and one paired fp32 fma (f32x2); a part's eight row sums leave the warp
// through a transposing shuffle reduction (nine shuffles), and the two
// parts meet in shared memory in part order.
// ---------------------------------------------------------------------------

// One row's 16 weights of a chunk (index word w of this lane) against the
// lane's activation pairs xp (in-features (2i, 2i+1) of its 16).
__device__ __forceinline__ void km8b1_row(uint64_t& acc, const uint4& w, const uint64_t (&xp)[8], uint32_t lb,
                                          uint32_t tb) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    acc = fma_f32x2(pack_f32x2(km8_lookup<0>(ws[s], lb, tb), km8_lookup<1>(ws[s], lb, tb)), xp[2 * s], acc);
    acc = fma_f32x2(pack_f32x2(km8_lookup<2>(ws[s], lb, tb), km8_lookup<3>(ws[s], lb, tb)), xp[2 * s + 1], acc);
  }
}

// Each lane holds one sum of each of 8 rows; returns, in lane l, the sum over
// the warp of row l / 4 (lanes exchange half of what they hold at each of
// the first three steps, then add whole values).
__device__ __forceinline__ float reduce_rows8(const float (&s)[8], int lane) {
  const bool h16 = (lane & 16) != 0, h8 = (lane & 8) != 0, h4 = (lane & 4) != 0;
  float v4[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // rows 4 h16 + i
    const float give = h16 ? s[i] : s[i + 4];
    const float keep = h16 ? s[i + 4] : s[i];
    v4[i] = keep + __shfl_xor_sync(0xffffffffu, give, 16);
  }
  float v2[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {  // rows 4 h16 + 2 h8 + i
    const float give = h8 ? v4[i] : v4[i + 2];
    const float keep = h8 ? v4[i + 2] : v4[i];
    v2[i] = keep + __shfl_xor_sync(0xffffffffu, give, 8);
  }
  const float give = h4 ? v2[0] : v2[1];
  const float keep = h4 ? v2[1] : v2[0];
  float v = keep + __shfl_xor_sync(0xffffffffu, give, 4);  // row 4 h16 + 2 h8 + h4 = l / 4
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v;
}

template <bool AM>
__global__ void __launch_bounds__(256, 2) km8b1_kernel(const __grid_constant__ MvParams p) {
  constexpr int kT = 256;
  constexpr int kR = 8;                  // rows per warp
  constexpr int KP = 2;                  // K parts per unit
  constexpr int EPW = 256 / 8;           // LUT entries per warp in a table build
  constexpr int kRedFloats = KP * 32;    // one partial-sum buffer: [part][32 rows]
  __shared__ unsigned long long s_best[kMaxCols];
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = smem_addr(km8_smem);  // the LUT table: [256][2 buffers][32] words (fp32 values)
  const uint32_t xbase = sbase + p.off_x;
  float* red0 = reinterpret_cast<float*>(km8_smem + p.off_red);
  const int64_t K = p.K;
  const int64_t total = p.tiles;  // row groups of 32
  const int64_t grid = gridDim.x;

  grid_launch_dependents();
  if (!p.prefetch) grid_wait_preceding();
  if (tid < kMaxCols) s_best[tid] = 0ull;

  auto unit_rows = [&](int64_t u) { return (int)min((int64_t)32, p.N - u * 32); };
  auto lut_entry = [&](int64_t u) -> uint32_t {
    const uint16_t* lut = reinterpret_cast<const uint16_t*>(p.aux) + u * 256;
    return lane < EPW ? __float_as_uint(__half2float(__ushort_as_half(lut[warp * EPW + lane]))) : 0u;
  };
  auto write_table = [&](uint32_t v, int b) {
#pragma unroll
    for (int j = 0; j < EPW / 4; ++j) {
      const int r = 4 * j + (lane >> 3);
      const uint32_t w = __shfl_sync(0xffffffffu, v, r);
      sts128(sbase + (uint32_t)(warp * EPW + r) * 256u + 128u * (uint32_t)b + 16u * (uint32_t)(lane & 7),
             make_uint4(w, w, w, w));
    }
  };
  const int rg = warp & 3, part = warp >> 2;
  const int nch = (int)((K + 511) / 512);
  const int cA = part * nch / KP, cB = (part + 1) * nch / KP;  // this warp's chunks, every unit
  const int64_t lk = 16 * (int64_t)lane;                       // this lane's first in-feature of a chunk

  // this lane's index word of row 8 rg + r of unit u, chunk c (zero where
  // past K or past the units; rows past N repeat the unit's last row)
  auto load_row = [&](int64_t u, int c, int r) -> uint4 {
    if (u < total && 512 * (int64_t)c + lk < K) {
      const int64_t row = u * 32 + min(kR * rg + r, unit_rows(u) - 1);
      return ldg_stream_128(p.codes + row * K + 512 * (int64_t)c + lk);
    }
    return make_uint4(0u, 0u, 0u, 0u);
  };

  // weights only before the wait (early weight reads): the first chunk's index words and LUT entries
  uint4 cw[kR];
#pragma unroll
  for (int r = 0; r < kR; ++r) cw[r] = cA < cB ? load_row(blockIdx.x, cA, r) : make_uint4(0u, 0u, 0u, 0u);
  const uint32_t lut0 = (int64_t)blockIdx.x < total ? lut_entry(blockIdx.x) : 0u;

  if (p.prefetch) grid_wait_preceding();
  {
    // fp32 activations: in-feature k = 512c + 16l + 4j + e at byte 2048c + 512j + 16l + 4e,
    // zero-padded to whole chunks
    const int64_t n8 = p.XS / 32;  // 8-feature pieces of the padded row
    for (int64_t j = tid; j < n8; j += kT) {
      float f[8];
      if (j < K / 8) {
        const uint4 v = ldg_nc_128(p.x + 8 * j);
        const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __half2 h = *reinterpret_cast<const __half2*>(&w4[e]);
          f[2 * e] = __low2float(h);
          f[2 * e + 1] = __high2float(h);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = 0.0f;
      }
      const int64_t k = 8 * j, c = k / 512, l = (k % 512) / 16, q = (k % 16) / 4;  // q even
      const uint32_t a = xbase + (uint32_t)(2048 * c + 512 * q + 16 * l);
      sts128(a, make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3])));
      sts128(a + 512u, make_uint4(__float_as_uint(f[4]), __float_as_uint(f[5]), __float_as_uint(f[6]), __float_as_uint(f[7])));
    }
  }
  if ((int64_t)blockIdx.x < total) write_table(lut0, 0);
  __syncthreads();  // the first table and the activations

  unsigned long long best[1] = {0ull};
  int bcol[1] = {-1};

  int buf = 0;
  for (int64_t u = blockIdx.x; u < total; u += grid, buf ^= 1) {
    const int nrows = unit_rows(u);
    const bool has_next = u + grid < total;
    float* red = red0 + (p.red_bufs == 2 ? buf : 0) * kRedFloats;
    if (p.red_bufs == 1) __syncthreads();  // one partial-sum buffer: the previous unit's sums have been read
    const uint32_t lutv = has_next ? lut_entry(u + grid) : 0u;
    const uint32_t lb = 128u * (uint32_t)buf + 4u * (uint32_t)lane;

    uint64_t acc[kR];
#pragma unroll
    for (int r = 0; r < kR; ++r) acc[r] = 0ull;
#pragma unroll 1
    for (int c = cA; c < cB; ++c) {
      const bool on = 512 * (int64_t)c + lk < K;  // the lane's in-features are inside K (else zero padding)
      uint64_t xp[8];
      const uint32_t xa = xbase + 2048u * (uint32_t)c + 16u * (uint32_t)lane;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 v = lds128(xa + 512u * (uint32_t)q);
        xp[2 * q] = pack_f32x2(v.x, v.y);
        xp[2 * q + 1] = pack_f32x2(v.z, v.w);
      }
      // the index words that follow: the next chunk of this part, else the next unit's first
      const int64_t un = c + 1 < cB ? u : u + grid;
      const int cn = c + 1 < cB ? c + 1 : cA;
      const bool ld = un < total && 512 * (int64_t)cn + lk < K;
      const uint8_t* nb = p.codes + (ld ? un * 32 * K + 512 * (int64_t)cn + lk : 0);
      const int nlast = ld ? unit_rows(un) - 1 : 0;
      if (512 * (int64_t)(c + 1) <= K) {  // (uniform) a whole chunk: no per-row branch
#pragma unroll
        for (int r = 0; r < kR; ++r) {
          km8b1_row(acc[r], cw[r], xp, lb, sbase);
          cw[r] = ld ? ldg_stream_128(nb + (int64_t)min(kR * rg + r, nlast) * K) : make_uint4(0u, 0u, 0u, 0u);
        }
      } else {
#pragma unroll
        for (int r = 0; r < kR; ++r) {
          if (on) km8b1_row(acc[r], cw[r], xp, lb, sbase);
          cw[r] = ld ? ldg_stream_128(nb + (int64_t)min(kR * rg + r, nlast) * K) : make_uint4(0u, 0u, 0u, 0u);
        }
      }
    }
    // this part's sums of the warp's 8 rows: lane pairs, then the warp (fixed order)
    float s[kR];
#pragma unroll
    for (int r = 0; r < kR; ++r) {
      const float2 a = unpack_f32x2(acc[r]);
      s[r] = a.x + a.y;
    }
    const float v = reduce_rows8(s, lane);
    if ((lane & 3) == 0) red[part * 32 + kR * rg + (lane >> 2)] = v;

    if (has_next) write_table(lutv, buf ^ 1);
    __syncthreads();

    if (tid < 32 && tid < nrows) {  // row tid of the unit: parts in order
      const float y = red[tid] + red[32 + tid];
      const int64_t nrow = u * 32 + tid;
      if constexpr (AM) {
        const unsigned long long key = argmax_key(y, nrow);
        best[0] = key > best[0] ? key : best[0];
        bcol[0] = 0;
      } else {
        p.y[nrow] = y;
      }
    }
  }

  if constexpr (AM) argmax_finish<1, kT>(best, bcol, s_best, s_last, p, tid, lane);
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
  p.n_xrows = p.gather ? (p.x_per_slot ? p.B * p.topk : p.B) : p.B;
  const int nt = p.B > 8 ? 2 : 1;
  const int64_t units = (p.gather ? (int64_t)p.B * p.topk : 1) * p.tiles;
  const int64_t dyn_limit = (int64_t)kSmemLimit - kStaticSmem;
  // dense batch 1 takes its own kernel (one fp32 activation row, in its own
  // chunk layout); where that row does not fit, the general kernel (fp16
  // rows, half the bytes)
  for (int one = (!p.gather && p.B == 1) ? 1 : 0; one >= 0; --one) {
    p.one = one;
    // staged activation rows: natural order, whole 64-wide chunks, the row
    // stride at 16 mod 128 bytes so the 16-byte reads of 8 lanes (two rows,
    // four in-feature quarters) fall in distinct banks
    p.XS = one ? (int)(2048 * ((p.K + 511) / 512)) : (int)(round_up8(2 * round_up8(p.K, 64), 128) + 16);
    const int64_t red_one = one ? (int64_t)2 * 32 * 4 : (int64_t)8 * 2 * nt * 4 * 32 * 4;  // one buffer
    // layouts in order of preference: two 8-warp CTAs per SM, one 16-warp CTA
    // (batch 1: one 8-warp CTA); two partial-sum buffers, else one
    const int cand[4][3] = {{8, 2, 2}, {16, 1, 2}, {8, 2, 1}, {16, 1, 1}};
    for (int ci = 0; ci < 4; ++ci) {
      const int warps = one ? 8 : cand[ci][0], ctas = cand[ci][1];
      p.warps = warps;
      p.red_bufs = cand[ci][2];
      p.off_tab = 0;  // 64 KB: 256 rows x 2 buffers x 128 bytes
      p.off_red = 256 * 256;
      p.off_x = (int)round_up8(p.off_red + p.red_bufs * red_one, 128);
      const int64_t bytes = p.off_x + (int64_t)p.n_xrows * p.XS;
      const int64_t stat = one ? 1024 : kStaticSmem;  // the batch-1 kernel's static shared memory is the argmax keys
      if (bytes <= dyn_limit && ctas * (bytes + stat + 1024) <= kSmemPerSM) {
        p.smem_bytes = (int)bytes;
        p.ctas_per_sm = ctas;
        const int64_t slots = (int64_t)num_sms * ctas;
        p.grid = (int)(units < slots ? units : slots);
        return true;
      }
    }
  }
  return false;
}

template <int NT, int WARPS, bool AM>
static cudaError_t launch_km8_t(const MvParams& p, cudaStream_t stream) {
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(km8_kernel<NT, WARPS, AM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemLimit - kStaticSmem);
    if (err != cudaSuccess) return err;
    attr_set[dev].store(true, std::memory_order_release);
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
static cudaError_t launch_km8b1_t(const MvParams& p, cudaStream_t stream) {
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(km8b1_kernel<AM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemLimit - kStaticSmem);
    if (err != cudaSuccess) return err;
    attr_set[dev].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.grid);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = (size_t)p.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, km8b1_kernel<AM>, p);
}

template <bool AM>
static cudaError_t launch_km8_a(const MvParams& p, cudaStream_t stream) {
  const bool wide = p.warps == 16;
  if (p.one) return launch_km8b1_t<AM>(p, stream);
  if (p.B > 8) return wide ? launch_km8_t<2, 16, AM>(p, stream) : launch_km8_t<2, 8, AM>(p, stream);
  return wide ? launch_km8_t<1, 16, AM>(p, stream) : launch_km8_t<1, 8, AM>(p, stream);
}

cudaError_t launch_km8(const MvParams& p, cudaStream_t stream) {
  return p.argmax ? launch_km8_a<true>(p, stream) : launch_km8_a<false>(p, stream);
}

}  // namespace qmv
