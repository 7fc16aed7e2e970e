// qmv_matvec.cu -- fused dequantize + matvec (dense and routed-expert gather)
// for weight-only block-quantized layers, sm_100a.
//
// What it computes (the pages' decode problem: "Dense-path int4km coverage +
// flagship Qwen3.6-35B -- session findings & methods", sec. 1-3 and 8; the
// gather formats of "Stream D -- Quantization (FP4 + QAT-int4): feasibility,
// first result, and plan", sec. 1):
//     y[c, n] = sum_k x[c, k] * Wdq[n, k],   c < B <= 16 activation rows,
// reading only the packed codes and their block scales / row palette.
//
// Design (B200): the op streams ~0.5 byte of weights per multiply-add, so HBM
// bandwidth bounds it and the instruction budget per weight is ~2-3.  Each CTA
// (one per SM, persistent) runs one producer warp that moves 16-row weight
// tiles into a ring of shared-memory stages with 1-D bulk async copies (TMA
// engine, mbarrier transaction counts), and eight consumer warps that split
// each tile along K.  A consumer turns one 32-bit word of codes into exact
// fp16 operands in registers and lets one m16n8k16 tensor-core step do 256
// multiply-adds (16 rows x 16 k, with the activations as the 8-column operand),
// so the per-weight cost is the decode alone.  Block scales are applied in fp32
// to each 32-block's partial sum; the palette format carries its scale in the
// table and accumulates straight through.  Tile partial sums are reduced in
// shared memory in a fixed warp order (deterministic), then written once.
#include "qmv_device.cuh"

namespace qmv {

template <int FMT>
struct FmtT;
template <>
struct FmtT<QMV_FMT_FP4> {
  static constexpr int kBits = 4, kSB = 1;
  static constexpr bool kLut = false, kPermX = false;
};
template <>
struct FmtT<QMV_FMT_INT4> {
  static constexpr int kBits = 4, kSB = 2;
  static constexpr bool kLut = false, kPermX = true;  // decoder emits (k0,k4),(k1,k5),...
};
template <>
struct FmtT<QMV_FMT_INT4KM> {
  static constexpr int kBits = 4, kSB = 0;
  static constexpr bool kLut = true, kPermX = false;
};
template <>
struct FmtT<QMV_FMT_INT8> {
  static constexpr int kBits = 8, kSB = 2;
  static constexpr bool kLut = false, kPermX = false;
};

// Column groups: the activation rows served by one pass over one expert's
// weights (dense: one group of all B rows).
struct GroupTable {
  int ngroups;
  int expert[kMaxPairs];
  int start[kMaxPairs];
  int count[kMaxPairs];
  int16_t sorted[kMaxPairs];  // (token, slot) pair indices ordered by expert
};

__device__ __forceinline__ uint32_t lds_u8(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts_u8(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u8 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void sts_f32x2(uint32_t a, float u, float v) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(a), "f"(u), "f"(v) : "memory");
}
__device__ __forceinline__ float lds_f32(uint32_t a) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint4 ldg_nc_128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// Barrier on named barrier `id` over `n` threads that also ORs a predicate.
__device__ __forceinline__ bool bar_red_or(uint32_t id, uint32_t n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred pi, po;\n setp.ne.u32 pi, %1, 0;\n barrier.red.or.pred po, %2, %3, pi;\n"
      " selp.u32 %0, 1, 0, po;\n}"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Block-scale of (row, block) from the staged scale region.
template <int FMT>
__device__ __forceinline__ float stage_scale(uint32_t a) {
  if constexpr (FMT == QMV_FMT_FP4) {
    return e8m0_to_f32(lds_u8(a));
  } else {
    return __half2float(__ushort_as_half((unsigned short)lds_u16(a)));
  }
}

template <int FMT, int NT>
__global__ void __launch_bounds__(kThreads, 1) mv_kernel(const __grid_constant__ MvParams p) {
  using F = FmtT<FMT>;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ GroupTable gt;
  __shared__ int s_ids[kMaxPairs];
  __shared__ int s_abort;
  __shared__ int s_nvalid;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = p.stages;
  const uint32_t sbase = smem_addr(smem);
  const uint32_t full0 = sbase, empty0 = sbase + 8u * S;  // mbarriers
  const int P = p.gather ? p.B * p.topk : p.B;

  // ---- set-up: barriers and the column groups ------------------------------
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8u * s, 1);
      mbar_init(empty0 + 8u * s, kConsumerWarps);
    }
    mbar_fence_init();
    s_abort = 0;
    s_nvalid = 0;
  }
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
        if (ng == 0 || gt.expert[ng - 1] != e || gt.count[ng - 1] == 8 * NT) {
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
    __syncthreads();
  }

  const int64_t total = (int64_t)gt.ngroups * p.tiles;
  if ((int64_t)blockIdx.x >= total) return;

  if (warp == 0) {
    // ======================= producer warp =======================
    uint32_t it = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < total && ok; u += gridDim.x) {
      const int grp = (int)(u / p.tiles);
      const int64_t tile = u - (int64_t)grp * p.tiles;
      const int64_t row0 = tile * kTileRows;
      const int nrows = (int)min((int64_t)kTileRows, p.N - row0);
      const int e = gt.expert[grp];
      const uint8_t* ce = p.codes + (int64_t)e * p.expert_code_bytes;
      const uint8_t* ae = p.aux + (int64_t)e * p.expert_aux_bytes;
      for (int c = 0; c < p.nchunks; ++c, ++it) {
        const int s = (int)(it % (uint32_t)S);
        const uint32_t ph = (it / (uint32_t)S) & 1u;
        const uint32_t fb = full0 + 8u * s;
        if (!mbar_wait(empty0 + 8u * s, ph ^ 1u, &s_abort, p.status)) {
          ok = false;
          break;
        }
        const int k0 = c * p.KC;
        const int kc = min(p.KC, (int)(p.K - k0));
        const uint32_t cbytes = (uint32_t)(kc * F::kBits / 8);
        const uint32_t stage = sbase + p.off_stage + (uint32_t)s * p.stage_bytes;
        const uint32_t auxs = stage + p.aux_off;
        uint32_t tx = kTileRows * cbytes;
        uint32_t arow = 0, lut_bytes = 0;
        const uint8_t* bsrc = nullptr;
        uint32_t bbytes = 0, bhead = 0, bmid = 0, bdst = 0;
        if constexpr (F::kLut) {
          lut_bytes = (c == 0) ? (uint32_t)nrows * 32u : 0u;
          tx += lut_bytes;
        } else if (p.aux_mode == kAuxRows) {
          arow = (uint32_t)(kc / 32) * F::kSB;
          tx += kTileRows * arow;
        } else {
          // whole tile scale block: bulk copy of its 16-byte-aligned middle,
          // head/tail bytes by plain loads; staged at offset (src & 15).
          bsrc = ae + row0 * p.aux_row_bytes;
          bbytes = (uint32_t)nrows * (uint32_t)p.aux_row_bytes;
          const uint32_t mis = (uint32_t)(reinterpret_cast<uintptr_t>(bsrc) & 15u);
          bhead = min(bbytes, (16u - mis) & 15u);
          bmid = (bbytes - bhead) & ~15u;
          bdst = auxs + mis;
          tx += bmid;
        }
        if (lane == 0) mbar_expect_tx(fb, tx);
        __syncwarp();
        if (lane < kTileRows) {
          const int r = min(lane, nrows - 1);  // rows past N re-read the last row
          bulk_g2s(stage + (uint32_t)lane * p.RS,
                   ce + (row0 + r) * p.code_row_bytes + (int64_t)k0 * F::kBits / 8, cbytes, fb);
        } else {
          const int r16 = lane - kTileRows;
          if constexpr (F::kLut) {
            if (r16 == 0 && lut_bytes) bulk_g2s(auxs, ae + row0 * 32, lut_bytes, fb);
          } else {
            if (p.aux_mode == kAuxRows) {
              const int r = min(r16, nrows - 1);
              bulk_g2s(auxs + (uint32_t)r16 * p.AS, ae + (row0 + r) * p.aux_row_bytes + (int64_t)(k0 / 32) * F::kSB,
                       arow, fb);
            } else if (r16 == 0 && bmid) {
              bulk_g2s(bdst + bhead, bsrc + bhead, bmid, fb);
            }
          }
        }
        if constexpr (!F::kLut) {
          if (p.aux_mode == kAuxBlock) {
            bool wrote = false;
            for (uint32_t i = lane; i < bhead; i += 32) {
              sts_u8(bdst + i, bsrc[i]);
              wrote = true;
            }
            for (uint32_t i = bhead + bmid + lane; i < bbytes; i += 32) {
              sts_u8(bdst + i, bsrc[i]);
              wrote = true;
            }
            if (wrote) fence_proxy_async();
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(fb);
      }
    }
    // Drain: every issued stage's copies must have landed before the CTA exits.
    if (lane == 0) {
      const uint32_t n = it < (uint32_t)S ? it : (uint32_t)S;
      for (uint32_t s = 0; s < n; ++s) {
        const uint32_t last = s + (uint32_t)S * ((it - 1u - s) / (uint32_t)S);
        mbar_wait(full0 + 8u * s, (last / (uint32_t)S) & 1u, &s_abort, p.status, /*respect_abort=*/false);
      }
    }
    return;
  }

  // ======================= consumer warps =======================
  const int cw = warp - 1;
  const int g = lane >> 2, t = lane & 3;
  const uint32_t xbase = sbase + p.off_x;

  // Stage the activations once: row r at xbase + r * XS, in the k order the
  // format's decoder emits (int4: (k0,k4),(k1,k5),(k2,k6),(k3,k7) per 8).
  {
    const int ct = tid - 32;
    const int64_t per_row = p.K / 8;
    const int64_t n16 = (int64_t)p.n_xrows * per_row;
    for (int64_t i = ct; i < n16; i += kConsumerWarps * 32) {
      const int64_t r = i / per_row, j = i - r * per_row;
      uint4 v = ldg_nc_128(p.x + r * p.K + 8 * j);
      if constexpr (F::kPermX) {
        v = make_uint4(prmt(v.x, v.z, 0x5410u), prmt(v.x, v.z, 0x7632u), prmt(v.y, v.w, 0x5410u),
                       prmt(v.y, v.w, 0x7632u));
      }
      sts128(xbase + (uint32_t)(r * p.XS + 16 * j), v);
    }
    named_bar_sync(1, kConsumerWarps * 32);
  }

  const uint32_t red0 = sbase + p.off_red;
  uint32_t it = 0;
  int par = 0;
  for (int64_t u = blockIdx.x; u < total; u += gridDim.x) {
    const int grp = (int)(u / p.tiles);
    const int64_t tile = u - (int64_t)grp * p.tiles;
    const int64_t row0 = tile * kTileRows;
    const int nrows = (int)min((int64_t)kTileRows, p.N - row0);
    const int ncols = gt.count[grp], gstart = gt.start[grp];

    uint32_t xa[NT];
    bool xv[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int col = 8 * n + g;
      xv[n] = col < ncols;
      const int pair = xv[n] ? gt.sorted[gstart + col] : 0;
      const int xrow = p.gather ? (p.x_per_slot ? pair : pair / p.topk) : pair;
      xa[n] = xbase + (uint32_t)xrow * p.XS + (uint32_t)t * 16u;
    }

    float acc[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.0f;
    Palette pg, pg8;
    bool tile_ok = true;

    for (int c = 0; c < p.nchunks; ++c, ++it) {
      const int s = (int)(it % (uint32_t)S);
      const uint32_t ph = (it / (uint32_t)S) & 1u;
      const bool ok = mbar_wait(full0 + 8u * s, ph, &s_abort, p.status);
      if (ok) {
        const uint32_t stage = sbase + p.off_stage + (uint32_t)s * p.stage_bytes;
        const uint32_t auxs = stage + p.aux_off;
        const int k0 = c * p.KC;
        const int kc = min(p.KC, (int)(p.K - k0));
        const int nbc = kc / 32;
        if constexpr (F::kLut) {
          if (c == 0) {
            uint32_t e0[8], e1[8];
            const uint4 a0 = lds128(auxs + (uint32_t)g * 32u), a1 = lds128(auxs + (uint32_t)g * 32u + 16u);
            const uint4 b0 = lds128(auxs + (uint32_t)(g + 8) * 32u), b1 = lds128(auxs + (uint32_t)(g + 8) * 32u + 16u);
            e0[0] = a0.x; e0[1] = a0.y; e0[2] = a0.z; e0[3] = a0.w;
            e0[4] = a1.x; e0[5] = a1.y; e0[6] = a1.z; e0[7] = a1.w;
            e1[0] = b0.x; e1[1] = b0.y; e1[2] = b0.z; e1[3] = b0.w;
            e1[4] = b1.x; e1[5] = b1.y; e1[6] = b1.z; e1[7] = b1.w;
            pg = palette_from_words(e0);
            pg8 = palette_from_words(e1);
          }
        }
        // scale addresses of rows g, g+8 for block 0 of this chunk
        uint32_t sa_g = 0, sa_g8 = 0;
        if constexpr (!F::kLut) {
          if (p.aux_mode == kAuxRows) {
            sa_g = auxs + (uint32_t)g * p.AS;
            sa_g8 = auxs + (uint32_t)(g + 8) * p.AS;
          } else {
            const uint8_t* bsrc = p.aux + (int64_t)gt.expert[grp] * p.expert_aux_bytes + row0 * p.aux_row_bytes;
            const uint32_t b0a = auxs + (uint32_t)(reinterpret_cast<uintptr_t>(bsrc) & 15u) +
                                 (uint32_t)(k0 / 32) * F::kSB;
            sa_g = b0a + (uint32_t)g * (uint32_t)p.aux_row_bytes;
            sa_g8 = b0a + (uint32_t)(g + 8) * (uint32_t)p.aux_row_bytes;
          }
        }
        const uint32_t crow_g = stage + (uint32_t)g * p.RS, crow_g8 = stage + (uint32_t)(g + 8) * p.RS;
        const int b_lo = cw * nbc / kConsumerWarps, b_hi = (cw + 1) * nbc / kConsumerWarps;
#pragma unroll 2
        for (int b = b_lo; b < b_hi; ++b) {
          uint4 xr[NT];
#pragma unroll
          for (int n = 0; n < NT; ++n)
            xr[n] = xv[n] ? lds128(xa[n] + (uint32_t)(k0 + 32 * b) * 2u) : make_uint4(0u, 0u, 0u, 0u);
          uint32_t g0lo, g0hi, g1lo, g1hi, h0lo, h0hi, h1lo, h1hi;  // row g / g+8, step 0 / 1
          if constexpr (F::kBits == 8) {
            const uint2 vg = lds64(crow_g + 32u * b + 8u * t);
            const uint2 vh = lds64(crow_g8 + 32u * b + 8u * t);
            dec_int8_word(vg.x, g0lo, g0hi);
            dec_int8_word(vg.y, g1lo, g1hi);
            dec_int8_word(vh.x, h0lo, h0hi);
            dec_int8_word(vh.y, h1lo, h1hi);
          } else {
            const uint32_t wg = lds32(crow_g + 16u * b + 4u * t);
            const uint32_t wh = lds32(crow_g8 + 16u * b + 4u * t);
            if constexpr (FMT == QMV_FMT_FP4) {
              DecFp4::run(wg, g0lo, g0hi, g1lo, g1hi);
              DecFp4::run(wh, h0lo, h0hi, h1lo, h1hi);
            } else if constexpr (FMT == QMV_FMT_INT4) {
              DecInt4::run(wg, g0lo, g0hi, g1lo, g1hi);
              DecInt4::run(wh, h0lo, h0hi, h1lo, h1hi);
            } else {
              dec_int4km(pg, wg, g0lo, g0hi, g1lo, g1hi);
              dec_int4km(pg8, wh, h0lo, h0hi, h1lo, h1hi);
            }
          }
          if constexpr (F::kLut) {
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              mma16816(acc[n], g0lo, h0lo, g0hi, h0hi, xr[n].x, xr[n].y);
              mma16816(acc[n], g1lo, h1lo, g1hi, h1hi, xr[n].z, xr[n].w);
            }
          } else {
            const float sg = stage_scale<FMT>(sa_g + (uint32_t)b * F::kSB);
            const float sh = stage_scale<FMT>(sa_g8 + (uint32_t)b * F::kSB);
#pragma unroll
            for (int n = 0; n < NT; ++n) {
              float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
              mma16816(d, g0lo, h0lo, g0hi, h0hi, xr[n].x, xr[n].y);
              mma16816(d, g1lo, h1lo, g1hi, h1hi, xr[n].z, xr[n].w);
              acc[n][0] = fmaf(d[0], sg, acc[n][0]);
              acc[n][1] = fmaf(d[1], sg, acc[n][1]);
              acc[n][2] = fmaf(d[2], sh, acc[n][2]);
              acc[n][3] = fmaf(d[3], sh, acc[n][3]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8u * s);
      tile_ok = tile_ok && ok;
    }

    // ---- deterministic split-K reduction over the consumer warps ----
    const uint32_t red = red0 + (uint32_t)par * (kConsumerWarps * kTileRows * kMaxCols * 4) +
                         (uint32_t)cw * (kTileRows * kMaxCols * 4);
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int c0 = 8 * n + 2 * t;
      sts_f32x2(red + (uint32_t)(g * kMaxCols + c0) * 4u, acc[n][0], acc[n][1]);
      sts_f32x2(red + (uint32_t)((g + 8) * kMaxCols + c0) * 4u, acc[n][2], acc[n][3]);
    }
    const bool stop = bar_red_or(1, kConsumerWarps * 32, !tile_ok || s_abort != 0);
    if (stop) break;
    const int ct = tid - 32;
    if (ct < kTileRows * ncols) {
      const int row = ct & (kTileRows - 1), col = ct >> 4;
      const uint32_t rp = red0 + (uint32_t)par * (kConsumerWarps * kTileRows * kMaxCols * 4) +
                          (uint32_t)(row * kMaxCols + col) * 4u;
      float sum = 0.0f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) sum += lds_f32(rp + (uint32_t)w * (kTileRows * kMaxCols * 4));
      if (row < nrows) {
        const int pair = gt.sorted[gstart + col];
        p.y[(int64_t)pair * p.N + row0 + row] = sum;
      }
    }
    par ^= 1;
  }
}

// ---------------------------------------------------------------------------
// Host side: geometry and launch
// ---------------------------------------------------------------------------

static int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

bool plan_matvec(int fmt, MvParams& p) {
  const FmtInfo fi = fmt_info(fmt);
  p.code_row_bytes = p.K * fi.bits / 8;
  p.aux_row_bytes = fi.lut ? 32 : (p.K / 32) * fi.scale_bytes;
  p.expert_code_bytes = p.N * p.code_row_bytes;
  p.expert_aux_bytes = p.N * p.aux_row_bytes;
  p.tiles = (p.N + kTileRows - 1) / kTileRows;
  p.KC = (int)(p.K < fi.kc_max ? p.K : fi.kc_max);
  p.nchunks = (int)((p.K + p.KC - 1) / p.KC);
  const int64_t cb = (int64_t)p.KC * fi.bits / 8;
  // Row strides chosen so the consumers' shared-memory reads are free of bank
  // conflicts: 4-bit rows at 16 mod 128 bytes (32-bit loads), 8-bit rows at
  // 32 mod 128 (64-bit loads).
  p.RS = (int)(round_up(cb, 128) + (fi.bits == 4 ? 16 : 32));
  int64_t aux_region;
  if (fi.lut) {
    p.aux_mode = kAuxLut;
    p.AS = 32;
    aux_region = kTileRows * 32;
  } else {
    const int64_t chunk_sc = (int64_t)(p.KC / 32) * fi.scale_bytes;
    const int64_t last_sc = ((p.K - (int64_t)(p.nchunks - 1) * p.KC) / 32) * fi.scale_bytes;
    const bool base16 = (reinterpret_cast<uintptr_t>(p.aux) & 15u) == 0;
    if (base16 && p.aux_row_bytes % 16 == 0 && chunk_sc % 16 == 0 && last_sc % 16 == 0) {
      p.aux_mode = kAuxRows;
      int64_t j = chunk_sc / 16;
      if (j % 2 == 0) ++j;  // odd multiple of 16 bytes: rows g = 0..7 hit distinct banks
      p.AS = (int)(16 * j);
      aux_region = kTileRows * p.AS;
    } else {
      p.aux_mode = kAuxBlock;
      p.AS = (int)p.aux_row_bytes;
      aux_region = round_up(kTileRows * p.aux_row_bytes + 16, 16);
    }
  }
  p.aux_off = kTileRows * p.RS;
  p.stage_bytes = (int)round_up(p.aux_off + aux_region, 128);
  p.XS = (int)(round_up(2 * p.K, 128) + 64);  // 64 mod 128: conflict-free 128-bit reads
  p.n_xrows = p.gather ? (p.x_per_slot ? p.B * p.topk : p.B) : p.B;
  p.off_red = 128;  // mbarriers live in the first 128 bytes
  p.off_x = p.off_red + 2 * kConsumerWarps * kTileRows * kMaxCols * 4;
  p.off_stage = (int)round_up(p.off_x + (int64_t)p.n_xrows * p.XS, 128);
  const int64_t static_reserve = 8 * 1024;  // the kernel's static shared memory (group table)
  const int64_t avail = (int64_t)kSmemLimit - static_reserve - p.off_stage;
  if (avail < 2 * (int64_t)p.stage_bytes) return false;
  int64_t st = avail / p.stage_bytes;
  if (st > kMaxStages) st = kMaxStages;
  p.stages = (int)st;
  p.smem_bytes = (int)(p.off_stage + st * p.stage_bytes);
  return true;
}

template <int FMT, int NT>
static cudaError_t launch_t(const MvParams& p, int num_sms, cudaStream_t stream) {
  static bool attr_set[64] = {false};
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && !attr_set[dev]) {
    err = cudaFuncSetAttribute(mv_kernel<FMT, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemLimit - 8 * 1024);
    if (err != cudaSuccess) return err;
    attr_set[dev] = true;
  }
  const int64_t upper = (p.gather ? (int64_t)p.B * p.topk : 1) * p.tiles;
  const int grid = (int)(upper < num_sms ? upper : num_sms);
  mv_kernel<FMT, NT><<<grid, kThreads, p.smem_bytes, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_matvec(int fmt, const MvParams& p, int num_sms, cudaStream_t stream) {
  // activation columns served per pass: dense B, gather at most B pairs per
  // expert when ids are distinct per token (groups are capped at 8 * NT)
  const bool two = p.B > 8;
  switch (fmt) {
    case QMV_FMT_FP4: return two ? launch_t<QMV_FMT_FP4, 2>(p, num_sms, stream) : launch_t<QMV_FMT_FP4, 1>(p, num_sms, stream);
    case QMV_FMT_INT4: return two ? launch_t<QMV_FMT_INT4, 2>(p, num_sms, stream) : launch_t<QMV_FMT_INT4, 1>(p, num_sms, stream);
    case QMV_FMT_INT4KM: return two ? launch_t<QMV_FMT_INT4KM, 2>(p, num_sms, stream) : launch_t<QMV_FMT_INT4KM, 1>(p, num_sms, stream);
    case QMV_FMT_INT8: return two ? launch_t<QMV_FMT_INT8, 2>(p, num_sms, stream) : launch_t<QMV_FMT_INT8, 1>(p, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace qmv
