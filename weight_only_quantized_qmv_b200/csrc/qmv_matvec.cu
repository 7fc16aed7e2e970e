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
// bandwidth bounds it and the instruction budget per weight is ~2-3.  Each
// warp of a persistent CTA is an independent pipeline over whole 16-row
// weight tiles: it copies its tile's next K-slice (16 rows x 512 weights,
// ~4.5 KB) with 16-byte asynchronous copies (cp.async) into a private
// shared-memory ring while it decodes and multiplies the previous slice, and
// it owns all of K of its tile, so no cross-warp reduction or CTA barrier
// sits on the streaming path.  Rows land at a padded stride so the warp's
// shared-memory reads are free of bank conflicts.  (Measured on B200: 16-byte
// asynchronous copies and 128-bit loads both reach the ~7.0 TB/s read ceiling
// with enough bytes in flight, while one-thread 1-D bulk copies cost ~225 ns
// per instruction.)  The warp turns one 32-bit word of codes into exact fp16
// operands in registers and lets one m16n8k16 tensor-core step do 256
// multiply-adds (16 rows x 16 k, with the activations as the 8-column
// operand), so the per-weight cost is the decode alone.  Block scales are
// applied in fp32 to each 32-block's partial sum; the palette format carries
// its scale in the table and accumulates straight through.  Each output is
// accumulated by one lane in a fixed order and written once (deterministic).
#include <atomic>

#include "qmv_device.cuh"
#include "qmv_kernel_common.cuh"

namespace qmv {

template <int FMT>
struct FmtT;
template <>
struct FmtT<QMV_FMT_FP4> {
  static constexpr int kBits = 4, kSB = 1;
  static constexpr bool kLut = false, kPermX = false, kZp = false;
};
template <>
struct FmtT<QMV_FMT_INT4> {
  static constexpr int kBits = 4, kSB = 2;
  static constexpr bool kLut = false, kPermX = true, kZp = false;  // decoder emits (k0,k4),(k1,k5),...
};
template <>
struct FmtT<QMV_FMT_INT4KM> {
  static constexpr int kBits = 4, kSB = 0;
  static constexpr bool kLut = true, kPermX = false, kZp = false;
};
template <>
struct FmtT<QMV_FMT_INT8> {
  static constexpr int kBits = 8, kSB = 2;
  static constexpr bool kLut = false, kPermX = false, kZp = false;
};
// affine int4: the int4 decoder with the block's own zero point instead of 8;
// a slice's zero points are staged after its scales, two per byte
template <>
struct FmtT<QMV_FMT_INT4AFF> {
  static constexpr int kBits = 4, kSB = 2;
  static constexpr bool kLut = false, kPermX = true, kZp = true;
};


__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most `n` (0..4; larger counts wait for 4) of this thread's
// committed copy groups are pending.
__device__ __forceinline__ void cp_async_wait(int n) {
  if (n <= 0)
    asm volatile("cp.async.wait_group 0;" ::: "memory");
  else if (n == 1)
    asm volatile("cp.async.wait_group 1;" ::: "memory");
  else if (n == 2)
    asm volatile("cp.async.wait_group 2;" ::: "memory");
  else if (n == 3)
    asm volatile("cp.async.wait_group 3;" ::: "memory");
  else
    asm volatile("cp.async.wait_group 4;" ::: "memory");
}

// Block-scale of (row, block) from the staged scale region (fp4: the e8m0
// scale times 2; the partial sums are halved once per tile).
template <int FMT>
__device__ __forceinline__ float stage_scale(uint32_t a, const Mul& m) {
  if constexpr (FMT == QMV_FMT_FP4) {
    return e8m0_x2_to_f32<3>(lds_u8(a) << 24, m);
  } else {
    return __half2float(__ushort_as_half((unsigned short)lds_u16(a)));
  }
}

// fp16 scale i of a 16-byte / 8-byte group -> float
template <int I>
__device__ __forceinline__ float half_at(const uint4& v) {
  const uint32_t w = (I / 2 == 0) ? v.x : (I / 2 == 1) ? v.y : (I / 2 == 2) ? v.z : v.w;
  const __half2 h = *reinterpret_cast<const __half2*>(&w);
  return (I % 2 == 0) ? __low2float(h) : __high2float(h);
}

// Decode one block's codes of rows g and g+8 into the two m16n8k16 A fragments
// (zg / zh: the block's zero points of rows g / g+8, affine int4 only; KMS:
// int4km row g+8 through the lane's palette copy at ktb in shared memory).
template <int FMT, bool KMS>
__device__ __forceinline__ void decode_block(uint32_t crow_g, uint32_t crow_g8, int b, int t, const Palette& pg,
                                             const Palette& pg8, const Mul& m, uint32_t (&a0)[4], uint32_t (&a1)[4],
                                             uint32_t zg, uint32_t zh, uint32_t ktb) {
  uint32_t g0lo, g0hi, g1lo, g1hi, h0lo, h0hi, h1lo, h1hi;  // row g / g+8, step 0 / 1
  if constexpr (FmtT<FMT>::kBits == 8) {
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
      DecFp4::run(wg, g0lo, g0hi, g1lo, g1hi, m);
      DecFp4::run(wh, h0lo, h0hi, h1lo, h1hi, m);
    } else if constexpr (FMT == QMV_FMT_INT4) {
      DecInt4::run(wg, g0lo, g0hi, g1lo, g1hi, m);
      DecInt4::run(wh, h0lo, h0hi, h1lo, h1hi, m);
    } else if constexpr (FMT == QMV_FMT_INT4AFF) {
      DecInt4::run_z(wg, g0lo, g0hi, g1lo, g1hi, int4_zp_sub(zg), int4_zp_neg(zg));
      DecInt4::run_z(wh, h0lo, h0hi, h1lo, h1hi, int4_zp_sub(zh), int4_zp_neg(zh));
    } else {
      dec_int4km(pg, wg, g0lo, g0hi, g1lo, g1hi, m);
      if constexpr (KMS)
        dec_int4km_smem(ktb, wh, h0lo, h0hi, h1lo, h1hi, m);
      else
        dec_int4km(pg8, wh, h0lo, h0hi, h1lo, h1hi, m);
    }
  }
  a0[0] = g0lo; a0[1] = h0lo; a0[2] = g0hi; a0[3] = h0hi;
  a1[0] = g1lo; a1[1] = h1lo; a1[2] = g1hi; a1[3] = h1hi;
}

// Multiply-accumulate one decoded block: palette formats accumulate directly,
// block-scaled formats scale the block's exact partial in fp32.
template <int FMT, int NT>
__device__ __forceinline__ void mac_block(float (&acc)[NT][4], const uint32_t (&a0)[4], const uint32_t (&a1)[4],
                                          const uint4 (&xr)[NT], float sg, float sh) {
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    if constexpr (FmtT<FMT>::kLut) {
      mma16816(acc[n], a0[0], a0[1], a0[2], a0[3], xr[n].x, xr[n].y);
      mma16816(acc[n], a1[0], a1[1], a1[2], a1[3], xr[n].z, xr[n].w);
    } else {
      float d[4];
      mma16816_zc(d, a0[0], a0[1], a0[2], a0[3], xr[n].x, xr[n].y);
      mma16816(d, a1[0], a1[1], a1[2], a1[3], xr[n].z, xr[n].w);
      acc[n][0] = fmaf(d[0], sg, acc[n][0]);
      acc[n][1] = fmaf(d[1], sg, acc[n][1]);
      acc[n][2] = fmaf(d[2], sh, acc[n][2]);
      acc[n][3] = fmaf(d[3], sh, acc[n][3]);
    }
  }
}

// A warp's NB blocks of a full K-slice, unrolled: every shared-memory address
// is a base plus an immediate, and the slice's scales of a row are read with
// one or two 128-bit loads (zo: offset of the zero points from the scales).
template <int FMT, int NT, int NB, bool KMS>
__device__ __forceinline__ void slice_full(float (&acc)[NT][4], uint32_t crow_g, uint32_t crow_g8, uint32_t sa_g,
                                           uint32_t sa_g8, uint32_t zo, const uint32_t (&xb)[NT], int t,
                                           const Palette& pg, const Palette& pg8, const Mul& m, uint32_t ktb) {
  using F = FmtT<FMT>;
  uint4 sg0 = make_uint4(0u, 0u, 0u, 0u), sh0 = sg0, sg1 = sg0, sh1 = sg0;
  if constexpr (!F::kLut) {
    sg0 = lds128(sa_g);
    sh0 = lds128(sa_g8);
    if constexpr (NB * F::kSB == 32) {
      sg1 = lds128(sa_g + 16u);
      sh1 = lds128(sa_g8 + 16u);
    }
  }
  uint2 zwg = make_uint2(0u, 0u), zwh = zwg;  // the slice's zero-point nibbles of rows g, g+8
  if constexpr (F::kZp) {
    static_assert(NB == 8 || NB == 16, "zero points come in 4- or 8-byte pieces");
    if constexpr (NB == 16) {
      zwg = lds64(sa_g + zo);
      zwh = lds64(sa_g8 + zo);
    } else {
      zwg.x = lds32(sa_g + zo);
      zwh.x = lds32(sa_g8 + zo);
    }
  }
#pragma unroll
  for (int i = 0; i < NB; ++i) {
    uint4 xr[NT];
#pragma unroll
    for (int n = 0; n < NT; ++n) xr[n] = lds128(xb[n] + 64u * (uint32_t)i);
    uint32_t a0[4], a1[4];
    uint32_t zg = 0u, zh = 0u;
    if constexpr (F::kZp) {
      zg = ((i < 8 ? zwg.x : zwg.y) >> (4 * (i & 7))) & 15u;
      zh = ((i < 8 ? zwh.x : zwh.y) >> (4 * (i & 7))) & 15u;
    }
    decode_block<FMT, KMS>(crow_g, crow_g8, i, t, pg, pg8, m, a0, a1, zg, zh, ktb);
    float sg = 0.0f, sh = 0.0f;
    if constexpr (FMT == QMV_FMT_FP4) {
      const uint32_t q = (uint32_t)i >> 2;
      const uint32_t wg = q == 0 ? sg0.x : q == 1 ? sg0.y : q == 2 ? sg0.z : sg0.w;
      const uint32_t wh = q == 0 ? sh0.x : q == 1 ? sh0.y : q == 2 ? sh0.z : sh0.w;
      if ((i & 3) == 0) { sg = e8m0_x2_to_f32<0>(wg, m); sh = e8m0_x2_to_f32<0>(wh, m); }
      if ((i & 3) == 1) { sg = e8m0_x2_to_f32<1>(wg, m); sh = e8m0_x2_to_f32<1>(wh, m); }
      if ((i & 3) == 2) { sg = e8m0_x2_to_f32<2>(wg, m); sh = e8m0_x2_to_f32<2>(wh, m); }
      if ((i & 3) == 3) { sg = e8m0_x2_to_f32<3>(wg, m); sh = e8m0_x2_to_f32<3>(wh, m); }
    } else if constexpr (!F::kLut) {
      const uint4& vg = (i < 8) ? sg0 : sg1;
      const uint4& vh = (i < 8) ? sh0 : sh1;
      switch (i & 7) {
        case 0: sg = half_at<0>(vg); sh = half_at<0>(vh); break;
        case 1: sg = half_at<1>(vg); sh = half_at<1>(vh); break;
        case 2: sg = half_at<2>(vg); sh = half_at<2>(vh); break;
        case 3: sg = half_at<3>(vg); sh = half_at<3>(vh); break;
        case 4: sg = half_at<4>(vg); sh = half_at<4>(vh); break;
        case 5: sg = half_at<5>(vg); sh = half_at<5>(vh); break;
        case 6: sg = half_at<6>(vg); sh = half_at<6>(vh); break;
        default: sg = half_at<7>(vg); sh = half_at<7>(vh); break;
      }
    }
    mac_block<FMT, NT>(acc, a0, a1, xr, sg, sh);
  }
}

// Batch 1: the eight MMA columns carry eight blocks instead of eight
// activation columns.  In a group of 8 blocks (16 MMA steps) lane (g, t)
// decodes blocks t (steps 0-7) and t+4 (steps 8-15) of rows g and g+8, so
// the k-slots 2t, 2t+1, 2t+8, 2t+9 of a step all belong to one block; B
// column n holds block n's activations and zeros elsewhere (lanes whose
// column is not their block read a zero region), so D[r][n] ends as block
// n's partial sum for row r and takes its own scale once per group.  Codes
// come in one 128-bit load per block and row (4-bit; two for int8).
//   crow_g / crow_g8: rows g, g+8 of the slice + this lane's block offset
//   sa_g / sa_g8:     their scale rows in the slice
//   xl0 / xl1:        activations of block t / t+4 of group 0, or the zero region
//
// int4 in this form: a nibble masked into the low bits of an fp16 is the
// subnormal n * 2^-24 (n * 2^-20 for the upper nibble of a byte), so the
// decode is one AND per two weights.  The two nibble positions accumulate
// in separate MMA sums (dlo, dhi); per block, 2^20 * (16 * dlo + dhi) is the
// exact sum of n * x, and the offset (8, or the block's zero point z for
// affine int4, staged zo bytes after the scales) is removed with the block's
// sum of activations (xsum, exact in fp64, rounded once to fp32).
template <int FMT, int NG, bool KMS>
__device__ __forceinline__ void slice_one(float (&acc)[2], float (&dl)[4], uint32_t crow_g, uint32_t crow_g8,
                                          uint32_t sa_g, uint32_t sa_g8, uint32_t zo, uint32_t xl0, uint32_t xl1,
                                          uint32_t xs_t, int t, const Palette& pg, const Palette& pg8, const Mul& m,
                                          uint32_t ktb) {
  using F = FmtT<FMT>;
  constexpr int kBB = F::kBits * 4;  // code bytes per block and row
  constexpr bool kSub = FMT == QMV_FMT_INT4 || FMT == QMV_FMT_INT4AFF;  // the subnormal int4 decode
#pragma unroll
  for (int gi = 0; gi < NG; ++gi) {
    float d[4], dh[4];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t cb = (uint32_t)((8 * gi + 4 * h) * kBB);
      uint32_t wg[8], wh[8];
      {
        const uint4 u = lds128(crow_g + cb), v = lds128(crow_g8 + cb);
        wg[0] = u.x; wg[1] = u.y; wg[2] = u.z; wg[3] = u.w;
        wh[0] = v.x; wh[1] = v.y; wh[2] = v.z; wh[3] = v.w;
        if constexpr (F::kBits == 8) {
          const uint4 u2 = lds128(crow_g + cb + 16u), v2 = lds128(crow_g8 + cb + 16u);
          wg[4] = u2.x; wg[5] = u2.y; wg[6] = u2.z; wg[7] = u2.w;
          wh[4] = v2.x; wh[5] = v2.y; wh[6] = v2.z; wh[7] = v2.w;
        }
      }
      const uint32_t xl = h ? xl1 : xl0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // word group i: in-features 8i..8i+7 of the block, MMA steps 2i and 2i+1
        const uint4 xv = lds128(xl + (uint32_t)(64 * (8 * gi + 4 * h) + 16 * i));
        uint32_t g0lo, g0hi, g1lo, g1hi, h0lo, h0hi, h1lo, h1hi;
        if constexpr (kSub) {
          // step 2i: (k0,k4), (k2,k6) as n * 2^-24; step 2i+1: (k1,k5), (k3,k7) as n * 2^-20
          const uint32_t g8 = wg[i] >> 8, h8 = wh[i] >> 8;
          const uint32_t gl0 = wg[i] & 0x000F000Fu, gl1 = g8 & 0x000F000Fu;
          const uint32_t hl0 = wh[i] & 0x000F000Fu, hl1 = h8 & 0x000F000Fu;
          const uint32_t gu0 = wg[i] & 0x00F000F0u, gu1 = g8 & 0x00F000F0u;
          const uint32_t hu0 = wh[i] & 0x00F000F0u, hu1 = h8 & 0x00F000F0u;
          if (h == 0 && i == 0) {
            mma16816_zc(d, gl0, hl0, gl1, hl1, xv.x, xv.y);
            mma16816_zc(dh, gu0, hu0, gu1, hu1, xv.z, xv.w);
          } else {
            mma16816(d, gl0, hl0, gl1, hl1, xv.x, xv.y);
            mma16816(dh, gu0, hu0, gu1, hu1, xv.z, xv.w);
          }
          continue;
        }
        if constexpr (F::kBits == 8) {
          dec_int8_word(wg[2 * i], g0lo, g0hi);
          dec_int8_word(wg[2 * i + 1], g1lo, g1hi);
          dec_int8_word(wh[2 * i], h0lo, h0hi);
          dec_int8_word(wh[2 * i + 1], h1lo, h1hi);
        } else if constexpr (FMT == QMV_FMT_FP4) {
          DecFp4::run(wg[i], g0lo, g0hi, g1lo, g1hi, m);
          DecFp4::run(wh[i], h0lo, h0hi, h1lo, h1hi, m);
        } else if constexpr (FMT == QMV_FMT_INT4) {
          DecInt4::run(wg[i], g0lo, g0hi, g1lo, g1hi, m);
          DecInt4::run(wh[i], h0lo, h0hi, h1lo, h1hi, m);
        } else {
          dec_int4km(pg, wg[i], g0lo, g0hi, g1lo, g1hi, m);
          if constexpr (KMS)  // row g+8 through the lane's palette copy in shared memory
            dec_int4km_smem(ktb, wh[i], h0lo, h0hi, h1lo, h1hi, m);
          else
            dec_int4km(pg8, wh[i], h0lo, h0hi, h1lo, h1hi, m);
        }
        if constexpr (F::kLut) {
          mma16816(dl, g0lo, h0lo, g0hi, h0hi, xv.x, xv.y);
          mma16816(dl, g1lo, h1lo, g1hi, h1hi, xv.z, xv.w);
        } else {
          if (h == 0 && i == 0)
            mma16816_zc(d, g0lo, h0lo, g0hi, h0hi, xv.x, xv.y);
          else
            mma16816(d, g0lo, h0lo, g0hi, h0hi, xv.x, xv.y);
          mma16816(d, g1lo, h1lo, g1hi, h1hi, xv.z, xv.w);
        }
      }
    }
    if constexpr (!F::kLut) {
      // lane (g, t) holds blocks 2t, 2t+1 of the group for rows g and g+8
      float s0, s1, s2, s3;
      if constexpr (FMT == QMV_FMT_FP4) {
        const uint32_t u = lds_u16(sa_g + (uint32_t)(8 * gi + 2 * t));
        const uint32_t v = lds_u16(sa_g8 + (uint32_t)(8 * gi + 2 * t));
        s0 = e8m0_x2_to_f32<0>(u, m); s1 = e8m0_x2_to_f32<1>(u, m);
        s2 = e8m0_x2_to_f32<0>(v, m); s3 = e8m0_x2_to_f32<1>(v, m);
      } else {
        const uint32_t u = lds32(sa_g + (uint32_t)(2 * (8 * gi + 2 * t)));
        const uint32_t v = lds32(sa_g8 + (uint32_t)(2 * (8 * gi + 2 * t)));
        const __half2 hu = *reinterpret_cast<const __half2*>(&u), hv = *reinterpret_cast<const __half2*>(&v);
        s0 = __low2float(hu); s1 = __high2float(hu);
        s2 = __low2float(hv); s3 = __high2float(hv);
      }
      if constexpr (FMT == QMV_FMT_INT4) {
        // block partial = 2^20 * (16 * dlo + dhi) - 8 * sum(x), one rounding each
        const float2 xs = *sptr<float2>(xs_t + (uint32_t)(4 * 8 * gi));  // blocks 2t, 2t+1 of the group
        d[0] = fmaf(fmaf(d[0], 16.0f, dh[0]), 1048576.0f, -8.0f * xs.x);
        d[1] = fmaf(fmaf(d[1], 16.0f, dh[1]), 1048576.0f, -8.0f * xs.y);
        d[2] = fmaf(fmaf(d[2], 16.0f, dh[2]), 1048576.0f, -8.0f * xs.x);
        d[3] = fmaf(fmaf(d[3], 16.0f, dh[3]), 1048576.0f, -8.0f * xs.y);
      } else if constexpr (kSub) {
        // block partial / 2^20 = (16 * dlo + dhi) - z * sum(x) / 2^20: one
        // rounding for the sum and one for the fma, as for int4 (the exact
        // power-of-two scale is restored once per row at the output); the
        // two blocks of a row go as one paired operation
        const float2 xs = *sptr<float2>(xs_t + (uint32_t)(4 * 8 * gi));  // block sums / 2^20
        const uint32_t zg = lds_u8(sa_g + zo + (uint32_t)(4 * gi + t));  // blocks 2t (low), 2t+1 (high)
        const uint32_t zh = lds_u8(sa_g8 + zo + (uint32_t)(4 * gi + t));
        // -z as floats: 2^23 minus (2^23 + z spliced into the mantissa), exact
        const uint64_t e23 = pack_f32x2(0x4B000000u, 0x4B000000u);
        const uint64_t nzg = sub_f32x2(e23, pack_f32x2(0x4B000000u | (zg & 15u), 0x4B000000u | (zg >> 4)));
        const uint64_t nzh = sub_f32x2(e23, pack_f32x2(0x4B000000u | (zh & 15u), 0x4B000000u | (zh >> 4)));
        const uint64_t x2 = pack_f32x2(__float_as_uint(xs.x), __float_as_uint(xs.y));
        const uint64_t c16 = pack_f32x2(0x41800000u, 0x41800000u);  // 16.0f
        const uint64_t tg = fma_f32x2(pack_f32x2(__float_as_uint(d[0]), __float_as_uint(d[1])), c16,
                                      pack_f32x2(__float_as_uint(dh[0]), __float_as_uint(dh[1])));
        const uint64_t th = fma_f32x2(pack_f32x2(__float_as_uint(d[2]), __float_as_uint(d[3])), c16,
                                      pack_f32x2(__float_as_uint(dh[2]), __float_as_uint(dh[3])));
        const float2 rg = unpack_f32x2(fma_f32x2(nzg, x2, tg)), rh = unpack_f32x2(fma_f32x2(nzh, x2, th));
        d[0] = rg.x;
        d[1] = rg.y;
        d[2] = rh.x;
        d[3] = rh.y;
      }
      acc[0] = fmaf(d[0], s0, acc[0]);
      acc[0] = fmaf(d[1], s1, acc[0]);
      acc[1] = fmaf(d[2], s2, acc[1]);
      acc[1] = fmaf(d[3], s3, acc[1]);
    }
  }
}


// NT: activation n-tiles of 8 columns (1 or 2); NT = 0 is the batch-1 form
// whose MMA columns carry blocks (slice_one).
// WARPS: warps per CTA (8, two CTAs per SM; or 16, one CTA per SM, when the
// staged activations leave room for only one 8-warp CTA).
// AM: fused argmax (outputs folded into per-row maxima instead of stored).
// KMS: int4km with lane palette copies in shared memory for rows g+8 (the
// host sets it where they fit; batch <= 8).
// PH: activations staged one K-phase at a time (p.xphase in-features), for
// activations beyond the on-chip staging (the general form, whole units).
template <int FMT, int NT, int WARPS, bool AM, bool KMS, bool PH>
__global__ void __launch_bounds__(32 * WARPS, WARPS == 8 ? kMinCtas : 1) mv_kernel(const __grid_constant__ MvParams p) {
  using F = FmtT<FMT>;
  constexpr bool kOne = NT == 0;
  constexpr int NTX = kOne ? 1 : NT;
  constexpr int kT = 32 * WARPS;  // threads per CTA
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ GroupTable gt;
  __shared__ int s_ids[kMaxPairs];
  __shared__ int s_nvalid;
  __shared__ unsigned long long s_best[kMaxCols];  // fused argmax: this CTA's best key per activation row
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sbase = smem_addr(smem);

  // Programmatic dependent launch: the next grid in the stream may become
  // resident as this one's blocks finish; this grid reads activations / ids
  // and writes outputs only after the preceding grid has completed.
  grid_launch_dependents();
  if (!p.prefetch) grid_wait_preceding();

  // ---- set-up (whole CTA): the column groups -----
  setup_groups<8 * NTX>(p, gt, s_ids, s_nvalid, s_best, tid);
  const uint32_t xbase = sbase + p.off_x;

  // ---- the warp's work items ------------------------------------------------
  // Units are (column group, 16-row tile) pairs, each taken by a group of P
  // warps of one CTA (P a power of two up to the CTA's warps): the group's
  // warps split the unit's K in whole granules of p.gk and add their partial
  // sums in shared memory in warp order (deterministic), behind the group's
  // own named barrier.  P is the largest power of two with P * units <= the
  // grid's warps whose parts keep at least p.min_part granules, so units are
  // spread over every warp without cutting K finer than needed; with at
  // least as many units as warps, P = 1 (whole units, no reduction).  Groups
  // are numbered group-major across CTAs, so the units of a partial last
  // round spread over the CTAs (and SMs) instead of filling whole CTAs
  // first.  Each warp streams its items through a private ring of S slices
  // (kc in-features of 16 rows) filled by 16-byte asynchronous copies S-1
  // slices ahead of the math.
  const int ngroups = gt.ngroups;
  const int64_t total = (int64_t)ngroups * p.tiles;
  const int grid = (int)gridDim.x;
  const int Kg = (int)((p.K + p.gk - 1) / p.gk);
  int P = 1;
  if (total < (int64_t)grid * WARPS && !(PH && !kOne)) {  // (then every count below fits 32 bits)
    const int units = (int)total, W = grid * WARPS;
    while (2 * P <= WARPS && units * 2 * P <= W && Kg >= 2 * P * p.min_part) P *= 2;
  }
  const int gi = warp / P, wr = warp - gi * P;  // this warp's group in the CTA, its rank in the group
  const int NG = grid * (WARPS / P);
  const int ggrp = gi * grid + (int)blockIdx.x;
  const int nitems = total > ggrp ? (int)((total - ggrp + NG - 1) / NG) : 0;
  // this warp's part of K: whole granules of p.gk
  const int kb_w = (int)min(p.K, (int64_t)(wr * Kg / P) * p.gk);
  const int ke_w = (int)min(p.K, (int64_t)((wr + 1) * Kg / P) * p.gk);
  const int KC = p.KC;
  const int nsl_w = ke_w > kb_w ? (ke_w - kb_w + KC - 1) / KC : 0;
  const int n_issue = nsl_w > 0 ? nitems : 0;  // items that move any bytes
  // a group's barrier: id 1 + gi (0 is the CTA barrier), its P warps
  auto group_sync = [&]() { asm volatile("bar.sync %0, %1;" ::"r"(1 + gi), "r"(32 * P) : "memory"); };

  struct Item {
    int64_t tile;
    int grp, kbeg, kend, nsl;
    bool split;
  };
  auto item_at = [&](int i) {
    Item it;
    const int64_t u = ggrp + (int64_t)i * NG;
    it.kbeg = kb_w; it.kend = ke_w; it.nsl = nsl_w; it.split = P > 1;
    if (ngroups == 1) {
      it.grp = 0; it.tile = u;
    } else {
      it.grp = (int)(u / p.tiles); it.tile = u - (int64_t)it.grp * p.tiles;
    }
    return it;
  };

  const int S = p.stages;
  const uint32_t ring = sbase + p.off_stage + (uint32_t)(warp * S) * p.stage_bytes;
  const uint32_t ring_end = ring + (uint32_t)S * p.stage_bytes;
  const int g = lane >> 2, t = lane & 3;
  const int cr = lane >> 1, ch = lane & 1;  // copy role: row cr of the tile, 16-byte half ch of each 32 bytes
  const Mul mul = Mul::make();
  const bool aux_fast = p.aux_mode != kAuxBlock;
  constexpr int kAuxSteps = (kSliceBytes * 8 / F::kBits / 32 * F::kSB + 15) / 16;  // 16-byte steps of scales

  // ---- issue cursor ----
  int ii = 0, ic = 0;
  Item iI{};
  // Code copies: lane (cc, rp) moves 16-byte column cc of rows 2j + rp, so each
  // instruction covers whole 128-byte lines of two rows.  Scale / palette
  // copies: lane (cr, ch) serves row cr.
  const int cc = lane & 15, rp = lane >> 4;
  const int64_t rb2 = 2 * p.code_row_bytes;
  const uint8_t* crow_base = nullptr;  // the item's tile row 0 at the next slice, + 16 * cc
  const uint8_t* asrc = nullptr;  // row cr's scales at the next slice (+ 8 * ch) / its palette (+ 16 * ch)
  const uint8_t* zsrc = nullptr;  // affine int4: row cr's zero points at the next slice (+ 4 * ch)
  int64_t irow0 = 0;
  int inrows = 0;
  auto load_issue_item = [&]() {
    iI = item_at(ii);
    irow0 = iI.tile * kTileRows;
    inrows = (int)min((int64_t)kTileRows, p.N - irow0);
    const int64_t row = min(irow0 + cr, p.N - 1);  // rows past N re-read the last row (outputs never stored)
    const int e = gt.expert[iI.grp];
    crow_base = p.codes + (int64_t)e * p.expert_code_bytes + irow0 * p.code_row_bytes + (int64_t)iI.kbeg * F::kBits / 8 + 16 * cc;
    if constexpr (F::kLut)
      asrc = p.aux + (int64_t)e * p.expert_aux_bytes + row * 32 + 16 * ch;
    else
      asrc = p.aux + (int64_t)e * p.expert_aux_bytes + row * p.aux_row_bytes + (int64_t)(iI.kbeg / 32) * F::kSB + 8 * ch;
    if constexpr (F::kZp)
      zsrc = p.aux + (int64_t)e * p.expert_aux_bytes + row * p.aux_row_bytes + p.zplane + iI.kbeg / 64 + 4 * ch;
  };
  if (n_issue > 0) load_issue_item();
  auto issue_next = [&](uint32_t stage) {
    const int k0 = iI.kbeg + ic * KC;
    const int kc = min(KC, iI.kend - k0);
    // codes: rows past N re-read the last row (their outputs are never stored)
    const int cb = kc * F::kBits / 8;  // code bytes per row, a multiple of 16
    if (16 * cc < cb) {
      uint32_t d = stage + (uint32_t)rp * p.RS + 16u * cc;
      if (inrows == kTileRows) {
        const uint8_t* q = crow_base + rp * p.code_row_bytes;
#pragma unroll
        for (int j = 0; j < kTileRows / 2; ++j) {
          cp_async16(d, q);
          q += rb2;
          d += 2u * p.RS;
        }
      } else {
#pragma unroll
        for (int j = 0; j < kTileRows / 2; ++j) {
          const int r = min(2 * j + rp, inrows - 1);
          cp_async16(d, crow_base + r * p.code_row_bytes);
          d += 2u * p.RS;
        }
      }
    }
    crow_base += cb;
    const uint32_t da = stage + p.aux_off;
    if constexpr (F::kLut) {
      if (ic == 0) cp_async16(da + (uint32_t)cr * 32u + 16u * ch, asrc);  // the palette rides with the first slice
    } else if (aux_fast) {
      const int sb = (kc / 32) * F::kSB;  // scale bytes per row, a multiple of 8
      const uint8_t* seg = asrc - 8 * ch;  // row cr's scale segment of this slice
      if ((reinterpret_cast<uintptr_t>(seg) & 15u) == 0 && sb % 16 == 0) {
        // 16-byte pieces, the row's two lanes alternating (8-byte copies of
        // scales cost several times the shared-memory wavefronts)
#pragma unroll
        for (int j = 0; j < kAuxSteps; j += 2)
          if (16 * (j + ch) < sb) cp_async16(da + (uint32_t)cr * p.AS + 16u * (j + ch), seg + 16 * (j + ch));
      } else {
#pragma unroll
        for (int j = 0; j < kAuxSteps; ++j)
          if (16 * j + 8 * ch < sb) cp_async8(da + (uint32_t)cr * p.AS + 16u * j + 8u * ch, asrc + 16 * j);
      }
      asrc += sb;
      if constexpr (F::kZp) {
        const int zb = kc / 64;  // zero-point bytes per row, a multiple of 4
        if (4 * ch < zb) cp_async4(da + (uint32_t)cr * p.AS + (uint32_t)p.zoff + 4u * ch, zsrc);
        zsrc += zb;
      }
    } else {
      // scale rows that are not 8-byte granular: plain byte loads
      const int sbytes = (kc / 32) * F::kSB;
      const int e = gt.expert[iI.grp];
      const uint8_t* abase = p.aux + (int64_t)e * p.expert_aux_bytes + irow0 * p.aux_row_bytes + (int64_t)(k0 / 32) * F::kSB;
      for (int i = lane; i < kTileRows * sbytes; i += 32) {
        const int row = i / sbytes, b = i - row * sbytes;
        const int r = min(row, inrows - 1);
        sts_u8(da + (uint32_t)row * p.AS + (uint32_t)b, ldg_u8(abase + (int64_t)r * p.aux_row_bytes + b));
      }
      if constexpr (F::kZp) {
        // slices start on even blocks: the slice's zero points are whole bytes
        const int zbytes = (kc / 32 + 1) / 2;
        const uint8_t* zbase = p.aux + (int64_t)e * p.expert_aux_bytes + irow0 * p.aux_row_bytes + p.zplane + k0 / 64;
        for (int i = lane; i < kTileRows * zbytes; i += 32) {
          const int row = i / zbytes, b = i - row * zbytes;
          const int r = min(row, inrows - 1);
          sts_u8(da + (uint32_t)row * p.AS + (uint32_t)p.zoff + (uint32_t)b,
                 ldg_u8(zbase + (int64_t)r * p.aux_row_bytes + b));
        }
      }
    }
    if (++ic == iI.nsl) {
      ic = 0;
      if (++ii < n_issue) load_issue_item();
    }
  };

  // prologue: S-1 slices in flight
  uint32_t fill = ring;
  for (int j = 0; j < S - 1; ++j) {
    if (ii < n_issue) issue_next(fill);
    cp_async_commit();
    fill += p.stage_bytes;
  }

  if (p.prefetch) grid_wait_preceding();  // weights only before this point

  // Activations are staged once per CTA: row r at xbase + r * XS, in the k
  // order the format's decoder emits (int4: (k0,k4),(k1,k5),(k2,k6),(k3,k7)
  // per 8).
  auto stage_x = [&](int64_t k_lo, int64_t k_hi) {
    const int64_t per_row = (k_hi - k_lo) / 8;
    const int64_t n16 = (int64_t)p.n_xrows * per_row;
    for (int64_t i = tid; i < n16; i += kT) {
      const int64_t r = i / per_row, j = i - r * per_row;
      const int64_t k = k_lo + 8 * j;
      uint4 v;
      if (p.xcols) {
        // the main columns of a wider activation row (the mixed format's
        // int4km part): in-feature k + e is column main_column(k + e)
        uint32_t h[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          h[e] = ldg_u16(p.x + r * p.xstride + main_column(p.xcols, p.ncols, k + e, p.xstride));
        v = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
      } else {
        v = ldg_nc_128(p.x + r * p.K + k);
      }
      if constexpr (F::kPermX && kOne) {  // (k0,k4), (k2,k6), (k1,k5), (k3,k7)
        v = make_uint4(prmt(v.x, v.z, 0x5410u), prmt(v.y, v.w, 0x5410u), prmt(v.x, v.z, 0x7632u),
                       prmt(v.y, v.w, 0x7632u));
      } else if constexpr (F::kPermX) {  // (k0,k4), (k1,k5), (k2,k6), (k3,k7)
        v = make_uint4(prmt(v.x, v.z, 0x5410u), prmt(v.x, v.z, 0x7632u), prmt(v.y, v.w, 0x5410u),
                       prmt(v.y, v.w, 0x7632u));
      }
      sts128(xbase + (uint32_t)(r * p.XS + 16 * j), v);
    }
  };
  // The activations are staged while the first weight slices are in flight
  // (all of K; or, where they do not fit on chip, one K-phase at a time in
  // the consume loop below).
  constexpr bool phased = PH && !kOne;
  {
    if (!phased) stage_x(0, p.K);
    if constexpr (kOne && (FMT == QMV_FMT_INT4 || FMT == QMV_FMT_INT4AFF)) {
      // per-block activation sums: exact in fp64 (32 fp16 terms), one rounding to fp32
      for (int64_t b = tid; b < p.K / 32; b += kT) {
        double sum = 0.0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 v = ldg_nc_128(p.x + 32 * b + 8 * q);
          const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __half2 hv = *reinterpret_cast<const __half2*>(&w4[e]);
            sum += (double)__low2float(hv) + (double)__high2float(hv);
          }
        }
        // affine int4 keeps its block partials scaled by 2^-20 (exact): the sums too
        if constexpr (FMT == QMV_FMT_INT4AFF) sum *= 0x1p-20;
        *reinterpret_cast<float*>(smem + p.off_xsum + 4 * b) = (float)sum;
      }
    }
    if constexpr (kOne) {  // the zero activations of the batch-1 form
      for (int j = tid; j < kZeroBytes / 16; j += kT) sts128(sbase + p.off_zero + 16u * j, make_uint4(0u, 0u, 0u, 0u));
    }
  }
  __syncthreads();

  // ---- consume ----
  float* red = reinterpret_cast<float*>(smem + p.off_red);  // split units: [warp][NT][4][lane]
  // One output y[pair, n]: stored, or folded into this thread's running
  // argmax for one of its columns (slot: a thread's columns are fixed for the
  // whole launch, and threads with the same t share them).
  unsigned long long best[2 * NTX];
  int bcol[2 * NTX];
#pragma unroll
  for (int i = 0; i < 2 * NTX; ++i) {
    best[i] = 0ull;
    bcol[i] = -1;
  }
  auto emit = [&](int slot, int pair, int64_t n, float v) {
    if constexpr (AM) {
      const unsigned long long k = argmax_key(v, n);
#pragma unroll
      for (int i = 0; i < 2 * NTX; ++i) {
        if (i == slot) {
          best[i] = k > best[i] ? k : best[i];
          bcol[i] = pair;
        }
      }
    } else {
      float* out = p.y + (int64_t)pair * p.N + n;
      *out = p.accum ? *out + v : v;  // accumulate: add to what the preceding kernel wrote
    }
  };
  float acc[NTX][4];
  float acc1[2], dl[4];  // batch-1 form: rows g, g+8 / the palette format's running MMA sums
  Palette pg, pg8;
  // int4km (KMS): this lane's copy of row g+8's palette, entry j at ktb +
  // 256 j.  Four warps share a 4 KB region (two 128-byte rows per entry, two
  // 16-bit halves per 4-byte slot); every lane stays in its own bank.
  const uint32_t ktb = ((sbase + (uint32_t)p.off_kmtab + 4095u) & ~4095u) + 4096u * (uint32_t)(warp >> 2) +
                       128u * (uint32_t)((warp >> 1) & 1) + 2u * (uint32_t)(warp & 1) + 4u * (uint32_t)lane;
  uint32_t xa[NTX];
  int xa_grp = -1;
  uint32_t cons = ring;
  // Phased staging: every warp runs the same rounds of whole units (a warp
  // without a unit in the last round only takes part in the staging), and
  // the CTA stages phase f's activations at the slice where it begins.
  const int rounds = phased ? (int)((total + NG - 1) / NG) : nitems;
  int xk0 = 0;  // first in-feature of the staged activations
  for (int i = 0; i < rounds; ++i) {
    const bool has = !phased || i < nitems;
    const Item it = item_at(has ? i : 0);
    const int grp = has ? it.grp : 0;
    const int64_t row0 = it.tile * kTileRows;
    const int nrows = (int)min((int64_t)kTileRows, p.N - row0);
    const int ncols = gt.count[grp], gstart = gt.start[grp];
    if (has && grp != xa_grp) {  // activation rows of this column group
      xa_grp = grp;
#pragma unroll
      for (int n = 0; n < NTX; ++n) {
        // a column the group does not use reads row 0: MMA columns are
        // independent and its outputs are never stored
        const int col = 8 * n + g;
        int xrow = 0;
        if (col < ncols) {
          const int pair = gt.sorted[gstart + col];
          xrow = p.gather ? (p.x_per_slot ? pair : pair / p.topk) : pair;
        }
        xa[n] = xbase + (uint32_t)xrow * p.XS + (uint32_t)t * 16u;
      }
    }
#pragma unroll
    for (int n = 0; n < NTX; ++n)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[n][q] = 0.0f;
    acc1[0] = acc1[1] = 0.0f;
    dl[0] = dl[1] = dl[2] = dl[3] = 0.0f;

    for (int c = 0; c < (has ? it.nsl : p.nchunks); ++c) {
      if (phased && (c * KC) % (int)p.xphase == 0) {
        // one K-phase of every activation row (the general form: natural
        // order, or int4's (k0,k4),(k1,k5),... per 8); 32-bit indices, the
        // staged phase fits in shared memory
        __syncthreads();  // every warp is done with the previous phase
        xk0 = c * KC;
        const int per_row = min((int)p.xphase, (int)p.K - xk0) / 8;
        const int n16 = p.n_xrows * per_row;
        for (int e = tid; e < n16; e += kT) {
          const int r = e / per_row, j = e - r * per_row;
          uint4 v = ldg_nc_128(p.x + (int64_t)r * p.K + xk0 + 8 * j);
          if constexpr (F::kPermX)
            v = make_uint4(prmt(v.x, v.z, 0x5410u), prmt(v.x, v.z, 0x7632u), prmt(v.y, v.w, 0x5410u),
                           prmt(v.y, v.w, 0x7632u));
          sts128(xbase + (uint32_t)(r * p.XS + 16 * j), v);
        }
        __syncthreads();
      }
      if (phased && !has) continue;
      // keep S-1 slices in flight: refill the stage freed by the previous slice
      if (ii < n_issue) issue_next(fill);
      cp_async_commit();
      fill = (fill + p.stage_bytes == ring_end) ? ring : fill + p.stage_bytes;
      cp_async_wait(S - 1);  // this slice's copies (all lanes) have landed
      __syncwarp();

      const uint32_t auxs = cons + p.aux_off;
      const int k0 = it.kbeg + c * KC;
      const int kc = min(KC, it.kend - k0);
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
          if constexpr (KMS) {
            // the lane's copy of row g+8's palette (read only by this lane,
            // after this lane's earlier lookups in program order)
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              sts_u16(ktb + 512u * j, e1[j] & 0xFFFFu);
              sts_u16(ktb + 512u * j + 256u, e1[j] >> 16);
            }
          } else {
            pg8 = palette_from_words(e1);
          }
        }
      }
      const uint32_t crow_g = cons + (uint32_t)g * p.RS, crow_g8 = cons + (uint32_t)(g + 8) * p.RS;
      const uint32_t sa_g = auxs + (uint32_t)g * p.AS, sa_g8 = auxs + (uint32_t)(g + 8) * p.AS;
      constexpr int kNB = kSliceBytes * 8 / F::kBits / 32;  // blocks in a full slice
      const uint32_t zo = (uint32_t)p.zoff;
      if constexpr (kOne) {
        // slices are whole groups of 8 blocks (the host requires K % 256 == 0)
        const uint32_t xs = xbase + (uint32_t)k0 * 2u, zb = sbase + p.off_zero;
        const uint32_t xl0 = (g == t) ? xs + 64u * t : zb;
        const uint32_t xl1 = (g == t + 4) ? xs + 64u * t : zb;
        const uint32_t tb = (uint32_t)(t * F::kBits * 4);
        const uint32_t xs_t = sbase + p.off_xsum + 4u * (uint32_t)(k0 / 32 + 2 * t);  // block sums of this lane
        if (kNB >= 16 && kc == kNB * 32)
          slice_one<FMT, (kNB >= 16 ? kNB / 8 : 1), KMS>(acc1, dl, crow_g + tb, crow_g8 + tb, sa_g, sa_g8, zo, xl0,
                                                         xl1, xs_t, t, pg, pg8, mul, ktb);
        else
          slice_one<FMT, 1, KMS>(acc1, dl, crow_g + tb, crow_g8 + tb, sa_g, sa_g8, zo, xl0, xl1, xs_t, t, pg, pg8,
                                 mul, ktb);
        __syncwarp();
        cons = (cons + p.stage_bytes == ring_end) ? ring : cons + p.stage_bytes;
        continue;
      }
      uint32_t xb[NTX];
#pragma unroll
      for (int n = 0; n < NTX; ++n) xb[n] = xa[n] + (uint32_t)(k0 - xk0) * 2u;
      if (kc == kNB * 32 && aux_fast) {
        slice_full<FMT, NTX, kNB, KMS>(acc, crow_g, crow_g8, sa_g, sa_g8, zo, xb, t, pg, pg8, mul, ktb);
      } else if (kc == kNB * 16 && aux_fast) {
        slice_full<FMT, NTX, kNB / 2, KMS>(acc, crow_g, crow_g8, sa_g, sa_g8, zo, xb, t, pg, pg8, mul, ktb);
      } else {
        const int nbc = kc / 32;
        for (int b = 0; b < nbc; ++b) {
          uint4 xr[NTX];
#pragma unroll
          for (int n = 0; n < NTX; ++n) xr[n] = lds128(xb[n] + 64u * (uint32_t)b);
          uint32_t a0[4], a1[4];
          uint32_t zg = 0u, zh = 0u;
          if constexpr (F::kZp) {
            zg = (lds_u8(sa_g + zo + (uint32_t)(b >> 1)) >> (4 * (b & 1))) & 15u;
            zh = (lds_u8(sa_g8 + zo + (uint32_t)(b >> 1)) >> (4 * (b & 1))) & 15u;
          }
          decode_block<FMT, KMS>(crow_g, crow_g8, b, t, pg, pg8, mul, a0, a1, zg, zh, ktb);
          float sg = 0.0f, sh = 0.0f;
          if constexpr (!F::kLut) {
            sg = stage_scale<FMT>(sa_g + (uint32_t)b * F::kSB, mul);
            sh = stage_scale<FMT>(sa_g8 + (uint32_t)b * F::kSB, mul);
          }
          mac_block<FMT, NTX>(acc, a0, a1, xr, sg, sh);
        }
      }
      __syncwarp();  // all lanes are done with this stage before it is refilled
      cons = (cons + p.stage_bytes == ring_end) ? ring : cons + p.stage_bytes;
    }
    if (phased && !has) continue;

    // ---- outputs: lane (g, t) holds rows g, g+8, columns 2t, 2t+1 of each n-tile ----
    const float f = (FMT == QMV_FMT_FP4) ? 0.5f : 1.0f;  // the fp4 block scales carried a factor 2
    if constexpr (kOne) {
      // (affine int4's batch-1 partials were kept scaled by 2^-20)
      const float f1 = FMT == QMV_FMT_INT4AFF ? 1048576.0f : f;
      // rows g, g+8: the four lanes of a row hold disjoint blocks; add them
      float r0 = F::kLut ? dl[0] + dl[1] : acc1[0];
      float r1 = F::kLut ? dl[2] + dl[3] : acc1[1];
      r0 += __shfl_xor_sync(0xffffffffu, r0, 1);
      r1 += __shfl_xor_sync(0xffffffffu, r1, 1);
      r0 += __shfl_xor_sync(0xffffffffu, r0, 2);
      r1 += __shfl_xor_sync(0xffffffffu, r1, 2);
      const int pair = gt.sorted[gstart];
      if (!it.split) {
        if (t == 0) {
          if (g < nrows) emit(0, pair, row0 + g, r0 * f1);
          if (g + 8 < nrows) emit(0, pair, row0 + g + 8, r1 * f1);
        }
      } else {
        if (t == 0) {
          red[warp * 16 + g] = r0;
          red[warp * 16 + g + 8] = r1;
        }
        group_sync();
        if (wr == 0 && lane < kTileRows) {  // the group's first warp adds its P partials in warp order
          float v = 0.0f;
#pragma unroll
          for (int w = 0; w < WARPS; ++w)
            if (w < P) v += red[(gi * P + w) * 16 + lane];
          if (lane < nrows) emit(0, pair, row0 + lane, v * f1);
        }
        group_sync();  // red is free again
      }
      continue;
    }
    if (!it.split) {
#pragma unroll
      for (int n = 0; n < NT; ++n) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = 8 * n + 2 * t + (q & 1);
          const int row = g + 8 * (q >> 1);
          if (col < ncols && row < nrows) {
            const int pair = gt.sorted[gstart + col];
            emit(2 * n + (q & 1), pair, row0 + row, acc[n][q] * f);
          }
        }
      }
    } else {
      // split unit: the group's P partial sums, added in warp order by the
      // group's first warp (lane (g, t) keeps its own outputs)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int q = 0; q < 4; ++q) red[((warp * NT + n) * 4 + q) * 32 + lane] = acc[n][q];
      group_sync();
      if (wr == 0) {
#pragma unroll
        for (int n = 0; n < NT; ++n) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v = 0.0f;
#pragma unroll
            for (int w = 0; w < WARPS; ++w)
              if (w < P) v += red[(((gi * P + w) * NT + n) * 4 + q) * 32 + lane];
            const int col = 8 * n + 2 * t + (q & 1);
            const int row = g + 8 * (q >> 1);
            if (col < ncols && row < nrows) {
              const int pair = gt.sorted[gstart + col];
              emit(2 * n + (q & 1), pair, row0 + row, v * f);
            }
          }
        }
      }
      group_sync();  // red is free again
    }
  }
  cp_async_wait(0);

  if constexpr (AM) argmax_finish<2 * NTX, kT>(best, bcol, s_best, s_last, p, tid, lane);
}

// ---------------------------------------------------------------------------
// Host side: geometry and launch
// ---------------------------------------------------------------------------

static int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

bool plan_matvec(int fmt, MvParams& p, int num_sms) {
  const FmtInfo fi = fmt_info(fmt);
  p.code_row_bytes = p.K * fi.bits / 8;
  p.aux_row_bytes = fi.lut ? 32 : fi.zp ? int4aff_aux_row_bytes(p.K) : (p.K / 32) * fi.scale_bytes;
  p.zplane = fi.zp ? 2 * (p.K / 32) : 0;
  p.expert_code_bytes = p.N * p.code_row_bytes;
  p.expert_aux_bytes = p.N * p.aux_row_bytes;
  p.tiles = (p.N + kTileRows - 1) / kTileRows;
  // batch 1 (dense, 4-bit formats): the block-column form, for K in whole
  // groups of 8 blocks (int8 measured faster on the general form)
  p.one = (!p.gather && p.B == 1 && p.K % 256 == 0 && fi.bits == 4) ? 1 : 0;
  p.zoff = 0;
  if (fi.lut) {
    p.aux_mode = kAuxLut;
  } else {
    // asynchronous 8-byte scale copies when every row's scales start on an
    // 8-byte boundary and come in whole 8-byte pieces (affine int4: and the
    // zero points of every slice in whole 4-byte pieces)
    const bool based = (reinterpret_cast<uintptr_t>(p.aux) % 8) == 0;
    const bool zp_ok = !fi.zp || (p.zplane % 4 == 0 && p.K % 256 == 0);
    p.aux_mode = (based && p.aux_row_bytes % 8 == 0 && zp_ok) ? kAuxRows : kAuxBlock;
    if (p.aux_mode == kAuxBlock) p.one = 0;
  }
  // A warp's K-slice: kSliceBytes of codes per row, or half of that where
  // the full ring leaves no room for enough warps (large staged activations).
  auto slice_geometry = [&](int slice_bytes) {
    const int slice = slice_bytes * 8 / fi.bits;
    p.KC = (int)(p.K < slice ? p.K : slice);
    p.nchunks = (int)((p.K + p.KC - 1) / p.KC);
    const int64_t cb = (int64_t)p.KC * fi.bits / 8;
    // Row strides chosen so a warp's shared-memory reads are free of bank
    // conflicts: 4-bit rows at 16 mod 128 bytes (32-bit loads), 8-bit rows at
    // 32 mod 128 (64-bit loads); the batch-1 form's 128-bit loads want 4-bit
    // rows at 64 mod 128 and 8-bit rows at 16 mod 128.
    if (p.one)
      p.RS = (int)(round_up(cb, 128) + (fi.bits == 4 ? 64 : 16));
    else
      p.RS = (int)(round_up(cb, 128) + (fi.bits == 4 ? 16 : 32));
    int64_t aux_region;
    if (fi.lut) {
      p.AS = 32;
      aux_region = kTileRows * 32;
    } else {
      const int64_t slice_sc = (int64_t)(p.KC / 32) * fi.scale_bytes;
      // a staged row: the slice's scales, then (affine int4) its zero points
      p.zoff = fi.zp ? (int)round_up(slice_sc, 8) : 0;
      const int64_t row_bytes = fi.zp ? p.zoff + (p.KC / 32 + 1) / 2 : slice_sc;
      int64_t j = (row_bytes + 15) / 16;
      // the batch-1 form reads 4 bytes of rows g = 0..7 per load: an odd
      // multiple of 16 bytes puts them in distinct banks (elsewhere the scale
      // loads are a few per slice and the tighter rows let more warps fit)
      if (p.one && j % 2 == 0) ++j;
      p.AS = (int)(16 * j);
      aux_region = kTileRows * p.AS;
    }
    p.aux_off = kTileRows * p.RS;
    p.stage_bytes = (int)round_up(p.aux_off + aux_region, 128);
  };
  p.n_xrows = p.gather ? (p.x_per_slot ? p.B * p.topk : p.B) : p.B;
  const int nt = p.B > 8 ? 2 : 1;
  const int64_t dyn_limit = (int64_t)kSmemLimit - kStaticSmem;
  // Layouts in order of preference (warps, CTAs per SM, slice halved):
  // two 8-warp CTAs per SM, else one 16-warp CTA (the staged activations
  // shared by 16 warps), then the 16-warp CTA with half slices (more warps
  // beat longer slices where the activations leave little room), else one
  // 8-warp CTA; within each the deepest ring (<= kStages slices per warp)
  // that fits.  (Half slices in two 8-warp CTAs measured slower than one
  // 16-warp CTA with whole slices, so that layout is not tried.)
  const int cand[5][3] = {{kWarps, kMinCtas, 0}, {2 * kWarps, 1, 0}, {2 * kWarps, 1, 1}, {kWarps, 1, 0}, {kWarps, 1, 1}};
  // one CTA per (group, tile) unit up to the resident-CTA slots
  const int64_t upper_units = (p.gather ? (int64_t)p.B * p.topk : 1) * p.tiles;
  // int4km up to 8 activation columns: lane palette copies in shared memory
  // (4 KB per four warps + alignment) where they fit beside the staging,
  // within each layout; without them otherwise.  (At 16 columns the copies
  // cost ring depth that the byte-permute lookups do not need: measured
  // slower.)
  const bool km_ok = fi.lut && p.B <= 8;
  auto try_layouts = [&](bool phased) -> bool {
    // split units divide K in granules whose code and scale segments start on
    // 16- and 8-byte boundaries
    // (affine int4: 256, so a granule's zero points start on a 4-byte boundary)
    p.gk = (p.one || fi.zp) ? 256 : (fi.lut ? 32 : (fi.scale_bytes == 1 ? 256 : 128));
    // a warp's part of a split unit keeps at least 256 in-features
    p.min_part = 256 / p.gk > 1 ? 256 / p.gk : 1;
    // staged activation rows: all of K, or one phase
    p.XS = (int)(round_up(2 * (p.xphase ? p.xphase : p.K), 128) + 64);  // 64 mod 128: conflict-free 128-bit reads
    for (int ci = 0; ci < 5; ++ci) {
      const int warps = cand[ci][0], ctas = cand[ci][1];
      if (warps != kWarps && p.one) continue;  // the batch-1 form fits two 8-warp CTAs
      if (phased && warps != 2 * kWarps) continue;  // phased staging: the 16-warp instances
      slice_geometry(cand[ci][2] ? kSliceBytes / 2 : kSliceBytes);
      for (int km = (km_ok && !phased) ? 1 : 0; km >= 0; --km) {
        p.warps = warps;
        p.km_smem = km;
        const int64_t slots = (int64_t)num_sms * ctas;
        p.grid = (int)(upper_units < slots ? upper_units : slots);
        // Units are split along K (partial sums meet in shared memory) only when
        // there are fewer than the grid's warps; a (group, tile) count of at
        // least p.tiles means that can happen only if p.tiles is below it.
        const bool may_split = p.tiles < (int64_t)p.grid * warps && p.xphase == 0;
        p.off_red = 0;  // split-unit partial sums: [warp][nt][4][32] floats
        p.off_x = may_split ? (int)round_up((int64_t)warps * nt * 4 * 32 * 4, 128) : 0;
        // the zero region starts 32 bytes past a 128-byte line: its reads and the
        // activation reads of the same instruction fall in different banks
        p.off_zero = (int)round_up(p.off_x + (int64_t)p.n_xrows * p.XS, 128) + 32;
        p.off_xsum = (int)round_up(p.off_zero + (p.one ? kZeroBytes : 0), 128);
        const bool xsum = p.one && (fmt == QMV_FMT_INT4 || fmt == QMV_FMT_INT4AFF);
        // the copies' region is aligned to 4 KB at run time: with the dynamic
        // shared memory 1 KB aligned and this offset a multiple of 1 KB, the
        // alignment moves it by at most 3 KB
        p.off_kmtab = (int)round_up(p.off_xsum + (xsum ? 4 * (p.K / 32) : 0), km ? 1024 : 128);
        const int64_t kmtab = km ? 4096 * (int64_t)((warps + 3) / 4) + 3072 : 0;
        p.off_stage = (int)round_up(p.off_kmtab + kmtab, 128);
        for (int st = kStages; st >= 2; --st) {
          const int64_t bytes = p.off_stage + (int64_t)warps * st * p.stage_bytes;
          if (bytes <= dyn_limit && ctas * (bytes + kStaticSmem + 1024) <= kSmemPerSM) {
            p.stages = st;
            p.smem_bytes = (int)bytes;
            p.ctas_per_sm = ctas;
            return true;
          }
        }
      }
    }
    return false;
  };
  p.xphase = 0;
  if (try_layouts(false)) return true;
  // Activations beyond the on-chip staging: stage them one K-phase at a time
  // (whole slices; the general form).  The fewest phases that fit.  (Not for
  // the mixed format's main part, whose staged columns are remapped.)
  if (p.xcols) return false;
  p.one = 0;
  const int64_t full_kc = kSliceBytes * 8 / fi.bits;
  int64_t prev = p.K;
  for (int64_t nph = 2; nph <= (p.K + full_kc - 1) / full_kc; ++nph) {
    p.xphase = round_up((p.K + nph - 1) / nph, full_kc);
    if (p.xphase >= prev) continue;  // the same phase as fewer phases gave
    prev = p.xphase;
    if (try_layouts(true)) return true;
  }
  p.xphase = 0;
  return false;
}

template <int FMT, int NT, int WARPS, bool AM, bool KMS = false, bool PH = false>
static cudaError_t launch_t(const MvParams& p, cudaStream_t stream) {
  static std::atomic<bool> attr_set[64];  // zero-initialised: false
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 64 && !attr_set[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(mv_kernel<FMT, NT, WARPS, AM, KMS, PH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  return cudaLaunchKernelEx(&cfg, mv_kernel<FMT, NT, WARPS, AM, KMS, PH>, p);
}

template <int FMT, bool AM>
static cudaError_t launch_fa(const MvParams& p, cudaStream_t stream) {
  // activation columns served per pass: dense B, gather at most B pairs per
  // expert when ids are distinct per token (groups are capped at 8 * NT)
  const bool wide = p.warps == 2 * kWarps;
  if (p.xphase)  // phased activation staging: 16-warp CTAs, register lookups
    return p.B > 8 ? launch_t<FMT, 2, 2 * kWarps, AM, false, true>(p, stream)
                   : launch_t<FMT, 1, 2 * kWarps, AM, false, true>(p, stream);
  if constexpr (FMT == QMV_FMT_INT4KM) {  // the palette-copy instances (batch <= 8)
    if (p.km_smem) {
      if (p.one) return launch_t<FMT, 0, kWarps, AM, true>(p, stream);
      return wide ? launch_t<FMT, 1, 2 * kWarps, AM, true>(p, stream) : launch_t<FMT, 1, kWarps, AM, true>(p, stream);
    }
  }
  if constexpr (FMT != QMV_FMT_INT8) {  // the batch-1 form (4-bit formats)
    if (p.one) return launch_t<FMT, 0, kWarps, AM>(p, stream);
  }
  if (p.B > 8) return wide ? launch_t<FMT, 2, 2 * kWarps, AM>(p, stream) : launch_t<FMT, 2, kWarps, AM>(p, stream);
  return wide ? launch_t<FMT, 1, 2 * kWarps, AM>(p, stream) : launch_t<FMT, 1, kWarps, AM>(p, stream);
}

template <int FMT>
static cudaError_t launch_f(const MvParams& p, cudaStream_t stream) {
  return p.argmax ? launch_fa<FMT, true>(p, stream) : launch_fa<FMT, false>(p, stream);
}

cudaError_t launch_matvec(int fmt, const MvParams& p, cudaStream_t stream) {
  switch (fmt) {
    case QMV_FMT_FP4: return launch_f<QMV_FMT_FP4>(p, stream);
    case QMV_FMT_INT4: return launch_f<QMV_FMT_INT4>(p, stream);
    case QMV_FMT_INT4KM: return launch_f<QMV_FMT_INT4KM>(p, stream);
    case QMV_FMT_INT8: return launch_f<QMV_FMT_INT8>(p, stream);
    case QMV_FMT_INT4AFF: return launch_f<QMV_FMT_INT4AFF>(p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace qmv
