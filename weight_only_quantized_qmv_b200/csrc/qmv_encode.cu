// qmv_encode.cu -- block encoders (FP4 E2M1 + e8m0, symmetric int4/int8 with
// MSE clip search) and the test-only dequantizer, sm_100a.
//
// Formats and procedures: "Stream D -- Quantization (FP4 + QAT-int4):
// feasibility, first result, and plan", sec. 1 (E2M1 with e8m0 scale
// 2^(floor(log2(max_abs)) - 2) per 32-block along in-features, two codes per
// byte) and sec. 2 (symmetric int4/int8 with an MSE-optimal clip).  Every
// step is IEEE-exact and written out in a fixed order (no contraction: the
// float and double operations use the _rn intrinsics), so the codes and scales
// are bit-identical to any other correct implementation of the same steps.
//
// One thread encodes one 32-block; offline conversion is not on the decode
// path, so the encoders favour exactness and simplicity over peak bandwidth.
#include "qmv_device.cuh"

namespace qmv {

__device__ __forceinline__ void load_block(const float* W, int64_t blk, float (&w)[32]) {
  const float4* src = reinterpret_cast<const float4*>(W + blk * 32);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const float4 v = __ldg(src + j);
    w[4 * j] = v.x;
    w[4 * j + 1] = v.y;
    w[4 * j + 2] = v.z;
    w[4 * j + 3] = v.w;
  }
}

// floor(log2(a)) for finite a > 0, from the exponent field (subnormals by the
// position of the leading mantissa bit).
__device__ __forceinline__ int floor_log2_f32(float a) {
  const uint32_t bits = __float_as_uint(a);
  const int ex = (int)(bits >> 23);
  if (ex == 0) return (31 - __clz((int)bits)) - 149;
  return ex - 127;
}

__global__ void enc_fp4_kernel(const float* __restrict__ W, int64_t nblocks, uint8_t* __restrict__ codes,
                               uint8_t* __restrict__ scales, uint32_t* status) {
  for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < nblocks;
       blk += (int64_t)gridDim.x * blockDim.x) {
    float w[32];
    load_block(W, blk, w);
    float amax = 0.0f;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      finite = finite && isfinite(w[i]);
      amax = fmaxf(amax, fabsf(w[i]));
    }
    uint4 out = make_uint4(0u, 0u, 0u, 0u);
    uint32_t sbyte = 0;
    if (!finite) {
      atomicOr(status, QMV_FLAG_NONFINITE);
    } else {
      int e = (amax == 0.0f) ? -127 : floor_log2_f32(amax) - 2;
      e = max(-127, min(127, e));
      sbyte = (uint32_t)(e + 127);
      const float inv = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, e in [-127, 125]
      uint32_t words[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        // magnitudes through the hardware conversion, signs copied from the
        // weights (a negative weight that rounds to zero keeps its sign bit)
        float v[8];
        uint32_t signs = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          v[j] = __fmul_rn(fabsf(w[8 * q + j]), inv);
          signs |= (__float_as_uint(w[8 * q + j]) >> 31) << (4 * j + 3);
        }
        words[q] = f32x8_to_e2m1x8(v) | signs;
      }
      out = make_uint4(words[0], words[1], words[2], words[3]);
    }
    *reinterpret_cast<uint4*>(codes + blk * 16) = out;
    scales[blk] = (uint8_t)sbyte;
  }
}

template <int QMAX>
__global__ void enc_int_kernel(const float* __restrict__ W, int64_t nblocks, ClipList clips,
                               uint8_t* __restrict__ codes, uint16_t* __restrict__ scales, uint32_t* status) {
  constexpr int kWords = (QMAX == 7) ? 4 : 8;  // packed codes per block
  for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < nblocks;
       blk += (int64_t)gridDim.x * blockDim.x) {
    float w[32];
    load_block(W, blk, w);
    float amax = 0.0f;
    bool finite = true;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      finite = finite && isfinite(w[i]);
      amax = fmaxf(amax, fabsf(w[i]));
    }
    uint32_t best[kWords];
#pragma unroll
    for (int j = 0; j < kWords; ++j) best[j] = (QMAX == 7) ? 0x88888888u : 0u;  // q = 0
    uint16_t best_s = 0;
    bool have = false;
    double best_err = 0.0;
    if (finite) {
      for (int c = 0; c < clips.n; ++c) {
        const float sf = __fdiv_rn(__fmul_rn(clips.v[c], amax), (float)QMAX);
        const __half sh = __float2half_rn(sf);
        const uint16_t sbits = __half_as_ushort(sh);
        if ((sbits & 0x7C00u) == 0x7C00u) continue;  // fp16 overflow: clip not representable
        const float s = __half2float(sh);
        uint32_t cur[kWords];
        double err = 0.0;
#pragma unroll
        for (int j = 0; j < kWords; ++j) cur[j] = 0u;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          float r = 0.0f;
          if (s != 0.0f) {
            r = rintf(__fdiv_rn(w[i], s));
            r = fminf(fmaxf(r, (float)-QMAX), (float)QMAX);
          }
          const int q = (int)r;
          const double d = __dsub_rn((double)w[i], __dmul_rn((double)q, (double)s));
          err = __dadd_rn(err, __dmul_rn(d, d));
          if (QMAX == 7)
            cur[i / 8] |= (uint32_t)(q + 8) << (4 * (i % 8));
          else
            cur[i / 4] |= ((uint32_t)q & 0xFFu) << (8 * (i % 4));
        }
        if (!have || err < best_err) {
          have = true;
          best_err = err;
          best_s = sbits;
#pragma unroll
          for (int j = 0; j < kWords; ++j) best[j] = cur[j];
        }
      }
    }
    if (!finite) atomicOr(status, QMV_FLAG_NONFINITE);
    else if (!have) atomicOr(status, QMV_FLAG_SCALE_OVERFLOW);
    if (!have) {
#pragma unroll
      for (int j = 0; j < kWords; ++j) best[j] = (QMAX == 7) ? 0x88888888u : 0u;
      best_s = 0;
    }
    uint4* dst = reinterpret_cast<uint4*>(codes + blk * (kWords * 4));
    dst[0] = make_uint4(best[0], best[1], best[2], best[3]);
    if constexpr (kWords == 8) dst[1] = make_uint4(best[4], best[5], best[6], best[7]);
    scales[blk] = best_s;
  }
}

// Affine (asymmetric) int4 per block of 32, in the oracle's float order
// ([P3] "Quantization" / "Theoretical size"; [P1] sec. 1 int4aff): one thread
// per pair of blocks, so each thread owns whole zero-point bytes.
//   range [lo, hi] = [min(min w, 0), max(max w, 0)]; s = fp16((hi - lo) / 15);
//   z = clamp(rint(-lo / s), 0, 15); q = clamp(rint(w / s) + z, 0, 15).
__global__ void enc_aff_kernel(const float* __restrict__ W, int64_t N, int64_t K, uint8_t* __restrict__ codes,
                               uint8_t* __restrict__ aux, uint32_t* status) {
  const int64_t nb = K / 32, npair = (nb + 1) / 2, arow = int4aff_aux_row_bytes(K);
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < N * npair;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = t / npair, pr = t - n * npair;
    uint8_t* ar = aux + n * arow;
    uint32_t zbyte = 0, flags = 0;
    for (int half = 0; half < 2; ++half) {
      const int64_t b = 2 * pr + half;
      if (b >= nb) break;
      const float* w = W + n * K + b * 32;
      float v[32];
      float lo = 0.0f, hi = 0.0f;
      bool finite = true;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        v[i] = w[i];
        finite = finite && isfinite(v[i]);
        if (v[i] < lo) lo = v[i];
        if (v[i] > hi) hi = v[i];
      }
      uint16_t sh = 0;
      uint32_t z = 0;
      uint32_t q[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) q[i] = 0;
      if (!finite) {
        flags |= QMV_FLAG_NONFINITE;
      } else {
        sh = __half_as_ushort(__float2half_rn(__fdiv_rn(__fsub_rn(hi, lo), 15.0f)));
        if ((sh & 0x7C00u) == 0x7C00u) {
          flags |= QMV_FLAG_SCALE_OVERFLOW;
          sh = 0;
        } else {
          const float s = __half2float(__ushort_as_half(sh));
          if (s != 0.0f) {
            const float zf = fminf(fmaxf(rintf(__fdiv_rn(-lo, s)), 0.0f), 15.0f);
            z = (uint32_t)zf;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              q[i] = (uint32_t)fminf(fmaxf(__fadd_rn(rintf(__fdiv_rn(v[i], s)), zf), 0.0f), 15.0f);
          }
        }
      }
      ar[2 * b] = (uint8_t)(sh & 0xFFu);  // rows of an odd byte count: byte stores
      ar[2 * b + 1] = (uint8_t)(sh >> 8);
      zbyte |= z << (4 * half);
      uint8_t* cb = codes + n * (K / 2) + b * 16;
#pragma unroll
      for (int i = 0; i < 32; i += 2) cb[i / 2] = (uint8_t)(q[i] | (q[i + 1] << 4));
    }
    ar[2 * nb + pr] = (uint8_t)zbyte;
    if (flags) atomicOr(status, flags);
  }
}

// Test-only dequantizer built on the matvec kernels' own decoders, so that
// its bit-exact comparison with the oracle also checks those decoders.
__device__ __forceinline__ void f16x2_to_f32(uint32_t v, float& lo, float& hi) {
  const __half2 h = *reinterpret_cast<const __half2*>(&v);
  lo = __low2float(h);
  hi = __high2float(h);
}

template <int FMT>
__global__ void dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ aux, int64_t N,
                               int64_t K, float* __restrict__ Wdq) {
  const int64_t nblocks = N * (K / 32);
  const int64_t nb_row = K / 32;
  for (int64_t blk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; blk < nblocks;
       blk += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = blk / nb_row, b = blk - n * nb_row;
    float out[32];
    if constexpr (FMT == QMV_FMT_INT8KM) {
      // one LUT of 256 fp16 entries per 32 rows
      const uint16_t* L = reinterpret_cast<const uint16_t*>(aux) + (n / 32) * 256;
      const uint8_t* src = codes + blk * 32;
#pragma unroll
      for (int i = 0; i < 32; ++i) out[i] = __half2float(__ushort_as_half(L[src[i]]));
    } else if constexpr (FMT == QMV_FMT_INT8) {
      const uint4* src = reinterpret_cast<const uint4*>(codes + blk * 32);
      const float s = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(aux)[blk]));
      const uint4 v0 = src[0], v1 = src[1];
      const uint32_t words[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint32_t lo, hi;
        dec_int8_word(words[q], lo, hi);
        f16x2_to_f32(lo, out[4 * q], out[4 * q + 1]);
        f16x2_to_f32(hi, out[4 * q + 2], out[4 * q + 3]);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) out[i] = __fmul_rn(out[i], s);
    } else {
      const uint4 v = *reinterpret_cast<const uint4*>(codes + blk * 16);
      const uint32_t words[4] = {v.x, v.y, v.z, v.w};
      Palette pal;
      const Mul mul = Mul::make();
      if constexpr (FMT == QMV_FMT_INT4KM) {
        const uint4* L = reinterpret_cast<const uint4*>(aux + n * 32);
        const uint4 a = L[0], c = L[1];
        const uint32_t e[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
        pal = palette_from_words(e);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t s0lo, s0hi, s1lo, s1hi;
        float* o = out + 8 * q;
        if constexpr (FMT == QMV_FMT_FP4) {
          DecFp4::run(words[q], s0lo, s0hi, s1lo, s1hi, mul);  // (k0,k1) (k2,k3) (k4,k5) (k6,k7)
          f16x2_to_f32(s0lo, o[0], o[1]);
          f16x2_to_f32(s0hi, o[2], o[3]);
          f16x2_to_f32(s1lo, o[4], o[5]);
          f16x2_to_f32(s1hi, o[6], o[7]);
        } else if constexpr (FMT == QMV_FMT_INT4AFF) {
          const uint8_t* ar = aux + n * int4aff_aux_row_bytes(K);
          const uint32_t z = (ar[2 * nb_row + b / 2] >> (4 * (b & 1))) & 15u;
          DecInt4::run_z(words[q], s0lo, s0hi, s1lo, s1hi, int4_zp_sub(z), int4_zp_neg(z));  // q - z
          f16x2_to_f32(s0lo, o[0], o[4]);
          f16x2_to_f32(s0hi, o[1], o[5]);
          f16x2_to_f32(s1lo, o[2], o[6]);
          f16x2_to_f32(s1hi, o[3], o[7]);
        } else if constexpr (FMT == QMV_FMT_INT4) {
          DecInt4::run(words[q], s0lo, s0hi, s1lo, s1hi, mul);  // (k0,k4) (k1,k5) (k2,k6) (k3,k7)
          f16x2_to_f32(s0lo, o[0], o[4]);
          f16x2_to_f32(s0hi, o[1], o[5]);
          f16x2_to_f32(s1lo, o[2], o[6]);
          f16x2_to_f32(s1hi, o[3], o[7]);
        } else {
          dec_int4km(pal, words[q], s0lo, s0hi, s1lo, s1hi, mul);
          f16x2_to_f32(s0lo, o[0], o[1]);
          f16x2_to_f32(s0hi, o[2], o[3]);
          f16x2_to_f32(s1lo, o[4], o[5]);
          f16x2_to_f32(s1hi, o[6], o[7]);
        }
      }
      if constexpr (FMT == QMV_FMT_FP4) {
        const float s = e8m0_to_f32(aux[blk]);
#pragma unroll
        for (int i = 0; i < 32; ++i) out[i] = __fmul_rn(out[i], s);
      } else if constexpr (FMT == QMV_FMT_INT4) {
        const float s = __half2float(__ushort_as_half(reinterpret_cast<const uint16_t*>(aux)[blk]));
#pragma unroll
        for (int i = 0; i < 32; ++i) out[i] = __fmul_rn(out[i], s);
      } else if constexpr (FMT == QMV_FMT_INT4AFF) {
        const uint8_t* ar = aux + n * int4aff_aux_row_bytes(K);  // rows may have an odd byte count
        const float s = __half2float(__ushort_as_half((unsigned short)(ar[2 * b] | (ar[2 * b + 1] << 8))));
#pragma unroll
        for (int i = 0; i < 32; ++i) out[i] = __fmul_rn(out[i], s);
      }
    }
    float4* dst = reinterpret_cast<float4*>(Wdq + n * K + b * 32);
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[j] = make_float4(out[4 * j], out[4 * j + 1], out[4 * j + 2], out[4 * j + 3]);
  }
}

static int grid_for(int64_t nblocks, int threads, int num_sms) {
  int64_t g = (nblocks + threads - 1) / threads;
  const int64_t cap = (int64_t)num_sms * 16;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return (int)g;
}

cudaError_t launch_encode_fp4(const float* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* scales,
                              uint32_t* status, int num_sms, cudaStream_t stream) {
  const int64_t nb = N * (K / 32);
  enc_fp4_kernel<<<grid_for(nb, 256, num_sms), 256, 0, stream>>>(W, nb, codes, scales, status);
  return cudaGetLastError();
}

cudaError_t launch_encode_int(int qmax, const float* W, int64_t N, int64_t K, const ClipList& clips,
                              uint8_t* codes, uint16_t* scales, uint32_t* status, int num_sms,
                              cudaStream_t stream) {
  const int64_t nb = N * (K / 32);
  if (qmax == 7)
    enc_int_kernel<7><<<grid_for(nb, 128, num_sms), 128, 0, stream>>>(W, nb, clips, codes, scales, status);
  else
    enc_int_kernel<127><<<grid_for(nb, 128, num_sms), 128, 0, stream>>>(W, nb, clips, codes, scales, status);
  return cudaGetLastError();
}

cudaError_t launch_encode_int4aff(const float* W, int64_t N, int64_t K, uint8_t* codes, uint8_t* aux,
                                  uint32_t* status, int num_sms, cudaStream_t stream) {
  const int64_t npairs = N * ((K / 32 + 1) / 2);
  enc_aff_kernel<<<grid_for(npairs, 128, num_sms), 128, 0, stream>>>(W, N, K, codes, aux, status);
  return cudaGetLastError();
}

cudaError_t launch_dequant(int fmt, const uint8_t* codes, const uint8_t* aux, int64_t N, int64_t K, float* Wdq,
                           int num_sms, cudaStream_t stream) {
  const int64_t nb = N * (K / 32);
  const int grid = grid_for(nb, 128, num_sms);
  switch (fmt) {
    case QMV_FMT_FP4: dequant_kernel<QMV_FMT_FP4><<<grid, 128, 0, stream>>>(codes, aux, N, K, Wdq); break;
    case QMV_FMT_INT4: dequant_kernel<QMV_FMT_INT4><<<grid, 128, 0, stream>>>(codes, aux, N, K, Wdq); break;
    case QMV_FMT_INT4KM: dequant_kernel<QMV_FMT_INT4KM><<<grid, 128, 0, stream>>>(codes, aux, N, K, Wdq); break;
    case QMV_FMT_INT8: dequant_kernel<QMV_FMT_INT8><<<grid, 128, 0, stream>>>(codes, aux, N, K, Wdq); break;
    case QMV_FMT_INT4AFF: dequant_kernel<QMV_FMT_INT4AFF><<<grid, 128, 0, stream>>>(codes, aux, N, K, Wdq); break;
    case QMV_FMT_INT8KM: dequant_kernel<QMV_FMT_INT8KM><<<grid, 128, 0, stream>>>(codes, aux, N, K, Wdq); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace qmv
