// qmv_device.cuh -- device helpers shared by the libqmv kernels (sm_100a):
// shared-memory loads, the m16n8k16 tensor-core step, and the per-format
// decoders that turn packed weight codes into exact fp16 tensor-core operands.
#pragma once
#include <cstdint>
#include <cuda_fp16.h>

#include "qmv_internal.h"

namespace qmv {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// Loads
// ---------------------------------------------------------------------------

// Loads from shared memory by 32-bit shared-window address.  Plain C++ loads
// (not volatile asm), so the compiler may schedule them freely between the
// barriers and fences that order them against the asynchronous copies.
template <typename T>
__device__ __forceinline__ const T* sptr(uint32_t a) {
  return reinterpret_cast<const T*>(__cvta_shared_to_generic(a));
}
__device__ __forceinline__ uint32_t lds32(uint32_t a) { return *sptr<uint32_t>(a); }
__device__ __forceinline__ uint2 lds64(uint32_t a) { return *sptr<uint2>(a); }
__device__ __forceinline__ uint4 lds128(uint32_t a) { return *sptr<uint4>(a); }

// ---------------------------------------------------------------------------
// Tensor-core step: D(16x8, f32) = A(16x16, f16, row) * B(16x8, f16, col) + C
// Fragment of lane l (g = l/4, t = l%4):
//   a0 = (row g,   k 2t,2t+1)   a1 = (row g+8, k 2t,2t+1)
//   a2 = (row g,   k 2t+8,2t+9) a3 = (row g+8, k 2t+8,2t+9)
//   b0 = (k 2t,2t+1; col g)     b1 = (k 2t+8,2t+9; col g)
//   d0,d1 = (row g, cols 2t,2t+1)   d2,d3 = (row g+8, cols 2t,2t+1)
// Products of fp16 operands are exact in fp32; the sum accumulates in fp32.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The same step with a zero accumulator input (no per-block zeroing of d).
__device__ __forceinline__ void mma16816_zc(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                            uint32_t b0, uint32_t b1) {
  const float z = 0.0f;
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%10,%10,%10};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
}

// ---------------------------------------------------------------------------
// Byte/bit helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {  // (a & b) | c
  uint32_t r;  // truth table: (0xF0 & 0xCC) | 0xAA = 0xEA
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

__device__ __forceinline__ uint32_t lop3_mux(uint32_t a, uint32_t b, uint32_t m) {  // m ? b : a, bitwise
  uint32_t r;
  // truth table over (a, b, m) = (0xF0, 0xCC, 0xAA): (m & b) | (~m & a) = 0xD8
  asm("lop3.b32 %0, %1, %2, %3, 0xD8;" : "=r"(r) : "r"(a), "r"(b), "r"(m));
  return r;
}

__device__ __forceinline__ uint32_t hsub2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t hfma2_u32(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

// byte `i` (0..3, compile-time) of w, two E2M1 codes -> f16x2 (low nibble in
// the low half).  Exact: every E2M1 value is an fp16 value.
template <int I>
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t w) {
  uint32_t r;
  if constexpr (I == 0)
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n cvt.rn.f16x2.e2m1x2 %0, b0;\n}" : "=r"(r) : "r"(w));
  else if constexpr (I == 1)
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n cvt.rn.f16x2.e2m1x2 %0, b1;\n}" : "=r"(r) : "r"(w));
  else if constexpr (I == 2)
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n cvt.rn.f16x2.e2m1x2 %0, b2;\n}" : "=r"(r) : "r"(w));
  else
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n cvt.rn.f16x2.e2m1x2 %0, b3;\n}" : "=r"(r) : "r"(w));
  return r;
}

// Eight non-negative floats -> four bytes of E2M1 code pairs (v[2j] in the low
// nibble of byte j), round to nearest even, saturating at 6 (hardware
// conversion; its first source operand fills the high nibble).
__device__ __forceinline__ uint32_t f32x8_to_e2m1x8(const float (&v)[8]) {
  uint32_t r;
  asm("{\n .reg .b8 c0, c1, c2, c3;\n"
      " cvt.rn.satfinite.e2m1x2.f32 c0, %2, %1;\n"
      " cvt.rn.satfinite.e2m1x2.f32 c1, %4, %3;\n"
      " cvt.rn.satfinite.e2m1x2.f32 c2, %6, %5;\n"
      " cvt.rn.satfinite.e2m1x2.f32 c3, %8, %7;\n"
      " mov.b32 %0, {c0, c1, c2, c3};\n}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// e8m0 byte -> float 2^(byte - 127), exact (byte 0 is the subnormal 2^-127).
__device__ __forceinline__ float e8m0_to_f32(uint32_t byte) {
  uint32_t bits = byte << 23;
  return __uint_as_float(bits > 0x00400000u ? bits : 0x00400000u);
}

// ---------------------------------------------------------------------------
// Per-format decoders: one 32-bit word of a row's codes (8 weights, k = 8t..8t+7
// of one 32-block for the 4-bit formats; 4 weights for int8) -> fp16 operands
// for the two m16n8k16 steps of that block.  The k order the decoder emits is
// the order the activations are staged in shared memory (see the kernel's
// activation staging).
// ---------------------------------------------------------------------------

// A 32-bit constant the compiler cannot fold, so that multiplies by powers of
// two stay integer multiply-adds (the FMA pipe) instead of turning into
// shifts and masks on the half-rate integer ALU pipe.
__device__ __forceinline__ uint32_t opaque(uint32_t c) {
  uint32_t r;
  asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(c));
  return r;
}

// Multipliers kept opaque so the decoders' shifts-by-multiply stay integer
// multiply-adds on the FMA pipe.
struct Mul {
  uint32_t p4, p8, p16, e23;  // 2^4, 2^8, 2^16, 2^23
  __device__ __forceinline__ static Mul make() {
    Mul m;
    m.p4 = opaque(1u << 4);
    m.p8 = opaque(1u << 8);
    m.p16 = opaque(1u << 16);
    m.e23 = opaque(1u << 23);
    return m;
  }
};

// two E2M1 codes in byte I of r -> f16x2
template <int I>
__device__ __forceinline__ uint32_t e2m1x2_byte_to_f16x2(uint32_t r) {
  uint32_t o;
  if constexpr (I == 0)
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n cvt.rn.f16x2.e2m1x2 %0, b0;\n}" : "=r"(o) : "r"(r));
  else if constexpr (I == 1)
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n cvt.rn.f16x2.e2m1x2 %0, b1;\n}" : "=r"(o) : "r"(r));
  else if constexpr (I == 2)
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n cvt.rn.f16x2.e2m1x2 %0, b2;\n}" : "=r"(o) : "r"(r));
  else
    asm("{\n .reg .b8 b0, b1, b2, b3;\n mov.b32 {b0, b1, b2, b3}, %1;\n cvt.rn.f16x2.e2m1x2 %0, b3;\n}" : "=r"(o) : "r"(r));
  return o;
}

// FP4: pairs (k0,k1) (k2,k3) for step 0, (k4,k5) (k6,k7) for step 1: one
// hardware conversion per byte, each reading its byte of w in place.
struct DecFp4 {
  __device__ __forceinline__ static void run(uint32_t w, uint32_t& s0lo, uint32_t& s0hi, uint32_t& s1lo,
                                             uint32_t& s1hi, const Mul& m) {
    (void)m;
    s0lo = e2m1x2_byte_to_f16x2<0>(w);
    s0hi = e2m1x2_byte_to_f16x2<1>(w);
    s1lo = e2m1x2_byte_to_f16x2<2>(w);
    s1hi = e2m1x2_byte_to_f16x2<3>(w);
  }
};

// Byte i (0..3) of u -> float 2^(byte - 126) (exact, always normal): the
// e8m0 scale times 2.  Callers fold the factor 1/2 into their outputs.
template <int I>
__device__ __forceinline__ float e8m0_x2_to_f32(uint32_t u, const Mul& m) {
  // bytes 0..2 by a byte permute (ALU), byte 3 by a multiply-high (FMA pipe)
  const uint32_t byte = (I < 3) ? prmt(u, 0u, 0x4440u + I) : (u >> 24);
  return __uint_as_float(byte * m.e23 + m.e23);
}

// INT4 (nibble = q + 8): 0x6400 | n is the fp16 1024 + n; subtracting 1032
// gives q exactly.  Nibbles at bits 4..7 of each half come out as 1024 + 16 n
// and are mapped with an exact fma: (1024 + 16 n) / 16 - 72 = n - 8.
// Emitted pairs: (k0,k4) (k1,k5) for step 0 and (k2,k6) (k3,k7) for step 1.
struct DecInt4 {
  __device__ __forceinline__ static void run(uint32_t w, uint32_t& s0lo, uint32_t& s0hi, uint32_t& s1lo,
                                             uint32_t& s1hi, const Mul& m) {
    (void)m;
    // zero point 8: subtract 1032 from the low nibbles, -72 after the 1/16 scaling of the high ones
    run_z(w, s0lo, s0hi, s1lo, s1hi, 0x64086408u, 0xD480D480u);
  }
  // Any zero point z (affine int4): sub = fp16x2 (1024 + z), neg = fp16x2 -(64 + z);
  // the results n - z are small integers, exact in fp16.
  __device__ __forceinline__ static void run_z(uint32_t w, uint32_t& s0lo, uint32_t& s0hi, uint32_t& s1lo,
                                               uint32_t& s1hi, uint32_t sub, uint32_t neg) {
    const uint32_t kMagic = 0x64006400u;      // fp16x2 (1024, 1024)
    const uint32_t kSixteenth = 0x2C002C00u;  // fp16x2 (1/16, 1/16)
    const uint32_t w8 = w >> 8;
    s0lo = hsub2_u32(lop3_and_or(w, 0x000F000Fu, kMagic), sub);
    s0hi = hfma2_u32(lop3_and_or(w, 0x00F000F0u, kMagic), kSixteenth, neg);
    s1lo = hsub2_u32(lop3_and_or(w8, 0x000F000Fu, kMagic), sub);
    s1hi = hfma2_u32(lop3_and_or(w8, 0x00F000F0u, kMagic), kSixteenth, neg);
  }
};
// The run_z constants of zero point z (0..15): fp16 1024 + z is 0x6400 + z,
// fp16 -(64 + z) is 0xD400 + 16 z (ulp 1/16 at 64).
__device__ __forceinline__ uint32_t int4_zp_sub(uint32_t z) { return (0x6400u + z) * 0x00010001u; }
__device__ __forceinline__ uint32_t int4_zp_neg(uint32_t z) { return (0xD400u + 16u * z) * 0x00010001u; }

// INT8: one word holds 4 weights (k0..k3).  Bias each byte by 128, splice it
// under 0x64 (fp16 1024 + u), subtract 1152: exact q.  Pairs (k0,k1) (k2,k3).
__device__ __forceinline__ void dec_int8_word(uint32_t w, uint32_t& lo, uint32_t& hi) {
  const uint32_t u = w ^ 0x80808080u;
  const uint32_t kSub = 0x64806480u;  // fp16x2 (1152, 1152)
  lo = hsub2_u32(prmt(u, 0x64646464u, 0x5140u), kSub);
  hi = hsub2_u32(prmt(u, 0x64646464u, 0x5342u), kSub);
}

// INT4KM: 16-entry fp16 palette of one row held as byte tables in registers:
// lo[0..3] = low bytes of entries 0..15, hi[0..3] = high bytes.  Four indices
// (one per byte lane of `sel`, bit 3 in `msk`) look up 4 bytes per table with
// two byte-permutes over the 8-entry halves and a bitwise select on bit 3.
struct Palette {
  uint32_t lo0, lo1, lo2, lo3, hi0, hi1, hi2, hi3;
};

__device__ __forceinline__ Palette palette_from_words(const uint32_t (&e)[8]) {
  // e[j] = entries 2j (low half) and 2j+1 (high half)
  Palette p;
  p.lo0 = prmt(e[0], e[1], 0x6420u);
  p.lo1 = prmt(e[2], e[3], 0x6420u);
  p.lo2 = prmt(e[4], e[5], 0x6420u);
  p.lo3 = prmt(e[6], e[7], 0x6420u);
  p.hi0 = prmt(e[0], e[1], 0x7531u);
  p.hi1 = prmt(e[2], e[3], 0x7531u);
  p.hi2 = prmt(e[4], e[5], 0x7531u);
  p.hi3 = prmt(e[6], e[7], 0x7531u);
  return p;
}

// w: 8 nibbles (k0..k7).  Emits (k0,k1) (k2,k3) (k4,k5) (k6,k7) as f16x2.
__device__ __forceinline__ void dec_int4km(const Palette& p, uint32_t w, uint32_t& s0lo, uint32_t& s0hi,
                                           uint32_t& s1lo, uint32_t& s1hi, const Mul& m) {
  const uint32_t w4 = w * m.p4;  // w << 4 on the multiply pipe (the lookups load the ALU)
  // byte permutes read only the low 16 bits of their selector
  const uint32_t sel0 = w & 0x77777777u;  // bit 3 of every nibble cleared; nibbles 0..3 in the low half
  const uint32_t sel1 = sel0 >> 16;       // nibbles 4..7
  const uint32_t m0 = prmt(w4, w, 0xD9C8u);  // byte i = 0xFF iff bit 3 of nibble i
  const uint32_t m1 = prmt(w4, w, 0xFBEAu);  // nibbles 4..7
  const uint32_t lo_a = lop3_mux(prmt(p.lo0, p.lo1, sel0), prmt(p.lo2, p.lo3, sel0), m0);
  const uint32_t hi_a = lop3_mux(prmt(p.hi0, p.hi1, sel0), prmt(p.hi2, p.hi3, sel0), m0);
  const uint32_t lo_b = lop3_mux(prmt(p.lo0, p.lo1, sel1), prmt(p.lo2, p.lo3, sel1), m1);
  const uint32_t hi_b = lop3_mux(prmt(p.hi0, p.hi1, sel1), prmt(p.hi2, p.hi3, sel1), m1);
  s0lo = prmt(lo_a, hi_a, 0x5140u);
  s0hi = prmt(lo_a, hi_a, 0x7362u);
  s1lo = prmt(lo_b, hi_b, 0x5140u);
  s1hi = prmt(lo_b, hi_b, 0x7362u);
}

// INT4KM through a lane-private copy of one row's palette in shared memory,
// a second lookup unit beside the byte permutes (which load the ALU pipe).
// Entry j of the lane's copy is the 16-bit word at tb + 256 j, in the lane's
// own bank, so the warp's 32 loads are one conflict-free wavefront; tb has
// bits 8..11 clear, so a nibble standing at bits 8..11 of a word is its own
// offset: one LOP3 ((v & 0xF00) | tb) forms each address.  Nibble 2 is in
// place, nibbles 0 and 1 move up by a multiply (FMA pipe), nibble 3 and the
// word's high half take one shift each, after which the high half's nibbles
// 4..6 move like 0..2.  Per 8 weights: 3 shifts and 8 address LOP3s on the
// ALU pipe (the byte-permute form takes 19), 8 16-bit loads, and 4
// multiply-adds pack entry pairs into f16x2.  Emits (k0,k1) (k2,k3) (k4,k5)
// (k6,k7) like dec_int4km.
__device__ __forceinline__ uint32_t km_entry(uint32_t v, uint32_t tb) {
  return *sptr<uint16_t>(lop3_and_or(v, 0xF00u, tb));
}

__device__ __forceinline__ void dec_int4km_smem(uint32_t tb, uint32_t w, uint32_t& s0lo, uint32_t& s0hi,
                                                uint32_t& s1lo, uint32_t& s1hi, const Mul& m) {
  const uint32_t hi = w >> 16;
  const uint32_t e0 = km_entry(w * m.p8, tb);
  const uint32_t e1 = km_entry(w * m.p4, tb);
  const uint32_t e2 = km_entry(w, tb);
  const uint32_t e3 = km_entry(w >> 4, tb);
  const uint32_t e4 = km_entry(hi * m.p8, tb);
  const uint32_t e5 = km_entry(hi * m.p4, tb);
  const uint32_t e6 = km_entry(hi, tb);
  const uint32_t e7 = km_entry(hi >> 4, tb);
  s0lo = e1 * m.p16 + e0;
  s0hi = e3 * m.p16 + e2;
  s1lo = e5 * m.p16 + e4;
  s1hi = e7 * m.p16 + e6;
}

}  // namespace qmv
