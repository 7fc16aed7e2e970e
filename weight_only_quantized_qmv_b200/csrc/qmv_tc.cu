// qmv_tc.cu -- fp4 (E2M1 + e8m0 per 32-block) matvec for the multi-token
// verify batch on the 5th-generation tensor cores (tcgen05, sm_100a): the
// alternative to the mma.sync path of qmv_matvec.cu for 2..16 activation
// columns ("Dense-path int4km coverage...", sec. 8: FP4 dense matvec, E2M1
// grid times a per-K-block e8m0 scale; "Kernel campaign -- session handoff",
// the spec-decode verify batch).
//
// What it computes: y[c, n] = sum_k x[c, k] * e2m1(code[n, k]) * 2^(s[n, k/32] - 127),
// exact products, fp32 accumulation.
//
// One persistent CTA per SM owns 128-row tiles (the MMA's M) round robin,
// its warps split by role:
//  * warp 8 (one thread) streams the tile's codes by TMA, 128 rows x 256
//    in-features (16 KB, 128-byte swizzle) per stage of a ring, and the
//    tile's scale rows (one padded 2D box) into one of two scale buffers;
//  * warps 0-7 decode: warp w owns tensor-memory lanes 32 (w % 4) .. + 31
//    (one row each) and half w / 4 of each chunk's in-features; a thread
//    turns its 128 codes into fp16 pairs by the hardware E2M1 conversion,
//    times the block scale as an exact fp16 power of two, and writes the 64
//    words into tensor memory as the MMA's A operand (two buffers);
//  * warps 9-12 (one thread each) issue the MMAs, MMA s of a chunk by
//    issuer s % 4 (an issuing thread waits ~60 cycles per MMA at N = 16;
//    four of them keep the tensor core fed): M = 128, N = 16, K = 16 each,
//    A from tensor memory, B = the activations staged once per CTA in
//    shared memory (no-swizzle K-major layout, columns >= B zero), fp32
//    accumulators in tensor memory: eight per tile (MMA s of a chunk adds
//    into accumulator s % 8, so consecutive MMAs do not wait on each
//    other's result), two tiles in flight;
//  * warps 13-16 read each finished tile's accumulators back (tcgen05.ld),
//    sum the eight and store y.
// Scaled E2M1 values are fp16-exact for exponents 2^-23 .. 2^13.  Each row
// is decoded relative to its largest block exponent (that block at 2^13) and
// the offset, a power of two, is restored in fp32 at the output; blocks more
// than 2^36 below the row's largest are dropped (below fp32's resolution of
// the row's result).  Every wait is bounded (a second of global time); on
// expiry the kernel sets QMV_FLAG_TIMEOUT and every role stops.
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "qmv_device.cuh"
#include "qmv_internal.h"

namespace qmv {
namespace {

constexpr int kTcRows = 128;                                // MMA M: rows per tile
constexpr int kTcCols = 16;                                 // MMA N: activation columns (zero-padded)
constexpr int kTcChunk = 256;                               // in-features per staged code chunk
constexpr int kTcChunkBytes = kTcRows * kTcChunk / 2;       // 16 KB
constexpr int kTcMaxStages = 8;
constexpr int kTcDecWarps = 8;                              // decoders: lanes 32 (w % 4).., in-feature half w / 4
constexpr int kTcProdWarp = 8;                              // TMA producer
constexpr int kTcMmaWarp0 = 9, kTcMmaWarps = 4;             // MMA issuers: MMA s of a chunk by issuer s % 4
constexpr int kTcEpiWarp0 = 13, kTcWarps = 17;              // epilogue: warps 13..16
constexpr int kTcThreads = kTcWarps * 32;
constexpr int kTcStageThreads = (kTcWarps - 1) * 32;        // every warp but the producer stages x
constexpr int kTcAcc = 8;                                   // independent accumulators per tile (MMA s -> s % 8)
constexpr uint32_t kTcTmemCols = 512;                       // A0 0..127, A1 128..255, D0 256..383, D1 384..511
constexpr uint64_t kTcWaitNs = 1000000000ull;               // bounded waits: 1 s of global time
constexpr int kTcMinSmem = 120 * 1024;                      // keeps one CTA per SM (the whole tensor memory)

struct TcShared {
  uint64_t full[kTcMaxStages], empty[kTcMaxStages];  // code stages: TMA landed / decoders done
  uint64_t sfull[2], sempty[2];                      // scale buffers
  uint64_t afull[2], aempty[2];                      // A buffers in tensor memory: decoded / MMAs done
  uint64_t dfull[2], dempty[2];                      // accumulators: tile done / read back
  uint32_t tmem;
  int abort;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- tensor memory -----------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 consecutive 32-bit columns of this thread's lane
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
// 32 consecutive 32-bit columns of this thread's lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr)
      : "memory");
}

// ---- MMA, completion, barriers, TMA ------------------------------------------
// D[128 x N] (+)= A[128 x 16] (tensor memory) * B[16 x N] (shared memory, by
// descriptor); no output lane masked.
__device__ __forceinline__ void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  const uint32_t z = 0u;
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(z)
      : "memory");
}
// the mbarrier receives one arrival when every MMA this thread issued before has completed
__device__ __forceinline__ void tc_commit(uint32_t mbar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar) : "memory");
}
__device__ __forceinline__ void mbar_init(uint32_t mbar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t mbar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(mbar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t mbar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(mbar), "r"(bytes) : "memory");
}
// true once the phase of parity `parity` has completed; the thread sleeps in
// the barrier (up to 1 ms) instead of spinning, so waiting warps take no issue slots
__device__ __forceinline__ bool mbar_try(uint32_t mbar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(done)
      : "r"(mbar), "r"(parity), "r"(1000000u)
      : "memory");
  return done != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Waits for the phase of parity `parity` to complete; false when a second of
// global time passed (the CTA's abort flag is then set) or another role gave up.
__device__ __noinline__ bool tc_wait_slow(uint32_t mbar, uint32_t parity, volatile int* abort) {
  const uint64_t t0 = global_ns();
  for (;;) {
    if (mbar_try(mbar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > kTcWaitNs) {
      *abort = 1;
      return false;
    }
  }
}
__device__ __forceinline__ bool tc_wait(uint32_t mbar, uint32_t parity, volatile int* abort) {
  return mbar_try(mbar, parity) || tc_wait_slow(mbar, parity, abort);
}
// Abort path: waits at most `ns` of global time for a phase, ignoring the
// abort flag (copies and MMAs already issued complete before the CTA exits).
__device__ __noinline__ void tc_drain(uint32_t mbar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = global_ns();
  while (!mbar_try(mbar, parity) && global_ns() - t0 < ns) {
  }
}
// a 2D tile of the tensor map at (x, y) (x in elements of the innermost
// dimension) into shared memory, completing bytes on the mbarrier
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t mbar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(mbar)
      : "memory");
}

// Shared-memory matrix descriptor, no swizzle, K-major: core matrices of 8
// rows x 16 bytes (rows 16 bytes apart), the next 8 in-features at +lbo, the
// next 8 rows at +sbo; byte offsets in 16-byte units; descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor: kind::f16, A and B fp16, both K-major, D fp32, M = 128, N = 16.
constexpr uint32_t kTcIdesc = (1u << 4) | ((uint32_t)(kTcCols >> 3) << 17) | ((uint32_t)(kTcRows >> 4) << 24);

// The activations in the B layout: for each K-step s (16 in-features) a
// 512-byte block: columns 0-7 in-features 0-7 at +0, in-features 8-15 at
// +128 (lbo), columns 8-15 at +256 (sbo); column c of a core matrix at +16 c.

// the largest byte of a staged scale row (n16 16-byte pieces)
__device__ __forceinline__ int row_emax(uint32_t srow, int n16) {
  uint32_t m = 0u;
  for (int i = 0; i < n16; ++i) {
    const uint4 v = lds128(srow + 16u * i);
    m = __vmaxu4(m, __vmaxu4(__vmaxu4(v.x, v.y), __vmaxu4(v.z, v.w)));
  }
  m = __vmaxu4(m, m >> 16);
  m = __vmaxu4(m, m >> 8);
  return (int)(m & 0xFFu);
}

// fp16x2 of the block scale relative to the row's largest block (at 2^13):
// 2^(e - emax + 13), zero below 2^-23 (those blocks are dropped)
__device__ __forceinline__ uint32_t block_scale_h2(int e, int emax) {
  const int se = e - emax + 13;
  uint32_t sb = 0u;
  if (se >= -14) sb = (uint32_t)(se + 15) << 10;
  else if (se >= -23) sb = 1u << (se + 24);
  return sb * 0x10001u;
}

// 16 code bytes (32 in-features, one block) times the block scale: 16 words
// of fp16 pairs (in-features 2j, 2j + 1 in word j)
__device__ __forceinline__ void decode_block16(const uint4 c, uint32_t s2, uint32_t* a, const Mul& m) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint32_t f0, f1, f2, f3;
    DecFp4::run(w[i], f0, f1, f2, f3, m);
    a[4 * i + 0] = hmul2_u32(f0, s2);
    a[4 * i + 1] = hmul2_u32(f1, s2);
    a[4 * i + 2] = hmul2_u32(f2, s2);
    a[4 * i + 3] = hmul2_u32(f3, s2);
  }
}

}  // namespace

// Geometry of one launch (host-computed).
struct TcGeom {
  int stages;      // code stages in the ring
  int srow;        // bytes per staged scale row (K/32 + 16: the padding makes 16-byte reads conflict-free)
  int off_scale;   // dynamic shared-memory offsets (from the 1024-aligned base)
  int off_x;
  int kc;          // code chunks per tile (K / 256)
};

__global__ void __launch_bounds__(kTcThreads, 1)
    mv_fp4_tc_kernel(const __grid_constant__ MvParams p, const __grid_constant__ CUtensorMap tmap_codes,
                     const __grid_constant__ CUtensorMap tmap_scales, const TcGeom g) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ TcShared sh;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t s_stage = base, s_scale = base + g.off_scale, s_x = base + g.off_x;
  const int K = (int)p.K;
  const int64_t tiles = (p.N + kTcRows - 1) / kTcRows;
  volatile int* abort = &sh.abort;

  if (tid == kTcProdWarp * 32) {
    for (int s = 0; s < g.stages; ++s) {
      mbar_init(smem_u32(&sh.full[s]), 1);
      mbar_init(smem_u32(&sh.empty[s]), kTcDecWarps);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&sh.sfull[b]), 1);
      mbar_init(smem_u32(&sh.sempty[b]), kTcDecWarps + 4);
      mbar_init(smem_u32(&sh.afull[b]), kTcDecWarps);
      mbar_init(smem_u32(&sh.aempty[b]), kTcMmaWarps);
      mbar_init(smem_u32(&sh.dfull[b]), kTcMmaWarps);
      mbar_init(smem_u32(&sh.dempty[b]), 4);
    }
    sh.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");  // inputs may come from the preceding grid
  if (warp == 0) {
    tmem_alloc(smem_u32(&sh.tmem), kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;  // this warp's tensor-memory lanes

  if (warp == kTcProdWarp) {
    // ---- producer: scale rows and code chunks by TMA ----
    if (lane == 0) {
      uint32_t gc = 0;
      int tt = 0, nt = 0;
      const uint32_t sbytes = (uint32_t)(kTcRows * g.srow);
      for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tt) {
        const int sb = tt & 1;
        if (!tc_wait(smem_u32(&sh.sempty[sb]), ((tt >> 1) & 1) ^ 1, abort)) break;
        mbar_expect_tx(smem_u32(&sh.sfull[sb]), sbytes);
        tma_load_2d(s_scale + sb * sbytes, &tmap_scales, 0, (int)(tile * kTcRows), smem_u32(&sh.sfull[sb]));
        nt = tt + 1;
        bool ok = true;
        for (int c = 0; c < g.kc; ++c, ++gc) {
          const int st = (int)(gc % g.stages);
          if (!tc_wait(smem_u32(&sh.empty[st]), ((gc / g.stages) & 1) ^ 1, abort)) {
            ok = false;
            break;
          }
          mbar_expect_tx(smem_u32(&sh.full[st]), kTcChunkBytes);
          tma_load_2d(s_stage + st * kTcChunkBytes, &tmap_codes, c * (kTcChunk / 2), (int)(tile * kTcRows),
                      smem_u32(&sh.full[st]));
        }
        if (!ok) break;
      }
      if (*abort) {  // let the copies in flight land before the CTA exits
        for (uint32_t i = gc > (uint32_t)g.stages ? gc - g.stages : 0u; i < gc; ++i)
          tc_drain(smem_u32(&sh.full[i % g.stages]), (i / g.stages) & 1, 10000000ull);
        for (int t = nt > 2 ? nt - 2 : 0; t < nt; ++t) tc_drain(smem_u32(&sh.sfull[t & 1]), (t >> 1) & 1, 10000000ull);
      }
    }
  }

  // activations into the B layout by every warp but the producer (columns >= B
  // zero), in shared-memory order: 16-byte unit u holds column c, in-features
  // 16 (u / 32) + 8 ((u / 8) & 1) .. + 7
  if (warp != kTcProdWarp) {
    const int idx = warp < kTcProdWarp ? tid : tid - 32;
    for (int u = idx; u < kTcCols * (K / 8); u += kTcStageThreads) {
      const int c = ((u >> 4) & 1) * 8 + (u & 7), k = (u >> 5) * 16 + ((u >> 3) & 1) * 8;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (c < p.B) v = *reinterpret_cast<const uint4*>(p.x + (int64_t)c * K + k);
      asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(s_x + 16u * u), "r"(v.x), "r"(v.y), "r"(v.z),
                   "r"(v.w)
                   : "memory");
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor core
    __syncwarp();
    asm volatile("bar.sync 1, %0;" ::"n"(kTcStageThreads) : "memory");
  }

  if (warp >= kTcMmaWarp0 && warp < kTcMmaWarp0 + kTcMmaWarps) {
    // ---- MMA issuers: issuer i takes MMAs i, i + 4, i + 8, i + 12 of each
    // chunk, into accumulators i and i + 4 (one thread's MMAs wait ~60 cycles
    // each at N = 16, so four issuers keep the tensor core fed) ----
    const int i0 = warp - kTcMmaWarp0;
    if (lane == 0) {
      uint32_t gc = 0;
      int tt = 0;
      for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tt) {
        const int db = tt & 1;
        if (!tc_wait(smem_u32(&sh.dempty[db]), ((tt >> 1) & 1) ^ 1, abort)) break;
        tc_fence_after();
        const uint32_t t_d = tmem + 256u + 128u * db;
        bool ok = true;
        for (int c = 0; c < g.kc; ++c, ++gc) {
          const int ab = (int)(gc & 1u);
          if (!tc_wait(smem_u32(&sh.afull[ab]), (gc >> 1) & 1, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t t_a = tmem + 128u * ab;
#pragma unroll
          for (int s = i0; s < kTcChunk / 16; s += kTcMmaWarps)
            tc_mma_f16_ts(t_d + 16u * (s % kTcAcc), t_a + 8u * s,
                          smem_desc(s_x + (uint32_t)((c * (kTcChunk / 16) + s) * 512), 128u, 256u), kTcIdesc,
                          (c > 0 || s >= kTcAcc) ? 1u : 0u);
          tc_commit(smem_u32(&sh.aempty[ab]));  // A buffer free once these MMAs complete
        }
        if (!ok) break;
        tc_commit(smem_u32(&sh.dfull[db]));  // the tile's accumulators complete
      }
      if (*abort && gc > 0) {  // the MMAs in flight complete before tensor memory is freed
        tc_commit(smem_u32(&sh.aempty[(gc - 1) & 1u]));
        tc_drain(smem_u32(&sh.aempty[(gc - 1) & 1u]), ((gc - 1) >> 1) & 1, 10000000ull);
      }
    }
  } else if (warp < kTcDecWarps) {
    // ---- decoders ----
    const int h = warp >> 2;                 // in-feature half of each chunk (four blocks)
    const int r = (warp & 3) * 32 + lane;    // row within the tile
    const Mul mul = Mul::make();
    uint32_t gc = 0;
    int tt = 0;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tt) {
      const int sb = tt & 1;
      bool ok = tc_wait(smem_u32(&sh.sfull[sb]), (tt >> 1) & 1, abort);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      const uint32_t srow = s_scale + (uint32_t)(sb * kTcRows * g.srow + r * g.srow);
      const int emax = row_emax(srow, K / 512);
      for (int c = 0; c < g.kc && ok; ++c, ++gc) {
        const int st = (int)(gc % g.stages);
        ok = tc_wait(smem_u32(&sh.full[st]), (gc / g.stages) & 1, abort);
        if (!__all_sync(0xFFFFFFFFu, ok)) {
          ok = false;
          break;
        }
        const uint32_t crow = s_stage + (uint32_t)(st * kTcChunkBytes + r * 128);
        uint4 cv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) cv[j] = lds128(crow + ((uint32_t)((4 * h + j) ^ (r & 7)) << 4));
        const uint32_t sc = lds32(srow + 8u * c + 4u * h);
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(smem_u32(&sh.empty[st]));
          if (c == g.kc - 1) mbar_arrive(smem_u32(&sh.sempty[sb]));
        }
        const int ab = (int)(gc & 1u);
        ok = tc_wait(smem_u32(&sh.aempty[ab]), ((gc >> 1) & 1) ^ 1, abort);
        if (!__all_sync(0xFFFFFFFFu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t t_a = tmem + lane_base + 128u * ab + 64u * h;
        uint32_t a[32];
        decode_block16(cv[0], block_scale_h2((int)(sc & 0xFFu), emax), a, mul);
        decode_block16(cv[1], block_scale_h2((int)((sc >> 8) & 0xFFu), emax), a + 16, mul);
        tmem_st32(t_a, a);
        decode_block16(cv[2], block_scale_h2((int)((sc >> 16) & 0xFFu), emax), a, mul);
        decode_block16(cv[3], block_scale_h2((int)(sc >> 24), emax), a + 16, mul);
        tmem_st32(t_a + 32u, a);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&sh.afull[ab]));
      }
      if (!ok) break;
    }
  } else if (warp >= kTcEpiWarp0) {
    // ---- epilogue: accumulators of each finished tile to y ----
    const int r = (warp & 3) * 32 + lane;
    int tt = 0;
    for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tt) {
      const int b = tt & 1;
      bool ok = tc_wait(smem_u32(&sh.sfull[b]), (tt >> 1) & 1, abort);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      const int emax = row_emax(s_scale + (uint32_t)(b * kTcRows * g.srow + r * g.srow), K / 512);
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sh.sempty[b]));
      ok = tc_wait(smem_u32(&sh.dfull[b]), (tt >> 1) & 1, abort);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      // the sum of the kTcAcc accumulators, 16 columns each
      float d[16];
#pragma unroll
      for (int c = 0; c < 16; ++c) d[c] = 0.f;
#pragma unroll
      for (int j = 0; j < kTcAcc; j += 2) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + 256u + 128u * b + 16u * j, v);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) d[c] += __uint_as_float(v[c]) + __uint_as_float(v[16 + c]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sh.dempty[b]));
      const int64_t row = tile * kTcRows + r;
      if (row < p.N) {
        // 2^(emax - 140) as two normal fp32 powers of two: exact
        const int off = emax - 140, o1 = off / 2, o2 = off - o1;
        const float f1 = __uint_as_float((uint32_t)(o1 + 127) << 23);
        const float f2 = __uint_as_float((uint32_t)(o2 + 127) << 23);
#pragma unroll
        for (int c = 0; c < kTcCols; ++c)
          if (c < p.B) p.y[(int64_t)c * p.N + row] = d[c] * f1 * f2;
      }
    }
  }

  __syncwarp();  // the single-thread roles rejoin their warps
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && sh.abort) atomicOr(p.status, QMV_FLAG_TIMEOUT);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static std::atomic<void*> fn{nullptr};
  void* f = fn.load(std::memory_order_acquire);
  if (!f) {
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn.store(f, std::memory_order_release);
  }
  return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
}

TcGeom tc_geom(const MvParams& p) {
  TcGeom g{};
  g.srow = (int)(p.K / 32) + 16;
  g.kc = (int)(p.K / kTcChunk);
  const int scale_bytes = 2 * kTcRows * g.srow;
  const int x_bytes = 32 * (int)p.K;  // 16 columns x K fp16
  const int fixed = 1024 + ((scale_bytes + 127) & ~127) + x_bytes;
  g.stages = (kSmemLimit - kStaticSmem - fixed) / kTcChunkBytes;
  if (g.stages > kTcMaxStages) g.stages = kTcMaxStages;
  g.off_scale = g.stages * kTcChunkBytes;
  g.off_x = g.off_scale + ((scale_bytes + 127) & ~127);
  return g;
}

}  // namespace

// Host: the shapes this path takes (dense fp4, B in [1, 16], K a multiple of
// 512 whose 16 activation columns and two code stages fit shared memory,
// K <= 4608; 16-byte aligned operands) and its geometry.
bool plan_fp4_tc(MvParams& p, int num_sms) {
  if (p.gather || p.B < 1 || p.B > kTcCols) return false;
  if (p.K % 512 != 0 || p.K / 32 + 16 > 256) return false;
  if ((reinterpret_cast<uintptr_t>(p.codes) | reinterpret_cast<uintptr_t>(p.aux) |
       reinterpret_cast<uintptr_t>(p.x)) & 15u)
    return false;
  const TcGeom g = tc_geom(p);
  if (g.stages < 2) return false;
  const int64_t tiles = (p.N + kTcRows - 1) / kTcRows;
  p.grid = (int)(tiles < num_sms ? tiles : num_sms);
  int smem = 1024 + g.off_x + 32 * (int)p.K;
  if (smem < kTcMinSmem) smem = kTcMinSmem;
  p.smem_bytes = smem;
  p.code_row_bytes = p.K / 2;
  p.aux_row_bytes = p.K / 32;
  return true;
}

cudaError_t launch_fp4_tc(const MvParams& p, cudaStream_t stream) {
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    err = cudaFuncSetAttribute(mv_fp4_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               kSmemLimit - kStaticSmem);
    if (err != cudaSuccess) return err;
    attr_set[dev].store(true, std::memory_order_release);
  }
  PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
  if (!encode) return cudaErrorNotSupported;
  const TcGeom g = tc_geom(p);
  CUtensorMap tc, ts;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)(p.K / 2), (cuuint64_t)p.N};
    const cuuint64_t strides[1] = {(cuuint64_t)(p.K / 2)};
    const cuuint32_t box[2] = {(cuuint32_t)(kTcChunk / 2), (cuuint32_t)kTcRows};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&tc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(p.codes), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const cuuint64_t dims[2] = {(cuuint64_t)(p.K / 32), (cuuint64_t)p.N};
    const cuuint64_t strides[1] = {(cuuint64_t)(p.K / 32)};
    const cuuint32_t box[2] = {(cuuint32_t)g.srow, (cuuint32_t)kTcRows};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&ts, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(p.aux), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.grid);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = (size_t)p.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mv_fp4_tc_kernel, p, tc, ts, g);
}

}  // namespace qmv
