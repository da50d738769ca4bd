// Blackwell (sm_100a) building blocks for the tensor-core chunk kernel:
// mbarriers with bounded waits, TMA tile loads, TMEM allocation, tcgen05 MMA
// issue/commit, TMEM loads, and the 128-byte-swizzled shared-memory operand
// layouts the MMA descriptors describe.
//
// Operand layouts (bf16, SWIZZLE_128B, 1024-byte aligned atoms):
//   K-major tile, R rows x (64*KA) columns: KA column blocks ("k-atoms") of
//     R rows x 128 bytes each, one after the other.  Element (row, col) lives
//     at  katom*R*128 + row*128 + (((col%64)/8) ^ (row%8))*16 + (col%8)*2.
//     Descriptor: SBO = 1024 (8-row group stride), LBO unused (1); the K=16
//     step ks starts at katom(ks)*R*128 + (ks%4)*32.
//   MN-major tile, K rows x (64*MB) MN-elements: MB blocks of 64 MN-elements,
//     each K rows x 128 bytes.  Element (mn, k) lives at
//     (mn/64)*K*128 + k*128 + (((mn%64)/8) ^ (k%8))*16 + (mn%8)*2.
//     Descriptor: LBO = K*128 (MN-block stride), SBO = 1024 (8-k-row group
//     stride); the K=16 step ks starts at ks*2048.
// The swizzle is the address-based XOR of byte-address bits [4,7) with bits
// [7,10), matching the hardware's SWIZZLE_128B mode.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "kda_common.cuh"

namespace kda {

// The driver's tensor-map encoder (cuTensorMapEncodeTiled), looked up once through
// the runtime; null if the driver does not provide it.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

namespace tc {

// ---------------------------------------------------------------------------
// Shared-memory addresses and proxies
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Make generic-proxy shared-memory writes visible to the async proxy (MMA/TMA).
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// mbarrier with bounded waits
// ---------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with the given parity to complete; give up after about
// `limit_ns` nanoseconds and return false (the caller records a timeout).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity,
                                          uint64_t limit_ns = 2000000000ull) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0 && globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// All threads of the CTA wait for a barrier phase; false (and a recorded
// timeout) if any thread gave up.  Also acts as a CTA-wide barrier.
__device__ __forceinline__ bool wait_all(uint64_t *bar, uint32_t parity, int *status) {
  const bool ok = mbar_wait(bar, parity);
  if (__syncthreads_or(!ok)) {
    if (threadIdx.x == 0) report(status, KDA_ERR_DEVICE_TIMEOUT);
    return false;
  }
  return true;
}

// Error exit of a kernel whose wait ran out: one thread waits (bounded) for the
// current phase of each of the CTA's mbarriers, so that a bulk copy or an MMA
// that is still in flight lands before the CTA frees its TMEM and exits.  A
// barrier with nothing in flight simply runs out after limit_ns.  The current
// phase's parity is read from the barrier itself: try_wait.parity(0) succeeds
// exactly when the current phase is odd.
__device__ __forceinline__ void drain(uint64_t *bar, uint64_t limit_ns = 100000000ull) {
  const uint32_t cur = mbar_try_wait(bar, 0u) ? 1u : 0u;
  (void)mbar_wait(bar, cur, limit_ns);
}

// ---------------------------------------------------------------------------
// TMA (tensor tile loads; no multicast)
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tma_prefetch_desc(const void *tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *smem_dst, const void *tmap, uint64_t *bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *smem_dst, const void *tmap, uint64_t *bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

// Untiled bulk copies (addresses 16-byte aligned, sizes multiples of 16 bytes).
// Global -> shared, completion counted in bytes on `bar`.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes,
                                          uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(gsrc)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// Shared -> global, tracked by bulk groups of the issuing thread.
__device__ __forceinline__ void bulk_store(void *gdst, const void *smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(gdst)),
               "r"(smem_u32(smem_src)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The issuing thread's bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// The issuing thread's bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMEM
// ---------------------------------------------------------------------------

// Whole-warp: allocate `ncols` TMEM columns, base address written to *slot.
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(slot)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t base, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Warp-collective: 32 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Warp-collective: 16 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Issue-only variants: the registers are valid after tmem_wait_ld.
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, float (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]),
        "=f"(v[7]), "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]),
        "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32_nowait(uint32_t taddr, float (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]),
        "=f"(v[7]), "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]),
        "=f"(v[13]), "=f"(v[14]), "=f"(v[15]), "=f"(v[16]), "=f"(v[17]), "=f"(v[18]),
        "=f"(v[19]), "=f"(v[20]), "=f"(v[21]), "=f"(v[22]), "=f"(v[23]), "=f"(v[24]),
        "=f"(v[25]), "=f"(v[26]), "=f"(v[27]), "=f"(v[28]), "=f"(v[29]), "=f"(v[30]),
        "=f"(v[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld8_nowait(uint32_t taddr, float (&v)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]),
        "=f"(v[7])
      : "r"(taddr));
}
// Wait for this thread's outstanding tcgen05.ld; the register arrays are tied
// to the wait so the compiler does not read them before it.
template <int A, int B>
__device__ __forceinline__ void tmem_wait_ld(float (&a)[A], float (&b)[B]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < A; ++i) asm volatile("" : "+f"(a[i]));
#pragma unroll
  for (int i = 0; i < B; ++i) asm volatile("" : "+f"(b[i]));
}

// Warp-collective: 8 consecutive fp32 columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------------------
// MMA descriptors and issue
// ---------------------------------------------------------------------------

// Instruction descriptor: kind::f16 with fp32 accumulate, dense; A and B
// share one input type (bf16 when `bf16`, else fp16).
__host__ __device__ constexpr uint32_t idesc_f16kind(int M, int N, bool a_mn_major,
                                                     bool b_mn_major, bool bf16) {
  return (1u << 4)                                 // D format: f32
         | ((bf16 ? 1u : 0u) << 7)                 // A format: 1 = bf16, 0 = f16
         | ((bf16 ? 1u : 0u) << 10)                // B format
         | ((a_mn_major ? 1u : 0u) << 15)          // A major
         | ((b_mn_major ? 1u : 0u) << 16)          // B major
         | ((uint32_t)(N >> 3) << 17)              // N / 8
         | ((uint32_t)(M >> 4) << 24);             // M / 16
}
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return idesc_f16kind(M, N, a_mn_major, b_mn_major, true);
}
__host__ __device__ constexpr uint32_t idesc_fp16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return idesc_f16kind(M, N, a_mn_major, b_mn_major, false);
}

// Instruction descriptor: kind::tf32 (fp32 operands read as tf32), fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                 // D format: f32
         | (2u << 7)                               // A format: tf32
         | (2u << 10)                              // B format: tf32
         | ((a_mn_major ? 1u : 0u) << 15)          // A major
         | ((b_mn_major ? 1u : 0u) << 16)          // B major
         | ((uint32_t)(N >> 3) << 17)              // N / 8
         | ((uint32_t)(M >> 4) << 24);             // M / 16
}

// Shared-memory matrix descriptor for a SWIZZLE_128B operand.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

// Shared-memory matrix descriptor for a SWIZZLE_64B MN-major operand of 32
// 16-bit MN-elements (one 64-byte swizzle atom wide): K-row stride 64 B,
// 8-row group stride (SBO) 512 B.  Element (mn, k) lives at
//   k*64 + (((mn/8) ^ ((k/2) % 4)) * 16) + (mn%8)*2
// (the XOR of byte-address bits [4,6) with [7,9), on 512-byte aligned tiles).
// Descriptor of K-step ks (16 K-rows).
__device__ __forceinline__ uint64_t desc_mn32_sw64(uint32_t tile, int ks) {
  const uint32_t saddr = tile + (uint32_t)(ks * 1024);
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((512u >> 4) & 0x3FFFu) << 16;   // LBO: next 32-element atom; unused at N=32
                                                   // (kept small so the tile's reads stay inside it)
  d |= (uint64_t)((512u >> 4) & 0x3FFFu) << 32;   // SBO: 8 K-rows
  d |= (uint64_t)1 << 46;                          // descriptor version (sm_100)
  d |= (uint64_t)4 << 61;                          // SWIZZLE_64B
  return d;
}

// Byte offset of the 16-byte chunk c (MN-elements [8c, 8c+8)) of K-row k in such a tile.
__device__ __forceinline__ uint32_t mn32_sw64_off(int k, int c) {
  return (uint32_t)(k * 64 + ((c ^ ((k >> 1) & 3)) << 4));
}

// K-major tile of `rows` rows: descriptor of K-step ks (16 bf16 columns).
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int rows, int ks) {
  return sdesc(tile + (uint32_t)((ks >> 2) * rows * 128 + (ks & 3) * 32), 16, 1024);
}

// MN-major tile of `krows` K-rows: descriptor of K-step ks (16 K-rows).
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int krows, int ks) {
  return sdesc(tile + (uint32_t)(ks * 2048), (uint32_t)(krows * 128), 1024);
}

// One thread: D[tmem] (+)= A * B^T for one K=16 step.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// One thread: D[tmem] (+)= A * B^T for one K=8 step of tf32 operands (32 bytes of K, the
// same byte step as a K=16 step of 16-bit operands).
__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// fp32 rounded to the nearest tf32 (10-bit significand), as the fp32 bit pattern.
__device__ __forceinline__ uint32_t tf32_rna(float x) {
  // Round to nearest, ties away from zero, on the bit pattern: add half of the dropped
  // 13-bit field to the magnitude and clear the field (a carry into the exponent is the
  // correct rounding up).  Finite inputs only.  Two integer operations; the same result
  // as the PTX conversion cvt.rna.tf32.f32, which issued more slowly here.
  return (__float_as_uint(x) + 0x1000u) & 0xffffe000u;
}

// One thread: arrive once on `bar` when all previously issued MMAs complete.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// Operand tile addressing (byte offsets inside a tile)
// ---------------------------------------------------------------------------

// K-major: 16-byte chunk c8 of `row` (columns [8*c8, 8*c8+8) of a 16-bit tile, or
// [4*c8, 4*c8+4) of a 32-bit one).
__device__ __forceinline__ uint32_t kmaj_off(int rows, int row, int c8) {
  return (uint32_t)((c8 >> 3) * rows * 128 + row * 128 + (((c8 & 7) ^ (row & 7)) << 4));
}

// MN-major: 16-byte chunk holding MN-elements [8*m8, 8*m8+8) of K-row `k`.
__device__ __forceinline__ uint32_t mnmaj_off(int krows, int k, int m8) {
  return (uint32_t)((m8 >> 3) * krows * 128 + k * 128 + (((m8 & 7) ^ (k & 7)) << 4));
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&f)[8]) {
  uint4 u;
  __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  return u;
}

__device__ __forceinline__ uint4 pack8_f16(const float (&f)[8]) {
  uint4 u;
  __half2 *h = reinterpret_cast<__half2 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(f[2 * i], f[2 * i + 1]);
  return u;
}

__device__ __forceinline__ void st_shared_16(uint8_t *base, uint32_t off, uint4 v) {
  *reinterpret_cast<uint4 *>(base + off) = v;
}

}  // namespace tc
}  // namespace kda
