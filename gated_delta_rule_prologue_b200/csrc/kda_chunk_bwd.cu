// Backward of the two-pass tensor-core prefill: gradients of o and of the final
// state with respect to q, k, v, g, beta and the initial state.
//
// The pages mention training ("Kimi K3的线性注意力：从源码看懂KDA如何更新记忆",
// 彩蛋) but give no backward; this is the chain rule through the chunk algebra
// of the forward (kda_chunk_record.cuh).  With R = diag(beta)(V - (K G) S),
// U = (I + A)^{-1} R, K' = K G_last / G, dO' = scale dO, and dS' the adjoint of a
// chunk's exit state:
//   dU  = P^T dO' + K' dS'                 dS = diag(G_last) dS' + (Q G)^T dO' - W^T dU
// (W = (I + A)^{-1} diag(beta) K G), so the adjoint state runs backwards through
// the chunks by the transpose of the forward's affine map ("KimiK3轻量化复刻实现KDA
// 并行解析，Chunkwise并行与状态压缩机制详解", Figure 1).  Two passes:
//
// * chunk_bwd_state_kernel: one CTA (128 threads) per (sequence, head, 32 value
//   channels), chunks in reverse order, on the forward's records.  Per chunk,
//   tcgen05 MMAs with fp32 accumulators in TMEM:
//     D_u = P^T (scale dO) + K' dS'        (M = 128 of which rows 0..63 are used;
//                                           P^T is the record's P tile read
//                                           MN-major, K' its K-major tile)
//     dU  = D_u + <q_r, k_r> scale dO_r    (fp32 diagonal term)
//     D_s = [W^T | (Q G)^T] [-dU ; scale dO]   (the record's [W; Q G] tile read
//                                               MN-major, K = 128)
//     dS  = diag(G_last) dS' + D_s         (fp32 registers; thread = key channel)
//   It writes dS' (the adjoint of every chunk's exit state) and the gradient of
//   the initial state.
//
// * chunk_bwd_local_kernel: one CTA (256 threads) per (chunk, head), fp32 on CUDA
//   cores.  From the chunk's entry state (saved by the forward state pass) and
//   dS', it walks the chunk in sub-chunks of 16 tokens: in a 16-token block the
//   in-block log-decay is at least -80 when g >= -5, so exp(+-gamma) stay in fp32
//   range and the chunk algebra applies with plain factors.  Sub-chunk sb is
//   reached by recomputing the forward through sub-chunks 0..sb-1 from the entry
//   state; its backward (the same relations as the float64 chunkwise backward
//   oracle) gives dq, dk, dv, dg, dbeta and the adjoint entering the sub-chunk
//   before it.
#include <cuda_fp16.h>

#include "kda_chunk_record.cuh"
#include "kda_common.cuh"
#include "kda_tcgen05.cuh"

namespace kda {
namespace {
using namespace tc;

// ----------------------------------------------------------------------------
// Reverse state pass
// ----------------------------------------------------------------------------

constexpr int kBT = 128;
constexpr int kSlices = 4;
constexpr uint32_t BB_A1 = 0;       // [W ; Q G] (record), read MN-major            32 KB
constexpr uint32_t BB_KP = 32768;   // K' (record, K-major 64 rows) then P          24 KB
constexpr uint32_t BB_P = 49152;
constexpr uint32_t BB_DS = 57344;   // dS' operand: 128 key rows x 32 values, 64-byte swizzle  8 KB
constexpr uint32_t BB_B2 = 65536;   // [-dU ; scale dO]: 128 token rows x 32 values             8 KB
constexpr uint32_t BB_BAR = 73728;  // three mbarriers, TMEM slot
constexpr uint32_t BB_ALLOC = BB_BAR + 64 + 1024;
constexpr uint32_t TB_DU = 0, TB_DS = 32, TB_COLS = 64;
// P^T is an M = 128 MN-major operand whose second MN block (rows 64..127 of D_u,
// never read back) lies over the dS' tile; K' as an M = 128 K-major operand reads
// its rows 64..127 from the next k-atom and P: all inside the allocation.
static_assert(BB_P + 8192 == BB_DS, "P^T's unused MN block overlays the dS' tile");

__global__ void __launch_bounds__(kBT, 3)
chunk_bwd_state_kernel(const uint8_t *__restrict__ ws, const int32_t *__restrict__ cu,
                       const float *dsN, const float *__restrict__ dout, float scale, int N,
                       int T, int H, float *__restrict__ dckpt, float *ds0, int *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int slice = blockIdx.x % kSlices;
  const int nh = blockIdx.x / kSlices, h = nh % H, n = nh / H;
  const int32_t *cprefix = reinterpret_cast<const int32_t *>(ws);
  const uint8_t *recs = ws + rec::header_bytes(N);
  uint64_t *bar_a1 = reinterpret_cast<uint64_t *>(sm + BB_BAR);
  uint64_t *bar_kp = bar_a1 + 1, *bar_mma = bar_a1 + 2;
  uint32_t *slot = reinterpret_cast<uint32_t *>(sm + BB_BAR + 32);

  int bos, eos;
  seq_bounds(cu, n, T, status, bos, eos);
  int cbase = 0, nch = (eos - bos + 63) / 64;
  if (cu) {
    cbase = cprefix[n];
    nch = cprefix[n + 1] - cbase;
  }
  {  // debug builds: the chain's chunks lie inside the workspace and its tokens inside T
    const long long cap = rec::chunk_capacity(N, T);
    if (nch > 0 && !(in_range(status, cbase, cap) && in_range(status, cbase + nch - 1, cap) &&
                     in_range(status, eos - 1, T)))
      return;
  }
  if (warp == 0) tmem_alloc(slot, TB_COLS);
  if (tid == 0) {
    mbar_init(bar_a1, 1);
    mbar_init(bar_kp, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
  }
  // dS[i] = dS'[key t][value 32 slice + i]; stored value-major [dv][dk] like the state.
  const int t = tid;
  const size_t head_off = ((size_t)n * H + h) * 128 * 128;
  const size_t sbase = (size_t)slice * 32 * 128 + t;
  float dS[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) dS[i] = dsN ? dsN[head_off + sbase + (size_t)i * 128] : 0.f;

  auto write_ds_operand = [&]() {
    float amax = 0.f;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        f[e] = dS[8 * x + e];
        amax = fmaxf(amax, fabsf(f[e]));
      }
      st_shared_16(sm + BB_DS, mn32_sw64_off(t, x), pack8_f16(f));
    }
    if (!(amax < 32768.f)) report(status, KDA_ERR_DEVICE_RANGE);
  };
  write_ds_operand();
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t lane_addr = static_cast<uint32_t>(32 * warp) << 16;

  auto rec_of = [&](int c) -> const uint8_t * {
    return recs + ((size_t)(cbase + c) * H + h) * rec::BYTES;
  };
  auto load_a1 = [&](int c) {
    mbar_arrive_expect_tx(bar_a1, 32768);
    bulk_load(sm + BB_A1, rec_of(c) + rec::A1, 32768, bar_a1);
  };
  auto load_kp = [&](int c) {
    mbar_arrive_expect_tx(bar_kp, 24576);
    bulk_load(sm + BB_KP, rec_of(c) + rec::KP, 24576, bar_kp);
  };
  if (tid == 0 && nch > 0) {
    load_a1(nch - 1);
    load_kp(nch - 1);
  }

  uint32_t pa = 0, pk = 0, pm = 0;
  bool failed = false;  // a wait ran out: copies or MMAs may still be in flight
  for (int c = nch - 1; c >= 0; --c) {
    const int t0 = bos + 64 * c, Lc = min(64, eos - t0);
    const uint8_t *rp = rec_of(c);
    {  // the adjoint of this chunk's exit state, for the local pass
      float *dst = dckpt + ((size_t)(cbase + c) * H + h) * (128 * 128) + sbase;
#pragma unroll
      for (int i = 0; i < 32; ++i) dst[(size_t)i * 128] = dS[i];
    }
    // scale dO of token r (warps 0-1: TMEM lanes 0..63 are the chunk's tokens)
    float sdo[32];
    float pd = 0.f;
    if (warp < 2) {
      const int r = tid;
      if (r < Lc) {
        const float4 *src = reinterpret_cast<const float4 *>(
            dout + ((size_t)(t0 + r) * H + h) * 128 + slice * 32);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float4 f = __ldg(src + x);
          sdo[4 * x] = scale * f.x;
          sdo[4 * x + 1] = scale * f.y;
          sdo[4 * x + 2] = scale * f.z;
          sdo[4 * x + 3] = scale * f.w;
        }
        pd = __ldg(reinterpret_cast<const float *>(rp + rec::PD) + r);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) sdo[i] = 0.f;
      }
      float amax = 0.f;
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          f[e] = sdo[8 * x + e];
          amax = fmaxf(amax, fabsf(f[e]));
        }
        st_shared_16(sm + BB_B2, mn32_sw64_off(64 + r, x), pack8_f16(f));
      }
      if (!(amax < 32768.f)) report(status, KDA_ERR_DEVICE_RANGE);
    }
    const float gl = __ldg(reinterpret_cast<const float *>(rp + rec::GL) + t);
    fence_async_smem();
    tc_fence_before();
    if (!wait_all(bar_kp, pk, status)) {
      failed = true;
      break;
    }  // K', P of this chunk; also a CTA barrier
    pk ^= 1;

    // ---- D_u = P^T (scale dO) + K' dS' -------------------------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t p = smem_u32(sm + BB_P), kp = smem_u32(sm + BB_KP);
      const uint32_t b2 = smem_u32(sm + BB_B2), dso = smem_u32(sm + BB_DS);
      constexpr uint32_t idT = idesc_fp16(128, 32, true, true);
      constexpr uint32_t idK = idesc_fp16(128, 32, false, true);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16(tmem + TB_DU, desc_mnmajor(p, 64, ks), desc_mn32_sw64(b2 + 4096, ks), idT,
                 ks > 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_bf16(tmem + TB_DU, desc_kmajor(kp, 64, ks), desc_mn32_sw64(dso, ks), idK, 1);
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, pm, status)) {
      failed = true;
      break;
    }
    pm ^= 1;
    tc_fence_after();
    if (tid == 0 && c > 0) load_kp(c - 1);  // K' and P have been read

    // ---- dU (fp32), then -dU as the upper half of the second B operand ----------------------
    if (warp < 2) {
      const int r = tid;
      float du[32];
      tmem_ld32(tmem + lane_addr + TB_DU, du);
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        du[i] = r < Lc ? -fmaf(pd, sdo[i], du[i]) : 0.f;
        amax = fmaxf(amax, fabsf(du[i]));
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = du[8 * x + e];
        st_shared_16(sm + BB_B2, mn32_sw64_off(r, x), pack8_f16(f));
      }
      if (!(amax < 32768.f)) report(status, KDA_ERR_DEVICE_RANGE);
    }
    fence_async_smem();
    tc_fence_before();
    if (!wait_all(bar_a1, pa, status)) {
      failed = true;
      break;
    }  // [W; Q G] of this chunk; also a CTA barrier
    pa ^= 1;

    // ---- D_s = [W^T | (Q G)^T] [-dU ; scale dO] ----------------------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t a1 = smem_u32(sm + BB_A1), b2 = smem_u32(sm + BB_B2);
      constexpr uint32_t idT = idesc_fp16(128, 32, true, true);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_bf16(tmem + TB_DS, desc_mnmajor(a1, 128, ks), desc_mn32_sw64(b2, ks), idT, ks > 0);
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, pm, status)) {
      failed = true;
      break;
    }
    pm ^= 1;
    tc_fence_after();
    if (tid == 0 && c > 0) load_a1(c - 1);  // [W; Q G] has been read
    {
      float ds[32];
      tmem_ld32(tmem + lane_addr + TB_DS, ds);
#pragma unroll
      for (int i = 0; i < 32; ++i) dS[i] = fmaf(gl, dS[i], ds[i]);
    }
    __syncthreads();
    write_ds_operand();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  if (ds0 && !failed) {
#pragma unroll
    for (int i = 0; i < 32; ++i) ds0[head_off + sbase + (size_t)i * 128] = dS[i];
  }
  if (failed && tid == 0) {  // let in-flight record copies and MMAs land first
    drain(bar_a1);
    drain(bar_kp);
    drain(bar_mma);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, TB_COLS);
}

// ----------------------------------------------------------------------------
// Local pass: fp32, 16-token sub-chunks
// ----------------------------------------------------------------------------

constexpr int kLT = 256;       // threads
constexpr int kSub = 16;       // tokens per sub-chunk
constexpr int RS = 132;        // row stride (floats) of the 128-wide shared matrices: eight
                               // consecutive rows start 4 banks apart
constexpr int SS = 17;         // row stride of the 16 x 16 matrices

struct LocalSmem {
  float S[128 * RS];    // entry state of the current sub-chunk, [key][value]
  float dS[128 * RS];   // adjoint of the current sub-chunk's exit state, [key][value]
  float G[kSub * RS];   // exp(gamma), gamma the in-sub-chunk inclusive cumsum of g
  float KG[kSub * RS];  // k exp(gamma)
  float KD[kSub * RS];  // k exp(-gamma)
  float QG[kSub * RS];  // q exp(gamma)
  float KP[kSub * RS];  // k exp(gamma_last - gamma)
  float E[kSub * RS];   // v - (K G) S
  float U[kSub * RS];   // (I + A)^{-1} diag(beta) E
  float dO[kSub * RS];  // scale dO
  float dU[kSub * RS];  // dU, then dR in place
  float A[kSub * SS];   // strict lower beta_r <k_r G_r, k_i / G_i>
  float KK[kSub * SS];  // <k_r G_r, k_i / G_i>
  float P[kSub * SS];   // lower <q_r G_r, k_i / G_i> (diagonal included)
  float dP[kSub * SS];
  float dA[kSub * SS];
  float beta[kSub];
  float gc[128];        // exp(gamma_last)
  float xch[2][128];    // per-key partial sums passed between the two row halves
};

// Pairs of fp32 lanes on the packed instructions (one issue for two lanes, each lane
// rounded as its scalar fma): the low and high halves of a float4.
__device__ __forceinline__ float2 lo2(const float4 &v) { return make_float2(v.x, v.y); }
__device__ __forceinline__ float2 hi2(const float4 &v) { return make_float2(v.z, v.w); }
__device__ __forceinline__ float2 dup2(float a) { return make_float2(a, a); }

// Persistent grid: one CTA per SM, each with a scratch slot for the entry states of
// sub-chunks 1..3 of its current chunk (written by the forward walk, read back by the
// backward walk; 192 KB per CTA, resident in L2).
constexpr int kLocalCTAs = 148;
constexpr size_t kLocalSlotFloats = (size_t)3 * 128 * 128;

template <typename Tin>
__global__ void __launch_bounds__(kLT, 1)
chunk_bwd_local_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k,
                       const Tin *__restrict__ v, const float *__restrict__ g,
                       const float *__restrict__ beta, const float *__restrict__ dout,
                       float scale, const int32_t *__restrict__ cu, const uint8_t *ws,
                       const float *__restrict__ ckpt, const float *__restrict__ dckpt,
                       float *__restrict__ scratch, long long items, int N, int T, int H,
                       float *__restrict__ dq, float *__restrict__ dk, float *__restrict__ dv,
                       float *__restrict__ dg, float *__restrict__ dbeta, int *status) {
  extern __shared__ float4 smem_f4[];
  LocalSmem &sm = *reinterpret_cast<LocalSmem *>(smem_f4);
  const int tid = threadIdx.x;
  const int32_t *cprefix = reinterpret_cast<const int32_t *>(ws);
  float *slot = scratch + (size_t)blockIdx.x * kLocalSlotFloats;

  // thread roles
  const int rr = tid >> 4, c8 = tid & 15;     // (row, 8 value columns) for 16 x 128 outputs
  const int ca = 4 * c8, cb = 64 + 4 * c8;    // its columns: [ca, ca+4) and [cb, cb+4)
  const int kt = tid & 127, rh = tid >> 7;    // (key, rows 8 rh .. 8 rh + 7): a warp holds 32 keys
  const int kq = tid & 63, q4 = tid >> 6;     // (keys kq and kq + 64, value chunks 16 m + 4 q4)

  // [value][key] in global <-> [key][value] in shared memory.  Lane l moves key
  // base + l % 8 of value row j0 + l / 8: the 32 lanes hit 32 distinct banks, and
  // the global side reads 32-byte runs of keys.
  auto load_state = [&](float *dst, const float *src) {
    for (int idx = tid; idx < 128 * 128; idx += kLT) {
      const int w = idx >> 5, l = idx & 31;           // w: 512 groups of 32
      const int key = 8 * (w & 15) + (l & 7), j = 4 * (w >> 4) + (l >> 3);
      dst[key * RS + j] = src[(size_t)j * 128 + key];
    }
  };
  auto store_state = [&](float *dst, const float *src) {
    for (int idx = tid; idx < 128 * 128; idx += kLT) {
      const int w = idx >> 5, l = idx & 31;
      const int key = 8 * (w & 15) + (l & 7), j = 4 * (w >> 4) + (l >> 3);
      dst[(size_t)j * 128 + key] = src[key * RS + j];
    }
  };

  for (long long it = blockIdx.x; it < items; it += gridDim.x) {
    const int h = (int)(it % H), ci = (int)(it / H);
    // ---- which chunk (uniform over the CTA) ---------------------------------------------
    int n = 0, c = ci;
    if (cu) {
      if (ci >= cprefix[N]) break;  // items are in chunk order: none left
      int lo = 0, hi = N - 1;       // last n with cprefix[n] <= ci
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cprefix[mid] <= ci) lo = mid;
        else hi = mid - 1;
      }
      n = lo;
      c = ci - cprefix[n];
    } else if (ci >= (T + 63) / 64) {
      break;
    }
    int bos, eos;
    seq_bounds(cu, n, T, status, bos, eos);
    const int t0 = bos + 64 * c, Lc = min(64, eos - t0);
    if (Lc <= 0) continue;
    // debug builds: the chunk's record and checkpoints, and its tokens, are in range
    if (!in_range(status, ci, rec::chunk_capacity(N, T)) || !in_range(status, t0 + Lc - 1, T))
      continue;
    const int nsub = (Lc + kSub - 1) / kSub;
    const size_t rec_idx = (size_t)ci * H + h;
    const float *S0 = ckpt + rec_idx * (128 * 128);
    const float *dS1 = dckpt + rec_idx * (128 * 128);

    // Inputs of sub-chunk sb: G, KG, KD, QG, KP, E (= v for now), dO (scaled), beta, gc.
    auto load_sub = [&](int sb, bool with_grad) {
      const int r0 = kSub * sb;
      {  // g (raw) into G, beta
        const int r = rr, tok = t0 + r0 + r;
        const bool ok = r0 + r < Lc;
        const size_t base = ((size_t)(ok ? tok : 0) * H + h) * 128;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const int col = part ? cb : ca;
          float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
          if (ok) f = __ldg(reinterpret_cast<const float4 *>(g + base + col));
          *reinterpret_cast<float4 *>(&sm.G[r * RS + col]) = f;
        }
        if (c8 == 0) sm.beta[r] = ok ? __ldg(beta + (size_t)tok * H + h) : 0.f;
      }
      __syncthreads();
      if (tid < 128) {  // inclusive cumsum over the rows, per key channel
        float run = 0.f;
#pragma unroll
        for (int r = 0; r < kSub; ++r) {
          run += sm.G[r * RS + tid];
          sm.G[r * RS + tid] = run;
        }
        sm.gc[tid] = __expf(run);
        // a 16-token block needs its log-decay within fp32's exp range (g >= -5 gives >= -80)
        if (!(run >= -87.f)) report(status, KDA_ERR_DEVICE_RANGE);
      }
      __syncthreads();
      {
        const int r = rr, tok = t0 + r0 + r;
        const bool ok = r0 + r < Lc;
        const size_t base = ((size_t)(ok ? tok : 0) * H + h) * 128;
        float gm[8];
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const int col = part ? cb : ca;
          float kv[4] = {0.f, 0.f, 0.f, 0.f}, qv[4] = {0.f, 0.f, 0.f, 0.f};
          float vv[4] = {0.f, 0.f, 0.f, 0.f}, dv4[4] = {0.f, 0.f, 0.f, 0.f};
          if (ok) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              kv[e] = to_f32(k[base + col + e]);
              qv[e] = to_f32(q[base + col + e]);
              vv[e] = to_f32(v[base + col + e]);
            }
            if (with_grad) {
              const float4 f = __ldg(reinterpret_cast<const float4 *>(dout + base + col));
              dv4[0] = scale * f.x; dv4[1] = scale * f.y; dv4[2] = scale * f.z; dv4[3] = scale * f.w;
            }
          }
          const float4 gam4 = *reinterpret_cast<const float4 *>(&sm.G[r * RS + col]);
          const float4 gl4 = *reinterpret_cast<const float4 *>(&sm.G[(kSub - 1) * RS + col]);
          const float gam[4] = {gam4.x, gam4.y, gam4.z, gam4.w};
          const float glast[4] = {gl4.x, gl4.y, gl4.z, gl4.w};
          float kg[4], kd[4], qg[4], kpv[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float Gv = __expf(gam[e]), Gi = __expf(-gam[e]);
            gm[4 * part + e] = Gv;
            kg[e] = kv[e] * Gv;
            kd[e] = kv[e] * Gi;
            qg[e] = qv[e] * Gv;
            kpv[e] = kv[e] * __expf(glast[e] - gam[e]);
          }
          const int o = r * RS + col;
          *reinterpret_cast<float4 *>(&sm.KG[o]) = make_float4(kg[0], kg[1], kg[2], kg[3]);
          *reinterpret_cast<float4 *>(&sm.KD[o]) = make_float4(kd[0], kd[1], kd[2], kd[3]);
          *reinterpret_cast<float4 *>(&sm.QG[o]) = make_float4(qg[0], qg[1], qg[2], qg[3]);
          *reinterpret_cast<float4 *>(&sm.KP[o]) = make_float4(kpv[0], kpv[1], kpv[2], kpv[3]);
          *reinterpret_cast<float4 *>(&sm.E[o]) = make_float4(vv[0], vv[1], vv[2], vv[3]);
          *reinterpret_cast<float4 *>(&sm.dO[o]) = make_float4(dv4[0], dv4[1], dv4[2], dv4[3]);
        }
        __syncthreads();  // gamma of the last row has been read by every thread
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const int col = part ? cb : ca;
          *reinterpret_cast<float4 *>(&sm.G[r * RS + col]) =
              make_float4(gm[4 * part], gm[4 * part + 1], gm[4 * part + 2], gm[4 * part + 3]);
        }
      }
      __syncthreads();
    };

    // E = V - (K G) S;  KK, A, P;  U = (I + A)^{-1} diag(beta) E.
    auto forward_local = [&](bool with_p) {
      {
        const float4 e1 = *reinterpret_cast<const float4 *>(&sm.E[rr * RS + ca]);
        const float4 e2 = *reinterpret_cast<const float4 *>(&sm.E[rr * RS + cb]);
        float2 acc[4] = {lo2(e1), hi2(e1), lo2(e2), hi2(e2)};
#pragma unroll 4
        for (int key = 0; key < 128; ++key) {
          const float2 na = dup2(-sm.KG[rr * RS + key]);
          const float4 s1 = *reinterpret_cast<const float4 *>(&sm.S[key * RS + ca]);
          const float4 s2 = *reinterpret_cast<const float4 *>(&sm.S[key * RS + cb]);
          acc[0] = __ffma2_rn(na, lo2(s1), acc[0]);
          acc[1] = __ffma2_rn(na, hi2(s1), acc[1]);
          acc[2] = __ffma2_rn(na, lo2(s2), acc[2]);
          acc[3] = __ffma2_rn(na, hi2(s2), acc[3]);
        }
        // each thread rewrites only the entries it read
        *reinterpret_cast<float4 *>(&sm.E[rr * RS + ca]) = make_float4(acc[0].x, acc[0].y, acc[1].x, acc[1].y);
        *reinterpret_cast<float4 *>(&sm.E[rr * RS + cb]) = make_float4(acc[2].x, acc[2].y, acc[3].x, acc[3].y);
      }
      {  // 16 x 16 Grams: thread (r, i)
        const int r = tid >> 4, i = tid & 15;
        float kk = 0.f, pp = 0.f;
#pragma unroll 4
        for (int key = 0; key < 128; key += 4) {
          const float4 kd = *reinterpret_cast<const float4 *>(&sm.KD[i * RS + key]);
          const float4 kg = *reinterpret_cast<const float4 *>(&sm.KG[r * RS + key]);
          kk = fmaf(kg.x, kd.x, kk); kk = fmaf(kg.y, kd.y, kk);
          kk = fmaf(kg.z, kd.z, kk); kk = fmaf(kg.w, kd.w, kk);
          if (with_p) {
            const float4 qg = *reinterpret_cast<const float4 *>(&sm.QG[r * RS + key]);
            pp = fmaf(qg.x, kd.x, pp); pp = fmaf(qg.y, kd.y, pp);
            pp = fmaf(qg.z, kd.z, pp); pp = fmaf(qg.w, kd.w, pp);
          }
        }
        sm.KK[r * SS + i] = kk;
        sm.A[r * SS + i] = i < r ? sm.beta[r] * kk : 0.f;
        sm.P[r * SS + i] = i <= r ? pp : 0.f;
      }
      __syncthreads();
      if (tid < 128) {  // forward substitution, one value column per thread
        const int j = tid;
        float u[kSub];
#pragma unroll
        for (int r = 0; r < kSub; ++r) {
          float x = sm.beta[r] * sm.E[r * RS + j];
#pragma unroll
          for (int i = 0; i < r; ++i) x = fmaf(-sm.A[r * SS + i], u[i], x);
          u[r] = x;
          sm.U[r * RS + j] = x;
        }
      }
      __syncthreads();
    };

    // S <- diag(G_last) S + K'^T U   (thread (keys kq, kq + 64; value chunks 16 m + 4 q4))
    auto advance_state = [&]() {
      float2 st[2][16];
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const int key = kq + 64 * kk;
        const float2 gck = dup2(sm.gc[key]);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const float4 x = *reinterpret_cast<const float4 *>(&sm.S[key * RS + 16 * m + 4 * q4]);
          st[kk][2 * m] = __fmul2_rn(gck, lo2(x));
          st[kk][2 * m + 1] = __fmul2_rn(gck, hi2(x));
        }
      }
#pragma unroll 2
      for (int r = 0; r < kSub; ++r) {
        const float2 kp0 = dup2(sm.KP[r * RS + kq]), kp1 = dup2(sm.KP[r * RS + kq + 64]);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const float4 u = *reinterpret_cast<const float4 *>(&sm.U[r * RS + 16 * m + 4 * q4]);
          st[0][2 * m] = __ffma2_rn(kp0, lo2(u), st[0][2 * m]);
          st[0][2 * m + 1] = __ffma2_rn(kp0, hi2(u), st[0][2 * m + 1]);
          st[1][2 * m] = __ffma2_rn(kp1, lo2(u), st[1][2 * m]);
          st[1][2 * m + 1] = __ffma2_rn(kp1, hi2(u), st[1][2 * m + 1]);
        }
      }
#pragma unroll
      for (int kk = 0; kk < 2; ++kk)
#pragma unroll
        for (int m = 0; m < 8; ++m)
          *reinterpret_cast<float4 *>(&sm.S[(kq + 64 * kk) * RS + 16 * m + 4 * q4]) =
              make_float4(st[kk][2 * m].x, st[kk][2 * m].y, st[kk][2 * m + 1].x, st[kk][2 * m + 1].y);
      __syncthreads();
    };

    // ---- forward walk: entry states of sub-chunks 1 .. nsub-1 into the scratch slot -------
    load_state(sm.S, S0);
    __syncthreads();
    for (int j = 0; j + 1 < nsub; ++j) {
      load_sub(j, false);
      forward_local(false);
      advance_state();
      store_state(slot + (size_t)j * 128 * 128, sm.S);
    }
    load_state(sm.dS, dS1);

    // ---- backward walk -------------------------------------------------------------------
    for (int sb = nsub - 1; sb >= 0; --sb) {
      if (sb < nsub - 1) {  // the last sub-chunk's entry state is still in place
        __syncthreads();    // every thread is done with the previous sub-chunk's state
        load_state(sm.S, sb == 0 ? S0 : slot + (size_t)(sb - 1) * 128 * 128);
      }
      __syncthreads();
      load_sub(sb, true);
      forward_local(true);
      const int r0 = kSub * sb;

      // ---- dU = P^T dO' + K' dS'  (thread (r, 8 value columns)) ----------------------------
      {
        float2 acc[4] = {dup2(0.f), dup2(0.f), dup2(0.f), dup2(0.f)};
#pragma unroll
        for (int i = 0; i < kSub; ++i) {
          const float2 p = dup2(sm.P[i * SS + rr]);
          const float4 d1 = *reinterpret_cast<const float4 *>(&sm.dO[i * RS + ca]);
          const float4 d2 = *reinterpret_cast<const float4 *>(&sm.dO[i * RS + cb]);
          acc[0] = __ffma2_rn(p, lo2(d1), acc[0]);
          acc[1] = __ffma2_rn(p, hi2(d1), acc[1]);
          acc[2] = __ffma2_rn(p, lo2(d2), acc[2]);
          acc[3] = __ffma2_rn(p, hi2(d2), acc[3]);
        }
#pragma unroll 4
        for (int key = 0; key < 128; ++key) {
          const float2 a = dup2(sm.KP[rr * RS + key]);
          const float4 s1 = *reinterpret_cast<const float4 *>(&sm.dS[key * RS + ca]);
          const float4 s2 = *reinterpret_cast<const float4 *>(&sm.dS[key * RS + cb]);
          acc[0] = __ffma2_rn(a, lo2(s1), acc[0]);
          acc[1] = __ffma2_rn(a, hi2(s1), acc[1]);
          acc[2] = __ffma2_rn(a, lo2(s2), acc[2]);
          acc[3] = __ffma2_rn(a, hi2(s2), acc[3]);
        }
        *reinterpret_cast<float4 *>(&sm.dU[rr * RS + ca]) = make_float4(acc[0].x, acc[0].y, acc[1].x, acc[1].y);
        *reinterpret_cast<float4 *>(&sm.dU[rr * RS + cb]) = make_float4(acc[2].x, acc[2].y, acc[3].x, acc[3].y);
      }
      {  // dP = lower(dO' U^T)   (thread (r, i))
        const int r = tid >> 4, i = tid & 15;
        float acc = 0.f;
        if (i <= r) {
#pragma unroll 8
          for (int j = 0; j < 128; j += 4) {
            const float4 a = *reinterpret_cast<const float4 *>(&sm.dO[r * RS + j]);
            const float4 b = *reinterpret_cast<const float4 *>(&sm.U[i * RS + j]);
            acc = fmaf(a.x, b.x, acc); acc = fmaf(a.y, b.y, acc);
            acc = fmaf(a.z, b.z, acc); acc = fmaf(a.w, b.w, acc);
          }
        }
        sm.dP[r * SS + i] = acc;
      }
      __syncthreads();
      if (tid < 128) {  // dR = (I + A)^{-T} dU, back substitution in place
        const int j = tid;
        float x[kSub];
#pragma unroll
        for (int r = kSub - 1; r >= 0; --r) {
          float y = sm.dU[r * RS + j];
#pragma unroll
          for (int i = r + 1; i < kSub; ++i) y = fmaf(-sm.A[i * SS + r], x[i], y);
          x[r] = y;
          sm.dU[r * RS + j] = y;
        }
      }
      __syncthreads();
      {  // dA = -strict_lower(dR U^T); dbeta; dv = beta dR
        const int r = tid >> 4, i = tid & 15;
        float acc = 0.f;
        if (i < r) {
#pragma unroll 8
          for (int j = 0; j < 128; j += 4) {
            const float4 a = *reinterpret_cast<const float4 *>(&sm.dU[r * RS + j]);
            const float4 b = *reinterpret_cast<const float4 *>(&sm.U[i * RS + j]);
            acc = fmaf(a.x, b.x, acc); acc = fmaf(a.y, b.y, acc);
            acc = fmaf(a.z, b.z, acc); acc = fmaf(a.w, b.w, acc);
          }
        }
        const float da = -acc;
        sm.dA[r * SS + i] = da;
        // dbeta_r = <dR_r, E_r> + sum_{i<r} dA[r,i] KK[r,i]; lanes (r, 0..15) share row r
        float part = i < r ? da * sm.KK[r * SS + i] : 0.f;
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const float4 a = *reinterpret_cast<const float4 *>(&sm.dU[r * RS + 8 * i + 4 * x]);
          const float4 b = *reinterpret_cast<const float4 *>(&sm.E[r * RS + 8 * i + 4 * x]);
          part = fmaf(a.x, b.x, part); part = fmaf(a.y, b.y, part);
          part = fmaf(a.z, b.z, part); part = fmaf(a.w, b.w, part);
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        if (i == 0 && r0 + r < Lc) dbeta[(size_t)(t0 + r0 + r) * H + h] = part;
      }
      if (r0 + rr < Lc) {
        const float b = sm.beta[rr];
        float *dst = dv + ((size_t)(t0 + r0 + rr) * H + h) * 128;
        const float4 a1 = *reinterpret_cast<const float4 *>(&sm.dU[rr * RS + ca]);
        const float4 a2 = *reinterpret_cast<const float4 *>(&sm.dU[rr * RS + cb]);
        *reinterpret_cast<float4 *>(dst + ca) = make_float4(b * a1.x, b * a1.y, b * a1.z, b * a1.w);
        *reinterpret_cast<float4 *>(dst + cb) = make_float4(b * a2.x, b * a2.y, b * a2.z, b * a2.w);
      }
      __syncthreads();

      // ---- key-indexed gradients: thread (key kt, rows 8 rh .. 8 rh + 7) -----------------------
      {
        const int rb = 8 * rh;
        float dqg[8], dkg[8], dkp[8];
        float sds;  // rowsum(S * dS') of key kt
        {
          // Dot products over the 128 value columns, as two interleaved partial sums (even
          // and odd columns) on the packed instructions, added at the end.
          float2 q2[8], k2[8], p2[8], sd2 = dup2(0.f);
#pragma unroll
          for (int x = 0; x < 8; ++x) q2[x] = k2[x] = p2[x] = dup2(0.f);
          const float *srow = &sm.S[kt * RS], *dsrow = &sm.dS[kt * RS];
#pragma unroll 2
          for (int j = 0; j < 128; j += 4) {
            const float4 sv = *reinterpret_cast<const float4 *>(srow + j);
            const float4 dv4 = *reinterpret_cast<const float4 *>(dsrow + j);
            sd2 = __ffma2_rn(lo2(sv), lo2(dv4), sd2);
            sd2 = __ffma2_rn(hi2(sv), hi2(dv4), sd2);
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              const int r = rb + x;  // the same row for the whole warp: broadcast reads
              const float4 o = *reinterpret_cast<const float4 *>(&sm.dO[r * RS + j]);
              const float4 rr4 = *reinterpret_cast<const float4 *>(&sm.dU[r * RS + j]);
              const float4 u = *reinterpret_cast<const float4 *>(&sm.U[r * RS + j]);
              q2[x] = __ffma2_rn(lo2(o), lo2(sv), q2[x]);
              q2[x] = __ffma2_rn(hi2(o), hi2(sv), q2[x]);
              k2[x] = __ffma2_rn(lo2(rr4), lo2(sv), k2[x]);
              k2[x] = __ffma2_rn(hi2(rr4), hi2(sv), k2[x]);
              p2[x] = __ffma2_rn(lo2(u), lo2(dv4), p2[x]);
              p2[x] = __ffma2_rn(hi2(u), hi2(dv4), p2[x]);
            }
          }
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            dqg[x] = q2[x].x + q2[x].y;
            dkg[x] = k2[x].x + k2[x].y;
            dkp[x] = p2[x].x + p2[x].y;
          }
          sds = sd2.x + sd2.y;
        }
        float dgam[8], dkd[8];
        float kps = 0.f;  // sum over this thread's rows of dK' K'
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const int r = rb + x;
          float pq = 0.f, pa = 0.f, kd = 0.f;
#pragma unroll
          for (int i = 0; i < kSub; ++i) {
            const float kdi = sm.KD[i * RS + kt];
            pq = fmaf(sm.dP[r * SS + i], kdi, pq);   // (dP K/G)[r]
            pa = fmaf(sm.dA[r * SS + i], kdi, pa);   // (dA K/G)[r]
            // ((diag(beta) dA)^T (K G) + dP^T (Q G))[r]
            kd = fmaf(sm.beta[i] * sm.dA[i * SS + r], sm.KG[i * RS + kt],
                      fmaf(sm.dP[i * SS + r], sm.QG[i * RS + kt], kd));
          }
          const float b = sm.beta[r], kpr = sm.KP[r * RS + kt];
          dqg[x] += pq;
          dkg[x] = b * (pa - dkg[x]);
          dkd[x] = kd;
          dgam[x] = dqg[x] * sm.QG[r * RS + kt] + dkg[x] * sm.KG[r * RS + kt] -
                    dkd[x] * sm.KD[r * RS + kt] - dkp[x] * kpr;
          kps = fmaf(dkp[x], kpr, kps);
        }
        // reverse cumulative sum within this thread's 8 rows
        float tot = 0.f;
#pragma unroll
        for (int x = 7; x >= 0; --x) {
          tot += dgam[x];
          dgam[x] = tot;
        }
        sm.xch[rh][kt] = rh ? tot : kps;  // upper half: its dgamma total; lower: its dK' K' sum
        __syncthreads();
        const float other = sm.xch[rh ^ 1][kt];
        __syncthreads();
        // the last row (row 15, upper half) gains G_last rowsum(S dS') + sum over all 16 rows
        // of dK' K'; every row at or above it sees that term in its suffix sum.
        const float last = rh ? sm.gc[kt] * sds + kps + other : 0.f;
        if (rh == 1) {
#pragma unroll
          for (int x = 0; x < 8; ++x) dgam[x] += last;
          sm.xch[0][kt] = tot + last;   // the whole upper half, for the lower half's suffixes
        }
        __syncthreads();
        if (rh == 0) {
          const float upper = sm.xch[0][kt];
#pragma unroll
          for (int x = 0; x < 8; ++x) dgam[x] += upper;
        }
        const float gck = sm.gc[kt];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const int r = rb + x;
          if (r0 + r < Lc) {
            const float Gv = sm.G[r * RS + kt];
            const size_t o = ((size_t)(t0 + r0 + r) * H + h) * 128 + kt;
            dq[o] = dqg[x] * Gv;
            dk[o] = dkg[x] * Gv + __fdividef(dkd[x] + dkp[x] * gck, Gv);
            dg[o] = dgam[x];
          }
        }
      }
      __syncthreads();

      // ---- dS <- diag(G_last) dS' + (Q G)^T dO' - (diag(beta) K G)^T dR  (keys kq, kq + 64) --
      {
        float2 st[2][16];
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const int key = kq + 64 * kk;
          const float2 gck = dup2(sm.gc[key]);
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float4 x = *reinterpret_cast<const float4 *>(&sm.dS[key * RS + 16 * m + 4 * q4]);
            st[kk][2 * m] = __fmul2_rn(gck, lo2(x));
            st[kk][2 * m + 1] = __fmul2_rn(gck, hi2(x));
          }
        }
#pragma unroll 2
        for (int r = 0; r < kSub; ++r) {
          const float nb = -sm.beta[r];
          const float2 a0 = dup2(sm.QG[r * RS + kq]), a1 = dup2(sm.QG[r * RS + kq + 64]);
          const float2 b0 = dup2(nb * sm.KG[r * RS + kq]), b1 = dup2(nb * sm.KG[r * RS + kq + 64]);
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            const float4 o = *reinterpret_cast<const float4 *>(&sm.dO[r * RS + 16 * m + 4 * q4]);
            const float4 d = *reinterpret_cast<const float4 *>(&sm.dU[r * RS + 16 * m + 4 * q4]);
            st[0][2 * m] = __ffma2_rn(a0, lo2(o), __ffma2_rn(b0, lo2(d), st[0][2 * m]));
            st[0][2 * m + 1] = __ffma2_rn(a0, hi2(o), __ffma2_rn(b0, hi2(d), st[0][2 * m + 1]));
            st[1][2 * m] = __ffma2_rn(a1, lo2(o), __ffma2_rn(b1, lo2(d), st[1][2 * m]));
            st[1][2 * m + 1] = __ffma2_rn(a1, hi2(o), __ffma2_rn(b1, hi2(d), st[1][2 * m + 1]));
          }
        }
#pragma unroll
        for (int kk = 0; kk < 2; ++kk)
#pragma unroll
          for (int m = 0; m < 8; ++m)
            *reinterpret_cast<float4 *>(&sm.dS[(kq + 64 * kk) * RS + 16 * m + 4 * q4]) =
                make_float4(st[kk][2 * m].x, st[kk][2 * m].y, st[kk][2 * m + 1].x, st[kk][2 * m + 1].y);
      }
    }
    __syncthreads();  // before the next item overwrites the shared matrices
  }
}

}  // namespace

cudaError_t launch_chunk_bwd_state(const void *ws, const int32_t *cu, const float *dsN,
                                   const float *dout, float scale, int N, int T, int H,
                                   float *dckpt, float *ds0, int *status, cudaStream_t s) {
  const long long blocks = (long long)N * H * kSlices;
  if (blocks >= (1LL << 31)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(chunk_bwd_state_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)BB_ALLOC);
  if (e != cudaSuccess) return e;
  chunk_bwd_state_kernel<<<(unsigned)blocks, kBT, BB_ALLOC, s>>>(
      static_cast<const uint8_t *>(ws), cu, dsN, dout, scale, N, T, H, dckpt, ds0, status);
  return cudaGetLastError();
}

namespace {
template <typename Tin>
cudaError_t launch_local_typed(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *dout, float scale,
                               const int32_t *cu, const void *ws, const float *ckpt,
                               const float *dckpt, float *scratch, int N, int T, int H,
                               float *dq, float *dk, float *dv, float *dg, float *dbeta,
                               int *status, cudaStream_t s) {
  const long long items = rec::chunk_capacity(N, T) * H;
  const int blocks = (int)(items < kLocalCTAs ? items : kLocalCTAs);
  const int bytes = (int)sizeof(LocalSmem);
  cudaError_t e = cudaFuncSetAttribute(chunk_bwd_local_kernel<Tin>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return e;
  chunk_bwd_local_kernel<Tin><<<blocks, kLT, bytes, s>>>(
      static_cast<const Tin *>(q), static_cast<const Tin *>(k), static_cast<const Tin *>(v), g,
      beta, dout, scale, cu, static_cast<const uint8_t *>(ws), ckpt, dckpt, scratch, items, N, T,
      H, dq, dk, dv, dg, dbeta, status);
  return cudaGetLastError();
}
}  // namespace

size_t chunk_bwd_local_scratch_bytes() { return (size_t)kLocalCTAs * kLocalSlotFloats * 4; }

cudaError_t launch_chunk_bwd_local(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, const float *dout, float scale,
                                   const int32_t *cu, const void *ws, const float *ckpt,
                                   const float *dckpt, float *scratch, int N, int T, int H,
                                   kda_dtype dt, float *dq, float *dk, float *dv, float *dg,
                                   float *dbeta, int *status, cudaStream_t s) {
  if (dt == KDA_BF16)
    return launch_local_typed<__nv_bfloat16>(q, k, v, g, beta, dout, scale, cu, ws, ckpt, dckpt,
                                             scratch, N, T, H, dq, dk, dv, dg, dbeta, status, s);
  if (dt == KDA_F16)
    return launch_local_typed<__half>(q, k, v, g, beta, dout, scale, cu, ws, ckpt, dckpt,
                                      scratch, N, T, H, dq, dk, dv, dg, dbeta, status, s);
  return cudaErrorInvalidValue;
}

}  // namespace kda
