// State pass of the two-pass tensor-core prefill, and the chunk index of a
// packed batch.
//
// Sources: "KimiK3轻量化复刻实现KDA并行解析，Chunkwise并行与状态压缩机制详解",
// Figure 1 (the state is carried chunk to chunk through an affine map built
// from per-chunk quantities); "AI-Workshop 文献分享 #16 — KDA：给长文本建立可更新的
// 记忆", §10.3 (the chunk update: read the entry state, correct with the
// in-chunk WY factors, decay and write).  Record contents and the algebra are
// in kda_chunk_record.cuh.
//
// One CTA (128 threads) per (sequence, head, slice of 32 value channels): the
// value columns of the state are independent of each other (W, A and the
// decay do not involve v), so the four slices of a head run side by side and
// a 96-head layer fills 384 CTAs.  Per chunk:
//   D1 = [W ; Q G] S_slice            (M = 128: rows 0..63 give W S, 64..127 Q G S)
//   U  = Ut - (W S)                   (fp32, warps 0-1; fp16 copy as MMA operand)
//   D1 += [* ; P] U                   (rows 64..127 += P U; rows 0..63 are dead)
//   D2 = K'^T U                       (M = 128 key channels)
//   o  = scale (D1[64 + r] + <q_r, k_r> U_r)     (warps 2-3, fp32)
//   S  = diag(G_last) S + D2          (fp32 registers; thread = key channel)
// Operand roundings are those of the one-pass kernel: fp16 S, W, Q G, U, P,
// K' with fp32 accumulation and fp32 diagonal terms.
#include <cuda_fp16.h>

#include <algorithm>

#include "kda_chunk_record.cuh"
#include "kda_common.cuh"
#include "kda_tcgen05.cuh"

namespace kda {
namespace {
using namespace tc;

constexpr int kBT = 128;      // threads per CTA
constexpr int kSlices = 4;    // value-channel slices per head
constexpr uint32_t SB_A1 = 0;            // [W ; Q G] (K-major 128 x 128)          32 KB
constexpr uint32_t SB_KP = 32768;        // K' (MN-major), then P: one copy       24 KB
constexpr uint32_t SB_P = 49152;
constexpr uint32_t SB_A2 = SB_P - 8192;  // A operand [* ; P]: rows 0..63 overlay the tail of
                                         // K' (finite fp16 values whose products land in
                                         // accumulator rows that are never read again)
constexpr uint32_t SB_S = 57344;         // S slice operand (value-contiguous, 128 key rows x 64 B,
                                         // 64-byte swizzle) 8 KB; between the two MMA groups:
                                         // <q_r, k_r> U exchange [32][64] f32
constexpr uint32_t SB_U = 65536;         // U operand (value-contiguous, 64 token rows x 64 B) 4 KB
constexpr uint32_t SB_BAR = 69632;       // three mbarriers, TMEM slot
constexpr uint32_t SB_ALLOC = SB_BAR + 64 + 1024;
// D1 is accumulated as two halves over the key channels (two independent MMA
// chains), summed at read-out; D2 = K'^T U.
constexpr uint32_t TB_D1 = 0, TB_D1B = 32, TB_D2 = 64, TB_COLS = 128;
static_assert(SB_KP + 24576 == SB_S, "K' and P are adjacent");

__global__ void __launch_bounds__(kBT, 3)
chunk_state_kernel(const uint8_t *__restrict__ ws, const int32_t *__restrict__ cu,
                   const float *s0, float scale, int N, int T, int H, float *__restrict__ o,
                   float *sN, int *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int slice = blockIdx.x % kSlices;
  const int nh = blockIdx.x / kSlices, h = nh % H, n = nh / H;
  const int32_t *cprefix = reinterpret_cast<const int32_t *>(ws);
  const uint8_t *recs = ws + rec::header_bytes(N);
  uint64_t *bar_a1 = reinterpret_cast<uint64_t *>(sm + SB_BAR);
  uint64_t *bar_kp = bar_a1 + 1, *bar_mma = bar_a1 + 2;
  uint32_t *slot = reinterpret_cast<uint32_t *>(sm + SB_BAR + 32);
  float *exch = reinterpret_cast<float *>(sm + SB_S);

  int bos, eos;
  seq_bounds(cu, n, T, status, bos, eos);
  int cbase = 0, nch = (eos - bos + 63) / 64;
  if (cu) {  // zero chunks for every sequence when the index pass rejected cu
    cbase = cprefix[n];
    nch = cprefix[n + 1] - cbase;
  }

  if (warp == 0) tmem_alloc(slot, TB_COLS);
  if (tid == 0) {
    mbar_init(bar_a1, 1);
    mbar_init(bar_kp, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
  }
  // S[i] = S[key tid][value 32 slice + i]; the state is stored value-major [dv][dk].
  const int t = tid;
  const size_t sbase = ((size_t)n * H + h) * 128 * 128 + (size_t)slice * 32 * 128 + t;
  float S[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) S[i] = s0 ? s0[sbase + (size_t)i * 128] : 0.f;

  auto write_s_operand = [&]() {  // S slice as the B operand: key row t, 32 values
    float amax = 0.f;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        f[e] = S[8 * x + e];
        amax = fmaxf(amax, fabsf(f[e]));
      }
      st_shared_16(sm + SB_S, mn32_sw64_off(t, x), pack8_f16(f));
    }
    if (!(amax < 32768.f)) report(status, KDA_ERR_DEVICE_RANGE);
  };
  write_s_operand();
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
    bulk_load(sm + SB_A1, rec_of(c) + rec::A1, 32768, bar_a1);
  };
  auto load_kp = [&](int c) {
    mbar_arrive_expect_tx(bar_kp, 24576);
    bulk_load(sm + SB_KP, rec_of(c) + rec::KP, 24576, bar_kp);
  };
  if (tid == 0 && nch > 0) {
    load_a1(0);
    load_kp(0);
  }

  // Record values read by threads (Ut slice and <q_r, k_r> of token tid for
  // warps 0-1, exp(gamma_last) of key t for all) are fetched one chunk ahead.
  float ut[32];
  float pd = 0.f, gl = 0.f;
  auto fetch_u = [&](int c) {
    if (warp < 2) {
      const uint8_t *rp = rec_of(c);
      const float4 *src =
          reinterpret_cast<const float4 *>(rp + rec::UT + ((size_t)tid * 128 + slice * 32) * 4);
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const float4 f = __ldcs(src + x);
        ut[4 * x] = f.x; ut[4 * x + 1] = f.y; ut[4 * x + 2] = f.z; ut[4 * x + 3] = f.w;
      }
      pd = __ldcs(reinterpret_cast<const float *>(rp + rec::PD) + tid);
    }
  };
  auto fetch_gl = [&](int c) { gl = __ldg(reinterpret_cast<const float *>(rec_of(c) + rec::GL) + t); };
  if (nch > 0) {
    fetch_u(0);
    fetch_gl(0);
  }

  uint32_t pa = 0, pk = 0, pm = 0;
  for (int c = 0; c < nch; ++c) {
    const int t0 = bos + 64 * c, Lc = min(64, eos - t0);

    // ---- D1 = [W ; Q G] S ----------------------------------------------------------
    if (!wait_all(bar_a1, pa, status)) break;
    pa ^= 1;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t a1 = smem_u32(sm + SB_A1), sop = smem_u32(sm + SB_S);
      constexpr uint32_t id = idesc_fp16(128, 32, false, true);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {  // key channels [0, 64) into D1, [64, 128) into D1B
        mma_bf16(tmem + TB_D1, desc_kmajor(a1, 128, ks), desc_mn32_sw64(sop, ks), id, ks > 0);
        mma_bf16(tmem + TB_D1B, desc_kmajor(a1, 128, ks + 4), desc_mn32_sw64(sop, ks + 4), id,
                 ks > 0);
      }
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, pm, status)) break;
    pm ^= 1;
    tc_fence_after();
    if (tid == 0 && c + 1 < nch) load_a1(c + 1);  // A1 has been read

    // ---- U = Ut - W S (warps 0-1: TMEM lanes 0..63 are the chunk's tokens) -------------
    if (warp < 2) {
      float y[32], y2[32];
      tmem_ld32_nowait(tmem + lane_addr + TB_D1, y);
      tmem_ld32_nowait(tmem + lane_addr + TB_D1B, y2);
      tmem_wait_ld(y, y2);
      const int r = tid;
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        y[i] = ut[i] - (y[i] + y2[i]);  // U
        amax = fmaxf(amax, fabsf(y[i]));
        exch[i * 64 + r] = pd * y[i];  // the S operand is dead until the next chunk
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = y[8 * x + e];
        st_shared_16(sm + SB_U, mn32_sw64_off(r, x), pack8_f16(f));
      }
      if (!(amax < 32768.f)) report(status, KDA_ERR_DEVICE_RANGE);
      if (c + 1 < nch) fetch_u(c + 1);
    }
    fence_async_smem();
    tc_fence_before();
    if (!wait_all(bar_kp, pk, status)) break;  // K', P of this chunk; also a CTA barrier
    pk ^= 1;

    // ---- D1 += [* ; P] U ;  D2 = K'^T U ----------------------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t a2 = smem_u32(sm + SB_A2), uop = smem_u32(sm + SB_U);
      const uint32_t kp = smem_u32(sm + SB_KP);
      constexpr uint32_t idO = idesc_fp16(128, 32, false, true);
      constexpr uint32_t idS = idesc_fp16(128, 32, true, true);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {  // the two accumulators' steps interleaved
        mma_bf16(tmem + TB_D1, desc_kmajor(a2, 128, ks), desc_mn32_sw64(uop, ks), idO, 1);
        mma_bf16(tmem + TB_D2, desc_mnmajor(kp, 64, ks), desc_mn32_sw64(uop, ks), idS, ks > 0);
      }
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, pm, status)) break;
    pm ^= 1;
    tc_fence_after();
    if (tid == 0 && c + 1 < nch) load_kp(c + 1);  // K' and P have been read

    // ---- outputs (warps 2-3: TMEM lanes 64..127) and the state update ---------------------
    {
      float ds[32];
      tmem_ld32(tmem + lane_addr + TB_D2, ds);
#pragma unroll
      for (int i = 0; i < 32; ++i) S[i] = fmaf(S[i], gl, ds[i]);
      if (c + 1 < nch) fetch_gl(c + 1);
    }
    if (warp >= 2) {
      float ov[32], ov2[32];
      tmem_ld32_nowait(tmem + lane_addr + TB_D1, ov);
      tmem_ld32_nowait(tmem + lane_addr + TB_D1B, ov2);
      tmem_wait_ld(ov, ov2);
#pragma unroll
      for (int i = 0; i < 32; ++i) ov[i] += ov2[i];
      const int r = tid - 64;
      if (r < Lc) {
        float4 *dst = reinterpret_cast<float4 *>(o + ((size_t)(t0 + r) * H + h) * 128 + slice * 32);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          float4 f;
          f.x = scale * (ov[4 * x] + exch[(4 * x) * 64 + r]);
          f.y = scale * (ov[4 * x + 1] + exch[(4 * x + 1) * 64 + r]);
          f.z = scale * (ov[4 * x + 2] + exch[(4 * x + 2) * 64 + r]);
          f.w = scale * (ov[4 * x + 3] + exch[(4 * x + 3) * 64 + r]);
          dst[x] = f;
        }
      }
    }
    __syncthreads();  // the exchange has been read; the S operand goes over it
    write_s_operand();
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  if (sN) {
#pragma unroll
    for (int i = 0; i < 32; ++i) sN[sbase + (size_t)i * 128] = S[i];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, TB_COLS);
}

// cprefix[n] = number of chunks of sequences 0..n-1 (cprefix[N] = total).  A
// malformed cu_seqlens (decreasing, or outside [0, T]) is recorded and gives
// every sequence zero chunks, so no pass reads or writes past the workspace.
__global__ void __launch_bounds__(1024)
chunk_index_kernel(const int32_t *__restrict__ cu, int N, int T, int32_t *cprefix, int *status) {
  __shared__ int bad;
  __shared__ int wsum[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int i = tid; i < N; i += 1024) {
    const int a = cu[i], b = cu[i + 1];
    if (a < 0 || b < a || b > T) bad = 1;
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) report(status, KDA_ERR_DEVICE_BOUNDS);
    for (int i = tid; i <= N; i += 1024) cprefix[i] = 0;
    return;
  }
  int carry = 0;
  for (int base = 0; base < N; base += 1024) {
    const int i = base + tid;
    const int cnt = i < N ? (cu[i + 1] - cu[i] + 63) / 64 : 0;
    int x = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, d);
      if (lane >= d) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int w = wsum[lane];
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, d);
        if (lane >= d) w += y;
      }
      wsum[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int before = warp > 0 ? wsum[warp - 1] : 0;
    if (i < N) cprefix[i] = carry + before + x - cnt;
    carry += wsum[31];
    __syncthreads();
  }
  if (tid == 0) cprefix[N] = carry;
}

// Fused two-pass prefill: a sequence without chunks (empty, or every sequence
// when the index pass rejected cu_seqlens) has no prep item to write its conv
// cache, so it is passed through here: cache_out[n] = cache_in[n], or zero.
// Elements are 16-bit (bf16 or fp16; +0.0 is all-zero bits in both).
__global__ void __launch_bounds__(256)
cache_pass_kernel(const int32_t *__restrict__ cprefix, const uint16_t *__restrict__ cache_in,
                  uint16_t *__restrict__ cache_out, long long per_seq) {
  const int n = blockIdx.x;
  if (cprefix[n + 1] != cprefix[n]) return;
  const size_t base = (size_t)n * per_seq;
  for (long long i = threadIdx.x; i < per_seq; i += blockDim.x)
    cache_out[base + i] = cache_in ? cache_in[base + i] : (uint16_t)0;
}

}  // namespace

cudaError_t launch_cache_pass(const void *ws, int N, int H, const void *cache_in,
                              void *cache_out, cudaStream_t s) {
  cache_pass_kernel<<<N, 256, 0, s>>>(static_cast<const int32_t *>(ws),
                                      static_cast<const uint16_t *>(cache_in),
                                      static_cast<uint16_t *>(cache_out), 3LL * 3 * H * 128);
  return cudaGetLastError();
}

cudaError_t launch_chunk_index(const int32_t *cu, int N, int T, void *ws, int *status,
                               cudaStream_t s) {
  chunk_index_kernel<<<1, 1024, 0, s>>>(cu, N, T, static_cast<int32_t *>(ws), status);
  return cudaGetLastError();
}

cudaError_t launch_chunk_state(const void *ws, const int32_t *cu, const float *s0, float scale,
                               int N, int T, int H, float *o, float *sN, int *status,
                               cudaStream_t s) {
  const long long blocks = (long long)N * H * kSlices;
  if (blocks >= (1LL << 31)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(chunk_state_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SB_ALLOC);
  if (e != cudaSuccess) return e;
  chunk_state_kernel<<<(unsigned)blocks, kBT, SB_ALLOC, s>>>(
      static_cast<const uint8_t *>(ws), cu, s0, scale, N, T, H, o, sN, status);
  return cudaGetLastError();
}

}  // namespace kda
