// Prologue kernel: causal depthwise short conv (width 4) + SiLU over the q/k/v
// projections, then per-(token, head) L2 normalisation of q and k.
//
// Source: "Kimi K3的线性注意力：从源码看懂KDA如何更新记忆", 第二站 (short conv
// of width 4 that never looks ahead, SiLU inside the conv module, q and k
// unit-normalised); "KimiK3轻量化复刻实现KDA并行解析，Chunkwise并行与状态压缩机制详解",
// ShortConv paragraph (per channel: the current token and the three before).
//
// Work decomposition (HBM-bound, 1536 B of traffic per token-head for bf16):
//   * one thread owns 8 consecutive channels of one (part, head) segment and
//     walks TT consecutive tokens, keeping the previous three inputs of its
//     channels in registers, so every input element is read from HBM once
//     (plus a 3-row halo per TT tokens, mostly served by L2);
//   * the D/8 threads of a segment sit in one warp and reduce the sum of
//     squares for the L2 norm with xor shuffles;
//   * 16-bit inputs (the common case) reach shared memory by 2-D TMA copies
//     into a three-slot ring per warp (below), so loads stay in flight while
//     the warp computes; fp32 inputs (and x not 16-byte aligned) take the
//     register form: loads of a batch of tokens are issued before any of them
//     is used, rows kept in their storage type until used.
#include <cstring>
#include <type_traits>

#include "kda_common.cuh"
#include "kda_tcgen05.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kTokensPerThread = 32;  // TT
// tokens whose loads are in flight together (fewer for 32-byte float rows)
template <typename Tin> __host__ __device__ constexpr int batch_of() { return sizeof(Tin) == 2 ? 6 : 3; }

// One token of a thread's 8 channels: y = SiLU(w0 x[t-3] + w1 x[t-2] + w2 x[t-1] + w3 x[t]),
// then, for q and k (norm = true), y / sqrt(sum over the head's D channels of y^2 + 1e-6);
// the G = D/8 lanes of a head are consecutive lanes of one warp.
template <int G>
__device__ __forceinline__ void conv_silu_norm(const float (&wt)[8][4], const float (&fm3)[8],
                                               const float (&fm2)[8], const float (&fm1)[8],
                                               const float (&f)[8], bool norm, float (&y)[8]) {
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    y[e] = fmaf(wt[e][2], fm1[e], fmaf(wt[e][1], fm2[e], wt[e][0] * fm3[e]));
    y[e] = silu(fmaf(wt[e][3], f[e], y[e]));
    ss = fmaf(y[e], y[e], ss);
  }
#pragma unroll
  for (int off = G / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if (norm) {
    const float r = rsqrtf(ss + 1e-6f);
#pragma unroll
    for (int e = 0; e < 8; ++e) y[e] *= r;
  }
}

template <typename Tin, typename Tout, int D>
__global__ void __launch_bounds__(kThreads, 2)
prologue_kernel(const Tin *__restrict__ x, const float *__restrict__ w,
                const Tin *__restrict__ cache_in, Tin *__restrict__ cache_out,
                const int32_t *__restrict__ cu, int N, int T, int H, Tout *__restrict__ q,
                Tout *__restrict__ k, Tout *__restrict__ v, int *status) {
  constexpr int G = D / 8;  // threads per (part, head) segment; divides 32
  const int HD = H * D;
  const int C = 3 * HD;
  const int c0 = (blockIdx.x * kThreads + threadIdx.x) * 8;
  const bool active = c0 < C;
  const int p = active ? c0 / HD : 0;
  const int h = active ? (c0 % HD) / D : 0;
  const int d0 = c0 % D;
  Tout *out = p == 0 ? q : (p == 1 ? k : v);
  auto load_or_zero = [&](const Tin *ptr, bool ok) { return ok ? load_raw8(ptr) : zero_raw8<Tin>(); };

  // Sequences with no tokens pass their cache through unchanged.
  if (blockIdx.y == 0 && cache_out != nullptr && active) {
    for (int n = 0; n < N; ++n) {
      const int a = cu ? cu[n] : 0, b = cu ? cu[n + 1] : T;
      if (a != b) continue;
      for (int r = 0; r < 3; ++r)
        store_raw8(cache_out + ((size_t)n * 3 + r) * C + c0,
                   load_or_zero(cache_in + ((size_t)n * 3 + r) * C + c0, cache_in != nullptr));
    }
  }

  const int t0 = blockIdx.y * kTokensPerThread;
  const int t_end = min(t0 + kTokensPerThread, T);
  if (t0 >= t_end) return;  // uniform over the block
  if (cu != nullptr && (cu[0] != 0 || cu[N] != T)) {
    report(status, KDA_ERR_DEVICE_BOUNDS);
    return;
  }

  float wt[8][4];
  if (active) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 f = __ldg(reinterpret_cast<const float4 *>(w + (size_t)(c0 + i) * 4));
      wt[i][0] = f.x; wt[i][1] = f.y; wt[i][2] = f.z; wt[i][3] = f.w;
    }
  }

  int n = seq_of_token(cu, N, t0);
  if (!in_range(status, n, N)) return;
  int bos, eos;
  seq_bounds(cu, n, T, status, bos, eos);
  while (t0 >= eos && n < N - 1) {  // skip empty sequences ending at t0
    ++n;
    seq_bounds(cu, n, T, status, bos, eos);
  }

  // History of t0: tokens t0-3, t0-2, t0-1 (from the cache before bos), packed
  // for the cache write-out and widened once for the convolution.
  Raw8<Tin> hm3, hm2, hm1;
  float fm3[8], fm2[8], fm1[8];
  {
    Raw8<Tin> hv[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const int tt = t0 - 3 + j;
      if (tt >= bos) {
        hv[j] = load_or_zero(x + (size_t)tt * C + c0, active && in_range(status, tt, T));
      } else {
        const int r = 3 - (bos - tt);  // cache row (0 = oldest)
        hv[j] = load_or_zero(cache_in + ((size_t)n * 3 + r) * C + c0,
                             active && cache_in != nullptr && in_range(status, r, 3));
      }
    }
    hm3 = hv[0];
    hm2 = hv[1];
    hm1 = hv[2];
    widen8(hm3, fm3);
    widen8(hm2, fm2);
    widen8(hm1, fm1);
  }

  constexpr int kBatch = batch_of<Tin>();
  for (int tb = t0; tb < t_end; tb += kBatch) {
    Raw8<Tin> xr[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i)
      xr[i] = load_or_zero(x + (size_t)(tb + i) * C + c0, active && tb + i < t_end);

#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int t = tb + i;
      if (t >= t_end) break;
      if (t >= eos) {  // next non-empty sequence starts at t: restart the history
        do {
          ++n;
          seq_bounds(cu, n, T, status, bos, eos);
        } while (t >= eos && n < N - 1);
        const Tin *cr = cache_in + (size_t)n * 3 * C + c0;
        const bool ok = active && cache_in != nullptr;
        hm3 = load_or_zero(cr, ok);
        hm2 = load_or_zero(cr + C, ok);
        hm1 = load_or_zero(cr + 2 * C, ok);
        widen8(hm3, fm3);
        widen8(hm2, fm2);
        widen8(hm1, fm1);
      }
      float y[8], f[8];
      widen8(xr[i], f);
      conv_silu_norm<G>(wt, fm3, fm2, fm1, f, p < 2, y);
      if (active) {
        if (in_range(status, t, T)) store8(out + ((size_t)t * H + h) * D + d0, y);
        if (cache_out != nullptr && t == eos - 1) {
          store_raw8(cache_out + ((size_t)n * 3 + 0) * C + c0, hm2);
          store_raw8(cache_out + ((size_t)n * 3 + 1) * C + c0, hm1);
          store_raw8(cache_out + ((size_t)n * 3 + 2) * C + c0, xr[i]);
        }
      }
      hm3 = hm2;
      hm2 = hm1;
      hm1 = xr[i];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        fm3[e] = fm2[e];
        fm2[e] = fm1[e];
        fm1[e] = f[e];
      }
    }
  }
}

// ---- 16-bit inputs: the x rows arrive by TMA into a ring per warp --------------------
// Each warp owns 256 consecutive channels (32 lanes x 8) and walks the CTA's tokens in
// boxes of kBoxTokens rows; a box is one 2-D TMA copy (kBoxTokens x 256 channels) into
// the warp's ring of kStages slots, so loads stay in flight while the warp computes and
// no thread holds loaded rows in registers.  A slot is refilled by lane 0 as soon as the
// warp has read it (the warp's own __syncwarp orders the reads before the refill).  No
// barrier spans warps.  Rows past T and channels past 3*H*D are zero-filled by the copy.
//
// The arithmetic runs on pairs of channels with the packed fp32 instructions (one
// issue for two lanes, each rounded as its scalar operation), and SiLU is written from
// its definition, a * sigma(a) with sigma(a) = 1 / (1 + 2^(-a log2 e)), on the
// hardware's approximate base-2 exponential and reciprocal (PTX ex2.approx,
// rcp.approx: relative errors of a few 2^-23).  The three-row history is a ring whose
// slots are compile-time indices (no register moves per token), and a box that neither
// ends a sequence nor the CTA's range runs without per-token checks.
constexpr int kBoxTokens = 6;    // a multiple of the 3-row history ring
constexpr int kStages = 3;
constexpr int kWarpChannels = 256;
constexpr int kBoxBytes = kBoxTokens * kWarpChannels * 2;
constexpr int kStagedTokens = 288;  // tokens per CTA: 48 boxes (32768 tokens x 96 heads: 2052
                                    // CTAs, 6.9 waves of 2 x 148)
constexpr int kStagedWarps = kThreads / 32;
constexpr int kStagedSmem = kStagedWarps * kStages * (kBoxBytes + 8);
static_assert(kStagedTokens % kBoxTokens == 0 && kBoxTokens % 3 == 0 && kBoxBytes % 128 == 0,
              "box plan");

__device__ __forceinline__ void store_pairs(__half *p, const float2 (&y)[4]) {
  *reinterpret_cast<uint4 *>(p) = pack_pairs(y, __half{});
}
__device__ __forceinline__ void store_pairs(__nv_bfloat16 *p, const float2 (&y)[4]) {
  *reinterpret_cast<uint4 *>(p) = pack_pairs(y, __nv_bfloat16{});
}
__device__ __forceinline__ void store_pairs(float *p, const float2 (&y)[4]) {
  reinterpret_cast<float4 *>(p)[0] = make_float4(y[0].x, y[0].y, y[1].x, y[1].y);
  reinterpret_cast<float4 *>(p)[1] = make_float4(y[2].x, y[2].y, y[3].x, y[3].y);
}

// One token of a thread's 4 channel pairs (taps w[0..3] apply to x[t-3], x[t-2], x[t-1],
// x[t]); q and k (norm = true) are divided by sqrt(sum of squares over the head + 1e-6).
template <int G>
__device__ __forceinline__ void conv_silu_norm_pairs(const float2 (&w)[4][4],
                                                     const float2 (&h3)[4],
                                                     const float2 (&h2)[4],
                                                     const float2 (&h1)[4],
                                                     const float2 (&f)[4], bool norm,
                                                     float2 (&y)[4]) {
  float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    y[i] = conv4_silu_pair(w[0][i], w[1][i], w[2][i], w[3][i], h3[i], h2[i], h1[i], f[i]);
    ss2 = __ffma2_rn(y[i], y[i], ss2);
  }
  float ss = ss2.x + ss2.y;
#pragma unroll
  for (int off = G / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if (norm) {
    const float r = rsqrtf(ss + 1e-6f);
    const float2 r2 = make_float2(r, r);
#pragma unroll
    for (int i = 0; i < 4; ++i) y[i] = __fmul2_rn(y[i], r2);
  }
}

template <typename Tin, typename Tout, int D>
__global__ void __launch_bounds__(kThreads, 2)
prologue_staged_kernel(const __grid_constant__ CUtensorMap tm_x, const Tin *__restrict__ x,
                       const float *__restrict__ w, const Tin *__restrict__ cache_in,
                       Tin *__restrict__ cache_out, const int32_t *__restrict__ cu, int N, int T,
                       int H, Tout *__restrict__ q, Tout *__restrict__ k, Tout *__restrict__ v,
                       int *status) {
  static_assert(sizeof(Tin) == 2, "16-bit inputs only");
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int G = D / 8;
  const int HD = H * D;
  const int C = 3 * HD;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cw = (blockIdx.x * kStagedWarps + warp) * kWarpChannels;
  if (cw >= C) return;  // warp-uniform: no barrier spans warps
  const int c0 = cw + lane * 8;
  const bool active = c0 < C;
  const int p = active ? c0 / HD : 0;
  const int h = active ? (c0 % HD) / D : 0;
  const int d0 = c0 % D;
  const bool norm = p < 2;
  Tout *out = p == 0 ? q : (p == 1 ? k : v);
  auto load_or_zero = [&](const Tin *ptr, bool ok) { return ok ? load_raw8(ptr) : zero_raw8<Tin>(); };

  if (blockIdx.y == 0 && cache_out != nullptr && active) {
    for (int n = 0; n < N; ++n) {
      const int a = cu ? cu[n] : 0, b = cu ? cu[n + 1] : T;
      if (a != b) continue;
      for (int r = 0; r < 3; ++r)
        store_raw8(cache_out + ((size_t)n * 3 + r) * C + c0,
                   load_or_zero(cache_in + ((size_t)n * 3 + r) * C + c0, cache_in != nullptr));
    }
  }

  const int t0 = blockIdx.y * kStagedTokens;
  const int t_end = min(t0 + kStagedTokens, T);
  if (t0 >= t_end) return;
  if (cu != nullptr && (cu[0] != 0 || cu[N] != T)) {
    if (lane == 0) report(status, KDA_ERR_DEVICE_BOUNDS);
    return;
  }
  const int nbox = (t_end - t0 + kBoxTokens - 1) / kBoxTokens;
  uint8_t *ring = smem + warp * kStages * kBoxBytes;
  uint64_t *full =
      reinterpret_cast<uint64_t *>(smem + kStagedWarps * kStages * kBoxBytes) + warp * kStages;
  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kStages; ++s) tc::mbar_init(full + s, 1);
    tc::fence_mbar_init();
    for (int s = 0; s < kStages && s < nbox; ++s) {
      tc::mbar_arrive_expect_tx(full + s, kBoxBytes);
      tc::tma_load_2d(ring + s * kBoxBytes, &tm_x, full + s, cw, t0 + s * kBoxTokens);
    }
  }
  __syncwarp();

  float2 wt[4][4];  // [tap][channel pair]
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (active) {
      a = __ldg(reinterpret_cast<const float4 *>(w + (size_t)(c0 + 2 * i) * 4));
      b = __ldg(reinterpret_cast<const float4 *>(w + (size_t)(c0 + 2 * i + 1) * 4));
    }
    wt[0][i] = make_float2(a.x, b.x);
    wt[1][i] = make_float2(a.y, b.y);
    wt[2][i] = make_float2(a.z, b.z);
    wt[3][i] = make_float2(a.w, b.w);
  }

  int n = seq_of_token(cu, N, t0);
  if (!in_range(status, n, N)) n = 0;  // the ring is already loading: no early exit
  int bos, eos;
  seq_bounds(cu, n, T, status, bos, eos);
  while (t0 >= eos && n < N - 1) {
    ++n;
    seq_bounds(cu, n, T, status, bos, eos);
  }
  // Raw row tt of the current sequence (tt >= bos - 3): from x, or from the cache before bos.
  auto raw_row = [&](int tt) {
    if (tt >= bos) return load_or_zero(x + (size_t)tt * C + c0, active && in_range(status, tt, T));
    return load_or_zero(cache_in + ((size_t)n * 3 + (3 - (bos - tt))) * C + c0,
                        active && cache_in != nullptr && in_range(status, bos - tt - 1, 3));
  };

  // History ring: before token i of a box, slot i % 3 holds x[t-3], (i+1) % 3 x[t-2] and
  // (i+2) % 3 x[t-1]; token i's own row then replaces slot i % 3.
  float2 hr[3][4];
#pragma unroll
  for (int j = 0; j < 3; ++j) widen_pairs(raw_row(t0 - 3 + j).u, hr[j], Tin{});

  int slot = 0;
  uint32_t par = 0;
  for (int j = 0; j < nbox; ++j) {
    if (!__all_sync(0xffffffffu, tc::mbar_wait(full + slot, par))) {
      // A box never landed: record it and let the copies still in flight land in this
      // warp's slots before the warp leaves (bounded waits).
      if (lane == 0) {
        report(status, KDA_ERR_DEVICE_TIMEOUT);
        for (int jj = j; jj < nbox && jj < j + kStages; ++jj)
          (void)tc::mbar_wait(full + jj % kStages, (uint32_t)(jj / kStages) & 1u, 100000000ull);
      }
      __syncwarp();
      return;
    }
    const uint8_t *box = ring + slot * kBoxBytes + lane * 16;
    const int tb = t0 + j * kBoxTokens;
    Tout *ob = out + ((size_t)tb * H + h) * D + d0;
    const bool box_ok = in_range(status, tb, T);
    if (tb + kBoxTokens < eos && tb + kBoxTokens <= t_end) {
      // Inside one sequence, not its last token, and inside the CTA's range.
#pragma unroll
      for (int i = 0; i < kBoxTokens; ++i) {
        float2 f[4], y[4];
        widen_pairs(*reinterpret_cast<const uint4 *>(box + i * (kWarpChannels * 2)), f, Tin{});
        conv_silu_norm_pairs<G>(wt, hr[i % 3], hr[(i + 1) % 3], hr[(i + 2) % 3], f, norm, y);
        if (active && box_ok) store_pairs(ob + (size_t)i * HD, y);
#pragma unroll
        for (int e = 0; e < 4; ++e) hr[i % 3][e] = f[e];
      }
    } else {
#pragma unroll
      for (int i = 0; i < kBoxTokens; ++i) {
        const int t = tb + i;
        if (t >= t_end) break;
        if (t >= eos) {  // next non-empty sequence starts at t: history from its cache
          do {
            ++n;
            seq_bounds(cu, n, T, status, bos, eos);
          } while (t >= eos && n < N - 1);
          const Tin *cr = cache_in + (size_t)n * 3 * C + c0;
          const bool ok = active && cache_in != nullptr;
          widen_pairs(load_or_zero(cr, ok).u, hr[i % 3], Tin{});
          widen_pairs(load_or_zero(cr + C, ok).u, hr[(i + 1) % 3], Tin{});
          widen_pairs(load_or_zero(cr + 2 * C, ok).u, hr[(i + 2) % 3], Tin{});
        }
        const uint4 xu = *reinterpret_cast<const uint4 *>(box + i * (kWarpChannels * 2));
        float2 f[4], y[4];
        widen_pairs(xu, f, Tin{});
        conv_silu_norm_pairs<G>(wt, hr[i % 3], hr[(i + 1) % 3], hr[(i + 2) % 3], f, norm, y);
        if (active && box_ok) {
          store_pairs(ob + (size_t)i * HD, y);
          if (cache_out != nullptr && t == eos - 1) {
            store_raw8(cache_out + ((size_t)n * 3 + 0) * C + c0, raw_row(t - 2));
            store_raw8(cache_out + ((size_t)n * 3 + 1) * C + c0, raw_row(t - 1));
            Raw8<Tin> xr;
            xr.u = xu;
            store_raw8(cache_out + ((size_t)n * 3 + 2) * C + c0, xr);
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) hr[i % 3][e] = f[e];
      }
    }
    __syncwarp();
    if (lane == 0 && j + kStages < nbox) {
      tc::mbar_arrive_expect_tx(full + slot, kBoxBytes);
      tc::tma_load_2d(ring + slot * kBoxBytes, &tm_x, full + slot, cw,
                      t0 + (j + kStages) * kBoxTokens);
    }
    if (++slot == kStages) {
      slot = 0;
      par ^= 1u;
    }
  }
}

// 2-D map over x [T][3*H*D] (16-bit): box = kBoxTokens rows x 256 channels.
bool make_x_map(CUtensorMap *m, const void *x, kda_dtype dt, int C, int T) {
  auto enc = tensor_map_encoder();
  if (!enc || (reinterpret_cast<uintptr_t>(x) & 15u) != 0 || T < 1) return false;
  cuuint64_t dims[2] = {(cuuint64_t)C, (cuuint64_t)T};
  cuuint64_t strides[1] = {(cuuint64_t)C * 2};
  cuuint32_t box[2] = {kWarpChannels, kBoxTokens};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType t =
      dt == KDA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return enc(m, t, 2, const_cast<void *>(x), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename Tin, typename Tout, int D>
cudaError_t launch_typed(const void *x, const float *w, const void *cache_in, void *cache_out,
                         const int32_t *cu, int N, int T, int H, void *q, void *k, void *v,
                         int *status, cudaStream_t s) {
  const int C = 3 * H * D;
  if constexpr (sizeof(Tin) == 2) {
    CUtensorMap tm;
    if (T > 0 && make_x_map(&tm, x, std::is_same<Tin, __half>::value ? KDA_F16 : KDA_BF16, C, T)) {
      const cudaError_t e = cudaFuncSetAttribute(prologue_staged_kernel<Tin, Tout, D>,
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kStagedSmem);
      if (e != cudaSuccess) return e;
      const int warps = (C + kWarpChannels - 1) / kWarpChannels;
      dim3 grid((warps + kStagedWarps - 1) / kStagedWarps,
                (T + kStagedTokens - 1) / kStagedTokens);
      prologue_staged_kernel<Tin, Tout, D><<<grid, kThreads, kStagedSmem, s>>>(
          tm, static_cast<const Tin *>(x), w, static_cast<const Tin *>(cache_in),
          static_cast<Tin *>(cache_out), cu, N, T, H, static_cast<Tout *>(q),
          static_cast<Tout *>(k), static_cast<Tout *>(v), status);
      return cudaGetLastError();
    }
  }
  const int groups = C / 8;
  dim3 grid((groups + kThreads - 1) / kThreads,
            max(1, (T + kTokensPerThread - 1) / kTokensPerThread));
  prologue_kernel<Tin, Tout, D><<<grid, kThreads, 0, s>>>(
      static_cast<const Tin *>(x), w, static_cast<const Tin *>(cache_in),
      static_cast<Tin *>(cache_out), cu, N, T, H, static_cast<Tout *>(q),
      static_cast<Tout *>(k), static_cast<Tout *>(v), status);
  return cudaGetLastError();
}

template <typename Tin, typename Tout>
cudaError_t launch_d(int D, const void *x, const float *w, const void *ci, void *co,
                     const int32_t *cu, int N, int T, int H, void *q, void *k, void *v,
                     int *status, cudaStream_t s) {
  switch (D) {
    case 16: return launch_typed<Tin, Tout, 16>(x, w, ci, co, cu, N, T, H, q, k, v, status, s);
    case 32: return launch_typed<Tin, Tout, 32>(x, w, ci, co, cu, N, T, H, q, k, v, status, s);
    case 64: return launch_typed<Tin, Tout, 64>(x, w, ci, co, cu, N, T, H, q, k, v, status, s);
    case 128: return launch_typed<Tin, Tout, 128>(x, w, ci, co, cu, N, T, H, q, k, v, status, s);
    default: return cudaErrorInvalidValue;
  }
}

template <typename Tin>
cudaError_t launch_out(kda_dtype out_dt, int D, const void *x, const float *w, const void *ci,
                       void *co, const int32_t *cu, int N, int T, int H, void *q, void *k,
                       void *v, int *status, cudaStream_t s) {
  switch (out_dt) {
    case KDA_BF16:
      return launch_d<Tin, __nv_bfloat16>(D, x, w, ci, co, cu, N, T, H, q, k, v, status, s);
    case KDA_F16: return launch_d<Tin, __half>(D, x, w, ci, co, cu, N, T, H, q, k, v, status, s);
    default: return launch_d<Tin, float>(D, x, w, ci, co, cu, N, T, H, q, k, v, status, s);
  }
}

}  // namespace

cudaError_t launch_prologue(const void *x, const float *w, const void *cache_in, void *cache_out,
                            const int32_t *cu, int N, int T, int H, int D, kda_dtype dt,
                            kda_dtype out_dt, void *q, void *k, void *v, int *status,
                            cudaStream_t s) {
  switch (dt) {
    case KDA_BF16:
      return launch_out<__nv_bfloat16>(out_dt, D, x, w, cache_in, cache_out, cu, N, T, H, q, k,
                                       v, status, s);
    case KDA_F16:
      return launch_out<__half>(out_dt, D, x, w, cache_in, cache_out, cu, N, T, H, q, k, v,
                                status, s);
    default:
      return launch_out<float>(out_dt, D, x, w, cache_in, cache_out, cu, N, T, H, q, k, v,
                               status, s);
  }
}

}  // namespace kda
