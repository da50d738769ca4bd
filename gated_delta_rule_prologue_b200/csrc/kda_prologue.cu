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
//   * loads of a batch of 8 tokens are issued before any of them is used, and
//     rows stay in their storage type until used (4 registers per 16-bit row),
//     so two 256-thread blocks fit per SM with 64 KB of loads in flight.
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;
constexpr int kTokensPerThread = 32;  // TT
// tokens whose loads are in flight together (fewer for 32-byte float rows)
template <typename Tin> __host__ __device__ constexpr int batch_of() { return sizeof(Tin) == 2 ? 6 : 3; }

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
        hv[j] = load_or_zero(x + (size_t)tt * C + c0, active);
      } else {
        const int r = 3 - (bos - tt);  // cache row (0 = oldest)
        hv[j] = load_or_zero(cache_in + ((size_t)n * 3 + r) * C + c0,
                             active && cache_in != nullptr);
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
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = fmaf(wt[e][2], fm1[e], fmaf(wt[e][1], fm2[e], wt[e][0] * fm3[e]));
      widen8(xr[i], f);
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        y[e] = silu(fmaf(wt[e][3], f[e], y[e]));
        ss = fmaf(y[e], y[e], ss);
      }
#pragma unroll
      for (int off = G / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
      if (p < 2) {
        const float r = rsqrtf(ss + 1e-6f);
#pragma unroll
        for (int e = 0; e < 8; ++e) y[e] *= r;
      }
      if (active) {
        store8(out + ((size_t)t * H + h) * D + d0, y);
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

template <typename Tin, typename Tout, int D>
cudaError_t launch_typed(const void *x, const float *w, const void *cache_in, void *cache_out,
                         const int32_t *cu, int N, int T, int H, void *q, void *k, void *v,
                         int *status, cudaStream_t s) {
  const int C = 3 * H * D;
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
