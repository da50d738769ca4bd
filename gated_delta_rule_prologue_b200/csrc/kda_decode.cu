// Batched decode step: for each (sequence, head) the prologue on the new token
// with the conv cache as history, then one step of the KDA recurrence on the
// fp32 state in place.
//
// Sources: "Kimi K3的线性注意力：从源码看懂KDA如何更新记忆" -- 第二站 (short conv,
// SiLU, L2 on q and k), 第三站 (rows of the key-first state decayed by
// alpha_t = exp(g_t)), 第四站 (error against the decayed state, delta write),
// 第五站 (read after the write), 彩蛋 (recurrent execution for generation).
//
// The state is stored value-major, state[n][h][j][i] = S[i][j] (S key-first),
// so row j of S^T is D contiguous floats.  Per row j:
//     s'  = alpha (.) S^T[j,:]
//     p_j = <s', k>,   r_j = <s', q>            (one fused shuffle tree)
//     e_j = v_j - p_j
//     S^T[j,:] = s' + beta e_j k
//     o_j = scale * <S^T[j,:], q> = scale * (r_j + beta e_j <k, q>)
// so both reductions are independent and <k, q> is one reduction per head, not per row.
// HBM traffic is dominated by the state: 2 * 4 * D^2 bytes per (seq, head).
// The block meets once, after the prologue: each warp then reduces the norms
// of q and k itself and writes the read-out of its own rows, so no warp waits
// for another while the state streams through.
#include "kda_common.cuh"

namespace kda {
namespace {

template <int D>
struct DecodeShape {
  static constexpr int kLanesPerRow = D / 4;                  // float4 per lane
  static constexpr int kRowsPerInstr = 32 / kLanesPerRow;     // rows per warp access
  static constexpr int kWarps = (D / kRowsPerInstr) < 8 ? (D / kRowsPerInstr) : 8;
  static constexpr int kThreads = kWarps * 32;
  static constexpr int kIters = D / (kRowsPerInstr * kWarps); // row groups per warp
  static_assert(kIters >= 1 && kIters * kRowsPerInstr * kWarps == D, "row split");
};

// kGated: g holds gate pre-activations of type Tin and the log-decay is
// lower_bound * sigmoid(exp(A_log[h]) * (g + dt_bias[h, :])) (pointers may be null).
template <typename Tin, int D, bool kGated>
__global__ void __launch_bounds__(DecodeShape<D>::kThreads, 2)  // two CTAs per SM: at most 128 registers
decode_kernel(const Tin *__restrict__ x, const float *__restrict__ w, Tin *__restrict__ cache,
              const void *__restrict__ g, const float *__restrict__ beta, float scale,
              float *__restrict__ state, int N, int H, float *__restrict__ o,
              const float *__restrict__ A_log, const float *__restrict__ dt_bias,
              float lower_bound) {
  using Sh = DecodeShape<D>;
  constexpr int LPR = Sh::kLanesPerRow;
  __shared__ float qkv[3 * D];

  const int nh = blockIdx.x;
  const int n = nh / H, h = nh % H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sub = lane % LPR;          // float4 slot within a row
  const int rsub = lane / LPR;         // row within the warp access
  const int dk0 = sub * 4;

  float4 g4;
  if constexpr (kGated) {
    const Tin *gr = static_cast<const Tin *>(g) + (size_t)nh * D + dk0;
    const float a = A_log ? __expf(__ldg(A_log + h)) : 1.f;
    const float4 b4 = dt_bias ? __ldg(reinterpret_cast<const float4 *>(dt_bias + (size_t)h * D + dk0))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    g4 = make_float4(bounded_gate(to_f32(gr[0]), a, b4.x, lower_bound),
                     bounded_gate(to_f32(gr[1]), a, b4.y, lower_bound),
                     bounded_gate(to_f32(gr[2]), a, b4.z, lower_bound),
                     bounded_gate(to_f32(gr[3]), a, b4.w, lower_bound));
  } else {
    g4 = __ldg(reinterpret_cast<const float4 *>(static_cast<const float *>(g) + (size_t)nh * D + dk0));
  }
  const float b = __ldg(beta + nh);

  // 1. Prologue for this head's 3*D channels; the conv cache is shifted in place.
  //    A thread's channels (two at most) have all their loads issued first, before
  //    the state's, and before any is used: the barrier waits for one round trip.
  const int C = 3 * H * D;
  constexpr int kCh = (3 * D + Sh::kThreads - 1) / Sh::kThreads;
  Tin r0[kCh], r1[kCh], r2[kCh], xin[kCh];
  float4 wc[kCh];
#pragma unroll
  for (int m = 0; m < kCh; ++m) {
    const int i = tid + m * Sh::kThreads;
    if (i < 3 * D) {
      const int c = (i / D) * H * D + h * D + i % D;
      const Tin *cr = cache + (size_t)n * 3 * C + c;
      r0[m] = cr[0];
      r1[m] = cr[C];
      r2[m] = cr[2 * C];
      xin[m] = x[(size_t)n * C + c];
      wc[m] = __ldg(reinterpret_cast<const float4 *>(w + (size_t)c * 4));
    }
  }
  // The state loads follow: the prologue is on the path to the barrier, the
  // state is first needed after it.
  float *base = state + (size_t)nh * D * D;
  float4 s[Sh::kIters];
#pragma unroll
  for (int it = 0; it < Sh::kIters; ++it) {
    const int j = (warp * Sh::kIters + it) * Sh::kRowsPerInstr + rsub;
    s[it] = __ldcs(reinterpret_cast<const float4 *>(base + (size_t)j * D + dk0));
  }
#pragma unroll
  for (int m = 0; m < kCh; ++m) {
    const int i = tid + m * Sh::kThreads;
    if (i < 3 * D) {
      const int c = (i / D) * H * D + h * D + i % D;
      float a = wc[m].x * to_f32(r0[m]);
      a = fmaf(wc[m].y, to_f32(r1[m]), a);
      a = fmaf(wc[m].z, to_f32(r2[m]), a);
      a = fmaf(wc[m].w, to_f32(xin[m]), a);
      qkv[i] = silu(a);
      Tin *cr = cache + (size_t)n * 3 * C + c;
      cr[0] = r1[m];
      cr[C] = r2[m];
      cr[2 * C] = xin[m];
    }
  }
  __syncthreads();
  // Every warp reduces |q|^2, |k|^2 and <k, q> itself (the same operations in the
  // same order, so the same values): no second block barrier.
  float sq = 0.f, sk = 0.f, skq = 0.f;
  for (int d = lane; d < D; d += 32) {
    const float qq = qkv[d], kk = qkv[D + d];
    sq = fmaf(qq, qq, sq);
    sk = fmaf(kk, kk, sk);
    skq = fmaf(kk, qq, skq);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, off);
    sk += __shfl_xor_sync(0xffffffffu, sk, off);
    skq += __shfl_xor_sync(0xffffffffu, skq, off);
  }
  const float rq = rsqrtf(sq + 1e-6f), rk = rsqrtf(sk + 1e-6f);
  const float kq = skq * rq * rk;  // <k, q> of the normalised vectors
  const float4 q4 = make_float4(qkv[dk0] * rq, qkv[dk0 + 1] * rq, qkv[dk0 + 2] * rq,
                                qkv[dk0 + 3] * rq);
  const float4 k4 = make_float4(qkv[D + dk0] * rk, qkv[D + dk0 + 1] * rk,
                                qkv[D + dk0 + 2] * rk, qkv[D + dk0 + 3] * rk);
  const float4 a4 = make_float4(expf(g4.x), expf(g4.y), expf(g4.z), expf(g4.w));

  // 2. State update, one row of S^T per LPR lanes.
#pragma unroll
  for (int it = 0; it < Sh::kIters; ++it) {
    const int j = (warp * Sh::kIters + it) * Sh::kRowsPerInstr + rsub;
    float4 sp = make_float4(a4.x * s[it].x, a4.y * s[it].y, a4.z * s[it].z, a4.w * s[it].w);
    float pk = sp.x * k4.x;
    pk = fmaf(sp.y, k4.y, pk);
    pk = fmaf(sp.z, k4.z, pk);
    pk = fmaf(sp.w, k4.w, pk);
    float pq = sp.x * q4.x;
    pq = fmaf(sp.y, q4.y, pq);
    pq = fmaf(sp.z, q4.z, pq);
    pq = fmaf(sp.w, q4.w, pq);
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) {
      pk += __shfl_xor_sync(0xffffffffu, pk, off);
      pq += __shfl_xor_sync(0xffffffffu, pq, off);
    }
    const float be = b * (qkv[2 * D + j] - pk);
    sp.x = fmaf(be, k4.x, sp.x);
    sp.y = fmaf(be, k4.y, sp.y);
    sp.z = fmaf(be, k4.z, sp.z);
    sp.w = fmaf(be, k4.w, sp.w);
    __stcs(reinterpret_cast<float4 *>(base + (size_t)j * D + dk0), sp);
    if (sub == 0) o[(size_t)nh * D + j] = scale * fmaf(be, kq, pq);
  }
}

// Gate of the gated step (null A_log / dt_bias: neutral; unused when not gated).
struct DecodeGate {
  const float *A_log;
  const float *dt_bias;
  float lower_bound;
  bool on;
};

template <typename Tin, int D>
cudaError_t launch_typed(const void *x, const float *w, void *cache, const void *g,
                         const float *beta, float scale, float *state, int N, int H, float *o,
                         const DecodeGate &gt, cudaStream_t s) {
  auto kern = gt.on ? decode_kernel<Tin, D, true> : decode_kernel<Tin, D, false>;
  kern<<<N * H, DecodeShape<D>::kThreads, 0, s>>>(static_cast<const Tin *>(x), w,
                                                  static_cast<Tin *>(cache), g, beta, scale,
                                                  state, N, H, o, gt.A_log, gt.dt_bias,
                                                  gt.lower_bound);
  return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_d(int D, const void *x, const float *w, void *cache, const void *g,
                     const float *beta, float scale, float *state, int N, int H, float *o,
                     const DecodeGate &gt, cudaStream_t s) {
  switch (D) {
    case 16: return launch_typed<Tin, 16>(x, w, cache, g, beta, scale, state, N, H, o, gt, s);
    case 32: return launch_typed<Tin, 32>(x, w, cache, g, beta, scale, state, N, H, o, gt, s);
    case 64: return launch_typed<Tin, 64>(x, w, cache, g, beta, scale, state, N, H, o, gt, s);
    case 128: return launch_typed<Tin, 128>(x, w, cache, g, beta, scale, state, N, H, o, gt, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_decode(const void *x, const float *w, void *cache, const void *g,
                          const float *beta, float scale, float *state, int N, int H, int D,
                          kda_dtype dt, float *o, const float *A_log, const float *dt_bias,
                          float lower_bound, bool gated, int *status, cudaStream_t s) {
  (void)status;  // the decode kernel has no waits or data-dependent indices
  if ((long long)N * H >= (1LL << 31)) return cudaErrorInvalidValue;
  const DecodeGate gt{A_log, dt_bias, lower_bound, gated};
  if (dt == KDA_BF16)
    return launch_d<__nv_bfloat16>(D, x, w, cache, g, beta, scale, state, N, H, o, gt, s);
  if (dt == KDA_F16) return launch_d<__half>(D, x, w, cache, g, beta, scale, state, N, H, o, gt, s);
  return launch_d<float>(D, x, w, cache, g, beta, scale, state, N, H, o, gt, s);
}

}  // namespace kda
