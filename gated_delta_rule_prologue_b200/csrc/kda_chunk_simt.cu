// Chunkwise KDA prefill on CUDA cores in fp32 (any activation type, D <= 128,
// chunk in {16, 32, 64}).  This is the exact-fp32 path and the cross-check for
// the tensor-core path; it favours clarity over speed.
//
// Sources: "Kimi K3的线性注意力：从源码看懂KDA如何更新记忆", 彩蛋 (chunked
// execution: the state is passed between chunks, work inside a chunk is
// matrix algebra, causality kept); "AI-Workshop 文献分享 #16 — KDA：给长文本建立可更新的记忆",
// §10.3 (chunkwise algorithm).
//
// Chunk algebra (derived from the recurrence; entry state S0 key-first,
// gamma_r = inclusive in-chunk cumsum of g, G_r = exp(gamma_r)):
//   A[r,i] = beta_r sum_d k_r[d] k_i[d] exp(gamma_r[d]-gamma_i[d])   (i < r)
//   P[r,i] =        sum_d q_r[d] k_i[d] exp(gamma_r[d]-gamma_i[d])   (i <= r)
//   (I + A) U = diag(beta) (V - (K*G) S0)          forward substitution
//   O = scale * ((Q*G) S0 + P U)
//   S_exit = diag(G_last) S0 + (K * exp(gamma_last - gamma))^T U
// Exponents are always differences gamma_r - gamma_i <= 0, so no factor can
// overflow whatever the decay.
//
// One CTA per (sequence, head, 32-wide slice of the value dimension).
#include "kda_common.cuh"

namespace kda {
namespace {

constexpr int kThreads = 256;

template <int D, int CH>
struct SimtSmem {
  static constexpr int DVS = D < 32 ? D : 32;  // value columns per CTA
  static constexpr int LD = D + 1;             // padded row stride (bank conflicts)
  static constexpr int LC = CH + 1;
  static constexpr size_t floats =
      3 * (size_t)CH * LD      // K, Q, GM (cumulative log-decay)
      + (size_t)CH * DVS       // V slice
      + 2 * (size_t)CH * LC    // A, P
      + (size_t)CH * DVS       // U
      + (size_t)D * DVS        // S slice, key-first
      + CH;                    // beta
  static constexpr size_t bytes = floats * sizeof(float);
};

template <typename Tin, int D, int CH>
__global__ void __launch_bounds__(kThreads)
chunk_simt_kernel(const Tin *__restrict__ q, const Tin *__restrict__ k, const Tin *__restrict__ v,
                  const float *__restrict__ g, const float *__restrict__ beta, float scale,
                  const float *s0, const int32_t *__restrict__ cu, int N, int T, int H,
                  float *__restrict__ o, float *sN, int *status) {
  using L = SimtSmem<D, CH>;
  constexpr int DVS = L::DVS, LD = L::LD, LC = L::LC, NSL = D / DVS;
  extern __shared__ float smem[];
  float *Ks = smem;
  float *Qs = Ks + CH * LD;
  float *GM = Qs + CH * LD;
  float *Vs = GM + CH * LD;
  float *As = Vs + CH * DVS;
  float *Ps = As + CH * LC;
  float *Us = Ps + CH * LC;
  float *Ss = Us + CH * DVS;
  float *Bs = Ss + D * DVS;

  const int slice = blockIdx.x % NSL;
  const int nh = blockIdx.x / NSL;
  const int n = nh / H, h = nh % H;
  const int tid = threadIdx.x;
  const int j0 = slice * DVS;
  int bos, eos;
  seq_bounds(cu, n, T, status, bos, eos);
  if (!in_range(status, n, N) || (eos > bos && !in_range(status, eos - 1, T))) return;

  // Entry state slice: Ss[d][j] = S[d][j0 + j] = state[n][h][j0 + j][d].
  for (int idx = tid; idx < D * DVS; idx += kThreads) {
    const int d = idx % D, j = idx / D;
    Ss[d * DVS + j] = s0 ? s0[(((size_t)n * H + h) * D + j0 + j) * D + d] : 0.f;
  }

  for (int c0 = bos; c0 < eos; c0 += CH) {
    const int Lc = min(CH, eos - c0);
    __syncthreads();
    for (int idx = tid; idx < CH * D; idx += kThreads) {
      const int r = idx / D, d = idx % D;
      float kk = 0.f, qq = 0.f, gg = 0.f;
      if (r < Lc) {
        const size_t off = ((size_t)(c0 + r) * H + h) * D + d;
        kk = to_f32(k[off]);
        qq = to_f32(q[off]);
        gg = g[off];
      }
      Ks[r * LD + d] = kk;
      Qs[r * LD + d] = qq;
      GM[r * LD + d] = gg;
    }
    for (int idx = tid; idx < CH * DVS; idx += kThreads) {
      const int r = idx / DVS, j = idx % DVS;
      Vs[idx] = r < Lc ? to_f32(v[((size_t)(c0 + r) * H + h) * D + j0 + j]) : 0.f;
    }
    for (int r = tid; r < CH; r += kThreads) Bs[r] = r < Lc ? beta[(size_t)(c0 + r) * H + h] : 0.f;
    __syncthreads();
    // inclusive cumulative log-decay along the chunk, per key channel
    for (int d = tid; d < D; d += kThreads) {
      float acc = 0.f;
      for (int r = 0; r < CH; ++r) {
        acc += GM[r * LD + d];
        GM[r * LD + d] = acc;
      }
    }
    __syncthreads();
    // Gram matrices A (strictly lower, scaled by beta_r) and P (lower incl.)
    for (int pi = tid; pi < CH * CH; pi += kThreads) {
      const int r = pi / CH, i = pi % CH;
      float sa = 0.f, sp = 0.f;
      if (i <= r && r < Lc) {
        for (int d = 0; d < D; ++d) {
          const float kd = Ks[i * LD + d] * expf(GM[r * LD + d] - GM[i * LD + d]);
          sa = fmaf(Ks[r * LD + d], kd, sa);
          sp = fmaf(Qs[r * LD + d], kd, sp);
        }
      }
      As[r * LC + i] = (i < r) ? Bs[r] * sa : 0.f;
      Ps[r * LC + i] = sp;
    }
    // right-hand side beta_r (v_r - S0^T (k_r * G_r))
    for (int idx = tid; idx < CH * DVS; idx += kThreads) {
      const int r = idx / DVS, j = idx % DVS;
      float acc = 0.f;
      for (int d = 0; d < D; ++d)
        acc = fmaf(Ks[r * LD + d] * expf(GM[r * LD + d]), Ss[d * DVS + j], acc);
      Us[idx] = Bs[r] * (Vs[idx] - acc);
    }
    __syncthreads();
    // forward substitution, one value column per thread
    for (int j = tid; j < DVS; j += kThreads) {
      for (int r = 1; r < Lc; ++r) {
        float u = Us[r * DVS + j];
        for (int i = 0; i < r; ++i) u = fmaf(-As[r * LC + i], Us[i * DVS + j], u);
        Us[r * DVS + j] = u;
      }
    }
    __syncthreads();
    // outputs
    for (int idx = tid; idx < Lc * DVS; idx += kThreads) {
      const int r = idx / DVS, j = idx % DVS;
      float acc = 0.f;
      for (int d = 0; d < D; ++d)
        acc = fmaf(Qs[r * LD + d] * expf(GM[r * LD + d]), Ss[d * DVS + j], acc);
      for (int i = 0; i <= r; ++i) acc = fmaf(Ps[r * LC + i], Us[i * DVS + j], acc);
      o[((size_t)(c0 + r) * H + h) * D + j0 + j] = scale * acc;
    }
    __syncthreads();
    // state update
    for (int idx = tid; idx < D * DVS; idx += kThreads) {
      const int d = idx / DVS, j = idx % DVS;
      const float gl = GM[(Lc - 1) * LD + d];
      float acc = expf(gl) * Ss[idx];
      for (int i = 0; i < Lc; ++i)
        acc = fmaf(Ks[i * LD + d] * expf(gl - GM[i * LD + d]), Us[i * DVS + j], acc);
      Ss[idx] = acc;
    }
  }
  __syncthreads();
  if (sN) {
    for (int idx = tid; idx < D * DVS; idx += kThreads) {
      const int d = idx % D, j = idx / D;
      sN[(((size_t)n * H + h) * D + j0 + j) * D + d] = Ss[d * DVS + j];
    }
  }
}

template <typename Tin, int D, int CH>
cudaError_t launch_typed(const void *q, const void *k, const void *v, const float *g,
                         const float *beta, float scale, const float *s0, const int32_t *cu,
                         int N, int T, int H, float *o, float *sN, int *status, cudaStream_t s) {
  using L = SimtSmem<D, CH>;
  auto kern = chunk_simt_kernel<Tin, D, CH>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)L::bytes);
  if (e != cudaSuccess) return e;
  const long long blocks = (long long)N * H * (D / L::DVS);
  if (blocks >= (1LL << 31)) return cudaErrorInvalidValue;
  kern<<<(unsigned)blocks, kThreads, L::bytes, s>>>(
      static_cast<const Tin *>(q), static_cast<const Tin *>(k), static_cast<const Tin *>(v), g,
      beta, scale, s0, cu, N, T, H, o, sN, status);
  return cudaGetLastError();
}

template <typename Tin, int D>
cudaError_t launch_c(int chunk, const void *q, const void *k, const void *v, const float *g,
                     const float *beta, float scale, const float *s0, const int32_t *cu, int N,
                     int T, int H, float *o, float *sN, int *status, cudaStream_t s) {
  switch (chunk) {
    case 16: return launch_typed<Tin, D, 16>(q, k, v, g, beta, scale, s0, cu, N, T, H, o, sN, status, s);
    case 32: return launch_typed<Tin, D, 32>(q, k, v, g, beta, scale, s0, cu, N, T, H, o, sN, status, s);
    case 64: return launch_typed<Tin, D, 64>(q, k, v, g, beta, scale, s0, cu, N, T, H, o, sN, status, s);
    default: return cudaErrorInvalidValue;
  }
}

template <typename Tin>
cudaError_t launch_d(int D, int chunk, const void *q, const void *k, const void *v,
                     const float *g, const float *beta, float scale, const float *s0,
                     const int32_t *cu, int N, int T, int H, float *o, float *sN, int *status,
                     cudaStream_t s) {
  switch (D) {
    case 16: return launch_c<Tin, 16>(chunk, q, k, v, g, beta, scale, s0, cu, N, T, H, o, sN, status, s);
    case 32: return launch_c<Tin, 32>(chunk, q, k, v, g, beta, scale, s0, cu, N, T, H, o, sN, status, s);
    case 64: return launch_c<Tin, 64>(chunk, q, k, v, g, beta, scale, s0, cu, N, T, H, o, sN, status, s);
    case 128: return launch_c<Tin, 128>(chunk, q, k, v, g, beta, scale, s0, cu, N, T, H, o, sN, status, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, float scale, const float *s0,
                              const int32_t *cu, int N, int T, int H, int D, int chunk,
                              kda_dtype dt, float *o, float *sN, int *status, cudaStream_t s) {
  if (dt == KDA_BF16)
    return launch_d<__nv_bfloat16>(D, chunk, q, k, v, g, beta, scale, s0, cu, N, T, H, o, sN,
                                   status, s);
  if (dt == KDA_F16)
    return launch_d<__half>(D, chunk, q, k, v, g, beta, scale, s0, cu, N, T, H, o, sN, status, s);
  return launch_d<float>(D, chunk, q, k, v, g, beta, scale, s0, cu, N, T, H, o, sN, status, s);
}

}  // namespace kda
