// Output epilogue: per-head RMSNorm of the read-out followed by the per-channel
// output gate ("Kimi K3的线性注意力：从源码看懂KDA如何更新记忆", 第六站):
//     out[t, h, :] = o[t, h, :] / sqrt(mean_d o^2 + eps) * weight * sigmoid(gate[t, h, :])
// (the gate a sigmoid of its pre-activation, a per-channel proportion; eps a
// parameter).  HBM-bound: D/4 lanes own one (token, head) row, one float4 of o
// per lane, the sum of squares is reduced with xor shuffles inside the row's
// lanes.  Bytes per row: 4 D (o) + 2 * D * sizeof(dt) (gate, out).
#include "kda_common.cuh"

namespace kda {
namespace {

template <typename Tg, int D>
__global__ void __launch_bounds__(256)
epilogue_kernel(const float *__restrict__ o, const Tg *__restrict__ gate,
                const float *__restrict__ weight, float eps, long long rows, Tg *__restrict__ out) {
  constexpr int LPR = D / 4;          // lanes per row
  constexpr int RPW = 32 / LPR;       // rows per warp
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPR, d0 = 4 * sub;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long row = warp * RPW + lane / LPR;
  const float4 w4 = __ldg(reinterpret_cast<const float4 *>(weight + d0));
  const bool ok = row < rows;
  const size_t base = (size_t)(ok ? row : 0) * D + d0;
  const float4 x = ok ? __ldcs(reinterpret_cast<const float4 *>(o + base))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
  float z[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) z[e] = ok ? to_f32(gate[base + e]) : 0.f;
  float ss = x.x * x.x;
  ss = fmaf(x.y, x.y, ss);
  ss = fmaf(x.z, x.z, ss);
  ss = fmaf(x.w, x.w, ss);
#pragma unroll
  for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float r = rsqrtf(ss * (1.f / D) + eps);
  const float xv[4] = {x.x, x.y, x.z, x.w}, wv[4] = {w4.x, w4.y, w4.z, w4.w};
  if (ok) {
#pragma unroll
    for (int e = 0; e < 4; ++e)
      out[base + e] = from_f32<Tg>(xv[e] * r * wv[e] * __fdividef(1.f, 1.f + __expf(-z[e])));
  }
}

template <typename Tg, int D>
cudaError_t launch_typed(const float *o, const void *gate, const float *weight, float eps,
                         long long rows, void *out, cudaStream_t s) {
  constexpr int RPW = 32 / (D / 4);
  const long long warps = (rows + RPW - 1) / RPW;
  const long long blocks = (warps + 7) / 8;
  if (blocks >= (1LL << 31)) return cudaErrorInvalidValue;
  epilogue_kernel<Tg, D><<<(unsigned)blocks, 256, 0, s>>>(
      o, static_cast<const Tg *>(gate), weight, eps, rows, static_cast<Tg *>(out));
  return cudaGetLastError();
}

template <typename Tg>
cudaError_t launch_d(int D, const float *o, const void *gate, const float *weight, float eps,
                     long long rows, void *out, cudaStream_t s) {
  switch (D) {
    case 16: return launch_typed<Tg, 16>(o, gate, weight, eps, rows, out, s);
    case 32: return launch_typed<Tg, 32>(o, gate, weight, eps, rows, out, s);
    case 64: return launch_typed<Tg, 64>(o, gate, weight, eps, rows, out, s);
    case 128: return launch_typed<Tg, 128>(o, gate, weight, eps, rows, out, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_epilogue(const float *o, const void *gate, const float *weight, float eps,
                            long long rows, int D, kda_dtype dt, void *out, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  if (dt == KDA_BF16) return launch_d<__nv_bfloat16>(D, o, gate, weight, eps, rows, out, s);
  if (dt == KDA_F16) return launch_d<__half>(D, o, gate, weight, eps, rows, out, s);
  return launch_d<float>(D, o, gate, weight, eps, rows, out, s);
}

}  // namespace kda
