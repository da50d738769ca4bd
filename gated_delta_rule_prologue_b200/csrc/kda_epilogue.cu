// Output epilogue: per-head RMSNorm of the read-out followed by the per-channel
// output gate ("Kimi K3的线性注意力：从源码看懂KDA如何更新记忆", 第六站):
//     out[t, h, :] = o[t, h, :] / sqrt(mean_d o^2 + eps) * weight * sigmoid(gate[t, h, :])
// (the gate a sigmoid of its pre-activation, a per-channel proportion; eps a
// parameter).  HBM-bound: D/4 lanes own one (token, head) row, one float4 of o and
// four gate values per lane in single vector accesses, four rows per lane group
// loaded before any is used; the sum of squares is reduced with xor shuffles
// inside the row's lanes.  Bytes per row: 4 D (o) + 2 * D * sizeof(dt) (gate, out).
#include "kda_common.cuh"

namespace kda {
namespace {

// Four gate (or output) values of a row, as one 8-byte (16-bit types) or 16-byte (fp32) access.
template <typename Tg> struct Vec4;
template <> struct Vec4<__nv_bfloat16> { using T = uint2; };
template <> struct Vec4<__half> { using T = uint2; };
template <> struct Vec4<float> { using T = float4; };

template <typename Tg>
__device__ __forceinline__ void unpack4(const typename Vec4<Tg>::T &v, float (&f)[4]) {
  const Tg *h = reinterpret_cast<const Tg *>(&v);
#pragma unroll
  for (int e = 0; e < 4; ++e) f[e] = to_f32(h[e]);
}
template <typename Tg>
__device__ __forceinline__ typename Vec4<Tg>::T pack4(const float (&f)[4]) {
  typename Vec4<Tg>::T v;
  Tg *h = reinterpret_cast<Tg *>(&v);
#pragma unroll
  for (int e = 0; e < 4; ++e) h[e] = from_f32<Tg>(f[e]);
  return v;
}

// Each lane group handles kRowsPerGroup rows, one per grid-wide stride of warps, with every
// load issued before any is used, so several rows' loads are in flight per thread.
constexpr int kRowsPerGroup = 4;

template <typename Tg, int D>
__global__ void __launch_bounds__(256)
epilogue_kernel(const float *__restrict__ o, const Tg *__restrict__ gate,
                const float *__restrict__ weight, float eps, long long rows, Tg *__restrict__ out) {
  using V = typename Vec4<Tg>::T;
  constexpr int LPR = D / 4;          // lanes per row
  constexpr int RPW = 32 / LPR;       // rows per warp access
  const int lane = threadIdx.x & 31;
  const int sub = lane % LPR, d0 = 4 * sub;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const float4 w4 = __ldg(reinterpret_cast<const float4 *>(weight + d0));
  const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
  float4 x[kRowsPerGroup];
  V zg[kRowsPerGroup];
#pragma unroll
  for (int i = 0; i < kRowsPerGroup; ++i) {
    const long long row = (warp + (long long)i * nwarps) * RPW + lane / LPR;
    const size_t base = (size_t)(row < rows ? row : 0) * D + d0;
    x[i] = row < rows ? __ldcs(reinterpret_cast<const float4 *>(o + base))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    zg[i] = *reinterpret_cast<const V *>(gate + base);
  }
#pragma unroll
  for (int i = 0; i < kRowsPerGroup; ++i) {
    const long long row = (warp + (long long)i * nwarps) * RPW + lane / LPR;
    float ss = x[i].x * x[i].x;
    ss = fmaf(x[i].y, x[i].y, ss);
    ss = fmaf(x[i].z, x[i].z, ss);
    ss = fmaf(x[i].w, x[i].w, ss);
#pragma unroll
    for (int off = LPR / 2; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float r = rsqrtf(ss * (1.f / D) + eps);
    const float xv[4] = {x[i].x, x[i].y, x[i].z, x[i].w};
    float z[4], y[4];
    unpack4<Tg>(zg[i], z);
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] = xv[e] * r * wv[e] * __fdividef(1.f, 1.f + __expf(-z[e]));
    if (row < rows) *reinterpret_cast<V *>(out + (size_t)row * D + d0) = pack4<Tg>(y);
  }
}

template <typename Tg, int D>
cudaError_t launch_typed(const float *o, const void *gate, const float *weight, float eps,
                         long long rows, void *out, cudaStream_t s) {
  constexpr int RPW = 32 / (D / 4);
  const long long per_warp = (long long)RPW * kRowsPerGroup;
  const long long warps = (rows + per_warp - 1) / per_warp;
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
