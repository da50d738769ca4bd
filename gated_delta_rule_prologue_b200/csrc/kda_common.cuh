// Shared device helpers for the libkda kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/kda.h"

namespace kda {

// ---------------------------------------------------------------------------
// Element access for the two activation types
// ---------------------------------------------------------------------------

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_f32(__half x) { return __half2float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}
template <> __device__ __forceinline__ __half from_f32<__half>(float x) { return __float2half_rn(x); }

// Load/store 8 consecutive elements (16 B for bf16, 32 B for f32) as floats.
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&out)[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
  const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __bfloat1622float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const __half *p, float (&out)[8]) {
  uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
  const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = __half22float2(h[i]);
    out[2 * i] = f.x;
    out[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float *p, float (&out)[8]) {
  float4 a = __ldg(reinterpret_cast<const float4 *>(p));
  float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
  out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
  out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float (&in)[8]) {
  uint4 u;
  __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(in[2 * i], in[2 * i + 1]);
  *reinterpret_cast<uint4 *>(p) = u;
}
__device__ __forceinline__ void store8(__half *p, const float (&in)[8]) {
  uint4 u;
  __half2 *h = reinterpret_cast<__half2 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(in[2 * i], in[2 * i + 1]);
  *reinterpret_cast<uint4 *>(p) = u;
}
__device__ __forceinline__ void store8(float *p, const float (&in)[8]) {
  reinterpret_cast<float4 *>(p)[0] = make_float4(in[0], in[1], in[2], in[3]);
  reinterpret_cast<float4 *>(p)[1] = make_float4(in[4], in[5], in[6], in[7]);
}

// Eight consecutive elements kept in their storage type (16 bytes for 16-bit
// types, 32 bytes for float) until they are used.
template <typename T> struct Raw8 { uint4 u; };
template <> struct Raw8<float> { float4 a, b; };

__device__ __forceinline__ Raw8<__nv_bfloat16> load_raw8(const __nv_bfloat16 *p) {
  return {__ldg(reinterpret_cast<const uint4 *>(p))};
}
__device__ __forceinline__ Raw8<__half> load_raw8(const __half *p) {
  return {__ldg(reinterpret_cast<const uint4 *>(p))};
}
__device__ __forceinline__ Raw8<float> load_raw8(const float *p) {
  return {__ldg(reinterpret_cast<const float4 *>(p)), __ldg(reinterpret_cast<const float4 *>(p) + 1)};
}
template <typename T> __device__ __forceinline__ Raw8<T> zero_raw8() {
  Raw8<T> r;
  r.u = make_uint4(0u, 0u, 0u, 0u);
  return r;
}
template <> __device__ __forceinline__ Raw8<float> zero_raw8<float>() {
  return {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
}
__device__ __forceinline__ void widen8(const Raw8<__nv_bfloat16> &r, float (&f)[8]) {
  const uint32_t w[4] = {r.u.x, r.u.y, r.u.z, r.u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
__device__ __forceinline__ void widen8(const Raw8<__half> &r, float (&f)[8]) {
  const __half2 *h = reinterpret_cast<const __half2 *>(&r.u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __half22float2(h[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}
__device__ __forceinline__ void widen8(const Raw8<float> &r, float (&f)[8]) {
  f[0] = r.a.x; f[1] = r.a.y; f[2] = r.a.z; f[3] = r.a.w;
  f[4] = r.b.x; f[5] = r.b.y; f[6] = r.b.z; f[7] = r.b.w;
}
__device__ __forceinline__ void store_raw8(__nv_bfloat16 *p, const Raw8<__nv_bfloat16> &r) {
  *reinterpret_cast<uint4 *>(p) = r.u;
}
__device__ __forceinline__ void store_raw8(__half *p, const Raw8<__half> &r) {
  *reinterpret_cast<uint4 *>(p) = r.u;
}
__device__ __forceinline__ void store_raw8(float *p, const Raw8<float> &r) {
  reinterpret_cast<float4 *>(p)[0] = r.a;
  reinterpret_cast<float4 *>(p)[1] = r.b;
}

// SiLU(x) = x * sigmoid(x) with the fast exponential and division intrinsics
// (a few ulp; for x -> -inf the denominator overflows and the result is 0).
__device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

// ---------------------------------------------------------------------------
// Channel pairs on the packed fp32 instructions (one issue for two lanes, each
// lane rounded as its scalar operation)
// ---------------------------------------------------------------------------

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Four channel pairs of a 16-byte segment of 16-bit values.
__device__ __forceinline__ void widen_pairs(const uint4 &u, float2 (&f)[4], __nv_bfloat16) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    f[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
}
__device__ __forceinline__ void widen_pairs(const uint4 &u, float2 (&f)[4], __half) {
  const __half2 *h = reinterpret_cast<const __half2 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) f[i] = __half22float2(h[i]);
}
__device__ __forceinline__ uint4 pack_pairs(const float2 (&y)[4], __half) {
  uint4 u;
  __half2 *h = reinterpret_cast<__half2 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2half2_rn(y[i].x, y[i].y);
  return u;
}
__device__ __forceinline__ uint4 pack_pairs(const float2 (&y)[4], __nv_bfloat16) {
  uint4 u;
  __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(y[i].x, y[i].y);
  return u;
}

// SiLU of a channel pair from its definition: a * sigma(a) with sigma(a) = 1 / (1 +
// 2^(-a log2 e)) on the hardware's approximate base-2 exponential and reciprocal
// (PTX ex2.approx, rcp.approx; relative errors of a few 2^-23).  For a -> -inf the
// exponential overflows to +inf and the result is -0.  conv4_silu_pair first applies
// the width-4 causal conv, taps w0..w3 on x[t-3], x[t-2], x[t-1], x[t], in that order.
__device__ __forceinline__ float2 silu_pair(float2 a) {
  float2 d = __fmul2_rn(a, make_float2(-1.4426950408889634f, -1.4426950408889634f));
  d.x = ex2_approx(d.x);
  d.y = ex2_approx(d.y);
  d = __fadd2_rn(d, make_float2(1.f, 1.f));
  d.x = rcp_approx(d.x);
  d.y = rcp_approx(d.y);
  return __fmul2_rn(a, d);
}
__device__ __forceinline__ float2 conv4_silu_pair(float2 w0, float2 w1, float2 w2, float2 w3,
                                                  float2 x3, float2 x2, float2 x1, float2 x0) {
  float2 a = __fmul2_rn(w0, x3);
  a = __ffma2_rn(w1, x2, a);
  a = __ffma2_rn(w2, x1, a);
  a = __ffma2_rn(w3, x0, a);
  return silu_pair(a);
}

// Bounded log-decay gate ("Kimi K3的线性注意力：从源码看懂KDA如何更新记忆", 彩蛋, the
// gate.py excerpt): g = lb * sigmoid(a * (graw + bias)) with a = exp(A_log[h]),
// bias = dt_bias[h][channel] and lb the lower bound (-5 in K3), in fp32.
__device__ __forceinline__ float bounded_gate(float graw, float a, float bias, float lb) {
  const float z = a * (graw + bias);
  return lb * __fdividef(1.f, 1.f + __expf(-z));  // 1/(1 + inf) = 0 for very negative z
}

// ---------------------------------------------------------------------------
// Device status word (one per device, a file-scope device variable)
// ---------------------------------------------------------------------------

// Record the first fault code; later faults keep the first one.
__device__ __forceinline__ void report(int *status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// Debug builds (compiled with -DKDA_DEBUG, the library libkda_debug.so): every
// index a kernel derives from the call's data or arithmetic (sequence, token,
// chunk, record, segment, state and cache indices) is checked against its extent
// before the access that uses it.  An index out of range records
// KDA_ERR_DEVICE_BOUNDS and the access (or the whole item, where the index is
// the same for the CTA) is skipped, so the fault shows in the status word and
// never as a memory fault.  In release builds the checks compile to nothing.
#ifdef KDA_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif

__device__ __forceinline__ bool in_range(int *status, long long i, long long n) {
  if constexpr (kDebugChecks) {
    if (i < 0 || i >= n) {
      if (status) atomicCAS(status, 0, KDA_ERR_DEVICE_BOUNDS);
      return false;
    }
  }
  return true;
}

// Sequence bounds from cu_seqlens with device-side validation: a malformed
// entry (decreasing or outside [0, T]) is clamped and recorded.
__device__ __forceinline__ void seq_bounds(const int32_t *cu, int n, int T, int *status,
                                           int &bos, int &eos) {
  if (cu == nullptr) {
    bos = 0;
    eos = T;
    return;
  }
  int a = cu[n], b = cu[n + 1];
  if (a < 0 || b < a || b > T) {
    report(status, KDA_ERR_DEVICE_BOUNDS);
    a = min(max(a, 0), T);
    b = min(max(b, a), T);
  }
  bos = a;
  eos = b;
}

// Index of the sequence containing token t (cu sorted); -1 if none.
__device__ __forceinline__ int seq_of_token(const int32_t *cu, int N, int t) {
  if (cu == nullptr) return 0;
  int lo = 0, hi = N - 1, ans = -1;
  while (lo <= hi) {
    int mid = (lo + hi) >> 1;
    if (cu[mid] <= t) {
      ans = mid;
      lo = mid + 1;
    } else {
      hi = mid - 1;
    }
  }
  return ans;
}

}  // namespace kda

// Host-side launchers implemented in the kernel files, called by kda_api.cu.
namespace kda {
// Device addresses of the file-scope __device__ status word (kda_status.cu)
// and of the fixed scratch of kda_chunk_fwd_static (kda_static.cu) on the
// current device, looked up once per device.
cudaError_t status_word_address(int **out);
cudaError_t static_scratch_address(void **out);
// One CTA whose bounded mbarrier wait runs out after limit_us (kda_selftest.cu).
cudaError_t launch_wait_timeout(unsigned limit_us, int *status, cudaStream_t s);
// One checked write of a four-slot probe array at `index` (debug builds only;
// cudaErrorNotSupported in release builds).
cudaError_t launch_bounds_probe(int index, int *status, cudaStream_t s);
cudaError_t launch_prologue(const void *x, const float *w, const void *cache_in, void *cache_out,
                            const int32_t *cu, int N, int T, int H, int D, kda_dtype dt,
                            kda_dtype out_dt, void *q, void *k, void *v, int *status,
                            cudaStream_t s);
cudaError_t launch_decode(const void *x, const float *w, void *cache, const void *g,
                          const float *beta, float scale, float *state, int N, int H, int D,
                          kda_dtype dt, float *o, const float *A_log, const float *dt_bias,
                          float lower_bound, bool gated, int *status, cudaStream_t s);
cudaError_t launch_epilogue(const float *o, const void *gate, const float *weight, float eps,
                            long long rows, int D, kda_dtype dt, void *out, cudaStream_t s);
cudaError_t launch_chunk_simt(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, float scale, const float *s0,
                              const int32_t *cu, int N, int T, int H, int D, int chunk,
                              kda_dtype dt, float *o, float *sN, int *status, cudaStream_t s);
cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float scale, const float *s0, const int32_t *cu,
                            int N, int T, int H, kda_dtype dt, float *o, float *sN, int *status,
                            cudaStream_t s);
// Two-pass tensor-core prefill (kda_chunk_record.cuh): the prep pass over all
// (chunk, head) items, then the state pass over (segment, head, value slice);
// L is the segment length in chunks (0: whole sequences), and with L > 0 the
// index pass must run (for cu == NULL too) and the state pass is the
// transition pass, the entry-state scan and the output pass.
// g: fp32 log-decay, or (gated) 16-bit gate pre-activations of type dt turned
// into the log-decay in the kernel (A_log, dt_bias may be null).
//
// Windows (kda_chunk_fwd_windowed_ws): the passes may run over a window [lo, hi) of
// the batch's chunk numbers (all sequences' chunks in order) at a time, with the
// window's records at slots 0 .. hi - lo of the workspace.  A sequence that starts
// before the window enters from carry_in and one that continues past it leaves its
// state in carry_out ([H][Dv][Dk] fp32 each; one sequence at most crosses a window
// boundary).  The default window is the whole batch.
struct ChunkWindow {
  int lo = 0;
  int hi = 0x7fffffff;
  const float *carry_in = nullptr;
  float *carry_out = nullptr;
};
cudaError_t launch_chunk_prep(const void *q, const void *k, const void *v, const void *g,
                              const float *beta, const int32_t *cu, int N, int T, int H,
                              kda_dtype dt, void *ws, const float *A_log, const float *dt_bias,
                              float lower_bound, bool gated, int *status, cudaStream_t s,
                              const ChunkWindow &win = ChunkWindow{});
cudaError_t launch_chunk_index(const int32_t *cu, int N, int T, int L, void *ws, int *status,
                               cudaStream_t s);
// ckpt (optional, [chunks][H][Dv][Dk] fp32 in record order): the entry state of
// every chunk, for the backward pass; o may then be NULL.
cudaError_t launch_chunk_state(const void *ws, const int32_t *cu, const float *s0, float scale,
                               int N, int T, int H, int L, float *o, float *sN, int *status,
                               cudaStream_t s, float *ckpt = nullptr,
                               const ChunkWindow &win = ChunkWindow{});
// Affine map of every sequence (one segment each; records from the prep pass):
// map_m [N][H][Dk][Dk] with M[t][k] at k * Dk + t, map_b [N][H][Dv][Dk] like a state.
cudaError_t launch_chunk_map(const void *ws, const int32_t *cu, int N, int T, int H, float *map_m,
                             float *map_b, int *status, cudaStream_t s);
// E_out = M E_in + B for NH (sequence, head) pairs (E_in NULL: zero); E_out must not
// overlap the inputs.
cudaError_t launch_state_compose(const float *M, const float *B, const float *E_in, float *E_out,
                                 int NH, cudaStream_t s);
// Backward of the two-pass prefill (kda_chunk_bwd.cu): the reverse state pass over
// (sequence, head, value slice) writing the adjoint of every chunk's exit state
// (dckpt, record order) and d_s0, then the local pass over (chunk, head).
cudaError_t launch_chunk_bwd_state(const void *ws, const int32_t *cu, const float *dsN,
                                   const float *dout, float scale, int N, int T, int H,
                                   float *dckpt, float *ds0, int *status, cudaStream_t s);
// scratch: chunk_bwd_local_scratch_bytes() (one slot per CTA of the persistent grid).
size_t chunk_bwd_local_scratch_bytes();
cudaError_t launch_chunk_bwd_local(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, const float *dout, float scale,
                                   const int32_t *cu, const void *ws, const float *ckpt,
                                   const float *dckpt, float *scratch, int N, int T, int H,
                                   kda_dtype dt, float *dq, float *dk, float *dv, float *dg,
                                   float *dbeta, int *status, cudaStream_t s);
cudaError_t launch_prologue_chunk_prep(const void *x, const float *conv_w, const void *cache_in,
                                       void *cache_out, const void *g, const float *beta,
                                       const int32_t *cu, int N, int T, int H, kda_dtype dt,
                                       void *ws, const float *A_log, const float *dt_bias,
                                       float lower_bound, bool gated, int *status,
                                       cudaStream_t s, const ChunkWindow &win = ChunkWindow{});
cudaError_t launch_cache_pass(const void *ws, int N, int H, const void *cache_in,
                              void *cache_out, cudaStream_t s);
cudaError_t launch_prologue_chunk_tc(const void *x, const float *conv_w, const void *cache_in,
                                     void *cache_out, const float *g, const float *beta,
                                     float scale, const float *s0, const int32_t *cu, int N,
                                     int T, int H, kda_dtype dt, float *o, float *sN,
                                     int *status, cudaStream_t s);
}  // namespace kda
