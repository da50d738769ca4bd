// Host side of the libkda C ABI: argument validation, error reporting and
// dispatch to the kernels.  No entry point allocates device memory: the status
// word (kda_status.cu) and the scratch of kda_chunk_fwd_static (kda_static.cu)
// are file-scope __device__ variables.
#include <algorithm>
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "kda_chunk_record.cuh"
#include "kda_common.cuh"

namespace {

thread_local std::string g_last_error = "no error";

kda_status fail(kda_status code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

kda_status cuda_fail(cudaError_t e, const char *what) {
  return fail(KDA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// The status word of the current device: a __device__ int of kda_status.cu,
// looked up once per device; nothing is allocated.
kda_status device_status_word(int **out) {
  cudaError_t e = kda::status_word_address(out);
  if (e != cudaSuccess) return cuda_fail(e, "status word address");
  return KDA_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void *a, size_t na, const void *b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  auto pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

size_t esize(kda_dtype dt) { return dt == KDA_F32 ? 4 : 2; }

bool valid_dtype(kda_dtype dt) { return dt == KDA_F32 || dt == KDA_BF16 || dt == KDA_F16; }

bool supported_d(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }

#define KDA_REQUIRE(cond, ...) \
  do {                         \
    if (!(cond)) return fail(KDA_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

#define KDA_REQUIRE_PTR(p, name)                                                    \
  do {                                                                              \
    if ((p) == nullptr) return fail(KDA_ERR_INVALID_ARG, "%s is NULL", name);       \
    if (!aligned16(p)) return fail(KDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name); \
  } while (0)

// Arrays read element by element (beta, cu_seqlens) only need 4-byte alignment.
#define KDA_REQUIRE_PTR4(p, name)                                                   \
  do {                                                                              \
    if ((p) == nullptr) return fail(KDA_ERR_INVALID_ARG, "%s is NULL", name);       \
    if (reinterpret_cast<uintptr_t>(p) & 3u)                                        \
      return fail(KDA_ERR_INVALID_ARG, "%s is not 4-byte aligned", name);           \
  } while (0)

#define KDA_OPT_PTR4(p, name)                                                       \
  do {                                                                              \
    if ((p) != nullptr && (reinterpret_cast<uintptr_t>(p) & 3u))                    \
      return fail(KDA_ERR_INVALID_ARG, "%s is not 4-byte aligned", name);           \
  } while (0)

#define KDA_OPT_PTR(p, name)                                                        \
  do {                                                                              \
    if ((p) != nullptr && !aligned16(p))                                            \
      return fail(KDA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);          \
  } while (0)

}  // namespace

extern "C" {

const char *kda_last_error(void) { return g_last_error.c_str(); }

const char *kda_version(void) { return "libkda 0.1 (sm_100a)"; }

kda_status kda_output_epilogue(const float *o, const void *gate, const float *weight, float eps,
                               int T, int H, int D, kda_dtype dt, void *out,
                               kda_stream_t stream) {
  KDA_REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  KDA_REQUIRE(T >= 0 && H >= 1 && D >= 1, "bad sizes T=%d H=%d D=%d", T, H, D);
  if (!supported_d(D)) return fail(KDA_ERR_UNSUPPORTED, "epilogue: D=%d not in {16,32,64,128}", D);
  KDA_REQUIRE(eps >= 0.f && eps < 1e30f, "eps must be finite and non-negative");
  KDA_REQUIRE_PTR(weight, "weight");
  if (T == 0) return KDA_OK;
  KDA_REQUIRE_PTR(o, "o");
  KDA_REQUIRE_PTR(gate, "gate");
  KDA_REQUIRE_PTR(out, "out");
  const size_t n = (size_t)T * H * D, es = esize(dt);
  KDA_REQUIRE(!overlaps(out, n * es, o, n * 4), "out overlaps o");
  KDA_REQUIRE(!overlaps(out, n * es, gate, n * es), "out overlaps gate");
  KDA_REQUIRE(!overlaps(out, n * es, weight, (size_t)D * 4), "out overlaps weight");
  cudaError_t e = kda::launch_epilogue(o, gate, weight, eps, (long long)T * H, D, dt, out,
                                       (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kda_output_epilogue launch");
  return KDA_OK;
}

kda_status kda_selftest_wait_timeout(unsigned limit_us, kda_stream_t stream) {
  KDA_REQUIRE(limit_us >= 1 && limit_us <= 2000000u, "limit_us=%u outside [1, 2000000]",
              limit_us);
  int *status = nullptr;
  kda_status st = device_status_word(&status);
  if (st != KDA_OK) return st;
  const cudaError_t e = kda::launch_wait_timeout(limit_us, status, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kda_selftest_wait_timeout launch");
  return KDA_OK;
}

int kda_debug_build(void) { return kda::kDebugChecks ? 1 : 0; }

kda_status kda_selftest_bounds(int index, kda_stream_t stream) {
  if (!kda::kDebugChecks)
    return fail(KDA_ERR_UNSUPPORTED,
                "kda_selftest_bounds: a release build (the index checks are compiled out)");
  int *status = nullptr;
  kda_status st = device_status_word(&status);
  if (st != KDA_OK) return st;
  const cudaError_t e = kda::launch_bounds_probe(index, status, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kda_selftest_bounds launch");
  return KDA_OK;
}

kda_status kda_get_device_status(int *code) {
  KDA_REQUIRE(code != nullptr, "code is NULL");
  int *word = nullptr;
  kda_status st = device_status_word(&word);
  if (st != KDA_OK) return st;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  int host = 0;
  e = cudaMemcpy(&host, word, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(status word)");
  e = cudaMemset(word, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(status word)");
  *code = host;
  return KDA_OK;
}

kda_status kda_prologue(const void *x, const float *conv_w, const void *cache_in,
                        void *cache_out, const int32_t *cu_seqlens, int N, int T, int H,
                        int D, kda_dtype dt, kda_dtype out_dt, void *q, void *k, void *v,
                        kda_stream_t stream) {
  KDA_REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  KDA_REQUIRE(valid_dtype(out_dt), "unknown output dtype %d", (int)out_dt);
  KDA_REQUIRE(N >= 1 && T >= 0 && H >= 1 && D >= 1, "bad sizes N=%d T=%d H=%d D=%d", N, T, H, D);
  KDA_REQUIRE(cu_seqlens != nullptr || N == 1, "cu_seqlens is NULL but N=%d", N);
  if (!supported_d(D)) return fail(KDA_ERR_UNSUPPORTED, "prologue: D=%d not in {16,32,64,128}", D);
  KDA_REQUIRE((long long)H * D * 3 < (1LL << 31), "3*H*D too large");
  if (T > 0) {
    KDA_REQUIRE_PTR(x, "x");
    KDA_REQUIRE_PTR(q, "q");
    KDA_REQUIRE_PTR(k, "k");
    KDA_REQUIRE_PTR(v, "v");
  }
  KDA_REQUIRE_PTR(conv_w, "conv_w");
  KDA_OPT_PTR(cache_in, "cache_in");
  KDA_OPT_PTR(cache_out, "cache_out");
  KDA_OPT_PTR4(cu_seqlens, "cu_seqlens");
  const size_t C = (size_t)3 * H * D, es = esize(dt);
  const size_t act = (size_t)T * H * D * esize(out_dt), cache_bytes = (size_t)N * 3 * C * es;
  KDA_REQUIRE(!overlaps(cache_in, cache_bytes, cache_out, cache_bytes),
              "cache_out overlaps cache_in");
  const void *outs[3] = {q, k, v};
  for (int i = 0; i < 3; ++i) {
    KDA_REQUIRE(!overlaps(outs[i], act, x, (size_t)T * C * es), "output overlaps x");
    for (int j = i + 1; j < 3; ++j)
      KDA_REQUIRE(!overlaps(outs[i], act, outs[j], act), "q/k/v outputs overlap");
  }
  int *status = nullptr;
  kda_status st = device_status_word(&status);
  if (st != KDA_OK) return st;
  cudaError_t e = kda::launch_prologue(x, conv_w, cache_in, cache_out, cu_seqlens, N, T, H, D,
                                       dt, out_dt, q, k, v, status, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kda_prologue launch");
  return KDA_OK;
}

}  // extern "C"

namespace {

bool chunk_tc_path(int T, int Dk, int Dv, int chunk, kda_dtype dt) {
  return dt != KDA_F32 && Dk == 128 && Dv == 128 && chunk == 64 && T > 0;
}

// Argument checks shared by kda_chunk_fwd and kda_chunk_fwd_ws.
kda_status check_chunk_args(const void *q, const void *k, const void *v, const void *g,
                            const float *beta, const float *initial_state,
                            const int32_t *cu_seqlens, int N, int T, int H, int Dk, int Dv,
                            int chunk, kda_dtype dt, float *o, float *final_state,
                            size_t g_elem_bytes = 4) {
  KDA_REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  KDA_REQUIRE(N >= 1 && T >= 0 && H >= 1 && Dk >= 1 && Dv >= 1,
              "bad sizes N=%d T=%d H=%d Dk=%d Dv=%d", N, T, H, Dk, Dv);
  KDA_REQUIRE(cu_seqlens != nullptr || N == 1, "cu_seqlens is NULL but N=%d", N);
  if (Dk != Dv || !supported_d(Dk))
    return fail(KDA_ERR_UNSUPPORTED, "chunk_fwd: Dk=%d Dv=%d (need Dk == Dv in {16,32,64,128})",
                Dk, Dv);
  if (chunk != 16 && chunk != 32 && chunk != 64)
    return fail(KDA_ERR_UNSUPPORTED, "chunk_fwd: chunk=%d not in {16,32,64}", chunk);
  if (T > 0) {
    KDA_REQUIRE_PTR(q, "q");
    KDA_REQUIRE_PTR(k, "k");
    KDA_REQUIRE_PTR(v, "v");
    KDA_REQUIRE_PTR(g, "g");
    KDA_REQUIRE_PTR4(beta, "beta");
    KDA_REQUIRE_PTR(o, "o");
  }
  KDA_OPT_PTR(initial_state, "initial_state");
  KDA_OPT_PTR(final_state, "final_state");
  KDA_OPT_PTR4(cu_seqlens, "cu_seqlens");
  const size_t es = esize(dt);
  const size_t act = (size_t)T * H * Dk * es, obytes = (size_t)T * H * Dv * sizeof(float);
  const size_t sbytes = (size_t)N * H * Dv * Dk * sizeof(float);
  const void *ins[5] = {q, k, v, g, beta};
  const size_t insz[5] = {act, act, (size_t)T * H * Dv * es, (size_t)T * H * Dk * g_elem_bytes,
                          (size_t)T * H * 4};
  for (int i = 0; i < 5; ++i)
    KDA_REQUIRE(!overlaps(o, obytes, ins[i], insz[i]), "o overlaps an input");
  KDA_REQUIRE(!overlaps(o, obytes, final_state, sbytes), "o overlaps final_state");
  KDA_REQUIRE(final_state == initial_state ||
                  !overlaps(final_state, sbytes, initial_state, sbytes),
              "final_state partially overlaps initial_state");
  return KDA_OK;
}

// Gate parameters of the *_gated entry points.  The chunk kernels need
// g >= -5 (their decay-range argument), so their lower bound is in [-5, 0).
kda_status check_gate_args(const float *A_log, const float *dt_bias, float lower_bound,
                           bool chunk_path) {
  KDA_REQUIRE(lower_bound == lower_bound && lower_bound < 0.f && lower_bound > -1e30f,
              "lower_bound must be finite and negative (got %g)", (double)lower_bound);
  if (chunk_path && lower_bound < -5.f)
    return fail(KDA_ERR_UNSUPPORTED,
                "gated chunk path: lower_bound %g < -5 is outside the decay range the tensor-core "
                "kernels are built for", (double)lower_bound);
  KDA_OPT_PTR4(A_log, "A_log");
  KDA_OPT_PTR(dt_bias, "dt_bias");
  return KDA_OK;
}

}  // namespace

extern "C" {

kda_status kda_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                         const float *beta, float scale, const float *initial_state,
                         const int32_t *cu_seqlens, int N, int T, int H, int Dk, int Dv,
                         int chunk, kda_dtype dt, float *o, float *final_state,
                         kda_stream_t stream) {
  kda_status st = check_chunk_args(q, k, v, g, beta, initial_state, cu_seqlens, N, T, H, Dk, Dv,
                                   chunk, dt, o, final_state);
  if (st != KDA_OK) return st;
  int *status = nullptr;
  st = device_status_word(&status);
  if (st != KDA_OK) return st;
  if (T == 0 && final_state == nullptr) return KDA_OK;
  cudaError_t e;
  if (chunk_tc_path(T, Dk, Dv, chunk, dt)) {
    e = kda::launch_chunk_tc(q, k, v, g, beta, scale, initial_state, cu_seqlens, N, T, H, dt, o,
                             final_state, status, (cudaStream_t)stream);
  } else {
    e = kda::launch_chunk_simt(q, k, v, g, beta, scale, initial_state, cu_seqlens, N, T, H, Dk,
                               chunk, dt, o, final_state, status, (cudaStream_t)stream);
  }
  if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd launch");
  return KDA_OK;
}

size_t kda_chunk_fwd_workspace_bytes(int N, int T, int H, int Dk, int Dv, int chunk,
                                     kda_dtype dt) {
  if (N < 1 || T < 0 || H < 1 || !chunk_tc_path(T, Dk, Dv, chunk, dt)) return 0;
  return kda::rec::workspace_bytes(N, T, H, kda::rec::segment_chunks(N, T, H));
}

size_t kda_chunk_fwd_segmented_workspace_bytes(int N, int T, int H, int Dk, int Dv, int chunk,
                                               kda_dtype dt, int segment_chunks) {
  if (N < 1 || T < 0 || H < 1 || segment_chunks < 0 || !chunk_tc_path(T, Dk, Dv, chunk, dt))
    return 0;
  return kda::rec::workspace_bytes(N, T, H, segment_chunks);
}

size_t kda_chunk_fwd_windowed_workspace_bytes(int N, int T, int H, int Dk, int Dv, int chunk,
                                              kda_dtype dt, int window_chunks) {
  if (N < 1 || T < 0 || H < 1 || window_chunks < 1 || !chunk_tc_path(T, Dk, Dv, chunk, dt))
    return 0;
  return kda::rec::windowed_workspace_bytes(N, H, window_chunks);
}

int kda_chunk_fwd_segment_chunks(int N, int T, int H) {
  if (N < 1 || T < 0 || H < 1) return 0;
  return kda::rec::segment_chunks(N, T, H);
}

}  // extern "C"

namespace {

// The two-pass tensor-core prefill on a caller workspace, with g either the
// fp32 log-decay or (gated) 16-bit gate pre-activations.  Arguments other than
// the workspace have been checked.
kda_status chunk_two_pass(const void *q, const void *k, const void *v, const void *g,
                          size_t g_elem_bytes, const float *A_log, const float *dt_bias,
                          float lower_bound, bool gated, const float *beta, float scale,
                          const float *initial_state, const int32_t *cu_seqlens, int N, int T,
                          int H, int Dk, int Dv, kda_dtype dt, float *o, float *final_state,
                          void *workspace, size_t workspace_bytes, cudaStream_t s,
                          const char *what, int L, int window = 0) {
  const size_t need = window > 0 ? kda::rec::windowed_workspace_bytes(N, H, window)
                                 : kda::rec::workspace_bytes(N, T, H, L);
  KDA_OPT_PTR(workspace, "workspace");
  KDA_REQUIRE(workspace_bytes >= need, "workspace holds %zu bytes, these sizes need %zu",
              workspace_bytes, need);
  {
    const size_t es = esize(dt), act = (size_t)T * H * Dk * es;
    const size_t sbytes = (size_t)N * H * Dv * Dk * sizeof(float);
    const void *others[10] = {q, k, v, g, beta, o, initial_state, final_state, A_log, dt_bias};
    const size_t osz[10] = {act, act, act, (size_t)T * H * Dk * g_elem_bytes, (size_t)T * H * 4,
                            (size_t)T * H * Dv * 4, sbytes, sbytes, (size_t)H * 4,
                            (size_t)H * Dk * 4};
    for (int i = 0; i < 10; ++i)
      KDA_REQUIRE(!overlaps(workspace, need, others[i], osz[i]),
                  "workspace overlaps another argument");
    KDA_REQUIRE(!overlaps(workspace, need, cu_seqlens, (size_t)(N + 1) * 4),
                "workspace overlaps cu_seqlens");
  }
  int *status = nullptr;
  kda_status st = device_status_word(&status);
  if (st != KDA_OK) return st;
  cudaError_t e = cudaSuccess;
  if (cu_seqlens || L > 0)
    e = kda::launch_chunk_index(cu_seqlens, N, T, L, workspace, status, s);
  if (window > 0) {
    // One window of chunk numbers at a time: the prep pass writes the window's records,
    // the state pass consumes them; a sequence crossing a window boundary hands its state
    // over through the two carry blocks (alternating).  The real chunk total is known on
    // the device only, so the windows cover the capacity bound; past the total they are
    // empty and their CTAs exit at once.
    float *carry = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                             kda::rec::windowed_carry_offset(N, H, window));
    const size_t carry_floats = (size_t)H * 128 * 128;
    const long long cap = kda::rec::chunk_capacity(N, T);
    for (long long lo = 0, w = 0; lo < cap && e == cudaSuccess; lo += window, ++w) {
      kda::ChunkWindow win;
      win.lo = (int)lo;
      win.hi = (int)std::min<long long>(lo + window, 0x7fffffffLL);
      win.carry_in = carry + (size_t)(w & 1) * carry_floats;
      win.carry_out = carry + (size_t)((w + 1) & 1) * carry_floats;
      e = kda::launch_chunk_prep(q, k, v, g, beta, cu_seqlens, N, T, H, dt, workspace, A_log,
                                 dt_bias, lower_bound, gated, status, s, win);
      if (e == cudaSuccess)
        e = kda::launch_chunk_state(workspace, cu_seqlens, initial_state, scale, N, T, H, 0, o,
                                    final_state, status, s, nullptr, win);
    }
    if (e != cudaSuccess) return cuda_fail(e, what);
    return KDA_OK;
  }
  if (e == cudaSuccess)
    e = kda::launch_chunk_prep(q, k, v, g, beta, cu_seqlens, N, T, H, dt, workspace, A_log,
                               dt_bias, lower_bound, gated, status, s);
  if (e == cudaSuccess)
    e = kda::launch_chunk_state(workspace, cu_seqlens, initial_state, scale, N, T, H, L, o,
                                final_state, status, s);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return KDA_OK;
}

}  // namespace

extern "C" {

kda_status kda_chunk_fwd_ws(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float scale, const float *initial_state,
                            const int32_t *cu_seqlens, int N, int T, int H, int Dk, int Dv,
                            int chunk, kda_dtype dt, float *o, float *final_state,
                            void *workspace, size_t workspace_bytes, kda_stream_t stream) {
  if (workspace == nullptr)
    return kda_chunk_fwd(q, k, v, g, beta, scale, initial_state, cu_seqlens, N, T, H, Dk, Dv,
                         chunk, dt, o, final_state, stream);
  kda_status st = check_chunk_args(q, k, v, g, beta, initial_state, cu_seqlens, N, T, H, Dk, Dv,
                                   chunk, dt, o, final_state);
  if (st != KDA_OK) return st;
  if (kda_chunk_fwd_workspace_bytes(N, T, H, Dk, Dv, chunk, dt) == 0)
    return kda_chunk_fwd(q, k, v, g, beta, scale, initial_state, cu_seqlens, N, T, H, Dk, Dv,
                         chunk, dt, o, final_state, stream);
  return chunk_two_pass(q, k, v, g, 4, nullptr, nullptr, 0.f, false, beta, scale, initial_state,
                        cu_seqlens, N, T, H, Dk, Dv, dt, o, final_state, workspace,
                        workspace_bytes, (cudaStream_t)stream, "kda_chunk_fwd_ws launch",
                        kda::rec::segment_chunks(N, T, H));
}

kda_status kda_chunk_fwd_segmented_ws(const void *q, const void *k, const void *v,
                                      const float *g, const float *beta, float scale,
                                      const float *initial_state, const int32_t *cu_seqlens,
                                      int N, int T, int H, int Dk, int Dv, int chunk,
                                      kda_dtype dt, float *o, float *final_state,
                                      int segment_chunks, void *workspace,
                                      size_t workspace_bytes, kda_stream_t stream) {
  kda_status st = check_chunk_args(q, k, v, g, beta, initial_state, cu_seqlens, N, T, H, Dk, Dv,
                                   chunk, dt, o, final_state);
  if (st != KDA_OK) return st;
  if (!chunk_tc_path(T, Dk, Dv, chunk, dt))
    return fail(KDA_ERR_UNSUPPORTED, "chunk_fwd_segmented: needs bf16/f16, Dk == Dv == 128, "
                                     "chunk 64 and T > 0 (got dt=%d Dk=%d chunk=%d T=%d)",
                (int)dt, Dk, chunk, T);
  KDA_REQUIRE(segment_chunks >= 0, "segment_chunks=%d is negative", segment_chunks);
  KDA_REQUIRE(workspace != nullptr, "chunk_fwd_segmented: workspace is NULL");
  return chunk_two_pass(q, k, v, g, 4, nullptr, nullptr, 0.f, false, beta, scale, initial_state,
                        cu_seqlens, N, T, H, Dk, Dv, dt, o, final_state, workspace,
                        workspace_bytes, (cudaStream_t)stream, "kda_chunk_fwd_segmented_ws launch",
                        segment_chunks);
}

kda_status kda_chunk_fwd_windowed_ws(const void *q, const void *k, const void *v,
                                     const float *g, const float *beta, float scale,
                                     const float *initial_state, const int32_t *cu_seqlens,
                                     int N, int T, int H, int Dk, int Dv, int chunk,
                                     kda_dtype dt, float *o, float *final_state,
                                     int window_chunks, void *workspace, size_t workspace_bytes,
                                     kda_stream_t stream) {
  kda_status st = check_chunk_args(q, k, v, g, beta, initial_state, cu_seqlens, N, T, H, Dk, Dv,
                                   chunk, dt, o, final_state);
  if (st != KDA_OK) return st;
  if (!chunk_tc_path(T, Dk, Dv, chunk, dt))
    return fail(KDA_ERR_UNSUPPORTED, "chunk_fwd_windowed: needs bf16/f16, Dk == Dv == 128, "
                                     "chunk 64 and T > 0 (got dt=%d Dk=%d chunk=%d T=%d)",
                (int)dt, Dk, chunk, T);
  KDA_REQUIRE(window_chunks >= 1, "window_chunks=%d must be at least 1", window_chunks);
  KDA_REQUIRE(workspace != nullptr, "chunk_fwd_windowed: workspace is NULL");
  return chunk_two_pass(q, k, v, g, 4, nullptr, nullptr, 0.f, false, beta, scale, initial_state,
                        cu_seqlens, N, T, H, Dk, Dv, dt, o, final_state, workspace,
                        workspace_bytes, (cudaStream_t)stream, "kda_chunk_fwd_windowed_ws launch",
                        0, window_chunks);
}

kda_status kda_chunk_fwd_gated_ws(const void *q, const void *k, const void *v, const void *g_raw,
                                  const float *A_log, const float *dt_bias, float lower_bound,
                                  const float *beta, float scale, const float *initial_state,
                                  const int32_t *cu_seqlens, int N, int T, int H, int Dk, int Dv,
                                  int chunk, kda_dtype dt, float *o, float *final_state,
                                  void *workspace, size_t workspace_bytes, kda_stream_t stream) {
  kda_status st = check_chunk_args(q, k, v, g_raw, beta, initial_state, cu_seqlens, N, T, H, Dk,
                                   Dv, chunk, dt, o, final_state, esize(dt));
  if (st != KDA_OK) return st;
  if (!chunk_tc_path(T, Dk, Dv, chunk, dt))
    return fail(KDA_ERR_UNSUPPORTED, "chunk_fwd_gated: needs bf16/f16, Dk == Dv == 128, chunk 64 "
                                     "and T > 0 (got dt=%d Dk=%d chunk=%d T=%d)",
                (int)dt, Dk, chunk, T);
  st = check_gate_args(A_log, dt_bias, lower_bound, true);
  if (st != KDA_OK) return st;
  KDA_REQUIRE(workspace != nullptr, "chunk_fwd_gated: workspace is NULL");
  return chunk_two_pass(q, k, v, g_raw, esize(dt), A_log, dt_bias, lower_bound, true, beta, scale,
                        initial_state, cu_seqlens, N, T, H, Dk, Dv, dt, o, final_state,
                        workspace, workspace_bytes, (cudaStream_t)stream,
                        "kda_chunk_fwd_gated_ws launch", kda::rec::segment_chunks(N, T, H));
}

kda_status kda_chunk_fwd_static(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, float scale, const float *initial_state,
                                const int32_t *cu_seqlens, int N, int T, int H, int Dk,
                                int Dv, int chunk, kda_dtype dt, float *o, float *final_state,
                                kda_stream_t stream) {
  kda_status st = check_chunk_args(q, k, v, g, beta, initial_state, cu_seqlens, N, T, H, Dk, Dv,
                                   chunk, dt, o, final_state);
  if (st != KDA_OK) return st;
  const size_t need = kda_chunk_fwd_workspace_bytes(N, T, H, Dk, Dv, chunk, dt);
  if (need == 0)
    return kda_chunk_fwd(q, k, v, g, beta, scale, initial_state, cu_seqlens, N, T, H, Dk, Dv,
                         chunk, dt, o, final_state, stream);
  if (need > KDA_CHUNK_STATIC_SCRATCH_BYTES)
    return fail(KDA_ERR_UNSUPPORTED,
                "kda_chunk_fwd_static: N=%d T=%d H=%d needs %zu bytes of scratch, the static "
                "buffer holds %zu (use kda_chunk_fwd_ws with a caller workspace)",
                N, T, H, need, (size_t)KDA_CHUNK_STATIC_SCRATCH_BYTES);
  void *scratch = nullptr;
  const cudaError_t e = kda::static_scratch_address(&scratch);
  if (e != cudaSuccess) return cuda_fail(e, "static scratch address");
  return chunk_two_pass(q, k, v, g, 4, nullptr, nullptr, 0.f, false, beta, scale, initial_state,
                        cu_seqlens, N, T, H, Dk, Dv, dt, o, final_state, scratch,
                        KDA_CHUNK_STATIC_SCRATCH_BYTES, (cudaStream_t)stream,
                        "kda_chunk_fwd_static launch", kda::rec::segment_chunks(N, T, H));
}

}  // extern "C"

namespace {

kda_status check_fused_args(const void *x, const float *conv_w, const void *cache_in,
                            void *cache_out, const void *g, const float *beta,
                            const float *initial_state, const int32_t *cu_seqlens, int N, int T,
                            int H, int D, kda_dtype dt, float *o, float *final_state,
                            size_t g_elem_bytes = 4) {
  KDA_REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  KDA_REQUIRE(N >= 1 && T >= 1 && H >= 1 && D >= 1, "bad sizes N=%d T=%d H=%d D=%d", N, T, H, D);
  KDA_REQUIRE(cu_seqlens != nullptr || N == 1, "cu_seqlens is NULL but N=%d", N);
  if (D != 128 || dt == KDA_F32)
    return fail(KDA_ERR_UNSUPPORTED, "prologue_chunk_fwd: needs D=128 and bf16/f16 x (D=%d)", D);
  KDA_REQUIRE((long long)H * D * 3 < (1LL << 31), "3*H*D too large");
  KDA_REQUIRE_PTR(x, "x");
  KDA_REQUIRE_PTR(conv_w, "conv_w");
  KDA_REQUIRE_PTR(g, "g");
  KDA_REQUIRE_PTR4(beta, "beta");
  KDA_REQUIRE_PTR(o, "o");
  KDA_OPT_PTR(cache_in, "cache_in");
  KDA_OPT_PTR(cache_out, "cache_out");
  KDA_OPT_PTR(initial_state, "initial_state");
  KDA_OPT_PTR(final_state, "final_state");
  KDA_OPT_PTR4(cu_seqlens, "cu_seqlens");
  const size_t C = (size_t)3 * H * D, es = esize(dt);
  const size_t obytes = (size_t)T * H * D * sizeof(float);
  const size_t sbytes = (size_t)N * H * D * D * sizeof(float);
  const size_t cache_bytes = (size_t)N * 3 * C * es;
  KDA_REQUIRE(!overlaps(o, obytes, x, (size_t)T * C * es), "o overlaps x");
  KDA_REQUIRE(!overlaps(o, obytes, g, (size_t)T * H * D * g_elem_bytes), "o overlaps g");
  KDA_REQUIRE(!overlaps(o, obytes, beta, (size_t)T * H * 4), "o overlaps beta");
  KDA_REQUIRE(!overlaps(o, obytes, final_state, sbytes), "o overlaps final_state");
  KDA_REQUIRE(!overlaps(cache_in, cache_bytes, cache_out, cache_bytes),
              "cache_out overlaps cache_in");
  KDA_REQUIRE(final_state == initial_state ||
                  !overlaps(final_state, sbytes, initial_state, sbytes),
              "final_state partially overlaps initial_state");
  return KDA_OK;
}

}  // namespace

extern "C" {

kda_status kda_prologue_chunk_fwd(const void *x, const float *conv_w, const void *cache_in,
                                  void *cache_out, const float *g, const float *beta,
                                  float scale, const float *initial_state,
                                  const int32_t *cu_seqlens, int N, int T, int H, int D,
                                  kda_dtype dt, float *o, float *final_state,
                                  kda_stream_t stream) {
  kda_status st = check_fused_args(x, conv_w, cache_in, cache_out, g, beta, initial_state,
                                   cu_seqlens, N, T, H, D, dt, o, final_state);
  if (st != KDA_OK) return st;
  int *status = nullptr;
  st = device_status_word(&status);
  if (st != KDA_OK) return st;
  cudaError_t e = kda::launch_prologue_chunk_tc(x, conv_w, cache_in, cache_out, g, beta, scale,
                                                initial_state, cu_seqlens, N, T, H, dt, o,
                                                final_state, status, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kda_prologue_chunk_fwd launch");
  return KDA_OK;
}

}  // extern "C"

namespace {

// The two-pass prefill with the prologue in the prep pass (see chunk_two_pass).
kda_status fused_two_pass(const void *x, const float *conv_w, const void *cache_in,
                          void *cache_out, const void *g, size_t g_elem_bytes,
                          const float *A_log, const float *dt_bias, float lower_bound, bool gated,
                          const float *beta, float scale, const float *initial_state,
                          const int32_t *cu_seqlens, int N, int T, int H, int D, kda_dtype dt,
                          float *o, float *final_state, void *workspace, size_t workspace_bytes,
                          cudaStream_t s, const char *what, int window = 0) {
  const size_t need = window > 0 ? kda::rec::windowed_workspace_bytes(N, H, window)
                                 : kda_chunk_fwd_workspace_bytes(N, T, H, D, D, 64, dt);
  KDA_OPT_PTR(workspace, "workspace");
  KDA_REQUIRE(workspace_bytes >= need, "workspace holds %zu bytes, these sizes need %zu",
              workspace_bytes, need);
  {
    const size_t C = (size_t)3 * H * D, es = esize(dt);
    const size_t sbytes = (size_t)N * H * D * D * sizeof(float);
    const void *others[11] = {x, conv_w, cache_in, cache_out, g, beta, o, initial_state,
                              final_state, A_log, dt_bias};
    const size_t osz[11] = {(size_t)T * C * es, C * 4 * 4, (size_t)N * 3 * C * es,
                            (size_t)N * 3 * C * es, (size_t)T * H * D * g_elem_bytes,
                            (size_t)T * H * 4, (size_t)T * H * D * 4, sbytes, sbytes,
                            (size_t)H * 4, (size_t)H * D * 4};
    for (int i = 0; i < 11; ++i)
      KDA_REQUIRE(!overlaps(workspace, need, others[i], osz[i]),
                  "workspace overlaps another argument");
    KDA_REQUIRE(!overlaps(workspace, need, cu_seqlens, (size_t)(N + 1) * 4),
                "workspace overlaps cu_seqlens");
  }
  int *status = nullptr;
  kda_status st = device_status_word(&status);
  if (st != KDA_OK) return st;
  cudaError_t e = cudaSuccess;
  const int L = window > 0 ? 0 : kda::rec::segment_chunks(N, T, H);
  if (cu_seqlens || L > 0)
    e = kda::launch_chunk_index(cu_seqlens, N, T, L, workspace, status, s);
  if (window > 0) {  // one window of chunk numbers at a time (see chunk_two_pass)
    float *carry = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) +
                                             kda::rec::windowed_carry_offset(N, H, window));
    const size_t carry_floats = (size_t)H * 128 * 128;
    const long long cap = kda::rec::chunk_capacity(N, T);
    for (long long lo = 0, w = 0; lo < cap && e == cudaSuccess; lo += window, ++w) {
      kda::ChunkWindow win;
      win.lo = (int)lo;
      win.hi = (int)std::min<long long>(lo + window, 0x7fffffffLL);
      win.carry_in = carry + (size_t)(w & 1) * carry_floats;
      win.carry_out = carry + (size_t)((w + 1) & 1) * carry_floats;
      e = kda::launch_prologue_chunk_prep(x, conv_w, cache_in, cache_out, g, beta, cu_seqlens, N,
                                          T, H, dt, workspace, A_log, dt_bias, lower_bound, gated,
                                          status, s, win);
      if (e == cudaSuccess)
        e = kda::launch_chunk_state(workspace, cu_seqlens, initial_state, scale, N, T, H, 0, o,
                                    final_state, status, s, nullptr, win);
    }
  } else {
    if (e == cudaSuccess)
      e = kda::launch_prologue_chunk_prep(x, conv_w, cache_in, cache_out, g, beta, cu_seqlens, N,
                                          T, H, dt, workspace, A_log, dt_bias, lower_bound, gated,
                                          status, s);
    if (e == cudaSuccess)
      e = kda::launch_chunk_state(workspace, cu_seqlens, initial_state, scale, N, T, H, L, o,
                                  final_state, status, s);
  }
  if (e == cudaSuccess && cu_seqlens && cache_out)
    e = kda::launch_cache_pass(workspace, N, H, cache_in, cache_out, s);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return KDA_OK;
}

}  // namespace

extern "C" {

kda_status kda_prologue_chunk_fwd_ws(const void *x, const float *conv_w, const void *cache_in,
                                     void *cache_out, const float *g, const float *beta,
                                     float scale, const float *initial_state,
                                     const int32_t *cu_seqlens, int N, int T, int H, int D,
                                     kda_dtype dt, float *o, float *final_state,
                                     void *workspace, size_t workspace_bytes,
                                     kda_stream_t stream) {
  if (workspace == nullptr)
    return kda_prologue_chunk_fwd(x, conv_w, cache_in, cache_out, g, beta, scale, initial_state,
                                  cu_seqlens, N, T, H, D, dt, o, final_state, stream);
  kda_status st = check_fused_args(x, conv_w, cache_in, cache_out, g, beta, initial_state,
                                   cu_seqlens, N, T, H, D, dt, o, final_state);
  if (st != KDA_OK) return st;
  return fused_two_pass(x, conv_w, cache_in, cache_out, g, 4, nullptr, nullptr, 0.f, false, beta,
                        scale, initial_state, cu_seqlens, N, T, H, D, dt, o, final_state,
                        workspace, workspace_bytes, (cudaStream_t)stream,
                        "kda_prologue_chunk_fwd_ws launch");
}

kda_status kda_prologue_chunk_fwd_windowed_ws(const void *x, const float *conv_w,
                                              const void *cache_in, void *cache_out,
                                              const float *g, const float *beta, float scale,
                                              const float *initial_state,
                                              const int32_t *cu_seqlens, int N, int T, int H,
                                              int D, kda_dtype dt, float *o, float *final_state,
                                              int window_chunks, void *workspace,
                                              size_t workspace_bytes, kda_stream_t stream) {
  kda_status st = check_fused_args(x, conv_w, cache_in, cache_out, g, beta, initial_state,
                                   cu_seqlens, N, T, H, D, dt, o, final_state);
  if (st != KDA_OK) return st;
  if (!chunk_tc_path(T, D, D, 64, dt))
    return fail(KDA_ERR_UNSUPPORTED, "prologue_chunk_fwd_windowed: needs bf16/f16, D == 128 "
                                     "and T > 0 (got dt=%d D=%d T=%d)", (int)dt, D, T);
  KDA_REQUIRE(window_chunks >= 1, "window_chunks=%d must be at least 1", window_chunks);
  KDA_REQUIRE(workspace != nullptr, "prologue_chunk_fwd_windowed: workspace is NULL");
  return fused_two_pass(x, conv_w, cache_in, cache_out, g, 4, nullptr, nullptr, 0.f, false, beta,
                        scale, initial_state, cu_seqlens, N, T, H, D, dt, o, final_state,
                        workspace, workspace_bytes, (cudaStream_t)stream,
                        "kda_prologue_chunk_fwd_windowed_ws launch", window_chunks);
}

kda_status kda_prologue_chunk_fwd_gated_ws(const void *x, const float *conv_w,
                                           const void *cache_in, void *cache_out,
                                           const void *g_raw, const float *A_log,
                                           const float *dt_bias, float lower_bound,
                                           const float *beta, float scale,
                                           const float *initial_state,
                                           const int32_t *cu_seqlens, int N, int T, int H, int D,
                                           kda_dtype dt, float *o, float *final_state,
                                           void *workspace, size_t workspace_bytes,
                                           kda_stream_t stream) {
  kda_status st = check_fused_args(x, conv_w, cache_in, cache_out, g_raw, beta, initial_state,
                                   cu_seqlens, N, T, H, D, dt, o, final_state, esize(dt));
  if (st != KDA_OK) return st;
  st = check_gate_args(A_log, dt_bias, lower_bound, true);
  if (st != KDA_OK) return st;
  KDA_REQUIRE(workspace != nullptr, "prologue_chunk_fwd_gated: workspace is NULL");
  return fused_two_pass(x, conv_w, cache_in, cache_out, g_raw, esize(dt), A_log, dt_bias,
                        lower_bound, true, beta, scale, initial_state, cu_seqlens, N, T, H, D, dt,
                        o, final_state, workspace, workspace_bytes, (cudaStream_t)stream,
                        "kda_prologue_chunk_fwd_gated_ws launch");
}

}  // extern "C"

namespace {

kda_status decode_step(const void *x, const float *conv_w, void *conv_cache, const void *g,
                       size_t g_elem_bytes, const float *A_log, const float *dt_bias,
                       float lower_bound, bool gated, const float *beta, float scale,
                       float *state, int N, int H, int D, kda_dtype dt, float *o,
                       kda_stream_t stream, const char *what) {
  KDA_REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  KDA_REQUIRE(N >= 0 && H >= 1 && D >= 1, "bad sizes N=%d H=%d D=%d", N, H, D);
  if (!supported_d(D)) return fail(KDA_ERR_UNSUPPORTED, "decode: D=%d not in {16,32,64,128}", D);
  if (N == 0) return KDA_OK;
  KDA_REQUIRE_PTR(x, "x");
  KDA_REQUIRE_PTR(conv_w, "conv_w");
  KDA_REQUIRE_PTR(conv_cache, "conv_cache");
  KDA_REQUIRE_PTR(g, "g");
  KDA_REQUIRE_PTR4(beta, "beta");
  KDA_REQUIRE_PTR(state, "state");
  KDA_REQUIRE_PTR(o, "o");
  if (gated && g_elem_bytes == 2)  // 4 pre-activations per lane: 8-byte loads
    KDA_REQUIRE((reinterpret_cast<uintptr_t>(g) & 7u) == 0, "g is not 8-byte aligned");
  const size_t es = esize(dt), C = (size_t)3 * H * D;
  const size_t obytes = (size_t)N * H * D * sizeof(float), sbytes = (size_t)N * H * D * D * 4;
  KDA_REQUIRE(!overlaps(o, obytes, state, sbytes), "o overlaps state");
  KDA_REQUIRE(!overlaps(o, obytes, conv_cache, (size_t)N * 3 * C * es), "o overlaps conv_cache");
  KDA_REQUIRE(!overlaps(o, obytes, x, (size_t)N * C * es), "o overlaps x");
  KDA_REQUIRE(!overlaps(o, obytes, g, (size_t)N * H * D * g_elem_bytes), "o overlaps g");
  KDA_REQUIRE(!overlaps(state, sbytes, conv_cache, (size_t)N * 3 * C * es),
              "state overlaps conv_cache");
  int *status = nullptr;
  kda_status st = device_status_word(&status);
  if (st != KDA_OK) return st;
  cudaError_t e = kda::launch_decode(x, conv_w, conv_cache, g, beta, scale, state, N, H, D, dt, o,
                                     A_log, dt_bias, lower_bound, gated, status,
                                     (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, what);
  return KDA_OK;
}

}  // namespace

extern "C" {

kda_status kda_decode_step(const void *x, const float *conv_w, void *conv_cache, const float *g,
                           const float *beta, float scale, float *state, int N, int H, int D,
                           kda_dtype dt, float *o, kda_stream_t stream) {
  return decode_step(x, conv_w, conv_cache, g, 4, nullptr, nullptr, 0.f, false, beta, scale,
                     state, N, H, D, dt, o, stream, "kda_decode_step launch");
}

kda_status kda_decode_step_gated(const void *x, const float *conv_w, void *conv_cache,
                                 const void *g_raw, const float *A_log, const float *dt_bias,
                                 float lower_bound, const float *beta, float scale, float *state,
                                 int N, int H, int D, kda_dtype dt, float *o,
                                 kda_stream_t stream) {
  KDA_REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  kda_status st = check_gate_args(A_log, dt_bias, lower_bound, false);
  if (st != KDA_OK) return st;
  return decode_step(x, conv_w, conv_cache, g_raw, esize(dt), A_log, dt_bias, lower_bound, true,
                     beta, scale, state, N, H, D, dt, o, stream, "kda_decode_step_gated launch");
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Backward of the two-pass prefill
// ---------------------------------------------------------------------------

extern "C" {

size_t kda_chunk_bwd_workspace_bytes(int N, int T, int H, int Dk, int Dv, int chunk,
                                     kda_dtype dt) {
  if (N < 1 || T < 0 || H < 1 || !chunk_tc_path(T, Dk, Dv, chunk, dt)) return 0;
  return kda::rec::workspace_bytes(N, T, H, 0) +
         2 * (size_t)kda::rec::chunk_capacity(N, T) * H * kda::rec::SEG_BLOCK +
         kda::chunk_bwd_local_scratch_bytes();
}

kda_status kda_chunk_bwd_ws(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float scale, const float *initial_state,
                            const int32_t *cu_seqlens, int N, int T, int H, int Dk, int Dv,
                            int chunk, kda_dtype dt, const float *d_o,
                            const float *d_final_state, float *dq, float *dk, float *dv,
                            float *dg, float *dbeta, float *d_initial_state, void *workspace,
                            size_t workspace_bytes, kda_stream_t stream) {
  KDA_REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  KDA_REQUIRE(N >= 1 && T >= 0 && H >= 1, "bad sizes N=%d T=%d H=%d", N, T, H);
  KDA_REQUIRE(cu_seqlens != nullptr || N == 1, "cu_seqlens is NULL but N=%d", N);
  if (!chunk_tc_path(T, Dk, Dv, chunk, dt))
    return fail(KDA_ERR_UNSUPPORTED, "chunk_bwd: needs bf16/f16, Dk == Dv == 128, chunk 64 and "
                                     "T > 0 (got dt=%d Dk=%d Dv=%d chunk=%d T=%d)",
                (int)dt, Dk, Dv, chunk, T);
  KDA_REQUIRE_PTR(q, "q");
  KDA_REQUIRE_PTR(k, "k");
  KDA_REQUIRE_PTR(v, "v");
  KDA_REQUIRE_PTR(g, "g");
  KDA_REQUIRE_PTR4(beta, "beta");
  KDA_REQUIRE_PTR(d_o, "d_o");
  KDA_REQUIRE_PTR(dq, "dq");
  KDA_REQUIRE_PTR(dk, "dk");
  KDA_REQUIRE_PTR(dv, "dv");
  KDA_REQUIRE_PTR(dg, "dg");
  KDA_REQUIRE_PTR4(dbeta, "dbeta");
  KDA_OPT_PTR(initial_state, "initial_state");
  KDA_OPT_PTR(d_final_state, "d_final_state");
  KDA_OPT_PTR(d_initial_state, "d_initial_state");
  KDA_OPT_PTR4(cu_seqlens, "cu_seqlens");
  KDA_REQUIRE(workspace != nullptr, "chunk_bwd: workspace is NULL");
  KDA_OPT_PTR(workspace, "workspace");
  const size_t need = kda_chunk_bwd_workspace_bytes(N, T, H, Dk, Dv, chunk, dt);
  KDA_REQUIRE(workspace_bytes >= need, "workspace holds %zu bytes, these sizes need %zu",
              workspace_bytes, need);
  {  // outputs must not overlap the inputs, each other or the workspace
    const size_t es = esize(dt), act = (size_t)T * H * 128 * es, f32 = (size_t)T * H * 128 * 4;
    const size_t sbytes = (size_t)N * H * 128 * 128 * 4, bb = (size_t)T * H * 4;
    const void *outs[6] = {dq, dk, dv, dg, dbeta, d_initial_state};
    const size_t osz[6] = {f32, f32, f32, f32, bb, sbytes};
    const void *ins[9] = {q, k, v, g, beta, d_o, initial_state, d_final_state, cu_seqlens};
    const size_t isz[9] = {act, act, act, f32, bb, f32, sbytes, sbytes, (size_t)(N + 1) * 4};
    for (int a = 0; a < 6; ++a) {
      for (int b = 0; b < 9; ++b)
        KDA_REQUIRE(!overlaps(outs[a], osz[a], ins[b], isz[b]), "an output overlaps an input");
      for (int b = a + 1; b < 6; ++b)
        KDA_REQUIRE(!overlaps(outs[a], osz[a], outs[b], osz[b]), "two outputs overlap");
      KDA_REQUIRE(!overlaps(outs[a], osz[a], workspace, need), "an output overlaps the workspace");
    }
    for (int b = 0; b < 9; ++b)
      KDA_REQUIRE(!overlaps(workspace, need, ins[b], isz[b]), "workspace overlaps an input");
  }
  int *status = nullptr;
  kda_status st = device_status_word(&status);
  if (st != KDA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  uint8_t *wsb = static_cast<uint8_t *>(workspace);
  float *ckpt = reinterpret_cast<float *>(wsb + kda::rec::workspace_bytes(N, T, H, 0));
  float *dckpt = ckpt + (size_t)kda::rec::chunk_capacity(N, T) * H * 128 * 128;
  float *scratch = dckpt + (size_t)kda::rec::chunk_capacity(N, T) * H * 128 * 128;
  cudaError_t e = cudaSuccess;
  if (cu_seqlens) e = kda::launch_chunk_index(cu_seqlens, N, T, 0, workspace, status, s);
  if (e == cudaSuccess)
    e = kda::launch_chunk_prep(q, k, v, g, beta, cu_seqlens, N, T, H, dt, workspace, nullptr,
                               nullptr, 0.f, false, status, s);
  if (e == cudaSuccess)
    e = kda::launch_chunk_state(workspace, cu_seqlens, initial_state, scale, N, T, H, 0, nullptr,
                                nullptr, status, s, ckpt);
  if (e == cudaSuccess)
    e = kda::launch_chunk_bwd_state(workspace, cu_seqlens, d_final_state, d_o, scale, N, T, H,
                                    dckpt, d_initial_state, status, s);
  if (e == cudaSuccess)
    e = kda::launch_chunk_bwd_local(q, k, v, g, beta, d_o, scale, cu_seqlens, workspace, ckpt,
                                    dckpt, scratch, N, T, H, dt, dq, dk, dv, dg, dbeta, status, s);
  if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_bwd_ws launch");
  return KDA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Affine chunk maps across ranks (sequence split)
// ---------------------------------------------------------------------------

extern "C" {

size_t kda_chunk_map_workspace_bytes(int N, int T, int H, int Dk, int Dv, int chunk,
                                     kda_dtype dt) {
  return kda_chunk_fwd_segmented_workspace_bytes(N, T, H, Dk, Dv, chunk, dt, 0);
}

kda_status kda_chunk_map_ws(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const int32_t *cu_seqlens, int N, int T, int H,
                            int Dk, int Dv, int chunk, kda_dtype dt, float *M, float *B,
                            void *workspace, size_t workspace_bytes, kda_stream_t stream) {
  KDA_REQUIRE(valid_dtype(dt), "unknown dtype %d", (int)dt);
  KDA_REQUIRE(N >= 1 && T >= 0 && H >= 1, "bad sizes N=%d T=%d H=%d", N, T, H);
  KDA_REQUIRE(cu_seqlens != nullptr || N == 1, "cu_seqlens is NULL but N=%d", N);
  if (!chunk_tc_path(T, Dk, Dv, chunk, dt))
    return fail(KDA_ERR_UNSUPPORTED, "chunk_map: needs bf16/f16, Dk == Dv == 128, chunk 64 and "
                                     "T > 0 (got dt=%d Dk=%d Dv=%d chunk=%d T=%d)",
                (int)dt, Dk, Dv, chunk, T);
  KDA_REQUIRE_PTR(q, "q");
  KDA_REQUIRE_PTR(k, "k");
  KDA_REQUIRE_PTR(v, "v");
  KDA_REQUIRE_PTR(g, "g");
  KDA_REQUIRE_PTR4(beta, "beta");
  KDA_REQUIRE_PTR(M, "M");
  KDA_REQUIRE_PTR(B, "B");
  KDA_OPT_PTR4(cu_seqlens, "cu_seqlens");
  KDA_REQUIRE(workspace != nullptr, "chunk_map: workspace is NULL");
  KDA_OPT_PTR(workspace, "workspace");
  const size_t need = kda_chunk_map_workspace_bytes(N, T, H, Dk, Dv, chunk, dt);
  KDA_REQUIRE(workspace_bytes >= need, "workspace holds %zu bytes, these sizes need %zu",
              workspace_bytes, need);
  {
    const size_t es = esize(dt), act = (size_t)T * H * 128 * es, sbytes = (size_t)N * H * 128 * 128 * 4;
    const void *ins[7] = {q, k, v, g, beta, cu_seqlens, workspace};
    const size_t isz[7] = {act, act, act, (size_t)T * H * 128 * 4, (size_t)T * H * 4,
                           (size_t)(N + 1) * 4, need};
    for (int i = 0; i < 7; ++i) {
      KDA_REQUIRE(!overlaps(M, sbytes, ins[i], isz[i]), "M overlaps an input or the workspace");
      KDA_REQUIRE(!overlaps(B, sbytes, ins[i], isz[i]), "B overlaps an input or the workspace");
    }
    KDA_REQUIRE(!overlaps(M, sbytes, B, sbytes), "M overlaps B");
    for (int i = 0; i < 6; ++i)
      KDA_REQUIRE(!overlaps(workspace, need, ins[i], isz[i]), "workspace overlaps an input");
  }
  int *status = nullptr;
  kda_status st = device_status_word(&status);
  if (st != KDA_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  if (cu_seqlens) e = kda::launch_chunk_index(cu_seqlens, N, T, 0, workspace, status, s);
  if (e == cudaSuccess)
    e = kda::launch_chunk_prep(q, k, v, g, beta, cu_seqlens, N, T, H, dt, workspace, nullptr,
                               nullptr, 0.f, false, status, s);
  if (e == cudaSuccess) e = kda::launch_chunk_map(workspace, cu_seqlens, N, T, H, M, B, status, s);
  if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_map_ws launch");
  return KDA_OK;
}

kda_status kda_state_compose(const float *M, const float *B, const float *E_in, float *E_out,
                             int N, int H, int D, kda_stream_t stream) {
  KDA_REQUIRE(N >= 1 && H >= 1, "bad sizes N=%d H=%d", N, H);
  if (D != 128) return fail(KDA_ERR_UNSUPPORTED, "state_compose: D=%d (needs 128)", D);
  KDA_REQUIRE_PTR(M, "M");
  KDA_REQUIRE_PTR(B, "B");
  KDA_REQUIRE_PTR(E_out, "E_out");
  KDA_OPT_PTR(E_in, "E_in");
  const size_t sbytes = (size_t)N * H * D * D * 4;
  KDA_REQUIRE(!overlaps(E_out, sbytes, M, sbytes) && !overlaps(E_out, sbytes, B, sbytes) &&
                  !overlaps(E_out, sbytes, E_in, sbytes),
              "E_out overlaps an input");
  cudaError_t e = kda::launch_state_compose(M, B, E_in, E_out, N * H, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "kda_state_compose launch");
  return KDA_OK;
}

}  // extern "C"
