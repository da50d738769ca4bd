/*
 * kda.h -- C ABI of libkda, a B200 (sm_100a) implementation of the Kimi Delta
 * Attention (KDA) recurrence hot path: the prologue (short conv, SiLU, L2),
 * the chunkwise-parallel prefill and the batched decode step.
 *
 * Sources (web pages; cited as [Wn section]):
 *   [W1] "Kimi K3的线性注意力：从源码看懂KDA如何更新记忆" (yeyulingfeng.com)
 *   [W3] "Kimi K3 记忆架构总览：KDA、MLA、AttnRes 各管什么" (moonzj.com)
 *   [W4] "KimiK3轻量化复刻实现KDA并行解析，Chunkwise并行与状态压缩机制详解"
 *   [W5] "AI-Workshop 文献分享 #16 — KDA：给长文本建立可更新的记忆"
 *
 * The recurrence, per head with state S in R^{Dk x Dv} ([W1 第三站-第五站]):
 *     S <- diag(exp(g_t)) S;  e <- v_t - S^T k_t;  S <- S + beta_t k_t e^T;
 *     o_t <- scale * S^T q_t.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers to contiguous row-major arrays
 *     owned by the caller.  The library never allocates device memory: its
 *     4-byte status word per device (see kda_get_device_status) is a
 *     file-scope __device__ variable, reserved with the library's device
 *     code and looked up once per device.
 *   - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  A synchronous return reports argument,
 *     support and launch errors only; faults detected inside a kernel
 *     (out-of-range cu_seqlens, a bounded wait that ran out) are recorded in
 *     the device status word.
 *   - Recurrent state layout is [N, H, Dv, Dk] float32: the key index is the
 *     contiguous one (the transpose of the pages' key-first S; [W1 第三站]
 *     allows a transposed storage layout).
 *   - Activations (q, k, v, x, conv cache) have the element type `dt`
 *     (KDA_F32, KDA_BF16 or KDA_F16).  g, beta, the state and every read-out o are
 *     always float32: o is heavy-tailed (its largest entries are many times
 *     its RMS), so rounding it to bf16 alone would exceed the parity bound
 *     max|o - o_ref| <= 2e-2 * RMS(o_ref).
 *   - Every pointer must be 16-byte aligned, except beta and cu_seqlens
 *     (4-byte aligned).  Outputs must not overlap inputs unless an argument
 *     says "in/out".
 *   - On any non-OK return, kda_last_error() gives a message (thread-local).
 *
 * Deliberate departures from the boundary first planned for this library
 *   - Every read-out o is float32 (`float *o`), not an array of the
 *     activation type `dt`.  Measured on the T=4096, H=8 bf16 workload,
 *     max|o| is about 20 RMS(o), so rounding the exact o to bf16 alone gives
 *     max|o - o_ref| / RMS(o_ref) = 0.040, twice the 2e-2 parity bound that
 *     bf16-input workloads must meet; no bf16 read-out can pass it.
 *   - kda_prologue takes an extra `out_dt`: the element type of q, k, v may
 *     differ from that of x (the tensor-core prefill reads fp16 q, k, v,
 *     whose 11-bit significand keeps its operands inside the parity bound,
 *     while the projections arrive as bf16).
 */
#ifndef KDA_H_
#define KDA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KDA_OK = 0,
  KDA_ERR_INVALID_ARG = 1,    /* null/misaligned pointer, bad size, aliasing   */
  KDA_ERR_UNSUPPORTED = 2,    /* valid request outside the compiled domain     */
  KDA_ERR_CUDA = 3,           /* a CUDA runtime call or kernel launch failed   */
  KDA_ERR_DEVICE_TIMEOUT = 4, /* (status word) a bounded device wait ran out   */
  KDA_ERR_DEVICE_BOUNDS = 5,  /* (status word) device-side index check failed  */
  KDA_ERR_DEVICE_RANGE = 6    /* (status word) a value left the range of the
                                 fp16 tensor-core operands (|x| >= 2^15)      */
} kda_status;

typedef enum { KDA_F32 = 0, KDA_BF16 = 1, KDA_F16 = 2 } kda_dtype;

typedef struct CUstream_st *kda_stream_t; /* same type as cudaStream_t */

/*
 * kda_prologue -- short conv + SiLU on the q/k/v projections, then per-head
 * L2 normalisation of q and k.  [W1 第二站]: a causal depthwise conv of
 * width 4 that never reads future tokens, SiLU inside the conv module, and
 * q, k unit-normalised inside the KDA operator; [W4 ShortConv paragraph]:
 * each channel sees the current token and the three before it.
 *
 *   x          [T, 3*H*D] dt   projections; channel p*H*D + h*D + d with
 *                              p = 0 (query), 1 (key), 2 (value)
 *   conv_w     [3*H*D, 4] f32  tap 3 multiplies the current token, tap 0 the
 *                              token three back; no bias
 *   cache_in   [N, 3, 3*H*D] dt or NULL: the three inputs before each
 *                              sequence, oldest first (NULL: zero history)
 *   cache_out  [N, 3, 3*H*D] dt or NULL: receives the last three inputs of
 *                              each sequence; must not overlap cache_in
 *   cu_seqlens [N+1] int32 device, or NULL (then N must be 1): packed
 *                              sequence boundaries; the conv never crosses one
 *   dt         element type of x and of both caches
 *   out_dt     element type of the outputs q, k, v
 *   q, k, v    [T, H, D] out_dt outputs; q, k are y/sqrt(sum y^2 + 1e-6) over
 *                              the head's D channels of y = SiLU(conv)
 * Supported: D in {16, 32, 64, 128}; T >= 0 (T == 0 only writes cache_out).
 */
kda_status kda_prologue(const void *x, const float *conv_w, const void *cache_in,
                        void *cache_out, const int32_t *cu_seqlens, int N, int T,
                        int H, int D, kda_dtype dt, kda_dtype out_dt, void *q, void *k,
                        void *v, kda_stream_t stream);

/*
 * kda_chunk_fwd -- chunkwise-parallel prefill of the recurrence.  [W1 彩蛋]
 * and [W5 §10.3]: tokens are grouped into chunks of `chunk`, the state is
 * carried from chunk to chunk, and the work inside a chunk is matrix algebra
 * (in-chunk cumulative log-decay, a unit-lower-triangular WY solve by
 * forward substitution, the state-dependent chunk update); [W4 Figure 1]:
 * the chunk map of the state is affine.  Results equal the token-by-token
 * recurrence up to rounding.
 *
 *   q, k          [T, H, Dk] dt  q and k already unit-normalised
 *   v             [T, H, Dv] dt
 *   g             [T, H, Dk] f32 log-decay, alpha = exp(g); the bf16 tensor-core
 *                                path requires g >= -5 (the bounded gate of
 *                                [W1 彩蛋]); other values may lose accuracy
 *   beta          [T, H] f32
 *   scale         multiplier on every read o_t ([W1 第五站])
 *   initial_state [N, H, Dv, Dk] f32 or NULL (zero state)
 *   cu_seqlens    [N+1] int32 device or NULL (N must be 1); sequences restart
 *                 from initial_state[n]
 *   o             [T, H, Dv] float32 output
 *   final_state   [N, H, Dv, Dk] f32 or NULL; may alias initial_state
 * Supported: Dk == Dv in {16, 32, 64, 128}, chunk in {16, 32, 64}.  With
 *   dt == KDA_BF16 or KDA_F16, Dk == Dv == 128 and chunk == 64 the call runs
 *   the tcgen05 tensor-core path; every other case runs the exact-fp32
 *   CUDA-core path.
 */
kda_status kda_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                         const float *beta, float scale, const float *initial_state,
                         const int32_t *cu_seqlens, int N, int T, int H, int Dk, int Dv,
                         int chunk, kda_dtype dt, float *o, float *final_state,
                         kda_stream_t stream);

/*
 * kda_chunk_fwd_workspace_bytes -- bytes of scratch kda_chunk_fwd_ws needs for
 * these sizes: one 88.75 KiB record per (chunk, head) plus a 1 KiB-aligned
 * chunk and segment index, sized for the worst case of N sequences in T
 * tokens (ceil(T/64) + N chunks per head), plus, when these sizes split
 * sequences into segments (kda_chunk_fwd_segment_chunks > 0), 192 KiB per
 * (segment, head) for the segment maps.  0 when the arguments do not select
 * the tensor-core path (dt == KDA_F32, Dk or Dv != 128, chunk != 64, T == 0).
 */
size_t kda_chunk_fwd_workspace_bytes(int N, int T, int H, int Dk, int Dv, int chunk,
                                     kda_dtype dt);

/*
 * kda_chunk_fwd_segment_chunks -- the segment length, in 64-token chunks, that
 * the workspace entry points (kda_chunk_fwd_ws, kda_chunk_fwd_gated_ws,
 * kda_chunk_fwd_static and the two-pass prologue entry points) use for these
 * sizes; 0 means every sequence is carried whole by one chain of CTAs.  A
 * batch whose (sequence, head, 32 value channels) chains already fill two
 * CTAs per SM is not split; otherwise sequences are cut into segments of at
 * most this many chunks (at least 4) so that the segment maps fill the GPU.
 * 0 for invalid sizes.
 */
int kda_chunk_fwd_segment_chunks(int N, int T, int H);

/*
 * kda_chunk_fwd_segmented_workspace_bytes -- kda_chunk_fwd_workspace_bytes
 * for an explicit segment length (segment_chunks >= 0; 0: whole sequences).
 * 0 for arguments off the tensor-core path or a negative segment_chunks.
 */
size_t kda_chunk_fwd_segmented_workspace_bytes(int N, int T, int H, int Dk, int Dv, int chunk,
                                               kda_dtype dt, int segment_chunks);

/*
 * kda_chunk_fwd_ws -- kda_chunk_fwd with a caller-owned scratch buffer, which
 * lets the tensor-core path run as two passes.  [W4 Figure 1]: inside a chunk
 * everything except the read of the entry state is independent of the
 * carried state, so the first pass computes it for all (chunk, head) pairs
 * at once (in-chunk log-decay, Gram products, the WY solve of [W5 §10.3]) and
 * the second carries the state through the chunks of each sequence in order,
 * one CTA per (sequence, head, 32 value channels), or per (segment, head, 32
 * value channels) when kda_chunk_fwd_segment_chunks splits the sequences (see
 * kda_chunk_fwd_segmented_ws).  Same arguments and
 * results as kda_chunk_fwd (equal up to rounding order), plus:
 *   workspace        device buffer of >= kda_chunk_fwd_workspace_bytes(...)
 *                    bytes, 16-byte aligned, owned by the caller; its contents
 *                    on entry do not matter and are unspecified on return.  It
 *                    must not overlap any other argument, and calls that may
 *                    run concurrently must not share one.  NULL: the call is
 *                    exactly kda_chunk_fwd.
 *   workspace_bytes  its size; KDA_ERR_INVALID_ARG if too small
 */
kda_status kda_chunk_fwd_ws(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float scale, const float *initial_state,
                            const int32_t *cu_seqlens, int N, int T, int H, int Dk, int Dv,
                            int chunk, kda_dtype dt, float *o, float *final_state,
                            void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_chunk_fwd_segmented_ws -- kda_chunk_fwd_ws with the sequence-parallel
 * state pass at an explicit segment length.  [W4 Figure 1, Figure 3]: the
 * chunk update is an affine map of the entry state, S -> M S + B with
 * M = diag(exp(gamma_last)) - K'^T W and B = K'^T Ut, so maps compose.  Each
 * sequence of nch chunks is cut into G = max(1, ceil(nch / segment_chunks))
 * segments of balanced length; a transition pass computes, for every segment
 * but the last, its map (M from the identity with Ut = 0, B from a zero
 * state; the first segment runs from the initial state) with the same
 * tensor-core chunk update; an fp32 scan composes the entry states; the output
 * pass then runs all segments at once from their entry states.
 * Same arguments and results as kda_chunk_fwd_ws (equal up to rounding), plus:
 *   segment_chunks   >= 0 (KDA_ERR_INVALID_ARG if negative); 0: whole sequences
 *   workspace        device buffer of >= kda_chunk_fwd_segmented_workspace_bytes
 *                    (..., segment_chunks) bytes, 16-byte aligned, caller-owned,
 *                    not NULL; the same overlap and concurrency rules
 * Tensor-core path only (else KDA_ERR_UNSUPPORTED).
 */
kda_status kda_chunk_fwd_segmented_ws(const void *q, const void *k, const void *v,
                                      const float *g, const float *beta, float scale,
                                      const float *initial_state, const int32_t *cu_seqlens,
                                      int N, int T, int H, int Dk, int Dv, int chunk,
                                      kda_dtype dt, float *o, float *final_state,
                                      int segment_chunks, void *workspace,
                                      size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_chunk_fwd_windowed_ws -- kda_chunk_fwd_ws with a workspace that does not
 * grow with T: the two passes run over windows of `window_chunks` consecutive
 * chunk numbers (the chunks of all sequences, in order) one window at a time,
 * so the workspace holds one window's records (88.75 KiB per chunk and head)
 * plus two fp32 carry states per head, through which a sequence that crosses
 * a window boundary hands its state to the next window.  This is the same
 * computation in the same order: every output and final state is bit for bit
 * that of kda_chunk_fwd_segmented_ws with segment_chunks = 0.  The cost is two
 * launches per window (ceil((ceil(T/64) + N) / window_chunks) windows).
 * Source: "KimiK3轻量化复刻实现KDA并行解析，Chunkwise并行与状态压缩机制详解",
 * Figure 1 (the in-chunk work is state-independent, so it can run ahead of the
 * state pass a window at a time).
 *   window_chunks    >= 1, else KDA_ERR_INVALID_ARG
 *   workspace        >= kda_chunk_fwd_windowed_workspace_bytes(...) bytes,
 *                    16-byte aligned, caller-owned, as for kda_chunk_fwd_ws
 * Supported: the tensor-core path only (dt KDA_BF16 or KDA_F16, Dk == Dv ==
 * 128, chunk 64, T > 0), else KDA_ERR_UNSUPPORTED.  Other arguments as in
 * kda_chunk_fwd_ws.
 */
kda_status kda_chunk_fwd_windowed_ws(const void *q, const void *k, const void *v,
                                     const float *g, const float *beta, float scale,
                                     const float *initial_state, const int32_t *cu_seqlens,
                                     int N, int T, int H, int Dk, int Dv, int chunk,
                                     kda_dtype dt, float *o, float *final_state,
                                     int window_chunks, void *workspace, size_t workspace_bytes,
                                     kda_stream_t stream);

/*
 * kda_prologue_chunk_fwd_windowed_ws -- kda_prologue_chunk_fwd_ws (the prologue
 * inside the prep pass) one window of `window_chunks` chunk numbers at a time,
 * as kda_chunk_fwd_windowed_ws: the workspace
 * (kda_chunk_fwd_windowed_workspace_bytes(N, T, H, D, D, 64, dt, window_chunks))
 * does not grow with T.  The conv cache out is written as by the unwindowed call;
 * o and final_state are bit for bit those of kda_prologue_chunk_fwd_ws when it
 * runs whole sequences (kda_chunk_fwd_segment_chunks(N, T, H) == 0).
 * Supported: dt KDA_BF16 or KDA_F16, D == 128, T > 0 (else KDA_ERR_UNSUPPORTED);
 * window_chunks >= 1 and a non-NULL workspace (else KDA_ERR_INVALID_ARG).
 * Other arguments as in kda_prologue_chunk_fwd_ws.
 */
kda_status kda_prologue_chunk_fwd_windowed_ws(const void *x, const float *conv_w,
                                              const void *cache_in, void *cache_out,
                                              const float *g, const float *beta, float scale,
                                              const float *initial_state,
                                              const int32_t *cu_seqlens, int N, int T, int H,
                                              int D, kda_dtype dt, float *o, float *final_state,
                                              int window_chunks, void *workspace,
                                              size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_chunk_fwd_windowed_workspace_bytes -- workspace of kda_chunk_fwd_windowed_ws:
 * a 1 KiB-aligned chunk index, window_chunks * H records of 88.75 KiB and
 * 2 * H carry states of 64 KiB.  0 for arguments off the tensor-core path or
 * window_chunks < 1.
 */
size_t kda_chunk_fwd_windowed_workspace_bytes(int N, int T, int H, int Dk, int Dv, int chunk,
                                              kda_dtype dt, int window_chunks);

/*
 * The *_gated entry points take the gate pre-activations instead of the
 * log-decay and apply the bounded gate inside the kernels ([W1 彩蛋], the
 * gate.py excerpt):
 *     g = lower_bound * sigmoid(exp(A_log[h]) * (g_raw + dt_bias[h, :]))
 * with lower_bound -5 in K3, so the fp32 log-decay is never stored.
 *   g_raw        [T, H, D] (prefill) or [N, H, D] (decode), element type dt
 *   A_log        [H] f32, 4-byte aligned, or NULL (exp(A_log) taken as 1)
 *   dt_bias      [H, D] f32, 16-byte aligned, or NULL (zero)
 *   lower_bound  finite and negative; the prefill entry points need it in
 *                [-5, 0) (their decay-range argument), else KDA_ERR_UNSUPPORTED
 */

/*
 * kda_chunk_fwd_gated_ws -- kda_chunk_fwd_ws with the in-kernel gate: the
 * two-pass tensor-core path only (dt KDA_BF16 or KDA_F16, Dk == Dv == 128,
 * chunk 64, T > 0, a workspace of kda_chunk_fwd_workspace_bytes(...) bytes),
 * else KDA_ERR_UNSUPPORTED / KDA_ERR_INVALID_ARG.  Other arguments as in
 * kda_chunk_fwd_ws.
 */
kda_status kda_chunk_fwd_gated_ws(const void *q, const void *k, const void *v, const void *g_raw,
                                  const float *A_log, const float *dt_bias, float lower_bound,
                                  const float *beta, float scale, const float *initial_state,
                                  const int32_t *cu_seqlens, int N, int T, int H, int Dk, int Dv,
                                  int chunk, kda_dtype dt, float *o, float *final_state,
                                  void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_chunk_fwd_static -- kda_chunk_fwd_ws without a caller workspace: the
 * scratch is a fixed device buffer inside the library, and the call
 * allocates and frees nothing.  The pages have no counterpart of this entry
 * point; it is an engineering variant for callers that must not allocate, and
 * it computes exactly what kda_chunk_fwd_ws computes (same kernels).
 *   Buffer    one file-scope device array of KDA_CHUNK_STATIC_SCRATCH_BYTES
 *             (64 MiB), 256-byte aligned, per device; its address is looked
 *             up once per device (cudaGetSymbolAddress) on first use, so
 *             the first call on a device should come before any stream
 *             capture.  The 64 MiB are reserved when the device module
 *             holding the array loads: at that first call under lazy
 *             module loading (the CUDA 12 default; the array sits in a
 *             module of its own, so the other entry points never load it),
 *             or when the context loads the library's device code under
 *             CUDA_MODULE_LOADING=EAGER.  They stay reserved for the life of
 *             the context.
 *   Sizes     if kda_chunk_fwd_workspace_bytes(...) exceeds the buffer the
 *             call returns KDA_ERR_UNSUPPORTED before launching anything
 *             (e.g. T=4096, H=8 needs 47.3 MB and fits; T=32768, H=96 needs
 *             4.5 GB and does not); if it is 0 the call is kda_chunk_fwd.
 *   Zeroing   nothing in the buffer has to start at zero: every byte a call
 *             reads was written earlier in the same call.
 *   Overlap   all calls on a device share the one buffer.  Calls that may run
 *             at the same time (different streams, or host threads without
 *             ordering between their streams) race on it and give undefined
 *             results; calls issued in order on one stream are safe.
 */
#define KDA_CHUNK_STATIC_SCRATCH_BYTES ((size_t)64 << 20)
kda_status kda_chunk_fwd_static(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, float scale, const float *initial_state,
                                const int32_t *cu_seqlens, int N, int T, int H, int Dk,
                                int Dv, int chunk, kda_dtype dt, float *o, float *final_state,
                                kda_stream_t stream);

/*
 * Affine chunk maps, for splitting one sequence across ranks.  [W4 Figure 1,
 * Figure 3]: the prefill maps its entry state affinely, final = M S0 + B, with
 * M (d_k x d_k) depending on k, g, beta only and B the final state from a
 * zero start.  A sequence cut into stretches held by different ranks is
 * evaluated by computing every stretch's (M, B) where it lives, exchanging
 * them, composing each stretch's entry state E_{r+1} = M_r E_r + B_r from the
 * ones before it, and running kda_chunk_fwd on each stretch from its entry
 * state (the Python package's kda_chunk_fwd_sequence_parallel does this over
 * torch.distributed).  No counterpart in code on the pages.
 *
 * kda_chunk_map_workspace_bytes -- scratch of kda_chunk_map_ws (the two-pass
 * records and chunk index); 0 off the tensor-core shapes.
 */
size_t kda_chunk_map_workspace_bytes(int N, int T, int H, int Dk, int Dv, int chunk,
                                     kda_dtype dt);

/*
 * kda_chunk_map_ws -- the affine map of each of the N sequences (cu_seqlens as
 * in kda_chunk_fwd; tensor-core shapes only, else KDA_ERR_UNSUPPORTED):
 *   M  [N, H, Dk, Dk] f32 output, 16-byte aligned; element (row t, column k) of
 *      the map at M[n][h][k][t] (stored like a state, column-major)
 *   B  [N, H, Dv, Dk] f32 output: the final state from a zero initial state
 *   workspace >= kda_chunk_map_workspace_bytes(...) bytes, caller-owned
 * Outputs must not overlap the inputs, each other or the workspace.  M is
 * computed by the tensor-core state pass from the identity with the value
 * term removed (one CTA per 32 of its columns), B from a zero state; the
 * rounding is that of kda_chunk_fwd_ws.
 */
kda_status kda_chunk_map_ws(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const int32_t *cu_seqlens, int N, int T, int H,
                            int Dk, int Dv, int chunk, kda_dtype dt, float *M, float *B,
                            void *workspace, size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_state_compose -- E_out = M E_in + B for N sequences x H heads, in fp32
 * (layouts as in kda_chunk_map_ws; E_in and E_out like a state [N, H, D, D]).
 * E_in NULL means zero (E_out = B).  D must be 128.  E_out must not overlap
 * M, B or E_in.
 */
kda_status kda_state_compose(const float *M, const float *B, const float *E_in, float *E_out,
                             int N, int H, int D, kda_stream_t stream);

/*
 * Backward of the chunkwise prefill.  The pages mention training ([W1 彩蛋])
 * but print no backward; these are the gradients of the loss
 *     L = sum(d_o * o) + sum(d_final_state * final_state)
 * with o and final_state those of kda_chunk_fwd on the same inputs, i.e. the
 * chain rule through the recurrence of [W1 第三站 - 第五站].  The adjoint of
 * the state is carried backwards through the chunks by the transpose of the
 * forward's affine chunk map [W4 Figure 1]; inside a chunk the gradients come
 * from the chunk algebra, evaluated in fp32 on 16-token blocks.
 *
 * kda_chunk_bwd_workspace_bytes -- scratch bytes of kda_chunk_bwd_ws: the
 * forward's records and chunk index (kda_chunk_fwd_segmented_workspace_bytes
 * with segment length 0) plus two fp32 128 x 128 blocks per (chunk, head)
 * (the entry state and the adjoint of the exit state of every chunk).  0 off
 * the tensor-core path (dt == KDA_F32, Dk or Dv != 128, chunk != 64, T == 0).
 */
size_t kda_chunk_bwd_workspace_bytes(int N, int T, int H, int Dk, int Dv, int chunk,
                                     kda_dtype dt);

/*
 * kda_chunk_bwd_ws -- gradients of kda_chunk_fwd.  Inputs as in kda_chunk_fwd
 * (q, k, v, g, beta, scale, initial_state, cu_seqlens, N, T, H, Dk, Dv, chunk,
 * dt; the tensor-core shapes only: dt KDA_BF16 or KDA_F16, Dk == Dv == 128,
 * chunk 64, T > 0, else KDA_ERR_UNSUPPORTED), plus:
 *   d_o              [T, H, Dv] f32, 16-byte aligned: dL/do
 *   d_final_state    [N, H, Dv, Dk] f32 or NULL (zero): dL/dfinal_state
 *   dq, dk, dg       [T, H, Dk] f32 outputs (dk, dg w.r.t. the k and g given)
 *   dv               [T, H, Dv] f32 output
 *   dbeta            [T, H] f32 output
 *   d_initial_state  [N, H, Dv, Dk] f32 output or NULL (not written)
 *   workspace        >= kda_chunk_bwd_workspace_bytes(...) bytes, 16-byte
 *                    aligned, caller-owned, not NULL; contents on entry do not
 *                    matter and are unspecified on return
 * The forward is recomputed inside the call (o is not needed).  Rows of tokens
 * outside every sequence are not written.  Outputs must not overlap the
 * inputs, each other or the workspace (KDA_ERR_INVALID_ARG).  g >= -5 is
 * required, as on the forward's tensor-core path; a 16-token block whose
 * log-decay falls below -87 is reported as KDA_ERR_DEVICE_RANGE.  Asynchronous
 * on `stream`; calls that may run concurrently must not share a workspace.
 */
kda_status kda_chunk_bwd_ws(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float scale, const float *initial_state,
                            const int32_t *cu_seqlens, int N, int T, int H, int Dk, int Dv,
                            int chunk, kda_dtype dt, const float *d_o,
                            const float *d_final_state, float *dq, float *dk, float *dv,
                            float *dg, float *dbeta, float *d_initial_state, void *workspace,
                            size_t workspace_bytes, kda_stream_t stream);

/*
 * kda_prologue_chunk_fwd -- the prologue fused into the chunkwise prefill: the
 * same result as kda_prologue followed by kda_chunk_fwd (chunk 64), with q, k
 * and v never written to memory.  Each chunk's projections are convolved
 * (causal width 4 with the carried three-row history), passed through SiLU
 * and L2-normalised in fp32 on chip ([W1 第二站], [W4 ShortConv paragraph]),
 * then used by the chunk update of kda_chunk_fwd ([W1 彩蛋]).
 *
 *   x             [T, 3*H*D] dt (KDA_BF16 or KDA_F16) projections, layout as in
 *                 kda_prologue
 *   conv_w        [3*H*D, 4] f32;  cache_in / cache_out as in kda_prologue
 *   g, beta, scale, initial_state, cu_seqlens, o, final_state as in
 *                 kda_chunk_fwd
 * Supported: D == 128, dt in {KDA_BF16, KDA_F16}; T >= 1.
 */
kda_status kda_prologue_chunk_fwd(const void *x, const float *conv_w, const void *cache_in,
                                  void *cache_out, const float *g, const float *beta,
                                  float scale, const float *initial_state,
                                  const int32_t *cu_seqlens, int N, int T, int H, int D,
                                  kda_dtype dt, float *o, float *final_state,
                                  kda_stream_t stream);

/*
 * kda_prologue_chunk_fwd_ws -- kda_prologue_chunk_fwd with a caller-owned
 * scratch buffer, run as two passes like kda_chunk_fwd_ws with the prologue
 * inside the parallel pass: each (chunk, head) item convolves its own 64 rows
 * ([W1 第二站], [W4 ShortConv paragraph]), taking the three raw rows before the
 * chunk, or cache_in at a sequence start, as the conv history; the state pass
 * then carries the state through the chunks ([W4 Figure 1]).  Same arguments
 * and results as kda_prologue_chunk_fwd (equal up to rounding order), plus
 * workspace / workspace_bytes exactly as in kda_chunk_fwd_ws, sized by
 * kda_chunk_fwd_workspace_bytes(N, T, H, D, D, 64, dt).  NULL workspace: the
 * call is kda_prologue_chunk_fwd.
 */
kda_status kda_prologue_chunk_fwd_ws(const void *x, const float *conv_w, const void *cache_in,
                                     void *cache_out, const float *g, const float *beta,
                                     float scale, const float *initial_state,
                                     const int32_t *cu_seqlens, int N, int T, int H, int D,
                                     kda_dtype dt, float *o, float *final_state,
                                     void *workspace, size_t workspace_bytes,
                                     kda_stream_t stream);

/*
 * kda_prologue_chunk_fwd_gated_ws -- kda_prologue_chunk_fwd_ws with the
 * in-kernel gate (see above; a workspace is required).
 */
kda_status kda_prologue_chunk_fwd_gated_ws(const void *x, const float *conv_w,
                                           const void *cache_in, void *cache_out,
                                           const void *g_raw, const float *A_log,
                                           const float *dt_bias, float lower_bound,
                                           const float *beta, float scale,
                                           const float *initial_state,
                                           const int32_t *cu_seqlens, int N, int T, int H, int D,
                                           kda_dtype dt, float *o, float *final_state,
                                           void *workspace, size_t workspace_bytes,
                                           kda_stream_t stream);

/*
 * kda_decode_step -- one new token for each of N independent sequences: the
 * prologue on that token with the conv cache as history, then one step of
 * the recurrence on the state in place (the recurrent mode used for
 * generation, [W1 彩蛋]; one fixed-size state update per token, [W1 回头看看]).
 *
 *   x          [N, 3*H*D] dt   the new token's projections (layout as above)
 *   conv_w     [3*H*D, 4] f32
 *   conv_cache [N, 3, 3*H*D] dt in/out: oldest first; after the call it holds
 *                              the last three inputs including x
 *   g          [N, H, D] f32;  beta [N, H] f32
 *   state      [N, H, Dv, Dk] f32 in/out
 *   o          [N, H, D] float32 output
 * Supported: D in {16, 32, 64, 128} (Dk == Dv == D).
 */
kda_status kda_decode_step(const void *x, const float *conv_w, void *conv_cache,
                           const float *g, const float *beta, float scale, float *state,
                           int N, int H, int D, kda_dtype dt, float *o,
                           kda_stream_t stream);

/*
 * kda_decode_step_gated -- kda_decode_step with the in-kernel gate: g_raw
 * [N, H, D] of type dt (16-byte aligned) replaces g; any finite negative
 * lower_bound.
 */
kda_status kda_decode_step_gated(const void *x, const float *conv_w, void *conv_cache,
                                 const void *g_raw, const float *A_log, const float *dt_bias,
                                 float lower_bound, const float *beta, float scale, float *state,
                                 int N, int H, int D, kda_dtype dt, float *o,
                                 kda_stream_t stream);

/*
 * kda_output_epilogue -- the output path after the read ([W1 第六站]): per-head
 * RMSNorm of the read-out, then the per-channel output gate:
 *     out[t, h, :] = o[t, h, :] / sqrt(mean_d o^2 + eps) * weight * sigmoid(gate[t, h, :])
 * The page's formula is lost in the extraction; the sigmoid gate (a
 * per-channel proportion) and the caller's eps are readings.  The gate
 * pre-activations come from the output-gate projection of x_t, which is not
 * part of this library.
 *   o       [T, H, D] f32 (a read-out of kda_chunk_fwd & co.)
 *   gate    [T, H, D] dt;  weight [D] f32 (shared by the heads);  eps >= 0
 *   out     [T, H, D] dt, must not overlap o, gate or weight
 * Supported: D in {16, 32, 64, 128}.
 */
kda_status kda_output_epilogue(const float *o, const void *gate, const float *weight, float eps,
                               int T, int H, int D, kda_dtype dt, void *out,
                               kda_stream_t stream);

/*
 * kda_get_device_status -- read and clear the current device's status word
 * (KDA_OK if no kernel recorded a fault).  Synchronises the device.
 */
kda_status kda_get_device_status(int *code);

/*
 * kda_selftest_wait_timeout -- exercise the failure path of the bounded device
 * waits.  The pages have no counterpart: this belongs to the library's failure
 * detection.  One CTA waits on an mbarrier that nothing ever arrives at,
 * gives up after about limit_us microseconds (the tensor-core kernels use
 * the same wait with a 2 s limit), records KDA_ERR_DEVICE_TIMEOUT in the
 * device status word and returns: no trap, no fault, so the context stays
 * usable and the next kda_get_device_status returns the code.
 *   limit_us  in [1, 2000000]; otherwise KDA_ERR_INVALID_ARG
 * Asynchronous on `stream`, like every entry point.
 */
kda_status kda_selftest_wait_timeout(unsigned limit_us, kda_stream_t stream);

/*
 * kda_debug_build -- 1 for the bounds-checked build of this library
 * (libkda_debug.so, compiled with KDA_DEBUG), 0 for the release build.  In the
 * debug build every kernel checks the indices it derives from the call's data
 * and arithmetic (sequence, token, chunk, record, segment, state and conv-cache
 * indices) against their extents before the access that uses them; an index
 * out of range records KDA_ERR_DEVICE_BOUNDS in the status word and the access
 * (or the kernel's whole item, where the index is the same for the CTA) is
 * skipped instead of made.  Results of valid calls are the same in both builds.
 */
int kda_debug_build(void);

/*
 * kda_selftest_bounds -- exercise the debug build's index check.  One thread
 * writes slot `index` of a four-slot device probe array through the check the
 * kernels use: in the debug build an index outside [0, 4) records
 * KDA_ERR_DEVICE_BOUNDS and skips the write.  KDA_ERR_UNSUPPORTED in the
 * release build, where the check is compiled out (nothing is launched).
 * Asynchronous on `stream`; read the outcome with kda_get_device_status.
 */
kda_status kda_selftest_bounds(int index, kda_stream_t stream);

/* Message for the last non-OK return on the calling thread (never NULL). */
const char *kda_last_error(void);

/* Library version string. */
const char *kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
