// Per-(chunk, head) record of the two-pass tensor-core prefill.
//
// The prep pass computes, for every chunk of 64 tokens and every head, the
// state-independent part of the chunk update (in-chunk log-decay, the Gram
// products, the WY solve) and stores it as one record; the state pass then
// walks the chunks of each (sequence, head) in order and applies them to the
// state.  This is the chunked form of "KimiK3轻量化复刻实现KDA并行解析，Chunkwise
// 并行与状态压缩机制详解" (Figure 1: within a chunk everything except the
// state read is independent of the carried state, so it can be computed for
// all chunks at once) and of the chunked execution in "Kimi K3的线性注意力：从
// 源码看懂KDA如何更新记忆" (彩蛋).
//
// With G_r = exp(gamma_r) (gamma the inclusive in-chunk cumsum of g), entry
// state S (key-first, d_k x d_v) and T = (I + A)^{-1}:
//   U   = Ut - W S                        Ut = T beta V,  W = T beta (K G)
//   O   = (Q G) S + P U                   P  = lower part of (Q G)(K / G)^T
//   S' = diag(G_last) S + K'^T U          K' = K G_last / G
// The record keeps the operand tiles in the exact 128-byte-swizzled layout
// the state pass's MMAs read (see kda_tcgen05.cuh), so they move with plain
// bulk copies:
//   A1  [W ; Q G]     fp16, K-major, 128 rows (tokens of W, then of Q G) x 128
//   KP  K'            fp16, MN-major (64 token rows x 128 key channels)
//   P   strict P      fp16, K-major 64 x 64 (rows 64..127 of a 128-row tile;
//                     its diagonal <q_r, k_r> is kept apart in fp32, PD)
//   UT  Ut            fp32 [64 tokens][128 value channels], with the fp32
//                     remainder beta v - f16(beta v) already added
//   GL  exp(gamma_63) fp32 [128]
//   PD  <q_r, k_r>    fp32 [64]
// The workspace is [cprefix: int32 [N + 1], sprefix: int32 [N + 1], padded to
// 1 KB][records][segment maps], record (ci, h) at index ci * H + h, where ci
// numbers the chunks of all sequences in order (cprefix[n] = first chunk of
// sequence n).
//
// Sequence-parallel state pass ("KimiK3轻量化复刻实现KDA并行解析，Chunkwise并行与
// 状态压缩机制详解", Figure 1 and Figure 3: the chunk map S -> M S + B is affine,
// so maps compose).  With a segment length of L chunks, sequence n is cut into
// G_n = max(1, ceil(nch_n / L)) segments of balanced length; sprefix[n] numbers
// the first segment of sequence n.  For every segment s that is not the last
// of its sequence the segment area holds, per head, three fp32 128 x 128
// blocks, each stored like a state (column-major: element (row r, column j)
// at j * 128 + r):
//   M  the segment's transition, end state = M * entry state + B (unused for
//      the first segment of a sequence)
//   B  the end state from a zero entry state
//   E  the entry state of segment s (for the first segment of a split
//      sequence, a copy of the caller's initial state)
// With L = 0 every sequence is one segment and there is no segment area.
//
// Windowed form: the passes run over windows of `window` consecutive chunk numbers,
// one window at a time, so the workspace holds the records of one window; a sequence
// that crosses a window boundary hands its fp32 state over through one of two carry
// blocks per head (alternating by window), placed after the records.
#pragma once

#include <stddef.h>
#include <stdint.h>

namespace kda {
namespace rec {

constexpr uint32_t A1 = 0;
constexpr uint32_t KP = 32768;
constexpr uint32_t P = 49152;
constexpr uint32_t UT = 57344;
constexpr uint32_t GL = 90112;
constexpr uint32_t PD = 90624;
constexpr uint32_t BYTES = 90880;
static_assert(BYTES % 16 == 0, "records keep 16-byte alignment");
static_assert(KP + 16384 == P, "K' and P are one contiguous copy");

// Upper bound on the number of chunks over all sequences of a batch of N
// sequences and T tokens: sum ceil(len_n / 64) <= ceil(T / 64) + N.
__host__ __device__ inline long long chunk_capacity(int N, int T) {
  return (long long)(T + 63) / 64 + N;
}

__host__ __device__ inline size_t header_bytes(int N) {
  return ((size_t)(N + 1) * 8 + 1023) & ~(size_t)1023;
}

// Bound on sum_n ceil(len_n / 64) for lengths summing to at most T:
// sum floor((len_n + 63) / 64) <= floor((T + 63 N) / 64).
__host__ __device__ inline long long chunk_sum_bound(int N, int T) {
  return ((long long)T + 63LL * N) / 64;
}

// Bound on the number of segments: sum_n max(1, ceil(nch_n / L)) <= N + floor(sum nch_n / L).
__host__ __device__ inline long long segment_capacity(int N, int T, int L) {
  return L > 0 ? N + chunk_sum_bound(N, T) / L : N;
}

constexpr int kStateSlots = 444;   // resident state-pass CTAs: 148 SMs x 3

// Model of the state pass's time (microseconds) for `ctas` CTAs that each walk
// L chunks: waves of at most kStateSlots CTAs; a chunk step takes 2.9 us with
// up to one CTA per SM, rising to 4.1 us at 2.5 CTAs per SM (the CTAs of an SM
// share its tensor and memory pipes).  Fitted to B200 measurements of the
// state kernel.
inline double state_pass_us(long long ctas, long long L) {
  if (ctas <= 0 || L <= 0) return 0.0;
  const long long waves = (ctas + kStateSlots - 1) / kStateSlots;
  const double occ = (double)((ctas + waves - 1) / waves) / 148.0;
  double f = (occ - 1.0) / 1.5;
  f = f < 0.0 ? 0.0 : f > 1.0 ? 1.0 : f;
  return (double)waves * (double)L * (2.9 + 1.2 * f);
}

// Segment length of the state pass for a batch (0: one segment per sequence).
// A batch whose (sequence, head, value slice) CTAs already fill two per SM
// keeps whole sequences.  Otherwise the search assumes the worst chain, one
// sequence holding all chunks: whole
// sequences cost one chain of them; G >= 3 segments cost the transition pass
// (8 CTAs per (segment, head) but 4 for the first segment), an entry-state
// scan of G - 2 steps (2.6 us each) and the output pass, plus two launches.
// The cheapest G wins if it saves at least 10%.
inline int segment_chunks(int N, int T, int H) {
  if (N < 1 || T < 1 || H < 1 || (long long)N * H * 4 >= 2 * 148) return 0;
  const long long cb = chunk_sum_bound(N, T);
  const double whole = state_pass_us((long long)N * H * 4, cb);
  double best = 0.9 * whole;
  int bestL = 0;
  for (long long G = 3; G <= cb && G <= 256; ++G) {
    const long long L = (cb + G - 1) / G, Gs = (cb + L - 1) / L;
    if (Gs < 3) continue;
    const double cost = state_pass_us(((Gs - 1) * 8 - 4) * H, L) +
                        state_pass_us((Gs + N - 1) * 4 * H, L) + 2.6 * (double)(Gs - 2) + 8.0;
    if (cost < best) {
      best = cost;
      bestL = (int)L;
    }
  }
  return bestL;
}

constexpr size_t SEG_BLOCK = 128 * 128 * sizeof(float);

__host__ __device__ inline size_t segment_area_offset(int N, int T, int H) {
  return header_bytes(N) + (size_t)chunk_capacity(N, T) * H * BYTES;
}

__host__ __device__ inline size_t workspace_bytes(int N, int T, int H, int L) {
  return segment_area_offset(N, T, H) +
         (L > 0 ? (size_t)segment_capacity(N, T, L) * H * 3 * SEG_BLOCK : 0);
}

// Windowed two-pass prefill (kda_chunk_fwd_windowed_ws): the header, records for
// `window` chunks of every head, then two carry states per head ([H][128][128] fp32
// each) that hand the state of a sequence over a window boundary.
__host__ __device__ inline size_t windowed_carry_offset(int N, int H, int window) {
  return header_bytes(N) + (size_t)window * H * BYTES;
}
__host__ __device__ inline size_t windowed_workspace_bytes(int N, int H, int window) {
  return windowed_carry_offset(N, H, window) + 2 * (size_t)H * SEG_BLOCK;
}

}  // namespace rec
}  // namespace kda
