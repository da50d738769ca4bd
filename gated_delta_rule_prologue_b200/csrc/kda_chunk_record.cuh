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
// The workspace is [cprefix: int32 [N + 1], padded to 1 KB][records], record
// (ci, h) at index ci * H + h, where ci numbers the chunks of all sequences
// in order (cprefix[n] = first chunk of sequence n).
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
  return ((size_t)(N + 1) * 4 + 1023) & ~(size_t)1023;
}

__host__ __device__ inline size_t workspace_bytes(int N, int T, int H) {
  return header_bytes(N) + (size_t)chunk_capacity(N, T) * H * BYTES;
}

}  // namespace rec
}  // namespace kda
