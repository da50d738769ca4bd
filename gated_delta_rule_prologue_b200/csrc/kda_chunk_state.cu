// State pass of the two-pass tensor-core prefill, and the chunk index of a
// packed batch.
//
// Sources: "KimiK3轻量化复刻实现KDA并行解析，Chunkwise并行与状态压缩机制详解",
// Figure 1 (the state is carried chunk to chunk through an affine map built
// from per-chunk quantities); "AI-Workshop 文献分享 #16 — KDA：给长文本建立可更新的
// 记忆", §10.3 (the chunk update: read the entry state, correct with the
// in-chunk WY factors, decay and write).  Record contents and the algebra are
// in kda_chunk_record.cuh.
//
// One CTA (128 threads) per (sequence, head, slice of 32 value channels): the
// value columns of the state are independent of each other (W, A and the
// decay do not involve v), so the four slices of a head run side by side and
// a 96-head layer fills 384 CTAs.  Per chunk:
//   D1 = [W ; Q G] S_slice            (M = 128: rows 0..63 give W S, 64..127 Q G S)
//   U  = Ut - (W S)                   (fp32, warps 0-1; fp16 copy as MMA operand)
//   D1 += [* ; P] U                   (rows 64..127 += P U; rows 0..63 are dead)
//   D2 = K'^T U                       (M = 128 key channels)
//   o  = scale (D1[64 + r] + <q_r, k_r> U_r)     (warps 2-3, fp32)
//   S  = diag(G_last) S + D2          (fp32 registers; thread = key channel)
// Operand roundings are those of the one-pass kernel: fp16 S, W, Q G, U, P,
// K' with fp32 accumulation and fp32 diagonal terms.
//
// Sequence-parallel form (segment length L > 0, layout in kda_chunk_record.cuh):
// a chunk maps S to M_c S + B_c with M_c = diag(G_last) - K'^T W and
// B_c = K'^T Ut, so the same kernel run over a segment from the identity with
// Ut = 0 yields the segment's transition M (value slices of the identity are
// its columns), and run from a zero state yields B.  The transition pass
// (kRole = kTransition, 8 CTAs per (segment, head): 4 column slices of M, 4
// value slices of B) writes them; state_scan_kernel composes the entry states
// E_{g+1} = M_g E_g + B_g in fp32; the output pass then runs every segment
// from its entry state at once.  The first segment of a sequence runs from
// the caller's initial state in the transition pass, so its B is E_1.
#include <cuda_fp16.h>

#include <algorithm>

#include "kda_chunk_record.cuh"
#include "kda_common.cuh"
#include "kda_tcgen05.cuh"

namespace kda {
namespace {
using namespace tc;

constexpr int kBT = 128;      // threads per CTA
constexpr int kSlices = 4;    // value-channel slices per head
constexpr uint32_t SB_A1 = 0;            // [W ; Q G] (K-major 128 x 128)          32 KB
constexpr uint32_t SB_KP = 32768;        // K' (MN-major), then P: one copy       24 KB
constexpr uint32_t SB_P = 49152;
constexpr uint32_t SB_A2 = SB_P - 8192;  // A operand [* ; P]: rows 0..63 overlay the tail of
                                         // K' (finite fp16 values whose products land in
                                         // accumulator rows that are never read again)
constexpr uint32_t SB_S = 57344;         // S slice operand (value-contiguous, 128 key rows x 64 B,
                                         // 64-byte swizzle) 8 KB; between the two MMA groups:
                                         // <q_r, k_r> U exchange [32][64] f32
constexpr uint32_t SB_U = 65536;         // U operand (value-contiguous, 64 token rows x 64 B) 4 KB
constexpr uint32_t SB_BAR = 69632;       // four mbarriers, TMEM slot
constexpr uint32_t SB_ALLOC = SB_BAR + 64 + 1024;
// D1 is one accumulator over the 128 key channels; D2 = K'^T U.
constexpr uint32_t TB_D1 = 0, TB_D2 = 64, TB_COLS = 128;
static_assert(SB_KP + 24576 == SB_S, "K' and P are adjacent");

enum { kOutputs = 0, kTransition = 1, kMap = 2 };

// Segment s (or sequence s when L == 0) of the batch: its sequence n, its
// index g among the G segments of n, and its chunk range [c_lo, c_hi) within n.
struct Segment {
  int n, g, G, c_lo, c_hi;
};

__device__ __forceinline__ bool segment_of(const int32_t *cprefix, const int32_t *sprefix,
                                           int N, int L, int s, int nch_whole, Segment &sg) {
  if (L == 0) {
    sg.n = s;
    sg.g = 0;
    sg.G = 1;
    sg.c_lo = 0;
    sg.c_hi = nch_whole;
    return true;
  }
  if (s >= sprefix[N]) return false;
  int lo = 0, hi = N - 1;  // last n with sprefix[n] <= s
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sprefix[mid] <= s) lo = mid;
    else hi = mid - 1;
  }
  const int nch = cprefix[lo + 1] - cprefix[lo];
  sg.n = lo;
  sg.g = s - sprefix[lo];
  sg.G = sprefix[lo + 1] - sprefix[lo];
  sg.c_lo = (int)((long long)sg.g * nch / sg.G);
  sg.c_hi = (int)((long long)(sg.g + 1) * nch / sg.G);
  return true;
}

template <int kRole>
__global__ void __launch_bounds__(kBT, 3)
chunk_state_kernel(const uint8_t *__restrict__ ws, const int32_t *__restrict__ cu,
                   const float *s0, float scale, int N, int T, int H, int L, float *__restrict__ o,
                   float *sN, float *ckpt, float *map_m, float *map_b, int *status,
                   ChunkWindow win) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5;
  constexpr int kParts = kRole == kOutputs ? 1 : 2;
  const int sub = blockIdx.x % (kSlices * kParts);
  const int slice = sub & 3, part = sub >> 2;  // part (transition pass): 0 = M, 1 = B
  const int item = blockIdx.x / (kSlices * kParts), h = item % H, s = item / H;
  const int32_t *cprefix = reinterpret_cast<const int32_t *>(ws);
  const int32_t *sprefix = cprefix + (N + 1);
  const uint8_t *recs = ws + rec::header_bytes(N);
  float *segbuf = reinterpret_cast<float *>(const_cast<uint8_t *>(ws) +
                                            rec::segment_area_offset(N, T, H));
  uint64_t *bar_a1 = reinterpret_cast<uint64_t *>(sm + SB_BAR);
  uint64_t *bar_kp = bar_a1 + 1, *bar_mma = bar_a1 + 2, *bar_m2 = bar_a1 + 3;
  uint32_t *slot = reinterpret_cast<uint32_t *>(sm + SB_BAR + 32);
  float *exch = reinterpret_cast<float *>(sm + SB_S);

  Segment sg;
  {
    const int n0 = L == 0 ? s : 0;
    int bos0, eos0;
    seq_bounds(cu, n0, T, status, bos0, eos0);
    if (!segment_of(cprefix, sprefix, N, L, s, (eos0 - bos0 + 63) / 64, sg)) return;
  }
  const int n = sg.n;
  int bos, eos;
  seq_bounds(cu, n, T, status, bos, eos);
  int cbase = 0;
  int c_lo = sg.c_lo, c_hi = sg.c_hi;
  if (cu || L > 0) {  // zero chunks for every sequence when the index pass rejected cu
    cbase = cprefix[n];
    if (L == 0) c_hi = cprefix[n + 1] - cbase;
  }
  // A window of chunk numbers [win.lo, win.hi) (whole sequences only): this chain runs the
  // sequence's chunks inside it, entering from the carry if the sequence began in an
  // earlier window and leaving its state in the carry if it goes on past this one.  An
  // empty sequence belongs to the window holding its chunk position.
  bool from_carry = false, to_carry = false;
  if (kRole == kOutputs && L == 0) {
    const int nch = c_hi;
    const int lo = max(0, win.lo - cbase);
    const int hi = (int)min((long long)nch, (long long)win.hi - cbase);
    if (nch > 0 ? lo >= hi : !(win.lo <= cbase && cbase < win.hi)) return;
    if (nch > 0) {
      from_carry = lo > 0;
      to_carry = hi < nch;
      c_lo = lo;
      c_hi = hi;
    }
  }
  {  // debug builds: the chain's sequence, chunks and segment slots lie inside the workspace
    const long long cap = min(rec::chunk_capacity(N, T), (long long)win.hi - win.lo);
    if (!in_range(status, n, N) ||
        (c_hi > c_lo && !(in_range(status, cbase + c_lo - win.lo, cap) &&
                          in_range(status, cbase + c_hi - 1 - win.lo, cap))) ||
        (L > 0 && !in_range(status, s, rec::segment_capacity(N, T, L))))
      return;
  }
  // Where the state comes from and goes to.  Slot (s, h, kind) of the segment area.
  auto seg_slot = [&](int seg, int kind) -> float * {
    return segbuf + (((size_t)seg * H + h) * 3 + kind) * (128 * 128);
  };
  const size_t head_off = ((size_t)n * H + h) * 128 * 128;
  const float *s_in = nullptr;
  float *s_out = nullptr, *s_copy = nullptr;
  bool identity = false, use_ut = true;
  if (kRole == kMap) {  // every sequence is one segment: its whole map, M and B
    if (part == 0) {
      identity = true;
      use_ut = false;
      s_out = map_m + head_off;
    } else {
      s_out = map_b + head_off;
    }
  } else if (kRole == kTransition) {
    if (sg.g == sg.G - 1) return;           // the last segment needs no map
    if (sg.g == 0 && part == 0) return;     // the first runs from the initial state
    if (part == 0) {
      identity = true;
      use_ut = false;
      s_out = seg_slot(s, 0);
    } else if (sg.g == 0) {
      s_in = s0 ? s0 + head_off : nullptr;
      s_copy = seg_slot(s, 2);
      s_out = seg_slot(s + 1, 2);
    } else {
      s_out = seg_slot(s, 1);
    }
  } else {
    // A split sequence reads its initial state from the copy the transition
    // pass took (E of its first segment): the final state may be written over
    // the initial state by the last segment while the first is still to run.
    s_in = sg.G > 1 ? seg_slot(s, 2) : s0 ? s0 + head_off : nullptr;
    s_out = sg.g == sg.G - 1 && sN ? sN + head_off : nullptr;
    if (from_carry) s_in = win.carry_in + (size_t)h * 128 * 128;
    if (to_carry) s_out = win.carry_out + (size_t)h * 128 * 128;
  }

  if (warp == 0) tmem_alloc(slot, TB_COLS);
  if (tid == 0) {
    mbar_init(bar_a1, 1);
    mbar_init(bar_kp, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_m2, 1);
    fence_mbar_init();
  }
  // S[i] = S[key tid][value 32 slice + i]; the state is stored value-major [dv][dk].
  const int t = tid;
  const size_t sbase = (size_t)slice * 32 * 128 + t;
  float S[32];
#pragma unroll
  for (int i = 0; i < 32; ++i)
    S[i] = identity ? (t == 32 * slice + i ? 1.f : 0.f) : s_in ? s_in[sbase + (size_t)i * 128] : 0.f;
  if (s_copy) {
#pragma unroll
    for (int i = 0; i < 32; ++i) s_copy[sbase + (size_t)i * 128] = S[i];
  }

  auto write_s_operand = [&]() {  // S slice as the B operand: key row t, 32 values
    float amax = 0.f;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      float f[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        f[e] = S[8 * x + e];
        amax = fmaxf(amax, fabsf(f[e]));
      }
      st_shared_16(sm + SB_S, mn32_sw64_off(t, x), pack8_f16(f));
    }
    if (!(amax < 32768.f)) report(status, KDA_ERR_DEVICE_RANGE);
  };
  write_s_operand();
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t lane_addr = static_cast<uint32_t>(32 * warp) << 16;

  auto rec_of = [&](int c) -> const uint8_t * {
    return recs + ((size_t)(cbase + c - win.lo) * H + h) * rec::BYTES;
  };
  auto load_a1 = [&](int c) {
    mbar_arrive_expect_tx(bar_a1, 32768);
    bulk_load(sm + SB_A1, rec_of(c) + rec::A1, 32768, bar_a1);
  };
  auto load_kp = [&](int c) {
    mbar_arrive_expect_tx(bar_kp, 24576);
    bulk_load(sm + SB_KP, rec_of(c) + rec::KP, 24576, bar_kp);
  };
  if (tid == 0 && c_lo < c_hi) {
    load_a1(c_lo);
    load_kp(c_lo);
  }

  // Record values read by threads (Ut slice and <q_r, k_r> of token tid for
  // warps 0-1, exp(gamma_last) of key t for all) are fetched one chunk ahead.
  float ut[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) ut[i] = 0.f;
  float pd = 0.f, gl = 0.f;
  auto fetch_u = [&](int c) {
    if (warp < 2 && use_ut) {
      const uint8_t *rp = rec_of(c);
      const float4 *src =
          reinterpret_cast<const float4 *>(rp + rec::UT + ((size_t)tid * 128 + slice * 32) * 4);
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const float4 f = __ldcs(src + x);
        ut[4 * x] = f.x; ut[4 * x + 1] = f.y; ut[4 * x + 2] = f.z; ut[4 * x + 3] = f.w;
      }
      pd = __ldcs(reinterpret_cast<const float *>(rp + rec::PD) + tid);
    }
  };
  auto fetch_gl = [&](int c) { gl = __ldg(reinterpret_cast<const float *>(rec_of(c) + rec::GL) + t); };
  if (c_lo < c_hi) {
    fetch_u(c_lo);
    fetch_gl(c_lo);
  }

  uint32_t pa = 0, pk = 0, pm = 0, pm2 = 0;
  bool failed = false;  // a wait ran out: copies or MMAs may still be in flight
  bool m2_ok = true;    // this thread's waits on the second MMA group completed
  for (int c = c_lo; c < c_hi; ++c) {
    const int t0 = bos + 64 * c, Lc = min(64, eos - t0);
    if (ckpt) {  // entry state of the chunk, for the backward pass
      float *dst = ckpt + ((size_t)(cbase + c) * H + h) * (128 * 128) + sbase;
#pragma unroll
      for (int i = 0; i < 32; ++i) dst[(size_t)i * 128] = S[i];
    }

    // ---- D1 = [W ; Q G] S ----------------------------------------------------------
    if (__syncthreads_or(!(mbar_wait(bar_a1, pa) && m2_ok))) {
      if (tid == 0) report(status, KDA_ERR_DEVICE_TIMEOUT);
      failed = true;
      break;
    }
    pa ^= 1;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t a1 = smem_u32(sm + SB_A1), sop = smem_u32(sm + SB_S);
      constexpr uint32_t id = idesc_fp16(128, 32, false, true);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)  // one accumulator over the 128 key channels
        mma_bf16(tmem + TB_D1, desc_kmajor(a1, 128, ks), desc_mn32_sw64(sop, ks), id, ks > 0);
      mma_commit(bar_mma);
    }
    // Only warps 0-1 read this group's result (W S, TMEM lanes 0..63); warps 2-3 go on
    // to the second group's wait.  A failed wait stops the issuing thread from starting
    // the second group, so every thread's wait on it then fails and the loop ends.
    bool ok1 = true;
    if (warp < 2) {
      ok1 = mbar_wait(bar_mma, pm);
      if (!ok1) report(status, KDA_ERR_DEVICE_TIMEOUT);
      tc_fence_after();
    } else if (tid == 64 && c + 1 < c_hi && mbar_wait(bar_mma, pm)) {
      load_a1(c + 1);  // A1 has been read (warp 2 is idle until the second group's result)
    }
    pm ^= 1;

    // ---- U = Ut - W S (warps 0-1: TMEM lanes 0..63 are the chunk's tokens) -------------
    if (warp < 2) {
      float y[32];
      tmem_ld32(tmem + lane_addr + TB_D1, y);
      const int r = tid;
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        y[i] = ut[i] - y[i];  // U
        amax = fmaxf(amax, fabsf(y[i]));
      }
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = y[8 * x + e];
        st_shared_16(sm + SB_U, mn32_sw64_off(r, x), pack8_f16(f));
      }
      if (!(amax < 32768.f)) report(status, KDA_ERR_DEVICE_RANGE);
      // Only warps 0-1 wrote the U operand and read D1: they alone meet before the
      // issuing thread (warp 0) starts the MMAs that read U and accumulate into D1.
      fence_async_smem();
      tc_fence_before();
      asm volatile("bar.sync 1, 64;" ::: "memory");

      // ---- D1 += [* ; P] U ;  D2 = K'^T U ------------------------------------------
      if (tid == 0) {
        if (ok1 && mbar_wait(bar_kp, pk)) {  // K', P of this chunk
          tc_fence_after();
          const uint32_t a2 = smem_u32(sm + SB_A2), uop = smem_u32(sm + SB_U);
          const uint32_t kp = smem_u32(sm + SB_KP);
          constexpr uint32_t idO = idesc_fp16(128, 32, false, true);
          constexpr uint32_t idS = idesc_fp16(128, 32, true, true);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {  // the two accumulators' steps interleaved
            mma_bf16(tmem + TB_D1, desc_kmajor(a2, 128, ks), desc_mn32_sw64(uop, ks), idO, 1);
            mma_bf16(tmem + TB_D2, desc_mnmajor(kp, 64, ks), desc_mn32_sw64(uop, ks), idS,
                     ks > 0);
          }
          mma_commit(bar_m2);
        } else {
          report(status, KDA_ERR_DEVICE_TIMEOUT);  // no commit: the wait below times out too
        }
      }
      // While the second group runs: the token's own term for warps 2-3 (the S operand
      // is dead until the next chunk) and the next chunk's Ut and <q_r, k_r>.
      if (kRole == kOutputs) {
#pragma unroll
        for (int i = 0; i < 32; ++i) exch[i * 64 + r] = pd * y[i];
        asm volatile("bar.arrive 2, 128;" ::: "memory");  // the exchange is written
      }
      if (c + 1 < c_hi) fetch_u(c + 1);
    }
    pk ^= 1;
    // Each thread waits for the second group by itself; a wait that ran out is acted on
    // at the next CTA-wide wait (the loop's next tile wait, or the check after the loop).
    m2_ok = mbar_wait(bar_m2, pm2) && m2_ok;
    pm2 ^= 1;
    tc_fence_after();
    // K' and P have been read: the next chunk's come in.  Warp 1 issues the copy (warp 0's
    // state update is on the chunk's critical path; warp 1 only waits at the chunk's end).
    if (tid == 32 && c + 1 < c_hi && m2_ok) load_kp(c + 1);

    // ---- outputs (warps 2-3: TMEM lanes 64..127) and the state update ---------------------
    {
      float ds[32];
      tmem_ld32(tmem + lane_addr + TB_D2, ds);
#pragma unroll
      for (int i = 0; i < 32; ++i) S[i] = fmaf(S[i], gl, ds[i]);
      if (c + 1 < c_hi) fetch_gl(c + 1);
    }
    if (kRole == kOutputs && warp >= 2) asm volatile("bar.sync 2, 128;" ::: "memory");
    if (kRole == kOutputs && warp >= 2 && o) {
      float ov[32];
      tmem_ld32(tmem + lane_addr + TB_D1, ov);
      const int r = tid - 64;
#pragma unroll
      for (int i = 0; i < 32; ++i) ov[i] = scale * (ov[i] + exch[i * 64 + r]);
      // Token r's 32 values go back over the exchange as a row of the read-out tile
      // (16-byte chunks swizzled by the row), so that the global stores below write whole
      // 128-byte rows with eight lanes each instead of one lane per row.
      asm volatile("bar.sync 4, 64;" ::: "memory");  // warps 2-3 have read the exchange
#pragma unroll
      for (int x = 0; x < 8; ++x)
        reinterpret_cast<float4 *>(exch)[r * 8 + (x ^ (r & 7))] =
            make_float4(ov[4 * x], ov[4 * x + 1], ov[4 * x + 2], ov[4 * x + 3]);
      asm volatile("bar.sync 4, 64;" ::: "memory");
      if (m2_ok) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int id = 64 * k + r, row = id >> 3, x = id & 7;
          if (row < Lc && in_range(status, t0 + row, T))
            __stcs(reinterpret_cast<float4 *>(o + ((size_t)(t0 + row) * H + h) * 128 + slice * 32) + x,
                   reinterpret_cast<const float4 *>(exch)[row * 8 + (x ^ (row & 7))]);
        }
      }
    }
    __syncthreads();  // the exchange has been read; the S operand goes over it
    write_s_operand();
    fence_async_smem();
    tc_fence_before();
    // the next chunk's wait on its [W; Q G] tile is the barrier before MMA1 reads S
  }

  if (!failed && __syncthreads_or(!m2_ok)) {  // the last chunk's second-group wait
    if (tid == 0) report(status, KDA_ERR_DEVICE_TIMEOUT);
    failed = true;
  }
  if (s_out && !failed) {
#pragma unroll
    for (int i = 0; i < 32; ++i) s_out[sbase + (size_t)i * 128] = S[i];
  }
  if (failed && tid == 0) {  // let in-flight record copies and MMAs land first
    drain(bar_a1);
    drain(bar_kp);
    drain(bar_mma);
    drain(bar_m2);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, TB_COLS);
}

// Inclusive-to-exclusive block scan step over 1024 threads: returns the
// exclusive prefix of x among the threads and adds the block total to carry.
__device__ __forceinline__ int block_exclusive_scan(int x, int *wsum, int &carry) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int v = x;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, d);
    if (lane >= d) v += y;
  }
  if (lane == 31) wsum[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int w = wsum[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += y;
    }
    wsum[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const int r = carry + (warp > 0 ? wsum[warp - 1] : 0) + v - x;
  carry += wsum[31];
  __syncthreads();
  return r;
}

// cprefix[n] = number of chunks of sequences 0..n-1 (cprefix[N] = total); with
// a segment length L > 0 also sprefix[n] = number of segments of sequences
// 0..n-1, sequence n having max(1, ceil(nch_n / L)).  cu == NULL is one
// sequence of T tokens.  A malformed cu_seqlens (decreasing, or outside
// [0, T]) is recorded and gives every sequence zero chunks and one segment,
// so no pass reads or writes past the workspace.  A segment total above
// seg_cap (not reachable for valid cu) falls back to one segment per sequence.
__global__ void __launch_bounds__(1024)
chunk_index_kernel(const int32_t *__restrict__ cu, int N, int T, int L, long long seg_cap,
                   int32_t *cprefix, int *status) {
  __shared__ int bad;
  __shared__ int wsum[32];
  int32_t *sprefix = cprefix + (N + 1);
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int i = tid; i < N && cu; i += 1024) {
    const int a = cu[i], b = cu[i + 1];
    if (a < 0 || b < a || b > T) bad = 1;
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) report(status, KDA_ERR_DEVICE_BOUNDS);
    for (int i = tid; i <= N; i += 1024) {
      cprefix[i] = 0;
      if (L > 0) sprefix[i] = i;
    }
    return;
  }
  int carry = 0, scarry = 0;
  for (int base = 0; base < N; base += 1024) {
    const int i = base + tid;
    const int len = i < N ? (cu ? cu[i + 1] - cu[i] : T) : 0;
    const int cnt = (len + 63) / 64;
    const int c = block_exclusive_scan(cnt, wsum, carry);
    if (i < N) cprefix[i] = c;
    if (L > 0) {
      const int sc = block_exclusive_scan(i < N ? max(1, (cnt + L - 1) / L) : 0, wsum, scarry);
      if (i < N) sprefix[i] = sc;
    }
  }
  if (tid == 0) {
    cprefix[N] = carry;
    if (L > 0) sprefix[N] = scarry;
  }
  if (L > 0 && scarry > seg_cap) {
    __syncthreads();
    for (int i = tid; i <= N; i += 1024) sprefix[i] = i;
  }
}

// Entry states of the segments: E_1 (written by the transition pass) and
// E_{g+1} = M_g E_g + B_g for g = 1 .. G-2, in fp32.  One CTA per (sequence,
// head, 8 value columns).  E_g sits in shared memory; M_g (64 KB, stored
// column by column) is brought into shared memory by a bulk copy,
// double-buffered so that M_{g+1} arrives while step g computes.  Warp w sums
// the key channels k in [32 w, 32 w + 32) and lane l rows l + 32 i (i < 4), so
// each broadcast read of a row of E_g feeds four rows; the four warps' partial
// sums meet in shared memory, where thread r adds up row r.
constexpr int kScanCols = 8;
constexpr uint32_t SC_M = 0;                                   // 2 x 64 KB
constexpr uint32_t SC_E = 2 * 65536;                           // [128][kScanCols] fp32
constexpr uint32_t SC_P = SC_E + 128 * kScanCols * 4;          // [4][128][kScanCols] fp32
constexpr uint32_t SC_BAR = SC_P + 4 * 128 * kScanCols * 4;    // two mbarriers
constexpr uint32_t SC_ALLOC = SC_BAR + 16 + 128;               // + alignment slack

__global__ void __launch_bounds__(128)
state_scan_kernel(const uint8_t *__restrict__ ws, int N, int T, int H, int *status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                            ~static_cast<uintptr_t>(127));
  const int r = threadIdx.x, lane = r & 31, warp = r >> 5;
  const int cb = blockIdx.x % (128 / kScanCols), nh = blockIdx.x / (128 / kScanCols);
  const int h = nh % H, n = nh / H;
  const int32_t *sprefix = reinterpret_cast<const int32_t *>(ws) + (N + 1);
  const int s0 = sprefix[n], G = sprefix[n + 1] - s0;
  if (G <= 2) return;
  // debug builds: the sequence's segments are among the batch's sprefix[N]
  if (!in_range(status, s0, sprefix[N]) || !in_range(status, s0 + G - 1, sprefix[N])) return;
  float *segbuf = reinterpret_cast<float *>(const_cast<uint8_t *>(ws) +
                                            rec::segment_area_offset(N, T, H));
  auto slot = [&](int seg, int kind) -> float * {
    return segbuf + (((size_t)seg * H + h) * 3 + kind) * (128 * 128);
  };
  constexpr int kQ = kScanCols / 4;  // float4 per row
  float4 *Es = reinterpret_cast<float4 *>(sm + SC_E);
  float4 *Ps = reinterpret_cast<float4 *>(sm + SC_P);
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + SC_BAR);
  if (r == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 1, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar, 65536);
    bulk_load(sm + SC_M, slot(s0 + 1, 0), 65536, bar);
  }
  const int j0 = cb * kScanCols;
  {
    const float *e = slot(s0 + 1, 2);
    float v[kScanCols];
#pragma unroll
    for (int j = 0; j < kScanCols; ++j) v[j] = e[(size_t)(j0 + j) * 128 + r];
#pragma unroll
    for (int q = 0; q < kQ; ++q)
      Es[r * kQ + q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  }
  __syncthreads();
  // B_g (row r) is read one step ahead, so its latency hides behind the step before.
  float bnext[kScanCols];
  auto load_b = [&](int g) {
    const float *B = slot(s0 + g, 1);
#pragma unroll
    for (int j = 0; j < kScanCols; ++j) bnext[j] = B[(size_t)(j0 + j) * 128 + r];
  };
  load_b(1);
  uint32_t phase = 0;  // bit b: parity of buffer b
  for (int g = 1; g + 1 < G; ++g) {
    const int b = (g - 1) & 1;
    if (r == 0 && g + 2 < G) {  // buffer b^1 was last read in step g - 1
      mbar_arrive_expect_tx(bar + (b ^ 1), 65536);
      bulk_load(sm + SC_M + (b ^ 1) * 65536, slot(s0 + g + 1, 0), 65536, bar + (b ^ 1));
    }
    float bcur[kScanCols];
#pragma unroll
    for (int j = 0; j < kScanCols; ++j) bcur[j] = bnext[j];
    if (g + 2 < G) load_b(g + 1);
    if (!wait_all(bar + b, (phase >> b) & 1, status)) {
      if (r == 0) {  // the other buffer's copy may still be in flight
        drain(bar);
        drain(bar + 1);
      }
      return;
    }
    phase ^= 1u << b;
    const float *Ms = reinterpret_cast<const float *>(sm + SC_M + b * 65536);
    float acc[4][kScanCols];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < kScanCols; ++j) acc[i][j] = 0.f;
#pragma unroll 4
    for (int kk = 0; kk < 32; ++kk) {
      const int k = 32 * warp + kk;
      float m[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) m[i] = Ms[k * 128 + lane + 32 * i];  // M_g[row][k]
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        const float4 e = Es[k * kQ + q];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[i][4 * q] = fmaf(m[i], e.x, acc[i][4 * q]);
          acc[i][4 * q + 1] = fmaf(m[i], e.y, acc[i][4 * q + 1]);
          acc[i][4 * q + 2] = fmaf(m[i], e.z, acc[i][4 * q + 2]);
          acc[i][4 * q + 3] = fmaf(m[i], e.w, acc[i][4 * q + 3]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int q = 0; q < kQ; ++q)
        Ps[(warp * 128 + lane + 32 * i) * kQ + q] =
            make_float4(acc[i][4 * q], acc[i][4 * q + 1], acc[i][4 * q + 2], acc[i][4 * q + 3]);
    __syncthreads();  // partial sums written; every thread has read E_g and M_g
    float out[kScanCols];
#pragma unroll
    for (int j = 0; j < kScanCols; ++j) out[j] = bcur[j];
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
      for (int q = 0; q < kQ; ++q) {
        const float4 p = Ps[(w * 128 + r) * kQ + q];
        out[4 * q] += p.x;
        out[4 * q + 1] += p.y;
        out[4 * q + 2] += p.z;
        out[4 * q + 3] += p.w;
      }
    float *e = slot(s0 + g + 1, 2);
#pragma unroll
    for (int j = 0; j < kScanCols; ++j) e[(size_t)(j0 + j) * 128 + r] = out[j];
#pragma unroll
    for (int q = 0; q < kQ; ++q)
      Es[r * kQ + q] = make_float4(out[4 * q], out[4 * q + 1], out[4 * q + 2], out[4 * q + 3]);
    __syncthreads();  // E_{g+1} in place; the partial sums have been read
  }
}

// Fused two-pass prefill: a sequence without chunks (empty, or every sequence
// when the index pass rejected cu_seqlens) has no prep item to write its conv
// cache, so it is passed through here: cache_out[n] = cache_in[n], or zero.
// Elements are 16-bit (bf16 or fp16; +0.0 is all-zero bits in both).
__global__ void __launch_bounds__(256)
cache_pass_kernel(const int32_t *__restrict__ cprefix, const uint16_t *__restrict__ cache_in,
                  uint16_t *__restrict__ cache_out, long long per_seq) {
  const int n = blockIdx.x;
  if (cprefix[n + 1] != cprefix[n]) return;
  const size_t base = (size_t)n * per_seq;
  for (long long i = threadIdx.x; i < per_seq; i += blockDim.x)
    cache_out[base + i] = cache_in ? cache_in[base + i] : (uint16_t)0;
}

}  // namespace

cudaError_t launch_cache_pass(const void *ws, int N, int H, const void *cache_in,
                              void *cache_out, cudaStream_t s) {
  cache_pass_kernel<<<N, 256, 0, s>>>(static_cast<const int32_t *>(ws),
                                      static_cast<const uint16_t *>(cache_in),
                                      static_cast<uint16_t *>(cache_out), 3LL * 3 * H * 128);
  return cudaGetLastError();
}

cudaError_t launch_chunk_index(const int32_t *cu, int N, int T, int L, void *ws, int *status,
                               cudaStream_t s) {
  chunk_index_kernel<<<1, 1024, 0, s>>>(cu, N, T, L, rec::segment_capacity(N, T, L),
                                        static_cast<int32_t *>(ws), status);
  return cudaGetLastError();
}

namespace {
template <int kRole>
cudaError_t launch_state_role(const void *ws, const int32_t *cu, const float *s0, float scale,
                              int N, int T, int H, int L, float *o, float *sN, float *ckpt,
                              int *status, cudaStream_t s, float *map_m = nullptr,
                              float *map_b = nullptr, const ChunkWindow &win = ChunkWindow{}) {
  const long long items = L > 0 ? rec::segment_capacity(N, T, L) : N;
  const long long blocks = items * H * kSlices * (kRole == kOutputs ? 1 : 2);
  if (blocks >= (1LL << 31)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(chunk_state_kernel<kRole>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SB_ALLOC);
  if (e != cudaSuccess) return e;
  chunk_state_kernel<kRole><<<(unsigned)blocks, kBT, SB_ALLOC, s>>>(
      static_cast<const uint8_t *>(ws), cu, s0, scale, N, T, H, L, o, sN, ckpt, map_m, map_b,
      status, win);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_chunk_map(const void *ws, const int32_t *cu, int N, int T, int H, float *map_m,
                             float *map_b, int *status, cudaStream_t s) {
  return launch_state_role<kMap>(ws, cu, nullptr, 1.f, N, T, H, 0, nullptr, nullptr, nullptr,
                                 status, s, map_m, map_b);
}

namespace {
// E_out = M E_in + B per (sequence, head), fp32: one CTA per (sequence, head, 8 value
// columns), thread r owns row r (key channel); E_in's 8 columns sit in shared memory
// and row r of M is read column by column (consecutive threads, consecutive words).
__global__ void __launch_bounds__(128)
state_compose_kernel(const float *__restrict__ M, const float *__restrict__ B,
                     const float *__restrict__ E_in, float *__restrict__ E_out, int NH) {
  __shared__ float Es[128][kScanCols];
  const int r = threadIdx.x;
  const int cb = blockIdx.x % (128 / kScanCols), nh = blockIdx.x / (128 / kScanCols);
  const size_t off = (size_t)nh * 128 * 128;
  const int j0 = cb * kScanCols;
#pragma unroll
  for (int j = 0; j < kScanCols; ++j) Es[r][j] = E_in ? E_in[off + (size_t)(j0 + j) * 128 + r] : 0.f;
  __syncthreads();
  float acc[kScanCols];
#pragma unroll
  for (int j = 0; j < kScanCols; ++j) acc[j] = B[off + (size_t)(j0 + j) * 128 + r];
  if (E_in) {
#pragma unroll 8
    for (int k = 0; k < 128; ++k) {
      const float m = M[off + (size_t)k * 128 + r];  // M[r][k]
#pragma unroll
      for (int j = 0; j < kScanCols; ++j) acc[j] = fmaf(m, Es[k][j], acc[j]);
    }
  }
#pragma unroll
  for (int j = 0; j < kScanCols; ++j) E_out[off + (size_t)(j0 + j) * 128 + r] = acc[j];
}
}  // namespace

cudaError_t launch_state_compose(const float *M, const float *B, const float *E_in, float *E_out,
                                 int NH, cudaStream_t s) {
  const long long blocks = (long long)NH * (128 / kScanCols);
  if (blocks >= (1LL << 31)) return cudaErrorInvalidValue;
  state_compose_kernel<<<(unsigned)blocks, 128, 0, s>>>(M, B, E_in, E_out, NH);
  return cudaGetLastError();
}

cudaError_t launch_chunk_state(const void *ws, const int32_t *cu, const float *s0, float scale,
                               int N, int T, int H, int L, float *o, float *sN, int *status,
                               cudaStream_t s, float *ckpt, const ChunkWindow &win) {
  cudaError_t e;
  if (L > 0) {
    e = launch_state_role<kTransition>(ws, cu, s0, scale, N, T, H, L, o, sN, nullptr, status,
                                       s);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(state_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SC_ALLOC);
    if (e != cudaSuccess) return e;
    state_scan_kernel<<<N * H * (128 / kScanCols), 128, SC_ALLOC, s>>>(
        static_cast<const uint8_t *>(ws), N, T, H, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return launch_state_role<kOutputs>(ws, cu, s0, scale, N, T, H, L, o, sN, ckpt, status, s,
                                     nullptr, nullptr, win);
}

}  // namespace kda
