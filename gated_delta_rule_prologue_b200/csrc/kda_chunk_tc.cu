// Chunkwise KDA prefill on the 5th-generation tensor cores (tcgen05 + TMEM,
// TMA tile loads), bf16 or fp16 q/k/v, d_k = d_v = 128, chunk 64, fp32 state
// and fp32 read-out.
//
// Sources: "Kimi K3的线性注意力：从源码看懂KDA如何更新记忆", 彩蛋 (chunked
// execution; the K3 report's observation that inside a 16-token block the
// cumulative log-decay of the bounded gate stays in [-80, 0], so the
// reciprocal scaling fits the bf16 range and the diagonal blocks can use dense
// tensor-core products); "AI-Workshop 文献分享 #16 — KDA：给长文本建立可更新的记忆",
// §10.3; "KimiK3轻量化复刻实现KDA并行解析，Chunkwise并行与状态压缩机制详解",
// Figure 1 (the chunk map of the state is affine).
//
// Per chunk (entry state S key-first; gamma = inclusive in-chunk cumsum of g).
// The 64 tokens form two halves, each with a reference in its middle:
// c_A = gamma_15 for tokens 0..31 and c_B = gamma_47 for tokens 32..63.  With
// g >= -5 a half spans at most 16 tokens on either side of its reference, so
// E_r = exp(gamma_r - c(r)) lies in [e^-80, e^75] and every factor below fits
// the fp32 exponent range:
//   Gram  D_G = [K*E ; Q*E] . [ver_A ; ver_B]^T          (M=128, N=96, K=128)
//         ver_A_i = k_i / E_i                     (i < 32, reference c_A)
//         ver_B_i = k_i / E_i * exp(c_B - c(i))   (i < 64, reference c_B; for i < 32
//                   the factor is applied as two halves: it alone can underflow
//                   while the product with the row factor of token 32 cannot)
//         rows of the first half read ver_A, rows of the second half ver_B.
//         A[r,i] = beta_r D_G[r, i] (i < r);  P[r,i] = D_G[64+r, i] (i < r)
//         P[r,r] = <q_r, k_r> is taken in fp32 from the unscaled tiles.
//         The Gram operands are fp32 rounded to tf32 (10-bit significand, fp32
//         range; MMA kind::tf32), one accumulator over the 128 key channels.
//   WY    T = (I + A)^{-1}: the four 16x16 diagonal blocks inverted by forward
//         substitution in fp32, the off-diagonal blocks by four fp16 MMA stages
//         W^T = (beta K G)^T T^T,  Ut^T = (beta V)^T T^T           (G_r = exp(gamma_r))
//   state U^T = Ut^T - S^T W^T,   O^T = S^T (Q G)^T + U^T P_strict^T
//         S <- diag(G_last) S + U^T (K * G_last / G)    (value-major registers)
//   Operand types: the Gram operands are tf32 (they need the e^+-80 range);
//   every other operand (T, beta K G, beta V, S^T, W, Q G, U^T, P, K') has a
//   modest range and is fp16, whose 11-bit significand keeps the read-out
//   within the parity bound when the decay is slow.  A value that would not
//   fit fp16 (|x| >= 2^15) is recorded in the status word.
//   fp32 diagonal terms: u_r gets beta_r v_r - f16(beta_r v_r) back, and
//   o_r gets <q_r, k_r> u_r in fp32, so a token's own (dominant) contribution
//   to its read-out is never rounded to bf16.
// One-pass modes: one CTA (512 threads) per (sequence, head); the chunks of a
// sequence run in order, the next chunk's tiles stream in by TMA during the
// current one.  Prep modes: the state-independent half per (chunk, head) item
// (see the mode list at the kernel).
#include <cuda.h>
#include <algorithm>
#include <cstring>
#include <type_traits>
#include <cudaTypedefs.h>

#include "kda_chunk_record.cuh"
#include "kda_common.cuh"
#include "kda_tcgen05.cuh"

namespace kda {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

namespace {
using namespace tc;

// Zeros for the inverse's 16-bit tiles (D16 + Zm, 16 KB; T32, 8 KB), copied in by the
// bulk-copy engine instead of written by threads.
__device__ __align__(128) uint8_t g_zero_tiles[16384];

constexpr int kThreads = 512;
constexpr int kHalf = kThreads / 2;

// Barriers of the first half of the CTA (warps 0-7) or of the second (warps 8-15) only.
__device__ __forceinline__ void bar_half() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ void bar_second_half() { asm volatile("bar.sync 2, 256;" ::: "memory"); }

// ---- shared memory plan (byte offsets from a 1024-aligned base) ----------------
constexpr uint32_t SM_Q = 0;                // raw q tile [64][128] bf16
constexpr uint32_t SM_K = SM_Q + 16384;     // raw k tile
constexpr uint32_t SM_V = SM_K + 16384;     // raw v tile
constexpr uint32_t SM_G = SM_V + 16384;     // raw g [64][128] f32 -> gamma -> E -> (A^T, T)
constexpr uint32_t SM_X = SM_G + 32768;     // 64 KB, reused within a chunk (the Gram's
                                            // two tiles also use TOP, POP and ST, 112 KB):
constexpr uint32_t SM_GA = SM_X;            //   Gram A operand, tf32 (K-major 128 x 128, 64 KB)
constexpr uint32_t SM_GB = SM_X + 65536;    //   Gram B operand, tf32 (K-major 96 x 128, 48 KB)
constexpr uint32_t SM_BKG = SM_X;           //   beta K G (MN-major, 64 k-rows)     16 KB; then W op
constexpr uint32_t SM_BV = SM_X + 16384;    //   beta V   (MN-major)                16 KB
constexpr uint32_t SM_QG = SM_X + 32768;    //   Q G      (K-major 64 x 128)        16 KB
constexpr uint32_t SM_KP = SM_X + 49152;    //   K G_last/G (MN-major)              16 KB
constexpr uint32_t SM_TOP = SM_X + 65536;   // T operand (K-major 64 x 64) 8 KB; before it is
constexpr uint32_t SM_XS = SM_TOP;          //   written: scratch (cumsum totals, inverse blocks)
constexpr uint32_t SM_POP = SM_TOP + 8192;  // P operand (K-major 64 x 64)          8 KB
constexpr uint32_t SM_ST = SM_POP + 8192;   // S^T operand (K-major 128 x 128) 32 KB; then U^T
constexpr uint32_t SM_F = SM_ST + 32768;    // per-channel fp32 factors [128] each:
constexpr uint32_t F_CA = SM_F;             //   c_A = gamma_15
constexpr uint32_t F_CB = F_CA + 512;       //   c_B = gamma_47
constexpr uint32_t F_ECA = F_CB + 512;      //   exp(c_A)
constexpr uint32_t F_ECB = F_ECA + 512;     //   exp(c_B)
constexpr uint32_t F_EBA = F_ECB + 512;     //   exp((c_B - c_A) / 2): applied twice, so no
                                            //   partial product underflows (c_B - c_A >= -160)
constexpr uint32_t F_ELA = F_EBA + 512;     //   exp(gamma_last - c_A)
constexpr uint32_t F_ELB = F_ELA + 512;     //   exp(gamma_last - c_B)
constexpr uint32_t F_EGC = F_ELB + 512;     //   exp(gamma_last)
constexpr uint32_t SM_BETA = F_EGC + 512;   // beta of the chunk     [64]
constexpr uint32_t SM_PDIAG = SM_BETA + 256;// <q_r, k_r> in fp32    [64]
constexpr uint32_t SM_BAR = SM_PDIAG + 256; // four mbarriers (tiles, MMAs, inverse MMAs, zero fill)
constexpr uint32_t SM_SLOT = SM_BAR + 32;   // TMEM base address
constexpr uint32_t SM_TOTAL = SM_SLOT + 16;
// Fused prologue only: fp32 correction beta*v - f16(beta*v_tile) kept as bf16
// [64][128], and two conv histories (3 parts x 3 rows x 128 raw values).
constexpr uint32_t SM_CORR = (SM_TOTAL + 1023) & ~1023u;
constexpr uint32_t SM_HIST = SM_CORR + 16384;
constexpr uint32_t SM_WCONV = SM_HIST + 2 * 3 * 3 * 128 * 2;  // conv weights of head h [3][4 taps][128] f32
constexpr uint32_t SM_TOTAL_FUSED = SM_WCONV + 3 * 128 * 4 * 4;
constexpr uint32_t SM_ALLOC = SM_TOTAL + 1024;  // slack for 1024-byte alignment
constexpr uint32_t SM_ALLOC_PREP = SM_CORR + 16384 + 1024;  // plus the remainder tile
constexpr uint32_t SM_ALLOC_FUSED = SM_TOTAL_FUSED + 1024;
static_assert(SM_ALLOC_FUSED <= 232448, "shared memory budget");
static_assert(SM_ALLOC_PREP <= SM_ALLOC_FUSED, "the prep plan is a prefix of the fused one");
static_assert(SM_GB + 49152 <= SM_ST + 32768, "Gram tiles stay inside X, TOP, POP and ST");
// The 64 x 64 inverse (P4b / P5) works in the S^T tile and the T tile, both dead
// from the Gram MMA to P6.  16-bit tiles are 64 rows x 128 bytes, row-major with
// the 128-byte swizzle: the same bytes serve as a K-major A operand (row = M
// index) and as an MN-major B operand (row = K index).  An A operand is read as
// M = 128 rows, so 8 KB past each A tile must be readable (those rows' products
// land in TMEM lanes 64..127, which nobody reads).
constexpr uint32_t SM_A16 = SM_ST;           // A = beta-scaled strict lower Gram, fp16; after
constexpr uint32_t SM_YM = SM_ST;            //   the third product, Y's lower-left block
constexpr uint32_t SM_D16 = SM_ST + 8192;    // D = inverses of the 16x16 diagonal blocks
constexpr uint32_t SM_ZM = SM_ST + 16384;    // the two in-half off-diagonal blocks of A D
constexpr uint32_t SM_ATD = SM_ST + 24576;   // fp32 diagonal 16x16 blocks of A, [blk][col][row]
constexpr uint32_t SM_T32 = SM_TOP;          // T at the 32x32-block level, then T itself
static_assert(SM_T32 + 16384 <= SM_ST && SM_D16 + 16384 <= SM_ST + 32768 &&
              SM_ATD + 4096 <= SM_ST + 32768 && SM_ST + 32768 <= SM_F,
              "A-operand reads stay inside shared memory");

// ---- TMEM columns (fp32 accumulators, 128 lanes) -------------------------------
constexpr uint32_t TM_G = 0;     // Gram, 96 columns
constexpr uint32_t TM_W = 160;   // W^T, 64
constexpr uint32_t TM_U = 224;   // U^T, 64
constexpr uint32_t TM_O = 288;   // O^T, 64
constexpr uint32_t TM_S = 352;   // delta S^T, 128
// The inverse's MMA stages (during P5 only, before W / Ut / O / delta S are written):
constexpr uint32_t TM_Z = 96;    // Z = A D, 64 columns; later T32 Y
constexpr uint32_t TM_T2 = 384;  // D Z, 64 (over delta S, written only after P5)
constexpr uint32_t TM_Y = 448;   // Y = A T32, 64
constexpr uint32_t TM_COLS = 512;
static_assert(TM_Z + 64 <= TM_W && TM_G + 96 <= TM_Z && TM_T2 + 64 <= TM_Y &&
              TM_Y + 64 <= TM_COLS && TM_S + 128 <= TM_COLS, "TMEM column plan");

constexpr uint32_t kHaloBytes = 3 * 3 * 128 * 2;  // three raw rows of the q, k, v parts


__device__ __forceinline__ void ld8_f32_pairs(const float *p, float2 (&f)[4]) {
  const float4 a = reinterpret_cast<const float4 *>(p)[0];
  const float4 b = reinterpret_cast<const float4 *>(p)[1];
  f[0] = make_float2(a.x, a.y); f[1] = make_float2(a.z, a.w);
  f[2] = make_float2(b.x, b.y); f[3] = make_float2(b.z, b.w);
}

// 8 consecutive K-elements [8*c8, 8*c8+8) of `row` of a K-major fp32 tile of `rows`
// rows, rounded to tf32: two 16-byte chunks.
__device__ __forceinline__ void st_tf32x8(uint8_t *tile, int rows, int row, int c8,
                                          const float (&f)[8]) {
  const uint4 lo = make_uint4(tf32_rna(f[0]), tf32_rna(f[1]), tf32_rna(f[2]), tf32_rna(f[3]));
  const uint4 hi = make_uint4(tf32_rna(f[4]), tf32_rna(f[5]), tf32_rna(f[6]), tf32_rna(f[7]));
  st_shared_16(tile, kmaj_off(rows, row, 2 * c8), lo);
  st_shared_16(tile, kmaj_off(rows, row, 2 * c8 + 1), hi);
}

template <typename Tin>
__device__ __forceinline__ uint4 pack8_in(const float (&f)[8]) {
  uint4 u;
  Tin *h = reinterpret_cast<Tin *>(&u);
#pragma unroll
  for (int i = 0; i < 8; ++i) h[i] = from_f32<Tin>(f[i]);
  return u;
}

// Modes.
//   kSingle: one CTA per (sequence, head) walks its chunks in order and carries
//            the state: the whole chunk update in one kernel.  q, k, v tiles
//            come from HBM as given (already unit-normalised).
//   kFused:  as kSingle, but the three tiles are the raw projections x (parts
//            q, k, v of head h); the prologue (causal width-4 conv with
//            history, SiLU, L2 on q and k) runs in fp32 in shared memory and
//            overwrites them with q, k, v.
//   kPrep:   the state-independent half only: persistent CTAs take the
//            (chunk, head) items blockIdx.x, blockIdx.x + gridDim.x, ... and
//            write one record per item (kda_chunk_record.cuh); the state pass
//            (kda_chunk_state.cu) applies the records in order.
//   kPrepFused: kPrep on raw projections with the prologue of kFused; each
//            item brings its own conv history (the three rows before the
//            chunk, or the cache at a sequence start), and the item holding a
//            sequence's last chunk writes that sequence's cache.
//   kPrepGated, kPrepFusedGated: kPrep / kPrepFused with the log-decay
//            computed from gate pre-activations in the cumsum phase (GateArgs).
//
// Thread layout (512 threads, 16 warps): warp w reads TMEM lanes
// 32*(w%4).. (its "quad") and handles column group w/4 of every accumulator it
// reads; element-wise phases walk (row, 8-channel chunk) pairs.
constexpr int kSingle = 0, kFusedMode = 1, kPrep = 2, kPrepFused = 3, kPrepGated = 4,
              kPrepFusedGated = 5;

// Parameters of the in-kernel bounded gate (the gated prep modes): the g tile
// holds the gate pre-activations (16-bit, like q/k/v or x) and
// g = lower_bound * sigmoid(exp(A_log[h]) * (g_raw + dt_bias[h, :])); either
// pointer may be null (exp(A_log) = 1, dt_bias = 0).
struct GateArgs {
  const float *A_log;
  const float *dt_bias;
  float lower_bound;
};

template <typename Tin, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                const float *__restrict__ beta, float scale, const float *s0,
                const int32_t *__restrict__ cu, int T, int H, float *__restrict__ o, float *sN,
                int *status, const float *__restrict__ conv_w, const Tin *cache_in,
                Tin *cache_out, uint8_t *recs, const int32_t *cprefix, int N, GateArgs gate,
                ChunkWindow win) {
  constexpr bool kFused = kMode == kFusedMode || kMode == kPrepFused || kMode == kPrepFusedGated;
  constexpr bool kGated = kMode == kPrepGated || kMode == kPrepFusedGated;
  constexpr bool kPrepM = kMode == kPrep || kMode == kPrepFused || kGated;
  // bytes of one work item's q, k, v (or x) tiles and its g tile (fp32 log-decay,
  // or 16-bit gate pre-activations)
  constexpr uint32_t kTileBytes = 3 * 16384 + (kGated ? 16384u : 32768u);
  // Element type of the q/k/v tiles the chunk phases read: the inputs as given,
  // or fp16 written by the fused prologue (q, k are unit vectors; v is guarded).
  using Tact = typename std::conditional<kFused, __half, Tin>::type;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                            ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, grp = warp >> 2;
  const int n = blockIdx.x / H, hb = blockIdx.x % H;  // kSingle / kFused
  uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + SM_BAR);
  uint64_t *bar_mma = bar_tma + 1;
  uint64_t *bar_inv = bar_tma + 2;
  uint64_t *bar_zero = bar_tma + 3;
  uint32_t *slot = reinterpret_cast<uint32_t *>(sm + SM_SLOT);
  float *Gf = reinterpret_cast<float *>(sm + SM_G);
  float *beta_s = reinterpret_cast<float *>(sm + SM_BETA);
  float *pdiag = reinterpret_cast<float *>(sm + SM_PDIAG);
  float *feca = reinterpret_cast<float *>(sm + F_ECA);
  float *fecb = reinterpret_cast<float *>(sm + F_ECB);
  float *feba = reinterpret_cast<float *>(sm + F_EBA);
  float *fela = reinterpret_cast<float *>(sm + F_ELA);
  float *felb = reinterpret_cast<float *>(sm + F_ELB);
  float *fegc = reinterpret_cast<float *>(sm + F_EGC);
  float *XS = reinterpret_cast<float *>(sm + SM_XS);

  // The work walk: (t0, Lc, head, chunk number) of step `it`.
  struct Work {
    int t0, Lc, h, ci;
    int n, bos, eos;  // the chunk's sequence
    bool ok;
  };
  int bos = 0, eos = 0, nchunks = 0;
  long long items = 0;
  int total_chunks = 0;
  if constexpr (kPrepM) {
    const long long cap = rec::chunk_capacity(N, T);
    total_chunks = cu ? (int)min((long long)cprefix[N], cap) : (T + 63) / 64;
    items = (long long)max(0, min(total_chunks, win.hi) - win.lo) * H;  // the window's items
  } else {
    seq_bounds(cu, n, T, status, bos, eos);
    nchunks = (eos - bos + 63) / 64;
  }
  auto work_of = [&](int it) -> Work {
    Work w;
    if constexpr (kPrepM) {
      const long long item = (long long)blockIdx.x + (long long)it * gridDim.x;
      w.ok = item < items;
      if (!w.ok) return w;
      w.ci = win.lo + (int)(item / H);
      w.h = (int)(item % H);
      int sb = 0, se = T, c0 = 0, lo = 0;
      if (cu) {  // sequence of chunk ci: the last n with cprefix[n] <= ci
        int hi = N - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (cprefix[mid] <= w.ci) lo = mid; else hi = mid - 1;
        }
        sb = min(max(cu[lo], 0), T);  // well-formed here: the index pass checked cu
        se = min(max(cu[lo + 1], sb), T);
        c0 = cprefix[lo];
      }
      w.t0 = sb + 64 * (w.ci - c0);
      w.Lc = min(64, se - w.t0);
      w.n = lo;
      w.bos = sb;
      w.eos = se;
      w.ok = w.Lc > 0 && in_range(status, w.n, N) &&
             in_range(status, w.ci, rec::chunk_capacity(N, T)) &&
             in_range(status, w.ci - win.lo,
                      min(rec::chunk_capacity(N, T), (long long)win.hi - win.lo)) &&
             in_range(status, w.t0 + w.Lc - 1, T);
    } else {
      w.ok = it < nchunks;
      w.ci = it;
      w.h = hb;
      w.t0 = bos + 64 * it;
      w.Lc = min(64, eos - w.t0);
      w.n = n;
      w.bos = bos;
      w.eos = eos;
      w.ok = w.ok && in_range(status, w.t0 + w.Lc - 1, T);
    }
    return w;
  };

  if (warp == 0) tmem_alloc(slot, TM_COLS);
  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_inv, 1);
    mbar_init(bar_zero, 1);
    fence_mbar_init();
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_g);
  }

  // State rows held in registers: row j of S^T, key columns [dk0, dk0 + 32).
  const int j = 32 * quad + lane;
  const int dk0 = 32 * grp;
  float S[32];
  {
    const float *src = (s0 && !kPrepM) ? s0 + (((size_t)n * H + hb) * 128 + j) * 128 + dk0 : nullptr;
#pragma unroll
    for (int x = 0; x < 32; x += 4) {
      float4 f = src ? *reinterpret_cast<const float4 *>(src + x) : make_float4(0.f, 0.f, 0.f, 0.f);
      S[x] = f.x; S[x + 1] = f.y; S[x + 2] = f.z; S[x + 3] = f.w;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t lane_addr = static_cast<uint32_t>(32 * quad) << 16;

  // The next chunk's tiles are requested as soon as each buffer is dead: q and k
  // after the Gram read-out, g after the inverse, v after the U read-out; one
  // mbarrier phase counts all four.
  // One mbarrier phase counts the four tiles of a work item; it is armed with
  // their total at the item's first issue (the tiles go out as buffers die).
  // kPrepFused: a chunk that does not start its sequence also brings the three
  // raw rows before it (its conv history) into history slot 0.
  auto has_halo = [&](const Work &w) {
    return (kMode == kPrepFused || kMode == kPrepFusedGated) && w.t0 > w.bos;
  };
  auto arm_tma = [&](const Work &w) {
    mbar_arrive_expect_tx(bar_tma, kTileBytes + (has_halo(w) ? kHaloBytes : 0u));
  };
  auto issue_tma_qk = [&](const Work &w) {
    if constexpr (kFused) {  // x viewed as [T, 3H, 128]: part p of head h is row p*H + h
      tma_load_3d(sm + SM_Q, &tm_q, bar_tma, 0, w.h, w.t0);
      tma_load_3d(sm + SM_K, &tm_q, bar_tma, 0, H + w.h, w.t0);
    } else {
      tma_load_3d(sm + SM_Q, &tm_q, bar_tma, 0, w.h, w.t0);
      tma_load_3d(sm + SM_K, &tm_k, bar_tma, 0, w.h, w.t0);
    }
  };
  auto issue_tma_g = [&](const Work &w) { tma_load_3d(sm + SM_G, &tm_g, bar_tma, 0, w.h, w.t0); };
  auto issue_tma_v = [&](const Work &w) {
    if constexpr (kFused)
      tma_load_3d(sm + SM_V, &tm_q, bar_tma, 0, 2 * H + w.h, w.t0);
    else
      tma_load_3d(sm + SM_V, &tm_v, bar_tma, 0, w.h, w.t0);
  };
  Tin *hist = reinterpret_cast<Tin *>(sm + SM_HIST);  // [2][3 parts][3 rows][128]
  auto issue_tma_halo = [&](const Work &w) {  // tm_k maps x with a 3-row box
    if (has_halo(w))
      for (int p = 0; p < 3; ++p)
        tma_load_3d(hist + p * 384, &tm_k, bar_tma, 0, p * H + w.h, w.t0 - 3);
  };
  auto issue_tma = [&](const Work &w) {
    arm_tma(w);
    issue_tma_qk(w);
    issue_tma_g(w);
    issue_tma_v(w);
    issue_tma_halo(w);
  };
  __nv_bfloat16 *corr = reinterpret_cast<__nv_bfloat16 *>(sm + SM_CORR);
  const int HD = H * 128;
  float *wconv = reinterpret_cast<float *>(sm + SM_WCONV);
  if constexpr (kMode == kFusedMode) {
    for (int idx = tid; idx < 3 * 128; idx += kThreads) {  // tap-major: lanes read consecutive channels
      const int p = idx >> 7, ch = idx & 127;
      const float4 w = __ldg(reinterpret_cast<const float4 *>(conv_w + ((size_t)p * HD + hb * 128 + ch) * 4));
      wconv[(p * 4 + 0) * 128 + ch] = w.x;
      wconv[(p * 4 + 1) * 128 + ch] = w.y;
      wconv[(p * 4 + 2) * 128 + ch] = w.z;
      wconv[(p * 4 + 3) * 128 + ch] = w.w;
    }
    // conv history before the sequence: the cache rows (oldest first) or zero
    for (int idx = tid; idx < 9 * 128; idx += kThreads) {
      const int pr = idx >> 7, ch = idx & 127, p = pr / 3, row = pr % 3;
      hist[idx] = cache_in ? cache_in[((size_t)n * 3 + row) * 3 * HD + p * HD + hb * 128 + ch]
                           : from_f32<Tin>(0.f);
    }
    __syncthreads();
  }
  Work cur = work_of(0);
  if (tid == 0 && cur.ok) issue_tma(cur);
  // beta of the current work item's tokens, fetched one item ahead
  float beta_next = (cur.ok && tid < cur.Lc) ? __ldg(beta + (size_t)(cur.t0 + tid) * H + cur.h) : 0.f;
  // kPrepFused: the item's conv weights [3 parts][128 channels][4 taps] (three
  // per thread), fetched one item ahead and stored tap-major at the item start
  float wnext[3] = {0.f, 0.f, 0.f};
  auto fetch_w = [&](const Work &w) {
    if constexpr (kPrepM && kFused) {
#pragma unroll
      for (int m = 0; m < 3; ++m)
        wnext[m] = __ldg(conv_w + (size_t)m * HD * 4 + (size_t)w.h * 512 + tid);
    }
  };
  if (cur.ok) fetch_w(cur);
  // gated modes: the item's exp(A_log[h]) and dt_bias[h][tid % 128], one item ahead
  float ga_next = 1.f, gb_next = 0.f, ga = 1.f, gb = 0.f;
  auto fetch_gate = [&](const Work &w) {
    if constexpr (kGated) {
      ga_next = gate.A_log ? __expf(__ldg(gate.A_log + w.h)) : 1.f;
      gb_next = gate.dt_bias ? __ldg(gate.dt_bias + (size_t)w.h * 128 + (tid & 127)) : 0.f;
    }
  };
  if (cur.ok) fetch_gate(cur);

  uint32_t tma_par = 0, mma_par = 0, inv_par = 0, zero_par = 0;
  bool failed = false;  // a wait ran out: copies or MMAs may still be in flight
  int c = 0;
  for (; cur.ok; ++c) {
    const Work nxt = work_of(c + 1);
    const int t0 = cur.t0, Lc = cur.Lc, h = cur.h;

    // ---- P0: raw tiles of this chunk ---------------------------------------------
    if (!wait_all(bar_tma, tma_par, status)) {
      failed = true;
      break;
    }
    tma_par ^= 1;
    if constexpr (!kFused) {
      // Rows past the chunk's end (the next sequence's tokens, or the zero fill past T)
      // are zeroed once here, so no later phase has to mask them (the fused prologue
      // writes zero rows there itself; the cumsum masks the g tile).
      if (Lc < 64) {
        for (int x = tid; x < (64 - Lc) * 48; x += kThreads) {
          const int row = Lc + x / 48, part = (x % 48) >> 4, c = x & 15;
          st_shared_16(sm + SM_Q + part * 16384, (uint32_t)(row * 256 + c * 16),
                       make_uint4(0u, 0u, 0u, 0u));
        }
      }
    }
    if constexpr (kGated) {
      ga = ga_next;
      gb = gb_next;
      if (nxt.ok) fetch_gate(nxt);
    }
    if constexpr (kPrepM && kFused) {
#pragma unroll
      for (int m = 0; m < 3; ++m) {  // element tid + 512 m of the head's [part][channel][tap]
        const int rem = tid, ch = rem >> 2, tap = rem & 3;
        wconv[(m * 4 + tap) * 128 + ch] = wnext[m];
      }
      if (nxt.ok) fetch_w(nxt);
      if (!has_halo(cur)) {  // sequence start: history from the cache rows or zero
        for (int idx = tid; idx < 9 * 128; idx += kThreads) {
          const int pr = idx >> 7, ch = idx & 127, p = pr / 3, row = pr % 3;
          hist[idx] = cache_in ? cache_in[((size_t)cur.n * 3 + row) * 3 * HD + p * HD + h * 128 + ch]
                               : from_f32<Tin>(0.f);
        }
      }
    }

    // ---- P1: beta, in-chunk cumulative log-decay, per-channel factors, E ------------
    if (tid < 64) {
      beta_s[tid] = beta_next;
      beta_next = (nxt.ok && tid < nxt.Lc) ? __ldg(beta + (size_t)(nxt.t0 + tid) * H + nxt.h) : 0.f;
    }
    if constexpr (kFused) {
      // ---- Pc: prologue in place on the x tiles (fp32 arithmetic) ----------------------
      // thread: 8 channels (c8) of two consecutive rows r0, r0+1 of all three parts;
      // all raw values are read before any tile is overwritten.
      __syncthreads();  // beta_s visible
      // history slots: alternate along the sequence (one pass), or slot 0 in,
      // slot 1 out (each prep item brings its own history)
      const Tin *hcur = hist + (kPrepM ? 0 : (c & 1) * 1152);
      Tin *hnxt = hist + (kPrepM ? 1152 : ((c + 1) & 1) * 1152);
      const int c8 = tid & 15, d0 = c8 * 8, r0 = 2 * (tid >> 4);
      uint4 packed[3][2];      // q, k, v of rows r0, r0+1 as fp16, written after the barrier
      uint4 corr_pk[2];        // beta*v - f16(beta*f16(v)) as bf16
      float2 q32[2][4];        // q in fp32 (channel pairs) until k is known
      float qk[2] = {0.f, 0.f};
      float vmax = 0.f;
      // The same arithmetic as the standalone prologue: channel pairs on the packed fp32
      // instructions, SiLU on the approximate exponential and reciprocal.
#pragma unroll
      for (int p = 0; p < 3; ++p) {
        const uint8_t *tile = sm + (p == 0 ? SM_Q : (p == 1 ? SM_K : SM_V));
        float2 w2[4][4];  // taps x 4 channel pairs
#pragma unroll
        for (int tp = 0; tp < 4; ++tp) {
          const float4 *src = reinterpret_cast<const float4 *>(wconv + (p * 4 + tp) * 128 + d0);
          const float4 lo = src[0], hi = src[1];
          w2[tp][0] = make_float2(lo.x, lo.y);
          w2[tp][1] = make_float2(lo.z, lo.w);
          w2[tp][2] = make_float2(hi.x, hi.y);
          w2[tp][3] = make_float2(hi.z, hi.w);
        }
        // Rows r0-3 .. r0+1 in order, each widened once and applied to both outputs (tap t - q2
        // of output row r0 + q2), so each output sees its taps in the order w0, w1, w2, w3.
        float2 acc[2][4];
#pragma unroll
        for (int t = 0; t < 5; ++t) {
          const int rr = r0 - 3 + t;
          float2 xr[4];
          widen_pairs(*reinterpret_cast<const uint4 *>(
                          rr >= 0 ? tile + rr * 256 + c8 * 16
                                  : reinterpret_cast<const uint8_t *>(hcur + (p * 3 + 3 + rr) * 128) +
                                        c8 * 16),
                      xr, Tin());
#pragma unroll
          for (int q2 = 0; q2 < 2; ++q2) {
            const int tap = t - q2;
            if (tap < 0 || tap > 3) continue;
#pragma unroll
            for (int i = 0; i < 4; ++i)
              acc[q2][i] = tap == 0 ? __fmul2_rn(w2[0][i], xr[i])
                                    : __ffma2_rn(w2[tap][i], xr[i], acc[q2][i]);
          }
        }

#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          float2 y[4];
          float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            y[i] = silu_pair(acc[q2][i]);
            ss2 = __ffma2_rn(y[i], y[i], ss2);
          }
          if (p < 2) {
            float ss = ss2.x + ss2.y;
            ss += __shfl_xor_sync(0xffffffffu, ss, 8);
            ss += __shfl_xor_sync(0xffffffffu, ss, 4);
            ss += __shfl_xor_sync(0xffffffffu, ss, 2);
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            const float sc = rsqrtf(ss + 1e-6f);
#pragma unroll
            for (int i = 0; i < 4; ++i) y[i] = __fmul2_rn(y[i], make_float2(sc, sc));
          }
          if (r0 + q2 >= Lc) {
#pragma unroll
            for (int i = 0; i < 4; ++i) y[i] = make_float2(0.f, 0.f);
          }
          packed[p][q2] = pack_pairs(y, Tact());
          if (p == 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) q32[q2][i] = y[i];
          } else if (p == 1) {
            float2 acc = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 4; ++i) acc = __ffma2_rn(q32[q2][i], y[i], acc);
            qk[q2] = acc.x + acc.y;
          } else {
            const float bt = beta_s[r0 + q2];
            float cr[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
              for (int hf = 0; hf < 2; ++hf) {
                const float ye = hf ? y[i].y : y[i].x;
                vmax = fmaxf(vmax, fabsf(ye));
                const float stored = to_f32(from_f32<Tact>(ye));
                cr[2 * i + hf] = bt * ye - __half2float(__float2half_rn(bt * stored));
              }
            }
            corr_pk[q2] = pack8_bf16(cr);
          }
        }
      }
      if (!(vmax < 32768.f)) report(status, KDA_ERR_DEVICE_RANGE);
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        qk[q2] += __shfl_xor_sync(0xffffffffu, qk[q2], 8);
        qk[q2] += __shfl_xor_sync(0xffffffffu, qk[q2], 4);
        qk[q2] += __shfl_xor_sync(0xffffffffu, qk[q2], 2);
        qk[q2] += __shfl_xor_sync(0xffffffffu, qk[q2], 1);
      }
      // history for the next chunk: raw rows Lc-3 .. Lc-1 of every part
      if (tid < 144) {
        const int p = tid / 48, hr = (tid % 48) >> 4, cc = tid & 15, src = Lc - 3 + hr;
        const uint8_t *tile = sm + (p == 0 ? SM_Q : (p == 1 ? SM_K : SM_V));
        const uint8_t *from = src >= 0 ? tile + src * 256 + cc * 16
                                       : reinterpret_cast<const uint8_t *>(hcur + (p * 3 + 3 + src) * 128) + cc * 16;
        *reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(hnxt + (p * 3 + hr) * 128) + cc * 16) =
            *reinterpret_cast<const uint4 *>(from);
      }
      __syncthreads();  // every raw value has been read
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        const int r = r0 + q2;
        st_shared_16(sm + SM_Q, r * 256 + c8 * 16, packed[0][q2]);
        st_shared_16(sm + SM_K, r * 256 + c8 * 16, packed[1][q2]);
        st_shared_16(sm + SM_V, r * 256 + c8 * 16, packed[2][q2]);
        st_shared_16(reinterpret_cast<uint8_t *>(corr), r * 256 + c8 * 16, corr_pk[q2]);
        if (c8 == 0) pdiag[r] = qk[q2];  // <q_r, k_r> of the fp32 prologue outputs
      }
      if constexpr (kPrepM) {
        if (cache_out && t0 + Lc == cur.eos) {  // the sequence's last three raw inputs
          for (int idx = tid; idx < 9 * 128; idx += kThreads) {
            const int pr = idx >> 7, ch = idx & 127, p = pr / 3, row = pr % 3;
            cache_out[((size_t)cur.n * 3 + row) * 3 * HD + p * HD + h * 128 + ch] = hnxt[idx];
          }
        }
      }
      __syncthreads();
    }
    {  // inclusive cumulative log-decay along the chunk, per key channel, then E in place
      const int d = tid & 127, part = tid >> 7;  // rows [16*part, 16*part + 16)
      float vals[16];
      float acc = 0.f;
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        const int rr = 16 * part + r;
        float gv;
        if constexpr (kGated)  // the 16-bit pre-activation tile, read before E overwrites it
          gv = bounded_gate(to_f32(reinterpret_cast<const Tin *>(Gf)[rr * 128 + d]), ga, gb,
                            gate.lower_bound);
        else
          gv = Gf[rr * 128 + d];
        acc += rr < Lc ? gv : 0.f;
        vals[r] = acc;
      }
      XS[part * 128 + d] = acc;
      __syncthreads();
      // every thread forms the prefix of its 16-row part and the references from the four
      // part totals: c_A = gamma_15, c_B = gamma_47, gamma_63
      const float s0 = XS[d], s1 = XS[128 + d], s2 = XS[256 + d], s3 = XS[384 + d];
      const float s01 = s0 + s1, ca = s0, cb = s01 + s2, cl = cb + s3;
      const float off = part == 0 ? 0.f : (part == 1 ? s0 : (part == 2 ? s01 : cb));
      const float ref = part < 2 ? ca : cb;
#pragma unroll
      for (int r = 0; r < 16; ++r) Gf[(16 * part + r) * 128 + d] = __expf((vals[r] + off) - ref);
      if (tid < 128) {
        feca[d] = __expf(ca);
        fecb[d] = __expf(cb);
        feba[d] = __expf(0.5f * (cb - ca));
        fela[d] = __expf(cl - ca);
        felb[d] = __expf(cl - cb);
        fegc[d] = __expf(cl);
      }
    }
    if constexpr (kPrepM) {
      if (tid == 0) bulk_wait_read_all();  // the previous record's tiles have left shared memory
    }
    __syncthreads();

    // ---- P2: Gram operands (fp32, rounded to tf32) -----------------------------------------
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int p = tid + kThreads * m;
      const int r = p >> 4, c8 = p & 15, d0 = c8 * 8;
      // channel pairs on the packed fp32 instructions (each lane rounded as its scalar op)
      float2 k2[4], q2[4], e2[4];
      widen_pairs(*reinterpret_cast<const uint4 *>(sm + SM_K + r * 256 + c8 * 16), k2, Tact());
      widen_pairs(*reinterpret_cast<const uint4 *>(sm + SM_Q + r * 256 + c8 * 16), q2, Tact());
      ld8_f32_pairs(Gf + r * 128 + d0, e2);
      float a[8], b[8], ki[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {  // rows past the chunk's end are zero
        const float2 ap = __fmul2_rn(k2[i], e2[i]), bp = __fmul2_rn(q2[i], e2[i]);
        a[2 * i] = ap.x; a[2 * i + 1] = ap.y;
        b[2 * i] = bp.x; b[2 * i + 1] = bp.y;
        // E in [e^-80, e^75]: inside the intrinsic's range
        ki[2 * i] = __fdividef(k2[i].x, e2[i].x);
        ki[2 * i + 1] = __fdividef(k2[i].y, e2[i].y);
      }
      st_tf32x8(sm + SM_GA, 128, r, c8, a);
      st_tf32x8(sm + SM_GA, 128, 64 + r, c8, b);
      if (r < 32) {
        st_tf32x8(sm + SM_GB, 96, r, c8, ki);
        float2 hf[4];
        ld8_f32_pairs(feba + d0, hf);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 kp = __fmul2_rn(__fmul2_rn(make_float2(ki[2 * i], ki[2 * i + 1]), hf[i]), hf[i]);
          ki[2 * i] = kp.x; ki[2 * i + 1] = kp.y;
        }
      }
      st_tf32x8(sm + SM_GB, 96, 32 + r, c8, ki);
    }
    fence_async_smem();
    __syncthreads();

    // ---- P3: Gram MMA: one accumulator, 16 K=8 steps --------------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ga = smem_u32(sm + SM_GA), gb = smem_u32(sm + SM_GB);
      constexpr uint32_t id = idesc_tf32(128, 96, false, false);
#pragma unroll
      for (int ks = 0; ks < 16; ++ks)
        mma_tf32(tmem + TM_G, desc_kmajor(ga, 128, ks), desc_kmajor(gb, 96, ks), id, ks > 0);
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, mma_par, status)) {
      failed = true;
      break;
    }
    mma_par ^= 1;
    tc_fence_after();
    if (tid == 0) {  // the Gram's operands are dead: D16, Zm and T32 start at zero
      mbar_arrive_expect_tx(bar_zero, 16384 + 8192);
      bulk_load(sm + SM_D16, g_zero_tiles, 16384, bar_zero);
      bulk_load(sm + SM_T32, g_zero_tiles, 8192, bar_zero);
    }

    // ---- P4: two warp groups ---------------------------------------------------------------
    //   warps 0-7:  P4b (Gram read-out -> A as an fp16 tile and its diagonal 16x16 blocks in
    //               fp32, strict P), P5 (T = (I + A)^-1)
    //   warps 8-15: P4a (the W / Ut / output operands; <q_r, k_r>), which needs neither
    // P4b / P5 work in the S^T and T tiles (dead from the Gram MMA to P6), so P4a can
    // still read E from the g tile.
    bool inv_ok = true;  // warps 0-1: every wait on the inverse's MMA stages completed
    if (tid < kHalf) {
      float *ATd = reinterpret_cast<float *>(sm + SM_ATD);  // [blk][col][row] of A's diagonal blocks
      // ---- P4b / P5 (i): warps 0-1 read only the diagonal 16x16 blocks of A out of TMEM and
      //      run the forward substitution at once, while warps 2-7 read out the whole of A
      //      (fp16 tile, zero on and above the diagonal) and the strict P operand
      //      (the inverse's 16-bit tiles start at zero: a bulk copy of zeros issued when
      //      the Gram MMA completed) -----------------------------------------------------
      // TMEM layout of the Gram: rows 0..31 hold columns i in [0, 32) (reference c_A), rows
      // 32..63 columns i in [0, 64) at TMEM columns 32 + i (reference c_B).
      // P5: T = (I + A)^{-1}, the blocked inverse of a lower triangular matrix.  D =
      // blockdiag of the inverses of the four 16x16 diagonal blocks of I + A (forward
      // substitution, fp32); then
      //   T32 = D - D Z      with Z = A D          (T at the 32x32-block level; only the
      //                                             blocks (1,0) and (3,2) of Z are used)
      //   T   = T32 - T32 Y  with Y = A T32        (only Y's lower-left 32x32 block)
      // The four products are tcgen05 MMAs (M = 128: rows 64..127 are not read) with fp16
      // operands and fp32 accumulation; each piece of T is rounded to fp16 once, for the
      // W / Ut MMAs.  Warps 0-1 run the substitution and the four stages.
      float amax = 0.f;
      if (warp < 2) {
        {  // warp 0: rows 0..31, TMEM columns 0..31; warp 1: rows 32..63, TMEM columns 64..95
          const int r = 32 * warp + lane;
          const float br = beta_s[r];
          float v[32];
          tmem_ld32(tmem + lane_addr + TM_G + 64 * warp, v);
          const bool hi = lane >= 16;  // the row's block starts at loaded column 16 * hi
          const int b = r >> 4, rr = r & 15;
#pragma unroll
          for (int ii = 0; ii < 16; ++ii) {
            const float g = hi ? v[16 + ii] : v[ii];
            if (ii < rr) ATd[(b * 16 + ii) * 16 + rr] = br * g;
          }
        }
        // Each warp's rows hold exactly the two diagonal blocks its own threads invert
        // (warp 0: blocks 0, 1; warp 1: blocks 2, 3), so the warps need not meet here.
        __syncwarp();
        // column jj of D_b, swept row by row; fp16 into D16 and T32
        const int b = tid >> 4, jj = tid & 15, base = 16 * b;
        // Rows in pairs on the packed fp32 instructions: every entry gets the same fma
        // sequence as a row-by-row sweep (so the same values), with half the issues.
        float2 acc2[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) acc2[p] = make_float2(0.f, 0.f);
#pragma unroll
        for (int ii = 0; ii < 16; ++ii) {
          float &aii = (ii & 1) ? acc2[ii >> 1].y : acc2[ii >> 1].x;
          aii = ii == jj ? 1.f : (ii < jj ? 0.f : -aii);
          const float *arow = ATd + (b * 16 + ii) * 16;  // A[base + rr][base + ii]
          if (!(ii & 1)) acc2[ii >> 1].y = fmaf(arow[ii + 1], aii, acc2[ii >> 1].y);
          const float2 a2 = make_float2(aii, aii);
#pragma unroll
          for (int p = (ii >> 1) + 1; p < 8; ++p)
            acc2[p] = __ffma2_rn(reinterpret_cast<const float2 *>(arow)[p], a2, acc2[p]);
        }
        float acc[16];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          acc[2 * p] = acc2[p].x;
          acc[2 * p + 1] = acc2[p].y;
        }
        const uint32_t col = (uint32_t)((base + jj) & 7) * 2;
        if (!mbar_wait(bar_zero, zero_par)) inv_ok = false;  // the zeros landed first
        zero_par ^= 1;
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
          const __half hv = __float2half_rn(acc[rr]);
          amax = fmaxf(amax, fabsf(acc[rr]));
          const uint32_t off = kmaj_off(64, base + rr, (base + jj) >> 3) + col;
          *reinterpret_cast<__half *>(sm + SM_D16 + off) = hv;
          *reinterpret_cast<__half *>(sm + SM_T32 + off) = hv;
        }
      } else {
        // warp 4: A rows 0..31 (quad 0), all four column groups of 8; warp 5: A rows 32..63
        // (quad 1), all four groups of 16; warps 2, 6 (quad 2) and 3, 7 (quad 3): the P rows,
        // column groups {0, 1} and {2, 3}
        const bool isP = quad >= 2;
        const int r = 32 * (quad & 1) + lane;
        const float br = beta_s[r];
        auto emit = [&](int cg, const float (&v)[16]) {
          const int i0s = (quad & 1) ? 16 * cg : 8 * cg;
#pragma unroll
          for (int g8 = 0; g8 < 2; ++g8) {
            if (g8 == 1 && !(quad & 1)) break;
            const int i0 = i0s + 8 * g8;
            float p8[8];
            if (!isP) {
#pragma unroll
              for (int e = 0; e < 8; ++e) p8[e] = i0 + e < r ? br * v[8 * g8 + e] : 0.f;
              st_shared_16(sm + SM_A16, kmaj_off(64, r, i0 >> 3), pack8_f16(p8));
            } else {  // every chunk of the strict P tile this thread reads is written
#pragma unroll
              for (int e = 0; e < 8; ++e) p8[e] = i0 + e < r ? v[8 * g8 + e] : 0.f;
              st_shared_16(sm + SM_POP, kmaj_off(64, r, i0 >> 3), pack8_f16(p8));
            }
          }
        };
        // two column groups per TMEM wait
        auto load_group = [&](int cg, float (&v)[16]) {
          if (quad & 1)
            tmem_ld16_nowait(tmem + lane_addr + TM_G + 32 + 16 * cg, v);
          else
            tmem_ld8_nowait(tmem + lane_addr + TM_G + 8 * cg, *reinterpret_cast<float(*)[8]>(v));
        };
        const int ng = warp >= 4 && warp < 6 ? 2 : 1;  // pairs of column groups
        const int cg0 = warp >= 6 ? 2 : 0;
#pragma unroll 1
        for (int pg = 0; pg < ng; ++pg) {
          const int cga = cg0 + 2 * pg;
          float v[16], w[16];
          load_group(cga, v);
          load_group(cga + 1, w);
          tmem_wait_ld(v, w);
          emit(cga, v);
          emit(cga + 1, w);
        }
        if (warp >= 6) {  // rows 0..31, columns 32..63 of A and P: above the diagonal, not read out
          const int t = tid - 192, rz = t >> 1, cz = 4 + 2 * (t & 1);
#pragma unroll
          for (int z = 0; z < 2; ++z) {
            st_shared_16(sm + SM_POP, kmaj_off(64, rz, cz + z), make_uint4(0u, 0u, 0u, 0u));
            st_shared_16(sm + SM_A16, kmaj_off(64, rz, cz + z), make_uint4(0u, 0u, 0u, 0u));
          }
        }

      }
      fence_async_smem();
      bar_half();
      if (warp < 2) {
        auto inv_mma = [&](uint32_t a_tile, uint32_t b_tile, uint32_t dcol) {
          if (tid == 0 && inv_ok) {
            tc_fence_after();
            constexpr uint32_t id = idesc_fp16(128, 64, false, true);
            const uint32_t a = smem_u32(sm + a_tile), bt = smem_u32(sm + b_tile);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
              mma_bf16(tmem + dcol, desc_kmajor(a, 128, ks), desc_mnmajor(bt, 64, ks), id, ks > 0);
            mma_commit(bar_inv);
          }
        };
        auto inv_wait = [&]() {
          if (!mbar_wait(bar_inv, inv_par)) inv_ok = false;
          inv_par ^= 1;
          tc_fence_after();
        };
        auto pair_sync = [&]() {  // warps 0-1: 16-bit tile writes -> the next MMA
          fence_async_smem();
          tc_fence_before();
          asm volatile("bar.sync 3, 64;" ::: "memory");
        };
        // the in-half off-diagonal blocks: warp 0 holds rows 16..31 (block column 0),
        // warp 1 rows 48..63 (block column 32), in its upper 16 lanes
        auto offdiag16 = [&](uint32_t col, uint32_t tile, float sign) {
          float z[16];
          tmem_ld16(tmem + lane_addr + col + 32 * warp, z);
          if (lane >= 16) {
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                f[e] = sign * z[8 * h8 + e];
                amax = fmaxf(amax, fabsf(f[e]));
              }
              st_shared_16(sm + tile, kmaj_off(64, 32 * warp + lane, 4 * warp + h8), pack8_f16(f));
            }
          }
        };
        // the lower-left 32x32 block: warp 1 (TMEM lanes 32..63), 32 columns
        auto lowerleft = [&](uint32_t col, uint32_t tile, float sign) {
          if (warp == 1) {
            float y[32];
            tmem_ld32(tmem + lane_addr + col, y);
#pragma unroll
            for (int h8 = 0; h8 < 4; ++h8) {
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                f[e] = sign * y[8 * h8 + e];
                amax = fmaxf(amax, fabsf(f[e]));
              }
              st_shared_16(sm + tile, kmaj_off(64, 32 + lane, h8), pack8_f16(f));
            }
          }
        };
        inv_mma(SM_A16, SM_D16, TM_Z);  // Z = A D
        inv_wait();
        offdiag16(TM_Z, SM_ZM, 1.f);
        pair_sync();
        inv_mma(SM_D16, SM_ZM, TM_T2);  // D Z
        inv_wait();
        offdiag16(TM_T2, SM_T32, -1.f);  // T32 = D - D Z
        pair_sync();
        inv_mma(SM_A16, SM_T32, TM_Y);  // A T32
        inv_wait();
        // Y goes over A (dead): the rest of that tile keeps A's finite values, which meet
        // only zeros of T32 in the rows read below
        lowerleft(TM_Y, SM_YM, 1.f);
        pair_sync();
        inv_mma(SM_T32, SM_YM, TM_Z);  // T32 Y (its rows 32..63: T_BR Y)
        inv_wait();
        lowerleft(TM_Z, SM_T32, -1.f);  // T's lower-left block; the T32 tile is now T
      }
      if (!(amax < 32768.f)) report(status, KDA_ERR_DEVICE_RANGE);
    } else {
      // ---- P4a: WY / output operands (the Gram operands are dead) -------------------------
#pragma unroll 2
      for (int m = 0; m < 4; ++m) {
        const int p = (tid - kHalf) + kHalf * m;
        const int r = p >> 4, c8 = p & 15, d0 = c8 * 8;
        const float bt = beta_s[r];
        const float *fec = r < 32 ? feca : fecb;
        const float *fel = r < 32 ? fela : felb;
        // channel pairs on the packed fp32 instructions (each lane rounded as its scalar op)
        float2 k2[4], q2[4], v2[4], e2[4], ec2[4], el2[4];
        widen_pairs(*reinterpret_cast<const uint4 *>(sm + SM_K + r * 256 + c8 * 16), k2, Tact());
        widen_pairs(*reinterpret_cast<const uint4 *>(sm + SM_Q + r * 256 + c8 * 16), q2, Tact());
        widen_pairs(*reinterpret_cast<const uint4 *>(sm + SM_V + r * 256 + c8 * 16), v2, Tact());
        ld8_f32_pairs(Gf + r * 128 + d0, e2);
        ld8_f32_pairs(fec + d0, ec2);
        ld8_f32_pairs(fel + d0, el2);
        float k8[8], q8[8], bkg[8], bv[8], qg[8], kp[8];
        const float2 bt2 = make_float2(bt, bt);
#pragma unroll
        for (int i = 0; i < 4; ++i) {  // zero past the chunk's end
          const float2 g_abs = __fmul2_rn(e2[i], ec2[i]);  // exp(gamma_r) per channel
          const float2 bk = __fmul2_rn(__fmul2_rn(bt2, k2[i]), g_abs);
          const float2 bvp = __fmul2_rn(bt2, v2[i]);
          const float2 qgp = __fmul2_rn(q2[i], g_abs);
          const float2 kpp = __fmul2_rn(make_float2(__fdividef(k2[i].x, e2[i].x),
                                                    __fdividef(k2[i].y, e2[i].y)), el2[i]);
          k8[2 * i] = k2[i].x; k8[2 * i + 1] = k2[i].y;
          q8[2 * i] = q2[i].x; q8[2 * i + 1] = q2[i].y;
          bkg[2 * i] = bk.x; bkg[2 * i + 1] = bk.y;
          bv[2 * i] = bvp.x; bv[2 * i + 1] = bvp.y;
          qg[2 * i] = qgp.x; qg[2 * i + 1] = qgp.y;
          kp[2 * i] = kpp.x; kp[2 * i + 1] = kpp.y;
        }
        const uint4 bv_h = pack8_f16(bv);
        st_shared_16(sm + SM_BKG, mnmaj_off(64, r, c8), pack8_f16(bkg));
        st_shared_16(sm + SM_BV, mnmaj_off(64, r, c8), bv_h);
        st_shared_16(sm + SM_QG, kmaj_off(64, r, c8), pack8_f16(qg));
        st_shared_16(sm + SM_KP, mnmaj_off(64, r, c8), pack8_f16(kp));
        if constexpr (!kFused) {  // <q_r, k_r> in fp32 over the row's 16 lanes
          float acc = 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc = fmaf(q8[e], k8[e], acc);
          acc += __shfl_xor_sync(0xffffffffu, acc, 1);
          acc += __shfl_xor_sync(0xffffffffu, acc, 2);
          acc += __shfl_xor_sync(0xffffffffu, acc, 4);
          acc += __shfl_xor_sync(0xffffffffu, acc, 8);
          if (c8 == 0) pdiag[r] = acc;
        }
        if constexpr (kPrepM && !kFused) {  // fp32 remainder beta v - f16(beta v), kept as bf16
          float cr[8], bvmax = 0.f;
          const __half2 *bh = reinterpret_cast<const __half2 *>(&bv_h);  // f16(beta v), packed above
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            const float2 f = __half22float2(bh[e2]);
            cr[2 * e2] = bv[2 * e2] - f.x;
            cr[2 * e2 + 1] = bv[2 * e2 + 1] - f.y;
            bvmax = fmaxf(bvmax, fmaxf(fabsf(bv[2 * e2]), fabsf(bv[2 * e2 + 1])));
          }
          st_shared_16(reinterpret_cast<uint8_t *>(corr), r * 256 + c8 * 16, pack8_bf16(cr));
          if (!(bvmax < 32768.f)) report(status, KDA_ERR_DEVICE_RANGE);
        }
      }
      if constexpr (kPrepM) {
        // the raw tiles (q, k, v, g; history slot 0) have no reader left in this item:
        // the next item's tiles start now, while the other warps finish the inverse
        bar_second_half();
        if (tid == kHalf && nxt.ok) {
          arm_tma(nxt);
          issue_tma_qk(nxt);
          issue_tma_g(nxt);
          issue_tma_v(nxt);
          issue_tma_halo(nxt);
        }
      }
    }
    fence_async_smem();
    tc_fence_before();
    if (__syncthreads_or(!inv_ok)) {
      if (tid == 0) report(status, KDA_ERR_DEVICE_TIMEOUT);
      failed = true;
      break;
    }
    if constexpr (!kPrepM) {
      if (tid == 0 && nxt.ok) {  // q, k and g are dead (v is read until the U read-out)
        arm_tma(nxt);
        issue_tma_qk(nxt);
        issue_tma_g(nxt);
      }
    }

    // ---- P6: W^T and Ut^T MMAs; meanwhile S^T -> fp16 operand ------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t top = smem_u32(sm + SM_TOP), bkg = smem_u32(sm + SM_BKG);
      const uint32_t bv = smem_u32(sm + SM_BV);
      constexpr uint32_t id = idesc_fp16(128, 64, true, false);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks) {  // two independent chains, interleaved
        mma_bf16(tmem + TM_W, desc_mnmajor(bkg, 64, ks), desc_kmajor(top, 64, ks), id, ks > 0);
        mma_bf16(tmem + TM_U, desc_mnmajor(bv, 64, ks), desc_kmajor(top, 64, ks), id, ks > 0);
      }
      mma_commit(bar_mma);
      if constexpr (kPrepM) {
        // the record's tiles that are complete already leave while the MMAs run: each
        // k-atom of A1 = [W ; Q G] holds the 64 W rows, then the 64 Q G rows
        uint8_t *rp = recs + rec::header_bytes(N) + ((size_t)(cur.ci - win.lo) * H + h) * rec::BYTES;
        bulk_store(rp + rec::A1 + 8192, sm + SM_QG, 8192);
        bulk_store(rp + rec::A1 + 24576, sm + SM_QG + 8192, 8192);
        bulk_store(rp + rec::KP, sm + SM_KP, 16384);
        bulk_store(rp + rec::P, sm + SM_POP, 8192);
        bulk_commit();
      }
    }
    if constexpr (!kPrepM) {
      float amax = 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          f[e] = S[8 * cc + e];
          amax = fmaxf(amax, fabsf(f[e]));
        }
        st_shared_16(sm + SM_ST, kmaj_off(128, j, 4 * grp + cc), pack8_f16(f));
      }
      if (!(amax < 32768.f)) report(status, KDA_ERR_DEVICE_RANGE);
    }
    fence_async_smem();
    if (!wait_all(bar_mma, mma_par, status)) {
      failed = true;
      break;
    }
    mma_par ^= 1;
    tc_fence_after();

    if constexpr (kPrepM) {
      // ---- record: W (K-major, over the dead beta K G tile), Ut + fp32 remainder,
      //      exp(gamma_63), <q_r, k_r>; then the tiles leave by bulk copies -------------
      uint8_t *rp = recs + rec::header_bytes(N) + ((size_t)(cur.ci - win.lo) * H + h) * rec::BYTES;
      {
        float w[16], u[16], cr[16];
        tmem_ld16_nowait(tmem + lane_addr + TM_W + 16 * grp, w);  // W[16 grp + i][j]
        tmem_ld16_nowait(tmem + lane_addr + TM_U + 16 * grp, u);  // Ut[16 grp + i][j]
#pragma unroll
        for (int i = 0; i < 16; ++i) cr[i] = __bfloat162float(corr[(16 * grp + i) * 128 + j]);
        tmem_wait_ld(w, u);
        __half *wt = reinterpret_cast<__half *>(sm + SM_BKG);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          wt[(kmaj_off(64, 16 * grp + i, j >> 3) >> 1) + (j & 7)] = __float2half_rn(w[i]);
        float *ut = reinterpret_cast<float *>(rp + rec::UT);
#pragma unroll
        for (int i = 0; i < 16; ++i) ut[(16 * grp + i) * 128 + j] = u[i] + cr[i];
      }
      if (tid < 128) reinterpret_cast<float *>(rp + rec::GL)[tid] = fegc[tid];
      if (tid < 64) reinterpret_cast<float *>(rp + rec::PD)[tid] = pdiag[tid];
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      if (tid == 0) {  // the W rows of A1's two k-atoms
        bulk_store(rp + rec::A1, sm + SM_BKG, 8192);
        bulk_store(rp + rec::A1 + 16384, sm + SM_BKG + 8192, 8192);
        bulk_commit();
      }
      cur = nxt;
      continue;
    }

    // ---- P7: W^T read-out -> -W operand (MN-major, over beta K G) --------------------------
    {
      float v[16];
      tmem_ld16(tmem + lane_addr + TM_W + 16 * grp, v);
#pragma unroll
      for (int g8 = 0; g8 < 2; ++g8) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = -v[8 * g8 + e];
        st_shared_16(sm + SM_BKG, mnmaj_off(128, j, 2 * grp + g8), pack8_f16(f));
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- P8: U^T = Ut^T - S^T W^T ;  O^T = S^T (Q G)^T -------------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t st = smem_u32(sm + SM_ST), wop = smem_u32(sm + SM_BKG);
      const uint32_t qg = smem_u32(sm + SM_QG);
      constexpr uint32_t idU = idesc_fp16(128, 64, false, true);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_bf16(tmem + TM_U, desc_kmajor(st, 128, ks), desc_mnmajor(wop, 128, ks), idU, 1);
      constexpr uint32_t idO = idesc_fp16(128, 64, false, false);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        mma_bf16(tmem + TM_O, desc_kmajor(st, 128, ks), desc_kmajor(qg, 64, ks), idO, ks > 0);
      mma_commit(bar_mma);
    }
    // ---- P9 (first half, overlapping the MMAs): the fp32 diagonal correction ---------------
    float dcorr[16], bvmax = 0.f;
    {
      const Tact *Vr = reinterpret_cast<const Tact *>(sm + SM_V);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * grp + i;
        const float vv = r < Lc ? to_f32(Vr[r * 128 + j]) : 0.f;
        const float bvv = beta_s[r] * vv;
        if constexpr (kFused)
          dcorr[i] = __bfloat162float(corr[r * 128 + j]);
        else
          dcorr[i] = bvv - __half2float(__float2half_rn(bvv));
        bvmax = fmaxf(bvmax, fabsf(bvv));
      }
    }
    if (!wait_all(bar_mma, mma_par, status)) {
      failed = true;
      break;
    }
    mma_par ^= 1;
    tc_fence_after();

    // ---- P9: U read-out (+ fp32 diagonal), U^T operand -----------------------------------
    float u[16];
    tmem_ld16(tmem + lane_addr + TM_U + 16 * grp, u);
    {
      float amax = bvmax;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        u[i] += dcorr[i];
        amax = fmaxf(amax, fabsf(u[i]));
      }
      if (!(amax < 32768.f)) report(status, KDA_ERR_DEVICE_RANGE);
#pragma unroll
      for (int g8 = 0; g8 < 2; ++g8) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = u[8 * g8 + e];
        st_shared_16(sm + SM_ST, kmaj_off(128, j, 2 * grp + g8), pack8_f16(f));
      }
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && nxt.ok) issue_tma_v(nxt);  // the v tile is dead

    // ---- P10: O^T += U^T P^T ; delta S^T = U^T K' ----------------------------------------
    if (tid == 0) {
      tc_fence_after();
      const uint32_t ut = smem_u32(sm + SM_ST), pop = smem_u32(sm + SM_POP);
      const uint32_t kp = smem_u32(sm + SM_KP);
      constexpr uint32_t idO = idesc_fp16(128, 64, false, false);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16(tmem + TM_O, desc_kmajor(ut, 128, ks), desc_kmajor(pop, 64, ks), idO, 1);
      constexpr uint32_t idS = idesc_fp16(128, 128, false, true);
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16(tmem + TM_S, desc_kmajor(ut, 128, ks), desc_mnmajor(kp, 64, ks), idS, ks > 0);
      mma_commit(bar_mma);
    }
    if (!wait_all(bar_mma, mma_par, status)) {
      failed = true;
      break;
    }
    mma_par ^= 1;
    tc_fence_after();

    // ---- P11: outputs and state update ----------------------------------------------------
    {
      float ov[16], dv[32];
      tmem_ld16_nowait(tmem + lane_addr + TM_O + 16 * grp, ov);
      tmem_ld32_nowait(tmem + lane_addr + TM_S + dk0, dv);
      tmem_wait_ld(ov, dv);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = 16 * grp + i;
        if (r < Lc) o[((size_t)(t0 + r) * H + h) * 128 + j] = scale * fmaf(pdiag[r], u[i], ov[i]);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) S[i] = fmaf(S[i], fegc[dk0 + i], dv[i]);
    }
    tc_fence_before();
    __syncthreads();
    cur = nxt;
  }

  if constexpr (kMode == kFusedMode) {
    if (cache_out) {  // the last three raw inputs of the sequence (oldest first)
      const Tin *hfin = hist + (nchunks & 1) * 1152;
      for (int idx = tid; idx < 9 * 128; idx += kThreads) {
        const int pr = idx >> 7, ch = idx & 127, p = pr / 3, row = pr % 3;
        cache_out[((size_t)n * 3 + row) * 3 * HD + p * HD + hb * 128 + ch] = hfin[idx];
      }
    }
  }
  if constexpr (kPrepM) {
    if (tid == 0) bulk_wait_all();
  }
  if (failed && tid == 0) {  // let in-flight tile loads and MMAs land first
    drain(bar_tma);
    drain(bar_mma);
    drain(bar_inv);
    drain(bar_zero);
  }
  if (sN && !kPrepM && !failed) {
    float *dst = sN + (((size_t)n * H + hb) * 128 + j) * 128 + dk0;
#pragma unroll
    for (int x = 0; x < 32; x += 4)
      *reinterpret_cast<float4 *>(dst + x) = make_float4(S[x], S[x + 1], S[x + 2], S[x + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, TM_COLS);
}

// 3-D map over a [T, H, 128] tensor: box = `rows` tokens x 1 head x 128 channels.
bool make_map(CUtensorMap *m, const void *ptr, CUtensorMapDataType dt, int esz, int H, int T,
              unsigned rows = 64) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)H, (cuuint64_t)T};
  cuuint64_t strides[2] = {(cuuint64_t)128 * esz, (cuuint64_t)H * 128 * esz};
  cuuint32_t box[3] = {128, 1, rows};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, dt, 3, const_cast<void *>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_chunk_tc(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, float scale, const float *s0, const int32_t *cu,
                            int N, int T, int H, kda_dtype dt, float *o, float *sN, int *status,
                            cudaStream_t s) {
  const CUtensorMapDataType act =
      dt == KDA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tq, tk, tv, tg;
  if (!make_map(&tq, q, act, 2, H, T) || !make_map(&tk, k, act, 2, H, T) ||
      !make_map(&tv, v, act, 2, H, T) ||
      !make_map(&tg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, T))
    return cudaErrorInvalidValue;
  const long long blocks = (long long)N * H;
  if (blocks >= (1LL << 31)) return cudaErrorInvalidValue;
  if (dt == KDA_BF16) {
    auto kern = chunk_tc_kernel<__nv_bfloat16, kSingle>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SM_ALLOC);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)blocks, kThreads, SM_ALLOC, s>>>(tq, tk, tv, tg, beta, scale, s0, cu, T, H, o,
                                                      sN, status, nullptr, nullptr, nullptr,
                                                      nullptr, nullptr, N, GateArgs{},
                                                      ChunkWindow{});
  } else {
    auto kern = chunk_tc_kernel<__half, kSingle>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SM_ALLOC);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)blocks, kThreads, SM_ALLOC, s>>>(tq, tk, tv, tg, beta, scale, s0, cu, T, H, o,
                                                      sN, status, nullptr, nullptr, nullptr,
                                                      nullptr, nullptr, N, GateArgs{},
                                                      ChunkWindow{});
  }
  return cudaGetLastError();
}

namespace {
// Grid of a persistent prep launch: one CTA per SM (each takes a whole SM's
// shared memory), at most one per work item.
cudaError_t prep_grid(int N, int T, int H, const ChunkWindow &win, unsigned *grid) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long chunks =
      std::min<long long>(rec::chunk_capacity(N, T), (long long)win.hi - win.lo);
  *grid = (unsigned)std::max<long long>(1, std::min<long long>(chunks * H, sms));
  return cudaSuccess;
}

template <typename Tin, int kMode>
cudaError_t launch_prep_typed(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv,
                              const CUtensorMap &tg, const float *beta, const int32_t *cu, int N,
                              int T, int H, uint8_t *ws, const GateArgs &gate, int *status,
                              cudaStream_t s, const ChunkWindow &win) {
  auto kern = chunk_tc_kernel<Tin, kMode>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SM_ALLOC_PREP);
  if (e != cudaSuccess) return e;
  unsigned grid = 0;
  if ((e = prep_grid(N, T, H, win, &grid)) != cudaSuccess) return e;
  kern<<<grid, kThreads, SM_ALLOC_PREP, s>>>(tq, tk, tv, tg, beta, 1.f, nullptr, cu, T, H, nullptr,
                                             nullptr, status, nullptr, nullptr, nullptr, ws,
                                             reinterpret_cast<const int32_t *>(ws), N, gate, win);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_chunk_prep(const void *q, const void *k, const void *v, const void *g,
                              const float *beta, const int32_t *cu, int N, int T, int H,
                              kda_dtype dt, void *ws, const float *A_log, const float *dt_bias,
                              float lower_bound, bool gated, int *status, cudaStream_t s,
                              const ChunkWindow &win) {
  const CUtensorMapDataType act =
      dt == KDA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  CUtensorMap tq, tk, tv, tg;
  if (!make_map(&tq, q, act, 2, H, T) || !make_map(&tk, k, act, 2, H, T) ||
      !make_map(&tv, v, act, 2, H, T) ||
      !(gated ? make_map(&tg, g, act, 2, H, T)
              : make_map(&tg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, T)))
    return cudaErrorInvalidValue;
  uint8_t *w = static_cast<uint8_t *>(ws);
  const GateArgs gate{A_log, dt_bias, lower_bound};
  if (dt == KDA_BF16)
    return gated ? launch_prep_typed<__nv_bfloat16, kPrepGated>(tq, tk, tv, tg, beta, cu, N, T, H,
                                                                 w, gate, status, s, win)
                 : launch_prep_typed<__nv_bfloat16, kPrep>(tq, tk, tv, tg, beta, cu, N, T, H, w,
                                                            gate, status, s, win);
  return gated ? launch_prep_typed<__half, kPrepGated>(tq, tk, tv, tg, beta, cu, N, T, H, w, gate,
                                                        status, s, win)
               : launch_prep_typed<__half, kPrep>(tq, tk, tv, tg, beta, cu, N, T, H, w, gate,
                                                   status, s, win);
}

namespace {
template <typename Tin>
cudaError_t launch_fused_typed(const void *x, const float *conv_w, const void *cache_in,
                               void *cache_out, const float *g, const float *beta, float scale,
                               const float *s0, const int32_t *cu, int N, int T, int H,
                               CUtensorMapDataType act, float *o, float *sN, int *status,
                               cudaStream_t s) {
  CUtensorMap tx, tg;
  if (!make_map(&tx, x, act, 2, 3 * H, T) ||
      !make_map(&tg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, T))
    return cudaErrorInvalidValue;
  const long long blocks = (long long)N * H;
  if (blocks >= (1LL << 31)) return cudaErrorInvalidValue;
  auto kern = chunk_tc_kernel<Tin, kFusedMode>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SM_ALLOC_FUSED);
  if (e != cudaSuccess) return e;
  kern<<<(unsigned)blocks, kThreads, SM_ALLOC_FUSED, s>>>(
      tx, tx, tx, tg, beta, scale, s0, cu, T, H, o, sN, status, conv_w,
      static_cast<const Tin *>(cache_in), static_cast<Tin *>(cache_out), nullptr, nullptr, N,
      GateArgs{}, ChunkWindow{});
  return cudaGetLastError();
}
}  // namespace

namespace {
template <typename Tin, int kMode>
cudaError_t launch_prep_fused_typed(const void *x, const float *conv_w, const void *cache_in,
                                    void *cache_out, const void *g, const float *beta,
                                    const int32_t *cu, int N, int T, int H,
                                    CUtensorMapDataType act, void *ws, const GateArgs &gate,
                                    int *status, cudaStream_t s, const ChunkWindow &win) {
  constexpr bool kGatedM = kMode == kPrepFusedGated;
  CUtensorMap tx, th, tg;
  if (!make_map(&tx, x, act, 2, 3 * H, T) || !make_map(&th, x, act, 2, 3 * H, T, 3) ||
      !(kGatedM ? make_map(&tg, g, act, 2, H, T)
                : make_map(&tg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, T)))
    return cudaErrorInvalidValue;
  auto kern = chunk_tc_kernel<Tin, kMode>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)SM_ALLOC_FUSED);
  if (e != cudaSuccess) return e;
  unsigned grid = 0;
  if ((e = prep_grid(N, T, H, win, &grid)) != cudaSuccess) return e;
  uint8_t *w = static_cast<uint8_t *>(ws);
  kern<<<grid, kThreads, SM_ALLOC_FUSED, s>>>(
      tx, th, tx, tg, beta, 1.f, nullptr, cu, T, H, nullptr, nullptr, status, conv_w,
      static_cast<const Tin *>(cache_in), static_cast<Tin *>(cache_out), w,
      reinterpret_cast<const int32_t *>(w), N, gate, win);
  return cudaGetLastError();
}
}  // namespace

cudaError_t launch_prologue_chunk_prep(const void *x, const float *conv_w, const void *cache_in,
                                       void *cache_out, const void *g, const float *beta,
                                       const int32_t *cu, int N, int T, int H, kda_dtype dt,
                                       void *ws, const float *A_log, const float *dt_bias,
                                       float lower_bound, bool gated, int *status,
                                       cudaStream_t s, const ChunkWindow &win) {
  const GateArgs gate{A_log, dt_bias, lower_bound};
  if (dt == KDA_BF16) {
    constexpr auto act = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    return gated ? launch_prep_fused_typed<__nv_bfloat16, kPrepFusedGated>(
                       x, conv_w, cache_in, cache_out, g, beta, cu, N, T, H, act, ws, gate, status, s, win)
                 : launch_prep_fused_typed<__nv_bfloat16, kPrepFused>(
                       x, conv_w, cache_in, cache_out, g, beta, cu, N, T, H, act, ws, gate, status, s, win);
  }
  constexpr auto act = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  return gated ? launch_prep_fused_typed<__half, kPrepFusedGated>(
                     x, conv_w, cache_in, cache_out, g, beta, cu, N, T, H, act, ws, gate, status, s, win)
               : launch_prep_fused_typed<__half, kPrepFused>(
                     x, conv_w, cache_in, cache_out, g, beta, cu, N, T, H, act, ws, gate, status, s, win);
}

cudaError_t launch_prologue_chunk_tc(const void *x, const float *conv_w, const void *cache_in,
                                     void *cache_out, const float *g, const float *beta,
                                     float scale, const float *s0, const int32_t *cu, int N,
                                     int T, int H, kda_dtype dt, float *o, float *sN,
                                     int *status, cudaStream_t s) {
  if (dt == KDA_BF16)
    return launch_fused_typed<__nv_bfloat16>(x, conv_w, cache_in, cache_out, g, beta, scale, s0,
                                             cu, N, T, H, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, o, sN,
                                             status, s);
  return launch_fused_typed<__half>(x, conv_w, cache_in, cache_out, g, beta, scale, s0, cu, N, T,
                                    H, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, o, sN, status, s);
}

}  // namespace kda
