// One CSA decode step in one cooperative launch: append, index, select,
// attend.
//
// Pages: jiwasawa.github.io DeepSeek-V4 article, section "Compressed Sparse
// Attention (CSA)" -- the indexer scores every compressed entry, a top-k
// selector keeps the best, and shared key-value MQA runs over them; section
// "Heavily Compressed Attention (HCA)" -- the sliding-window branch over the
// latest tokens; "DeepSeek V4とOpenCode" (hazakura.dev), "衝撃1：CSA + HCA" --
// 4 tokens per entry, an FP4 Lightning Indexer, a 128-token window, 1M-token
// contexts; "DeepSeek V4 Flash" (studioglobal.ai), "アテンションのブレイクスルー"
// -- softmax-gated pooling, top 512 blocks per query.
//
// A decode step with separate launches is a chain of short dependent phases
// (pool the new tokens; stream every indexer key; find the row's threshold;
// rank the survivors; gather the selected rows; attend; merge item splits),
// each of which leaves most of the GPU idle while it waits on memory.  Here
// one CTA per SM runs them all, separated by bounded grid barriers:
//
//   A0  append: the CTA that owns the end of each sequence pools the step's
//       new tokens into entries (softmax-gated, E4M3 + scale) and stores the
//       tokens themselves in the window ring; the new entries' indexer keys
//       are copied into the key cache and scored directly from the input.
//   A1  scan: per_row CTAs per sequence each stream a contiguous range of
//       indexer keys through a 4-stage ring of TMA loads; per 1,024 keys
//       eight kind::mxf4 MMAs give exact q.k sums in TMEM (two buffers, the
//       MMAs of batch b overlap the epilogue of b - 1); integer scores stay in
//       shared memory and are counted in a 4,096-bin histogram of score >> 8.
//       The attention's Q tile is loaded by TMA as soon as the key ring is
//       free, and the unit's window rows are prefetched into L2.
//   A2  select: row histograms in the workspace give the threshold bin; the
//       keys at or above it become candidates (unique 64-bit keys score,
//       ~index, their cache rows prefetched into L2), with an exact
//       refinement when ties flood the bin; every candidate is ranked by
//       counting the larger ones (the row's CTAs share the candidates), and
//       the K best are written in rank order.
//   B   attend: every CTA becomes one attention unit (sequence, quarter of
//       D, item split) and runs the tensor-core MQA over its chunks of the
//       sequence's item list (selected entries, then window tokens).  Q lives
//       in TMEM as the A operand of S = Q K^T (M = 128 heads, N = 128 items,
//       K = 512), so the tensor core streams only the item tile from shared
//       memory; E4M3 rows are converted exactly to bf16; the softmax (two
//       threads per head, 64 items each, one pass over S, lazy rescaling)
//       writes P = p * item scale straight into TMEM over S, the A operand
//       of O += P V (N = 128, the unit's quarter of D).
//       Item splits write unnormalised partials and count themselves done
//       per (sequence, quarter); each unit then merges its share of the heads.
//
// Grid barriers count arrivals on a 64-bit word that only ever grows by one
// per CTA and barrier, and the per-(sequence, quarter) merge counters only
// grow too; the per-call selection counters are cleared by each call after
// their last use.  So a workspace needs zero filling once, before its first
// use, and again only when the shape changes or a call timed out.
// Every wait is bounded by wall time; on expiry the kernel sets the status
// word's timeout bit, stops waiting, and unwinds.
#include "common.cuh"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int kThreads = 288;          // warps 0-7 work, warp 8 issues TMA and MMA
constexpr int kWork = 256;
constexpr int kBins = 4096;
constexpr int kCandCap = 2048;
constexpr int kLocalCap = 8192;        // indexer keys one CTA scores
constexpr int kStages = 4;
constexpr int kTileKeys = 128;
constexpr int kBatchTiles = 8;
constexpr int kBatchKeys = kTileKeys * kBatchTiles;
constexpr uint32_t kBatchBytes = kBatchKeys * 32;
constexpr unsigned long long kWaitNs = 2000000000ull;

constexpr int TH = 128;                // attention heads = MMA M
constexpr int TD = 512;                // entry width
constexpr int CH = 128;                // items per chunk = QK MMA N
constexpr int DQ = 128;                // output columns per unit (a quarter of D) = PV MMA N
constexpr int kMaxSelLocal = 2304;     // selected items one unit may hold
constexpr int kMaxNew = 16;            // appended tokens per step
constexpr int kMaxSplits = 64;         // item splits per (sequence, quarter) at most
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;

// shared memory: the scan/select phase and the attention phase overlay
constexpr uint32_t A_KBUF = 0;                                  // key ring
constexpr uint32_t A_SC = A_KBUF + kStages * kBatchBytes;       // u32 scores; later candidate keys
constexpr uint32_t A_HIST = A_SC + kLocalCap * 4;               // u32 [4096]
constexpr uint32_t A_QI = A_HIST + kBins * 4;                   // indexer queries (MMA B operand)
constexpr uint32_t A_END = A_QI + 256;
// Q is staged at 0 (TMA: [32 d-blocks][128 heads][16 d] bf16) and moved into
// TMEM; the region then holds the item tile [128 items][512 d] bf16.
constexpr uint32_t B_Q = 0;
constexpr uint32_t B_KV = 0;
constexpr uint32_t KV_BYTES = CH * TD * 2;                      // 128 KiB
constexpr uint32_t B_SEL = B_KV + KV_BYTES;                     // int32 [kMaxSelLocal]
constexpr uint32_t B_SCALE = B_SEL + kMaxSelLocal * 4;          // fp32 [128] item scales
constexpr uint32_t B_MX = B_SCALE + CH * 4;                     // fp32 [2][128] per-half maxima / sums
constexpr uint32_t B_END = B_MX + 2 * TH * 4;
constexpr uint32_t OFF_BAR = ((A_END > B_END ? A_END : B_END) + 127u) & ~127u;
constexpr int NBAR = 15;
constexpr uint32_t OFF_MISC = (OFF_BAR + NBAR * 8 + 127u) & ~127u;

enum { A_FULL = 0, A_MDONE = 4, BAR_KV_FULL = 6, BAR_KV_FREE = 7, BAR_S_FULL = 8, BAR_P_FULL = 9,
       BAR_PV_DONE = 10, BAR_FIN = 11, BAR_Q = 12, BAR_QT = 13, BAR_MX = 14 };

constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TCOL_SFA = 128, TCOL_SFB = 132;   // scan: accumulators at 0..127
// attention: Q (bf16, the A operand of S = Q K^T), S of the current chunk,
// the unit's quarter of O
constexpr uint32_t TCOL_Q = 0, TCOL_S = 256, TCOL_O = 384;

struct Misc {
  unsigned long long base_ctr;  // grid-barrier counter at the start of this call
  uint32_t nbar;                // grid barriers this CTA has arrived at
  uint32_t pair_base;           // this unit's pair counter at the start of this call
  uint32_t cbase_a, cbase_b;    // candidate counters of the scan row and the unit's row at the start
  uint32_t token;               // this call's token (never 0)
  uint32_t tmem;
  int abort;
  int bin;
  uint32_t above;
  uint32_t tstar, take, base;
  uint32_t warp_tot[8];
  uint32_t knew_score[kMaxNew];
  float red[8];
};
constexpr uint32_t SMEM_BYTES = OFF_MISC + ((sizeof(Misc) + 127u) & ~127u);
static_assert(SMEM_BYTES <= 232448, "shared memory");

struct Ws {
  unsigned long long *bar;   // grid-barrier arrivals (only grows; a multiple of the grid between calls)
  uint32_t *zone;     // start of the per-call counters below (zeroed by the kernel)
  uint32_t zone_u4;   // their size in 16-byte words
  uint32_t *hist;     // [B][4096]
  uint32_t *hist2;    // [B][256]
  uint32_t *tiecnt;   // [B * per_row]
  uint32_t zone_hist_u4;  // the histograms' part of the zone, in 16-byte words
  uint32_t *ccount;   // [B] candidates listed (only grows; each call reads its base first)
  uint32_t *flag;     // the call's token when some row needs the tie refinement
  uint32_t *pair_done;  // [B * 4] item splits of (sequence, quarter) whose partials are written (only grows)
  uint64_t *cand;     // [B][kCandCap]
  float4 *ws_o;       // [B * 4 * S][32 column quads][128 heads] partial outputs
  float2 *ws_ml;      // [B * 4 * S][128]                      (max, sum) in log2 units
};

struct StepArgs {
  const float *x_new, *z_new;   // [B][n_new][512]
  const uint8_t *kI_new;        // [B][n_new / m][32] or null
  const int32_t *q_pos;         // [B]
  const uint8_t *qI;            // [B][HI][32]
  const float *w;               // [B][HI]
  uint8_t *codes;
  float *scales;
  uint8_t *kI;
  uint8_t *wcodes;
  float *wscales;
  int B, m, K, W, n_entries, win_cap, n_new;
  int64_t entry_cap;
  float sm_scale;
  int per_row;                  // scan CTAs per sequence
  int S, cps;                   // item splits per (sequence, quarter) and chunks per split
  int32_t *idx_out;
  float *score_out;
  __nv_bfloat16 *out;
  float *lse;
  Ws ws;
  unsigned *status;
};

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// barrier 1 over the 256 working threads (warp 8 does not take part)
__device__ __forceinline__ void wsync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ uint64_t make_key(uint32_t score, uint32_t idx) {
  return ((uint64_t)score << 32) | (uint64_t)(0xFFFFFFFFu - idx);
}

__device__ __forceinline__ int e2m1x2(uint32_t code) {   // 2 * value of one E2M1 code
  const int mag = (int)((0xC8643210u >> (4 * (code & 7))) & 0xF);
  return (code & 8) ? -mag : mag;
}

// ---------------------------------------------------------------------------
// grid barrier (thread 0 of each CTA)
// ---------------------------------------------------------------------------
// One 64-bit counter that only grows: every CTA adds 1 per barrier, so with
// G CTAs and every earlier call complete it holds a multiple of G when a call
// starts.  Each CTA reads that base before its first arrival; barrier k is
// complete once the counter reaches base + k * G.  Nothing is ever reset.
// The counter's value at the start of the call, rounded down to a multiple of
// G.  Read by each CTA before its first arrival (barrier 0 cannot complete
// before that arrival, so the value lies in [base, base + G)).
__device__ __forceinline__ void gb_read_base(const unsigned long long *ctr, uint32_t G, Misc *misc) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ctr) : "memory");
  misc->base_ctr = v - v % G;
  misc->nbar = 0;
}

__device__ __forceinline__ void gb_arrive(unsigned long long *ctr, Misc *misc) {
  __threadfence();
  asm volatile("red.release.gpu.global.add.u64 [%0], 1;" ::"l"(ctr) : "memory");
  misc->nbar += 1;
}

// wait for the barrier of the last arrival
__device__ __forceinline__ void gb_wait(const unsigned long long *ctr, uint32_t G, Misc *misc, unsigned *status) {
  if (misc->abort) return;
  const unsigned long long target = misc->base_ctr + (unsigned long long)misc->nbar * G;
  uint64_t t0 = 0;
  uint32_t n = 0;
  unsigned long long v;
  for (;;) {
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(ctr) : "memory");
    if (v >= target) break;
    if ((++n & 63u) == 0) {
      const uint64_t now = gtimer();
      if (t0 == 0) t0 = now;
      else if (now - t0 > kWaitNs) {
        misc->abort = 1;
        raise_status(status, STATUS_TIMEOUT);
        break;
      }
    }
  }
  __threadfence();
}

__device__ __forceinline__ void grid_sync(unsigned long long *ctr, uint32_t G, Misc *misc, unsigned *status) {
  tc::fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0) {
    gb_arrive(ctr, misc);
    gb_wait(ctr, G, misc, status);
  }
  __syncthreads();
  tc::fence_after_sync();
}

// bounded wait on an mbarrier phase; false (and the CTA marked) on expiry
__device__ __forceinline__ bool bwait(uint64_t *b, uint32_t parity, Misc *misc, unsigned *status) {
  if (tc::mbar_try_wait(b, parity)) return true;
  const uint64_t t0 = gtimer();
  uint32_t n = 0;
  while (!tc::mbar_try_wait(b, parity)) {
    if ((++n & 255u) == 0) {
      if (*(volatile int *)&misc->abort) return false;
      if (gtimer() - t0 > kWaitNs) {
        *(volatile int *)&misc->abort = 1;
        raise_status(status, STATUS_TIMEOUT);
        return false;
      }
    }
  }
  return true;
}

// ---------------------------------------------------------------------------
// selection helpers over the 256 working threads
// ---------------------------------------------------------------------------
// Bin where the count of keys in this-or-higher bins first reaches `need`,
// and the count strictly above it (16 bins per thread).
__device__ void find_bin_w(const uint32_t *hist, uint32_t need, Misc *misc) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hi_bin = kBins - 1 - 16 * tid;
  uint32_t c[16], local = 0;
  const uint4 *h4 = reinterpret_cast<const uint4 *>(hist + hi_bin - 15);
#pragma unroll
  for (int k4 = 0; k4 < 4; ++k4) {
    const uint4 v = h4[k4];
    c[15 - 4 * k4] = v.x;
    c[14 - 4 * k4] = v.y;
    c[13 - 4 * k4] = v.z;
    c[12 - 4 * k4] = v.w;
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) local += c[k];
  uint32_t v = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += x;
  }
  if (lane == 31) misc->warp_tot[warp] = v;
  wsync();
  uint32_t before = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) before += (k < warp) ? misc->warp_tot[k] : 0u;
  const uint32_t incl = v + before;
  const uint32_t excl = incl - local;
  if (excl < need && incl >= need) {
    uint32_t run = excl;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if (run + c[k] >= need) { misc->bin = hi_bin - k; misc->above = run; break; }
      run += c[k];
    }
  }
  wsync();
}

// Exclusive prefix of v over the 256 working threads, and the total.
__device__ __forceinline__ uint32_t block_scan_w(uint32_t v, Misc *misc, uint32_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  wsync();
  if (lane == 31) misc->warp_tot[warp] = x;
  wsync();
  uint32_t before = 0, tot = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const uint32_t t = misc->warp_tot[k];
    before += (k < warp) ? t : 0u;
    tot += t;
  }
  *total = tot;
  return before + x - v;
}

// Warp-aggregated append of `key` (when take) to a global list with counter.
__device__ __forceinline__ void list_append(bool take, uint64_t key, uint32_t *count, uint32_t cbase, uint64_t *list) {
  const int lane = threadIdx.x & 31;
  const unsigned msk = __ballot_sync(0xffffffffu, take);
  if (!msk) return;
  const int leader = __ffs(msk) - 1;
  uint32_t base = 0;
  if (lane == leader) base = atomicAdd(count, (uint32_t)__popc(msk));
  base = __shfl_sync(0xffffffffu, base, leader);
  if (take) {
    const uint32_t pos = base - cbase + __popc(msk & ((1u << lane) - 1u));
    if (pos < (uint32_t)kCandCap) list[pos] = key;
  }
}

// ---------------------------------------------------------------------------
// pooling of the step's new tokens (128 threads, 4 channels each)
// ---------------------------------------------------------------------------
// Per-channel online softmax over a block's tokens: the same update order
// and rounding as the library's pooling kernel, so that an entry appended
// here is bit-identical to one pooled by csa_compress.
struct Pool4 {
  float mx[4], l[4], acc[4];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int c = 0; c < 4; ++c) { mx[c] = -INFINITY; l[c] = 0.f; acc[c] = 0.f; }
  }
  __device__ __forceinline__ void push(const float4 &xv, const float4 &zv) {
    const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
    const float zs[4] = {zv.x, zv.y, zv.z, zv.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if (zs[c] > mx[c]) {
        const float r = expf(mx[c] - zs[c]);
        l[c] = fmaf(l[c], r, 1.f);
        acc[c] = fmaf(acc[c], r, xs[c]);
        mx[c] = zs[c];
      } else {
        const float p = expf(zs[c] - mx[c]);
        l[c] += p;
        acc[c] = fmaf(p, xs[c], acc[c]);
      }
    }
  }
};

// amax over 128 threads (4 warps starting at warp w0) through misc->red[w0..]
__device__ __forceinline__ float amax128(float a, Misc *misc, int w0, int barrier_id) {
  const int warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) misc->red[warp] = a;
  asm volatile("bar.sync %0, 128;" ::"r"(barrier_id) : "memory");
  const float r = fmaxf(fmaxf(misc->red[w0], misc->red[w0 + 1]), fmaxf(misc->red[w0 + 2], misc->red[w0 + 3]));
  asm volatile("bar.sync %0, 128;" ::"r"(barrier_id) : "memory");
  return r;
}

// E4M3 word of 4 channels with entry scale s (s = amax / 448, 1 for a zero entry)
__device__ __forceinline__ uint32_t quant4(const float (&C)[4], float s) {
  uint32_t word = 0;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float r = __fdiv_rn(C[c], s);
    word |= (uint32_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3) << (8 * c);
  }
  return word;
}

// ---------------------------------------------------------------------------
// attention helpers
// ---------------------------------------------------------------------------
// Core-matrix layout (8 rows x 16 B) of the item tile KV [128 items][512 d]:
// g = d / 8, g-stride 2 KiB, item-group stride 128 B.
__device__ __forceinline__ uint32_t kv_off(int i, int g) { return g * 2048 + (i >> 3) * 128 + (i & 7) * 16; }


__device__ __forceinline__ uint4 ldcg16(const void *p) { return __ldcg(reinterpret_cast<const uint4 *>(p)); }

// The same decision in every lane of the warp (after a bounded wait that may
// give up in some lanes only), so that warp-collective TMEM loads and stores
// and votes that follow are never reached by part of a warp.
__device__ __forceinline__ bool uniform(bool v) { return __all_sync(0xffffffffu, v); }

// 2^x (hardware approximation, a few ulp; flushes results below 2^-126 to 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Combines the S item splits' partials of heads [h0, h0 + nh) of one
// (sequence, quarter).  One task per (head, column quad); each loads its
// splits' (max, sum) and partial quad 8 at a time, all in flight, and folds
// them into a running maximum, sum and accumulator.
//   src_o: [S][32 quads][128 heads] float4,  src_ml: [S][128 heads],
//   dst: the sequence's output at this quarter's first column,
//   lse: the sequence's log-sum-exp row (or null).
__device__ __forceinline__ void merge_quarter(const float4 *src_o, const float2 *src_ml, int S, int h0, int nh,
                                              __nv_bfloat16 *dst, float *lse) {
  const int ntask = nh * (DQ / 4);
  for (int t = threadIdx.x; t < ntask; t += kThreads) {
    const int h = h0 + t / (DQ / 4), c = t % (DQ / 4);
    float M = -INFINITY, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < S; j0 += 8) {
      float2 ml[8];
      float4 v[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const int j = j0 + jj;
        ml[jj] = j < S ? __ldcg(src_ml + (int64_t)j * TH + h) : make_float2(-INFINITY, 0.f);
        v[jj] = j < S ? __ldcg(src_o + ((int64_t)j * (DQ / 4) + c) * TH + h) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float Mg = M;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj)
        if (ml[jj].y > 0.f) Mg = fmaxf(Mg, ml[jj].x);
      if (Mg == -INFINITY) continue;
      const float f = M == -INFINITY ? 0.f : exp2f(M - Mg);
      acc.x *= f; acc.y *= f; acc.z *= f; acc.w *= f;
      L *= f;
      M = Mg;
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        const float wj = ml[jj].y > 0.f ? exp2f(ml[jj].x - M) : 0.f;
        L += wj * ml[jj].y;
        acc.x += wj * v[jj].x; acc.y += wj * v[jj].y; acc.z += wj * v[jj].z; acc.w += wj * v[jj].w;
      }
    }
    const float il = 1.f / L;
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * il, acc.y * il);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * il, acc.w * il);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t *>(&lo);
    pk.y = *reinterpret_cast<const uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(dst + (int64_t)h * TD + c * 4) = pk;
    if (lse && c == 0) lse[h] = (M + log2f(L)) * 0.6931471805599453f;
  }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
template <int HI>
__global__ void __launch_bounds__(kThreads, 1)
decode_step_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap qmap,
                   const StepArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  Misc *misc = reinterpret_cast<Misc *>(smem + OFF_MISC);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t G = gridDim.x;
  const Ws &ws = a.ws;

  // ---------------------------------------------------------------- phase A set-up
  const int rowA = blockIdx.x / a.per_row, part = blockIdx.x - rowA * a.per_row;
  const bool scanA = rowA < a.B;
  const int64_t tA = scanA ? (int64_t)a.q_pos[rowA] : -1;
  const int nvisA = tA < 0 ? 0 : (int)min((tA + 1) / a.m, (int64_t)a.n_entries);
  // contiguous key ranges; the last part, which also pools the new tokens,
  // takes half a share: part p starts at 2 p nvis / (2 per_row - 1)
  const int64_t den = 2 * (int64_t)a.per_row - 1;
  const int s0 = (int)((2 * (int64_t)part * nvisA) / den);
  const int s1 = part == a.per_row - 1 ? nvisA : (int)((2 * (int64_t)(part + 1) * nvisA) / den);
  const int n = s1 - s0;
  const int nb = (n + kBatchKeys - 1) / kBatchKeys;
  const int ybase = (int)((int64_t)rowA * a.entry_cap + s0);
  // the step's new entries [e0, e1): whole blocks ending at the query token
  const int nbn = a.n_new / a.m;
  const int64_t e1 = tA < 0 ? 0 : (tA + 1) / a.m;
  const int64_t e0 = e1 - nbn;
  const bool append_ok = tA >= 0 && (tA + 1) % a.m == 0 && e0 >= 0 && e1 <= a.entry_cap && tA + 1 >= a.n_new;
  if (scanA && part == 0 && tid == 0 && !append_ok) raise_status(a.status, STATUS_BAD_POSITION);

  // the attention unit this CTA runs after the selection: (sequence, quarter
  // of D, item split)
  const int S = a.S;
  const int units = a.B * 4 * S;
  const bool attB = (int)blockIdx.x < units;
  const int split = (int)blockIdx.x % S;
  const int pair = (int)blockIdx.x / S;
  const int qd = pair & 3;
  const int rowB = min(pair >> 2, a.B - 1);

  uint64_t *full = bar + A_FULL;
  uint64_t *mdone = bar + A_MDONE;
  unsigned char *kbuf = smem + A_KBUF;
  auto issue = [&](int bb) {   // key batch bb: <= 4 boxes of 256 rows (32 B each)
    const int slot = bb % kStages;
    const int boxes = min(4, (n - bb * kBatchKeys + 255) >> 8);
    tc::mbar_arrive_expect_tx(&full[slot], (uint32_t)boxes * 8192u);
    for (int i = 0; i < boxes; ++i)
      tc::tma_load_2d(kbuf + slot * kBatchBytes + i * 8192, &kmap, 0, ybase + bb * kBatchKeys + i * 256,
                      &full[slot]);
  };
  if (tid == 0) {
    gb_read_base(ws.bar, G, misc);
    // the unit's pair counter before any unit of this call adds to it (they
    // do so only after the selection, which every CTA reaches after this)
    if (attB) asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(misc->pair_base) : "l"(ws.pair_done + pair) : "memory");
    // the candidate counters grow during the selection, after every CTA read them here
    if (scanA) asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(misc->cbase_a) : "l"(ws.ccount + rowA) : "memory");
    if (attB) asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(misc->cbase_b) : "l"(ws.ccount + rowB) : "memory");
    misc->token = (uint32_t)(misc->base_ctr / G) + 1u;
  }
  if (tid == kWork) {
    for (int i = 0; i < NBAR; ++i)
      tc::mbar_init(&bar[i], (i == BAR_KV_FULL || i == BAR_P_FULL || i == BAR_MX) ? 256u : i == BAR_QT ? 128u : 1u);
    misc->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int bb = 0; bb < min(kStages, nb); ++bb) issue(bb);
  }
  __syncwarp();
  if (warp == 8) tc::tmem_alloc(&misc->tmem, TMEM_COLS);

  uint32_t *hist = reinterpret_cast<uint32_t *>(smem + A_HIST);
  uint32_t *sc = reinterpret_cast<uint32_t *>(smem + A_SC);
  int w16[HI];
#pragma unroll
  for (int h = 0; h < HI; ++h) w16[h] = 0;
  if (warp < 8) {
    for (int i = tid; i < kBins; i += kWork) hist[i] = 0;
    if (scanA && tid < 16) {
      const int r = tid & 7, c = tid >> 3;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (r < HI) v = *reinterpret_cast<const uint4 *>(a.qI + ((int64_t)rowA * HI + r) * 32 + c * 16);
      *reinterpret_cast<uint4 *>(smem + A_QI + c * 128 + r * 16) = v;
    }
    if (scanA) {
#pragma unroll
      for (int h = 0; h < HI; ++h) {
        const float f = a.w[(int64_t)rowA * HI + h] * 16.f;
        const int r = __float2int_rn(f);
        if (tid == 0 && part == 0 && !((float)r == f && r >= 0 && r <= 16)) raise_status(a.status, STATUS_BAD_WEIGHT);
        w16[h] = min(max(r, 0), 16);
      }
    }
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = misc->tmem;
  if (warp < 4) {     // block scales 2^0 (UE8M0 127) wherever the MMA may read them
    const uint32_t ones[4] = {0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu};
    tc::tmem_st4(tbase + ((uint32_t)(warp * 32) << 16) + TCOL_SFA, ones);
    tc::tmem_st4(tbase + ((uint32_t)(warp * 32) << 16) + TCOL_SFB, ones);
    tc::tmem_wait_st();
  }

  // ---------------------------------------------------------------- A0 append
  if (scanA && append_ok && warp < 8) {
    const int b = rowA;
    if (part == a.per_row - 1) {
      const int g = tid & 127;
      if (warp < 4) {
        // pooled entries e0 .. e1-1; the loads of 4 tokens are issued together
        for (int j = 0; j < nbn; ++j) {
          Pool4 pl;
          pl.init();
          for (int i0 = 0; i0 < a.m; i0 += 4) {
            float4 xv[4], zv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              if (i0 + u < a.m) {
                const int64_t tok = (int64_t)b * a.n_new + (int64_t)j * a.m + i0 + u;
                xv[u] = __ldg(reinterpret_cast<const float4 *>(a.x_new + tok * TD) + g);
                zv[u] = __ldg(reinterpret_cast<const float4 *>(a.z_new + tok * TD) + g);
              }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (i0 + u < a.m) pl.push(xv[u], zv[u]);
          }
          float C[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) C[c] = __fdiv_rn(pl.acc[c], pl.l[c]);
          const float am = amax128(fmaxf(fmaxf(fabsf(C[0]), fabsf(C[1])), fmaxf(fabsf(C[2]), fabsf(C[3]))),
                                   misc, 0, 2);
          float s = __fdiv_rn(am, 448.f);
          if (!(s > 0.f)) s = 1.f;
          const int64_t ent = (int64_t)b * a.entry_cap + e0 + j;
          reinterpret_cast<uint32_t *>(a.codes + ent * TD)[g] = quant4(C, s);
          if (g == 0) a.scales[ent] = s;
        }
      } else {
        // the new tokens enter the window ring (loads of 4 tokens issued together)
        for (int i0 = 0; i0 < a.n_new; i0 += 4) {
          float4 xv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (i0 + u < a.n_new)
              xv[u] = __ldg(reinterpret_cast<const float4 *>(a.x_new + ((int64_t)b * a.n_new + i0 + u) * TD) + g);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (i0 + u >= a.n_new) break;
            const float C[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
            const float am = amax128(fmaxf(fmaxf(fabsf(C[0]), fabsf(C[1])), fmaxf(fabsf(C[2]), fabsf(C[3]))),
                                     misc, 4, 3);
            float s = __fdiv_rn(am, 448.f);
            if (!(s > 0.f)) s = 1.f;
            const int64_t p = tA - a.n_new + 1 + i0 + u;
            const int64_t ent = (int64_t)b * a.win_cap + p % a.win_cap;
            reinterpret_cast<uint32_t *>(a.wcodes + ent * TD)[g] = quant4(C, s);
            if (g == 0) a.wscales[ent] = s;
          }
        }
      }
      if (a.kI_new && tid < 2 * nbn) {
        const int j = tid >> 1, hf = tid & 1;
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(a.kI_new + ((int64_t)b * nbn + j) * 32 + hf * 16));
        *reinterpret_cast<uint4 *>(a.kI + ((int64_t)b * a.entry_cap + e0 + j) * 32 + hf * 16) = v;
      }
    }
    // exact scores of the new entries in this CTA's range, from the given keys
    // (the key cache rows are being written in this launch)
    if (a.kI_new && tid < nbn) {
      const int64_t e = e0 + tid;
      uint32_t s64 = 0;
      if (e >= s0 && e < s1) {
        const uint8_t *kr = a.kI_new + ((int64_t)b * nbn + tid) * 32;
#pragma unroll
        for (int h = 0; h < HI; ++h) {
          const uint8_t *qr = a.qI + ((int64_t)b * HI + h) * 32;
          int dot = 0;
          for (int k = 0; k < 32; ++k) {
            const uint32_t qb = qr[k], kb = kr[k];
            dot += e2m1x2(qb & 15) * e2m1x2(kb & 15) + e2m1x2(qb >> 4) * e2m1x2(kb >> 4);
          }
          s64 += (uint32_t)(w16[h] * max(dot, 0));
        }
      }
      misc->knew_score[tid] = s64;
    }
  }

  // ---------------------------------------------------------------- A1 scan
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const bool knew = scanA && append_ok && a.kI_new != nullptr;
  const uint32_t idesc = tc::idesc_mxf4(128, 8);
  const uint64_t bdesc = tc::smem_desc(tc::smem_u32(smem + A_QI), 128, 256);
  for (int bb = 0; bb <= nb; ++bb) {
    if (tid == kWork) {
      if (bb < nb) {
        const int slot = bb % kStages;
        if (bwait(&full[slot], (uint32_t)(bb / kStages) & 1u, misc, a.status)) {
          tc::fence_after_sync();
          const uint32_t buf = tc::smem_u32(kbuf + slot * kBatchBytes);
          const uint32_t acc = tbase + (uint32_t)(bb & 1) * 64;
#pragma unroll
          for (int i = 0; i < kBatchTiles; ++i)
            tc::mma_mxf4_ss(acc + i * 8, tc::smem_desc_sw32(buf + i * 4096), bdesc, idesc, tbase + TCOL_SFA,
                            tbase + TCOL_SFB, 0);
        }
        tc::mma_commit(&mdone[bb & 1]);
      }
      // the ring slot of batch bb - 1 is free once its MMAs are done
      const int pb = bb - 1;
      if (pb >= 0 && pb + kStages < nb && bwait(&mdone[pb & 1], (uint32_t)(pb >> 1) & 1u, misc, a.status))
        issue(pb + kStages);
    }
    if (bb > 0 && warp < 8) {
      const int pb = bb - 1;
      const bool ok = uniform(bwait(&mdone[pb & 1], (uint32_t)(pb >> 1) & 1u, misc, a.status));
      tc::fence_after_sync();
      const int q = warp & 3;
      uint32_t acc[4][4];
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        acc[i4][0] = acc[i4][1] = acc[i4][2] = acc[i4][3] = 0u;
        if (ok)
          tc::tmem_ld4(tbase + ((uint32_t)(q * 32) << 16) + (uint32_t)(pb & 1) * 64 + ((warp >> 2) * 4 + i4) * 8,
                       acc[i4]);
      }
      tc::tmem_wait_ld();
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        const int tile = (warp >> 2) * 4 + i4;
        const int j = pb * kBatchKeys + tile * kTileKeys + q * 32 + lane;
        if (j < n) {
          uint32_t s = 0;
#pragma unroll
          for (int h = 0; h < HI; ++h)
            s += (uint32_t)(w16[h] * max(0, __float2int_rn(4.f * __uint_as_float(acc[i4][h]))));
          if (knew && (int64_t)(s0 + j) >= e0 && (int64_t)(s0 + j) < e1) s = misc->knew_score[s0 + j - e0];
          sc[j] = s;
          atomicAdd(&hist[s >> 8], 1u);
        }
      }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
  }

  // ---------------------------------------------------------------- attention unit of this CTA
  int64_t tB = a.q_pos[rowB];
  if (tB < 0) tB = 0;
  const int nvisB = (int)min((tB + 1) / a.m, (int64_t)a.n_entries);
  const int nsel = min(a.K, nvisB);
  const int nwin = (int)min((int64_t)a.W, tB + 1);
  const int64_t p0 = tB - nwin + 1;
  const int n_items = nsel + nwin;
  const int nch = (n_items + CH - 1) / CH;
  const int c_begin = split * a.cps;
  const int c_end = min(c_begin + a.cps, nch);
  const int nloc = attB ? max(0, c_end - c_begin) : 0;
  if (tid == kWork && nloc > 0) {
    // the key ring is idle: Q of the unit's sequence in one 3-D TMA,
    // [32 d-blocks][128 heads][16 d]
    tc::mbar_arrive_expect_tx(&bar[BAR_Q], TH * TD * 2);
    tc::tma_load_3d(smem + B_Q, &qmap, 0, rowB * TH, 0, &bar[BAR_Q]);
  }

  // ---------------------------------------------------------------- A2 select
  uint32_t *ghist = ws.hist + (int64_t)rowA * kBins;
  if (scanA && warp < 8) {
    for (int i = tid; i < kBins; i += kWork) {
      const uint32_t c = hist[i];
      if (c) atomicAdd(&ghist[i], c);
    }
  }
  grid_sync(ws.bar, G, misc, a.status);             // barrier 1: row histograms complete

  uint32_t bstar = 0, above = 0, C = (uint32_t)nvisA;
  bool refine = false;
  uint64_t *cand = ws.cand + (int64_t)rowA * kCandCap;
  uint32_t *ccount = ws.ccount + rowA;
  if (scanA && warp < 8) {
    if (nvisA > a.K) {
      const uint4 *G4 = reinterpret_cast<const uint4 *>(ghist);
      for (int i = tid; i < kBins / 4; i += kWork) reinterpret_cast<uint4 *>(hist)[i] = __ldcg(G4 + i);
      wsync();
      find_bin_w(hist, (uint32_t)a.K, misc);
      bstar = (uint32_t)misc->bin;
      above = misc->above;
      C = above + hist[bstar];
    }
    refine = C > (uint32_t)kCandCap;
    if (!refine) {
      uint32_t mine = 0;
      for (int j = tid; j < n; j += kWork) mine += (sc[j] >> 8) >= bstar ? 1u : 0u;
      uint32_t total;
      uint32_t pos = block_scan_w(mine, misc, &total);
      if (tid == 0) misc->base = total ? atomicAdd(ccount, total) - misc->cbase_a : 0u;
      wsync();
      pos += misc->base;
      for (int j = tid; j < n; j += kWork) {
        const uint32_t s = sc[j];
        if ((s >> 8) >= bstar) {
          if (pos < (uint32_t)kCandCap) cand[pos] = make_key(s, (uint32_t)(s0 + j));
          ++pos;
          // a candidate's cache row is likely to be gathered by the attention
          if (nvisA > a.K)
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.codes + ((int64_t)rowA * a.entry_cap + s0 + j) * TD),
                         "r"(TD)
                         : "memory");
        }
      }
    } else {
      if (tid == 0 && part == 0) atomicExch(ws.flag, misc->token);
      wsync();
      for (int i = tid; i < 256; i += kWork) hist[i] = 0;
      wsync();
      for (int j = tid; j < n; j += kWork) {
        const uint32_t s = sc[j];
        if ((s >> 8) == bstar) atomicAdd(&hist[s & 255u], 1u);
      }
      wsync();
      for (int i = tid; i < 256; i += kWork)
        if (hist[i]) atomicAdd(&ws.hist2[rowA * 256 + i], hist[i]);
    }
  }
  grid_sync(ws.bar, G, misc, a.status);             // barrier 2: candidates listed

  // the same decision in every CTA; the histograms' last reads are done
  const bool refine_any = *(volatile uint32_t *)ws.flag == misc->token;
  if (warp < 8) {
    const uint32_t per = (ws.zone_hist_u4 + G - 1) / G;
    const uint32_t z0 = min(blockIdx.x * per, ws.zone_hist_u4), z1 = min(z0 + per, ws.zone_hist_u4);
    uint4 *zp = reinterpret_cast<uint4 *>(ws.zone);
    for (uint32_t i = z0 + tid; i < z1; i += kWork) zp[i] = make_uint4(0, 0, 0, 0);
  }
  if (refine_any) {
    uint32_t tstar = 0, take_ties = 0;
    if (scanA && refine && warp < 8) {
      if (tid == 0) {
        const uint32_t need = (uint32_t)a.K - above;
        uint32_t run = 0;
        int lo = 255;
        for (; lo > 0; --lo) {
          const uint32_t c = __ldcg(ws.hist2 + rowA * 256 + lo);
          if (run + c >= need) break;
          run += c;
        }
        misc->tstar = (bstar << 8) | (uint32_t)lo;
        misc->take = need - run;
      }
      wsync();
      tstar = misc->tstar;
      take_ties = misc->take;
      uint32_t myties = 0;
      for (int j0 = 0; j0 < n; j0 += kWork) {
        const int j = j0 + tid;
        const uint32_t s = j < n ? sc[j] : 0u;
        list_append(j < n && s > tstar, make_key(s, (uint32_t)(s0 + j)), ccount, misc->cbase_a, cand);
        myties += (j < n && s == tstar) ? 1u : 0u;
      }
      myties = __reduce_add_sync(0xffffffffu, myties);
      wsync();
      if (lane == 0) misc->warp_tot[warp] = myties;
      wsync();
      if (tid == 0) {
        uint32_t tot = 0;
        for (int k = 0; k < 8; ++k) tot += misc->warp_tot[k];
        ws.tiecnt[blockIdx.x] = tot;
      }
    }
    grid_sync(ws.bar, G, misc, a.status);           // barrier 3r: tie counts published
    if (scanA && refine && warp == 0) {
      uint32_t before = 0;
      for (int p = 0; p < part; ++p) before += __ldcg(ws.tiecnt + rowA * a.per_row + p);
      const uint32_t want = take_ties > before ? take_ties - before : 0u;
      uint32_t got = 0;
      for (int j0 = 0; j0 < n && got < want; j0 += 32) {
        const int j = j0 + lane;
        const bool tie = j < n && sc[j] == tstar;
        const unsigned msk = __ballot_sync(0xffffffffu, tie);
        const uint32_t r = got + __popc(msk & ((1u << lane) - 1u));
        list_append(tie && r < want, make_key(tstar, (uint32_t)(s0 + j)), ccount, misc->cbase_a, cand);
        got += __popc(msk);
      }
    }
    grid_sync(ws.bar, G, misc, a.status);           // barrier 4r: candidates listed
    // the tie counters' last reads are done
    if (warp < 8) {
      const uint32_t nz = ws.zone_u4 - ws.zone_hist_u4;
      const uint32_t per = (nz + G - 1) / G;
      const uint32_t z0 = min(blockIdx.x * per, nz), z1 = min(z0 + per, nz);
      uint4 *zp = reinterpret_cast<uint4 *>(ws.zone) + ws.zone_hist_u4;
      for (uint32_t i = z0 + tid; i < z1; i += kWork) zp[i] = make_uint4(0, 0, 0, 0);
    }
  }

  // rank: each candidate's position is the number of larger keys, counted
  // by a warp; the row's CTAs share its candidates
  if (scanA && warp < 8) {
    const int cnt = min(a.K, nvisA);
    int32_t *oi = a.idx_out + (int64_t)rowA * a.K;
    float *os = a.score_out ? a.score_out + (int64_t)rowA * a.K : nullptr;
    const uint32_t nc = min(__ldcg(ccount) - misc->cbase_a, (uint32_t)kCandCap);
    uint64_t *ck = reinterpret_cast<uint64_t *>(smem + A_SC);   // the scores are no longer needed
    wsync();
    for (uint32_t i = tid; i < nc; i += kWork) ck[i] = __ldcg(cand + i);
    wsync();
    for (uint32_t i = (uint32_t)(part + a.per_row * warp); i < nc; i += (uint32_t)(a.per_row * 8)) {
      const uint64_t key = ck[i];
      uint32_t r = 0;
      for (uint32_t j = lane; j < nc; j += 32) r += ck[j] > key ? 1u : 0u;
      r = __reduce_add_sync(0xffffffffu, r);
      if (lane == 0 && r < (uint32_t)cnt) {
        const uint32_t e = 0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFu);
        oi[r] = (int32_t)e;
        if (os) os[r] = (float)(uint32_t)(key >> 32) * (1.f / 64.f);
        // the attention gathers this row next (the candidates of a tie-flooded
        // threshold bin were not prefetched when they were listed)
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a.codes + ((int64_t)rowA * a.entry_cap + e) * TD),
                     "r"(TD)
                     : "memory");
      }
    }
    if (part == 0) {
      for (int j = cnt + tid; j < a.K; j += kWork) {
        oi[j] = -1;
        if (os) os[j] = 0.f;
      }
    }
  }
  // barrier 5: selections and appended rows visible.  While the other CTAs
  // finish their selection, the unit's Q goes from its staging buffer into
  // TMEM (the scan's accumulators are done with): warps 4-7, one head row per
  // thread; d-block k of the buffer holds d = 16 k .. 16 k + 15, and 32 TMEM
  // columns take 4 d-blocks (two bf16 per column)
  tc::fence_before_sync();
  __syncthreads();
  if (tid == 0) gb_arrive(ws.bar, misc);
  if (attB && nloc > 0 && warp >= 4 && warp < 8) {
    const int h = (warp & 3) * 32 + lane;
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const bool qok = uniform(bwait(&bar[BAR_Q], 0, misc, a.status));
#pragma unroll 1
    for (int cb = 0; cb < 8 && qok; ++cb) {
      uint32_t v[32];
#pragma unroll
      for (int db = 0; db < 4; ++db) {
        const uint4 *q4 = reinterpret_cast<const uint4 *>(smem + B_Q + ((cb * 4 + db) * TH + h) * 32);
        const uint4 x0 = q4[0], x1 = q4[1];
        v[db * 8 + 0] = x0.x; v[db * 8 + 1] = x0.y; v[db * 8 + 2] = x0.z; v[db * 8 + 3] = x0.w;
        v[db * 8 + 4] = x1.x; v[db * 8 + 5] = x1.y; v[db * 8 + 6] = x1.z; v[db * 8 + 7] = x1.w;
      }
      tc::tmem_st32(misc->tmem + lane_off + TCOL_Q + cb * 32, v);
    }
    tc::tmem_wait_st();
    tc::fence_before_sync();
    tc::mbar_arrive(&bar[BAR_QT]);
  }
  if (tid == 0) gb_wait(ws.bar, G, misc, a.status);
  __syncthreads();
  tc::fence_after_sync();

  // ---------------------------------------------------------------- B attend
  int *sel = reinterpret_cast<int *>(smem + B_SEL);
  float *iscale = reinterpret_cast<float *>(smem + B_SCALE);
  const int nsel_loc = max(0, min(nloc * CH, nsel - c_begin * CH));
  if (warp < 8)
    for (int i = tid; i < nsel_loc; i += kWork) sel[i] = __ldcg(a.idx_out + (int64_t)rowB * a.K + c_begin * CH + i);
  __syncthreads();
  const uint32_t sbase = tc::smem_u32(smem);
  bool ok_b = true;
  float m_used = -INFINITY, l_sum = 0.f;
  if (warp < 8) {
    // ------------------------------------------------------------ workers
    // Every worker gathers a share of each chunk; the softmax of a head runs
    // on the two warps that own its TMEM lane (warp w and w + 4), each over
    // half of the chunk's items; warps 4-7 also move Q into TMEM and run the
    // epilogue.
    const bool soft = warp >= 4;
    const int quad = warp & 3;
    const int half = soft ? 0 : 1;                    // items [64 half, 64 half + 64) of a chunk
    const int h = quad * 32 + lane;                   // this thread's head (TMEM lane)
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    float *mxx = reinterpret_cast<float *>(smem + B_MX);   // [2][128]
    const float qs = a.sm_scale * kLog2e;
    for (int c = 0; c < nloc && ok_b; ++c) {
      // gather: 4 threads per item row (8 x 16 B each), 2 rows per thread;
      // the loads are issued before anything else waits
      uint4 cv[2][8];
      float scr[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int t = tid + kWork * r;
        const int item = t >> 2, pq = t & 3;
        const int u = (c_begin + c) * CH + item;
        const uint8_t *src;
        const float *scp;
        if (u < nsel) {
          const int64_t ent = (int64_t)rowB * a.entry_cap + sel[u - c_begin * CH];
          src = a.codes + ent * TD;
          scp = a.scales + ent;
        } else {
          // items past the list read a valid row (the first window token);
          // their logits are masked and their P is zero
          const int64_t pp = p0 + (u < n_items ? u - nsel : 0);
          const int64_t ent = (int64_t)rowB * a.win_cap + (pp % a.win_cap);
          src = a.wcodes + ent * TD;
          scp = a.wscales + ent;
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) cv[r][k] = ldcg16(src + 16 * (pq + 4 * k));
        scr[r] = u < n_items ? __ldcg(scp) : 0.f;
      }
      if (c == 0) {
        // Q is in TMEM (moved during barrier 5); the tile overlays its
        // staging buffer, so every head must have been copied
        if (!uniform(bwait(&bar[BAR_QT], 0, misc, a.status) && ok_b)) { ok_b = false; break; }
      } else if (!uniform(bwait(&bar[BAR_KV_FREE], (c - 1) & 1, misc, a.status))) {
        ok_b = false;
        break;
      }
      unsigned char *kv = smem + B_KV;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int t = tid + kWork * r;
        const int item = t >> 2, pq = t & 3;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int pc = pq + 4 * k;
          uint4 lo, hi;
          e4m3x16_to_bf16x16(cv[r][k], lo, hi);
          *reinterpret_cast<uint4 *>(kv + kv_off(item, 2 * pc)) = lo;
          *reinterpret_cast<uint4 *>(kv + kv_off(item, 2 * pc + 1)) = hi;
        }
        if (pq == 0) iscale[item] = scr[r];
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bar[BAR_KV_FULL]);
      // -------------------------------------------------------- softmax of chunk c
      if (!uniform(bwait(&bar[BAR_S_FULL], c & 1, misc, a.status))) { ok_b = false; break; }
      tc::fence_after_sync();
      const int valid = min(CH, n_items - (c_begin + c) * CH);
      const int i_lo = half * (CH / 2);
      // one pass over this half's 64 scores: all of them into registers
      // (every TMEM read of S is done before the half's P overwrites part of S)
      uint32_t sr[CH / 2];
#pragma unroll
      for (int jb = 0; jb < CH / 64; ++jb)
        tc::tmem_ld32(tbase + lane_off + TCOL_S + i_lo + jb * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + jb * 32));
      tc::tmem_wait_ld();
      float sv[CH / 2];
      float pmx = -INFINITY;
#pragma unroll
      for (int j = 0; j < CH / 2; ++j) {
        const int i = i_lo + j;
        sv[j] = i < valid ? __uint_as_float(sr[j]) * iscale[i] * qs : -INFINITY;
        pmx = fmaxf(pmx, sv[j]);
      }
      // the two halves agree on the chunk maximum through shared memory
      mxx[half * TH + h] = pmx;
      tc::mbar_arrive(&bar[BAR_MX]);
      if (!uniform(bwait(&bar[BAR_MX], c & 1, misc, a.status))) { ok_b = false; break; }
      const float mx = fmaxf(mxx[h], mxx[TH + h]);
      const bool need = mx > m_used + kRescaleLog2;
      if (c > 0 && __any_sync(0xffffffffu, need)) {
        // O holds earlier chunks: wait for the last PV, then rescale this
        // warp's half of the head rows' quarter (2 of 4 column blocks)
        if (!uniform(bwait(&bar[BAR_PV_DONE], (c - 1) & 1, misc, a.status))) { ok_b = false; break; }
        tc::fence_after_sync();
        const float f = need ? ex2(m_used - mx) : 1.f;
#pragma unroll 1
        for (int blk = 2 * half; blk < 2 * half + 2; ++blk) {
          uint32_t o[32];
          tc::tmem_ld32(tbase + lane_off + TCOL_O + blk * 32, o);
          tc::tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
          tc::tmem_st32(tbase + lane_off + TCOL_O + blk * 32, o);
        }
        tc::tmem_wait_st();
      }
      if (need) {
        l_sum = (m_used == -INFINITY) ? 0.f : l_sum * ex2(m_used - mx);
        m_used = mx;
      }
      // P = p * item scale (bf16) for this half's items into TMEM over the
      // first 64 columns of S (row h, items 2j, 2j + 1 in column j): half h
      // writes columns 32 half .. 32 half + 31, the A operand of the PV MMAs
      float lsum = 0.f;
      uint32_t pw[32];
#pragma unroll
      for (int j = 0; j < CH / 2; j += 2) {
        const int i0 = i_lo + j;
        const float pa = ex2(sv[j] - m_used), pb = ex2(sv[j + 1] - m_used);
        lsum += pa + pb;
        const __nv_bfloat162 v = __floats2bfloat162_rn(pa * iscale[i0], pb * iscale[i0 + 1]);
        pw[j >> 1] = *reinterpret_cast<const uint32_t *>(&v);
      }
      tc::tmem_st32(tbase + lane_off + TCOL_S + half * 32, pw);
      tc::tmem_wait_st();
      l_sum += lsum;
      tc::fence_before_sync();
      tc::mbar_arrive(&bar[BAR_P_FULL]);
    }
    // the row sums of the two halves (every worker arrives here, whatever
    // happened in the loop)
    asm volatile("bar.sync 6, 256;" ::: "memory");
    mxx[half * TH + h] = l_sum;
    asm volatile("bar.sync 6, 256;" ::: "memory");
    if (soft) {
      l_sum = mxx[h] + mxx[TH + h];
      // epilogue: the normalised quarter row (one split) or the unnormalised
      // partial.  FIN completes once, after every MMA of the CTA.
      const int64_t orow = (int64_t)rowB * TH + h;
      const bool have = uniform(nloc > 0 && ok_b && bwait(&bar[BAR_FIN], 0, misc, a.status));
      tc::fence_after_sync();
      if (attB && S == 1) {
        if (have) {
          const float inv = 1.f / l_sum;
#pragma unroll 1
          for (int blk = 0; blk < DQ / 32; ++blk) {
            uint32_t o[32];
            tc::tmem_ld32(tbase + lane_off + TCOL_O + blk * 32, o);
            tc::tmem_wait_ld();
            uint32_t wv[16];
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
              const __nv_bfloat162 v =
                  __floats2bfloat162_rn(__uint_as_float(o[j]) * inv, __uint_as_float(o[j + 1]) * inv);
              wv[j >> 1] = *reinterpret_cast<const uint32_t *>(&v);
            }
            uint4 *dst = reinterpret_cast<uint4 *>(a.out + orow * TD + qd * DQ + blk * 32);
#pragma unroll
            for (int k = 0; k < 4; ++k) dst[k] = make_uint4(wv[4 * k], wv[4 * k + 1], wv[4 * k + 2], wv[4 * k + 3]);
          }
          if (a.lse && qd == 0) a.lse[orow] = (m_used + log2f(l_sum)) * 0.6931471805599453f;
        }
      } else if (attB) {
        // the unnormalised partial as [32 column quads][128 heads] float4 (a
        // warp's store covers 512 contiguous bytes), then (max, sum); each
        // writer makes its stores visible before the unit is counted done
        const int64_t slot = (int64_t)pair * S + split;
        float4 *dst = ws.ws_o + slot * (DQ / 4) * TH + h;
#pragma unroll 1
        for (int blk = 0; blk < DQ / 32; ++blk) {
          uint32_t o[32];
          if (have) {
            tc::tmem_ld32(tbase + lane_off + TCOL_O + blk * 32, o);
            tc::tmem_wait_ld();
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[(blk * 8 + k) * TH] = make_float4(__uint_as_float(o[4 * k]), __uint_as_float(o[4 * k + 1]),
                                                  __uint_as_float(o[4 * k + 2]), __uint_as_float(o[4 * k + 3]));
        }
        ws.ws_ml[slot * TH + h] = have ? make_float2(m_used, l_sum) : make_float2(-INFINITY, 0.f);
        __threadfence();
        asm volatile("bar.sync 4, 128;" ::: "memory");
        if (h == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ws.pair_done + pair) : "memory");
      }
    }
  } else {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nloc > 0) {
      const uint32_t idesc_qk = tc::idesc_bf16_f32(128, CH, 0, 0);
      const uint32_t idesc_pv = tc::idesc_bf16_f32(128, DQ, 0, 1);
      bool ok = bwait(&bar[BAR_QT], 0, misc, a.status);
      for (int c = 0; c < nloc && ok; ++c) {
        if (!bwait(&bar[BAR_KV_FULL], c & 1, misc, a.status)) break;
        tc::fence_after_sync();
        // S = Q K^T: A = Q from TMEM (8 columns per K step of 16 d), B = the
        // item tile, K-major core matrices (LBO = d-group step, SBO = 8 items)
#pragma unroll 4
        for (int k = 0; k < TD / 16; ++k)
          tc::mma_bf16_ts(tbase + TCOL_S, tbase + TCOL_Q + 8 * k, tc::smem_desc(sbase + B_KV + k * 4096, 2048, 128),
                          idesc_qk, k > 0);
        tc::mma_commit(&bar[BAR_S_FULL]);
        if (!bwait(&bar[BAR_P_FULL], c & 1, misc, a.status)) break;
        tc::fence_after_sync();
        // O += P V: A = P in TMEM over S (8 columns per 16 items), B = the
        // item tile read MN-major for this quarter of D (LBO = item-group
        // step, SBO = d-group step)
        const uint32_t vb = sbase + B_KV + qd * (DQ / 8) * 2048;
#pragma unroll
        for (int kk = 0; kk < CH / 16; ++kk)
          tc::mma_bf16_ts(tbase + TCOL_O, tbase + TCOL_S + 8 * kk, tc::smem_desc(vb + kk * 256, 128, 2048), idesc_pv,
                          (c > 0 || kk > 0));
        tc::mma_commit(&bar[BAR_KV_FREE]);
        tc::mma_commit(&bar[BAR_PV_DONE]);
      }
      tc::mma_commit(&bar[BAR_FIN]);
      bwait(&bar[BAR_FIN], 0, misc, a.status);
    }
    __syncwarp();
  }

  // ---------------------------------------------------------------- merge of the item splits
  // Each unit combines heads [h0, h1) of its (sequence, quarter) once all S
  // partials of that pair are counted:
  //   out = sum_j 2^(m_j - M) O_j / sum_j 2^(m_j - M) l_j,  M = max_j m_j.
  if (S > 1 && attB) {
    if (tid == 0 && !misc->abort) {
      const uint32_t target = misc->pair_base + (uint32_t)S;
      const uint64_t t0 = gtimer();
      uint32_t v, it = 0;
      for (;;) {
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ws.pair_done + pair) : "memory");
        if ((int32_t)(v - target) >= 0) break;
        if ((++it & 63u) == 0 && gtimer() - t0 > kWaitNs) {
          misc->abort = 1;
          raise_status(a.status, STATUS_TIMEOUT);
          break;
        }
      }
      __threadfence();
    }
    __syncthreads();
    const int h0 = split * TH / S, h1 = (split + 1) * TH / S;
    const int64_t slot0 = (int64_t)pair * S;
    merge_quarter(ws.ws_o + slot0 * (DQ / 4) * TH, ws.ws_ml + slot0 * TH, S, h0, h1 - h0,
                  a.out + (int64_t)rowB * TH * TD + qd * DQ, (a.lse && qd == 0) ? a.lse + (int64_t)rowB * TH : nullptr);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 8) tc::tmem_dealloc(tbase, TMEM_COLS);
}

int g_sms[64] = {0};

int ds_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (!g_sms[dev]) {
    int sms = 0, occ = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (set_smem_once((const void *)decode_step_kernel<4>, (int)SMEM_BYTES, "decode_step_kernel")) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, decode_step_kernel<4>, kThreads, SMEM_BYTES) !=
            cudaSuccess || occ < 1)
      return 0;
    g_sms[dev] = sms;
  }
  return g_sms[dev];
}

struct Plan {
  int G, per_row, S, cps;
};

// The launch shape, or false (with the reason in the error message) when the
// shape is outside the fused step's set.
bool ds_plan(const csa_dims *d, int n_new, Plan *p) {
  if (d->Tq != 1) return fail(CSA_ERR_UNSUPPORTED, "csa_decode_step: Tq=%d (one query per sequence)", d->Tq), false;
  if (d->H != TH || d->D != TD || d->dI != 64 || d->HI < 1 || d->HI > 4)
    return fail(CSA_ERR_UNSUPPORTED, "csa_decode_step: H=%d D=%d HI=%d dI=%d (supported: 128 heads, D 512, "
                "indexer 1..4 x 64)", d->H, d->D, d->HI, d->dI), false;
  if (d->K < 1 || d->K > kCandCap) return fail(CSA_ERR_UNSUPPORTED, "csa_decode_step: K=%d (1..2048)", d->K), false;
  if (n_new < d->m || n_new % d->m || n_new > kMaxNew || n_new > d->win_cap)
    return fail(CSA_ERR_UNSUPPORTED, "csa_decode_step: n_new=%d (a multiple of m=%d, at most %d and win_cap)",
                n_new, d->m, kMaxNew), false;
  const int G = ds_sms();
  if (G < 1) return fail(CSA_ERR_CUDA, "csa_decode_step: cannot size the grid (no device?)"), false;
  if (d->B < 1 || 4 * d->B > G)
    return fail(CSA_ERR_UNSUPPORTED, "csa_decode_step: B=%d (1..%d sequences)", d->B, G / 4), false;
  const int per_row = G / d->B;
  if ((2 * (int64_t)d->n_entries + 2 * per_row - 2) / (2 * per_row - 1) + 1 > kLocalCap)
    return fail(CSA_ERR_UNSUPPORTED, "csa_decode_step: %d entries over %d CTAs per sequence (at most %d each)",
                d->n_entries, per_row, kLocalCap), false;
  const int nch = (d->K + d->W + CH - 1) / CH;
  int S = min(min(G / (4 * d->B), nch), kMaxSplits);
  const int cps = (nch + S - 1) / S;
  S = (nch + cps - 1) / cps;
  if (cps * CH > kMaxSelLocal)
    return fail(CSA_ERR_UNSUPPORTED, "csa_decode_step: K + W = %d items per sequence is too many", d->K + d->W),
           false;
  if ((int64_t)d->B * d->entry_cap >= (1ll << 31))
    return fail(CSA_ERR_UNSUPPORTED, "csa_decode_step: key cache too large for one tensor map"), false;
  p->G = G;
  p->per_row = per_row;
  p->S = S;
  p->cps = cps;
  return true;
}

size_t ds_workspace(const csa_dims *d, const Plan &p, Ws *ws, void *base) {
  const int64_t B = d->B;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off += (bytes + 255) & ~(size_t)255; return o; };
  const size_t o_bar = take(8);
  const size_t o_cnt = take((size_t)(B * 4));
  const size_t o_flag = take(4);
  const size_t o_hist = take((size_t)(B * kBins * 4));
  const size_t hist_end = off;
  const size_t o_hist2 = take((size_t)(B * 256 * 4));
  const size_t o_tie = take((size_t)(B * p.per_row * 4));
  const size_t zone_end = off;
  const size_t o_pair = take((size_t)(B * 4 * 4));
  const size_t o_cand = take((size_t)(B * kCandCap * 8));
  const int64_t slots = p.S > 1 ? B * 4 * p.S : 0;
  const size_t o_o = take((size_t)(slots * TH * DQ * 4));
  const size_t o_ml = take((size_t)(slots * TH * 8));
  if (ws && base) {
    char *c = static_cast<char *>(base);
    ws->bar = reinterpret_cast<unsigned long long *>(c + o_bar);
    ws->zone = reinterpret_cast<uint32_t *>(c + o_hist);
    ws->zone_u4 = (uint32_t)((zone_end - o_hist) / 16);
    ws->zone_hist_u4 = (uint32_t)((hist_end - o_hist) / 16);
    ws->hist = reinterpret_cast<uint32_t *>(c + o_hist);
    ws->hist2 = reinterpret_cast<uint32_t *>(c + o_hist2);
    ws->ccount = reinterpret_cast<uint32_t *>(c + o_cnt);
    ws->flag = reinterpret_cast<uint32_t *>(c + o_flag);
    ws->tiecnt = reinterpret_cast<uint32_t *>(c + o_tie);
    ws->pair_done = reinterpret_cast<uint32_t *>(c + o_pair);
    ws->cand = reinterpret_cast<uint64_t *>(c + o_cand);
    ws->ws_o = reinterpret_cast<float4 *>(c + o_o);
    ws->ws_ml = reinterpret_cast<float2 *>(c + o_ml);
  }
  return off;
}

}  // namespace

size_t decode_step_workspace(const csa_dims *d, int n_new) {
  Plan p;
  if (!ds_plan(d, n_new, &p)) return 0;
  return ds_workspace(d, p, nullptr, nullptr);
}

int launch_decode_step(const float *x_new, const float *z_new, int n_new, const uint8_t *kI_new,
                       const uint16_t *q, const uint8_t *qI, const float *w, const int32_t *q_pos,
                       uint8_t *codes, float *scales, uint8_t *kI, uint8_t *win_codes, float *win_scales,
                       const csa_dims *d, int32_t *idx_out, float *score_out, uint16_t *out, float *lse,
                       void *workspace, size_t workspace_bytes, cudaStream_t stream) {
  Plan p;
  if (!ds_plan(d, n_new, &p)) return CSA_ERR_UNSUPPORTED;
  StepArgs a;
  const size_t need = ds_workspace(d, p, &a.ws, workspace);
  if (!workspace || workspace_bytes < need)
    return fail(CSA_ERR_WORKSPACE, "csa_decode_step: workspace needs %zu bytes (got %zu)", need, workspace_bytes);
  a.x_new = x_new; a.z_new = z_new; a.kI_new = kI_new; a.q_pos = q_pos; a.qI = qI; a.w = w;
  a.codes = codes; a.scales = scales; a.kI = kI; a.wcodes = win_codes; a.wscales = win_scales;
  a.B = d->B; a.m = d->m; a.K = d->K; a.W = d->W; a.n_entries = d->n_entries; a.win_cap = d->win_cap;
  a.n_new = n_new; a.entry_cap = d->entry_cap; a.sm_scale = d->softmax_scale;
  a.per_row = p.per_row; a.S = p.S; a.cps = p.cps;
  a.idx_out = idx_out; a.score_out = score_out;
  a.out = reinterpret_cast<__nv_bfloat16 *>(out);
  a.lse = lse;
  a.status = status_word_device_ptr();
  CUtensorMap kmap, qmap;
  if (!encode_tmap_2d(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, kI, 32, (uint64_t)d->B * d->entry_cap, 32, 32, 256,
                      CU_TENSOR_MAP_SWIZZLE_32B))
    return fail(CSA_ERR_INVALID, "csa_decode_step: cannot map the indexer keys for TMA");
  // Q as [32 d-blocks][B * 128 rows][16 d]: one box of 16 x 128 x 32 lands as
  // [d-block][head][16 d] in shared memory
  const uint64_t qdims[3] = {16, (uint64_t)d->B * TH, TD / 16};
  const uint64_t qstrides[2] = {TD * 2, 32};
  const uint32_t qbox[3] = {16, TH, TD / 16};
  if (!encode_tmap_3d(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, qdims, qstrides, qbox))
    return fail(CSA_ERR_INVALID, "csa_decode_step: cannot map the queries for TMA");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.G);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  switch (d->HI) {
#define CSA_DS(HI_)                                                                                       \
  case HI_:                                                                                               \
    if (int rc = set_smem_once((const void *)decode_step_kernel<HI_>, (int)SMEM_BYTES, "decode_step_kernel")) \
      return rc;                                                                                          \
    e = cudaLaunchKernelEx(&cfg, decode_step_kernel<HI_>, kmap, qmap, a);                                 \
    break;
    CSA_DS(1) CSA_DS(2) CSA_DS(3) CSA_DS(4)
#undef CSA_DS
    default: return fail(CSA_ERR_UNSUPPORTED, "csa_decode_step: HI=%d", d->HI);
  }
  count_launches(1);
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "decode_step_kernel launch: %s", cudaGetErrorString(e));
  return check_launch("decode_step_kernel");
}

}  // namespace csa
