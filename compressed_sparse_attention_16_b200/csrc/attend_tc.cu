// Shared-KV multi-query attention on the sm_100a tensor cores (tcgen05 +
// TMEM) for 128 query heads and 512-wide entries.
//
// Page: jiwasawa.github.io DeepSeek-V4 article, section "Compressed Sparse
// Attention (CSA)" -- multi-query attention with shared key-value over the
// k selected entries; section "Heavily Compressed Attention (HCA)" -- dense
// attention over the compressed sequence plus a sliding-window branch;
// "DeepSeek V4 Flash" (studioglobal.ai), "アテンションのブレイクスルー" -- the
// window covers the latest 128 tokens.  The same key/value row serves as key
// and as value, so one shared-memory tile feeds both products.
//
// Work split: one CTA per (query row, half of D, item split).  With M = 128
// query heads, S = Q K^T (K = 512) lands in TMEM with one head per lane; the
// output half O[:, dh*256 : dh*256+256] = P V accumulates in 256 TMEM columns
// across the CTA's chunks of 64 items.  Both halves of a row compute the same
// S (each needs the full 512-wide dot products) and keep bit-identical softmax
// state, so their halves combine without exchange.  The item splits of one
// (row, half) (1, 2, 4 or 8) form a thread-block cluster: each CTA writes its
// unnormalised partial O and per-head (max, sum) to the workspace (L2), one
// hardware cluster barrier orders them, and CTA c then combines the final
// rows of heads [c * 128 / S, +128 / S):
//   out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s.
//
// Tensor memory (512 columns): O (256), S double-buffered (2 x 64), and the
// first half of Q (d < 256, 128 columns of bf16 pairs) as the A operand of
// the first 16 QK MMAs; the second half of Q stays in shared memory (16 TMA
// boxes of 128 heads x 16 d, 32-byte swizzle).  That frees the room for two
// 64-item tiles, so the loaders fill one tile while the tensor core reads the
// other.  P (bf16) overwrites the first 32 columns of its S buffer and is the
// TMEM A operand of the PV MMAs, so it never touches shared memory.  A
// tcgen05 MMA with M = 128 and K = 16 costs about the same for N = 32 and
// N = 64 (about 50 cycles, its issue floor, against 135 at N = 256), so the
// QK product runs at N = 64.
//
// Roles (416 threads):
//   warps 0-7  gather 64 items per chunk, one item row per thread and half
//              of d (dense lists: one bulk L2 prefetch of the chunk two
//              ahead), convert E4M3 codes exactly to bf16 and store them in
//              the "core matrix" layout (8 rows x 16 B); with four warps the
//              conversion and stores of a chunk (~2 us) paced the CTA;
//   warps 8-11 first half of Q into TMEM, then softmax: one head per thread,
//              lazy rescaling of O (only when a chunk raises the running max
//              by more than 2^8), P = p * scale written to TMEM;
//   warp 12    TMEM allocation, the Q TMA, and the single MMA-issuing thread,
//              which issues whichever of PV(c) and QK(c + 2) is ready first.
// Item scales multiply the logits and P, never the codes, so the bf16 tiles
// hold the E4M3 values exactly.  Every mbarrier wait is bounded by wall time;
// on expiry the CTA sets the library's status word and unwinds.
#include "common.cuh"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int TH = 128;          // heads = MMA M
constexpr int TD = 512;          // entry width
constexpr int DHALF = 256;       // output columns per CTA = PV MMA N
constexpr int CH = 64;           // items per chunk = QK MMA N
constexpr uint32_t GS = CH * 16; // byte step between d-groups of a KV tile
constexpr int kLoadWarps = 8;    // warps 0-7 gather and convert the item tiles
constexpr int kSoftWarp0 = 8;    // warps 8-11 run the softmax (TMEM lane quadrant = warp % 4)
constexpr int kMmaWarp = 12;     // TMEM allocation, Q TMA, MMA issue
constexpr int kThreads = 32 * (kMmaWarp + 1);
constexpr int kMaxSel = 2048;
constexpr int kPrefetchAhead = 2;  // chunks
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;
constexpr unsigned long long kWaitNs = 2000000000ull;   // 2 s per wait

// Shared memory map (bytes):
//   QH    128 heads x d 256..511 bf16 = 64 KiB (16 boxes of 4 KiB)
//   KV    2 x (64 x 512 bf16) = 128 KiB
//   SEL   int32 [2048] (sparse instances only)
//   SCALE fp32 [2][64] item scales (for P) and [2][64] scales x softmax
//         scale x log2(e) (for the logits)
template <bool SEL>
struct Lay {
  static constexpr uint32_t OFF_QH = 0;
  static constexpr uint32_t OFF_KV = OFF_QH + TH * (TD / 2) * 2;
  static constexpr uint32_t KV_BYTES = CH * TD * 2;
  static constexpr uint32_t OFF_SEL = OFF_KV + 2 * KV_BYTES;
  static constexpr uint32_t OFF_SCALE = OFF_SEL + (SEL ? kMaxSel * 4 : 0);
  static constexpr uint32_t OFF_BAR = OFF_SCALE + 2 * 2 * CH * 4;
  static constexpr uint32_t OFF_MISC = OFF_BAR + 16 * 8;
  static constexpr uint32_t SMEM_BYTES = OFF_MISC + 64;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// TMEM columns
constexpr uint32_t TCOL_O = 0;        // 256
constexpr uint32_t TCOL_S = 256;      // 2 x 64
constexpr uint32_t TCOL_QL = 384;     // 128: Q[:, 0:256] as bf16 pairs
constexpr uint32_t TMEM_COLS = 512;

// Each item tile is written in two halves of d: half A (the 256 columns
// this CTA's PV product does not read, needed only by the QK MMAs over
// them) and half B (this CTA's output half).  Half A of a slot is free once
// the QK MMAs over it are done, half B once PV is done, so the loaders
// refill half A of chunk c + 2 while PV(c) is still pending.
enum { BAR_FULL_A = 0, BAR_FULL_B = 2, BAR_FREE_A = 4, BAR_FREE_B = 6, BAR_S_FULL = 8, BAR_P_FULL = 10,
       BAR_PV_DONE = 12, BAR_FIN = 13, BAR_Q = 14, BAR_QT = 15, kNumBars = 16 };

struct Misc {
  uint32_t tmem_base;
  int abort;
  int nsel;
  int wcount[9];
};

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on an mbarrier phase; false (and the abort flag set) on expiry.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, Misc *misc, unsigned *status) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  uint32_t n = 0;
  while (!tc::mbar_try_wait(bar, parity)) {
    if ((++n & 255u) == 0) {
      if (*(volatile int *)&misc->abort) return false;
      if (globaltimer() - t0 > kWaitNs) {
        misc->abort = 1;
        raise_status(status, STATUS_TIMEOUT);
        return false;
      }
    }
  }
  return true;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Byte offsets in the core-matrix layouts.  g counts 16-byte groups along
// the contraction-side dimension of each tile (8 bf16).
//   QH [128 heads][256 d]:   not core matrices: 16 TMA boxes [128 heads][16 d]
//                            of 4 KiB with 32-byte swizzle, box k at k * 4096
//   KV [64 items][512 d]:    g = d/8,     g-stride 1 KiB,  item-group stride 128 B
__device__ __forceinline__ uint32_t kv_off(int i, int g) { return g * GS + (i >> 3) * 128 + (i & 7) * 16; }

// packed fp32 pairs (low word first) and the two-lane PTX arithmetic
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t v;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
  return v;
}
__device__ __forceinline__ void unpack2(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// 2^x by the hardware approximation (PTX ex2.approx.ftz.f32: a few ulp;
// results below 2^-126 flush to zero, far below what a bf16 P or the fp32
// row sum can hold next to the row's largest term, which is >= 2^-8)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}


struct Args {
  const __nv_bfloat16 *q;
  const uint8_t *codes;
  const float *scales;
  const int32_t *idx;       // nullptr: dense (HCA)
  const uint8_t *wcodes;
  const float *wscales;
  const int32_t *q_pos;
  int Tq, K, W, m, n_entries, win_cap;
  int64_t entry_cap;
  float sm_scale;
  int splits, cps;          // splits per row, chunks per split
  __nv_bfloat16 *out;
  float *lse;
  float *ws_o;              // [rows * 2][splits][8 blocks][128][32] partial outputs (splits > 1)
  float2 *ws_ml;            // [rows * 2][splits][128] (max, sum) in log2 units
  unsigned *status;
};

// Combine the S <= JMAX split partials of `nh` (<= NH) heads h0, h0 + 8, ...
// of one (row, half) into the bf16 output (and the log-sum-exp):
//   out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s.
// Lane l handles d = 8 l .. 8 l + 7 of the half; all loads are issued first.
template <int JMAX, int NH>
__device__ __forceinline__ void merge_heads(const Args &a, int64_t slot0, int S, int h0, int nh, int row, int dh,
                                            int lane) {
  float2 ml[NH];
  float4 v0[NH][JMAX], v1[NH][JMAX];
#pragma unroll
  for (int n = 0; n < NH; ++n) {
    const int h = h0 + 8 * n;
    const bool live = n < nh;
    ml[n] = (live && lane < S) ? __ldcg(a.ws_ml + (slot0 + lane) * TH + h) : make_float2(-INFINITY, 0.f);
#pragma unroll
    for (int j = 0; j < JMAX; ++j) {
      v0[n][j] = v1[n][j] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (live && j < S) {
        // d = 8 lane .. 8 lane + 7: block lane / 4, offset 8 (lane % 4)
        const float4 *src = reinterpret_cast<const float4 *>(
            a.ws_o + (slot0 + j) * TH * DHALF + ((int64_t)(lane >> 2) * TH + h) * 32 + (lane & 3) * 8);
        v0[n][j] = __ldcg(src);
        v1[n][j] = __ldcg(src + 1);
      }
    }
  }
#pragma unroll
  for (int n = 0; n < NH; ++n) {
    if (n >= nh) break;
    const int h = h0 + 8 * n;
    float M = ml[n].x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    const float wgt = (ml[n].y > 0.f) ? exp2f(ml[n].x - M) : 0.f;
    float L = wgt * ml[n].y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;
#pragma unroll
    for (int j = 0; j < JMAX; ++j) {
      const float wj = __shfl_sync(0xffffffffu, wgt, j);
      acc[0] += wj * v0[n][j].x; acc[1] += wj * v0[n][j].y; acc[2] += wj * v0[n][j].z; acc[3] += wj * v0[n][j].w;
      acc[4] += wj * v1[n][j].x; acc[5] += wj * v1[n][j].y; acc[6] += wj * v1[n][j].z; acc[7] += wj * v1[n][j].w;
    }
    const float inv = 1.f / L;
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 8; k += 2) {
      const __nv_bfloat162 v = __floats2bfloat162_rn(acc[k] * inv, acc[k + 1] * inv);
      w[k >> 1] = *reinterpret_cast<const uint32_t *>(&v);
    }
    const int64_t orow = (int64_t)row * TH + h;
    *reinterpret_cast<uint4 *>(a.out + orow * TD + dh * DHALF + lane * 8) = make_uint4(w[0], w[1], w[2], w[3]);
    if (a.lse && dh == 0 && lane == 0) a.lse[orow] = (M + log2f(L)) * 0.6931471805599453f;
  }
}

template <bool SEL>
__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                const Args a) {
  using Lt = Lay<SEL>;
  constexpr uint32_t OFF_QH = Lt::OFF_QH, OFF_KV = Lt::OFF_KV, KV_BYTES = Lt::KV_BYTES;
  constexpr uint32_t OFF_SEL = Lt::OFF_SEL, OFF_SCALE = Lt::OFF_SCALE;
  constexpr uint32_t OFF_BAR = Lt::OFF_BAR, OFF_MISC = Lt::OFF_MISC;
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  Misc *misc = reinterpret_cast<Misc *>(smem + OFF_MISC);
  int *sel = reinterpret_cast<int *>(smem + OFF_SEL);
  float *iscale = reinterpret_cast<float *>(smem + OFF_SCALE);        // [2][CH] item scales
  float *lscale = iscale + 2 * CH;                                     // [2][CH] logit factors

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x % a.splits;        // == rank in the cluster
  const int pair = blockIdx.x / a.splits;
  const int dh = pair & 1;
  const int row = pair >> 1;
  const int b = row / a.Tq;

  int64_t t = a.q_pos[row];
  if (t < 0) {
    if (tid == 0) raise_status(a.status, STATUS_BAD_POSITION);
    t = 0;
  }
  const int nvis = (int)min((t + 1) / a.m, (int64_t)a.n_entries);
  const int nwin = (int)min((int64_t)a.W, t + 1);
  const int64_t p0 = t - nwin + 1;

  if (tid == 0) {
    misc->abort = 0;
    for (int i = 0; i < kNumBars; ++i)
      tc::mbar_init(&bars[i], i < BAR_FREE_A ? 32 * kLoadWarps
                                  : (i == BAR_P_FULL || i == BAR_P_FULL + 1 || i == BAR_QT) ? 128 : 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (warp == kMmaWarp) {
    tc::tmem_alloc(&misc->tmem_base, TMEM_COLS);
  } else if (warp < 8 && SEL && a.idx) {
    // ordered compaction of the valid selected entries (warps 0-7)
    const int32_t *irow = a.idx + (int64_t)row * a.K;
    int base = 0;
    for (int j0 = 0; j0 < a.K; j0 += 256) {
      const int j = j0 + tid;
      int e = (j < a.K) ? irow[j] : -1;
      if (e >= a.n_entries || e < -1) { raise_status(a.status, STATUS_BAD_INDEX); e = -1; }
      const bool f = e >= 0;
      const unsigned bal = __ballot_sync(0xffffffffu, f);
      if (lane == 0) misc->wcount[warp] = __popc(bal);
      asm volatile("bar.sync 2, 256;" ::: "memory");
      int before = 0, tot = 0;
      for (int k = 0; k < 8; ++k) { if (k < warp) before += misc->wcount[k]; tot += misc->wcount[k]; }
      if (f) sel[base + before + __popc(bal & ((1u << lane) - 1u))] = e;
      base += tot;
      asm volatile("bar.sync 2, 256;" ::: "memory");
    }
    if (tid == 0) misc->nsel = base;
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const int nsel = (SEL && a.idx) ? misc->nsel : nvis;
  const int n_items = nsel + nwin;
  const int nch = (n_items + CH - 1) / CH;
  const int c_begin = split * a.cps;
  const int c_end = min(c_begin + a.cps, nch);
  const int nloc = max(0, c_end - c_begin);
  const uint32_t tbase = misc->tmem_base;
  const uint32_t sbase = tc::smem_u32(smem);
  // source row of item u of the list (selected entries, then the window);
  // items past the list read the first window token (masked, P = 0)
  auto item_src = [&](int u, const float **scp) -> const uint8_t * {
    if (u < nsel) {
      const int e = (SEL && a.idx) ? sel[u] : u;
      const int64_t ent = (int64_t)b * a.entry_cap + e;
      *scp = a.scales + ent;
      return a.codes + ent * TD;
    }
    const int64_t p = p0 + (u < n_items ? u - nsel : 0);
    const int64_t ent = (int64_t)b * a.win_cap + (p % a.win_cap);
    *scp = a.wscales + ent;
    return a.wcodes + ent * TD;
  };
  if (warp == kMmaWarp && lane == 0 && nloc > 0) {
    // second half of Q: 16 boxes of 128 heads x 16 d (32-byte swizzle, the
    // layout the MMA reads), box k = d 256 + 16 k
    tc::mbar_arrive_expect_tx(&bars[BAR_Q], TH * (TD / 2) * 2);
    for (int k = 0; k < TD / 32; ++k)
      tc::tma_load_2d(smem + OFF_QH + k * 4096, &qmap, TD / 2 + 16 * k, row * TH, &bars[BAR_Q]);
  }

  if (warp < kLoadWarps) {
    // ------------------------------------------------------------ loaders
    // 4 threads per item row; warp w takes items 8 w + (0..7) of each chunk,
    // thread (i8, pq) the 16-byte groups pq + 4 k of the row: k < 4 lie in
    // d < 256, k >= 4 in d >= 256.  Half A (d outside this CTA's output half)
    // first, half B after; each half's loads for the next chunk are issued as
    // soon as the previous half is stored.
    const int i8 = lane & 7, pq = lane >> 3;
    const int item = warp * 8 + i8;
    const float qs = a.sm_scale * kLog2e;
    const int u_end = min(c_end * CH, n_items);
    const int ka = (1 - dh) * 4, kb = dh * 4;      // first k of half A / half B
    uint4 ra[4], rb[4];
    float sc = 0.f;
    auto load_half = [&](int lc, int k0, uint4 (&r)[4], bool with_scale) {
      const int u = (c_begin + lc) * CH + item;
      const float *scp;
      const uint8_t *src = item_src(u, &scp);
#pragma unroll
      for (int k = 0; k < 4; ++k) r[k] = __ldg(reinterpret_cast<const uint4 *>(src) + pq + 4 * (k0 + k));
      // consumed only when the half is stored (items past the list get 0
      // there), so the load's latency stays hidden
      if (with_scale) sc = __ldg(scp);
      // dense lists: the entries of the chunk kPrefetchAhead ahead are
      // contiguous rows; one bulk prefetch pulls them into L2
      if (!SEL && with_scale && warp == 0 && lane == 0) {
        const int f0 = (c_begin + lc + kPrefetchAhead) * CH;
        const int f1 = min(min(f0 + CH, u_end), nsel);
        if (f0 < f1)
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;"
                       ::"l"(a.codes + ((int64_t)b * a.entry_cap + f0) * TD), "r"((f1 - f0) * TD) : "memory");
      }
    };
    auto store_half = [&](unsigned char *kv, int k0, const uint4 (&r)[4]) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int p = pq + 4 * (k0 + k);
        uint4 lo, hi;
        e4m3x16_to_bf16x16(r[k], lo, hi);
        *reinterpret_cast<uint4 *>(kv + kv_off(item, 2 * p)) = lo;
        *reinterpret_cast<uint4 *>(kv + kv_off(item, 2 * p + 1)) = hi;
      }
    };
    if (nloc > 0) {
      load_half(0, ka, ra, false);
      load_half(0, kb, rb, true);
    }
    for (int lc = 0; lc < nloc; ++lc) {
      const int kslot = lc & 1;
      unsigned char *kv = smem + OFF_KV + kslot * KV_BYTES;
      // half A: free once QK(lc - 2) has read it
      if (lc >= 2 && !wait_bar(&bars[BAR_FREE_A + kslot], ((lc - 2) >> 1) & 1, misc, a.status)) break;
      store_half(kv, ka, ra);
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[BAR_FULL_A + kslot]);
      if (lc + 1 < nloc) load_half(lc + 1, ka, ra, false);
      // half B and the item scales: free once PV(lc - 2) is done
      if (lc >= 2 && !wait_bar(&bars[BAR_FREE_B + kslot], ((lc - 2) >> 1) & 1, misc, a.status)) break;
      store_half(kv, kb, rb);
      if (pq == 0) {
        const float v = (c_begin + lc) * CH + item < n_items ? sc : 0.f;
        iscale[kslot * CH + item] = v;
        lscale[kslot * CH + item] = v * qs;
      }
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[BAR_FULL_B + kslot]);
      if (lc + 1 < nloc) load_half(lc + 1, kb, rb, true);
    }
  } else if (warp < kSoftWarp0 + 4) {
    // ------------------------------------------------------------ softmax
    const int quad = warp - kSoftWarp0;
    const int h = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    bool ok = true;
    if (nloc > 0) {
      // first half of Q into TMEM: lane h, column 384 + j holds d = 2j, 2j + 1
      const uint4 *qrow = reinterpret_cast<const uint4 *>(a.q + ((int64_t)row * TH + h) * TD);
#pragma unroll 1
      for (int blk = 0; blk < 4; ++blk) {
        uint32_t v[32];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 x = __ldg(qrow + blk * 8 + k);
          v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
        }
        tc::tmem_st32(tbase + lane_off + TCOL_QL + blk * 32, v);
      }
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[BAR_QT]);
    }
    float m_used = -INFINITY, l = 0.f;
    for (int c = 0; c < nloc && ok; ++c) {
      const int buf = c & 1;          // S buffer and item tile
      // full_b orders the loaders' scale writes before this thread's reads
      // one decision per warp: the TMEM accesses and votes below are warp-collective
      if (!__all_sync(0xffffffffu, wait_bar(&bars[BAR_FULL_B + buf], (c >> 1) & 1, misc, a.status) &&
                                       wait_bar(&bars[BAR_S_FULL + buf], (c >> 1) & 1, misc, a.status))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      const int valid = min(CH, n_items - (c_begin + c) * CH);
      const uint64_t *isc2 = reinterpret_cast<const uint64_t *>(iscale + buf * CH);
      const uint64_t *lsc2 = reinterpret_cast<const uint64_t *>(lscale + buf * CH);
      // logits in log2 units, as fp32 pairs: s = S * scale * softmax scale * log2(e)
      uint64_t s2[CH / 2];
      {
        uint32_t sr[CH];
#pragma unroll
        for (int jb = 0; jb < CH / 32; ++jb)
          tc::tmem_ld32(tbase + lane_off + TCOL_S + buf * CH + jb * 32, *reinterpret_cast<uint32_t(*)[32]>(sr + jb * 32));
        tc::tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < CH / 2; j += 2) {
          const uint4 l4 = *reinterpret_cast<const uint4 *>(lsc2 + j);
          s2[j] = mul2(pack2(__uint_as_float(sr[2 * j]), __uint_as_float(sr[2 * j + 1])),
                       (uint64_t)l4.x | ((uint64_t)l4.y << 32));
          s2[j + 1] = mul2(pack2(__uint_as_float(sr[2 * j + 2]), __uint_as_float(sr[2 * j + 3])),
                           (uint64_t)l4.z | ((uint64_t)l4.w << 32));
        }
      }
      if (valid < CH) {
#pragma unroll
        for (int j = 0; j < CH / 2; ++j) {
          float x0, x1;
          unpack2(s2[j], x0, x1);
          s2[j] = pack2(2 * j < valid ? x0 : -INFINITY, 2 * j + 1 < valid ? x1 : -INFINITY);
        }
      }
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < CH / 2; ++j) {
        float x0, x1;
        unpack2(s2[j], x0, x1);
        mx = max3(mx, x0, x1);
      }
      const bool need = mx > m_used + kRescaleLog2;
      if (c > 0 && __any_sync(0xffffffffu, need)) {
        // O holds earlier chunks: once PV(c - 1) is done, rescale this warp's rows
        if (!__all_sync(0xffffffffu, wait_bar(&bars[BAR_PV_DONE], (c - 1) & 1, misc, a.status))) { ok = false; break; }
        tc::fence_after_sync();
        const float f = need ? exp2f(m_used - mx) : 1.f;
#pragma unroll 1
        for (int blk = 0; blk < DHALF / 32; ++blk) {
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
        l = (m_used == -INFINITY) ? 0.f : l * exp2f(m_used - mx);
        m_used = mx;
      }
      // p = 2^(s - m); P = p * item scale, rounded to bf16
      const uint64_t negm = pack2(-m_used, -m_used);
      uint64_t lsum2 = pack2(0.f, 0.f);
      uint32_t pw[CH / 2];
#pragma unroll
      for (int j = 0; j < CH / 2; ++j) {
        float x0, x1;
        unpack2(add2(s2[j], negm), x0, x1);
        const uint64_t p2 = pack2(ex2(x0), ex2(x1));
        lsum2 = add2(lsum2, p2);
        float w0, w1;
        unpack2(mul2(p2, isc2[j]), w0, w1);
        const __nv_bfloat162 v = __floats2bfloat162_rn(w0, w1);
        pw[j] = *reinterpret_cast<const uint32_t *>(&v);
      }
      float l0, l1;
      unpack2(lsum2, l0, l1);
      l += l0 + l1;
      // P replaces the first 32 columns of its S buffer (row h, items
      // 2j, 2j + 1 in column j), the A operand of the PV MMAs
      tc::tmem_st32(tbase + lane_off + TCOL_S + buf * CH, pw);
      tc::tmem_wait_st();
      tc::fence_before_sync();
      tc::mbar_arrive(&bars[BAR_P_FULL + buf]);
    }
    // epilogue
    const int64_t orow = (int64_t)row * TH + h;
    // FIN completes once, after every MMA of the CTA (a parity wait on
    // PV_DONE could see a phase from chunks earlier when the PV MMAs lag)
    const bool have = __all_sync(0xffffffffu, nloc > 0 && ok && wait_bar(&bars[BAR_FIN], 0, misc, a.status));
    tc::fence_after_sync();
    if (a.splits == 1) {
      if (have) {
        const float inv = 1.f / l;
#pragma unroll 1
        for (int blk = 0; blk < DHALF / 32; ++blk) {
          uint32_t o[32];
          tc::tmem_ld32(tbase + lane_off + TCOL_O + blk * 32, o);
          tc::tmem_wait_ld();
          uint32_t w[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[j]) * inv, __uint_as_float(o[j + 1]) * inv);
            w[j >> 1] = *reinterpret_cast<const uint32_t *>(&v);
          }
          uint4 *dst = reinterpret_cast<uint4 *>(a.out + orow * TD + dh * DHALF + blk * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        }
        if (a.lse && dh == 0) a.lse[orow] = (m_used + log2f(l)) * 0.6931471805599453f;
      }
    } else {
      // partial rows (zeros when this split had no items) straight from TMEM
      // to the workspace, laid out [32-column block][head][32] so that each
      // thread writes whole 128-byte lines
      const int64_t slot = (int64_t)pair * a.splits + split;
      float *dstb = a.ws_o + slot * TH * DHALF;
      // two 32-column blocks per round: both TMEM loads in flight together
#pragma unroll 1
      for (int blk = 0; blk < DHALF / 32; blk += 2) {
        uint32_t o[2][32];
        if (have) {
          tc::tmem_ld32(tbase + lane_off + TCOL_O + blk * 32, o[0]);
          tc::tmem_ld32(tbase + lane_off + TCOL_O + (blk + 1) * 32, o[1]);
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o[0][j] = o[1][j] = 0u;
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          uint4 *dst = reinterpret_cast<uint4 *>(dstb + ((int64_t)(blk + u) * TH + h) * 32);
#pragma unroll
          for (int k = 0; k < 8; ++k) dst[k] = make_uint4(o[u][4 * k], o[u][4 * k + 1], o[u][4 * k + 2], o[u][4 * k + 3]);
        }
      }
      a.ws_ml[slot * TH + h] = have ? make_float2(m_used, l) : make_float2(-INFINITY, 0.f);
    }
  } else {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nloc > 0) {
      constexpr uint32_t idesc_qk = tc::idesc_bf16_f32(128, CH, 0, 0);
      constexpr uint32_t idesc_pv = tc::idesc_bf16_f32(128, DHALF, 0, 1);
      // Descriptors are built once; a K step only advances the start-address
      // field (bits 0..13 hold address / 16, and every address in shared
      // memory stays below 2^18, so the additions never carry out of it).
      // QK B = items, K-major core matrices: LBO = step between d-groups, SBO = 8-row groups
      const uint64_t bd_kv0 = tc::smem_desc(sbase + OFF_KV, GS, 128);
      const uint64_t bd_kv1 = tc::smem_desc(sbase + OFF_KV + KV_BYTES, GS, 128);
      // QK A (second half) = QH, K-major with 32-byte swizzle, one box per K step
      const uint64_t ad_qh = tc::smem_desc_sw32(sbase + OFF_QH);
      // PV A = P in TMEM (over its S buffer); B = the same item tile read
      // MN-major (N = d): LBO = step between item groups (K), SBO = between d-groups (N)
      const uint64_t bd_v0 = tc::smem_desc(sbase + OFF_KV + dh * (DHALF / 8) * GS, 128, GS);
      const uint64_t bd_v1 = tc::smem_desc(sbase + OFF_KV + KV_BYTES + dh * (DHALF / 8) * GS, 128, GS);
      // QK over one half of d: half 0 (d < 256) reads Q from TMEM, half 1
      // from shared memory; accumulation starts with half A
      auto issue_qk_half = [&](int c, int half, bool first) {
        const int buf = c & 1;
        const uint64_t bd = (buf ? bd_kv1 : bd_kv0) + (uint64_t)((half * (TD / 32) * 2 * GS) >> 4);
        const uint32_t dt = tbase + TCOL_S + buf * CH;
        if (half == 0) {
#pragma unroll
          for (int k = 0; k < TD / 32; ++k)
            tc::mma_bf16_ts(dt, tbase + TCOL_QL + 8 * k, bd + (uint64_t)((k * 2 * GS) >> 4), idesc_qk, !first || k > 0);
        } else {
#pragma unroll
          for (int k = 0; k < TD / 32; ++k)
            tc::mma_bf16_ss(dt, ad_qh + (uint64_t)((k * 4096) >> 4), bd + (uint64_t)((k * 2 * GS) >> 4), idesc_qk,
                            !first || k > 0);
        }
      };
      auto issue_pv = [&](int c) {
        const int buf = c & 1;
        const uint64_t bd = buf ? bd_v1 : bd_v0;
#pragma unroll
        for (int kk = 0; kk < CH / 16; ++kk)
          tc::mma_bf16_ts(tbase + TCOL_O, tbase + TCOL_S + buf * CH + 8 * kk, bd + (uint64_t)((kk * 256) >> 4), idesc_pv,
                          (c > 0 || kk > 0));
        tc::mma_commit(&bars[BAR_FREE_B + buf]);
        tc::mma_commit(&bars[BAR_PV_DONE]);
      };
      bool ok = wait_bar(&bars[BAR_Q], 0, misc, a.status) && wait_bar(&bars[BAR_QT], 0, misc, a.status);
      // QK_A(c) (over half A) needs that half of tile c in place and S buffer
      // c & 1 read (PV(c - 2) issued); QK_B(c) needs half B; PV(c) needs P(c).
      // The first ready of PV, QK_B, QK_A goes next, so the tensor core works
      // on one chunk while the loaders and the softmax warps handle others.
      // (Each product goes out whole: issuing QK in groups of 2-8 K steps, to
      // let a ready PV in sooner, made the call 20-80 % slower.)
      const int half_a = 1 - dh, half_b = dh;
      int nqa = 0, nqb = 0, npv = 0;
      const uint64_t t0 = globaltimer();
      uint32_t spins = 0;
      while (ok && npv < nloc) {
        bool did = false;
        const uint32_t pbar = BAR_P_FULL + (npv & 1);
        const uint32_t ppar = (npv >> 1) & 1;
        if (npv < nqb && tc::mbar_try_wait(&bars[pbar], ppar)) {
          tc::fence_after_sync();
          issue_pv(npv);
          ++npv;
          did = true;
        }
        if (nqb < nqa && tc::mbar_try_wait(&bars[BAR_FULL_B + (nqb & 1)], (nqb >> 1) & 1)) {
          tc::fence_after_sync();
          issue_qk_half(nqb, half_b, false);
          tc::mma_commit(&bars[BAR_S_FULL + (nqb & 1)]);
          ++nqb;
          did = true;
        }
        if (nqa < nloc && nqa < npv + 2 && tc::mbar_try_wait(&bars[BAR_FULL_A + (nqa & 1)], (nqa >> 1) & 1)) {
          tc::fence_after_sync();
          issue_qk_half(nqa, half_a, true);
          tc::mma_commit(&bars[BAR_FREE_A + (nqa & 1)]);
          ++nqa;
          did = true;
        }
        if (did) {
          spins = 0;
          continue;
        }
        if ((++spins & 255u) == 0) {
          if (*(volatile int *)&misc->abort) { ok = false; break; }
          if (globaltimer() - t0 > kWaitNs * 4) {
            misc->abort = 1;
            raise_status(a.status, STATUS_TIMEOUT);
            ok = false;
            break;
          }
        }
      }
      // drain: every MMA issued above has completed once FIN fires
      tc::mma_commit(&bars[BAR_FIN]);
      wait_bar(&bars[BAR_FIN], 0, misc, a.status);
    }
    __syncwarp();
  }

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  if (a.splits > 1) {
    // ---- combine heads [rank * 128 / S, +128 / S) of this (row, half) from
    // the partials every CTA of the cluster wrote before the barrier
    cluster_sync_all();
    const int S = a.splits;
    const int hper = TH / S;
    if (warp < 8) {
      const int64_t slot0 = (int64_t)pair * S;
      // S <= 4: two heads per round, so both heads' partials are in flight together
      if (S <= 4) {
        for (int hl = warp; hl < hper; hl += 16)
          merge_heads<4, 2>(a, slot0, S, split * hper + hl, hl + 8 < hper ? 2 : 1, row, dh, lane);
      } else {
        for (int hl = warp; hl < hper; hl += 8) merge_heads<8, 1>(a, slot0, S, split * hper + hl, 1, row, dh, lane);
      }
    }
  }
  if (warp == kMmaWarp) tc::tmem_dealloc(tbase, TMEM_COLS);
}

}  // namespace

// Item splits per (row, half): a power of two <= 8 (one thread-block cluster)
// so that rows * 2 * splits CTAs fill about one wave of the SMs.
static void tc_plan(const csa_dims *d, bool dense, int *splits, int *cps) {
  const int64_t rows = (int64_t)d->B * d->Tq;
  const int64_t max_items = (dense ? (int64_t)d->n_entries : (int64_t)d->K) + d->W;
  const int nch = (int)((max_items + CH - 1) / CH);
  const int64_t per = 148 / (2 * (rows > 0 ? rows : 1));
  int s = 1;
  while (s < 8 && 2 * s <= per && 2 * s <= nch) s *= 2;
  *cps = (nch + s - 1) / s;
  *splits = s;
}

bool attend_tc_supported(const csa_dims *d) { return d->H == TH && d->D == TD; }

size_t attend_tc_workspace(const csa_dims *d, bool dense) {
  int splits, cps;
  tc_plan(d, dense, &splits, &cps);
  if (splits == 1) return 0;
  const int64_t slots = (int64_t)d->B * d->Tq * 2 * splits;
  return (size_t)(slots * TH * (DHALF * 4 + 8)) + 256;
}

int launch_attend_tc(const uint16_t *q, const uint8_t *codes, const float *scales, const int32_t *idx,
                     const uint8_t *wcodes, const float *wscales, const int32_t *q_pos,
                     const csa_dims *d, uint16_t *out, float *lse, void *workspace,
                     cudaStream_t stream) {
  const bool dense = idx == nullptr;
  int splits, cps;
  tc_plan(d, dense, &splits, &cps);
  const int64_t rows = (int64_t)d->B * d->Tq;
  Args a;
  a.q = reinterpret_cast<const __nv_bfloat16 *>(q);
  a.codes = codes; a.scales = scales; a.idx = idx; a.wcodes = wcodes; a.wscales = wscales;
  a.q_pos = q_pos; a.Tq = d->Tq; a.K = d->K; a.W = d->W; a.m = d->m; a.n_entries = d->n_entries;
  a.win_cap = d->win_cap; a.entry_cap = d->entry_cap; a.sm_scale = d->softmax_scale;
  a.splits = splits; a.cps = cps;
  a.out = reinterpret_cast<__nv_bfloat16 *>(out);
  a.lse = lse;
  const int64_t slots = rows * 2 * splits;
  a.ws_o = splits > 1 ? static_cast<float *>(workspace) : nullptr;
  a.ws_ml = splits > 1 ? reinterpret_cast<float2 *>(static_cast<char *>(workspace) + (size_t)(slots * TH * DHALF * 4))
                       : nullptr;
  if (splits > 1 && !workspace) return fail(CSA_ERR_WORKSPACE, "attend: workspace required");
  a.status = status_word_device_ptr();
  // sparse instances keep room for the compacted selection
  const void *kfn = dense ? (const void *)attend_tc_kernel<false> : (const void *)attend_tc_kernel<true>;
  const uint32_t SMEM_BYTES = dense ? Lay<false>::SMEM_BYTES : Lay<true>::SMEM_BYTES;
  if (int rc = set_smem_once(kfn, (int)SMEM_BYTES, "attend_tc_kernel")) return rc;
  const int64_t grid = rows * 2 * splits;
  if (grid > 0x7fffffffLL) return fail(CSA_ERR_UNSUPPORTED, "attend: too many rows");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)splits;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // Q viewed as [rows * 128 heads][512 d] bf16; boxes of 16 d x 128 heads
  CUtensorMap qmap;
  if (!encode_tmap_2d(&qmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, TD, (uint64_t)(rows * TH), TD * 2, 16, TH,
                      CU_TENSOR_MAP_SWIZZLE_32B))
    return fail(CSA_ERR_INVALID, "attend: cannot map the queries for TMA (misaligned?)");
  const cudaError_t e = dense ? cudaLaunchKernelEx(&cfg, attend_tc_kernel<false>, qmap, a)
                              : cudaLaunchKernelEx(&cfg, attend_tc_kernel<true>, qmap, a);
  count_launches(1);
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "attend_tc_kernel launch: %s", cudaGetErrorString(e));
  return check_launch("attend_tc_kernel");
}

}  // namespace csa
