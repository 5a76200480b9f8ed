// Prefill indexer: exact per-query top-k over FP4 tensor-core scores in two
// streaming passes over the keys (more only for queries whose threshold bin
// is crowded).
//
// Pages: jiwasawa.github.io DeepSeek-V4 article, section "Compressed Sparse
// Attention (CSA)" -- every query scores the compressed entries with a
// lightweight indexer and keeps the top k; "DeepSeek V4とOpenCode"
// (hazakura.dev), "衝撃1：CSA + HCA" -- the indexer runs at FP4; "DeepSeek V4
// Flash" (studioglobal.ai), "アテンションのブレイクスルー" -- top 512 blocks.
//
// One CTA owns 128 consecutive queries of a sequence (one TMEM lane each) and
// streams their visible keys in tiles of 32 (TMA, 32-byte swizzle).  Per tile
// and indexer head one kind::mxf4 MMA (M = 128 queries, N = 32 keys, K = 64)
// gives exact q.k sums; the score 64 * sum_h w_h max(q_h.k, 0) is an integer
// below 2^20, exact in fp32.  Two groups of four warps take turns: group 0
// reads the first half of each pass's tiles, group 1 the second half, the
// control warp issuing the MMAs alternately into the group's own TMEM buffer
// so that one group computes while the other waits.  Each query thus has one
// thread per group, and each thread sees its keys in index order.
//
//   pass 0  a 321-bin histogram per query of the score's float exponent and
//           top 4 mantissa bits (bins about 6 % wide at any magnitude, so the
//           bin holding the k-th score is narrow whatever the query's scale);
//           counts go to shared memory with fire-and-forget atomics.  The
//           threshold bin follows from the counts.
//   (1, 2)  only if the threshold bin of some query would overflow the
//           candidate buffer: histograms of the next 8 score bits inside it.
//   last    every key above the threshold bin, and the whole threshold bin,
//           is appended to the query's candidate list (capacity 2k); when the
//           threshold is an exact score, each of the query's two threads takes
//           at most the k - above ties of its own keys (the first ties overall
//           are among them).  Group 0 fills the list from the front, group 1
//           from the back, each in index order, so that the list read as
//           front part then reversed back part is in index order.
// A second kernel sorts each query's candidates by score (a stable radix
// sort, so equal scores stay in index order) and writes the k best.
#include "common.cuh"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int kQ = 128;                  // queries per CTA = TMEM lanes = MMA M
constexpr int kN = 48;                   // keys per tile = MMA N (three chunks of 16)
constexpr int kStg = 8;                  // key-tile ring
constexpr int kThr = 320;                // warps 0-7 epilogue (two groups of 4), 8 MMA issue, 9 key loads
constexpr int kEpi = 256;
constexpr int kBins0 = 321;              // 0: score 0; 1..320: exponent (0..19) x 16 + mantissa bits
constexpr int kHistRows = 324;
constexpr uint32_t kCols = 512;          // 2 accumulator buffers x 4 heads x 48 + scale columns
constexpr uint32_t kBufCols = 4 * kN;
constexpr uint32_t kColSFA = 2 * kBufCols, kColSFB = kColSFA + 4;
constexpr int kTileBytes = kN * 32;      // one key tile in shared memory
constexpr int kStage = 64;               // collection: candidates staged per thread before a flush
constexpr unsigned long long kWaitNs = 2000000000ull;

constexpr uint32_t OFF_Q = 0;                             // 4 heads x 128 queries x 32 B (core matrices)
constexpr uint32_t OFF_K = OFF_Q + 4 * 4096;              // kStg x kN keys x 32 B
constexpr uint32_t OFF_H = OFF_K + kStg * kTileBytes;     // u32 [kHistRows][128]; the collection's staging
constexpr uint32_t OFF_ST = OFF_H + kHistRows * kQ * 4;   // per-query selection state
constexpr uint32_t OFF_BAR = OFF_ST + kQ * 16;
constexpr uint32_t OFF_MISC = OFF_BAR + 32 * 8;
constexpr uint32_t SMEM = OFF_MISC + 64;
static_assert(SMEM <= 232448, "shared memory");
static_assert(kStage * kEpi * 8 <= kHistRows * kQ * 4, "staging fits in the histogram area");

struct QState {          // one query's threshold so far
  uint32_t prefix;       // (score bits) >> shift of the threshold bin
  uint32_t shift;        // 19, 11 or 3
  uint32_t above;        // keys in higher bins (all taken)
  uint32_t mode;         // 0 all visible keys, 1 whole bin, 2 exact score (ties limited), 3 refine next
};

struct Misc {
  uint32_t tmem;
  int nvmax;
  int abort;
  int passes_known;      // passes that certainly exist
  int passes_final;      // total passes once known (0 = not yet)
  int refine;            // some query needs another histogram pass
};

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void esync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// 16 * w as an integer weight clamped to [0, 16]; `bad` when w is off the grid
__device__ __forceinline__ int weight16p(float w, bool &bad) {
  const float f = w * 16.f;
  const int r = __float2int_rn(f);
  bad = !((float)r == f && r >= 0 && r <= 16);
  return min(max(r, 0), 16);
}

// level-0 bin of a score given as fp32 bits (score 0 -> bin 0)
__device__ __forceinline__ uint32_t bin0(uint32_t bits) {
  return bits >= 0x3F800000u ? (bits >> 19) - 2031u : 0u;
}

// packed pair of fp32 (low word first) and the two-lane fused multiply-add
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t v;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "f"(lo), "f"(hi));
  return v;
}
__device__ __forceinline__ void unpack2(uint64_t v, float &lo, float &hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// max(x, 0) of an fp32 given by its bits (negative values have the sign bit
// set, so they are negative as integers too)
__device__ __forceinline__ float relu_bits(uint32_t b) { return __int_as_float(max((int)b, 0)); }

// fp32 bits of 16 scores from the TMEM registers of 16 keys: 64 * score =
// sum_h w64_h * max(q_h . k, 0), exact (integers below 2^20)
template <int HI>
__device__ __forceinline__ void scores16(const uint32_t (&r)[4][16], const uint64_t (&w2)[4], uint32_t (&bits)[16]) {
#pragma unroll
  for (int j = 0; j < 16; j += 2) {
    uint64_t acc = pack2(0.f, 0.f);
#pragma unroll
    for (int h = 0; h < HI; ++h) acc = fma2(w2[h], pack2(relu_bits(r[h][j]), relu_bits(r[h][j + 1])), acc);
    float a, b;
    unpack2(acc, a, b);
    bits[j] = __float_as_uint(a);
    bits[j + 1] = __float_as_uint(b);
  }
}

__device__ __forceinline__ void red_add_shared(uint32_t saddr) {
  asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(saddr) : "memory");
}

template <int HI>
__device__ __forceinline__ void tmem_ld_heads16(uint32_t taddr, uint32_t (&r)[4][16]) {
#pragma unroll
  for (int h = 0; h < HI; ++h)
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[h][0]), "=r"(r[h][1]), "=r"(r[h][2]), "=r"(r[h][3]), "=r"(r[h][4]), "=r"(r[h][5]),
          "=r"(r[h][6]), "=r"(r[h][7]), "=r"(r[h][8]), "=r"(r[h][9]), "=r"(r[h][10]), "=r"(r[h][11]),
          "=r"(r[h][12]), "=r"(r[h][13]), "=r"(r[h][14]), "=r"(r[h][15])
        : "r"(taddr + h * kN));
}

// Bin where the count of this query's keys in this-or-higher bins first
// reaches `need`; the count strictly above it; the bin's own count.  The
// column is cleared for the next histogram.
__device__ __forceinline__ uint32_t find_bin_col(uint32_t *col, int nbins, uint32_t need, uint32_t &above,
                                                 uint32_t &cnt) {
  uint32_t cum = 0, sel = 0, c_sel = 0;
  bool found = false;
  for (int b = nbins - 1; b >= 0; --b) {
    const uint32_t c = col[b * kQ];
    if (!found) {
      if (cum + c >= need) { found = true; sel = (uint32_t)b; c_sel = c; }
      else cum += c;
    }
    col[b * kQ] = 0;
  }
  above = cum;
  cnt = c_sel;
  return sel;
}

// Step k of a pass of n_et tiles goes to group k & 1 as that group's
// (k >> 1)-th tile; group 0 takes tiles [0, ceil(n_et / 2)), group 1 the
// rest.  Tiles a group takes per pass:
__device__ __forceinline__ int group_tiles(int g, int n_et) { return g ? n_et >> 1 : (n_et + 1) >> 1; }

template <int HI>
__global__ void __launch_bounds__(kThr, 1)
index_prefill_kernel(const __grid_constant__ CUtensorMap kmap, const uint8_t *__restrict__ qI,
                     const float *__restrict__ w, const int32_t *__restrict__ q_pos, int Tq, int m, int n_entries,
                     int64_t entry_cap, int K, int cap, int tiles_per_seq, int ntiles, uint64_t *__restrict__ cand,
                     uint32_t *__restrict__ ccount, unsigned *status) {
  extern __shared__ __align__(1024) unsigned char smem[];
  uint32_t *hist = reinterpret_cast<uint32_t *>(smem + OFF_H);
  QState *qst = reinterpret_cast<QState *>(smem + OFF_ST);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *full = bars, *sempty = bars + kStg, *tfull = bars + 2 * kStg, *tempty = bars + 2 * kStg + 2;
  Misc *misc = reinterpret_cast<Misc *>(smem + OFF_MISC);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = ntiles - 1 - (int)blockIdx.x;           // the heaviest tiles first
  const int seq = tile / tiles_per_seq;
  const int q0 = (tile - seq * tiles_per_seq) * kQ;
  const int nq = min(kQ, Tq - q0);
  const int64_t row0 = (int64_t)seq * Tq + q0;

  // this thread's query and group (warps w and w + 4 share a lane quadrant)
  const int quad = warp & 3, grp = (warp >> 2) & 1;
  const int qi = quad * 32 + lane;
  const bool epi = warp < 8;
  const bool active = epi && qi < nq;
  int nvis = 0;
  float w64[HI];
  uint64_t w2[4];
#pragma unroll
  for (int h = 0; h < HI; ++h) w64[h] = 0.f;
  if (active) {
    const int64_t t = q_pos[row0 + qi];
    if (t < 0 && grp == 0) raise_status(status, STATUS_BAD_POSITION);
    nvis = t < 0 ? 0 : (int)min((t + 1) / m, (int64_t)n_entries);
#pragma unroll
    for (int h = 0; h < HI; ++h) {
      bool bad;
      w64[h] = (float)(4 * weight16p(w[(row0 + qi) * HI + h], bad));
      if (bad && grp == 0) raise_status(status, STATUS_BAD_WEIGHT);
    }
  }
#pragma unroll
  for (int h = 0; h < 4; ++h) w2[h] = h < HI ? pack2(w64[h], w64[h]) : 0ull;
  if (tid == 0) {
    misc->nvmax = 0;
    misc->abort = 0;
    misc->passes_final = 0;
    misc->refine = 0;
  }
  if (tid == kEpi) {
    for (int i = 0; i < kStg; ++i) { tc::mbar_init(&full[i], 1); tc::mbar_init(&sempty[i], 1); }
    for (int i = 0; i < 2; ++i) { tc::mbar_init(&tfull[i], 1); tc::mbar_init(&tempty[i], 4); }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 8) tc::tmem_alloc(&misc->tmem, kCols);
  // query tiles (A operands) in the FP4 core-matrix layout; rows past the tile are zero
  for (int c = tid; c < 4 * kQ * 2; c += kThr) {
    const int h = c / (kQ * 2), r = (c >> 1) % kQ, hf = c & 1;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (h < HI && r < nq) v = *reinterpret_cast<const uint4 *>(qI + ((row0 + r) * HI + h) * 32 + hf * 16);
    *reinterpret_cast<uint4 *>(smem + OFF_Q + h * 4096 + (r >> 3) * 256 + hf * 128 + (r & 7) * 16) = v;
  }
  for (int i = tid; i < kHistRows * kQ; i += kThr) hist[i] = 0u;
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (active && grp == 0 && nvis > 0) atomicMax(&misc->nvmax, nvis);
  const uint32_t tbase = misc->tmem;
  if (warp < 4) {     // block scales 2^0 (UE8M0 127) wherever the MMA may read them
    const uint32_t ones[4] = {0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu};
    tc::tmem_st4(tbase + ((uint32_t)(warp * 32) << 16) + kColSFA, ones);
    tc::tmem_st4(tbase + ((uint32_t)(warp * 32) << 16) + kColSFB, ones);
    tc::tmem_wait_st();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const int nvmax = misc->nvmax;
  const int n_et = (nvmax + kN - 1) / kN;
  const bool any_radix = nvmax > K;
  // pass 0 always exists; with any query over k visible keys so does pass 1
  // (histogram, then at least the collection)
  const int passes_at_start = n_et == 0 ? 0 : (any_radix ? 2 : 1);
  if (tid == 0) {
    misc->passes_known = passes_at_start;
    if (!any_radix) misc->passes_final = passes_at_start;
  }
  __syncthreads();

  auto bwait = [&](uint64_t *bar, uint32_t par) -> bool {
    if (tc::mbar_try_wait(bar, par)) return true;
    const uint64_t t0 = gtimer();
    uint32_t it = 0;
    while (!tc::mbar_try_wait(bar, par)) {
      if ((++it & 255u) == 0) {
        if (*(volatile int *)&misc->abort) return false;
        if (gtimer() - t0 > kWaitNs) { *(volatile int *)&misc->abort = 1; raise_status(status, STATUS_TIMEOUT); return false; }
      }
    }
    return true;
  };
  if (warp >= 8) {
    // ------------------------------------------------------------ control: warp 9 loads key tiles, warp 8 issues MMAs
    if (lane == 0 && n_et > 0) {
      int known = passes_at_start, fin = any_radix ? 0 : passes_at_start;
      // does pass p exist?  Past the passes known so far, wait for the
      // epilogue's decision at the end of the histogram pass before it.
      auto pass_exists = [&](int p) -> bool {
        if (p < known) return true;
        if (fin != 0) return false;
        const uint64_t t0 = gtimer();
        for (uint32_t it = 1;; ++it) {
          known = *(volatile int *)&misc->passes_known;
          fin = *(volatile int *)&misc->passes_final;
          if (p < known) return true;
          if (fin != 0 || *(volatile int *)&misc->abort) return false;
          if ((it & 255u) == 0 && gtimer() - t0 > kWaitNs) {
            *(volatile int *)&misc->abort = 1;
            raise_status(status, STATUS_TIMEOUT);
            return false;
          }
        }
      };
      bool ok = true;
      if (warp == 9) {
        // step k of a pass loads tile step_tile(k) into ring stage u % kStg
        // once the MMAs of step u - kStg are done with it
        const int ybase = (int)((int64_t)seq * entry_cap);
        const int h0 = (n_et + 1) >> 1;
        int u = 0, stg = 0, round = 0;
        for (int p = 0; ok && pass_exists(p); ++p) {
          for (int k = 0; k < n_et; ++k) {
            if (round > 0 && !bwait(&sempty[stg], (uint32_t)(round - 1) & 1u)) { ok = false; break; }
            tc::mbar_arrive_expect_tx(&full[stg], (uint32_t)kTileBytes);
            tc::tma_load_2d(smem + OFF_K + stg * kTileBytes, &kmap, 0, ybase + ((k & 1) ? h0 + (k >> 1) : (k >> 1)) * kN,
                            &full[stg]);
            ++u;
            if (++stg == kStg) { stg = 0; ++round; }
          }
        }
        // every load that was issued has landed before the CTA may exit
        for (int v = max(0, u - kStg); v < u; ++v) bwait(&full[v % kStg], (uint32_t)(v / kStg) & 1u);
      } else {
        const uint32_t idesc = tc::idesc_mxf4(128, kN);
        uint64_t adesc[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) adesc[h] = tc::smem_desc(tc::smem_u32(smem + OFF_Q + h * 4096), 128, 256);
        // stage s's descriptor: the start-address field (bits 0-13, in 16-byte units) advances by kTileBytes / 16
        const uint64_t bdesc0 = tc::smem_desc_sw32(tc::smem_u32(smem + OFF_K));
        int stg = 0, round = 0, use0 = 0, use1 = 0;
        for (int p = 0; ok && pass_exists(p); ++p) {
          for (int k = 0; k < n_et; ++k) {
            const int buf = k & 1;
            const int use = buf ? use1 : use0;   // this buffer's use count
            if (!bwait(&full[stg], (uint32_t)round & 1u)) { ok = false; break; }
            if (use >= 1 && !bwait(&tempty[buf], (uint32_t)(use - 1) & 1u)) { ok = false; break; }
            tc::fence_after_sync();
            const uint64_t bd = bdesc0 + (uint64_t)(stg * (kTileBytes >> 4));
#pragma unroll
            for (int h = 0; h < HI; ++h)
              tc::mma_mxf4_ss(tbase + buf * kBufCols + h * kN, adesc[h], bd, idesc, tbase + kColSFA, tbase + kColSFB, 0);
            tc::mma_commit(&tfull[buf]);
            tc::mma_commit(&sempty[stg]);
            if (buf) ++use1; else ++use0;
            if (++stg == kStg) { stg = 0; ++round; }
          }
        }
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue: scores, histograms, candidates
    const uint32_t taddr0 = tbase + ((uint32_t)(quad * 32) << 16) + (uint32_t)grp * kBufCols;
    uint32_t *col = hist + qi;
    // shared address of this query's level-0 counter for (score bits >> 19) = b: hbase + b * 512
    const uint32_t hbase = tc::smem_u32(col) - 2031u * (uint32_t)(kQ * 4);
    const bool radix = nvis > K;
    // mode 3 (counting) until the query's threshold is known
    uint32_t prefix = 0, shift = 19, above = 0, mode = radix ? 3u : 0u, need_eq = 0, eq_taken = 0;
    uint32_t thr = 0;                          // collection: lowest score bits taken (modes 0 and 1)
    uint32_t ncand = 0;                        // candidates this thread has written out
    uint32_t nst = 0;                          // candidates staged in shared memory
    // group 0 appends from the front of the row's list, group 1 from the back
    const int64_t cstep = grp ? -1 : 1;
    // the collection stages candidates in the (then idle) histogram area:
    // entry e of epilogue thread t at [e][t], so a warp's stores hit distinct banks
    uint64_t *stage = reinterpret_cast<uint64_t *>(smem + OFF_H);
    const uint32_t stage_me = tc::smem_u32(stage + tid);
    // Candidates of the lanes in `mask` go from shared to global memory, the
    // whole warp writing one lane's run at a time (contiguous, coalesced).
    auto flush = [&](uint32_t mask) {
      while (mask) {
        const int L = __ffs(mask) - 1;
        mask &= mask - 1;
        const uint32_t nL = __shfl_sync(0xffffffffu, nst, L);
        const uint32_t cL = __shfl_sync(0xffffffffu, ncand, L);
        const uint64_t *src = stage + (warp * 32 + L);
        uint64_t *dst = cand + (row0 + quad * 32 + L) * (int64_t)cap + (grp ? cap - 1 : 0);
        for (uint32_t e = lane; e < nL; e += 32)
          if (cL + e < (uint32_t)cap) dst[cstep * (int64_t)(cL + e)] = src[e * kEpi];
      }
    };
    // stage one candidate: fp32 bits of 64 * score above, ~index below
    auto put = [&](uint32_t bits, uint32_t s) {
      asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(stage_me + nst * (kEpi * 8)), "r"(0xFFFFFFFFu - s), "r"(bits)
                   : "memory");
      ++nst;
    };
    auto drain = [&](bool all) {   // write out staged candidates (all, or of lanes near full)
      const uint32_t m = __ballot_sync(0xffffffffu, all ? nst > 0 : nst > (uint32_t)(kStage - 16));
      if (m) {
        __syncwarp();
        flush(m);
        __syncwarp();
        if ((m >> lane) & 1u) { ncand += nst; nst = 0; }
      }
    };
    const int gt = group_tiles(grp, n_et);
    int level = any_radix ? 0 : -1;     // histogram level of the current pass, -1 = collection

    // one chunk of 16 keys starting at key s0 (registers r)
    auto chunk = [&](const uint32_t (&r)[4][16], int s0, bool ok) {
      const bool whole = active && s0 + 16 <= nvis;
      if (level == 0 && __all_sync(0xffffffffu, ok && whole && radix && mode == 3)) {
        // level-0 histogram over 16 visible keys: no per-key checks
        uint32_t bits[16];
        scores16<HI>(r, w2, bits);
#pragma unroll
        for (int j = 0; j < 16; ++j) red_add_shared(hbase + (max(bits[j] >> 19, 2031u) << 9));
        return;
      }
      if (level < 0) {
        if (__all_sync(0xffffffffu, ok && whole && mode != 2)) {
          // collection over 16 visible keys: every key at or above the
          // threshold bin's lower edge (all keys for queries in mode 0)
          uint32_t bits[16];
          scores16<HI>(r, w2, bits);
#pragma unroll
          for (int j = 0; j < 16; ++j)
            if (bits[j] >= thr) put(bits[j], (uint32_t)(s0 + j));
        } else if (active && ok) {
          // collection with per-key checks: the tail of the visible keys, or
          // an exact threshold score whose ties are taken in index order
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int s = s0 + j;
            if (s >= nvis) break;
            float f = 0.f;
#pragma unroll
            for (int h = 0; h < HI; ++h) f = fmaf(w64[h], fmaxf(__uint_as_float(r[h][j]), 0.f), f);
            const uint32_t bits = __float_as_uint(f);
            bool take = true;
            if (radix) {
              const uint32_t v = bits >> shift;
              if (v > prefix) take = true;
              else if (v < prefix) take = false;
              else if (mode == 1) take = true;
              else { take = eq_taken < need_eq; eq_taken += take ? 1u : 0u; }
            }
            if (take) put(bits, (uint32_t)s);
          }
        }
        drain(false);
        return;
      }
      // histogram of a level with per-key checks (queries past their threshold skip it)
      if (!active || !ok || !radix || mode != 3) return;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (s0 + j >= nvis) break;
        float f = 0.f;
#pragma unroll
        for (int h = 0; h < HI; ++h) f = fmaf(w64[h], fmaxf(__uint_as_float(r[h][j]), 0.f), f);
        const uint32_t bits = __float_as_uint(f);
        uint32_t b;
        if (level == 0) b = bin0(bits);
        else if ((bits >> shift) == prefix) b = (bits >> (shift - 8)) & 0xFFu;
        else continue;
        atomicAdd(&col[b * kQ], 1u);
      }
    };

    for (int p = 0; n_et > 0; ++p) {
      for (int t = 0; t < gt; ++t) {
        const int use = p * gt + t;
        const int et = grp ? ((n_et + 1) >> 1) + t : t;
        const bool ok = __all_sync(0xffffffffu, bwait(&tfull[grp], (uint32_t)use & 1u));
        tc::fence_after_sync();
        uint32_t r[4][16];
#pragma unroll
        for (int c = 0; c < kN / 16 - 1; ++c) {
          tmem_ld_heads16<HI>(taddr0 + c * 16, r);
          tc::tmem_wait_ld();
          chunk(r, et * kN + c * 16, ok);
        }
        tmem_ld_heads16<HI>(taddr0 + kN - 16, r);
        tc::tmem_wait_ld();
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&tempty[grp]);   // the buffer is free once its last chunk is in registers
        chunk(r, et * kN + kN - 16, ok);
      }
      if (level < 0) break;    // the collection was the last pass
      // ---- thresholds after histogram level `level`
      esync();
      if (radix && mode == 3 && grp == 0) {
        // mode 3 = refining; initial state enters here at level 0
        uint32_t a = 0, c = 0;
        const uint32_t need = (uint32_t)K - above;
        if (level == 0) {
          const uint32_t b = find_bin_col(col, kBins0, need, a, c);
          above += a;
          if (b == 0) { prefix = 0; shift = 19; mode = 2; need_eq = (uint32_t)K - above; }
          else { prefix = b + 2031u; shift = 19; mode = (above + c > (uint32_t)cap) ? 3 : 1; }
        } else {
          const uint32_t b = find_bin_col(col, 256, need, a, c);
          above += a;
          prefix = (prefix << 8) | b;
          shift -= 8;
          if (shift == 3) { mode = 2; need_eq = (uint32_t)K - above; }
          else mode = (above + c > (uint32_t)cap) ? 3 : 1;
        }
        qst[qi] = QState{prefix, shift, above, mode};
        if (mode == 3) atomicOr(&misc->refine, 1);
      }
      esync();
      if (radix && mode == 3 && grp == 1) {
        const QState q = qst[qi];
        prefix = q.prefix; shift = q.shift; above = q.above; mode = q.mode;
        need_eq = mode == 2 ? (uint32_t)K - above : 0u;
      }
      if (mode == 1) thr = prefix << shift;
      const bool more = *(volatile int *)&misc->refine != 0;
      esync();
      if (tid == 0) {
        misc->refine = 0;
        // pass p + 1 exists (histogram or collection); p + 2 only after another histogram
        if (more) *(volatile int *)&misc->passes_known = p + 3;
        else *(volatile int *)&misc->passes_final = p + 2;
      }
      level = more ? level + 1 : -1;
    }
    drain(true);
    if (active) ccount[2 * (row0 + qi) + grp] = min(ncand, (uint32_t)cap);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 8) tc::tmem_dealloc(tbase, kCols);
}

// Rank order: one warp per row sorts the row's candidates by score
// (descending) with a stable least-significant-digit radix sort, 8 bits per
// pass, over the score's span within the row; the candidates enter in index
// order, so equal scores leave in index order.  When span and index range fit
// in 32 bits the sort moves 32-bit composites ((max - score) << ib | (index -
// min index)) between two shared buffers; otherwise 64-bit keys move between
// a shared buffer and the row's own candidate list.  Each pass scatters in
// chunks of 32 in list order: eight ballots give every lane the set of lanes
// holding its digit, so equal digits are placed in lane order (stable), and
// the next pass's digits are counted on the way.  Writes the first k
// entries; -1 / 0 padding when the row has fewer.
constexpr int kFinWarps = 4;

__host__ __device__ constexpr int fin_warp_bytes(int cap) { return cap * 8 + 2048; }

// lanes whose 8-bit digit equals this lane's (invalid lanes pass 0x100 | x
// and match no valid lane)
__device__ __forceinline__ uint32_t same_digit_lanes(uint32_t dg, bool valid) {
  uint32_t peers = __ballot_sync(0xffffffffu, valid);
  if (!valid) peers = ~peers;
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    const uint32_t bit = (dg >> b) & 1u;
    const uint32_t B = __ballot_sync(0xffffffffu, bit != 0u);
    peers &= B ^ (bit - 1u);      // B where the bit is set, ~B where it is clear
  }
  return peers;
}

// one stable pass: digit (key >> sh) & 255, destination offsets in `cnt`
// (exclusive prefix of this pass's counts); with count_next, the counts of
// the digit at sh + 8 go to `cnt_next` (zero on entry)
template <typename T>
__device__ __forceinline__ void fin_pass(const T *src, T *dst, int c, int sh, uint32_t *cnt, uint32_t *cnt_next,
                                         bool count_next, int lane) {
  const uint32_t lt = (1u << lane) - 1u;
  for (int b0 = 0; b0 < c; b0 += 32) {
    const int j = b0 + lane;
    const bool valid = j < c;
    const T k = valid ? src[j] : (T)0;
    const uint32_t dg = (uint32_t)(k >> sh) & 255u;
    const uint32_t peers = same_digit_lanes(dg, valid);
    const int leader = __ffs(peers) - 1;
    uint32_t base = 0;
    if (valid && lane == leader) base = atomicAdd(&cnt[dg], (uint32_t)__popc(peers));
    if (count_next && valid) atomicAdd(&cnt_next[(uint32_t)(k >> (sh + 8)) & 255u], 1u);
    base = __shfl_sync(0xffffffffu, base, leader);
    if (valid) dst[base + __popc(peers & lt)] = k;
    __syncwarp();      // this chunk's offsets are taken before the next chunk's
  }
}

// exclusive prefix of the 256 counts in place: 8 per lane, then across lanes
__device__ __forceinline__ void fin_scan(uint32_t *cnt, int lane) {
  uint32_t v[8], run = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) { v[i] = run; run += cnt[lane * 8 + i]; }
  uint32_t inc = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t t = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += t;
  }
  const uint32_t excl = inc - run;
#pragma unroll
  for (int i = 0; i < 8; ++i) cnt[lane * 8 + i] = excl + v[i];
}

__global__ void __launch_bounds__(kFinWarps * 32)
topk_finish_kernel(int64_t rows, int K, int cap, uint64_t *__restrict__ cand, const uint32_t *__restrict__ ccount,
                   int32_t *__restrict__ idx_out, float *__restrict__ score_out) {
  extern __shared__ __align__(16) unsigned char fsm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kFinWarps + warp;
  if (row >= rows) return;
  unsigned char *mine = fsm + warp * fin_warp_bytes(cap);
  uint32_t *cnt0 = reinterpret_cast<uint32_t *>(mine + cap * 8);
  uint32_t *cnt1 = cnt0 + 256;
  uint32_t *k32 = reinterpret_cast<uint32_t *>(mine);
  uint64_t *k64 = reinterpret_cast<uint64_t *>(mine);
  uint64_t *gl = cand + row * cap;
  const int n0 = (int)min(ccount[2 * row], (uint32_t)cap);
  const int n1 = (int)min(ccount[2 * row + 1], (uint32_t)(cap - n0));
  const int c = n0 + n1;
  // the list in index order (front part, then the back part reversed) into
  // shared memory, all loads in flight at once; candidates carry the fp32
  // bits of 64 * score (an integer) above ~index
  for (int j = lane; j < c; j += 32)
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(tc::smem_u32(k64 + j)),
                 "l"(gl + (j < n0 ? j : cap - 1 - (j - n0)))
                 : "memory");
  asm volatile("cp.async.wait_all;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) cnt0[lane * 16 + i] = 0u;     // cnt0 and cnt1
  __syncwarp();
  uint32_t smax = 0, smin = 0xFFFFFFFFu, imax = 0, imin = 0xFFFFFFFFu;
  for (int j = lane; j < c; j += 32) {
    const uint64_t k = k64[j];
    const uint32_t sc = (uint32_t)__uint_as_float((uint32_t)(k >> 32)), ix = 0xFFFFFFFFu - (uint32_t)k;
    smax = max(smax, sc); smin = min(smin, sc);
    imax = max(imax, ix); imin = min(imin, ix);
  }
  smax = __reduce_max_sync(0xffffffffu, smax);
  smin = __reduce_min_sync(0xffffffffu, smin);
  imax = __reduce_max_sync(0xffffffffu, imax);
  imin = __reduce_min_sync(0xffffffffu, imin);
  const int sb = c > 0 ? 32 - __clz((int)(smax - smin)) : 0;   // bits of the score span
  const int ib = c > 0 ? 32 - __clz((int)(imax - imin)) : 0;   // bits of the index span
  const int passes = (sb + 7) >> 3;
  const bool narrow = sb + ib <= 32;
  const int sh0 = narrow ? ib : 32;
  __syncwarp();
  // pass keys (the score part above the index part), in place; the first
  // pass's digits counted on the way.  A narrow key j overwrites bytes of
  // wide keys below j / 2 + 16, all read by this or an earlier chunk.
  for (int b0 = 0; b0 < c; b0 += 32) {
    const int j = b0 + lane;
    const bool valid = j < c;
    uint64_t key = 0;
    if (valid) {
      const uint64_t k = k64[j];
      const uint32_t sc = (uint32_t)__uint_as_float((uint32_t)(k >> 32)), ix = 0xFFFFFFFFu - (uint32_t)k;
      key = narrow ? (((uint64_t)(smax - sc) << ib) | (uint64_t)(ix - imin)) : (((uint64_t)(smax - sc) << 32) | ix);
      atomicAdd(&cnt0[(uint32_t)(key >> sh0) & 255u], 1u);
    }
    __syncwarp();
    if (valid) {
      if (narrow) k32[j] = (uint32_t)key;
      else k64[j] = key;
    }
  }
  __syncwarp();
  // passes: narrow keys alternate between the two halves of the shared
  // buffer, wide keys between the shared buffer and the candidate list
  uint32_t *cur = cnt0, *nxt = cnt1;
  for (int p = 0; p < passes; ++p) {
    fin_scan(cur, lane);
    __syncwarp();
    const bool more = p + 1 < passes;
    const int sh = sh0 + 8 * p;
    if (narrow) {
      uint32_t *src = k32 + (p & 1) * cap, *dst = k32 + ((p + 1) & 1) * cap;
      fin_pass<uint32_t>(src, dst, c, sh, cur, nxt, more, lane);
    } else {
      uint64_t *src = (p & 1) ? gl : k64, *dst = (p & 1) ? k64 : gl;
      fin_pass<uint64_t>(src, dst, c, sh, cur, nxt, more, lane);
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) cur[lane * 8 + i] = 0u;
    uint32_t *t = cur; cur = nxt; nxt = t;
    __syncwarp();
  }
  const uint32_t imask = narrow && ib ? (uint32_t)((1ull << ib) - 1ull) : 0u;
  for (int j = lane; j < K; j += 32) {
    int32_t id = -1;
    float sc = 0.f;
    if (j < c) {
      if (narrow) {
        const uint32_t k = k32[(passes & 1) * cap + j];
        id = (int32_t)(imin + (k & imask));
        sc = (float)(smax - (uint32_t)((uint64_t)k >> ib)) * (1.f / 64.f);
      } else {
        const uint64_t k = (passes & 1) ? gl[j] : k64[j];
        id = (int32_t)(uint32_t)k;
        sc = (float)(smax - (uint32_t)(k >> 32)) * (1.f / 64.f);
      }
    }
    idx_out[row * K + j] = id;
    if (score_out) score_out[row * K + j] = sc;
  }
}

}  // namespace

// Two-pass prefill selection: shapes with more than 64 query rows, the
// 4 x 64 (or fewer heads) indexer and k <= 1024.
bool prefill2_plan(const csa_dims *d) {
  const int64_t rows = (int64_t)d->B * d->Tq;
  return d->dI == 64 && d->HI >= 1 && d->HI <= 4 && rows > 64 && d->K <= 1024 && d->n_entries >= 1 &&
         (int64_t)d->B * d->entry_cap < (1ll << 31);
}

size_t prefill2_workspace(const csa_dims *d) {
  const int64_t rows = (int64_t)d->B * d->Tq;
  const int64_t cap = 2 * (int64_t)d->K;
  return (size_t)(rows * cap * 8 + ((rows * 8 + 255) & ~255LL) + 256);
}

int launch_prefill2(const uint8_t *qI, const float *w, const uint8_t *kI, const int32_t *q_pos, const csa_dims *d,
                    int32_t *idx_out, float *score_out, void *workspace, cudaStream_t stream) {
  const int64_t rows = (int64_t)d->B * d->Tq;
  const int cap = 2 * d->K;
  uint64_t *cand = static_cast<uint64_t *>(workspace);
  uint32_t *cnt = reinterpret_cast<uint32_t *>(static_cast<char *>(workspace) + rows * cap * 8);
  CUtensorMap kmap;
  if (!encode_tmap_2d(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, kI, 32, (uint64_t)d->B * d->entry_cap, 32, 32, kN,
                      CU_TENSOR_MAP_SWIZZLE_32B))
    return fail(CSA_ERR_INVALID, "csa_index_topk: cannot map the indexer keys for TMA");
  const int tiles_per_seq = (d->Tq + kQ - 1) / kQ;
  const int ntiles = d->B * tiles_per_seq;
  unsigned *st = status_word_device_ptr();
  switch (d->HI) {
#define CSA_P2(HI_)                                                                                        \
  case HI_:                                                                                                \
    if (int rc = set_smem_once((const void *)index_prefill_kernel<HI_>, (int)SMEM, "index_prefill_kernel")) \
      return rc;                                                                                           \
    index_prefill_kernel<HI_><<<ntiles, kThr, SMEM, stream>>>(kmap, qI, w, q_pos, d->Tq, d->m, d->n_entries,  \
                                                              d->entry_cap, d->K, cap, tiles_per_seq, ntiles, \
                                                              cand, cnt, st);                              \
    break;
    CSA_P2(1) CSA_P2(2) CSA_P2(3) CSA_P2(4)
#undef CSA_P2
    default: return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk: HI=%d", d->HI);
  }
  count_launches(1);
  if (int rc = check_launch("index_prefill_kernel")) return rc;
  if (int rc = set_smem_once((const void *)topk_finish_kernel, kFinWarps * fin_warp_bytes(2048), "topk_finish_kernel"))
    return rc;
  const int fsmem = kFinWarps * fin_warp_bytes(cap);
  topk_finish_kernel<<<(unsigned)((rows + kFinWarps - 1) / kFinWarps), kFinWarps * 32, fsmem, stream>>>(
      rows, d->K, cap, cand, cnt, idx_out, score_out);
  count_launches(1);
  return check_launch("topk_finish_kernel");
}

}  // namespace csa
