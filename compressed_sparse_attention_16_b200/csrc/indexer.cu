// Lightning Indexer (FP4) scores and exact top-k selection.
//
// Page: jiwasawa.github.io DeepSeek-V4 article, section "Compressed Sparse
// Attention (CSA)" -- every query scores the compressed KV entries with a
// lightweight indexer and a top-k selector keeps the k best (DSA); page
// "DeepSeek V4とOpenCode" (hazakura.dev), section "衝撃1：CSA + HCA" -- the
// indexer runs at FP4; page "DeepSeek V4 Flash" (studioglobal.ai), section
// "アテンションのブレイクスルー" -- top 512 compressed blocks per query.
//
// Score form used by this library:
//     score(t, s) = sum_h w[t,h] * ReLU(sum_j qI[t,h,j] * kI[s,j])
// qI, kI are E2M1 and w a multiple of 1/16, so 64*score is an integer below
// 2^24.  Scores are computed in integers: 2*E2M1 is an int8 in [-12, 12] and
// 4-way int8 dot products (dp4a) give 4*(q.k) exactly.  The nibble -> int8
// conversion uses byte permutes against an 8-entry magnitude table; the sign
// of each key element is handled by splitting the key into its positive and
// negative parts (prmt's sign-replicate mode zeroes the other half).
//
// Selection: a key (score64, index) is ranked by score descending, then index
// ascending.  Each query row's threshold score is found with a two-digit
// radix select (12 bits per digit) over a shared-memory histogram, ties at
// the threshold are resolved by index, and the K survivors are sorted with a
// bitonic network.
#include "common.cuh"
#include "tc.cuh"
#include "select.cuh"

namespace csa {
namespace {

constexpr uint32_t kMagLo = 0x03020100u;   // 2*|E2M1| for codes 0..3
constexpr uint32_t kMagHi = 0x0C080604u;   // 2*|E2M1| for codes 4..7

// 16 * w as an integer weight, clamped to [0, 16] so that an off-contract
// weight (negative, above 1, NaN) can never wrap the unsigned score; `bad` is
// set when w is not a multiple of 1/16 in [0, 1] (the caller raises
// STATUS_BAD_WEIGHT for it).
__device__ __forceinline__ int weight16(float w, bool &bad) {
  const float f = w * 16.f;
  const int r = __float2int_rn(f);
  bad = !((float)r == f && r >= 0 && r <= 16);
  return min(max(r, 0), 16);
}

__device__ __forceinline__ int e2m1x2_int(uint32_t code) {   // 2*value of one 4-bit code
  const int mag = (int)((0xC8643210u >> (4 * (code & 7))) & 0xF);
  return (code & 8) ? -mag : mag;
}

// ---------------------------------------------------------------------------
// scores
// ---------------------------------------------------------------------------
constexpr int kScoreThreads = 256;
constexpr int kEPT = 4;   // entries per thread per CTA

// One query row of the indexer: 2*q as packed int8 (word 2k holds elements
// 8k..8k+3, word 2k+1 elements 8k+4..8k+7) and 16*w as integers.
template <int HI, int DI>
struct IndexQuery {
  static constexpr int NW = DI / 8;     // 32-bit key words (8 codes each)
  int qw[HI][2 * NW];
  int w16[HI];

  __device__ __forceinline__ void load(const uint8_t *qrow, const float *wrow, unsigned *status,
                                       bool report) {
#pragma unroll
    for (int h = 0; h < HI; ++h) {
      bool bad;
      w16[h] = weight16(wrow[h], bad);
      if (report && bad) raise_status(status, STATUS_BAD_WEIGHT);
#pragma unroll
      for (int k = 0; k < NW; ++k) {
        const uint32_t word = *reinterpret_cast<const uint32_t *>(qrow + h * (DI / 2) + 4 * k);
        uint32_t lo = 0, hi = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          lo |= (uint32_t)(e2m1x2_int((word >> (4 * e)) & 0xF) & 0xFF) << (8 * e);
          hi |= (uint32_t)(e2m1x2_int((word >> (4 * e + 16)) & 0xF) & 0xFF) << (8 * e);
        }
        qw[h][2 * k] = (int)lo;
        qw[h][2 * k + 1] = (int)hi;
      }
    }
  }

  __device__ __forceinline__ static void load_key(const uint8_t *krow, int64_t s, uint32_t (&kw)[NW]) {
    if constexpr (DI == 64) {
      const uint4 a = __ldg(reinterpret_cast<const uint4 *>(krow + s * 32));
      const uint4 c = __ldg(reinterpret_cast<const uint4 *>(krow + s * 32 + 16));
      kw[0] = a.x; kw[1] = a.y; kw[2] = a.z; kw[3] = a.w;
      kw[4] = c.x; kw[5] = c.y; kw[6] = c.z; kw[7] = c.w;
    } else {
      const uint4 a = __ldg(reinterpret_cast<const uint4 *>(krow + s * 16));
      kw[0] = a.x; kw[1] = a.y; kw[2] = a.z; kw[3] = a.w;
    }
  }

  // 64 * score of entry s (exact, < 2^24)
  __device__ __forceinline__ uint32_t score(const uint8_t *krow, int64_t s) const {
    uint32_t kw[NW];
    load_key(krow, s, kw);
    return score_words(kw);
  }

  __device__ __forceinline__ uint32_t score_words(const uint32_t (&kw)[NW]) const {
    int accP[HI], accN[HI];
#pragma unroll
    for (int h = 0; h < HI; ++h) { accP[h] = 0; accN[h] = 0; }
#pragma unroll
    for (int k = 0; k < NW; ++k) {
      const uint32_t u0 = kw[k];
      const uint32_t un = u0 ^ 0x88888888u;
      const int p0 = (int)prmt(kMagLo, kMagHi, u0);          // elements 0..3, positive part
      const int p1 = (int)prmt(kMagLo, kMagHi, u0 >> 16);    // elements 4..7
      const int n0 = (int)prmt(kMagLo, kMagHi, un);          // negative part magnitudes
      const int n1 = (int)prmt(kMagLo, kMagHi, un >> 16);
#pragma unroll
      for (int h = 0; h < HI; ++h) {
        accP[h] = __dp4a(p0, qw[h][2 * k], accP[h]);
        accP[h] = __dp4a(p1, qw[h][2 * k + 1], accP[h]);
        accN[h] = __dp4a(n0, qw[h][2 * k], accN[h]);
        accN[h] = __dp4a(n1, qw[h][2 * k + 1], accN[h]);
      }
    }
    uint32_t sc = 0;
#pragma unroll
    for (int h = 0; h < HI; ++h) sc += (uint32_t)(w16[h] * max(accP[h] - accN[h], 0));
    return sc;
  }
};

template <int HI, int DI>
__global__ void __launch_bounds__(kScoreThreads)
index_scores_kernel(const uint8_t *__restrict__ qI, const float *__restrict__ w,
                    const uint8_t *__restrict__ kI, const int32_t *__restrict__ q_pos, int row0,
                    int Tq, int m, int n_entries, int64_t entry_cap, uint32_t *__restrict__ scores,
                    int64_t ld, unsigned *status) {
  const int row = row0 + blockIdx.y;
  const int b = row / Tq;
  const int64_t t = q_pos[row];
  const int nvis = (int)min((t + 1) / m, (int64_t)n_entries);
  const int base = blockIdx.x * (kScoreThreads * kEPT);
  if (base >= nvis) return;
  IndexQuery<HI, DI> iq;
  iq.load(qI + (int64_t)row * HI * (DI / 2), w + (int64_t)row * HI, status,
          threadIdx.x == 0 && blockIdx.x == 0);
  const uint8_t *krow = kI + (int64_t)b * entry_cap * (DI / 2);
  uint32_t *srow = scores + (int64_t)row * ld;
#pragma unroll
  for (int u = 0; u < kEPT; ++u) {
    const int s = base + u * kScoreThreads + threadIdx.x;
    if (s >= nvis) break;
    srow[s] = iq.score(krow, s);
  }
}

// ---------------------------------------------------------------------------
// top-k selection, one CTA per query row
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 1024;
constexpr int kHistBits = 12;
constexpr int kBins = 1 << kHistBits;
constexpr int kTieCap = 2048;
constexpr int kMaxK = 2048;

__device__ __forceinline__ uint64_t make_key(uint32_t score, uint32_t idx) {
  return ((uint64_t)score << 32) | (uint64_t)(0xFFFFFFFFu - idx);
}

// Block-wide inclusive suffix sums over kBins bins, 4 bins per thread:
// finds the bin where the count of elements in higher-or-equal bins first
// reaches `need`.  Returns (bin, count strictly above bin) via shared vars.
__device__ void find_threshold_bin(const uint32_t *hist, uint32_t need, uint32_t *warp_tot,
                                   int *out_bin, uint32_t *out_above) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // thread tid owns bins [kBins - 4*(tid+1), kBins - 4*tid): thread 0 has the top bins
  const int hi_bin = kBins - 1 - 4 * tid;
  uint32_t c[4], local = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) { c[k] = hist[hi_bin - k]; local += c[k]; }
  // inclusive scan over threads (descending bin order)
  uint32_t v = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t wv = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xffffffffu, wv, o);
      if (lane >= o) wv += n;
    }
    warp_tot[lane] = wv;   // inclusive over warps
  }
  __syncthreads();
  const uint32_t incl = v + (warp > 0 ? warp_tot[warp - 1] : 0u);
  const uint32_t excl = incl - local;
  if (excl < need && incl >= need) {
    uint32_t run = excl;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if (run + c[k] >= need) { *out_bin = hi_bin - k; *out_above = run; break; }
      run += c[k];
    }
  }
  __syncthreads();
}

// Bitonic sort of n (power of two) keys in shared memory, descending.
__device__ void bitonic_desc_u64(uint64_t *a, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int p = i ^ j;
        if (p > i) {
          const bool desc = (i & k) == 0;
          const uint64_t x = a[i], y = a[p];
          if (desc ? (x < y) : (x > y)) { a[i] = y; a[p] = x; }
        }
      }
      __syncthreads();
    }
  }
}

// Bitonic sort of n (power of two) u32 in shared memory, ascending.
__device__ void bitonic_asc_u32(uint32_t *a, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int p = i ^ j;
        if (p > i) {
          const bool asc = (i & k) == 0;
          const uint32_t x = a[i], y = a[p];
          if (asc ? (x > y) : (x < y)) { a[i] = y; a[p] = x; }
        }
      }
      __syncthreads();
    }
  }
}

struct RowSelSmem {
  uint32_t hist[kBins];
  uint64_t keys[kMaxK];
  uint32_t ties[kTieCap];
  uint32_t warp_tot[32];
  int s_bin;
  uint32_t s_above, s_cgt, s_ceq, s_run;
};

// Exact top-K of the n scores S[0..n) (the entry index is the position), in
// rank order, into out_idx[0..K) / out_score[0..K) (padding -1 / 0).
// Called by all kSelThreads threads of a CTA.
__device__ void select_row(const uint32_t *__restrict__ S, int n, int K, int32_t *__restrict__ out_idx,
                           float *__restrict__ out_score, RowSelSmem &sm) {
  uint32_t *hist = sm.hist;
  uint64_t *keys = sm.keys;
  uint32_t *ties = sm.ties;
  uint32_t *warp_tot = sm.warp_tot;
  int &s_bin = sm.s_bin;
  uint32_t &s_above = sm.s_above, &s_cgt = sm.s_cgt, &s_ceq = sm.s_ceq, &s_run = sm.s_run;
  const int tid = threadIdx.x;
  int cnt;

  if (n <= K) {
    for (int j = tid; j < n; j += kSelThreads) keys[j] = make_key(S[j], (uint32_t)j);
    cnt = n;
  } else {
    // digit 1: bits [23:12]
    for (int j = tid; j < kBins; j += kSelThreads) hist[j] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += kSelThreads) atomicAdd(&hist[S[j] >> kHistBits], 1u);
    __syncthreads();
    find_threshold_bin(hist, (uint32_t)K, warp_tot, &s_bin, &s_above);
    const uint32_t b1 = (uint32_t)s_bin;
    const uint32_t above1 = s_above;
    __syncthreads();
    // digit 2: bits [11:0] within bin b1
    for (int j = tid; j < kBins; j += kSelThreads) hist[j] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += kSelThreads) {
      const uint32_t v = S[j];
      if ((v >> kHistBits) == b1) atomicAdd(&hist[v & (kBins - 1)], 1u);
    }
    __syncthreads();
    find_threshold_bin(hist, (uint32_t)K - above1, warp_tot, &s_bin, &s_above);
    const uint32_t tau = (b1 << kHistBits) | (uint32_t)s_bin;
    const uint32_t count_gt = above1 + s_above;
    const uint32_t n_eq = hist[s_bin];
    const uint32_t need_eq = (uint32_t)K - count_gt;
    if (tid == 0) { s_cgt = 0; s_ceq = 0; s_run = 0; }
    __syncthreads();
    const bool take_all_eq = (n_eq == need_eq);
    const bool tie_buffer = !take_all_eq && n_eq <= kTieCap;
    for (int j = tid; j < n; j += kSelThreads) {
      const uint32_t v = S[j];
      if (v > tau) {
        keys[atomicAdd(&s_cgt, 1u)] = make_key(v, (uint32_t)j);
      } else if (v == tau) {
        if (take_all_eq) keys[count_gt + atomicAdd(&s_ceq, 1u)] = make_key(v, (uint32_t)j);
        else if (tie_buffer) ties[atomicAdd(&s_ceq, 1u)] = (uint32_t)j;
      }
    }
    __syncthreads();
    if (tie_buffer) {
      int np = 1;
      while (np < (int)n_eq) np <<= 1;
      for (int j = (int)n_eq + tid; j < np; j += kSelThreads) ties[j] = 0xFFFFFFFFu;
      __syncthreads();
      bitonic_asc_u32(ties, np);
      for (int r = tid; r < (int)need_eq; r += kSelThreads) keys[count_gt + r] = make_key(tau, ties[r]);
    } else if (!take_all_eq) {
      // many ties: take the lowest indices by an ordered block scan
      const int lane = tid & 31, warp = tid >> 5;
      for (int j0 = 0; j0 < n; j0 += kSelThreads) {
        const int j = j0 + tid;
        const bool f = (j < n) && (S[j] == tau);
        const unsigned bal = __ballot_sync(0xffffffffu, f);
        const uint32_t wpre = __popc(bal & ((1u << lane) - 1u));
        if (lane == 0) warp_tot[warp] = __popc(bal);
        __syncthreads();
        uint32_t before = 0, total = 0;
        for (int k = 0; k < kSelThreads / 32; ++k) {
          const uint32_t c = warp_tot[k];
          if (k < warp) before += c;
          total += c;
        }
        const uint32_t rank = s_run + before + wpre;
        if (f && rank < need_eq) keys[count_gt + rank] = make_key(tau, (uint32_t)j);
        __syncthreads();
        if (tid == 0) s_run += total;
        __syncthreads();
        if (s_run >= need_eq) break;
      }
    }
    cnt = K;
  }
  __syncthreads();
  int np = 1;
  while (np < cnt) np <<= 1;
  for (int j = cnt + tid; j < np; j += kSelThreads) keys[j] = 0ull;
  __syncthreads();
  bitonic_desc_u64(keys, np);
  for (int j = tid; j < K; j += kSelThreads) {
    int32_t id = -1;
    float sc = 0.f;
    if (j < cnt) {
      const uint64_t k = keys[j];
      id = (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFu));
      sc = (float)(uint32_t)(k >> 32) * (1.f / 64.f);
    }
    out_idx[j] = id;
    if (out_score) out_score[j] = sc;
  }
}

__global__ void __launch_bounds__(kSelThreads)
topk_rows_kernel(const uint32_t *__restrict__ scores, int64_t ld, const int32_t *__restrict__ q_pos,
                 int m, int n_entries, int K, int32_t *__restrict__ idx_out,
                 float *__restrict__ score_out, unsigned *status) {
  __shared__ RowSelSmem sm;
  const int row = blockIdx.x;
  const int64_t t = q_pos[row];
  if (t < 0 && threadIdx.x == 0) raise_status(status, STATUS_BAD_POSITION);
  const int n = t < 0 ? 0 : (int)min((t + 1) / m, (int64_t)n_entries);
  select_row(scores + (int64_t)row * ld, n, K, idx_out + (int64_t)row * K,
             score_out ? score_out + (int64_t)row * K : nullptr, sm);
}

template <int HI, int DI>
void launch_scores(const uint8_t *qI, const float *w, const uint8_t *kI, const int32_t *q_pos,
                   int rows, int Tq, int m, int n_entries, int64_t entry_cap, uint32_t *scores,
                   int64_t ld, cudaStream_t stream) {
  const unsigned gx = (unsigned)((n_entries + kScoreThreads * kEPT - 1) / (kScoreThreads * kEPT));
  for (int r0 = 0; r0 < rows; r0 += 65535) {          // grid.y is limited to 65535
    const int r = rows - r0 < 65535 ? rows - r0 : 65535;
    index_scores_kernel<HI, DI><<<dim3(gx, (unsigned)r), kScoreThreads, 0, stream>>>(
        qI, w, kI, q_pos, r0, Tq, m, n_entries, entry_cap, scores, ld, status_word_device_ptr());
    count_launches(1);
  }
}

// ---------------------------------------------------------------------------
// split path for few query rows over many entries (decode): each CTA scores a
// slice of entries and keeps its exact top-K as 64-bit keys; one CTA per row
// then selects the final top-K among the slices' candidates.
// ---------------------------------------------------------------------------
constexpr int kPartThreads = 512;
constexpr int kSliceMax = 8192;
constexpr int kMergeThreads = 1024;
constexpr int kMergeCap = 20480;     // candidate keys per row held by the merge CTA (160 KiB)

using sel::find_bin;
using sel::kth_largest_key;
using sel::SelShared;
static_assert(kBins == sel::kSelBins, "selection bins");

template <int HI, int DI>
__global__ void __launch_bounds__(kPartThreads)
index_partial_kernel(const uint8_t *__restrict__ qI, const float *__restrict__ w,
                     const uint8_t *__restrict__ kI, const int32_t *__restrict__ q_pos, int Tq, int m,
                     int n_entries, int64_t entry_cap, int K, int splits, int slice,
                     uint64_t *__restrict__ cand, unsigned *status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);                 // [kSliceMax]
  uint32_t *hist = reinterpret_cast<uint32_t *>(keys + kSliceMax);         // [4096]
  SelShared *sh = reinterpret_cast<SelShared *>(hist + kBins);
  const int row = blockIdx.y, split = blockIdx.x, tid = threadIdx.x;
  const int b = row / Tq;
  int64_t t = q_pos[row];
  if (t < 0) {
    if (tid == 0 && split == 0) raise_status(status, STATUS_BAD_POSITION);
    t = -1;
  }
  const int nvis = t < 0 ? 0 : (int)min((t + 1) / m, (int64_t)n_entries);
  const int s0 = split * slice;
  const int n = max(0, min(s0 + slice, nvis) - s0);
  uint64_t *out = cand + ((int64_t)row * splits + split) * K;
  if (n == 0) {
    for (int j = tid; j < K; j += kPartThreads) out[j] = 0ull;
    return;
  }
  IndexQuery<HI, DI> iq;
  iq.load(qI + (int64_t)row * HI * (DI / 2), w + (int64_t)row * HI, status, tid == 0 && split == 0);
  const uint8_t *krow = kI + (int64_t)b * entry_cap * (DI / 2);
  constexpr int U = 4;
  for (int j0 = 0; j0 < n; j0 += kPartThreads * U) {
    uint32_t kw[U][IndexQuery<HI, DI>::NW];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * kPartThreads + tid;
      if (j < n) IndexQuery<HI, DI>::load_key(krow, s0 + j, kw[u]);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int j = j0 + u * kPartThreads + tid;
      if (j < n) keys[j] = make_key(iq.score_words(kw[u]), (uint32_t)(s0 + j));
    }
  }
  __syncthreads();
  if (n <= K) {
    for (int j = tid; j < K; j += kPartThreads) out[j] = j < n ? keys[j] : 0ull;
    return;
  }
  const uint64_t T = kth_largest_key<kPartThreads>(keys, n, K, hist, sh);
  if (tid == 0) sh->count = 0;
  __syncthreads();
  for (int j = tid; j < n; j += kPartThreads) {
    const uint64_t k = keys[j];
    if (k >= T) out[atomicAdd(&sh->count, 1u)] = k;
  }
}

// WIDE: the keys carry fp32 score bits (the block-scaled indexer) rather
// than 64 * score as an integer below 2^24.
template <bool WIDE>
__global__ void __launch_bounds__(kMergeThreads)
topk_merge_kernel(const uint64_t *__restrict__ cand, int splits, int K, const int32_t *__restrict__ q_pos,
                  int m, int n_entries, int32_t *__restrict__ idx_out, float *__restrict__ score_out) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint64_t *keys = reinterpret_cast<uint64_t *>(smem_raw);                 // [kMergeCap]
  uint64_t *best = keys + kMergeCap;                                       // [kMaxK]
  uint32_t *hist = reinterpret_cast<uint32_t *>(best + kMaxK);             // [4096]
  SelShared *sh = reinterpret_cast<SelShared *>(hist + kBins);
  const int row = blockIdx.x, tid = threadIdx.x;
  const int64_t t = q_pos[row];
  const int nvis = t < 0 ? 0 : (int)min((t + 1) / m, (int64_t)n_entries);
  const int n = splits * K;
  const uint64_t *src = cand + (int64_t)row * n;
  for (int j = tid; j < n; j += kMergeThreads) keys[j] = src[j];
  if (tid == 0) sh->count = 0;
  __syncthreads();
  const int cnt = min(K, nvis);
  // real candidates are non-zero keys; padding keys are 0 and rank last
  const uint64_t T = (nvis > K) ? kth_largest_key<kMergeThreads, WIDE>(keys, n, K, hist, sh) : 1ull;
  for (int j = tid; j < n; j += kMergeThreads) {
    const uint64_t k = keys[j];
    if (k >= T) best[atomicAdd(&sh->count, 1u)] = k;
  }
  __syncthreads();
  int np = 1;
  while (np < cnt) np <<= 1;
  for (int j = cnt + tid; j < np; j += kMergeThreads) best[j] = 0ull;
  __syncthreads();
  bitonic_desc_u64(best, np);
  for (int j = tid; j < K; j += kMergeThreads) {
    int32_t id = -1;
    float sc = 0.f;
    if (j < cnt) {
      const uint64_t k = best[j];
      id = (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFu));
      sc = WIDE ? __uint_as_float((uint32_t)(k >> 32)) : (float)(uint32_t)(k >> 32) * (1.f / 64.f);
    }
    idx_out[(int64_t)row * K + j] = id;
    if (score_out) score_out[(int64_t)row * K + j] = sc;
  }
}

// Split-path plan: slices of at most kSliceMax entries, at most kMergeCap
// candidates per row, about two CTAs per SM.  False when the row path applies.
bool split_plan(const csa_dims *d, int *splits, int *slice) {
  const int64_t rows = (int64_t)d->B * d->Tq;
  const int n = d->n_entries;
  if (rows < 1 || rows > 64 || n < 2048) return false;
  int s = (int)((2 * 148 + rows - 1) / rows);
  s = min(s, (n + 1023) / 1024);
  s = min(s, kMergeCap / d->K);
  s = max(s, (n + kSliceMax - 1) / kSliceMax);
  if (s * d->K > kMergeCap || s < 2) return false;
  *splits = s;
  *slice = (n + s - 1) / s;
  return *slice <= kSliceMax;
}

template <int HI, int DI>
void launch_partial(const uint8_t *qI, const float *w, const uint8_t *kI, const int32_t *q_pos,
                    const csa_dims *d, int splits, int slice, uint64_t *cand, cudaStream_t stream) {
  const size_t smem = kSliceMax * 8 + kBins * 4 + sizeof(SelShared);
  if (set_smem_once((const void *)index_partial_kernel<HI, DI>, (int)smem, "index_partial_kernel")) return;
  index_partial_kernel<HI, DI><<<dim3(splits, d->B * d->Tq), kPartThreads, smem, stream>>>(
      qI, w, kI, q_pos, d->Tq, d->m, d->n_entries, d->entry_cap, d->K, splits, slice, cand,
      status_word_device_ptr());
  count_launches(1);
}

// ---------------------------------------------------------------------------
// tensor-core decode path (dI = 64, HI <= 4, few query rows over many
// entries).  Scores come from one block-scaled FP4 MMA per 128 keys
// (kind::mxf4, M = 128 keys, N = 8 query rows = the heads padded with zeros,
// K = 64, every scale 2^0).  The MMA's fp32 sums of E2M1 products are exact
// (multiples of 1/4 below 2^12), so 4*acc is an integer and the score is
// rebuilt in integers.
//   scan:    keys stream HBM -> shared memory (cp.async, FP4 core-matrix
//            layout); per 1024 keys 8 MMAs into TMEM; the epilogue writes each
//            score to the workspace and counts it in a 4096-bin histogram of
//            score >> 8, added into the row's global histogram.
//   collect: every CTA derives the row's threshold bin (the bin holding the
//            K-th best score) from the global histogram and appends the keys
//            at or above it; the last CTA of the row (atomic ticket after a
//            memory fence) ranks those candidates by counting, which yields
//            the rank order directly.  If ties flood the threshold bin beyond
//            the candidate buffer, it runs the exact radix select on the
//            stored scores instead.
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 256;
constexpr int kTileKeys = 128;
constexpr int kBatchTiles = 8;
constexpr int kBatchKeys = kTileKeys * kBatchTiles;      // 1024
constexpr uint32_t kBatchBytes = kBatchKeys * 32;        // 32 KiB of packed keys
constexpr int kStages = 3;                               // key batches in shared memory
constexpr uint32_t kScanTmemCols = 256;                  // 3 x 64 accumulator + 8 scale columns
constexpr uint32_t kColSFA = 192, kColSFB = 196;
constexpr uint32_t kScanSmem = kStages * kBatchBytes + 256 + kBins * 4 + 256;   // ~113 KiB: at most 2 CTAs/SM
constexpr int kCollectSpan = 32768;                      // scores read by one collect CTA
constexpr int kCandCap = 2048;
constexpr int kCollectThreads = kSelThreads;
constexpr unsigned long long kScanWaitNs = 2000000000ull;

struct TcWs {
  uint32_t *scores;   // [rows][ld]
  uint32_t *hist;     // [rows][4096]
  uint64_t *cand;     // [rows][kCandCap]
  uint32_t *ccount;   // [rows]
  uint32_t *done;     // [rows] collect tickets
  uint32_t *sdone;    // [rows] scan tickets
  uint32_t *meta;     // [rows][2]: threshold bin, candidate count (written by the last scan CTA)
};

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

template <int HI>
__global__ void __launch_bounds__(kScanThreads, 2)
index_scan_tc_kernel(const uint8_t *__restrict__ qI, const float *__restrict__ w,
                     const uint8_t *__restrict__ kI, const int32_t *__restrict__ q_pos, int Tq, int m,
                     int n_entries, int64_t entry_cap, int K, int slice, TcWs ws, int64_t ld,
                     unsigned *status) {
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char *kbuf = smem;                                          // [kStages][32 KiB]
  unsigned char *qbuf = smem + kStages * kBatchBytes;                  // 8 rows x 32 B
  uint32_t *hist = reinterpret_cast<uint32_t *>(qbuf + 256);           // [4096]
  uint64_t *bars = reinterpret_cast<uint64_t *>(hist + kBins);         // [kStages]
  uint32_t *tptr = reinterpret_cast<uint32_t *>(bars + kStages);
  int *abort_flag = reinterpret_cast<int *>(tptr + 1);
  int *last_flag = abort_flag + 1;
  SelShared *sel = reinterpret_cast<SelShared *>(abort_flag + 2);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.y, split = blockIdx.x;
  const int b = row / Tq;
  const int64_t t = q_pos[row];
  if (t < 0 && tid == 0 && split == 0) raise_status(status, STATUS_BAD_POSITION);
  const int nvis = t < 0 ? 0 : (int)min((t + 1) / m, (int64_t)n_entries);
  const int s0 = split * slice;
  const int s1 = min(s0 + slice, nvis);
  const uint8_t *krow = kI + (int64_t)b * entry_cap * 32;
  const int n = max(0, s1 - s0);
  const int nb = (n + kBatchKeys - 1) / kBatchKeys;
  auto load = [&](int bb) {
    unsigned char *buf = kbuf + (bb % kStages) * kBatchBytes;
    const int base = s0 + bb * kBatchKeys;
    for (int c = tid; c < 2 * kBatchKeys; c += kScanThreads) {
      const int r = c >> 1, h = c & 1;
      const int s = base + r;
      unsigned char *dst = buf + (r >> 7) * 4096 + ((r & 127) >> 3) * 256 + h * 128 + (r & 7) * 16;
      const bool ok = s < s1;
      tc::cp_async16(dst, ok ? (const void *)(krow + (int64_t)s * 32 + h * 16) : (const void *)krow, ok ? 16u : 0u);
    }
    tc::cp_async_commit();
  };
  // start the key stream before any set-up
  for (int bb = 0; bb < kStages - 1; ++bb) {
    if (bb < nb) load(bb); else tc::cp_async_commit();
  }

  if (warp == 0) tc::tmem_alloc(tptr, kScanTmemCols);
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) tc::mbar_init(&bars[i], 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int i = tid; i < kBins; i += kScanThreads) hist[i] = 0;
  // query tile, FP4 core-matrix layout: row r, K-half c at c*128 + r*16 (rows >= HI are zero)
  if (tid < 16) {
    const int r = tid & 7, c = tid >> 3;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < HI) v = *reinterpret_cast<const uint4 *>(qI + ((int64_t)row * HI + r) * 32 + c * 16);
    *reinterpret_cast<uint4 *>(qbuf + c * 128 + r * 16) = v;
  }
  int w16[HI];
#pragma unroll
  for (int h = 0; h < HI; ++h) {
    bool bad;
    w16[h] = weight16(w[(int64_t)row * HI + h], bad);
    if (tid == 0 && split == 0 && bad) raise_status(status, STATUS_BAD_WEIGHT);
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tptr;
  if (warp < 4) {     // block scales = 2^0 (UE8M0 127) in every byte the MMA may read
    const uint32_t ones[4] = {0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu};
    tc::tmem_st4(tbase + ((uint32_t)(warp * 32) << 16) + kColSFA, ones);
    tc::tmem_st4(tbase + ((uint32_t)(warp * 32) << 16) + kColSFB, ones);
    tc::tmem_wait_st();
  }

  const uint32_t idesc = tc::idesc_mxf4(128, 8);
  for (int bb = 0; bb < nb; ++bb) {
    tc::cp_async_wait<kStages - 2>();      // batch bb has landed (one group is committed per batch)
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const int stg = bb % kStages;
    const uint32_t par = (uint32_t)(bb / kStages) & 1u;
    if (tid == 0) {
      const uint32_t buf = tc::smem_u32(kbuf + stg * kBatchBytes);
      const uint64_t bd = tc::smem_desc(tc::smem_u32(qbuf), 128, 256);
#pragma unroll
      for (int i = 0; i < kBatchTiles; ++i)
        tc::mma_mxf4_ss(tbase + stg * 64 + i * 8, tc::smem_desc(buf + i * 4096, 128, 256), bd, idesc,
                        tbase + kColSFA, tbase + kColSFB, 0);
      tc::mma_commit(&bars[stg]);
    }
    // bounded wait for the batch's MMAs
    bool ok = tc::mbar_try_wait(&bars[stg], par);
    if (!ok) {
      const uint64_t t0 = gtimer();
      uint32_t it = 0;
      while (!(ok = tc::mbar_try_wait(&bars[stg], par))) {
        if ((++it & 255u) == 0 && (*(volatile int *)abort_flag || gtimer() - t0 > kScanWaitNs)) {
          if (!*(volatile int *)abort_flag) raise_status(status, STATUS_TIMEOUT);
          *(volatile int *)abort_flag = 1;
          break;
        }
      }
    }
    tc::fence_after_sync();
    if (ok) {
      const int q = warp & 3;
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        const int tile = (warp >> 2) * 4 + i4;
        uint32_t acc[4];
        tc::tmem_ld4(tbase + ((uint32_t)(q * 32) << 16) + stg * 64 + tile * 8, acc);
        tc::tmem_wait_ld();
        const int s = s0 + bb * kBatchKeys + tile * kTileKeys + q * 32 + lane;
        if (s < s1) {
          uint32_t sc = 0;
#pragma unroll
          for (int h = 0; h < HI; ++h)
            sc += (uint32_t)(w16[h] * max(0, __float2int_rn(4.f * __uint_as_float(acc[h]))));
          ws.scores[(int64_t)row * ld + s] = sc;
          atomicAdd(&hist[sc >> 8], 1u);
        }
      }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (*(volatile int *)abort_flag) break;
    if (bb + kStages - 1 < nb) load(bb + kStages - 1); else tc::cp_async_commit();
  }
  tc::cp_async_wait<0>();
  for (int i = tid; i < kBins; i += kScanThreads) {
    const uint32_t c = hist[i];
    if (c) atomicAdd(&ws.hist[(int64_t)row * kBins + i], c);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tbase, kScanTmemCols);
  // the row's last scan CTA derives the threshold bin from the complete histogram
  __threadfence();
  if (tid == 0) *last_flag = atomicAdd(&ws.sdone[row], 1u) == gridDim.x - 1;
  __syncthreads();
  if (!*last_flag) return;
  __threadfence();
  uint32_t bstar = 0, C = (uint32_t)nvis;
  if (nvis > K) {
    // L2-coherent loads (not cached in L1), issued together
    const uint4 *G = reinterpret_cast<const uint4 *>(ws.hist + (int64_t)row * kBins);
    for (int i = tid; i < kBins / 4; i += kScanThreads) reinterpret_cast<uint4 *>(hist)[i] = __ldcg(G + i);
    __syncthreads();
    find_bin<kScanThreads>(hist, (uint32_t)K, sel->warp_tot, &sel->bin, &sel->above);
    bstar = (uint32_t)sel->bin;
    C = sel->above + hist[bstar];
  }
  if (tid == 0) {
    ws.meta[2 * row] = bstar;
    ws.meta[2 * row + 1] = C;
  }
}

__global__ void __launch_bounds__(kCollectThreads)
index_collect_kernel(const int32_t *__restrict__ q_pos, int m, int n_entries, int K, int span, TcWs ws,
                     int64_t ld, int32_t *__restrict__ idx_out, float *__restrict__ score_out) {
  __shared__ RowSelSmem sm;
  __shared__ int s_last;
  const int tid = threadIdx.x;
  const int row = blockIdx.y, split = blockIdx.x;
  const int64_t t = q_pos[row];
  const int nvis = t < 0 ? 0 : (int)min((t + 1) / m, (int64_t)n_entries);
  const uint32_t *S = ws.scores + (int64_t)row * ld;
  uint32_t bstar = 0, C = (uint32_t)nvis;
  if (nvis > 0) {
    bstar = ws.meta[2 * row];
    C = ws.meta[2 * row + 1];
  }
  const int slice = span;
  const bool degenerate = C > (uint32_t)kCandCap;
  if (!degenerate) {
    // slice starts are multiples of 4 and rows are 16-byte aligned: read 4 scores at a time
    const int j0 = split * slice;
    const int j1 = min(j0 + slice, nvis);
    uint64_t *cand = ws.cand + (int64_t)row * kCandCap;
    const uint4 *S4 = reinterpret_cast<const uint4 *>(S + j0);
    const int nq = (j1 - j0 + 3) >> 2;
    constexpr int U = 4;
    for (int q0 = 0; q0 < nq; q0 += kCollectThreads * U) {
      uint4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int qi = q0 + u * kCollectThreads + tid;
        v[u] = qi < nq ? __ldcg(S4 + qi) : make_uint4(0, 0, 0, 0);
      }
      const int lane = tid & 31;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int jb = j0 + 4 * (q0 + u * kCollectThreads + tid);
        const uint32_t sv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = jb + e;
          const bool take = j < j1 && (sv[e] >> 8) >= bstar;
          // one atomic per warp for all of its candidates
          const unsigned msk = __ballot_sync(0xffffffffu, take);
          if (msk) {
            const int leader = __ffs(msk) - 1;
            uint32_t base = 0;
            if (lane == leader) base = atomicAdd(&ws.ccount[row], (uint32_t)__popc(msk));
            base = __shfl_sync(0xffffffffu, base, leader);
            if (take) {
              const uint32_t pos = base + __popc(msk & ((1u << lane) - 1u));
              if (pos < (uint32_t)kCandCap) cand[pos] = make_key(sv[e], (uint32_t)j);
            }
          }
        }
      }
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicAdd(&ws.done[row], 1u) == gridDim.x - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  int32_t *oi = idx_out + (int64_t)row * K;
  float *os = score_out ? score_out + (int64_t)row * K : nullptr;
  if (degenerate) {
    select_row(S, nvis, K, oi, os, sm);
    return;
  }
  const int cnt = min(K, nvis);
  C = min(C, min(*(volatile uint32_t *)&ws.ccount[row], (uint32_t)kCandCap));
  uint64_t *keys = sm.keys;                         // C <= kCandCap == kMaxK
  const uint64_t *cand = ws.cand + (int64_t)row * kCandCap;
  int np = 1;
  while (np < (int)C) np <<= 1;
  for (int i = tid; i < np; i += kCollectThreads) keys[i] = i < (int)C ? __ldcg(cand + i) : 0ull;
  __syncthreads();
  // keys are distinct: after a descending sort the first cnt are the answer in rank order
  bitonic_desc_u64(keys, np);
  for (int r = tid; r < cnt; r += kCollectThreads) {
    const uint64_t k = keys[r];
    oi[r] = (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFu));
    if (os) os[r] = (float)(uint32_t)(k >> 32) * (1.f / 64.f);
  }
  for (int j = cnt + tid; j < K; j += kCollectThreads) {
    oi[j] = -1;
    if (os) os[j] = 0.f;
  }
}

// Tensor-core decode plan: about two CTAs per SM over the rows' entries.
bool tc_plan(const csa_dims *d, int *splits, int *slice) {
  const int64_t rows = (int64_t)d->B * d->Tq;
  const int n = d->n_entries;
  if (d->dI != 64 || d->HI > 4 || rows < 1 || rows > 64 || n < 2048 || d->K > kMaxK) return false;
  int s = (int)((2 * 148 + rows - 1) / rows);
  s = min(s, (n + 1023) / 1024);
  s = max(s, 1);
  *splits = s;
  *slice = (n + s - 1) / s;
  return true;
}

size_t tc_workspace(const csa_dims *d, TcWs *ws, void *base) {
  const int64_t rows = (int64_t)d->B * d->Tq;
  const int64_t ld = ((int64_t)d->n_entries + 3) & ~3LL;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off += (bytes + 255) & ~(size_t)255; return o; };
  const size_t o_scores = take((size_t)(rows * ld * 4));
  const size_t o_hist = take((size_t)(rows * kBins * 4));
  const size_t o_cand = take((size_t)(rows * kCandCap * 8));
  const size_t o_cnt = take((size_t)(rows * 4));
  const size_t o_done = take((size_t)(rows * 4));
  const size_t o_sdone = take((size_t)(rows * 4));
  const size_t o_meta = take((size_t)(rows * 8));
  if (ws && base) {
    char *p = static_cast<char *>(base);
    ws->scores = reinterpret_cast<uint32_t *>(p + o_scores);
    ws->hist = reinterpret_cast<uint32_t *>(p + o_hist);
    ws->cand = reinterpret_cast<uint64_t *>(p + o_cand);
    ws->ccount = reinterpret_cast<uint32_t *>(p + o_cnt);
    ws->done = reinterpret_cast<uint32_t *>(p + o_done);
    ws->sdone = reinterpret_cast<uint32_t *>(p + o_sdone);
    ws->meta = reinterpret_cast<uint32_t *>(p + o_meta);
  }
  return off;
}

int launch_tc(const uint8_t *qI, const float *w, const uint8_t *kI, const int32_t *q_pos,
              const csa_dims *d, int splits, int slice, int32_t *idx_out, float *score_out,
              void *workspace, cudaStream_t stream) {
  TcWs ws;
  tc_workspace(d, &ws, workspace);
  const int rows = d->B * d->Tq;
  const int64_t ld = ((int64_t)d->n_entries + 3) & ~3LL;
  // the histogram and the counters start at zero on every call
  const size_t zero_bytes = (size_t)((char *)ws.meta - (char *)ws.hist) + (size_t)rows * 8;
  if (cudaMemsetAsync(ws.hist, 0, zero_bytes, stream) != cudaSuccess) return check_launch("cudaMemsetAsync");
  if (int rc = set_smem_once((const void *)index_scan_tc_kernel<4>, (int)kScanSmem, "index_scan_tc_kernel")) return rc;
  if (int rc = set_smem_once((const void *)index_scan_tc_kernel<2>, (int)kScanSmem, "index_scan_tc_kernel")) return rc;
  if (int rc = set_smem_once((const void *)index_scan_tc_kernel<1>, (int)kScanSmem, "index_scan_tc_kernel")) return rc;
  if (int rc = set_smem_once((const void *)index_scan_tc_kernel<3>, (int)kScanSmem, "index_scan_tc_kernel")) return rc;
  const dim3 grid(splits, rows);
  unsigned *st = status_word_device_ptr();
  switch (d->HI) {
    case 1: index_scan_tc_kernel<1><<<grid, kScanThreads, kScanSmem, stream>>>(qI, w, kI, q_pos, d->Tq, d->m, d->n_entries, d->entry_cap, d->K, slice, ws, ld, st); break;
    case 2: index_scan_tc_kernel<2><<<grid, kScanThreads, kScanSmem, stream>>>(qI, w, kI, q_pos, d->Tq, d->m, d->n_entries, d->entry_cap, d->K, slice, ws, ld, st); break;
    case 3: index_scan_tc_kernel<3><<<grid, kScanThreads, kScanSmem, stream>>>(qI, w, kI, q_pos, d->Tq, d->m, d->n_entries, d->entry_cap, d->K, slice, ws, ld, st); break;
    default: index_scan_tc_kernel<4><<<grid, kScanThreads, kScanSmem, stream>>>(qI, w, kI, q_pos, d->Tq, d->m, d->n_entries, d->entry_cap, d->K, slice, ws, ld, st); break;
  }
  count_launches(1);
  if (int rc = check_launch("index_scan_tc_kernel")) return rc;
  const int csplits = (d->n_entries + kCollectSpan - 1) / kCollectSpan;
  const int cspan = (((d->n_entries + csplits - 1) / csplits) + 3) & ~3;   // multiple of 4
  index_collect_kernel<<<dim3(csplits, rows), kCollectThreads, 0, stream>>>(q_pos, d->m, d->n_entries, d->K, cspan,
                                                                           ws, ld, idx_out, score_out);
  count_launches(1);
  return check_launch("index_collect_kernel");
}

// ---------------------------------------------------------------------------
// fused decode path: one cooperative launch, one CTA per SM, per_row CTAs per
// query row, each owning a contiguous range of <= 8192 visible entries.
//   scan     keys stream through a 4-stage ring of TMA tensor loads (32-byte
//            swizzle, the layout the MMA reads); per 1024-key batch eight
//            kind::mxf4 MMAs give exact q.k sums into one of two TMEM
//            buffers, so the MMAs of batch b overlap the epilogue of b - 1;
//            the integer scores stay in shared memory and are counted in a
//            4096-bin histogram of score >> 8, which the CTA then adds into
//            the row's global histogram.
//   barrier  (bounded grid barrier)
//   collect  every CTA finds the row's threshold bin b* and appends its keys
//            of bin >= b* to the row's candidate list.  If b* holds so many
//            keys that the list would overflow (heavy ties), the row is
//            refined instead: a 256-bin histogram of the low score byte inside
//            b* fixes the exact threshold score t*; keys above t* are taken,
//            and the ties at t* in index order, each CTA taking its share after
//            the tie counts of the CTAs before it (two more barriers, entered
//            by the whole grid when any row needs them).
//   rank     the candidates are unique 64-bit keys (score, ~index); each is
//            ranked by counting the larger ones, spread over the row's CTAs,
//            and written at its rank when that is below K.
// ---------------------------------------------------------------------------
constexpr int kFdThreads = 256;
constexpr int kFdStages = 4;
constexpr int kFdLocalCap = 8192;
constexpr uint32_t kFdOffScores = kFdStages * kBatchBytes;            // u32 [8192]
constexpr uint32_t kFdOffHist = kFdOffScores + kFdLocalCap * 4;       // u32 [4096]
constexpr uint32_t kFdOffQ = kFdOffHist + kBins * 4;                  // 8 rows x 32 B
constexpr uint32_t kFdOffBar = kFdOffQ + 256;
constexpr uint32_t kFdOffMisc = kFdOffBar + 64;
constexpr uint32_t kFdSmem = kFdOffMisc + 256;
constexpr uint32_t kFdTmemCols = 256;                                 // 2 x 64 accumulator + scale columns
constexpr uint32_t kFdColSFA = 128, kFdColSFB = 132;

struct FdWs {
  uint64_t *cand;     // [rows][kCandCap]
  uint32_t *hist;     // [rows][4096]     (zeroed per call from here on)
  uint32_t *hist2;    // [rows][256]
  uint32_t *ccount;   // [rows]
  uint32_t *tiecnt;   // [rows * per_row]
  uint32_t *sync;     // grid barrier counter
  uint32_t *flag;     // some row needs the refinement
};

struct FdMisc {
  uint32_t tmem;
  int abort;
  SelShared sel;
  uint32_t cnt[8];
  uint32_t tstar, take, base;
};

// Bounded grid barrier number k (1, 2, ...) over G CTAs of a cooperative
// launch: arrive, then wait until all G arrived.  A CTA whose wait gave up
// raises STATUS_TIMEOUT and stops waiting at later barriers (it still arrives).
__device__ __forceinline__ void fd_grid_barrier(uint32_t *ctr, uint32_t k, uint32_t G, FdMisc *misc,
                                                unsigned *status) {
  __syncthreads();
  if (threadIdx.x == 0) {
    // release: the CTA's writes (ordered before by the CTA barrier) become
    // visible before the arrival; acquire on the loads that see all arrivals
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
    if (!misc->abort) {
      const uint64_t t0 = gtimer();
      uint32_t v, n = 0;
      for (;;) {
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= k * G) break;
        if ((++n & 63u) == 0 && gtimer() - t0 > kScanWaitNs) {
          misc->abort = 1;
          raise_status(status, STATUS_TIMEOUT);
          break;
        }
      }
    }
  }
  __syncthreads();
}

// Warp-aggregated append of `key` (when take) to a global list with counter.
__device__ __forceinline__ void fd_append(bool take, uint64_t key, uint32_t *count, uint64_t *list, uint32_t cap) {
  const int lane = threadIdx.x & 31;
  const unsigned msk = __ballot_sync(0xffffffffu, take);
  if (!msk) return;
  const int leader = __ffs(msk) - 1;
  uint32_t base = 0;
  if (lane == leader) base = atomicAdd(count, (uint32_t)__popc(msk));
  base = __shfl_sync(0xffffffffu, base, leader);
  if (take) {
    const uint32_t pos = base + __popc(msk & ((1u << lane) - 1u));
    if (pos < cap) list[pos] = key;
  }
}

// Exclusive prefix of v over the CTA (kFdThreads threads) and the total.
__device__ __forceinline__ uint32_t fd_block_scan(uint32_t v, uint32_t *warp_tot, uint32_t *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  uint32_t before = 0, tot = 0;
#pragma unroll
  for (int k = 0; k < kFdThreads / 32; ++k) {
    const uint32_t t = warp_tot[k];
    before += (k < warp) ? t : 0u;
    tot += t;
  }
  *total = tot;
  return before + x - v;
}

template <int HI>
__global__ void __launch_bounds__(kFdThreads, 1)
index_decode_kernel(const __grid_constant__ CUtensorMap kmap, const uint8_t *__restrict__ qI,
                    const float *__restrict__ w, const int32_t *__restrict__ q_pos, int Tq, int m, int n_entries,
                    int64_t entry_cap, int K, int per_row, FdWs ws, int32_t *__restrict__ idx_out,
                    float *__restrict__ score_out, unsigned *status) {
  extern __shared__ __align__(1024) unsigned char smem[];
  unsigned char *kbuf = smem;
  uint32_t *sc = reinterpret_cast<uint32_t *>(smem + kFdOffScores);
  uint32_t *hist = reinterpret_cast<uint32_t *>(smem + kFdOffHist);
  unsigned char *qbuf = smem + kFdOffQ;
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + kFdOffBar);
  FdMisc *misc = reinterpret_cast<FdMisc *>(smem + kFdOffMisc);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t G = gridDim.x;
  const int row = blockIdx.x / per_row, part = blockIdx.x - row * per_row;
  const int b = row / Tq;
  const int64_t t = q_pos[row];
  if (t < 0 && tid == 0 && part == 0) raise_status(status, STATUS_BAD_POSITION);
  const int nvis = t < 0 ? 0 : (int)min((t + 1) / m, (int64_t)n_entries);
  const int slice = (nvis + per_row - 1) / per_row;
  const int s0 = min(part * slice, nvis), s1 = min(s0 + slice, nvis);
  const int n = s1 - s0;
  const int nb = (n + kBatchKeys - 1) / kBatchKeys;
  const int ybase = (int)((int64_t)b * entry_cap + s0);    // row of the key tensor (< 2^31)
  uint64_t *full = bar;                                    // [kFdStages] key batch landed
  uint64_t *mdone = bar + kFdStages;                       // [2] accumulator buffer complete
  // batch bb: keys [bb * 1024, +1024) of the range, as 256-row TMA boxes
  // (boxes wholly past the range are skipped; rows past it inside a box are
  // loaded and masked)
  auto issue = [&](int bb) {
    const int slot = bb % kFdStages;
    const int boxes = min(4, (n - bb * kBatchKeys + 255) >> 8);
    tc::mbar_arrive_expect_tx(&full[slot], (uint32_t)boxes * 8192u);
    for (int i = 0; i < boxes; ++i)
      tc::tma_load_2d(kbuf + slot * kBatchBytes + i * 8192, &kmap, 0, ybase + bb * kBatchKeys + i * 256,
                      &full[slot]);
  };
  if (tid == 0) {
    for (int i = 0; i < kFdStages + 2; ++i) tc::mbar_init(&bar[i], 1);
    misc->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int bb = 0; bb < min(kFdStages, nb); ++bb) issue(bb);
  }
  if (warp == 0) tc::tmem_alloc(&misc->tmem, kFdTmemCols);
  for (int i = tid; i < kBins; i += kFdThreads) hist[i] = 0;
  if (tid < 16) {
    const int r = tid & 7, c = tid >> 3;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < HI) v = *reinterpret_cast<const uint4 *>(qI + ((int64_t)row * HI + r) * 32 + c * 16);
    *reinterpret_cast<uint4 *>(qbuf + c * 128 + r * 16) = v;
  }
  int w16[HI];
#pragma unroll
  for (int h = 0; h < HI; ++h) {
    bool bad;
    w16[h] = weight16(w[(int64_t)row * HI + h], bad);
    if (tid == 0 && part == 0 && bad) raise_status(status, STATUS_BAD_WEIGHT);
  }
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = misc->tmem;
  if (warp < 4) {     // block scales = 2^0 (UE8M0 127) in every byte the MMA may read
    const uint32_t ones[4] = {0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu};
    tc::tmem_st4(tbase + ((uint32_t)(warp * 32) << 16) + kFdColSFA, ones);
    tc::tmem_st4(tbase + ((uint32_t)(warp * 32) << 16) + kFdColSFB, ones);
    tc::tmem_wait_st();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();

  // bounded wait on an mbarrier phase; gives up (and marks the CTA) after 2 s
  auto bwait = [&](uint64_t *bb_, uint32_t par) -> bool {
    if (*(volatile int *)&misc->abort) return false;
    if (tc::mbar_try_wait(bb_, par)) return true;
    const uint64_t t0 = gtimer();
    uint32_t it = 0;
    while (!tc::mbar_try_wait(bb_, par)) {
      if ((++it & 255u) == 0 && (*(volatile int *)&misc->abort || gtimer() - t0 > kScanWaitNs)) {
        if (!*(volatile int *)&misc->abort) raise_status(status, STATUS_TIMEOUT);
        *(volatile int *)&misc->abort = 1;
        return false;
      }
    }
    return true;
  };

  // ---- scan
  const uint32_t idesc = tc::idesc_mxf4(128, 8);
  const uint64_t bd = tc::smem_desc(tc::smem_u32(qbuf), 128, 256);
  for (int bb = 0; bb <= nb; ++bb) {
    if (bb < nb && tid == 0) {
      const int slot = bb % kFdStages;
      if (bwait(&full[slot], (uint32_t)(bb / kFdStages) & 1u)) {
        tc::fence_after_sync();
        const uint32_t buf = tc::smem_u32(kbuf + slot * kBatchBytes);
        const uint32_t acc = tbase + (uint32_t)(bb & 1) * 64;
#pragma unroll
        for (int i = 0; i < kBatchTiles; ++i)
          tc::mma_mxf4_ss(acc + i * 8, tc::smem_desc_sw32(buf + i * 4096), bd, idesc, tbase + kFdColSFA,
                          tbase + kFdColSFB, 0);
      }
      tc::mma_commit(&mdone[bb & 1]);
    }
    if (bb > 0) {
      const int pb = bb - 1;
      // one decision per warp: the TMEM loads below are warp-collective
      const bool ok = __all_sync(0xffffffffu, bwait(&mdone[pb & 1], (uint32_t)(pb >> 1) & 1u));
      tc::fence_after_sync();
      // the key slot of batch pb is free again
      if (tid == 0 && pb + kFdStages < nb) issue(pb + kFdStages);
      const int q = warp & 3;
      uint32_t acc[4][4];
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        acc[i4][0] = acc[i4][1] = acc[i4][2] = acc[i4][3] = 0u;
        if (ok) tc::tmem_ld4(tbase + ((uint32_t)(q * 32) << 16) + (uint32_t)(pb & 1) * 64 + ((warp >> 2) * 4 + i4) * 8,
                             acc[i4]);
      }
      tc::tmem_wait_ld();
#pragma unroll
      for (int i4 = 0; i4 < 4; ++i4) {
        const int tile = (warp >> 2) * 4 + i4;
        const int j = pb * kBatchKeys + tile * kTileKeys + q * 32 + lane;   // local index
        const bool valid = j < n;
        uint32_t s = 0;
#pragma unroll
        for (int h = 0; h < HI; ++h)
          s += (uint32_t)(w16[h] * max(0, __float2int_rn(4.f * __uint_as_float(acc[i4][h]))));
        if (valid) {
          sc[j] = s;
          atomicAdd(&hist[s >> 8], 1u);
        }
      }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
  }
  // add the CTA's histogram into the row's (the scores occupy few bins)
  uint32_t *ghist = ws.hist + (int64_t)row * kBins;
  for (int i = tid; i < kBins; i += kFdThreads) {
    const uint32_t c = hist[i];
    if (c) atomicAdd(&ghist[i], c);
  }
  fd_grid_barrier(ws.sync, 1, G, misc, status);

  // ---- collect
  uint32_t bstar = 0, above = 0, C = (uint32_t)nvis;
  if (nvis > K) {
    const uint4 *G4 = reinterpret_cast<const uint4 *>(ghist);
    for (int i = tid; i < kBins / 4; i += kFdThreads) reinterpret_cast<uint4 *>(hist)[i] = __ldcg(G4 + i);
    __syncthreads();
    find_bin<kFdThreads>(hist, (uint32_t)K, misc->sel.warp_tot, &misc->sel.bin, &misc->sel.above);
    bstar = (uint32_t)misc->sel.bin;
    above = misc->sel.above;
    C = above + hist[bstar];
  }
  const bool refine = C > (uint32_t)kCandCap;
  uint64_t *cand = ws.cand + (int64_t)row * kCandCap;
  uint32_t *ccount = ws.ccount + row;
  if (!refine) {
    // count, reserve the CTA's block of the list with one atomic, then write
    uint32_t mine = 0;
    for (int j = tid; j < n; j += kFdThreads) mine += (sc[j] >> 8) >= bstar ? 1u : 0u;
    uint32_t total;
    uint32_t pos = fd_block_scan(mine, misc->cnt, &total);
    if (tid == 0) misc->base = total ? atomicAdd(ccount, total) : 0u;
    __syncthreads();
    pos += misc->base;
    for (int j = tid; j < n; j += kFdThreads) {
      const uint32_t s = sc[j];
      if ((s >> 8) >= bstar) {
        if (pos < (uint32_t)kCandCap) cand[pos] = make_key(s, (uint32_t)(s0 + j));
        ++pos;
      }
    }
  } else {
    if (tid == 0 && part == 0) atomicOr(ws.flag, 1u);
    __syncthreads();
    for (int i = tid; i < 256; i += kFdThreads) hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < n; j += kFdThreads) {
      const uint32_t s = sc[j];
      if ((s >> 8) == bstar) atomicAdd(&hist[s & 255u], 1u);
    }
    __syncthreads();
    for (int i = tid; i < 256; i += kFdThreads)
      if (hist[i]) atomicAdd(&ws.hist2[row * 256 + i], hist[i]);
  }
  fd_grid_barrier(ws.sync, 2, G, misc, status);

  if (*(volatile uint32_t *)ws.flag) {       // the same decision in every CTA
    uint32_t tstar = 0, take_ties = 0;
    if (refine) {
      if (tid == 0) {
        const uint32_t need = (uint32_t)K - above;
        uint32_t run = 0;
        int lo = 255;
        for (; lo > 0; --lo) {
          const uint32_t c = __ldcg(ws.hist2 + row * 256 + lo);
          if (run + c >= need) break;
          run += c;
        }
        misc->tstar = (bstar << 8) | (uint32_t)lo;
        misc->take = need - run;   // ties at t* to take
      }
      __syncthreads();
      tstar = misc->tstar;
      take_ties = misc->take;
      uint32_t myties = 0;
      for (int j0 = 0; j0 < n; j0 += kFdThreads) {
        const int j = j0 + tid;
        const uint32_t s = j < n ? sc[j] : 0u;
        fd_append(j < n && s > tstar, make_key(s, (uint32_t)(s0 + j)), ccount, cand, kCandCap);
        myties += (j < n && s == tstar) ? 1u : 0u;
      }
      myties = __reduce_add_sync(0xffffffffu, myties);
      if (lane == 0) misc->cnt[warp] = myties;
      __syncthreads();
      if (tid == 0) {
        uint32_t tot = 0;
        for (int k = 0; k < kFdThreads / 32; ++k) tot += misc->cnt[k];
        ws.tiecnt[blockIdx.x] = tot;
      }
      __syncthreads();
    }
    fd_grid_barrier(ws.sync, 3, G, misc, status);
    if (refine) {
      // ties before this CTA's range, then this CTA's first (take - before) ties in index order
      uint32_t before = 0;
      for (int p = 0; p < part; ++p) before += __ldcg(ws.tiecnt + row * per_row + p);
      const uint32_t want = take_ties > before ? take_ties - before : 0u;
      if (warp == 0 && want > 0) {
        uint32_t got = 0;
        for (int j0 = 0; j0 < n && got < want; j0 += 32) {
          const int j = j0 + lane;
          const bool tie = j < n && sc[j] == tstar;
          const unsigned msk = __ballot_sync(0xffffffffu, tie);
          const uint32_t r = got + __popc(msk & ((1u << lane) - 1u));
          fd_append(tie && r < want, make_key(tstar, (uint32_t)(s0 + j)), ccount, cand, kCandCap);
          got += __popc(msk);
        }
      }
    }
    fd_grid_barrier(ws.sync, 4, G, misc, status);
  }

  // ---- rank
  const int cnt = min(K, nvis);
  int32_t *oi = idx_out + (int64_t)row * K;
  float *os = score_out ? score_out + (int64_t)row * K : nullptr;
  const uint32_t nc = min(__ldcg(ccount), (uint32_t)kCandCap);
  uint64_t *ck = reinterpret_cast<uint64_t *>(kbuf);   // the key ring is idle now
  for (uint32_t i = tid; i < nc; i += kFdThreads) ck[i] = __ldcg(cand + i);
  __syncthreads();
  for (uint32_t i = (uint32_t)(part + per_row * warp); i < nc; i += (uint32_t)(per_row * (kFdThreads / 32))) {
    const uint64_t key = ck[i];
    uint32_t r = 0;
    for (uint32_t j = lane; j < nc; j += 32) r += ck[j] > key ? 1u : 0u;
    r = __reduce_add_sync(0xffffffffu, r);
    if (lane == 0 && r < (uint32_t)cnt) {
      oi[r] = (int32_t)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFu));
      if (os) os[r] = (float)(uint32_t)(key >> 32) * (1.f / 64.f);
    }
  }
  if (part == 0) {
    for (int j = cnt + tid; j < K; j += kFdThreads) {
      oi[j] = -1;
      if (os) os[j] = 0.f;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tbase, kFdTmemCols);
}

int fd_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  if (!cache[dev]) {
    int sms = 0, occ = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (set_smem_once((const void *)index_decode_kernel<4>, (int)kFdSmem, "index_decode_kernel")) return 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, index_decode_kernel<4>, kFdThreads, kFdSmem) !=
            cudaSuccess || occ < 1)
      return 0;
    cache[dev] = sms;   // one CTA per SM
  }
  return cache[dev];
}

// Fused decode plan: per_row CTAs per row, all co-resident (one per SM).
bool fd_plan(const csa_dims *d, int *per_row) {
  const int rows = d->B * d->Tq;
  if (d->dI != 64 || d->HI > 4 || d->HI < 1 || rows < 1 || d->K > kCandCap || d->n_entries < 1) return false;
  const int sms = fd_sms();
  if (sms < 1 || rows > sms) return false;
  const int pr = sms / rows;
  if ((d->n_entries + pr - 1) / pr > kFdLocalCap) return false;
  *per_row = pr;
  return true;
}

size_t fd_workspace(const csa_dims *d, int per_row, FdWs *ws, void *base, size_t *zero_off) {
  const int64_t rows = (int64_t)d->B * d->Tq;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off += (bytes + 255) & ~(size_t)255; return o; };
  const size_t o_cand = take((size_t)(rows * kCandCap * 8));
  const size_t o_hist = take((size_t)(rows * kBins * 4));
  const size_t o_hist2 = take((size_t)(rows * 256 * 4));
  const size_t o_cnt = take((size_t)(rows * 4));
  const size_t o_tie = take((size_t)(rows * per_row * 4));
  const size_t o_sync = take(4);
  const size_t o_flag = take(4);
  if (zero_off) *zero_off = o_hist;
  if (ws && base) {
    char *p = static_cast<char *>(base);
    ws->cand = reinterpret_cast<uint64_t *>(p + o_cand);
    ws->hist = reinterpret_cast<uint32_t *>(p + o_hist);
    ws->hist2 = reinterpret_cast<uint32_t *>(p + o_hist2);
    ws->ccount = reinterpret_cast<uint32_t *>(p + o_cnt);
    ws->tiecnt = reinterpret_cast<uint32_t *>(p + o_tie);
    ws->sync = reinterpret_cast<uint32_t *>(p + o_sync);
    ws->flag = reinterpret_cast<uint32_t *>(p + o_flag);
  }
  return off;
}

// Tensor map over the indexer keys viewed as [B * entry_cap rows][32 bytes],
// 256-row boxes, 32-byte swizzle (the layout the MMA descriptor reads).
bool fd_key_map(const uint8_t *kI, const csa_dims *d, CUtensorMap *map) {
  const int64_t rows = (int64_t)d->B * d->entry_cap;
  if (rows >= (1ll << 31)) return false;
  return encode_tmap_2d(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, kI, 32, (uint64_t)rows, 32, 32, 256,
                        CU_TENSOR_MAP_SWIZZLE_32B);
}

int launch_fd(const CUtensorMap &kmap, const uint8_t *qI, const float *w, const int32_t *q_pos, const csa_dims *d,
              int per_row, int32_t *idx_out, float *score_out, void *workspace, cudaStream_t stream) {
  FdWs ws;
  size_t zoff = 0;
  const size_t total = fd_workspace(d, per_row, &ws, workspace, &zoff);
  if (cudaMemsetAsync(static_cast<char *>(workspace) + zoff, 0, total - zoff, stream) != cudaSuccess)
    return check_launch("cudaMemsetAsync");
  const int rows = d->B * d->Tq;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(rows * per_row));
  cfg.blockDim = dim3(kFdThreads);
  cfg.dynamicSmemBytes = kFdSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  unsigned *st = status_word_device_ptr();
  cudaError_t e;
  switch (d->HI) {
    case 1: if (set_smem_once((const void *)index_decode_kernel<1>, (int)kFdSmem, "index_decode_kernel")) return CSA_ERR_CUDA;
            e = cudaLaunchKernelEx(&cfg, index_decode_kernel<1>, kmap, qI, w, q_pos, d->Tq, d->m, d->n_entries, d->entry_cap, d->K, per_row, ws, idx_out, score_out, st); break;
    case 2: if (set_smem_once((const void *)index_decode_kernel<2>, (int)kFdSmem, "index_decode_kernel")) return CSA_ERR_CUDA;
            e = cudaLaunchKernelEx(&cfg, index_decode_kernel<2>, kmap, qI, w, q_pos, d->Tq, d->m, d->n_entries, d->entry_cap, d->K, per_row, ws, idx_out, score_out, st); break;
    case 3: if (set_smem_once((const void *)index_decode_kernel<3>, (int)kFdSmem, "index_decode_kernel")) return CSA_ERR_CUDA;
            e = cudaLaunchKernelEx(&cfg, index_decode_kernel<3>, kmap, qI, w, q_pos, d->Tq, d->m, d->n_entries, d->entry_cap, d->K, per_row, ws, idx_out, score_out, st); break;
    default: e = cudaLaunchKernelEx(&cfg, index_decode_kernel<4>, kmap, qI, w, q_pos, d->Tq, d->m, d->n_entries, d->entry_cap, d->K, per_row, ws, idx_out, score_out, st); break;
  }
  count_launches(1);
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "index_decode_kernel launch: %s", cudaGetErrorString(e));
  return check_launch("index_decode_kernel");
}

// ---------------------------------------------------------------------------
// tensor-core prefill path: one CTA per 128 query rows (one TMEM lane per
// query), streaming 16-entry key tiles.  Per tile and head one kind::mxf4 MMA
// (M = 128 queries, N = 16 entries, K = 64) gives exact q.k sums; each
// epilogue thread turns its query's 16 columns into integer scores and runs an
// exact radix threshold over four streaming passes on a private 256-bin
// histogram column (bits 19..12, 11..4, 3..0, then collection).  Entries are
// visited in increasing index order, so the ties kept at the threshold are
// the lowest-indexed ones.  Survivors are written in index order and put in
// rank order by topk_sort_kernel.
// ---------------------------------------------------------------------------
constexpr int kPfQ = 128;                 // queries per CTA
constexpr int kPfN = 16;                  // entries per MMA tile
constexpr int kPfStages = 8;              // key-tile ring
constexpr int kPfThreads = 160;           // warps 0-3 epilogue, warp 4 control
constexpr uint32_t kPfTmemCols = 256;     // 2 x (4 heads x 16) accumulator columns + scales
constexpr uint32_t kPfColSFA = 128, kPfColSFB = 132;
constexpr uint32_t kPfOffQ = 0;                                   // 4 heads x 4 KiB
constexpr uint32_t kPfOffK = kPfOffQ + 4 * 4096;                  // stages x 512 B
constexpr uint32_t kPfOffH = kPfOffK + kPfStages * 512;           // u16 [256 bins][128 queries]
constexpr uint32_t kPfOffBar = kPfOffH + 256 * kPfQ * 2;
constexpr uint32_t kPfSmem = kPfOffBar + 32 * 8 + 64;

template <int HI>
__global__ void __launch_bounds__(kPfThreads, 2)
index_prefill_tc_kernel(const uint8_t *__restrict__ qI, const float *__restrict__ w,
                        const uint8_t *__restrict__ kI, const int32_t *__restrict__ q_pos, int Tq, int m,
                        int n_entries, int64_t entry_cap, int K, int tiles_per_seq, int ntiles,
                        int32_t *__restrict__ idx_out, uint32_t *__restrict__ sc_out, unsigned *status) {
  extern __shared__ __align__(1024) unsigned char smem[];
  uint16_t *hist = reinterpret_cast<uint16_t *>(smem + kPfOffH);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kPfOffBar);
  uint64_t *tfull = bars, *tempty = bars + 2, *sempty = bars + 4;      // [2], [2], [kPfStages]
  uint32_t *tptr = reinterpret_cast<uint32_t *>(bars + 4 + kPfStages);
  int *nvmax_s = reinterpret_cast<int *>(tptr + 1);
  int *abort_flag = nvmax_s + 1;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = ntiles - 1 - (int)blockIdx.x;          // the heaviest tiles first
  const int seq = tile / tiles_per_seq;
  const int q0 = (tile - seq * tiles_per_seq) * kPfQ;       // first query of the tile in its sequence
  const int nq = min(kPfQ, Tq - q0);
  const int64_t row0 = (int64_t)seq * Tq + q0;
  const uint8_t *krow = kI + (int64_t)seq * entry_cap * 32;

  // this thread's query (epilogue threads only)
  int nvis = 0;
  float w64[HI];            // 64 * w: with it, sum_h w64_h * max(acc_h, 0) is 64 * score, an exact fp32 integer
#pragma unroll
  for (int h = 0; h < HI; ++h) w64[h] = 0.f;
  if (warp < 4 && tid < nq) {
    const int64_t t = q_pos[row0 + tid];
    if (t < 0) raise_status(status, STATUS_BAD_POSITION);
    nvis = t < 0 ? 0 : (int)min((t + 1) / m, (int64_t)n_entries);
#pragma unroll
    for (int h = 0; h < HI; ++h) {
      bool bad;
      const int w16 = weight16(w[(row0 + tid) * HI + h], bad);
      if (bad) raise_status(status, STATUS_BAD_WEIGHT);
      w64[h] = (float)(4 * w16);
    }
  }
  if (tid == 0) { *nvmax_s = 0; *abort_flag = 0; }
  if (warp == 4) tc::tmem_alloc(tptr, kPfTmemCols);
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) { tc::mbar_init(&tfull[i], 1); tc::mbar_init(&tempty[i], 4); }
    for (int i = 0; i < kPfStages; ++i) tc::mbar_init(&sempty[i], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // query tiles (A operands), FP4 core-matrix layout; rows beyond the tile are zero
  for (int c = tid; c < 4 * kPfQ * 2; c += kPfThreads) {
    const int h = c / (kPfQ * 2), r = (c >> 1) % kPfQ, half = c & 1;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (h < HI && r < nq) v = *reinterpret_cast<const uint4 *>(qI + ((row0 + r) * HI + h) * 32 + half * 16);
    *reinterpret_cast<uint4 *>(smem + kPfOffQ + h * 4096 + (r >> 3) * 256 + half * 128 + (r & 7) * 16) = v;
  }
  // histogram columns start at zero
  for (int i = tid; i < 256 * kPfQ / 2; i += kPfThreads) reinterpret_cast<uint32_t *>(hist)[i] = 0u;
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  if (warp < 4 && nvis > 0) atomicMax(nvmax_s, nvis);
  tc::fence_after_sync();
  const uint32_t tbase = *tptr;
  if (warp < 4) {
    const uint32_t ones[4] = {0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu, 0x7F7F7F7Fu};
    tc::tmem_st4(tbase + ((uint32_t)(warp * 32) << 16) + kPfColSFA, ones);
    tc::tmem_st4(tbase + ((uint32_t)(warp * 32) << 16) + kPfColSFB, ones);
    tc::tmem_wait_st();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const int nvmax = *nvmax_s;
  const int npass = nvmax > K ? 4 : 1;
  const int n_et = (nvmax + kPfN - 1) / kPfN;
  const int total = npass * n_et;

  auto bounded_wait = [&](uint64_t *bar, uint32_t par) -> bool {
    if (tc::mbar_try_wait(bar, par)) return true;
    const uint64_t t0 = gtimer();
    uint32_t it = 0;
    while (!tc::mbar_try_wait(bar, par)) {
      if ((++it & 255u) == 0) {
        if (*(volatile int *)abort_flag) return false;
        if (gtimer() - t0 > kScanWaitNs) { *(volatile int *)abort_flag = 1; raise_status(status, STATUS_TIMEOUT); return false; }
      }
    }
    return true;
  };

  if (warp == 4) {
    // ---------------------------------------------------------------- control warp
    const uint32_t idesc = tc::idesc_mxf4(128, kPfN);
    auto load = [&](int i) {
      const int stg = i % kPfStages;
      const int et = i % n_et;
      const int r = lane >> 1, half = lane & 1;           // 16 entries x 2 halves = 32 chunks
      const int s = et * kPfN + r;
      const bool okk = s < n_entries;
      tc::cp_async16(smem + kPfOffK + stg * 512 + (r >> 3) * 256 + half * 128 + (r & 7) * 16,
                     okk ? (const void *)(krow + (int64_t)s * 32 + half * 16) : (const void *)krow, okk ? 16u : 0u);
    };
    constexpr int LA = kPfStages - 1;
    for (int i = 0; i < LA; ++i) { if (i < total) load(i); tc::cp_async_commit(); }
    bool ok = true;
    for (int i = 0; i < total && ok; ++i) {
      // refill the stage of tile i-1 with tile i+LA once MMA(i-1) is done
      const int nxt = i + LA;
      if (nxt < total) {
        if (nxt >= kPfStages) ok = bounded_wait(&sempty[nxt % kPfStages], (uint32_t)((nxt / kPfStages) - 1) & 1u);
        if (ok) load(nxt);
      }
      tc::cp_async_commit();
      tc::cp_async_wait<LA>();
      tc::fence_proxy_async_smem();
      __syncwarp();
      const int buf = i & 1;
      if (lane == 0 && ok) {
        if (i >= 2) ok = bounded_wait(&tempty[buf], (uint32_t)((i >> 1) - 1) & 1u);
        if (ok) {
          tc::fence_after_sync();
          const uint64_t bd = tc::smem_desc(tc::smem_u32(smem + kPfOffK + (i % kPfStages) * 512), 128, 256);
#pragma unroll
          for (int h = 0; h < HI; ++h)
            tc::mma_mxf4_ss(tbase + buf * 64 + h * kPfN, tc::smem_desc(tc::smem_u32(smem + kPfOffQ + h * 4096), 128, 256),
                            bd, idesc, tbase + kPfColSFA, tbase + kPfColSFB, 0);
          tc::mma_commit(&tfull[buf]);
          tc::mma_commit(&sempty[i % kPfStages]);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    tc::cp_async_wait<0>();
  } else {
    // ---------------------------------------------------------------- epilogue: one query per thread
    const bool active = tid < nq;
    const bool radix = nvis > K;
    uint32_t b1 = 0, b2 = 0, tau = 0, need_eq = 0, above = 0;
    int cnt = 0;
    uint32_t eq_taken = 0;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    // this query's u16 counters: slot(tid) puts the 32 lanes of a warp in 32 different banks
    uint16_t *hcol = hist + (lane * 2 + (warp & 1) + (warp >> 1) * 64);
    auto find = [&](int nb, uint32_t need, uint32_t &above_out) -> uint32_t {
      uint32_t cum = 0;
      int bsel = 0;
      for (int bn = nb - 1; bn >= 0; --bn) {
        const uint32_t c = hcol[bn * kPfQ];
        if (cum + c >= need) { bsel = bn; break; }
        cum += c;
      }
      above_out = cum;
      for (int bn = 0; bn < 256; ++bn) hcol[bn * kPfQ] = 0;
      return (uint32_t)bsel;
    };
    bool ok = true;
    for (int i = 0; i < total && ok; ++i) {
      const int pass = npass == 4 ? i / n_et : 3;
      const int et = i % n_et;
      const int buf = i & 1;
      ok = bounded_wait(&tfull[buf], (uint32_t)(i >> 1) & 1u);
      tc::fence_after_sync();
      // the 4 heads' 16 columns: 4 x 16 columns issued together, one wait
      uint32_t r[4][16];
#pragma unroll
      for (int h = 0; h < HI; ++h)
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                     : "=r"(r[h][0]), "=r"(r[h][1]), "=r"(r[h][2]), "=r"(r[h][3]), "=r"(r[h][4]), "=r"(r[h][5]),
                       "=r"(r[h][6]), "=r"(r[h][7]), "=r"(r[h][8]), "=r"(r[h][9]), "=r"(r[h][10]), "=r"(r[h][11]),
                       "=r"(r[h][12]), "=r"(r[h][13]), "=r"(r[h][14]), "=r"(r[h][15])
                     : "r"(tbase + lane_off + buf * 64 + h * kPfN));
      tc::tmem_wait_ld();
      uint32_t sc[kPfN];
#pragma unroll
      for (int j = 0; j < kPfN; ++j) {
        float f = 0.f;
#pragma unroll
        for (int h = 0; h < HI; ++h) f = fmaf(w64[h], fmaxf(__uint_as_float(r[h][j]), 0.f), f);
        sc[j] = __float2uint_rz(f);          // exact: an integer below 2^20
      }
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&tempty[buf]);
      if (!active) continue;
      const int s0 = et * kPfN;
      if (pass == 0) {
        if (radix)
#pragma unroll
          for (int j = 0; j < kPfN; ++j)
            if (s0 + j < nvis) hcol[(sc[j] >> 12) * kPfQ] += 1;
      } else if (pass == 1) {
        if (radix)
#pragma unroll
          for (int j = 0; j < kPfN; ++j)
            if (s0 + j < nvis && (sc[j] >> 12) == b1) hcol[((sc[j] >> 4) & 0xFF) * kPfQ] += 1;
      } else if (pass == 2) {
        if (radix)
#pragma unroll
          for (int j = 0; j < kPfN; ++j)
            if (s0 + j < nvis && (sc[j] >> 4) == ((b1 << 8) | b2)) hcol[(sc[j] & 0xF) * kPfQ] += 1;
      } else {
        int32_t *oi = idx_out + (row0 + tid) * K;
        uint32_t *os = sc_out + (row0 + tid) * K;
#pragma unroll
        for (int j = 0; j < kPfN; ++j) {
          const int s = s0 + j;
          if (s >= nvis) break;
          bool take;
          if (!radix) take = true;
          else if (sc[j] > tau) take = true;
          else if (sc[j] == tau && eq_taken < need_eq) { take = true; ++eq_taken; }
          else take = false;
          if (take) { oi[cnt] = s; os[cnt] = sc[j]; ++cnt; }
        }
      }
      // pass boundaries: per-query thresholds
      if (et == n_et - 1 && radix) {
        uint32_t a;
        if (pass == 0) { b1 = find(256, (uint32_t)K, a); above = a; }
        else if (pass == 1) { b2 = find(256, (uint32_t)K - above, a); above += a; }
        else if (pass == 2) {
          const uint32_t b3 = find(16, (uint32_t)K - above, a);
          above += a;
          tau = (b1 << 12) | (b2 << 4) | b3;
          need_eq = (uint32_t)K - above;
        }
      }
    }
    if (active) {
      int32_t *oi = idx_out + (row0 + tid) * K;
      uint32_t *os = sc_out + (row0 + tid) * K;
      for (int j = cnt; j < K; ++j) { oi[j] = -1; os[j] = 0; }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 4) tc::tmem_dealloc(tbase, kPfTmemCols);
}

// Rank order for rows written in index order: sort (score desc, index asc).
__global__ void __launch_bounds__(256)
topk_sort_kernel(int K, int32_t *__restrict__ idx_out, const uint32_t *__restrict__ sc_in,
                 float *__restrict__ score_out) {
  __shared__ uint64_t keys[kMaxK];
  const int64_t row = blockIdx.x;
  int np = 1;
  while (np < K) np <<= 1;
  for (int j = threadIdx.x; j < np; j += 256) {
    uint64_t k = 0;
    if (j < K) {
      const int32_t id = idx_out[row * K + j];
      if (id >= 0) k = make_key(sc_in[row * K + j], (uint32_t)id);
    }
    keys[j] = k;
  }
  __syncthreads();
  bitonic_desc_u64(keys, np);
  for (int j = threadIdx.x; j < K; j += 256) {
    const uint64_t k = keys[j];
    idx_out[row * K + j] = k ? (int32_t)(0xFFFFFFFFu - (uint32_t)(k & 0xFFFFFFFFu)) : -1;
    if (score_out) score_out[row * K + j] = k ? (float)(uint32_t)(k >> 32) * (1.f / 64.f) : 0.f;
  }
}

bool prefill_tc_plan(const csa_dims *d) {
  const int64_t rows = (int64_t)d->B * d->Tq;
  return d->dI == 64 && d->HI <= 4 && rows > 64 && d->n_entries <= 65535 && d->K <= kMaxK && d->n_entries >= 1;
}

int launch_prefill_tc(const uint8_t *qI, const float *w, const uint8_t *kI, const int32_t *q_pos,
                      const csa_dims *d, int32_t *idx_out, float *score_out, void *workspace,
                      cudaStream_t stream) {
  const int tiles_per_seq = (d->Tq + kPfQ - 1) / kPfQ;
  const int ntiles = d->B * tiles_per_seq;
  uint32_t *sc = static_cast<uint32_t *>(workspace);
  unsigned *st = status_word_device_ptr();
#define CSA_PF(HI_)                                                                                  \
  case HI_:                                                                                          \
    if (int rc = set_smem_once((const void *)index_prefill_tc_kernel<HI_>, (int)kPfSmem, "index_prefill_tc_kernel")) \
      return rc;                                                                                     \
    index_prefill_tc_kernel<HI_><<<ntiles, kPfThreads, kPfSmem, stream>>>(                           \
        qI, w, kI, q_pos, d->Tq, d->m, d->n_entries, d->entry_cap, d->K, tiles_per_seq, ntiles, idx_out, sc, st); \
    break;
  switch (d->HI) {
    CSA_PF(1) CSA_PF(2) CSA_PF(3) CSA_PF(4)
    default: return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk: HI=%d", d->HI);
  }
#undef CSA_PF
  count_launches(1);
  if (int rc = check_launch("index_prefill_tc_kernel")) return rc;
  topk_sort_kernel<<<(unsigned)((int64_t)d->B * d->Tq), 256, 0, stream>>>(d->K, idx_out, sc, score_out);
  count_launches(1);
  return check_launch("topk_sort_kernel");
}

}  // namespace

// The K best of each row's splits x K candidate keys, in rank order.
int launch_topk_merge(const uint64_t *cand, int splits, const csa_dims *d, const int32_t *q_pos, int32_t *idx_out,
                      float *score_out, bool float_scores, cudaStream_t stream) {
  const int64_t rows = (int64_t)d->B * d->Tq;
  const size_t smem = (kMergeCap + kMaxK) * 8 + kBins * 4 + sizeof(SelShared);
  const void *fn = float_scores ? (const void *)topk_merge_kernel<true> : (const void *)topk_merge_kernel<false>;
  if (int rc = set_smem_once(fn, (int)smem, "topk_merge_kernel")) return rc;
  if (float_scores)
    topk_merge_kernel<true><<<rows, kMergeThreads, smem, stream>>>(cand, splits, d->K, q_pos, d->m, d->n_entries,
                                                                   idx_out, score_out);
  else
    topk_merge_kernel<false><<<rows, kMergeThreads, smem, stream>>>(cand, splits, d->K, q_pos, d->m, d->n_entries,
                                                                    idx_out, score_out);
  count_launches(1);
  return check_launch("topk_merge_kernel");
}

bool prefill2_plan(const csa_dims *d);
size_t prefill2_workspace(const csa_dims *d);
int launch_prefill2(const uint8_t *qI, const float *w, const uint8_t *kI, const int32_t *q_pos, const csa_dims *d,
                    int32_t *idx_out, float *score_out, void *workspace, cudaStream_t stream);

size_t index_topk_workspace(const csa_dims *d) {
  int splits, slice, per_row;
  if (fd_plan(d, &per_row)) {
    // the launch falls back to the two-kernel path when the keys cannot be mapped
    const size_t a = fd_workspace(d, per_row, nullptr, nullptr, nullptr);
    const size_t b = tc_plan(d, &splits, &slice) ? tc_workspace(d, nullptr, nullptr) : 0;
    return a > b ? a : b;
  }
  if (tc_plan(d, &splits, &slice)) return tc_workspace(d, nullptr, nullptr);
  if (prefill2_plan(d)) return prefill2_workspace(d);
  if (prefill_tc_plan(d)) return (size_t)((int64_t)d->B * d->Tq * d->K * 4);
  if (split_plan(d, &splits, &slice)) return (size_t)((int64_t)d->B * d->Tq * splits * d->K * 8);
  const int64_t ld = ((int64_t)d->n_entries + 3) & ~3LL;
  return (size_t)((int64_t)d->B * d->Tq * ld * 4);
}

int launch_index_topk(const uint8_t *qI, const float *w, const uint8_t *kI, const int32_t *q_pos,
                      const csa_dims *d, int32_t *idx_out, float *score_out, void *workspace,
                      cudaStream_t stream) {
  const int rows = d->B * d->Tq;
  if (rows == 0) return CSA_OK;
  if (d->K > kMaxK) return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk: K > %d", kMaxK);
  int splits, slice, per_row;
  if (fd_plan(d, &per_row)) {
    CUtensorMap kmap;
    if (fd_key_map(kI, d, &kmap))
      return launch_fd(kmap, qI, w, q_pos, d, per_row, idx_out, score_out, workspace, stream);
  }
  if (tc_plan(d, &splits, &slice))
    return launch_tc(qI, w, kI, q_pos, d, splits, slice, idx_out, score_out, workspace, stream);
  if (prefill2_plan(d)) return launch_prefill2(qI, w, kI, q_pos, d, idx_out, score_out, workspace, stream);
  if (prefill_tc_plan(d)) return launch_prefill_tc(qI, w, kI, q_pos, d, idx_out, score_out, workspace, stream);
  if (split_plan(d, &splits, &slice)) {
    uint64_t *cand = static_cast<uint64_t *>(workspace);
#define CSA_PARTIAL(HI_, DI_)                                                                   \
  if (d->HI == HI_ && d->dI == DI_) {                                                           \
    launch_partial<HI_, DI_>(qI, w, kI, q_pos, d, splits, slice, cand, stream);                 \
  } else
    CSA_PARTIAL(1, 32) CSA_PARTIAL(1, 64) CSA_PARTIAL(2, 32) CSA_PARTIAL(2, 64) CSA_PARTIAL(4, 32)
    CSA_PARTIAL(4, 64) CSA_PARTIAL(8, 32) {
      return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk: (HI=%d, dI=%d) not compiled", d->HI, d->dI);
    }
#undef CSA_PARTIAL
    if (int rc = check_launch("index_partial_kernel")) return rc;
    return launch_topk_merge(cand, splits, d, q_pos, idx_out, score_out, false, stream);
  }
  const int64_t ld = ((int64_t)d->n_entries + 3) & ~3LL;
  uint32_t *scores = static_cast<uint32_t *>(workspace);
  if (d->n_entries > 0) {
#define CSA_SCORES(HI_, DI_)                                                                    \
  if (d->HI == HI_ && d->dI == DI_) {                                                           \
    launch_scores<HI_, DI_>(qI, w, kI, q_pos, rows, d->Tq, d->m, d->n_entries, d->entry_cap,     \
                            scores, ld, stream);                                                \
  } else
    CSA_SCORES(1, 32) CSA_SCORES(1, 64) CSA_SCORES(2, 32) CSA_SCORES(2, 64) CSA_SCORES(4, 32)
    CSA_SCORES(4, 64) CSA_SCORES(8, 32) {
      return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk: (HI=%d, dI=%d) not compiled", d->HI, d->dI);
    }
#undef CSA_SCORES
    int rc = check_launch("index_scores_kernel");
    if (rc) return rc;
  }
  topk_rows_kernel<<<rows, kSelThreads, 0, stream>>>(scores, ld, q_pos, d->m, d->n_entries, d->K,
                                                     idx_out, score_out, status_word_device_ptr());
  count_launches(1);
  return check_launch("topk_rows_kernel");
}

}  // namespace csa
