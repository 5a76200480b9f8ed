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

namespace csa {
namespace {

constexpr uint32_t kMagLo = 0x03020100u;   // 2*|E2M1| for codes 0..3
constexpr uint32_t kMagHi = 0x0C080604u;   // 2*|E2M1| for codes 4..7

__device__ __forceinline__ int e2m1x2_int(uint32_t code) {   // 2*value of one 4-bit code
  const int mag = (int)((0xC8643210u >> (4 * (code & 7))) & 0xF);
  return (code & 8) ? -mag : mag;
}

// ---------------------------------------------------------------------------
// scores
// ---------------------------------------------------------------------------
constexpr int kScoreThreads = 256;
constexpr int kEPT = 4;   // entries per thread per CTA

template <int HI, int DI>
__global__ void __launch_bounds__(kScoreThreads)
index_scores_kernel(const uint8_t *__restrict__ qI, const float *__restrict__ w,
                    const uint8_t *__restrict__ kI, const int32_t *__restrict__ q_pos, int row0,
                    int Tq, int m, int n_entries, int64_t entry_cap, uint32_t *__restrict__ scores,
                    int64_t ld, unsigned *status) {
  constexpr int NW = DI / 8;           // 32-bit key words (8 codes each)
  const int row = row0 + blockIdx.y;
  const int b = row / Tq;
  const int64_t t = q_pos[row];
  const int nvis = (int)min((t + 1) / m, (int64_t)n_entries);
  const int base = blockIdx.x * (kScoreThreads * kEPT);
  if (base >= nvis) return;

  // query as packed int8 (2*q): qw[h][2*k] holds elements 8k..8k+3, qw[h][2k+1] 8k+4..8k+7
  int qw[HI][2 * NW];
  int w16[HI];
  const uint8_t *qrow = qI + (int64_t)row * HI * (DI / 2);
#pragma unroll
  for (int h = 0; h < HI; ++h) {
    const float wf = w[(int64_t)row * HI + h];
    const float w16f = wf * 16.f;
    w16[h] = __float2int_rn(w16f);
    if (threadIdx.x == 0 && blockIdx.x == 0 && ((float)w16[h] != w16f || w16[h] < 0 || w16[h] > 16))
      raise_status(status, STATUS_BAD_WEIGHT);
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

  const uint8_t *krow = kI + (int64_t)b * entry_cap * (DI / 2);
  uint32_t *srow = scores + (int64_t)row * ld;
#pragma unroll
  for (int u = 0; u < kEPT; ++u) {
    const int s = base + u * kScoreThreads + threadIdx.x;
    if (s >= nvis) break;
    uint32_t kw[NW];
    if constexpr (DI == 64) {
      const uint4 a = __ldg(reinterpret_cast<const uint4 *>(krow + (int64_t)s * 32));
      const uint4 c = __ldg(reinterpret_cast<const uint4 *>(krow + (int64_t)s * 32 + 16));
      kw[0] = a.x; kw[1] = a.y; kw[2] = a.z; kw[3] = a.w;
      kw[4] = c.x; kw[5] = c.y; kw[6] = c.z; kw[7] = c.w;
    } else {
      const uint4 a = __ldg(reinterpret_cast<const uint4 *>(krow + (int64_t)s * 16));
      kw[0] = a.x; kw[1] = a.y; kw[2] = a.z; kw[3] = a.w;
    }
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
    srow[s] = sc;
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

__global__ void __launch_bounds__(kSelThreads)
topk_rows_kernel(const uint32_t *__restrict__ scores, int64_t ld, const int32_t *__restrict__ q_pos,
                 int m, int n_entries, int K, int32_t *__restrict__ idx_out,
                 float *__restrict__ score_out, unsigned *status) {
  __shared__ uint32_t hist[kBins];
  __shared__ uint64_t keys[kMaxK];
  __shared__ uint32_t ties[kTieCap];
  __shared__ uint32_t warp_tot[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above, s_cgt, s_ceq, s_run;

  const int row = blockIdx.x;
  const int tid = threadIdx.x;
  const int64_t t = q_pos[row];
  if (t < 0 && tid == 0) raise_status(status, STATUS_BAD_POSITION);
  const int n = t < 0 ? 0 : (int)min((t + 1) / m, (int64_t)n_entries);
  const uint32_t *S = scores + (int64_t)row * ld;
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
    idx_out[(int64_t)row * K + j] = id;
    if (score_out) score_out[(int64_t)row * K + j] = sc;
  }
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

}  // namespace

size_t index_topk_workspace(const csa_dims *d) {
  const int64_t ld = ((int64_t)d->n_entries + 3) & ~3LL;
  return (size_t)((int64_t)d->B * d->Tq * ld * 4);
}

int launch_index_topk(const uint8_t *qI, const float *w, const uint8_t *kI, const int32_t *q_pos,
                      const csa_dims *d, int32_t *idx_out, float *score_out, void *workspace,
                      cudaStream_t stream) {
  const int rows = d->B * d->Tq;
  if (rows == 0) return CSA_OK;
  if (d->K > kMaxK) return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk: K > %d", kMaxK);
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
