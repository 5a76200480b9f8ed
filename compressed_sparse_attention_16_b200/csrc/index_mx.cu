// Block-scaled FP4 indexer: queries and keys in MXFP4 (E2M1 elements, one
// UE8M0 power-of-two scale per 32 elements), top-k per query.
//
// Pages: jiwasawa.github.io DeepSeek-V4 article, sections "Compressed Sparse
// Attention (CSA)" (the indexer scores every compressed entry, a top-k
// selector keeps the best) and "限界を押し広げるインフラストラクチャの最適化"
// (FP4 on the indexer's QK path); "DeepSeek V4 Flash" (studioglobal.ai),
// "FP4/FP8混合精度" (MXFP4, two values per byte).
//
// score(t, s) = sum_h w[t,h] * max(0, sum_j q[t,h,j] k[s,j]) with
// q[t,h,j] = e2m1 * 2^(qs[t,h,j/32] - 127) and k[s,j] likewise.  The scales
// are applied inside the tensor core: one tcgen05.mma.kind::mxf4.block_scale
// per 128 keys (M = 128 keys, N = 8 query heads, K = 64) reads the keys'
// scale factors from TMEM (lane r holds key r's two block scales in bytes 0
// and 1 of column SFA + r / 32) and the query heads' from TMEM (column n's
// in lane 32 q + n of every lane quadrant q, column SFB, bytes 0 and 1).
// The scores are fp32, no longer exact integers: the top-k keys carry the
// fp32 bits of the score above ~index, and near-ties may order differently
// from an exact evaluation (see the tie-tolerant check in the tests).
//
// One CTA per (query row, slice of at most 4,096 entries): the slice's keys
// land in shared memory in one wave of 16-byte copies, the scales go to
// TMEM, 32 MMAs are issued back to back (accumulators of tile t at columns
// 8 t .. 8 t + 7), then every key's score becomes a 64-bit key and a radix
// select keeps the slice's k best.  A merge kernel keeps each row's k best
// of its slices in rank order.
#include "common.cuh"
#include "tc.cuh"
#include "select.cuh"

namespace csa {
namespace {

constexpr int kThr = 256;
constexpr int kTile = 128;                 // keys per MMA (M)
constexpr int kMaxTiles = 32;
constexpr int kSlice = kTile * kMaxTiles;  // 4,096 entries per CTA at most
constexpr uint32_t kColSFA = 256;          // 4 columns per tile
constexpr uint32_t kColSFB = 384;
constexpr uint32_t kCols = 512;
constexpr unsigned long long kWaitNs = 2000000000ull;

constexpr uint32_t OFF_A = 0;                                // key tiles, 4 KiB each, core-matrix layout
constexpr uint32_t OFF_B = OFF_A + kMaxTiles * 4096;         // query heads (8 rows x 32 B)
constexpr uint32_t OFF_KEYS = OFF_B + 1024;                  // u64 [kSlice]
constexpr uint32_t OFF_HIST = OFF_KEYS + kSlice * 8;         // u32 [4096]
constexpr uint32_t OFF_SH = OFF_HIST + sel::kSelBins * 4;
constexpr uint32_t OFF_BAR = OFF_SH + ((sizeof(sel::SelShared) + 15) & ~15u);
constexpr uint32_t SMEM = OFF_BAR + 64;
static_assert(SMEM <= 232448, "shared memory");

__device__ __forceinline__ uint64_t gtimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t v) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(v) : "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

// two UE8M0 scales as the low bytes of a TMEM scale word (the other bytes 2^0)
__device__ __forceinline__ uint32_t sf_word(const uint8_t *p) {
  return 0x7F7F0000u | (uint32_t)p[0] | ((uint32_t)p[1] << 8);
}

template <int HI>
__global__ void __launch_bounds__(kThr, 1)
index_mx_partial_kernel(const uint8_t *__restrict__ qI, const uint8_t *__restrict__ qs, const float *__restrict__ w,
                        const uint8_t *__restrict__ kI, const uint8_t *__restrict__ ks,
                        const int32_t *__restrict__ q_pos, int row0, int Tq, int m, int n_entries,
                        int64_t entry_cap, int K, int splits, int slice, uint64_t *__restrict__ cand,
                        unsigned *status) {
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t *keys = reinterpret_cast<uint64_t *>(smem + OFF_KEYS);
  uint32_t *hist = reinterpret_cast<uint32_t *>(smem + OFF_HIST);
  sel::SelShared *sh = reinterpret_cast<sel::SelShared *>(smem + OFF_SH);
  uint64_t *bar = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint32_t *tslot = reinterpret_cast<uint32_t *>(smem + OFF_BAR + 8);
  int *abort_flag = reinterpret_cast<int *>(smem + OFF_BAR + 12);

  const int row = row0 + (int)blockIdx.y, split = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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
    for (int j = tid; j < K; j += kThr) out[j] = 0ull;
    return;
  }
  const int ntiles = (n + kTile - 1) / kTile;

  // weights: finite and non-negative, else reported and taken as 0
  float wt[HI];
#pragma unroll
  for (int h = 0; h < HI; ++h) {
    const float v = w[(int64_t)row * HI + h];
    const bool good = v >= 0.f && v <= 3.402823466e38f;
    if (!good && tid == 0 && split == 0) raise_status(status, STATUS_BAD_WEIGHT);
    wt[h] = good ? v : 0.f;
  }
  // query heads as the B operand (rows past HI are zero), core-matrix layout
  if (tid < 16) {
    const int h = tid >> 1, hf = tid & 1;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (h < HI) v = *reinterpret_cast<const uint4 *>(qI + ((int64_t)row * HI + h) * 32 + hf * 16);
    *reinterpret_cast<uint4 *>(smem + OFF_B + hf * 128 + h * 16) = v;
  }
  // the slice's keys: one 16-byte copy per half row, all in flight at once;
  // rows past the slice are zero
  const uint8_t *krow = kI + ((int64_t)b * entry_cap + s0) * 32;
  for (int c = tid; c < ntiles * kTile * 2; c += kThr) {
    const int r = c >> 1, hf = c & 1;
    const int tile = r / kTile, rr = r % kTile;
    unsigned char *dst = smem + OFF_A + tile * 4096 + (rr >> 3) * 256 + hf * 128 + (rr & 7) * 16;
    tc::cp_async16(dst, krow + (int64_t)(r < n ? r : 0) * 32 + hf * 16, r < n ? 16u : 0u);
  }
  tc::cp_async_commit();
  if (tid == 0) {
    tc::mbar_init(bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tc::tmem_alloc(tslot, kCols);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tslot;
  // scale factors: warp w writes lane quadrant q = w % 4 of the tiles t with
  // t % 2 == w / 4 (column SFA + 4 t + q: key t * 128 + 32 q + lane); warps
  // 0-3 also write the query heads' scales (lane 32 q + n holds head n's)
  const int q = warp & 3;
  const uint32_t lane_base = (uint32_t)(q * 32) << 16;
  const uint8_t *kscale = ks + ((int64_t)b * entry_cap + s0) * 2;
  bool bad_scale = false;
  for (int tt = warp >> 2; tt < ntiles; tt += 2) {
    const int r = tt * kTile + q * 32 + lane;
    uint32_t v = 0x7F7F7F7Fu;
    if (r < n) {
      v = sf_word(kscale + (int64_t)r * 2);
      bad_scale |= ((v & 0xFFu) == 0xFFu) || (((v >> 8) & 0xFFu) == 0xFFu);
    }
    tmem_st1(tbase + lane_base + kColSFA + 4 * tt + q, v);
  }
  if (warp < 4) {
    uint32_t v = 0x7F7F7F7Fu;
    if (lane < HI) {
      v = sf_word(qs + ((int64_t)row * HI + lane) * 2);
      bad_scale |= ((v & 0xFFu) == 0xFFu) || (((v >> 8) & 0xFFu) == 0xFFu);
    }
    tmem_st1(tbase + lane_base + kColSFB, v);
  }
  if (bad_scale) raise_status(status, STATUS_BAD_WEIGHT);
  tc::tmem_wait_st();
  tc::cp_async_wait<0>();
  tc::fence_proxy_async_smem();
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (tid == 0) {
    const uint32_t idesc = tc::idesc_mxf4(kTile, 8);
    const uint64_t bd = tc::smem_desc(tc::smem_u32(smem + OFF_B), 128, 256);
    for (int tt = 0; tt < ntiles; ++tt)
      tc::mma_mxf4_ss(tbase + 8 * tt, tc::smem_desc(tc::smem_u32(smem + OFF_A + tt * 4096), 128, 256), bd, idesc,
                      tbase + kColSFA + 4 * tt, tbase + kColSFB, 0);
    tc::mma_commit(bar);
  }
  __syncwarp();
  // wait for the MMAs (bounded)
  bool ok = tc::mbar_try_wait(bar, 0);
  if (!ok) {
    const uint64_t t0 = gtimer();
    uint32_t it = 0;
    while (!(ok = tc::mbar_try_wait(bar, 0))) {
      if ((++it & 255u) == 0) {
        if (*(volatile int *)abort_flag) break;
        if (gtimer() - t0 > kWaitNs) {
          *(volatile int *)abort_flag = 1;
          raise_status(status, STATUS_TIMEOUT);
          break;
        }
      }
    }
  }
  ok = __all_sync(0xffffffffu, ok);
  tc::fence_after_sync();
  // scores -> keys (fp32 bits of the score above ~index)
  for (int tt = warp >> 2; tt < ntiles; tt += 2) {
    uint32_t d[8];
    if (ok) {
      tmem_ld8(tbase + lane_base + 8 * tt, d);
      tc::tmem_wait_ld();
    }
    const int r = tt * kTile + q * 32 + lane;
    if (r < n) {
      float sc = 0.f;
#pragma unroll
      for (int h = 0; h < HI; ++h) sc = fmaf(wt[h], fmaxf(__uint_as_float(d[h]), 0.f), sc);
      if (!ok) sc = 0.f;
      keys[r] = ((uint64_t)__float_as_uint(sc) << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)(s0 + r));
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tbase, kCols);
  if (n <= K) {
    for (int j = tid; j < K; j += kThr) out[j] = j < n ? keys[j] : 0ull;
    return;
  }
  const uint64_t T = sel::kth_largest_key<kThr, true>(keys, n, K, hist, sh);
  if (tid == 0) sh->count = 0;
  __syncthreads();
  for (int j = tid; j < n; j += kThr) {
    const uint64_t k = keys[j];
    if (k >= T) out[atomicAdd(&sh->count, 1u)] = k;
  }
}

}  // namespace

// Slices of at most 4,096 entries, at most 20,480 / K of them per row (the
// merge kernel's candidate capacity).
bool index_mx_plan(const csa_dims *d, int *splits, int *slice) {
  if (d->dI != 64 || d->HI < 1 || d->HI > 8 || d->K < 1 || d->K > 2048) return false;
  const int n = max(d->n_entries, 1);
  const int64_t rows = (int64_t)d->B * d->Tq;
  // aim for about two CTAs per SM when there are few rows
  int s = (int)max((int64_t)1, (2 * 148 + rows - 1) / rows);
  s = min(s, (n + kTile - 1) / kTile);
  s = max(s, (n + kSlice - 1) / kSlice);
  const int sl = ((n + s - 1) / s + kTile - 1) / kTile * kTile;
  s = (n + sl - 1) / sl;
  if ((int64_t)s * d->K > 20480) return false;
  *splits = s;
  *slice = sl;
  return true;
}

size_t index_mx_workspace(const csa_dims *d) {
  int splits, slice;
  if (!index_mx_plan(d, &splits, &slice)) return 0;
  return (size_t)((int64_t)d->B * d->Tq * splits * d->K * 8);
}

int launch_index_mx(const uint8_t *qI, const uint8_t *qs, const float *w, const uint8_t *kI, const uint8_t *ks,
                    const int32_t *q_pos, const csa_dims *d, int32_t *idx_out, float *score_out, void *workspace,
                    cudaStream_t stream) {
  int splits, slice;
  if (!index_mx_plan(d, &splits, &slice))
    return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk_mx: dI=%d HI=%d K=%d n_entries=%d (dI 64, HI 1..8, at most "
                "20,480 / K slices of 4,096 entries)", d->dI, d->HI, d->K, d->n_entries);
  const int64_t rows = (int64_t)d->B * d->Tq;
  uint64_t *cand = static_cast<uint64_t *>(workspace);
  unsigned *st = status_word_device_ptr();
  if (rows >= (1ll << 31)) return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk_mx: too many rows");
  for (int64_t r0 = 0; r0 < rows; r0 += 65535) {          // grid.y is limited to 65,535
    const int r = (int)min(rows - r0, (int64_t)65535);
    const dim3 grid((unsigned)splits, (unsigned)r);
    switch (d->HI) {
#define CSA_MX(HI_)                                                                                         \
  case HI_:                                                                                                 \
    if (int rc = set_smem_once((const void *)index_mx_partial_kernel<HI_>, (int)SMEM, "index_mx_partial_kernel")) \
      return rc;                                                                                            \
    index_mx_partial_kernel<HI_><<<grid, kThr, SMEM, stream>>>(qI, qs, w, kI, ks, q_pos, (int)r0, d->Tq, d->m,   \
                                                               d->n_entries, d->entry_cap, d->K, splits, slice, \
                                                               cand, st);                                   \
    break;
      CSA_MX(1) CSA_MX(2) CSA_MX(3) CSA_MX(4) CSA_MX(5) CSA_MX(6) CSA_MX(7) CSA_MX(8)
#undef CSA_MX
      default: return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk_mx: HI=%d", d->HI);
    }
    count_launches(1);
    if (int rc = check_launch("index_mx_partial_kernel")) return rc;
  }
  return launch_topk_merge(cand, splits, d, q_pos, idx_out, score_out, true, stream);
}

}  // namespace csa
