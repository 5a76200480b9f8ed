// Shared-KV multi-query attention on the tensor cores for 64 query heads and
// 512-wide entries (the prefill shape: many query rows, each with its own
// item set).
//
// Page: jiwasawa.github.io DeepSeek-V4 article, section "Compressed Sparse
// Attention (CSA)" -- MQA with shared key-value over the k selected entries;
// section "Heavily Compressed Attention (HCA)" -- the sliding-window branch;
// "DeepSeek V4 Flash" (studioglobal.ai), "アテンションのブレイクスルー" -- top
// 512 blocks per query, 128-token window.
//
// With only 64 heads per query the items fill the tensor core's M = 128
// dimension instead:
//   pass 1   S^T[item, head] = K_items . Q^T   (M = 128 items per tile,
//            N = 64 heads, K = 512 in four 128-wide blocks); all <= 5 tiles of
//            the row stay in TMEM (<= 320 columns);
//   softmax  per head over items, i.e. across TMEM lanes: each warp reduces its
//            32 lanes with a transposing butterfly, four quadrants combine in
//            shared memory; P^T = p * entry scale is written as bf16;
//   pass 2   O^T[d, head] = V^T . P^T  (M = 128 d per block, N = 64 heads,
//            K = items), reading the same [item][d] tiles MN-major; O^T reuses
//            the S^T columns;
//   epilogue O / l through a shared-memory transpose to coalesced bf16 rows.
// Each key/value tile is gathered twice (once per pass) and converted exactly
// from E4M3 to bf16; the conversion of block j+1 overlaps the MMAs of block j.
// CTAs are persistent (one per SM) and walk the query rows round-robin.
#include "common.cuh"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int PH = 64;             // heads (MMA N)
constexpr int PD = 512;            // entry width
constexpr int PT = 128;            // items per tile (MMA M of pass 1)
constexpr int PDB = 128;           // d per block
constexpr int kMaxTiles = 5;       // <= 640 items per row
constexpr int kPThreads = 256;
constexpr int kPMaxSel = 2048;
constexpr float kPLog2e = 1.4426950408889634f;
constexpr unsigned long long kPWaitNs = 2000000000ull;

// shared memory map (bytes)
constexpr uint32_t P_OFF_Q = 0;                                  // 64 x 512 bf16   = 64 KiB
constexpr uint32_t P_OFF_KV = P_OFF_Q + PH * PD * 2;             // 2 x (128 x 128 bf16) = 64 KiB
constexpr uint32_t P_KV_BYTES = PT * PDB * 2;
constexpr uint32_t P_OFF_PT = P_OFF_KV + 2 * P_KV_BYTES;         // 640 x 64 bf16   = 80 KiB
constexpr uint32_t P_OFF_SEL = P_OFF_PT + kMaxTiles * PT * PH * 2;   // int32 [2048]
constexpr uint32_t P_OFF_SCALE = P_OFF_SEL + kPMaxSel * 4;       // fp32 [640]
constexpr uint32_t P_OFF_RED = P_OFF_SCALE + kMaxTiles * PT * 4; // fp32 [4][64] + [64] x 3
constexpr uint32_t P_OFF_BAR = P_OFF_RED + (4 * PH + 3 * PH) * 4;
constexpr uint32_t P_OFF_MISC = P_OFF_BAR + 8 * 8;
constexpr uint32_t P_SMEM = P_OFF_MISC + 64;

// Q  [64 h][512 d]:   d-group stride 1024, head-group stride 128
// KV [128 i][128 d]:  d-group stride 2048, item-group stride 128
// PT [640 i][64 h]:   item-group stride 1024, head-group stride 128
__device__ __forceinline__ uint32_t pq_off(int h, int g) { return g * 1024 + (h >> 3) * 128 + (h & 7) * 16; }
__device__ __forceinline__ uint32_t pkv_off(int i, int g) { return g * 2048 + (i >> 3) * 128 + (i & 7) * 16; }
__device__ __forceinline__ uint32_t ppt_off(int i, int hg) { return (i >> 3) * 1024 + hg * 128 + (i & 7) * 16; }

struct PMisc {
  uint32_t tmem_base;
  int abort;
  int wcount[8];
};

__device__ __forceinline__ uint64_t ptimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool pwait(uint64_t *bar, uint32_t parity, PMisc *misc, unsigned *status) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptimer();
  uint32_t n = 0;
  while (!tc::mbar_try_wait(bar, parity)) {
    if ((++n & 255u) == 0) {
      if (*(volatile int *)&misc->abort) return false;
      if (ptimer() - t0 > kPWaitNs) {
        misc->abort = 1;
        raise_status(status, STATUS_TIMEOUT);
        return false;
      }
    }
  }
  return true;
}

__device__ __forceinline__ void cvt16(const uint4 &c, uint4 &lo, uint4 &hi) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t o[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __nv_bfloat162 a = __float22bfloat162_rn(e4m3x2_to_float2((uint16_t)(w[k] & 0xFFFF)));
    const __nv_bfloat162 b = __float22bfloat162_rn(e4m3x2_to_float2((uint16_t)(w[k] >> 16)));
    o[2 * k] = *reinterpret_cast<const uint32_t *>(&a);
    o[2 * k + 1] = *reinterpret_cast<const uint32_t *>(&b);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// Transposing butterfly over a warp: on entry every lane holds v[0..31]
// (one value per column); on exit lane l holds op over all lanes of column l.
template <bool kMax>
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, s);
      v[i] = kMax ? fmaxf(keep, got) : keep + got;
    }
  }
  return v[0];
}

struct PArgs {
  const __nv_bfloat16 *q;
  const uint8_t *codes;
  const float *scales;
  const int32_t *idx;
  const uint8_t *wcodes;
  const float *wscales;
  const int32_t *q_pos;
  int rows, Tq, K, W, m, n_entries, win_cap;
  int64_t entry_cap;
  float sm_scale;
  __nv_bfloat16 *out;
  float *lse;
  unsigned *status;
};

__global__ void __launch_bounds__(kPThreads, 1) attend_prefill_kernel(const PArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  int *sel = reinterpret_cast<int *>(smem + P_OFF_SEL);
  float *iscale = reinterpret_cast<float *>(smem + P_OFF_SCALE);
  float *red = reinterpret_cast<float *>(smem + P_OFF_RED);        // [4][64]
  float *Mh = red + 4 * PH;                                         // [64] row max (log2 units)
  float *Lh = Mh + PH;                                              // [64] row sum
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + P_OFF_BAR);  // [0],[1]: KV buffers
  PMisc *misc = reinterpret_cast<PMisc *>(smem + P_OFF_MISC);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3;            // TMEM lane quadrant
  const int hhalf = warp >> 2;          // which 32 heads / which block pair this warp handles

  if (tid == 0) {
    misc->abort = 0;
    tc::mbar_init(&bars[0], 1);
    tc::mbar_init(&bars[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tc::tmem_alloc(&misc->tmem_base, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = misc->tmem_base;
  const uint32_t sbase = tc::smem_u32(smem);
  const uint32_t idesc_qk = tc::idesc_bf16_f32(128, PH, 0, 0);
  const uint32_t idesc_pv = tc::idesc_bf16_f32(128, PH, 1, 1);
  const float qs = a.sm_scale * kPLog2e;
  // MMA commits issued / completions consumed per KV buffer (mbarrier phases);
  // each buffer has at most one commit in flight.
  uint32_t issued[2] = {0u, 0u}, done[2] = {0u, 0u};
  // Wait (bounded) until buffer `buf` has no MMA in flight.  All threads call
  // this together; the result is made uniform across the CTA.
  auto drain = [&](int buf) -> bool {
    bool r = true;
    if (issued[buf] != done[buf]) {
      r = pwait(&bars[buf], done[buf] & 1u, misc, a.status);
      done[buf] += 1u;
    }
    return __syncthreads_and(r) != 0;
  };
  bool ok = true;

  for (int row = blockIdx.x; row < a.rows && ok; row += gridDim.x) {
    const int b = row / a.Tq;
    int64_t t = a.q_pos[row];
    if (t < 0) {
      if (tid == 0) raise_status(a.status, STATUS_BAD_POSITION);
      t = 0;
    }
    const int nwin = (int)min((int64_t)a.W, t + 1);
    const int64_t p0 = t - nwin + 1;
    // ordered compaction of the valid selected entries
    const int32_t *irow = a.idx + (int64_t)row * a.K;
    int nsel = 0;
    for (int j0 = 0; j0 < a.K; j0 += kPThreads) {
      const int j = j0 + tid;
      int e = (j < a.K) ? irow[j] : -1;
      if (e >= a.n_entries || e < -1) { raise_status(a.status, STATUS_BAD_INDEX); e = -1; }
      const bool f = e >= 0;
      const unsigned bal = __ballot_sync(0xffffffffu, f);
      if (lane == 0) misc->wcount[warp] = __popc(bal);
      __syncthreads();
      int before = 0, tot = 0;
      for (int k = 0; k < kPThreads / 32; ++k) { if (k < warp) before += misc->wcount[k]; tot += misc->wcount[k]; }
      if (f) sel[nsel + before + __popc(bal & ((1u << lane) - 1u))] = e;
      nsel += tot;
      __syncthreads();
    }
    const int n_items = min(nsel + nwin, kMaxTiles * PT);
    const int ntiles = (n_items + PT - 1) / PT;
    // item scales
    for (int u = tid; u < ntiles * PT; u += kPThreads) {
      float sc = 0.f;
      if (u < nsel) sc = a.scales[(int64_t)b * a.entry_cap + sel[u]];
      else if (u < n_items) sc = a.wscales[(int64_t)b * a.win_cap + ((p0 + (u - nsel)) % a.win_cap)];
      iscale[u] = sc;
    }
    // Q -> shared memory (B operand of pass 1, K-major)
    {
      const uint4 *qrow = reinterpret_cast<const uint4 *>(a.q + (int64_t)row * PH * PD);
      for (int c = tid; c < PH * PD / 8; c += kPThreads) {
        const int h = (c >> 1) & 63, g = (c & 1) + 2 * (c >> 7);
        tc::cp_async16(smem + P_OFF_Q + pq_off(h, g), qrow + h * (PD / 8) + g, 16u);
      }
      tc::cp_async_commit();
    }

    // Block j of a pass covers items [tile*128, +128) and d [dblk*128, +128)
    // with tile = j / 4, dblk = j % 4.  Its 16 KiB of E4M3 codes are gathered
    // with cp.async into a staging ring that lives in shared memory the pass
    // does not use (pass 1: the P^T region, 5 slots; pass 2: the Q region, 4
    // slots), several blocks ahead; convert() turns a staged block into bf16
    // tiles.  Staging layout [item][8 x 16 B], chunk c of item i at slot
    // c ^ (i & 7) so that the conversion reads hit distinct banks.
    constexpr uint32_t STG = PT * PDB;                  // 16 KiB per block
    const int nblk_row = ntiles * (PD / PDB);
    auto issue = [&](int pass, int j) {
      if (j < nblk_row) {
        const int tile = j / (PD / PDB), dblk = j % (PD / PDB);
        const int nslot = pass == 0 ? 5 : 4;
        unsigned char *st = smem + (pass == 0 ? P_OFF_PT : P_OFF_Q) + (j % nslot) * STG;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c = tid + kPThreads * k;
          const int item = c >> 3, ch = c & 7;
          const int u = tile * PT + item;
          const uint8_t *src = nullptr;
          if (u < nsel) src = a.codes + ((int64_t)b * a.entry_cap + sel[u]) * PD;
          else if (u < n_items) src = a.wcodes + ((int64_t)b * a.win_cap + ((p0 + (u - nsel)) % a.win_cap)) * PD;
          tc::cp_async16(st + item * 128 + ((ch ^ (item & 7)) << 4),
                         src ? (const void *)(src + dblk * PDB + ch * 16) : (const void *)a.codes, src ? 16u : 0u);
        }
      }
      tc::cp_async_commit();
    };
    const int i8 = lane & 7, pq = lane >> 3;
    auto convert = [&](int pass, int j, int buf) {
      const int nslot = pass == 0 ? 5 : 4;
      const unsigned char *st = smem + (pass == 0 ? P_OFF_PT : P_OFF_Q) + (j % nslot) * STG;
      unsigned char *kv = smem + P_OFF_KV + buf * P_KV_BYTES;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int item = (warp * 2 + r) * 8 + i8;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int p = pq + 4 * k;                     // 16 codes -> d-groups 2p, 2p+1
          const uint4 c = *reinterpret_cast<const uint4 *>(st + item * 128 + ((p ^ (item & 7)) << 4));
          uint4 lo, hi;
          cvt16(c, lo, hi);
          *reinterpret_cast<uint4 *>(kv + pkv_off(item, 2 * p)) = lo;
          *reinterpret_cast<uint4 *>(kv + pkv_off(item, 2 * p + 1)) = hi;
        }
      }
      tc::fence_proxy_async_smem();
    };
    constexpr int AHEAD1 = 4, AHEAD2 = 3;               // blocks in flight per pass

    // ---------------------------------------------------------------- pass 1
    const int nblk = nblk_row;
    for (int j = 0; j < AHEAD1; ++j) issue(0, j);
    for (int j = 0; j < nblk && ok; ++j) {
      const int buf = j & 1;
      const int tile = j / (PD / PDB), dblk = j % (PD / PDB);
      issue(0, j + AHEAD1);                              // into the slot block j-1 used
      tc::cp_async_wait<AHEAD1>();                       // block j (and Q) have landed
      __syncthreads();
      if (!drain(buf)) { ok = false; break; }
      convert(0, j, buf);
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      if (tid == 0) {
        const uint32_t kvb = sbase + P_OFF_KV + buf * P_KV_BYTES;
#pragma unroll
        for (int k = 0; k < PDB / 16; ++k) {
          const uint64_t ad = tc::smem_desc(kvb + k * 4096, 2048, 128);
          const uint64_t bd = tc::smem_desc(sbase + P_OFF_Q + (dblk * 16 + 2 * k) * 1024, 1024, 128);
          tc::mma_bf16_ss(tbase + tile * PH, ad, bd, idesc_qk, (dblk > 0 || k > 0));
        }
        tc::mma_commit(&bars[buf]);
      }
      issued[buf] += 1u;
    }
    // all of pass 1 complete; Q is no longer read, so pass 2 may stage into it
    if (ok) ok = drain(0) && drain(1);
    if (!ok) break;
    tc::cp_async_wait<0>();
    __syncthreads();
    for (int j = 0; j < AHEAD2; ++j) issue(1, j);
    tc::fence_after_sync();

    // ---------------------------------------------------------------- softmax
    {
      const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
      float mx[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) mx[j] = -INFINITY;
      for (int tl = 0; tl < ntiles; ++tl) {
        uint32_t r[32];
        tc::tmem_ld32(tbase + lane_off + tl * PH + hhalf * 32, r);
        tc::tmem_wait_ld();
        const int it = tl * PT + quad * 32 + lane;
        const float f = (it < n_items) ? iscale[it] * qs : 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) mx[j] = fmaxf(mx[j], (it < n_items) ? __uint_as_float(r[j]) * f : -INFINITY);
      }
      const float wm = warp_transpose_reduce<true>(mx);      // max of head hhalf*32+lane over this quadrant
      red[quad * PH + hhalf * 32 + lane] = wm;
      __syncthreads();
      if (tid < PH) Mh[tid] = fmaxf(fmaxf(red[tid], red[PH + tid]), fmaxf(red[2 * PH + tid], red[3 * PH + tid]));
      __syncthreads();
      float sm_[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) sm_[j] = 0.f;
      float mrow[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) mrow[j] = Mh[hhalf * 32 + j];
      for (int tl = 0; tl < ntiles; ++tl) {
        uint32_t r[32];
        tc::tmem_ld32(tbase + lane_off + tl * PH + hhalf * 32, r);
        tc::tmem_wait_ld();
        const int it = tl * PT + quad * 32 + lane;
        const bool valid = it < n_items;
        const float sc = valid ? iscale[it] : 0.f;
        uint32_t pw[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float pa = valid ? exp2f(__uint_as_float(r[j]) * sc * qs - mrow[j]) : 0.f;
          const float pb = valid ? exp2f(__uint_as_float(r[j + 1]) * sc * qs - mrow[j + 1]) : 0.f;
          sm_[j] += pa;
          sm_[j + 1] += pb;
          const __nv_bfloat162 v = __floats2bfloat162_rn(pa * sc, pb * sc);
          pw[j >> 1] = *reinterpret_cast<const uint32_t *>(&v);
        }
#pragma unroll
        for (int hg = 0; hg < 4; ++hg)
          *reinterpret_cast<uint4 *>(smem + P_OFF_PT + ppt_off(it, hhalf * 4 + hg)) =
              make_uint4(pw[4 * hg], pw[4 * hg + 1], pw[4 * hg + 2], pw[4 * hg + 3]);
      }
      const float ws_ = warp_transpose_reduce<false>(sm_);
      red[quad * PH + hhalf * 32 + lane] = ws_;
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      if (tid < PH) Lh[tid] = red[tid] + red[PH + tid] + red[2 * PH + tid] + red[3 * PH + tid];
    }

    // ---------------------------------------------------------------- pass 2
    for (int j = 0; j < nblk && ok; ++j) {
      const int buf = j & 1;
      const int tile = j / (PD / PDB), dblk = j % (PD / PDB);
      issue(1, j + AHEAD2);
      tc::cp_async_wait<AHEAD2>();
      __syncthreads();
      if (!drain(buf)) { ok = false; break; }
      convert(1, j, buf);
      tc::fence_before_sync();
      __syncthreads();
      tc::fence_after_sync();
      if (tid == 0) {
        const uint32_t kvb = sbase + P_OFF_KV + buf * P_KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < PT / 16; ++kk) {
          // A = V^T (M = d, K = items), MN-major: LBO = item-group step (K), SBO = d-group step (M)
          const uint64_t ad = tc::smem_desc(kvb + kk * 256, 128, 2048);
          // B = P^T (N = heads, K = items), MN-major: LBO = item-group step (K), SBO = head-group step (N)
          const uint64_t bd = tc::smem_desc(sbase + P_OFF_PT + (tile * 16 + 2 * kk) * 1024, 1024, 128);
          tc::mma_bf16_ss(tbase + dblk * PH, ad, bd, idesc_pv, (tile > 0 || kk > 0));
        }
        tc::mma_commit(&bars[buf]);
      }
      issued[buf] += 1u;
    }
    tc::cp_async_wait<0>();
    if (ok) ok = drain(0) && drain(1);
    if (!ok) break;
    tc::fence_after_sync();

    // ---------------------------------------------------------------- epilogue
    // O^T block dblk: lanes = d (128), columns = heads.  Stage O[h][d] bf16 in
    // the (now idle) KV buffers, then write 64 x 512 bf16 rows coalesced.
    {
      const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
      __nv_bfloat16 *stage = reinterpret_cast<__nv_bfloat16 *>(smem + P_OFF_KV);   // [64][512]
      float inv[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) inv[j] = 1.f / Lh[hhalf * 32 + j];
      for (int dblk = 0; dblk < PD / PDB; ++dblk) {
        uint32_t r[32];
        tc::tmem_ld32(tbase + lane_off + dblk * PH + hhalf * 32, r);
        tc::tmem_wait_ld();
        const int d = dblk * PDB + quad * 32 + lane;
#pragma unroll
        for (int j = 0; j < 32; ++j) stage[(hhalf * 32 + j) * PD + d] = __float2bfloat16_rn(__uint_as_float(r[j]) * inv[j]);
      }
      tc::fence_before_sync();
      __syncthreads();
      uint4 *orow = reinterpret_cast<uint4 *>(a.out + (int64_t)row * PH * PD);
      const uint4 *src = reinterpret_cast<const uint4 *>(stage);
      for (int c = tid; c < PH * PD / 8; c += kPThreads) orow[c] = src[c];
      if (a.lse && tid < PH) a.lse[(int64_t)row * PH + tid] = (Mh[tid] + log2f(Lh[tid])) * 0.6931471805599453f;
      __syncthreads();
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tbase, 512);
}

}  // namespace

bool attend_prefill_supported(const csa_dims *d) {
  return d->H == PH && d->D == PD && (int64_t)d->K + d->W <= kMaxTiles * PT;
}

int launch_attend_prefill(const uint16_t *q, const uint8_t *codes, const float *scales, const int32_t *idx,
                          const uint8_t *wcodes, const float *wscales, const int32_t *q_pos,
                          const csa_dims *d, uint16_t *out, float *lse, cudaStream_t stream) {
  PArgs a;
  a.q = reinterpret_cast<const __nv_bfloat16 *>(q);
  a.codes = codes; a.scales = scales; a.idx = idx; a.wcodes = wcodes; a.wscales = wscales; a.q_pos = q_pos;
  a.rows = d->B * d->Tq; a.Tq = d->Tq; a.K = d->K; a.W = d->W; a.m = d->m; a.n_entries = d->n_entries;
  a.win_cap = d->win_cap; a.entry_cap = d->entry_cap; a.sm_scale = d->softmax_scale;
  a.out = reinterpret_cast<__nv_bfloat16 *>(out);
  a.lse = lse;
  a.status = status_word_device_ptr();
  if (int rc = set_smem_once((const void *)attend_prefill_kernel, (int)P_SMEM, "attend_prefill_kernel")) return rc;
  static int sms_cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return fail(CSA_ERR_CUDA, "attend: no device");
  if (!sms_cache[dev] && cudaDeviceGetAttribute(&sms_cache[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return fail(CSA_ERR_CUDA, "attend: cannot query the SM count");
  const int sms = sms_cache[dev];
  const int grid = a.rows < sms ? a.rows : sms;
  attend_prefill_kernel<<<grid, kPThreads, P_SMEM, stream>>>(a);
  count_launches(1);
  return check_launch("attend_prefill_kernel");
}

}  // namespace csa
