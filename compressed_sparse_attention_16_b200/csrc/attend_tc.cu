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
// across the CTA's chunks of 32 items.  Both halves of a row compute the same
// S (each needs the full 512-wide dot products) and keep bit-identical softmax
// state, so their halves combine without exchange.  The item splits of one
// (row, half) (1, 2, 4 or 8) form a thread-block cluster: each CTA writes its
// unnormalised partial O and per-head (max, sum) to the workspace (L2), one
// hardware cluster barrier orders them, and CTA c then combines the final
// rows of heads [c * 128 / S, +128 / S):
//   out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s.
// Q arrives by 32 TMA boxes of 128 heads x 16 d (32-byte swizzle, the layout
// the MMA reads); the CTA's gathered rows are prefetched into L2 right after
// the selection is compacted.
//
// Roles (288 threads):
//   warps 0-3  gather 32 items per chunk, convert E4M3 codes exactly to bf16
//              and store them in the "core matrix" layout (8 rows x 16 B);
//   warps 4-7  Q to shared memory (while the first chunks are gathered), then
//              softmax: one head per thread, lazy rescaling of O (only when a
//              chunk raises the running max by more than 2^8), P = p * scale
//              written to shared memory;
//   warp 8     TMEM allocation and the single MMA-issuing thread.
// Item scales multiply the logits and P, never the codes, so the bf16 tiles
// hold the E4M3 values exactly.  Every mbarrier wait is bounded by wall time;
// on expiry the CTA sets the library's status word and unwinds.
#include "common.cuh"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int TH = 128;          // heads = MMA M
constexpr int TD = 512;          // entry width
constexpr int CH = 32;           // items per chunk = QK MMA N
constexpr int DHALF = 256;       // output columns per CTA = PV MMA N
constexpr int kThreads = 288;
constexpr int kMaxSel = 2048;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;
constexpr unsigned long long kWaitNs = 2000000000ull;   // 2 s per wait

// shared memory map (bytes)
constexpr uint32_t OFF_Q = 0;                              // 128 x 512 bf16 = 128 KiB
constexpr uint32_t OFF_KV = OFF_Q + TH * TD * 2;           // 2 x (32 x 512 bf16) = 64 KiB
constexpr uint32_t KV_BYTES = CH * TD * 2;
constexpr uint32_t OFF_P = OFF_KV + 2 * KV_BYTES;          // 2 x (128 x 32 bf16) = 16 KiB
constexpr uint32_t P_BYTES = TH * CH * 2;
constexpr uint32_t OFF_SEL = OFF_P + 2 * P_BYTES;          // int32 [2048]
constexpr uint32_t OFF_SCALE = OFF_SEL + kMaxSel * 4;      // fp32 [2][32]
constexpr uint32_t OFF_BAR = OFF_SCALE + 2 * CH * 4;       // mbarriers
constexpr uint32_t OFF_MISC = OFF_BAR + 16 * 8;
constexpr uint32_t SMEM_BYTES = OFF_MISC + 64;

// TMEM columns
constexpr uint32_t TCOL_O = 0;        // 256 columns
constexpr uint32_t TCOL_S = 256;      // 2 x 32 columns
constexpr uint32_t TMEM_COLS = 512;

enum { BAR_KV_FULL = 0, BAR_KV_FREE = 2, BAR_S_FULL = 4, BAR_P_FULL = 6, BAR_PV_DONE = 8, BAR_FIN = 9,
       BAR_Q = 10 };

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
// the contraction-side dimension of each tile (8 bf16).  Every tile keeps
// the 8-row-group stride at 128 B and the other stride at most 2 KiB, so all
// descriptor strides stay small.
//   Q  [128 heads][512 d]:  not core matrices: 32 TMA boxes [128 heads][16 d]
//                           of 4 KiB with 32-byte swizzle, box k at k * 4096
//   KV [32 items][512 d]:   g = d/8,     g-stride 512 B,  item-group stride 128 B
//   P  [128 heads][32 items]: g = item/8, g-stride 2048 B, head-group stride 128 B
__device__ __forceinline__ uint32_t kv_off(int i, int g) { return g * 512 + (i >> 3) * 128 + (i & 7) * 16; }
__device__ __forceinline__ uint32_t p_off(int h, int g) { return g * 2048 + (h >> 3) * 128 + (h & 7) * 16; }

// 16 E4M3 codes -> 16 bf16 (exact), as two 16-byte words
__device__ __forceinline__ void e4m3x16_to_bf16(const uint4 &c, uint4 &lo, uint4 &hi) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
  uint32_t o[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 a = e4m3x2_to_float2((uint16_t)(w[k] & 0xFFFF));
    const float2 b = e4m3x2_to_float2((uint16_t)(w[k] >> 16));
    const __nv_bfloat162 ab = __float22bfloat162_rn(a);
    const __nv_bfloat162 bb = __float22bfloat162_rn(b);
    o[2 * k] = *reinterpret_cast<const uint32_t *>(&ab);
    o[2 * k + 1] = *reinterpret_cast<const uint32_t *>(&bb);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
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

__global__ void __launch_bounds__(kThreads, 1) attend_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                const Args a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  Misc *misc = reinterpret_cast<Misc *>(smem + OFF_MISC);
  int *sel = reinterpret_cast<int *>(smem + OFF_SEL);
  float *iscale = reinterpret_cast<float *>(smem + OFF_SCALE);

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
    for (int i = 0; i < 10; ++i) tc::mbar_init(&bars[i], (i == BAR_KV_FULL || i == BAR_KV_FULL + 1) ? 128
                                                       : (i == BAR_P_FULL || i == BAR_P_FULL + 1) ? 128 : 1);
    tc::mbar_init(&bars[BAR_Q], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (warp == 8) {
    tc::tmem_alloc(&misc->tmem_base, TMEM_COLS);
  } else if (a.idx) {
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
  const int nsel = a.idx ? misc->nsel : nvis;
  const int n_items = nsel + nwin;
  const int nch = (n_items + CH - 1) / CH;
  const int c_begin = split * a.cps;
  const int c_end = min(c_begin + a.cps, nch);
  const int nloc = max(0, c_end - c_begin);
  const uint32_t tbase = misc->tmem_base;
  const uint32_t sbase = tc::smem_u32(smem);
  if (warp == 8) {
    // Q (32 boxes of 128 heads x 16 d, 32-byte swizzle: box k is the A
    // operand of the k-th K step) while the loaders gather the first chunks
    if (lane == 0) {
      tc::mbar_arrive_expect_tx(&bars[BAR_Q], TH * TD * 2);
      for (int k = 0; k < TD / 16; ++k) tc::tma_load_2d(smem + OFF_Q + k * 4096, &qmap, 16 * k, row * TH, &bars[BAR_Q]);
    }
    // pull this CTA's gathered rows into L2 ahead of the loaders
    const int u1 = min(c_end * CH, n_items);
    for (int u = c_begin * CH + lane; u < u1; u += 32) {
      const uint8_t *src;
      if (u < nsel) src = a.codes + ((int64_t)b * a.entry_cap + (a.idx ? sel[u] : u)) * TD;
      else src = a.wcodes + ((int64_t)b * a.win_cap + ((p0 + (u - nsel)) % a.win_cap)) * TD;
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(TD) : "memory");
    }
  }

  if (warp < 4) {
    // ------------------------------------------------------------ loaders
    const int i8 = lane & 7, pq = lane >> 3;
    for (int lc = 0; lc < nloc; ++lc) {
      const int buf = lc & 1;
      const int item = warp * 8 + i8;
      const int u = (c_begin + lc) * CH + item;
      // Items past the list read a valid row (the first window token): their
      // logits are masked and their P is zero, so the finite codes do not
      // matter.  The loads are issued before waiting for the buffer.
      const uint8_t *src;
      const float *scp;
      if (u < nsel) {
        const int e = a.idx ? sel[u] : u;
        const int64_t ent = (int64_t)b * a.entry_cap + e;
        src = a.codes + ent * TD;
        scp = a.scales + ent;
      } else {
        const int64_t p = p0 + (u < n_items ? u - nsel : 0);
        const int64_t ent = (int64_t)b * a.win_cap + (p % a.win_cap);
        src = a.wcodes + ent * TD;
        scp = a.wscales + ent;
      }
      uint4 c[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) c[k] = __ldg(reinterpret_cast<const uint4 *>(src) + pq + 4 * k);
      const float sc_raw = __ldg(scp);
      if (lc >= 2 && !wait_bar(&bars[BAR_KV_FREE + buf], ((lc - 2) >> 1) & 1, misc, a.status)) break;
      const float sc = u < n_items ? sc_raw : 0.f;
      unsigned char *kv = smem + OFF_KV + buf * KV_BYTES;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const int p = pq + 4 * k;
        uint4 lo, hi;
        e4m3x16_to_bf16(c[k], lo, hi);
        *reinterpret_cast<uint4 *>(kv + kv_off(item, 2 * p)) = lo;
        *reinterpret_cast<uint4 *>(kv + kv_off(item, 2 * p + 1)) = hi;
      }
      if (pq == 0) iscale[buf * CH + item] = sc;
      tc::fence_proxy_async_smem();
      tc::mbar_arrive(&bars[BAR_KV_FULL + buf]);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ softmax
    const int quad = warp - 4;
    const int h = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float qs = a.sm_scale * kLog2e;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int c = 0; c < nloc && ok; ++c) {
      const int buf = c & 1;
      // kv_full orders the loaders' scale writes before this thread's reads
      // one decision per warp: the TMEM accesses and votes below are warp-collective
      if (!__all_sync(0xffffffffu, wait_bar(&bars[BAR_KV_FULL + buf], (c >> 1) & 1, misc, a.status) &&
                                       wait_bar(&bars[BAR_S_FULL + buf], (c >> 1) & 1, misc, a.status))) {
        ok = false;
        break;
      }
      tc::fence_after_sync();
      uint32_t sr[32];
      tc::tmem_ld32(tbase + lane_off + TCOL_S + buf * CH, sr);
      tc::tmem_wait_ld();
      const int valid = min(CH, n_items - (c_begin + c) * CH);
      float s[32];
      float mx = -INFINITY;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        s[j] = (j < valid) ? __uint_as_float(sr[j]) * iscale[buf * CH + j] * qs : -INFINITY;
        mx = fmaxf(mx, s[j]);
      }
      const bool need = mx > m_used + kRescaleLog2;
      if (c > 0 && __any_sync(0xffffffffu, need)) {
        // O holds earlier chunks: wait for the last PV, then rescale this warp's rows
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
      uint32_t pw[16];
      float lsum = 0.f;
#pragma unroll
      for (int j = 0; j < 32; j += 2) {
        const float pa = exp2f(s[j] - m_used), pb = exp2f(s[j + 1] - m_used);
        lsum += pa + pb;
        const __nv_bfloat162 v = __floats2bfloat162_rn(pa * iscale[buf * CH + j], pb * iscale[buf * CH + j + 1]);
        pw[j >> 1] = *reinterpret_cast<const uint32_t *>(&v);
      }
      l += lsum;
      unsigned char *P = smem + OFF_P + buf * P_BYTES;
#pragma unroll
      for (int g = 0; g < 4; ++g)
        *reinterpret_cast<uint4 *>(P + p_off(h, g)) = make_uint4(pw[4 * g], pw[4 * g + 1], pw[4 * g + 2], pw[4 * g + 3]);
      tc::fence_proxy_async_smem();
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
#pragma unroll 1
      for (int blk = 0; blk < DHALF / 32; ++blk) {
        uint32_t o[32];
        if (have) {
          tc::tmem_ld32(tbase + lane_off + TCOL_O + blk * 32, o);
          tc::tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = 0u;
        }
        uint4 *dst = reinterpret_cast<uint4 *>(dstb + ((int64_t)blk * TH + h) * 32);
#pragma unroll
        for (int k = 0; k < 8; ++k) dst[k] = make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
      }
      a.ws_ml[slot * TH + h] = have ? make_float2(m_used, l) : make_float2(-INFINITY, 0.f);
    }
  } else {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nloc > 0) {
      const uint32_t idesc_qk = tc::idesc_bf16_f32(128, CH, 0, 0);
      const uint32_t idesc_pv = tc::idesc_bf16_f32(128, DHALF, 0, 1);
      auto issue_qk = [&](int c) {
        const int buf = c & 1;
        const uint32_t kvb = sbase + OFF_KV + buf * KV_BYTES;
#pragma unroll 4
        for (int k = 0; k < TD / 16; ++k) {
          // A = Q, K-major with 32-byte swizzle (one TMA box per K step);
          // B = items, K-major core matrices: LBO = step between d-groups, SBO = 8-row groups
          const uint64_t ad = tc::smem_desc_sw32(sbase + OFF_Q + k * 4096);
          const uint64_t bd = tc::smem_desc(kvb + k * 1024, 512, 128);
          tc::mma_bf16_ss(tbase + TCOL_S + buf * CH, ad, bd, idesc_qk, k > 0);
        }
        tc::mma_commit(&bars[BAR_S_FULL + buf]);
      };
      bool ok = wait_bar(&bars[BAR_Q], 0, misc, a.status) && wait_bar(&bars[BAR_KV_FULL + 0], 0, misc, a.status);
      if (ok) { tc::fence_after_sync(); issue_qk(0); }
      if (ok && nloc > 1) {
        ok = wait_bar(&bars[BAR_KV_FULL + 1], 0, misc, a.status);
        if (ok) { tc::fence_after_sync(); issue_qk(1); }
      }
      for (int c = 0; c < nloc && ok; ++c) {
        const int buf = c & 1;
        if (!wait_bar(&bars[BAR_P_FULL + buf], (c >> 1) & 1, misc, a.status)) break;
        tc::fence_after_sync();
        const uint32_t pb = sbase + OFF_P + buf * P_BYTES;
        const uint32_t vb = sbase + OFF_KV + buf * KV_BYTES + dh * (DHALF / 8) * 512;
#pragma unroll
        for (int kk = 0; kk < CH / 16; ++kk) {
          // A = P, K-major (K = items).  B = the same item tile read MN-major
          // (N = d): LBO = step between item groups (K), SBO = between d-groups (N)
          const uint64_t ad = tc::smem_desc(pb + kk * 4096, 2048, 128);
          const uint64_t bd = tc::smem_desc(vb + kk * 256, 128, 512);
          tc::mma_bf16_ss(tbase + TCOL_O, ad, bd, idesc_pv, (c > 0 || kk > 0));
        }
        tc::mma_commit(&bars[BAR_KV_FREE + buf]);
        tc::mma_commit(&bars[BAR_PV_DONE]);
        if (c + 2 < nloc) {
          if (!wait_bar(&bars[BAR_KV_FULL + buf], ((c + 2) >> 1) & 1, misc, a.status)) break;
          tc::fence_after_sync();
          issue_qk(c + 2);
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
      for (int hl = warp; hl < hper; hl += 8) {
        const int h = split * hper + hl;
        const float2 ml = lane < S ? __ldcg(a.ws_ml + (slot0 + lane) * TH + h) : make_float2(-INFINITY, 0.f);
        // every source's row in flight before any use
        float4 v0[8], v1[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          v0[j] = v1[j] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (j < S) {
            // d = 8 lane .. 8 lane + 7: block lane / 4, offset 8 (lane % 4)
            const float4 *src = reinterpret_cast<const float4 *>(
                a.ws_o + (slot0 + j) * TH * DHALF + ((int64_t)(lane >> 2) * TH + h) * 32 + (lane & 3) * 8);
            v0[j] = __ldcg(src);
            v1[j] = __ldcg(src + 1);
          }
        }
        float M = ml.x;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float wgt = (ml.y > 0.f) ? exp2f(ml.x - M) : 0.f;
        float L = wgt * ml.y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        float acc[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float wj = __shfl_sync(0xffffffffu, wgt, j);
          acc[0] += wj * v0[j].x; acc[1] += wj * v0[j].y; acc[2] += wj * v0[j].z; acc[3] += wj * v0[j].w;
          acc[4] += wj * v1[j].x; acc[5] += wj * v1[j].y; acc[6] += wj * v1[j].z; acc[7] += wj * v1[j].w;
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
  }
  if (warp == 8) tc::tmem_dealloc(tbase, TMEM_COLS);
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
  if (int rc = set_smem_once((const void *)attend_tc_kernel, (int)SMEM_BYTES, "attend_tc_kernel")) return rc;
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
  const cudaError_t e = cudaLaunchKernelEx(&cfg, attend_tc_kernel, qmap, a);
  count_launches(1);
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "attend_tc_kernel launch: %s", cudaGetErrorString(e));
  return check_launch("attend_tc_kernel");
}

}  // namespace csa
