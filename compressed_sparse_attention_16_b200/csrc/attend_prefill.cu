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
//            shared memory; P^T = p * entry scale is written as fp16;
//   pass 2   O^T[d, head] = V^T . P^T  (M = 128 d per block, N = 64 heads,
//            K = items), reading the same [item][d] tiles MN-major, one
//            128-wide d block at a time into two alternating 64-column TMEM
//            buffers;
//   epilogue O / l straight from TMEM to the bf16 output rows.
//
// Roles (persistent CTAs, one per SM, query rows round-robin):
//   warps 0-7   producers: per row, compact the selection into item row
//               numbers and scales, convert Q, then gather every 128 x 128
//               block of E4M3 codes (twice: once per pass) through registers,
//               three blocks ahead, convert it exactly to fp16 and hand it to
//               the tensor core through a two-slot shared-memory ring;
//   warps 8-11  softmax of a row, then its epilogue (which overlaps pass 1 of
//               the next row);
//   warp 12     issues the MMAs (one thread) and commits them to mbarriers.
// Every wait is bounded; a wait that gives up raises STATUS_TIMEOUT and turns
// every later wait of the CTA into a no-op, so all roles run to the end.
//
// fp16 operands: E4M3 -> fp16 is exact.  Q and P^T are brought into fp16's
// range by exact powers of two:
//   Q    one factor 2^kq per row puts max|q| in [2^14, 2^15): every bf16 value
//        down to 2^-31 of the row maximum converts exactly; the factor is
//        divided out of the scores in fp32;
//   P^T  exp2(x - max_h - E), with the integer E chosen from the row's largest
//        entry scale so that p * scale <= 2^15.  The same shift divides the
//        softmax denominator, so O = sum(P^T v) / sum(p) needs no correction
//        and the log-sum-exp adds E back.
#include "common.cuh"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int PH = 64;             // heads (MMA N)
constexpr int PD = 512;            // entry width
constexpr int PT = 128;            // items per tile (MMA M of pass 1)
constexpr int PDB = 128;           // d per block
constexpr int kMaxTiles = 5;       // <= 640 items per row
constexpr int kMaxItems = kMaxTiles * PT;
constexpr int kProd = 256;         // producer threads (warps 0-7)
constexpr int kSoft = 128;         // softmax / epilogue threads (warps 8-11)
constexpr int kThreads = kProd + kSoft + 32;
constexpr int kMmaWarp = (kProd + kSoft) / 32;
constexpr float kPLog2e = 1.4426950408889634f;
constexpr unsigned long long kPWaitNs = 2000000000ull;
constexpr uint32_t kOCol = kMaxTiles * PH;   // O^T buffers: columns [320, 448)

// shared memory map (bytes)
constexpr uint32_t S_Q = 0;                                  // fp16 [64 h][512 d]          64 KiB
constexpr uint32_t S_PT = S_Q + PH * PD * 2;                 // fp16 [640 i][64 h]          80 KiB
constexpr uint32_t S_KV = S_PT + kMaxItems * PH * 2;         // fp16 2 x [128 i][128 d]     64 KiB
constexpr uint32_t KV_BYTES = PT * PDB * 2;
constexpr uint32_t S_ITEM = S_KV + 2 * KV_BYTES;             // int32 [2][640] item rows
constexpr uint32_t S_SCALE = S_ITEM + 2 * kMaxItems * 4;     // fp32 [2][640] item scales
constexpr uint32_t S_INFO = S_SCALE + 2 * kMaxItems * 4;     // RowInfo [2]
constexpr uint32_t S_RED = S_INFO + 2 * 32;                  // fp32 [4][64], M[64], L[64], 1/L[64]
constexpr uint32_t S_PRED = S_RED + 8 * PH * 4;              // producer reductions, u32 [16]
constexpr uint32_t S_BAR = S_PRED + 16 * 4;
constexpr int kNumBars = 16;
constexpr uint32_t S_MISC = S_BAR + kNumBars * 8;
constexpr uint32_t P_SMEM = S_MISC + 32;
static_assert(P_SMEM <= 232448, "shared memory");

// mbarriers
enum : int {
  B_FULL = 0,      // [2] producers -> MMA: ring slot converted (one arrival per warp)
  B_EMPTY = 2,     // [2] MMA -> producers: ring slot read (commit)
  B_READY = 4,     // [2] producers -> all: row set-up done, by row parity (one per warp)
  B_P1DONE = 6,    // MMA -> softmax, producers: S^T complete, Q no longer read (commit)
  B_PTFULL = 7,    // softmax -> MMA: P^T written, S^T read (1 arrival)
  B_P2DONE = 8,    // MMA -> softmax: P^T no longer read (commit)
  B_OFULL = 9,     // [2] MMA -> epilogue: O^T buffer complete (commit)
  B_OEMPTY = 11,   // [2] epilogue -> MMA: O^T buffer read (one arrival per warp)
  B_FINAL = 13,    // all MMAs complete (commit)
};

// Q  [64 h][512 d]:   d-group stride 1024, head-group stride 128
// KV [128 i][128 d]:  d-group stride 2048, item-group stride 128
// PT [640 i][64 h]:   item-group stride 1024, head-group stride 128
__device__ __forceinline__ uint32_t pq_off(int h, int g) { return g * 1024 + (h >> 3) * 128 + (h & 7) * 16; }
__device__ __forceinline__ uint32_t pkv_off(int i, int g) { return g * 2048 + (i >> 3) * 128 + (i & 7) * 16; }
__device__ __forceinline__ uint32_t ppt_off(int i, int hg) { return (i >> 3) * 1024 + hg * 128 + (i & 7) * 16; }

struct RowInfo {
  int row, n_items, ntiles, pad0;
  float qscale;      // softmax scale * log2(e) / 2^kq
  float eshift;      // E
  float pad1[2];
};

struct PMisc {
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ uint64_t ptimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait for the phase of parity `parity`.  After any wait of the CTA
// has given up, returns false at once.
__device__ __forceinline__ bool pwait(uint64_t *bar, uint32_t parity, PMisc *misc, unsigned *status) {
  volatile int *abort = &misc->abort;
  if (*abort) return false;
  if (tc::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptimer();
  uint32_t n = 0;
  while (!tc::mbar_try_wait(bar, parity)) {
    if ((++n & 63u) == 0) {
      if (*abort) return false;
      if (ptimer() - t0 > kPWaitNs) {
        *abort = 1;
        raise_status(status, STATUS_TIMEOUT);
        return false;
      }
    }
  }
  return true;
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two E4M3 codes -> two fp16 (exact: every finite E4M3 value is an fp16).
__device__ __forceinline__ uint32_t e4m3x2_to_h2(uint32_t two) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

__device__ __forceinline__ void cvt16(const uint4 &c, uint4 &lo, uint4 &hi) {
  lo = make_uint4(e4m3x2_to_h2(c.x & 0xFFFFu), e4m3x2_to_h2(c.x >> 16), e4m3x2_to_h2(c.y & 0xFFFFu),
                  e4m3x2_to_h2(c.y >> 16));
  hi = make_uint4(e4m3x2_to_h2(c.z & 0xFFFFu), e4m3x2_to_h2(c.z >> 16), e4m3x2_to_h2(c.w & 0xFFFFu),
                  e4m3x2_to_h2(c.w >> 16));
}

// Two bf16 (packed) times an exact power of two -> two fp16 (packed).
__device__ __forceinline__ uint32_t bf2_to_h2(uint32_t w, float f) {
  const __half2 h = __floats2half2_rn(__uint_as_float(w << 16) * f, __uint_as_float(w & 0xFFFF0000u) * f);
  return *reinterpret_cast<const uint32_t *>(&h);
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

// ------------------------------------------------------------------ producers
// The producers walk one stream of blocks over all rows of the CTA.  Row it
// has nbt = 8 * ntiles blocks: j < nb1 = 4 * ntiles is pass 1, tile j / 4, d
// block j % 4; j = nb1 + jj is pass 2, d block jj / ntiles, tile jj % ntiles.
// Blocks are gathered into registers three ahead of the one being converted
// (across row boundaries); the set-up of row it + 1 (selection, scales, Q)
// runs once pass 1 of row it has been handed over, while the softmax of row it
// keeps the tensor core waiting anyway.
__device__ __forceinline__ void run_producers(const PArgs &a, unsigned char *smem, int nrows) {
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S_BAR);
  PMisc *misc = reinterpret_cast<PMisc *>(smem + S_MISC);
  RowInfo *info = reinterpret_cast<RowInfo *>(smem + S_INFO);
  uint32_t *pred = reinterpret_cast<uint32_t *>(smem + S_PRED);
  const int tid = threadIdx.x, pw = tid >> 5, lane = tid & 31;
  const int i8 = lane & 7, cq = lane >> 3;
  const float qs = a.sm_scale * kPLog2e;
  int ni0 = 0, ni1 = 0, nt0 = 0, nt1 = 0;   // n_items / ntiles of the rows of parity 0 / 1

  // ---- per-row set-up: item rows and scales, Q in fp16, RowInfo
  auto setup = [&](int it) {
    const int row = blockIdx.x + it * gridDim.x;
    const int par = it & 1;
    int *irow = reinterpret_cast<int *>(smem + S_ITEM) + par * kMaxItems;
    float *isc = reinterpret_cast<float *>(smem + S_SCALE) + par * kMaxItems;
    const int b = row / a.Tq;
    int64_t t = a.q_pos[row];
    if (t < 0) {
      if (tid == 0) raise_status(a.status, STATUS_BAD_POSITION);
      t = 0;
    }
    const int nwin = (int)min((int64_t)a.W, t + 1);
    const int64_t p0 = t - nwin + 1;
    // ordered compaction of the valid selected entries into item rows:
    // r >= 0 is row r of the entry cache, r < 0 row -r-1 of the window ring
    const int32_t *idx = a.idx + (int64_t)row * a.K;
    int nsel = 0;
    for (int j0 = 0; j0 < a.K; j0 += kProd) {
      const int j = j0 + tid;
      int e = (j < a.K) ? idx[j] : -1;
      if (e >= a.n_entries || e < -1) { raise_status(a.status, STATUS_BAD_INDEX); e = -1; }
      const bool f = e >= 0;
      const unsigned bal = __ballot_sync(0xffffffffu, f);
      if (lane == 0) pred[pw] = __popc(bal);
      named_sync(1, kProd);
      int before = 0, tot = 0;
#pragma unroll
      for (int k = 0; k < kProd / 32; ++k) {
        const int c = (int)pred[k];
        before += (k < pw) ? c : 0;
        tot += c;
      }
      if (f) {
        const int u = nsel + before + __popc(bal & ((1u << lane) - 1u));
        const int64_t r = (int64_t)b * a.entry_cap + e;
        irow[u] = (int)r;
        isc[u] = a.scales[r];
      }
      nsel += tot;
      named_sync(1, kProd);
    }
    const int n_items = min(nsel + nwin, kMaxItems);
    for (int u = nsel + tid; u < n_items; u += kProd) {
      const int64_t r = (int64_t)b * a.win_cap + (p0 + (u - nsel)) % a.win_cap;
      irow[u] = (int)(-r - 1);
      isc[u] = a.wscales[r];
    }
    const int ntiles = (n_items + PT - 1) / PT;
    if (par) { ni1 = n_items; nt1 = ntiles; } else { ni0 = n_items; nt0 = ntiles; }
    named_sync(1, kProd);

    // Q: thread (pw, lane) holds head (lane & 7) + 8 pw, d-groups (lane >> 3) + 4 k;
    // read twice (max, then convert) to keep few registers live
    const uint4 *qg = reinterpret_cast<const uint4 *>(a.q + (int64_t)row * PH * PD);
    const int h = i8 + 8 * pw;
    uint32_t mq = 0;
#pragma unroll 4
    for (int k = 0; k < 16; ++k) {
      const uint4 v = __ldg(qg + h * (PD / 8) + cq + 4 * k);
      mq = __vmaxu2(mq, __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                 __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
    }
    float smax = 0.f;
    for (int u = tid; u < n_items; u += kProd) smax = fmaxf(smax, isc[u]);
    mq = __reduce_max_sync(0xffffffffu, max(mq & 0xFFFFu, mq >> 16));
    const uint32_t sbits = __reduce_max_sync(0xffffffffu, __float_as_uint(smax));   // smax >= 0
    if (lane == 0) { pred[pw] = mq; pred[8 + pw] = sbits; }
    named_sync(1, kProd);
    uint32_t amax = 0, smb = 0;
#pragma unroll
    for (int k = 0; k < kProd / 32; ++k) { amax = max(amax, pred[k]); smb = max(smb, pred[8 + k]); }
    // bf16 |q| max in [2^(eb-127), 2^(eb-126)) -> times 2^(141-eb) in [2^14, 2^15)
    const int kq = amax ? min(126, 141 - (int)((amax >> 7) & 0xFFu)) : 0;
    const float fq = __int_as_float((kq + 127) << 23);
    if (tid == 0) {
      RowInfo ri;
      ri.row = row; ri.n_items = n_items; ri.ntiles = ntiles; ri.pad0 = 0;
      ri.qscale = qs * __int_as_float((127 - kq) << 23);
      // largest scale < 2^(e - 126) for biased exponent e; p * scale * 2^-E <= 2^15
      const int e = (int)((smb >> 23) & 0xFFu);
      ri.eshift = (float)min(104, max(-110, e - 141));
      ri.pad1[0] = ri.pad1[1] = 0.f;
      info[par] = ri;
    }
    // the Q buffer is free once pass 1 of the previous row is complete
    if (it > 0) pwait(&bars[B_P1DONE], (it - 1) & 1, misc, a.status);
    unsigned char *qs_ = smem + S_Q;
#pragma unroll 4
    for (int k = 0; k < 16; ++k) {
      const uint4 v = __ldg(qg + h * (PD / 8) + cq + 4 * k);
      *reinterpret_cast<uint4 *>(qs_ + pq_off(h, cq + 4 * k)) =
          make_uint4(bf2_to_h2(v.x, fq), bf2_to_h2(v.y, fq), bf2_to_h2(v.z, fq), bf2_to_h2(v.w, fq));
    }
    tc::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&bars[B_READY + par]);
  };

  // ---- block gather: thread (pw, lane) holds items (2 pw + (k & 1)) * 8 +
  // (lane & 7) of the tile, 16-byte chunks (k >> 1) * 4 + (lane >> 3) of the
  // d block, k = 0..3.  Items past n_items read item 0 (always valid): their
  // scores are masked and their P^T rows are zero.
  auto block_of = [&](int it, int j, int &tile, int &dblk) {
    const int ntiles = (it & 1) ? nt1 : nt0;
    const int nb1 = ntiles * (PD / PDB);
    if (j < nb1) { tile = j >> 2; dblk = j & 3; }
    else { const int jj = j - nb1; dblk = jj / ntiles; tile = jj - dblk * ntiles; }
  };
  auto load_blk = [&](int it, int j, uint4 (&v)[4]) {
    int tile, dblk;
    block_of(it, j, tile, dblk);
    const int n_items = (it & 1) ? ni1 : ni0;
    const int *irow = reinterpret_cast<const int *>(smem + S_ITEM) + (it & 1) * kMaxItems;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int u = tile * PT + (2 * pw + (k & 1)) * 8 + i8;
      u = u < n_items ? u : 0;
      const int r = irow[u];
      const uint8_t *base = r >= 0 ? a.codes + (int64_t)r * PD : a.wcodes + (int64_t)(-r - 1) * PD;
      v[k] = __ldg(reinterpret_cast<const uint4 *>(base + dblk * PDB + ((k >> 1) * 4 + cq) * 16));
    }
  };
  uint32_t nblk = 0;   // blocks handed over so far (ring slot = nblk & 1)
  auto produce = [&](const uint4 (&v)[4]) {
    const uint32_t slot = nblk & 1u, use = nblk >> 1;
    if (use > 0 && lane == 0) pwait(&bars[B_EMPTY + slot], (use - 1) & 1u, misc, a.status);
    __syncwarp();
    unsigned char *kv = smem + S_KV + slot * KV_BYTES;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int il = (2 * pw + (k & 1)) * 8 + i8;
      const int ch = (k >> 1) * 4 + cq;
      uint4 lo, hi;
      cvt16(v[k], lo, hi);
      *reinterpret_cast<uint4 *>(kv + pkv_off(il, 2 * ch)) = lo;
      *reinterpret_cast<uint4 *>(kv + pkv_off(il, 2 * ch + 1)) = hi;
    }
    // every lane's writes reach the async proxy before the warp's single arrival
    tc::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&bars[B_FULL + slot]);
    ++nblk;
  };
  auto nbt_of = [&](int it) { return ((it & 1) ? nt1 : nt0) * 2 * (PD / PDB); };

  if (nrows <= 0) return;
  setup(0);
  int p_it = 0, p_j = 0;   // next block to hand over
  int l_it = 0, l_j = 0;   // next block to gather
  auto step = [&](uint4 (&v)[4]) {
    if (p_it < nrows) {
      if (p_j == nbt_of(p_it) / 2 && p_it + 1 < nrows) setup(p_it + 1);
      produce(v);
      if (++p_j == nbt_of(p_it)) { ++p_it; p_j = 0; }
    }
    if (l_it < nrows) {
      load_blk(l_it, l_j, v);
      if (++l_j == nbt_of(l_it)) { ++l_it; l_j = 0; }
    }
  };
  uint4 A[4], B[4], C[4];
  load_blk(0, 0, A);
  load_blk(0, 1, B);
  load_blk(0, 2, C);
  l_j = 3;   // a row has at least 8 blocks
  while (p_it < nrows) {
    step(A);
    step(B);
    step(C);
  }
}

// -------------------------------------------------------------------- softmax
__device__ __forceinline__ void run_softmax(const PArgs &a, unsigned char *smem, int nrows, uint32_t tbase) {
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S_BAR);
  PMisc *misc = reinterpret_cast<PMisc *>(smem + S_MISC);
  const RowInfo *info = reinterpret_cast<const RowInfo *>(smem + S_INFO);
  float *red = reinterpret_cast<float *>(smem + S_RED);   // [4][64]
  float *Mh = red + 4 * PH;
  float *Lh = Mh + PH;
  float *invL = Lh + PH;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sq = warp - kProd / 32;        // TMEM lane quadrant
  const int stid = tid - kProd;
  const uint32_t lane_off = (uint32_t)(sq * 32) << 16;
  uint32_t ouse = 0;

  for (int it = 0; it < nrows; ++it) {
    const int par = it & 1;
    pwait(&bars[B_READY + par], (it >> 1) & 1, misc, a.status);
    const RowInfo ri = info[par];
    const float *isc = reinterpret_cast<const float *>(smem + S_SCALE) + par * kMaxItems;
    pwait(&bars[B_P1DONE], it & 1, misc, a.status);
    tc::fence_after_sync();

    // max over items of x = score * scale * log2(e), per head
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
      float mx[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) mx[j] = -INFINITY;
      for (int tl = 0; tl < ri.ntiles; ++tl) {
        uint32_t r[32];
        tc::tmem_ld32(tbase + lane_off + tl * PH + hh * 32, r);
        tc::tmem_wait_ld();
        const int u = tl * PT + sq * 32 + lane;
        const bool valid = u < ri.n_items;
        const float f = valid ? isc[u] * ri.qscale : 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) mx[j] = fmaxf(mx[j], valid ? __uint_as_float(r[j]) * f : -INFINITY);
      }
      red[sq * PH + hh * 32 + lane] = warp_transpose_reduce<true>(mx);
    }
    named_sync(2, kSoft);
    if (stid < PH) Mh[stid] = fmaxf(fmaxf(red[stid], red[PH + stid]), fmaxf(red[2 * PH + stid], red[3 * PH + stid]));
    named_sync(2, kSoft);

    // P^T may be overwritten once pass 2 of the previous row is complete
    if (it > 0) pwait(&bars[B_P2DONE], (it - 1) & 1, misc, a.status);
#pragma unroll 1
    for (int hh = 0; hh < 2; ++hh) {
      // the shifted row maxima stay in shared memory (broadcast reads): fewer live registers
      float *Ms = invL;                              // [64] free until the epilogue
      if (hh == 0 && stid < PH) Ms[stid] = Mh[stid] + ri.eshift;
      named_sync(2, kSoft);
      float sm[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) sm[j] = 0.f;
      for (int tl = 0; tl < ri.ntiles; ++tl) {
        uint32_t r[32];
        tc::tmem_ld32(tbase + lane_off + tl * PH + hh * 32, r);
        tc::tmem_wait_ld();
        const int u = tl * PT + sq * 32 + lane;
        const bool valid = u < ri.n_items;
        const float sc = valid ? isc[u] : 0.f;
        const float f = sc * ri.qscale;
        uint32_t pw[16];
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 mm = *reinterpret_cast<const float2 *>(Ms + hh * 32 + j);
          const float pa = valid ? ex2(__uint_as_float(r[j]) * f - mm.x) : 0.f;
          const float pb = valid ? ex2(__uint_as_float(r[j + 1]) * f - mm.y) : 0.f;
          sm[j] += pa;
          sm[j + 1] += pb;
          const __half2 v = __floats2half2_rn(pa * sc, pb * sc);
          pw[j >> 1] = *reinterpret_cast<const uint32_t *>(&v);
        }
#pragma unroll
        for (int hg = 0; hg < 4; ++hg)
          *reinterpret_cast<uint4 *>(smem + S_PT + ppt_off(u, hh * 4 + hg)) =
              make_uint4(pw[4 * hg], pw[4 * hg + 1], pw[4 * hg + 2], pw[4 * hg + 3]);
      }
      red[sq * PH + hh * 32 + lane] = warp_transpose_reduce<false>(sm);
    }
    tc::fence_proxy_async_smem();
    tc::fence_before_sync();
    named_sync(2, kSoft);
    if (stid == 0) tc::mbar_arrive(&bars[B_PTFULL]);
    if (stid < PH) {
      const float L = red[stid] + red[PH + stid] + red[2 * PH + stid] + red[3 * PH + stid];
      Lh[stid] = L;
      invL[stid] = 1.f / L;
      if (a.lse) a.lse[(int64_t)ri.row * PH + stid] = (Mh[stid] + ri.eshift + log2f(L)) * 0.6931471805599453f;
    }
    named_sync(2, kSoft);

    // epilogue: O^T block dblk, lanes = d, columns = heads
    __nv_bfloat16 *orow = a.out + (int64_t)ri.row * PH * PD;
#pragma unroll 1
    for (int dblk = 0; dblk < PD / PDB; ++dblk) {
      const uint32_t ob = ouse & 1u, use = ouse >> 1;
      pwait(&bars[B_OFULL + ob], use & 1u, misc, a.status);
      tc::fence_after_sync();
      uint32_t r0[32], r1[32];
      tc::tmem_ld32(tbase + lane_off + kOCol + ob * PH, r0);
      tc::tmem_ld32(tbase + lane_off + kOCol + ob * PH + 32, r1);
      tc::tmem_wait_ld();
      tc::fence_before_sync();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&bars[B_OEMPTY + ob]);
      ++ouse;
      __nv_bfloat16 *o = orow + dblk * PDB + sq * 32 + lane;
#pragma unroll
      for (int j = 0; j < 32; ++j) o[j * PD] = __float2bfloat16_rn(__uint_as_float(r0[j]) * invL[j]);
#pragma unroll
      for (int j = 0; j < 32; ++j) o[(32 + j) * PD] = __float2bfloat16_rn(__uint_as_float(r1[j]) * invL[32 + j]);
    }
  }
}

// ------------------------------------------------------------------------ MMA
__device__ __forceinline__ void run_mma(const PArgs &a, unsigned char *smem, int nrows, uint32_t tbase) {
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S_BAR);
  PMisc *misc = reinterpret_cast<PMisc *>(smem + S_MISC);
  const RowInfo *info = reinterpret_cast<const RowInfo *>(smem + S_INFO);
  const bool leader = (threadIdx.x & 31) == 0;
  const uint32_t sbase = tc::smem_u32(smem);
  const uint32_t idesc_qk = tc::idesc_f16_f32(128, PH, 0, 0);
  const uint32_t idesc_pv = tc::idesc_f16_f32(128, PH, 1, 1);
  uint32_t ncons = 0, ouse = 0;

  for (int it = 0; it < nrows; ++it) {
    const int par = it & 1;
    pwait(&bars[B_READY + par], (it >> 1) & 1, misc, a.status);
    const int ntiles = info[par].ntiles;
    // pass 1: S^T[tile] += K[tile, dblk] . Q[:, dblk]^T
    for (int j = 0; j < ntiles * (PD / PDB); ++j) {
      const uint32_t slot = ncons & 1u, use = ncons >> 1;
      pwait(&bars[B_FULL + slot], use & 1u, misc, a.status);
      tc::fence_after_sync();
      if (leader) {
        const int tile = j >> 2, dblk = j & 3;
        const uint32_t kvb = sbase + S_KV + slot * KV_BYTES;
#pragma unroll
        for (int k = 0; k < PDB / 16; ++k) {
          // A = K tile (M = items, K = d), K-major: LBO = d-group step, SBO = item-group step
          const uint64_t ad = tc::smem_desc(kvb + k * 4096, 2048, 128);
          // B = Q (N = heads, K = d), K-major: LBO = d-group step, SBO = head-group step
          const uint64_t bd = tc::smem_desc(sbase + S_Q + (dblk * 16 + 2 * k) * 1024, 1024, 128);
          tc::mma_bf16_ss(tbase + tile * PH, ad, bd, idesc_qk, (dblk > 0 || k > 0));
        }
        tc::mma_commit(&bars[B_EMPTY + slot]);
      }
      __syncwarp();
      ++ncons;
    }
    if (leader) tc::mma_commit(&bars[B_P1DONE]);
    __syncwarp();
    pwait(&bars[B_PTFULL], it & 1, misc, a.status);
    tc::fence_after_sync();
    // pass 2: O^T[dblk] = sum over tiles of V^T[tile, dblk] . P^T[tile]
    for (int dblk = 0; dblk < PD / PDB; ++dblk) {
      const uint32_t ob = ouse & 1u, ou = ouse >> 1;
      if (ou > 0) pwait(&bars[B_OEMPTY + ob], (ou - 1) & 1u, misc, a.status);
      tc::fence_after_sync();
      for (int tile = 0; tile < ntiles; ++tile) {
        const uint32_t slot = ncons & 1u, use = ncons >> 1;
        pwait(&bars[B_FULL + slot], use & 1u, misc, a.status);
        tc::fence_after_sync();
        if (leader) {
          const uint32_t kvb = sbase + S_KV + slot * KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < PT / 16; ++kk) {
            // A = V^T (M = d, K = items), MN-major: LBO = item-group step, SBO = d-group step
            const uint64_t ad = tc::smem_desc(kvb + kk * 256, 128, 2048);
            // B = P^T (N = heads, K = items), MN-major: LBO = item-group step, SBO = head-group step
            const uint64_t bd = tc::smem_desc(sbase + S_PT + (tile * 16 + 2 * kk) * 1024, 1024, 128);
            tc::mma_bf16_ss(tbase + kOCol + ob * PH, ad, bd, idesc_pv, (tile > 0 || kk > 0));
          }
          tc::mma_commit(&bars[B_EMPTY + slot]);
        }
        __syncwarp();
        ++ncons;
      }
      if (leader) tc::mma_commit(&bars[B_OFULL + ob]);
      __syncwarp();
      ++ouse;
    }
    if (leader) tc::mma_commit(&bars[B_P2DONE]);
    __syncwarp();
  }
  // every MMA issued above completes before the TMEM is released
  if (leader) tc::mma_commit(&bars[B_FINAL]);
  __syncwarp();
  const uint64_t t0 = ptimer();
  while (!tc::mbar_try_wait(&bars[B_FINAL], 0)) {
    if (ptimer() - t0 > kPWaitNs) { raise_status(a.status, STATUS_TIMEOUT); break; }
  }
}

__global__ void __launch_bounds__(kThreads, 1) attend_prefill_kernel(const PArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S_BAR);
  PMisc *misc = reinterpret_cast<PMisc *>(smem + S_MISC);
  const int tid = threadIdx.x, warp = tid >> 5;
  if (tid == 0) {
    misc->abort = 0;
    tc::mbar_init(&bars[B_FULL + 0], kProd / 32);
    tc::mbar_init(&bars[B_FULL + 1], kProd / 32);
    tc::mbar_init(&bars[B_EMPTY + 0], 1);
    tc::mbar_init(&bars[B_EMPTY + 1], 1);
    tc::mbar_init(&bars[B_READY + 0], kProd / 32);
    tc::mbar_init(&bars[B_READY + 1], kProd / 32);
    tc::mbar_init(&bars[B_P1DONE], 1);
    tc::mbar_init(&bars[B_PTFULL], 1);
    tc::mbar_init(&bars[B_P2DONE], 1);
    tc::mbar_init(&bars[B_OFULL + 0], 1);
    tc::mbar_init(&bars[B_OFULL + 1], 1);
    tc::mbar_init(&bars[B_OEMPTY + 0], kSoft / 32);
    tc::mbar_init(&bars[B_OEMPTY + 1], kSoft / 32);
    tc::mbar_init(&bars[B_FINAL], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) tc::tmem_alloc(&misc->tmem_base, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = misc->tmem_base;
  const int nrows = (int)blockIdx.x < a.rows ? (a.rows - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp < kProd / 32) run_producers(a, smem, nrows);
  else if (warp < kMmaWarp) run_softmax(a, smem, nrows, tbase);
  else run_mma(a, smem, nrows, tbase);

  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  if (warp == 0) tc::tmem_dealloc(tbase, 512);
}

}  // namespace

bool attend_prefill_supported(const csa_dims *d) {
  // item rows are kept as 32-bit row numbers
  return d->H == PH && d->D == PD && (int64_t)d->K + d->W <= kMaxItems &&
         (int64_t)d->B * d->entry_cap < (1ll << 31) && (int64_t)d->B * d->win_cap < (1ll << 31);
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
  if (a.rows <= 0) return CSA_OK;
  if (int rc = set_smem_once((const void *)attend_prefill_kernel, (int)P_SMEM, "attend_prefill_kernel")) return rc;
  static int sms_cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return fail(CSA_ERR_CUDA, "attend: no device");
  if (!sms_cache[dev] && cudaDeviceGetAttribute(&sms_cache[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return fail(CSA_ERR_CUDA, "attend: cannot query the SM count");
  const int sms = sms_cache[dev];
  const int grid = a.rows < sms ? a.rows : sms;
  attend_prefill_kernel<<<grid, kThreads, P_SMEM, stream>>>(a);
  count_launches(1);
  return check_launch("attend_prefill_kernel");
}

}  // namespace csa
