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
// dimension instead.  A row's items (<= 640) are processed in tiles of 128;
// each tile is gathered and converted once and feeds both products:
//   S^T[item, head] = K_tile . Q^T      (M = 128 items, N = 64 heads, K = 512)
//   online softmax per head over the tile's items, i.e. across TMEM lanes:
//            each warp reduces its 32 lanes with a transposing butterfly, the
//            four quadrants combine in shared memory; the running maximum is
//            raised lazily (only when a tile exceeds it by more than 2^8), and
//            then O^T and the running sum are rescaled; P^T = p * entry scale
//            is written as fp16;
//   O^T[d, head] += V^T_tile . P^T      (M = 128 d per block, four blocks,
//            N = 64 heads, K = 128 items), reading the same [item][d] tile
//            MN-major; O^T for all 512 d stays in TMEM (256 columns);
//   epilogue O / l straight from TMEM to the bf16 output rows.
// The tile sits in shared memory as four 128 x 128 fp16 blocks, one slot per
// 128-wide d block; a slot is refilled with the next tile's block as soon as
// the MMAs of this tile's O^T block have read it.
//
// Roles (persistent CTAs, one per SM, query rows round-robin):
//   warps 0-7   producers: gather every 128 x 128 block of E4M3 codes through
//               registers, three blocks ahead (across rows), convert it
//               exactly to fp16 and hand it to the tensor core;
//   warps 8-11  softmax of each tile, then the row's epilogue (which overlaps
//               the first scores of the next row);
//   warp 12     issues the MMAs (one thread) and commits them to mbarriers;
//   warps 13-14 per-row set-up, up to a row ahead: compact the selection
//               into item row numbers and scales, the Q and scale maxima,
//               then Q in fp16 once the previous row's scores are complete.
// After the first tile of a row the softmax computes P^T against the running
// maximum straight away and takes the separate maximum pass only when some
// score exceeds it by more than 2^8.
// Every wait is bounded; a wait that gives up raises STATUS_TIMEOUT and turns
// every later wait of the CTA into a no-op, so all roles run to the end.
//
// fp16 operands: E4M3 -> fp16 is exact.  Q and P^T are brought into fp16's
// range by exact powers of two:
//   Q    one factor 2^kq per row puts max|q| in [2^14, 2^15): every bf16 value
//        down to 2^-31 of the row maximum converts exactly; the factor is
//        divided out of the scores in fp32;
//   P^T  exp2(x - m_h - E), with the integer E chosen from the row's largest
//        entry scale: the lazy maximum lets exp2(x - m_h) reach 2^8, and
//        E = e - 133 for a largest scale below 2^(e - 126) keeps
//        p * scale < 2^15.  The same shift divides the softmax denominator,
//        so O = sum(P^T v) / sum(p) needs no correction and the log-sum-exp
//        adds E back.
#include "common.cuh"
#include "tc.cuh"

namespace csa {
namespace {

constexpr int PH = 64;             // heads (MMA N)
constexpr int PD = 512;            // entry width
constexpr int PT = 128;            // items per tile (MMA M of the scores)
constexpr int PDB = 128;           // d per block
constexpr int kNdb = PD / PDB;     // d blocks (= ring slots)
constexpr int kMaxTiles = 5;       // <= 640 items per row
constexpr int kMaxItems = kMaxTiles * PT;
constexpr int kProd = 256;         // producer threads (warps 0-7)
constexpr int kSoft = 128;         // softmax / epilogue threads (warps 8-11)
constexpr int kSetup = 64;         // set-up threads (warps 13-14)
constexpr int kMmaWarp = (kProd + kSoft) / 32;
constexpr int kSetupWarp0 = kMmaWarp + 1;
constexpr int kThreads = kProd + kSoft + 32 + kSetup;
constexpr float kPLog2e = 1.4426950408889634f;
constexpr float kPRescaleLog2 = 8.f;
constexpr unsigned long long kPWaitNs = 2000000000ull;
constexpr uint32_t kSCol = 0;      // S^T: TMEM columns [0, 64)
constexpr uint32_t kOCol = PH;     // O^T: four blocks of 64 columns, [64, 320)

// shared memory map (bytes)
constexpr uint32_t S_Q = 0;                                  // fp16 [64 h][512 d]          64 KiB
constexpr uint32_t S_PT = S_Q + PH * PD * 2;                 // fp16 [128 i][64 h]          16 KiB
constexpr uint32_t S_KV = S_PT + PT * PH * 2;                // fp16 4 x [128 i][128 d]    128 KiB
constexpr uint32_t KV_BYTES = PT * PDB * 2;
constexpr uint32_t S_ITEM = S_KV + kNdb * KV_BYTES;          // int32 [2][640] item rows
constexpr uint32_t S_SCALE = S_ITEM + 2 * kMaxItems * 4;     // fp32 [2][640] item scales
constexpr uint32_t S_INFO = S_SCALE + 2 * kMaxItems * 4;     // RowInfo [2]
constexpr uint32_t S_RED = S_INFO + 2 * 32;                  // fp32: max [4][64], sum [4][64], M, L, Ms, invL, fac [64]
constexpr uint32_t S_PRED = S_RED + 13 * PH * 4;             // set-up reductions, u32 [16]
constexpr uint32_t S_FLAG = S_PRED + 16 * 4;                 // int [2] rescale, int [2] slow path
constexpr uint32_t S_BAR = S_FLAG + 16;
constexpr int kNumBars = 20;
constexpr uint32_t S_MISC = S_BAR + kNumBars * 8;
constexpr uint32_t P_SMEM = S_MISC + 32;
static_assert(P_SMEM <= 232448, "shared memory");
static_assert(S_KV % 1024 == 0 && S_PT % 1024 == 0, "tile alignment");

// mbarriers
enum : int {
  B_FULL = 0,      // [4] producers -> MMA: d-block slot converted (one arrival per warp)
  B_EMPTY = 4,     // [4] MMA -> producers: d-block slot read by the tile's last MMA (commit)
  B_READY = 8,     // [2] set-up -> softmax, MMA: RowInfo and Q in place, by row parity (one per warp)
  B_ITEMS = 10,    // [2] set-up -> producers: item rows in place, by row parity (one per warp)
  B_FREE = 12,     // [2] producers (one per warp) + softmax (one) -> set-up: the row's item
                   //     rows and scales are no longer read
  B_QFREE = 14,    // MMA -> set-up: the row's last scores complete, Q no longer read (commit)
  B_SFULL = 15,    // MMA -> softmax: S^T of a tile complete (commit)
  B_PFULL = 16,    // softmax -> MMA: P^T written, S^T read, O^T rescaled (1 arrival)
  B_OFULL = 17,    // MMA -> epilogue: the row's O^T complete (commit)
  B_OEMPTY = 18,   // epilogue -> MMA: O^T read (one arrival per warp)
  B_FINAL = 19,    // all MMAs complete (commit)
};

// Q  [64 h][512 d]:   d-group stride 1024, head-group stride 128
// KV [128 i][128 d]:  d-group stride 2048, item-group stride 128
// PT [128 i][64 h]:   item-group stride 1024, head-group stride 128
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

// Four E4M3 codes (byte i of w is code i) -> four fp16, codes 0-1 in `lo`
// and 2-3 in `hi`, the lower code in the lower half (exact: every finite
// E4M3 value is an fp16).  One PTX cvt per pair of codes.
__device__ __forceinline__ void e4m3x4_to_h2x2(uint32_t w, uint32_t &lo, uint32_t &hi) {
  asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// 16 E4M3 codes -> 16 fp16, codes 0-7 in `lo` and 8-15 in `hi`
__device__ __forceinline__ void cvt16(const uint4 &c, uint4 &lo, uint4 &hi) {
  e4m3x4_to_h2x2(c.x, lo.x, lo.y);
  e4m3x4_to_h2x2(c.y, lo.z, lo.w);
  e4m3x4_to_h2x2(c.z, hi.x, hi.y);
  e4m3x4_to_h2x2(c.w, hi.z, hi.w);
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

// ------------------------------------------------------------------- set-up
// Row it uses the item, scale and RowInfo buffers of parity it & 1; they are
// rewritten for row it + 2 once the producers have gathered row it's last
// block and the softmax has used row it's last scales (B_FREE).
__device__ __forceinline__ void run_setup(const PArgs &a, unsigned char *smem, int nrows) {
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S_BAR);
  PMisc *misc = reinterpret_cast<PMisc *>(smem + S_MISC);
  RowInfo *info = reinterpret_cast<RowInfo *>(smem + S_INFO);
  uint32_t *pred = reinterpret_cast<uint32_t *>(smem + S_PRED);
  const int st = threadIdx.x - kSetupWarp0 * 32, sw = st >> 5, lane = threadIdx.x & 31;
  const float qs = a.sm_scale * kPLog2e;

  for (int it = 0; it < nrows; ++it) {
    const int row = blockIdx.x + it * gridDim.x;
    const int par = it & 1;
    if (it >= 2) pwait(&bars[B_FREE + par], ((it >> 1) - 1) & 1, misc, a.status);
    int *irow = reinterpret_cast<int *>(smem + S_ITEM) + par * kMaxItems;
    float *isc = reinterpret_cast<float *>(smem + S_SCALE) + par * kMaxItems;
    const int b = row / a.Tq;
    int64_t t = a.q_pos[row];
    if (t < 0) {
      if (st == 0) raise_status(a.status, STATUS_BAD_POSITION);
      t = 0;
    }
    const int nwin = (int)min((int64_t)a.W, t + 1);
    const int64_t p0 = t - nwin + 1;
    // ordered compaction of the valid selected entries into item rows:
    // r >= 0 is row r of the entry cache, r < 0 row -r-1 of the window ring.
    // The indices are read eight per thread up front, so that their loads
    // (and the scale loads they lead to) overlap.
    const int32_t *idx = a.idx + (int64_t)row * a.K;
    constexpr int kPer = 8;
    int nsel = 0;
    for (int j0 = 0; j0 < a.K; j0 += kSetup * kPer) {
      int e[kPer];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int j = j0 + k * kSetup + st;
        e[k] = (j < a.K) ? idx[j] : -1;
      }
      float sv[kPer];
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        if (e[k] >= a.n_entries || e[k] < -1) { raise_status(a.status, STATUS_BAD_INDEX); e[k] = -1; }
        sv[k] = e[k] >= 0 ? a.scales[(int64_t)b * a.entry_cap + e[k]] : 0.f;
      }
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const bool f = e[k] >= 0;
        const unsigned bal = __ballot_sync(0xffffffffu, f);
        if (lane == 0) pred[2 * k + sw] = __popc(bal);
      }
      named_sync(3, kSetup);
      int base = nsel;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const bool f = e[k] >= 0;
        const unsigned bal = __ballot_sync(0xffffffffu, f);
        const int c0 = (int)pred[2 * k], c1 = (int)pred[2 * k + 1];
        if (f) {
          const int u = base + (sw ? c0 : 0) + __popc(bal & ((1u << lane) - 1u));
          irow[u] = (int)((int64_t)b * a.entry_cap + e[k]);
          isc[u] = sv[k];
        }
        base += c0 + c1;
      }
      nsel = base;
      named_sync(3, kSetup);
    }
    const int n_items = min(nsel + nwin, kMaxItems);
    for (int u = nsel + st; u < n_items; u += kSetup) {
      const int64_t r = (int64_t)b * a.win_cap + (p0 + (u - nsel)) % a.win_cap;
      irow[u] = (int)(-r - 1);
      isc[u] = a.wscales[r];
    }
    const int ntiles = (n_items + PT - 1) / PT;
    named_sync(3, kSetup);
    // the producers may gather this row now
    __syncwarp();
    if (lane == 0) {
      if (sw == 0) {
        info[par].n_items = n_items;
        info[par].ntiles = ntiles;
      }
    }
    named_sync(3, kSetup);
    if (lane == 0) tc::mbar_arrive(&bars[B_ITEMS + par]);

    // Q row max (thread st holds head st) and the largest scale
    const uint4 *qg = reinterpret_cast<const uint4 *>(a.q + (int64_t)row * PH * PD) + st * (PD / 8);
    uint32_t mq = 0;
#pragma unroll 16
    for (int k = 0; k < PD / 8; ++k) {
      const uint4 v = __ldg(qg + k);
      mq = __vmaxu2(mq, __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                 __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
    }
    float smax = 0.f;
    for (int u = st; u < n_items; u += kSetup) smax = fmaxf(smax, isc[u]);
    mq = __reduce_max_sync(0xffffffffu, max(mq & 0xFFFFu, mq >> 16));
    const uint32_t sbits = __reduce_max_sync(0xffffffffu, __float_as_uint(smax));   // smax >= 0
    if (lane == 0) { pred[sw] = mq; pred[8 + sw] = sbits; }
    named_sync(3, kSetup);
    const uint32_t amax = max(pred[0], pred[1]), smb = max(pred[8], pred[9]);
    // bf16 |q| max in [2^(eb-127), 2^(eb-126)) -> times 2^(141-eb) in [2^14, 2^15)
    const int kq = amax ? min(126, 141 - (int)((amax >> 7) & 0xFFu)) : 0;
    const float fq = __int_as_float((kq + 127) << 23);
    if (st == 0) {
      RowInfo &ri = info[par];
      ri.row = row;
      ri.pad0 = 0;
      ri.qscale = qs * __int_as_float((127 - kq) << 23);
      // largest scale < 2^(e - 126) for biased exponent e; p <= 2^8 under the
      // lazy maximum, so p * scale * 2^-E < 2^15 with E = e - 133
      const int e = (int)((smb >> 23) & 0xFFu);
      ri.eshift = (float)min(112, max(-110, e - 133));
      ri.pad1[0] = ri.pad1[1] = 0.f;
    }
    // Q in fp16, 16 chunks of 8 per batch (the first batch is loaded before
    // the wait): the buffer is free once the previous row's last scores are
    // complete
    unsigned char *qs_ = smem + S_Q;
    constexpr int kQb = 16;
    uint4 qv[kQb];
#pragma unroll
    for (int k = 0; k < kQb; ++k) qv[k] = __ldg(qg + k);
    if (it > 0) pwait(&bars[B_QFREE], (it - 1) & 1, misc, a.status);
#pragma unroll 1
    for (int k0 = 0; k0 < PD / 8; k0 += kQb) {
#pragma unroll
      for (int k = 0; k < kQb; ++k) {
        const uint4 v = qv[k];
        *reinterpret_cast<uint4 *>(qs_ + pq_off(st, k0 + k)) =
            make_uint4(bf2_to_h2(v.x, fq), bf2_to_h2(v.y, fq), bf2_to_h2(v.z, fq), bf2_to_h2(v.w, fq));
      }
      if (k0 + kQb < PD / 8) {
#pragma unroll
        for (int k = 0; k < kQb; ++k) qv[k] = __ldg(qg + k0 + kQb + k);
      }
    }
    tc::fence_proxy_async_smem();
    // pred is reused by the next row
    named_sync(3, kSetup);
    if (lane == 0) tc::mbar_arrive(&bars[B_READY + par]);
  }
}

// ------------------------------------------------------------------ producers
// The producers walk one stream of blocks over all rows of the CTA.  Row it
// has 4 * ntiles blocks: block j is tile j / 4, d block j % 4, and goes to
// ring slot j % 4.  Blocks are gathered into registers three ahead of the one
// being converted, across row boundaries.
__device__ __forceinline__ void run_producers(const PArgs &a, unsigned char *smem, int nrows) {
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S_BAR);
  PMisc *misc = reinterpret_cast<PMisc *>(smem + S_MISC);
  const RowInfo *info = reinterpret_cast<const RowInfo *>(smem + S_INFO);
  const int tid = threadIdx.x, pw = tid >> 5, lane = tid & 31;
  const int i8 = lane & 7, cq = lane >> 3;
  int ni0 = 0, ni1 = 0, nt0 = 0, nt1 = 0;   // n_items / ntiles of the rows of parity 0 / 1

  auto row_items = [&](int it) {
    const int par = it & 1;
    pwait(&bars[B_ITEMS + par], (it >> 1) & 1, misc, a.status);
    const int n = info[par].n_items, t = info[par].ntiles;
    if (par) { ni1 = n; nt1 = t; } else { ni0 = n; nt0 = t; }
  };

  // ---- block gather: thread (pw, lane) holds items (2 pw + (k & 1)) * 8 +
  // (lane & 7) of the tile, 16-byte chunks (k >> 1) * 4 + (lane >> 3) of the
  // d block, k = 0..3.  Items past n_items read item 0 (always valid): their
  // scores are masked and their P^T rows are zero.
  auto load_blk = [&](int it, int j, uint4 (&v)[4]) {
    const int tile = j >> 2, dblk = j & 3;
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
  uint32_t nblk = 0;   // blocks handed over so far (ring slot = nblk & 3 = d block)
  auto produce = [&](const uint4 (&v)[4]) {
    const uint32_t slot = nblk & 3u, use = nblk >> 2;
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
  auto nbt_of = [&](int it) { return ((it & 1) ? nt1 : nt0) * kNdb; };

  if (nrows <= 0) return;
  int p_it = 0, p_j = 0;   // next block to hand over
  int l_it = 0, l_j = 0;   // next block to gather
  auto gather = [&](uint4 (&v)[4]) {
    if (l_it < nrows) {
      if (l_j == 0) row_items(l_it);
      load_blk(l_it, l_j, v);
      if (++l_j == nbt_of(l_it)) {
        // this row's item rows are no longer read by the producers
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars[B_FREE + (l_it & 1)]);
        ++l_it;
        l_j = 0;
      }
    }
  };
  auto step = [&](uint4 (&v)[4]) {
    if (p_it < nrows) {
      produce(v);
      if (++p_j == nbt_of(p_it)) { ++p_it; p_j = 0; }
    }
    gather(v);
  };
  uint4 A[4], B[4], C[4];
  gather(A);
  gather(B);
  gather(C);
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
  float *redm = reinterpret_cast<float *>(smem + S_RED);   // [4][64] tile maxima per quadrant
  float *reds = redm + 4 * PH;                              // [4][64] tile sums per quadrant
  float *Mh = reds + 4 * PH;                                // running maximum
  float *Lh = Mh + PH;                                      // running sum
  float *Ms = Lh + PH;                                      // running maximum + E
  float *invL = Ms + PH;
  float *fac = invL + PH;                                   // rescale factor of this tile
  int *flag = reinterpret_cast<int *>(smem + S_FLAG);       // [2] rescale O^T
  int *slow = flag + 2;                                     // [2] the running maximum is too low
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int sq = warp - kProd / 32;        // TMEM lane quadrant
  const int stid = tid - kProd;
  const uint32_t lane_off = (uint32_t)(sq * 32) << 16;
  uint32_t ntile = 0;                      // tiles processed by this CTA

  for (int it = 0; it < nrows; ++it) {
    const int par = it & 1;
    pwait(&bars[B_READY + par], (it >> 1) & 1, misc, a.status);
    const RowInfo ri = info[par];
    const float *isc = reinterpret_cast<const float *>(smem + S_SCALE) + par * kMaxItems;
    // exp2(x - m) <= 2^8 <=> (x - m - E) <= 8 - E
    const float thr = kPRescaleLog2 - ri.eshift;
    if (stid < PH) { Mh[stid] = -INFINITY; Lh[stid] = 0.f; }

    for (int tl = 0; tl < ri.ntiles; ++tl, ++ntile) {
      pwait(&bars[B_SFULL], ntile & 1, misc, a.status);
      tc::fence_after_sync();
      const int u = tl * PT + sq * 32 + lane;
      const bool valid = u < ri.n_items;
      const float sc = valid ? isc[u] : 0.f;
      const float f = sc * ri.qscale;

      // P^T = exp2(x - m - E) * scale and the tile's sums of exp2(x - m - E);
      // with `detect`, report any item whose exp2(x - m) would exceed 2^8
      auto p_phase = [&](bool detect) {
        bool over = false;
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t r[32];
          tc::tmem_ld32(tbase + lane_off + kSCol + hh * 32, r);
          tc::tmem_wait_ld();
          float sm[32];
          uint32_t pk[16];
#pragma unroll
          for (int j = 0; j < 32; j += 2) {
            const float2 mm = *reinterpret_cast<const float2 *>(Ms + hh * 32 + j);
            const float da = valid ? __uint_as_float(r[j]) * f - mm.x : -INFINITY;
            const float db = valid ? __uint_as_float(r[j + 1]) * f - mm.y : -INFINITY;
            over |= (da > thr) | (db > thr);
            const float pa = ex2(da), pb = ex2(db);
            sm[j] = pa;
            sm[j + 1] = pb;
            const __half2 v = __floats2half2_rn(pa * sc, pb * sc);
            pk[j >> 1] = *reinterpret_cast<const uint32_t *>(&v);
          }
          const int ul = sq * 32 + lane;
#pragma unroll
          for (int hg = 0; hg < 4; ++hg)
            *reinterpret_cast<uint4 *>(smem + S_PT + ppt_off(ul, hh * 4 + hg)) =
                make_uint4(pk[4 * hg], pk[4 * hg + 1], pk[4 * hg + 2], pk[4 * hg + 3]);
          reds[sq * PH + hh * 32 + lane] = warp_transpose_reduce<false>(sm);
        }
        if (detect && over) slow[ntile & 1] = 1;
      };

      bool need_max = tl == 0;
      if (!need_max) {
        p_phase(true);
        named_sync(2, kSoft);
        need_max = slow[ntile & 1] != 0;
        // the next tile's flags (last read before this barrier) start clear
        if (stid == 0) { slow[(ntile + 1) & 1] = 0; flag[(ntile + 1) & 1] = 0; }
      }
      if (need_max) {
        // tile maximum of x = score * scale * log2(e), per head
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t r[32];
          tc::tmem_ld32(tbase + lane_off + kSCol + hh * 32, r);
          tc::tmem_wait_ld();
          float mx[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) mx[j] = valid ? __uint_as_float(r[j]) * f : -INFINITY;
          redm[sq * PH + hh * 32 + lane] = warp_transpose_reduce<true>(mx);
        }
        named_sync(2, kSoft);
        if (stid == 0) { slow[(ntile + 1) & 1] = 0; flag[(ntile + 1) & 1] = 0; }
        if (stid < PH) {
          const float mt = fmaxf(fmaxf(redm[stid], redm[PH + stid]), fmaxf(redm[2 * PH + stid], redm[3 * PH + stid]));
          const float mo = Mh[stid];
          float fc = 1.f;
          if (mt > mo + kPRescaleLog2) {
            fc = mo == -INFINITY ? 0.f : ex2(mo - mt);
            Lh[stid] *= fc;
            Mh[stid] = mt;
            if (tl > 0) flag[ntile & 1] = 1;
          }
          fac[stid] = fc;
          Ms[stid] = Mh[stid] + ri.eshift;
        }
        named_sync(2, kSoft);
        if (flag[ntile & 1]) {
          // O^T holds the row's earlier tiles (their MMAs completed before this
          // tile's scores): scale head column h of every d block by fac[h]
#pragma unroll 1
          for (int c = 0; c < kNdb * 2; ++c) {
            uint32_t o[32];
            tc::tmem_ld32(tbase + lane_off + kOCol + c * 32, o);
            tc::tmem_wait_ld();
            const float *fcp = fac + (c & 1) * 32;
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * fcp[j]);
            tc::tmem_st32(tbase + lane_off + kOCol + c * 32, o);
          }
          tc::tmem_wait_st();
        }
        p_phase(false);
      }
      tc::fence_proxy_async_smem();
      tc::fence_before_sync();
      named_sync(2, kSoft);
      if (stid == 0) {
        tc::mbar_arrive(&bars[B_PFULL]);
        // the row's scales are no longer read
        if (tl == ri.ntiles - 1) tc::mbar_arrive(&bars[B_FREE + par]);
      }
      if (stid < PH) Lh[stid] += (reds[stid] + reds[PH + stid]) + (reds[2 * PH + stid] + reds[3 * PH + stid]);
    }

    // epilogue: O^T block dblk, lanes = d, columns = heads
    pwait(&bars[B_OFULL], it & 1, misc, a.status);
    tc::fence_after_sync();
    named_sync(2, kSoft);
    if (stid < PH) {
      const float L = Lh[stid];
      invL[stid] = 1.f / L;
      if (a.lse) a.lse[(int64_t)ri.row * PH + stid] = (Mh[stid] + ri.eshift + log2f(L)) * 0.6931471805599453f;
    }
    named_sync(2, kSoft);
    __nv_bfloat16 *orow = a.out + (int64_t)ri.row * PH * PD;
#pragma unroll 1
    for (int dblk = 0; dblk < kNdb; ++dblk) {
      uint32_t r0[32], r1[32];
      tc::tmem_ld32(tbase + lane_off + kOCol + dblk * PH, r0);
      tc::tmem_ld32(tbase + lane_off + kOCol + dblk * PH + 32, r1);
      tc::tmem_wait_ld();
      if (dblk == kNdb - 1) {
        tc::fence_before_sync();
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&bars[B_OEMPTY]);
      }
      __nv_bfloat16 *o = orow + dblk * PDB + sq * 32 + lane;
#pragma unroll
      for (int j = 0; j < 32; ++j) o[j * PD] = __float2bfloat16_rn(__uint_as_float(r0[j]) * invL[j]);
#pragma unroll
      for (int j = 0; j < 32; ++j) o[(32 + j) * PD] = __float2bfloat16_rn(__uint_as_float(r1[j]) * invL[32 + j]);
    }
    // invL, Mh and Lh are reset or rewritten only after every thread is done
    named_sync(2, kSoft);
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
  uint32_t ntile = 0;

  for (int it = 0; it < nrows; ++it) {
    const int par = it & 1;
    pwait(&bars[B_READY + par], (it >> 1) & 1, misc, a.status);
    const int ntiles = info[par].ntiles;
    for (int tl = 0; tl < ntiles; ++tl, ++ntile) {
      // S^T = K_tile . Q^T, one d block per ring slot
      for (int dblk = 0; dblk < kNdb; ++dblk) {
        pwait(&bars[B_FULL + dblk], ntile & 1, misc, a.status);
        tc::fence_after_sync();
        if (leader) {
          const uint32_t kvb = sbase + S_KV + dblk * KV_BYTES;
#pragma unroll
          for (int k = 0; k < PDB / 16; ++k) {
            // A = K tile (M = items, K = d), K-major: LBO = d-group step, SBO = item-group step
            const uint64_t ad = tc::smem_desc(kvb + k * 4096, 2048, 128);
            // B = Q (N = heads, K = d), K-major: LBO = d-group step, SBO = head-group step
            const uint64_t bd = tc::smem_desc(sbase + S_Q + (dblk * 16 + 2 * k) * 1024, 1024, 128);
            tc::mma_bf16_ss(tbase + kSCol, ad, bd, idesc_qk, (dblk > 0 || k > 0));
          }
        }
        __syncwarp();
      }
      if (leader) {
        tc::mma_commit(&bars[B_SFULL]);
        if (tl == ntiles - 1) tc::mma_commit(&bars[B_QFREE]);
      }
      __syncwarp();
      // the previous row's epilogue has read O^T before its first tile overwrites it
      if (tl == 0 && it > 0) pwait(&bars[B_OEMPTY], (it - 1) & 1, misc, a.status);
      pwait(&bars[B_PFULL], ntile & 1, misc, a.status);
      tc::fence_after_sync();
      // O^T[dblk] += V^T_tile[dblk] . P^T; the slot is free after these MMAs
      if (leader) {
        for (int dblk = 0; dblk < kNdb; ++dblk) {
          const uint32_t kvb = sbase + S_KV + dblk * KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < PT / 16; ++kk) {
            // A = V^T (M = d, K = items), MN-major: LBO = item-group step, SBO = d-group step
            const uint64_t ad = tc::smem_desc(kvb + kk * 256, 128, 2048);
            // B = P^T (N = heads, K = items), MN-major: LBO = item-group step, SBO = head-group step
            const uint64_t bd = tc::smem_desc(sbase + S_PT + (2 * kk) * 1024, 1024, 128);
            tc::mma_bf16_ss(tbase + kOCol + dblk * PH, ad, bd, idesc_pv, (tl > 0 || kk > 0));
          }
          tc::mma_commit(&bars[B_EMPTY + dblk]);
        }
      }
      __syncwarp();
    }
    if (leader) tc::mma_commit(&bars[B_OFULL]);
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
    for (int s = 0; s < kNdb; ++s) {
      tc::mbar_init(&bars[B_FULL + s], kProd / 32);
      tc::mbar_init(&bars[B_EMPTY + s], 1);
    }
    for (int p = 0; p < 2; ++p) {
      tc::mbar_init(&bars[B_READY + p], kSetup / 32);
      tc::mbar_init(&bars[B_ITEMS + p], kSetup / 32);
      tc::mbar_init(&bars[B_FREE + p], kProd / 32 + 1);
    }
    tc::mbar_init(&bars[B_QFREE], 1);
    tc::mbar_init(&bars[B_SFULL], 1);
    tc::mbar_init(&bars[B_PFULL], 1);
    tc::mbar_init(&bars[B_OFULL], 1);
    tc::mbar_init(&bars[B_OEMPTY], kSoft / 32);
    tc::mbar_init(&bars[B_FINAL], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (tid < 4) reinterpret_cast<int *>(smem + S_FLAG)[tid] = 0;
  if (warp == 0) tc::tmem_alloc(&misc->tmem_base, 512);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = misc->tmem_base;
  const int nrows = (int)blockIdx.x < a.rows ? (a.rows - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp < kProd / 32) run_producers(a, smem, nrows);
  else if (warp < kMmaWarp) run_softmax(a, smem, nrows, tbase);
  else if (warp == kMmaWarp) run_mma(a, smem, nrows, tbase);
  else run_setup(a, smem, nrows);

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
