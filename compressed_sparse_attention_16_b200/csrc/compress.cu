// Softmax-gated pooling of m-token blocks into FP8-E4M3 entries with a
// per-entry fp32 scale.
//
// Page: "DeepSeek V4 Flash：知っておくべき284Bパラメータのオープンソースモデル"
// (studioglobal.ai), section "アテンションのブレイクスルー：CSAとHCA" --
// softmax-gated pooling compresses the KV entries along the sequence; page
// "DeepSeek V4とOpenCode" (hazakura.dev), section "衝撃1：CSA + HCA" -- m = 4
// for CSA, m' = 128 for HCA; page "DeepSeek V4 1M context window agent
// efficient inference" (ai-papers.net), section "ハイブリッドアテンションの
// 仕組み" -- KV entries stored in FP8.
//
// The op is HBM-bound: 8 bytes read per (token, channel), 1/m byte written
// (4 bytes read when m = 1: a one-token block needs no gate logits).
// One group of D/4 threads owns one entry; each thread owns 4 channels and
// streams the block's tokens with 16-byte loads, keeping a per-channel online
// softmax (running max, normaliser and weighted sum).  The group then reduces
// the entry's amax, and every thread quantises its 4 channels and stores them
// as one 32-bit word.
#include "common.cuh"

namespace csa {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct OnlineSoftmax4 {
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
        const float r = expf(mx[c] - zs[c]);     // 0 on the first token
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

__global__ void __launch_bounds__(kThreads)
compress_kernel(const float *__restrict__ x, const float *__restrict__ z, int n_per_seq,
                int64_t n_total, int D, int m, int64_t x_bstride, uint8_t *__restrict__ codes,
                float *__restrict__ scales, int64_t dst_first, int64_t dst_bstride, int ring_cap,
                float *__restrict__ pooled) {
  __shared__ float red[kThreads / 32];
  const int L = D >> 2;                       // threads per entry
  const int groups = kThreads / L;            // entries per CTA (L divides 256 or L >= 256 handled by host)
  const int g = threadIdx.x / L;
  const int lane = threadIdx.x - g * L;
  const int64_t e = (int64_t)blockIdx.x * groups + g;
  int64_t b = 0, i = 0;
  if (g < groups && e < n_total) {
    b = e / n_per_seq;
    i = e - b * n_per_seq;
  }
  // With a ring of ring_cap slots only the call's last ring_cap blocks survive;
  // earlier blocks would share their slots, so they are not written at all.
  const bool active = (g < groups) && (e < n_total) && !(ring_cap > 0 && i + ring_cap < n_per_seq);

  float C[4] = {0.f, 0.f, 0.f, 0.f};
  if (active && m == 1) {
    // a one-token block: the softmax weight is exactly 1, so C = x and the
    // gate logits are not read at all
    const float4 v = __ldg(reinterpret_cast<const float4 *>(x + b * x_bstride + i * (int64_t)D) + lane);
    C[0] = v.x; C[1] = v.y; C[2] = v.z; C[3] = v.w;
  } else if (active) {
    const float4 *xp = reinterpret_cast<const float4 *>(x + b * x_bstride + i * (int64_t)m * D) + lane;
    const float4 *zp = reinterpret_cast<const float4 *>(z + b * x_bstride + i * (int64_t)m * D) + lane;
    OnlineSoftmax4 sm;
    sm.init();
    int j = 0;
    for (; j + kUnroll <= m; j += kUnroll) {
      float4 xv[kUnroll], zv[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        xv[u] = __ldg(xp + (int64_t)(j + u) * L);
        zv[u] = __ldg(zp + (int64_t)(j + u) * L);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) sm.push(xv[u], zv[u]);
    }
    for (; j < m; ++j) sm.push(__ldg(xp + (int64_t)j * L), __ldg(zp + (int64_t)j * L));
#pragma unroll
    for (int c = 0; c < 4; ++c) C[c] = __fdiv_rn(sm.acc[c], sm.l[c]);
  }

  // amax over the entry's L threads
  float a = fmaxf(fmaxf(fabsf(C[0]), fabsf(C[1])), fmaxf(fabsf(C[2]), fabsf(C[3])));
  const int width = L < 32 ? L : 32;
  for (int o = width >> 1; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if (L > 32) {
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) red[warp] = a;
    __syncthreads();
    const int w0 = (g * L) >> 5, nw = L >> 5;
    a = 0.f;
    for (int k = 0; k < nw; ++k) a = fmaxf(a, red[w0 + k]);
  }
  if (!active) return;

  float s = __fdiv_rn(a, 448.f);
  if (!(s > 0.f)) s = 1.f;
  uint32_t word = 0;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const float r = __fdiv_rn(C[c], s);
    const uint32_t q = __nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E4M3);
    word |= q << (8 * c);
  }
  int64_t slot = dst_first + i;
  if (ring_cap > 0) slot %= ring_cap;
  const int64_t ent = b * dst_bstride + slot;
  reinterpret_cast<uint32_t *>(codes + ent * D)[lane] = word;
  if (lane == 0) scales[ent] = s;
  if (pooled) {
    reinterpret_cast<float4 *>(pooled + (b * n_per_seq + i) * (int64_t)D)[lane] =
        make_float4(C[0], C[1], C[2], C[3]);
  }
}

// Large blocks (m >= 16): one CTA per entry; G groups of D/4 threads each run
// the online softmax over tokens g, g+G, g+2G, ... and the G partial states
// (max, normaliser, weighted sum) are merged per channel in shared memory.
__global__ void __launch_bounds__(1024)
compress_tokens_kernel(const float *__restrict__ x, const float *__restrict__ z, int n_per_seq,
                       int D, int m, int G, int64_t x_bstride, uint8_t *__restrict__ codes,
                       float *__restrict__ scales, int64_t dst_first, int64_t dst_bstride,
                       int ring_cap, float *__restrict__ pooled) {
  extern __shared__ float part[];            // [3][G][D]: max, normaliser, weighted sum
  __shared__ float red[32];
  const int L = D >> 2;
  const int g = threadIdx.x / L, lane = threadIdx.x - g * L;
  const int64_t e = blockIdx.x;
  const int64_t b = e / n_per_seq, i = e - b * n_per_seq;
  if (ring_cap > 0 && i + ring_cap < n_per_seq) return;     // overwritten later in this call
  const float4 *xp = reinterpret_cast<const float4 *>(x + b * x_bstride + i * (int64_t)m * D) + lane;
  const float4 *zp = reinterpret_cast<const float4 *>(z + b * x_bstride + i * (int64_t)m * D) + lane;
  OnlineSoftmax4 sm;
  sm.init();
  int j = g;
  for (; j + (kUnroll - 1) * G < m; j += kUnroll * G) {
    float4 xv[kUnroll], zv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      xv[u] = __ldg(xp + (int64_t)(j + u * G) * L);
      zv[u] = __ldg(zp + (int64_t)(j + u * G) * L);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) sm.push(xv[u], zv[u]);
  }
  for (; j < m; j += G) sm.push(__ldg(xp + (int64_t)j * L), __ldg(zp + (int64_t)j * L));
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    part[(0 * G + g) * D + 4 * lane + c] = sm.mx[c];
    part[(1 * G + g) * D + 4 * lane + c] = sm.l[c];
    part[(2 * G + g) * D + 4 * lane + c] = sm.acc[c];
  }
  __syncthreads();
  float C[4] = {0.f, 0.f, 0.f, 0.f};
  float a = 0.f;
  if (g == 0) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int ch = 4 * lane + c;
      float M = -INFINITY;
      for (int k = 0; k < G; ++k) M = fmaxf(M, part[(0 * G + k) * D + ch]);
      float l = 0.f, acc = 0.f;
      for (int k = 0; k < G; ++k) {
        const float mk = part[(0 * G + k) * D + ch];
        if (mk == -INFINITY) continue;                  // a group that saw no token
        const float f = expf(mk - M);
        l = fmaf(part[(1 * G + k) * D + ch], f, l);
        acc = fmaf(part[(2 * G + k) * D + ch], f, acc);
      }
      C[c] = __fdiv_rn(acc, l);
    }
    a = fmaxf(fmaxf(fabsf(C[0]), fabsf(C[1])), fmaxf(fabsf(C[2]), fabsf(C[3])));
    const unsigned gm = L < 32 ? ((1u << L) - 1u) : 0xffffffffu;   // group 0's lanes of warp 0
    for (int o = (L < 32 ? L : 32) >> 1; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(gm, a, o));
    if (L > 32 && (threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
  }
  __syncthreads();
  if (g != 0) return;
  if (L > 32) {
    a = 0.f;
    for (int k = 0; k < (L >> 5); ++k) a = fmaxf(a, red[k]);
  }
  float s = __fdiv_rn(a, 448.f);
  if (!(s > 0.f)) s = 1.f;
  uint32_t word = 0;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t q = __nv_cvt_float_to_fp8(__fdiv_rn(C[c], s), __NV_SATFINITE, __NV_E4M3);
    word |= q << (8 * c);
  }
  int64_t slot = dst_first + i;
  if (ring_cap > 0) slot %= ring_cap;
  const int64_t ent = b * dst_bstride + slot;
  reinterpret_cast<uint32_t *>(codes + ent * D)[lane] = word;
  if (lane == 0) scales[ent] = s;
  if (pooled) {
    reinterpret_cast<float4 *>(pooled + (b * n_per_seq + i) * (int64_t)D)[lane] =
        make_float4(C[0], C[1], C[2], C[3]);
  }
}

// Large blocks on many SMs (m >= 16, D a multiple of 64): the channels of
// one entry are split over a thread-block cluster of D / 64 CTAs (the
// softmax is per channel, so the CTAs pool independently); in each CTA 16
// token groups of 16 threads run the online softmax over tokens g, g + 16,
// ... for 4 channels each, and the 16 partial states are merged per channel
// in shared memory.  Only the entry's amax couples the channels: each CTA
// publishes its 64-channel amax and reads the others' through distributed
// shared memory, so every CTA derives the same scale and quantises its own
// channels.  With window outputs (wcodes, m <= 128 and a multiple of 16:
// every token is in registers), each of the block's tokens is also
// quantised on its own exactly as the one-token rule does (C = x, s = amax /
// 448, the token's amax shared the same way), so the tokens are read once.
constexpr int kClChannels = 64;                   // channels per CTA
constexpr int kClGroups = 16;                     // token groups per CTA
constexpr int kClThreads = kClGroups * (kClChannels / 4);
constexpr int kClUnroll = 8;                      // tokens per thread in one batch; window fusion needs m = 128

__device__ __forceinline__ void cl_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ float cl_load_f32(const float *p, uint32_t rank) {
  uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p)), r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(r) : "memory");
  return v;
}

__global__ void __launch_bounds__(kClThreads)
compress_cluster_kernel(const float *__restrict__ x, const float *__restrict__ z, int n_per_seq, int D, int m,
                        int64_t x_bstride, uint8_t *__restrict__ codes, float *__restrict__ scales,
                        int64_t dst_first, int64_t dst_bstride, int ring_cap, float *__restrict__ pooled,
                        int T, uint8_t *__restrict__ wcodes, float *__restrict__ wscales, int64_t w_first,
                        int64_t w_bstride, int w_ring) {
  __shared__ float part[3][kClGroups][kClChannels];   // max, normaliser, weighted sum
  __shared__ float cpool[kClChannels];
  __shared__ float tok_amax[kClGroups * 8];           // window: this CTA's 64-channel amax per token
  __shared__ float tok_scale[kClGroups * 8];
  __shared__ float wmax[kClChannels / 32];
  __shared__ float amax_cta;
  const int CG = D / kClChannels;                     // CTAs per entry (= cluster size)
  const int rank = (int)(blockIdx.x % CG);
  const int64_t e = blockIdx.x / CG;
  const int64_t b = e / n_per_seq, i = e - b * n_per_seq;
  // with a ring only the call's last ring_cap blocks survive (the whole
  // cluster leaves together, before its barriers)
  const bool win = wcodes != nullptr;                 // the host fuses only when m <= 128, m % 16 == 0
  if (!win && ring_cap > 0 && i + ring_cap < n_per_seq) return;
  const bool entry_live = !(ring_cap > 0 && i + ring_cap < n_per_seq);
  const int L = kClChannels / 4;
  const int g = threadIdx.x / L, lane = threadIdx.x - g * L;
  const int64_t col = (int64_t)rank * L + lane;       // float4 column of the row
  const float4 *xp = reinterpret_cast<const float4 *>(x + b * x_bstride + i * (int64_t)m * D) + col;
  const float4 *zp = reinterpret_cast<const float4 *>(z + b * x_bstride + i * (int64_t)m * D) + col;
  const int64_t rs = D / 4;                           // float4 per token row
  OnlineSoftmax4 sm;
  sm.init();
  // up to 8 tokens per thread in flight together (one HBM round trip for m <= 128)
  float4 keep[kClUnroll];
  int j = g;
  for (; j + (kClUnroll - 1) * kClGroups < m; j += kClUnroll * kClGroups) {
    float4 xv[kClUnroll], zv[kClUnroll];
#pragma unroll
    for (int u = 0; u < kClUnroll; ++u) {
      xv[u] = __ldg(xp + (int64_t)(j + u * kClGroups) * rs);
      zv[u] = __ldg(zp + (int64_t)(j + u * kClGroups) * rs);
    }
#pragma unroll
    for (int u = 0; u < kClUnroll; ++u) sm.push(xv[u], zv[u]);
    if (win) {
      // window (m = 128: this is the thread's only batch): each token's amax
      // over this CTA's channels (the 16 lanes of a token group are one half
      // of a warp); the tokens stay in registers for their codes below
#pragma unroll
      for (int u = 0; u < kClUnroll; ++u) {
        float t = fmaxf(fmaxf(fabsf(xv[u].x), fabsf(xv[u].y)), fmaxf(fabsf(xv[u].z), fabsf(xv[u].w)));
        for (int o = 8; o > 0; o >>= 1) t = fmaxf(t, __shfl_xor_sync(0xffffffffu, t, o));
        if (lane == 0) tok_amax[g + u * kClGroups] = t;
        keep[u] = xv[u];
      }
    }
  }
  for (; j < m; j += kClGroups) sm.push(__ldg(xp + (int64_t)j * rs), __ldg(zp + (int64_t)j * rs));
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    part[0][g][4 * lane + c] = sm.mx[c];
    part[1][g][4 * lane + c] = sm.l[c];
    part[2][g][4 * lane + c] = sm.acc[c];
  }
  __syncthreads();
  if (threadIdx.x < kClChannels) {
    const int ch = threadIdx.x;
    float M = -INFINITY;
    for (int k = 0; k < kClGroups; ++k) M = fmaxf(M, part[0][k][ch]);
    float l = 0.f, acc = 0.f;
    for (int k = 0; k < kClGroups; ++k) {
      const float mk = part[0][k][ch];
      if (mk == -INFINITY) continue;                  // a group that saw no token
      const float f = expf(mk - M);
      l = fmaf(part[1][k][ch], f, l);
      acc = fmaf(part[2][k][ch], f, acc);
    }
    const float C = __fdiv_rn(acc, l);
    cpool[ch] = C;
    float a = fabsf(C);
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((ch & 31) == 0) wmax[ch >> 5] = a;
  }
  __syncthreads();
  if (threadIdx.x == 0) amax_cta = fmaxf(wmax[0], wmax[1]);
  // every CTA's amax visible to the cluster
  cl_sync();
  float a = 0.f;
  for (int r = 0; r < CG; ++r) a = fmaxf(a, cl_load_f32(&amax_cta, (uint32_t)r));
  float s = __fdiv_rn(a, 448.f);
  if (!(s > 0.f)) s = 1.f;
  int64_t slot = dst_first + i;
  if (ring_cap > 0) slot %= ring_cap;
  const int64_t ent = b * dst_bstride + slot;
  if (threadIdx.x < L && entry_live) {
    uint32_t word = 0;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t q = __nv_cvt_float_to_fp8(__fdiv_rn(cpool[4 * threadIdx.x + c], s), __NV_SATFINITE, __NV_E4M3);
      word |= q << (8 * c);
    }
    reinterpret_cast<uint32_t *>(codes + ent * D)[rank * L + threadIdx.x] = word;
    if (pooled)
      reinterpret_cast<float4 *>(pooled + (b * n_per_seq + i) * (int64_t)D)[rank * L + threadIdx.x] =
          make_float4(cpool[4 * threadIdx.x], cpool[4 * threadIdx.x + 1], cpool[4 * threadIdx.x + 2],
                      cpool[4 * threadIdx.x + 3]);
  }
  if (rank == 0 && threadIdx.x == 0 && entry_live) scales[ent] = s;
  if (win) {
    // each token's scale from the cluster's per-token amaxima, then its codes
    if (threadIdx.x < m) {
      float ta = 0.f;
      for (int r = 0; r < CG; ++r) ta = fmaxf(ta, cl_load_f32(&tok_amax[threadIdx.x], (uint32_t)r));
      float ts = __fdiv_rn(ta, 448.f);
      if (!(ts > 0.f)) ts = 1.f;
      tok_scale[threadIdx.x] = ts;
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kClUnroll; ++u) {
      const int jt = g + u * kClGroups;               // token within the block
      const int64_t t = i * (int64_t)m + jt;          // token within the call
      if (w_ring > 0 && t + w_ring < T) continue;     // overwritten later in this call
      int64_t wslot = w_first + t;
      if (w_ring > 0) wslot %= w_ring;
      const int64_t went = b * w_bstride + wslot;
      const float ts = tok_scale[jt];
      const float xs[4] = {keep[u].x, keep[u].y, keep[u].z, keep[u].w};
      uint32_t word = 0;
#pragma unroll
      for (int c = 0; c < 4; ++c)
        word |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(xs[c], ts), __NV_SATFINITE, __NV_E4M3) << (8 * c);
      reinterpret_cast<uint32_t *>(wcodes + went * D)[rank * L + lane] = word;
      if (rank == 0 && lane == 0) wscales[went] = ts;
    }
  }
  // no CTA leaves while another may still read its amaxima
  cl_sync();
}

// Entries and window in one pass: each group of D/4 threads pools one block
// of m tokens (m = 2, 4 or 8) into an entry exactly as compress_kernel does,
// and also quantises each of the block's m tokens on its own as a window
// entry (the one-token case of the same rule: C = x, s = amax / 448).  The
// block's tokens are read once; the m + 1 amax reductions run together.
// Instantiated for m = 2, 4 and 8 (M).
constexpr int kMaxEwM = 8;

template <int M>
__global__ void __launch_bounds__(kThreads)
compress_ew_kernel(const float *__restrict__ x, const float *__restrict__ z, int n_per_seq, int64_t n_total,
                   int D, int T, int64_t x_bstride, uint8_t *__restrict__ codes, float *__restrict__ scales,
                   int64_t dst_first, int64_t dst_bstride, int ring_cap, uint8_t *__restrict__ wcodes,
                   float *__restrict__ wscales, int64_t w_first, int64_t w_bstride, int w_ring,
                   float *__restrict__ pooled) {
  constexpr int m = M;
  __shared__ float red[kThreads / 32][M + 1];
  const int L = D >> 2;
  const int groups = kThreads / L;
  const int g = threadIdx.x / L;
  const int lane = threadIdx.x - g * L;
  const int64_t e = (int64_t)blockIdx.x * groups + g;
  int64_t b = 0, i = 0;
  const bool valid = g < groups && e < n_total;
  if (valid) {
    b = e / n_per_seq;
    i = e - b * n_per_seq;
  }
  const bool write_entry = valid && !(ring_cap > 0 && i + ring_cap < n_per_seq);
  float4 xv[M];
  float C[4] = {0.f, 0.f, 0.f, 0.f};
  float v[M + 1];
#pragma unroll
  for (int u = 0; u <= M; ++u) v[u] = 0.f;
  if (valid) {
    const float4 *xp = reinterpret_cast<const float4 *>(x + b * x_bstride + i * (int64_t)m * D) + lane;
    const float4 *zp = reinterpret_cast<const float4 *>(z + b * x_bstride + i * (int64_t)m * D) + lane;
    float4 zv[M];
#pragma unroll
    for (int u = 0; u < M; ++u) {
      xv[u] = __ldg(xp + (int64_t)u * L);
      zv[u] = __ldg(zp + (int64_t)u * L);
    }
    OnlineSoftmax4 sm;
    sm.init();
#pragma unroll
    for (int u = 0; u < M; ++u) sm.push(xv[u], zv[u]);
#pragma unroll
    for (int c = 0; c < 4; ++c) C[c] = __fdiv_rn(sm.acc[c], sm.l[c]);
    v[0] = fmaxf(fmaxf(fabsf(C[0]), fabsf(C[1])), fmaxf(fabsf(C[2]), fabsf(C[3])));
#pragma unroll
    for (int u = 0; u < M; ++u)
      v[u + 1] = fmaxf(fmaxf(fabsf(xv[u].x), fabsf(xv[u].y)), fmaxf(fabsf(xv[u].z), fabsf(xv[u].w)));
  }
  // the m + 1 maxima over the group's L threads
  const int width = L < 32 ? L : 32;
#pragma unroll
  for (int u = 0; u <= M; ++u)
    for (int o = width >> 1; o > 0; o >>= 1) v[u] = fmaxf(v[u], __shfl_xor_sync(0xffffffffu, v[u], o));
  if (L > 32) {
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) {
#pragma unroll
      for (int u = 0; u <= M; ++u) red[warp][u] = v[u];
    }
    __syncthreads();
    const int w0 = (g * L) >> 5, nw = L >> 5;
#pragma unroll
    for (int u = 0; u <= M; ++u) {
      float a = 0.f;
      for (int k = 0; k < nw; ++k) a = fmaxf(a, red[w0 + k][u]);
      v[u] = a;
    }
  }
  if (!valid) return;
  auto quant = [&](const float (&c)[4], float a, uint32_t &word) {
    float s = __fdiv_rn(a, 448.f);
    if (!(s > 0.f)) s = 1.f;
    word = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t q = __nv_cvt_float_to_fp8(__fdiv_rn(c[k], s), __NV_SATFINITE, __NV_E4M3);
      word |= q << (8 * k);
    }
    return s;
  };
  if (write_entry) {
    uint32_t word;
    const float s = quant(C, v[0], word);
    int64_t slot = dst_first + i;
    if (ring_cap > 0) slot %= ring_cap;
    const int64_t ent = b * dst_bstride + slot;
    reinterpret_cast<uint32_t *>(codes + ent * D)[lane] = word;
    if (lane == 0) scales[ent] = s;
  }
  if (pooled)
    reinterpret_cast<float4 *>(pooled + (b * n_per_seq + i) * (int64_t)D)[lane] = make_float4(C[0], C[1], C[2], C[3]);
#pragma unroll
  for (int u = 0; u < M; ++u) {
    const int64_t p = i * m + u;                      // token of the call
    if (w_ring > 0 && p + w_ring < T) continue;
    const float c4[4] = {xv[u].x, xv[u].y, xv[u].z, xv[u].w};
    uint32_t word;
    const float s = quant(c4, v[u + 1], word);
    int64_t slot = w_first + p;
    if (w_ring > 0) slot %= w_ring;
    const int64_t ent = b * w_bstride + slot;
    reinterpret_cast<uint32_t *>(wcodes + ent * D)[lane] = word;
    if (lane == 0) wscales[ent] = s;
  }
}

}  // namespace

int launch_compress(const float *x, const float *z, int B, int T, int D, int m, int64_t x_bstride,
                    uint8_t *codes, float *scales, int64_t dst_first, int64_t dst_bstride,
                    int ring_cap, float *pooled, cudaStream_t stream);

int launch_compress_ew(const float *x, const float *z, int B, int T, int D, int m, int64_t x_bstride, uint8_t *codes,
                       float *scales, int64_t dst_first, int64_t dst_bstride, int ring_cap, uint8_t *wcodes,
                       float *wscales, int64_t w_first, int64_t w_bstride, int w_ring, float *pooled,
                       cudaStream_t stream) {
  const int L = D / 4;
  const int n = T / m;
  if (m == kClGroups * kClUnroll && D % kClChannels == 0 && D / kClChannels <= 8 && n > 0) {
    // large blocks: entries and window in one channel-split cluster pass
    const int CG = D / kClChannels;
    const int64_t grid = (int64_t)B * n * CG;
    if (grid > 0x7fffffffLL) return fail(CSA_ERR_UNSUPPORTED, "csa_compress_ew: too many entries");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kClThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)CG;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, compress_cluster_kernel, x, z, n, D, m, x_bstride, codes, scales,
                                             dst_first, dst_bstride, ring_cap, pooled, T, wcodes, wscales, w_first,
                                             w_bstride, w_ring);
    count_launches(1);
    if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "compress_cluster_kernel launch: %s", cudaGetErrorString(e));
    if (int rc = check_launch("compress_cluster_kernel")) return rc;
    const int tail = T - n * m;                       // tokens past the last full block: window only
    if (tail == 0) return CSA_OK;
    const int64_t off = (int64_t)n * m * D;
    return launch_compress(x + off, z + off, B, tail, D, 1, x_bstride, wcodes, wscales, w_first + (int64_t)n * m,
                           w_bstride, w_ring, nullptr, stream);
  }
  if ((m != 2 && m != 4 && m != 8) || L > kThreads || n == 0) {
    // not fused: the entries, then every token as a window entry
    if (int rc = launch_compress(x, z, B, T, D, m, x_bstride, codes, scales, dst_first, dst_bstride, ring_cap,
                                 pooled, stream))
      return rc;
    return launch_compress(x, z, B, T, D, 1, x_bstride, wcodes, wscales, w_first, w_bstride, w_ring, nullptr,
                           stream);
  }
  const int64_t total = (int64_t)B * n;
  const int groups = kThreads / L;
  const int64_t grid = (total + groups - 1) / groups;
  if (grid > 0x7fffffffLL) return fail(CSA_ERR_UNSUPPORTED, "csa_compress_ew: too many entries");
#define CSA_EW(M_)                                                                                       \
  compress_ew_kernel<M_><<<(unsigned)grid, kThreads, 0, stream>>>(x, z, n, total, D, T, x_bstride, codes, scales, \
                                                                  dst_first, dst_bstride, ring_cap, wcodes,       \
                                                                  wscales, w_first, w_bstride, w_ring, pooled)
  if (m == 2) CSA_EW(2);
  else if (m == 4) CSA_EW(4);
  else CSA_EW(8);
#undef CSA_EW
  count_launches(1);
  if (int rc = check_launch("compress_ew_kernel")) return rc;
  const int tail = T - n * m;                         // tokens past the last full block: window only
  if (tail == 0) return CSA_OK;
  // tokens [n m, T) of each sequence: the call's tokens n m .. T - 1 (the ring
  // keeps the same ones: token n m + j is skipped iff j + w_ring < tail)
  const int64_t off = (int64_t)n * m * D;
  return launch_compress(x + off, z + off, B, tail, D, 1, x_bstride, wcodes, wscales, w_first + (int64_t)n * m,
                         w_bstride, w_ring, nullptr, stream);
}

int launch_compress(const float *x, const float *z, int B, int T, int D, int m, int64_t x_bstride,
                    uint8_t *codes, float *scales, int64_t dst_first, int64_t dst_bstride,
                    int ring_cap, float *pooled, cudaStream_t stream) {
  const int n = T / m;
  const int64_t total = (int64_t)B * n;
  if (total == 0) return CSA_OK;
  const int L = D / 4;
  if (m >= 16 && D % kClChannels == 0 && D / kClChannels <= 8) {
    // channel-split clusters: D / 64 CTAs per entry
    const int CG = D / kClChannels;
    const int64_t grid = total * CG;
    if (grid > 0x7fffffffLL) return fail(CSA_ERR_UNSUPPORTED, "csa_compress: too many entries");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kClThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)CG;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, compress_cluster_kernel, x, z, n, D, m, x_bstride, codes, scales,
                                             dst_first, dst_bstride, ring_cap, pooled, T, (uint8_t *)nullptr,
                                             (float *)nullptr, (int64_t)0, (int64_t)0, 0);
    count_launches(1);
    if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "compress_cluster_kernel launch: %s", cudaGetErrorString(e));
    return check_launch("compress_cluster_kernel");
  }
  if (m >= 16 && L <= 512) {
    int G = 1024 / L;
    while (G > 1 && G * 8 > m) G >>= 1;                 // at least 8 tokens per group
    const size_t smem = (size_t)3 * G * D * sizeof(float);     // <= 3 * 1024 * 4 * 4 = 48 KiB
    if (int rc = set_smem_once((const void *)compress_tokens_kernel, 3 * 1024 * 4 * 4, "compress_tokens_kernel"))
      return rc;
    if (total <= 0x7fffffffLL) {
      compress_tokens_kernel<<<(unsigned)total, G * L, smem, stream>>>(
          x, z, n, D, m, G, x_bstride, codes, scales, dst_first, dst_bstride, ring_cap, pooled);
      count_launches(1);
      return check_launch("compress_tokens_kernel");
    }
  }
  const int groups = kThreads / L;
  const int64_t grid = (total + groups - 1) / groups;
  if (grid > 0x7fffffffLL) return fail(CSA_ERR_UNSUPPORTED, "csa_compress: too many entries");
  compress_kernel<<<(unsigned)grid, kThreads, 0, stream>>>(x, z, n, total, D, m, x_bstride, codes,
                                                           scales, dst_first, dst_bstride, ring_cap,
                                                           pooled);
  count_launches(1);
  return check_launch("compress_kernel");
}

}  // namespace csa
