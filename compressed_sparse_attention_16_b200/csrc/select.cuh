// Radix selection helpers over 64-bit keys (score above, ~index below),
// shared by the indexer's selection kernels.  Included inside each file's
// own namespace.
#pragma once

#include <stdint.h>

namespace csa {
namespace sel {

constexpr int kSelBins = 4096;

// Bin (0..4095) where the count of keys in this-or-higher bins first reaches
// `need`, and the count strictly above it.  NT threads, 4096/NT bins each.
template <int NT>
__device__ __forceinline__ void find_bin(const uint32_t *hist, uint32_t need, uint32_t *warp_tot, int *out_bin,
                                         uint32_t *out_above) {
  constexpr int BPT = kSelBins / NT;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int hi_bin = kSelBins - 1 - BPT * tid;
  uint32_t c[BPT], local = 0;
  if (((uintptr_t)hist & 15u) == 0) {
    // this thread's BPT bins are contiguous and 16-byte aligned: vector loads
    // (scalar loads at a stride of BPT words would conflict on the banks)
    const uint4 *h4 = reinterpret_cast<const uint4 *>(hist + hi_bin - (BPT - 1));
#pragma unroll
    for (int k4 = 0; k4 < BPT / 4; ++k4) {
      const uint4 v = h4[k4];
      c[BPT - 1 - 4 * k4] = v.x;
      c[BPT - 2 - 4 * k4] = v.y;
      c[BPT - 3 - 4 * k4] = v.z;
      c[BPT - 4 - 4 * k4] = v.w;
    }
  } else {
#pragma unroll
    for (int k = 0; k < BPT; ++k) c[k] = hist[hi_bin - k];
  }
#pragma unroll
  for (int k = 0; k < BPT; ++k) local += c[k];
  uint32_t v = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += x;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t wv = lane < NT / 32 ? warp_tot[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, wv, o);
      if (lane >= o) wv += x;
    }
    if (lane < NT / 32) warp_tot[lane] = wv;
  }
  __syncthreads();
  const uint32_t incl = v + (warp > 0 ? warp_tot[warp - 1] : 0u);
  const uint32_t excl = incl - local;
  if (excl < need && incl >= need) {
    uint32_t run = excl;
#pragma unroll
    for (int k = 0; k < BPT; ++k) {
      if (run + c[k] >= need) { *out_bin = hi_bin - k; *out_above = run; break; }
      run += c[k];
    }
  }
  __syncthreads();
}

struct SelShared {
  uint32_t warp_tot[32];
  int bin;
  uint32_t above;
  uint32_t count;
};

// Threshold T such that exactly K of the n keys are >= T (keys distinct, K <= n):
// radix select over the key bits, 12 bits per pass, stopping as soon as the
// threshold bin is taken whole.  Narrow keys (scores below 2^24) start at
// bit 55; WIDE keys (fp32 score bits) use all 64 bits.
template <int NT, bool WIDE = false>
__device__ uint64_t kth_largest_key(const uint64_t *keys, int n, int K, uint32_t *hist, SelShared *sh) {
  uint64_t prefix = 0, pmask = 0;
  uint32_t need = (uint32_t)K;
  constexpr int ND = WIDE ? 6 : 5;
  const int shifts[6] = {WIDE ? 52 : 44, WIDE ? 40 : 32, WIDE ? 28 : 20, WIDE ? 16 : 8, WIDE ? 4 : 0, 0};
  const uint32_t dmask[6] = {0xFFFu, 0xFFFu, 0xFFFu, 0xFFFu, WIDE ? 0xFFFu : 0xFFu, 0xFu};
  for (int dgt = 0; dgt < ND; ++dgt) {
    const int sft = shifts[dgt];
    const uint32_t dm = dmask[dgt];
    for (int i = threadIdx.x; i < kSelBins; i += NT) hist[i] = 0;
    __syncthreads();
    for (int j = threadIdx.x; j < n; j += NT) {
      const uint64_t k = keys[j];
      if ((k & pmask) == prefix) atomicAdd(&hist[(uint32_t)(k >> sft) & dm], 1u);
    }
    __syncthreads();
    find_bin<NT>(hist, need, sh->warp_tot, &sh->bin, &sh->above);
    const uint32_t bin = (uint32_t)sh->bin;
    need -= sh->above;
    prefix |= (uint64_t)bin << sft;
    pmask |= (uint64_t)dm << sft;
    const uint32_t in_bin = hist[bin];
    __syncthreads();
    if (in_bin == need) break;       // the whole bin is taken: keys >= prefix
  }
  return prefix;
}

}  // namespace sel
}  // namespace csa
