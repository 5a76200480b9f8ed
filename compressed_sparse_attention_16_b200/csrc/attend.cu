// Shared-KV multi-query attention over (selected compressed entries) plus
// (sliding-window tokens), one joint softmax -- the generic CUDA-core kernel.
//
// Page: jiwasawa.github.io DeepSeek-V4 article, section "Compressed Sparse
// Attention (CSA)" -- MQA with shared key-value over the k selected entries;
// section "Heavily Compressed Attention (HCA)" -- dense attention over the
// compressed sequence, plus a sliding-window branch over recent uncompressed
// tokens; page "DeepSeek V4 Flash" (studioglobal.ai), section
// "アテンションのブレイクスルー" -- the window always covers the latest 128
// tokens.
//
// One CTA serves one query row and a group of heads (one warp per head).  The
// row's key/value items (valid selected entries, or every visible entry for
// HCA, then the window tokens) are gathered in chunks of 32: their E4M3 codes
// are converted exactly to fp32 in shared memory, each lane owns D/32
// channels, QK dot products are reduced across the warp by a transposing
// butterfly (lane j ends with item j's logit), and an online softmax folds
// every chunk into the fp32 output accumulators.  The entry scale multiplies
// the logit and the probability, never the codes.
#include "common.cuh"

namespace csa {
namespace {

constexpr int kChunk = 32;
constexpr int kMaxSel = 2048;
constexpr float kLog2e = 1.4426950408889634f;

template <int D>
__global__ void __launch_bounds__(256)
attend_generic_kernel(const __nv_bfloat16 *__restrict__ q, const uint8_t *__restrict__ codes,
                      const float *__restrict__ scales, const int32_t *__restrict__ idx,
                      const uint8_t *__restrict__ wcodes, const float *__restrict__ wscales,
                      const int32_t *__restrict__ q_pos, int Tq, int H, int K, int W, int m,
                      int n_entries, int64_t entry_cap, int win_cap, float sm_scale,
                      __nv_bfloat16 *__restrict__ out, float *__restrict__ lse, unsigned *status) {
  constexpr int EPL = D / 32;            // channels per lane
  static_assert(D % 64 == 0, "D must be a multiple of 64");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  float *vs = reinterpret_cast<float *>(smem_raw);                  // [kChunk][D]
  float *ps = vs + kChunk * D;                                       // [warps][kChunk]
  const uint8_t **iptr = reinterpret_cast<const uint8_t **>(ps + 8 * kChunk);   // [kChunk]
  float *iscale = reinterpret_cast<float *>(iptr + kChunk);         // [kChunk]
  int *sel = reinterpret_cast<int *>(iscale + kChunk);              // [kMaxSel]
  __shared__ int s_nsel;
  __shared__ int s_wcount[8];

  const int warps = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.y;
  const int b = row / Tq;
  const int h = blockIdx.x * warps + warp;
  int64_t t = q_pos[row];
  if (t < 0) {
    if (threadIdx.x == 0) raise_status(status, STATUS_BAD_POSITION);
    t = 0;
  }
  const int nvis = (int)min((t + 1) / m, (int64_t)n_entries);
  const int nwin = (int)min((int64_t)W, t + 1);

  // compact list of valid selected entries (ordered), or the dense count
  int nsel;
  if (idx) {
    const int32_t *irow = idx + (int64_t)row * K;
    if (threadIdx.x == 0) s_nsel = 0;
    __syncthreads();
    int base = 0;
    for (int j0 = 0; j0 < K; j0 += blockDim.x) {
      const int j = j0 + threadIdx.x;
      int e = (j < K) ? irow[j] : -1;
      if (e >= n_entries || e < -1) { raise_status(status, STATUS_BAD_INDEX); e = -1; }
      const bool f = e >= 0;
      const unsigned bal = __ballot_sync(0xffffffffu, f);
      if (lane == 0) s_wcount[warp] = __popc(bal);
      __syncthreads();
      int before = 0, tot = 0;
      for (int k = 0; k < warps; ++k) { if (k < warp) before += s_wcount[k]; tot += s_wcount[k]; }
      if (f) sel[base + before + __popc(bal & ((1u << lane) - 1u))] = e;
      base += tot;
      __syncthreads();
    }
    nsel = base;
  } else {
    nsel = nvis;
  }
  const int n_items = nsel + nwin;
  const int64_t p0 = t - nwin + 1;       // first window position

  // this lane's query channels: c = lane*2 + 64*k + {0,1}
  float qv[EPL];
  const float qscale = sm_scale * kLog2e;
  const __nv_bfloat16 *qrow = q + ((int64_t)row * H + (h < H ? h : 0)) * D;
#pragma unroll
  for (int k = 0; k < EPL / 2; ++k) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(qrow + lane * 2 + 64 * k));
    qv[2 * k] = f.x * qscale;
    qv[2 * k + 1] = f.y * qscale;
  }
  float o[EPL];
#pragma unroll
  for (int k = 0; k < EPL; ++k) o[k] = 0.f;
  float mrun = -INFINITY, lrun = 0.f;

  for (int c0 = 0; c0 < n_items; c0 += kChunk) {
    const int nc = min(kChunk, n_items - c0);
    __syncthreads();
    if (threadIdx.x < nc) {
      const int u = c0 + threadIdx.x;
      if (u < nsel) {
        const int e = idx ? sel[u] : u;
        const int64_t ent = (int64_t)b * entry_cap + e;
        iptr[threadIdx.x] = codes + ent * D;
        iscale[threadIdx.x] = scales[ent];
      } else {
        const int64_t p = p0 + (u - nsel);
        const int64_t ent = (int64_t)b * win_cap + (p % win_cap);
        iptr[threadIdx.x] = wcodes + ent * D;
        iscale[threadIdx.x] = wscales[ent];
      }
    }
    __syncthreads();
    // gather + exact E4M3 -> fp32, 16 bytes per thread per step
    constexpr int V16 = D / 16;
    for (int i = threadIdx.x; i < nc * V16; i += blockDim.x) {
      const int item = i / V16, part = i - item * V16;
      const uint4 c = __ldg(reinterpret_cast<const uint4 *>(iptr[item]) + part);
      float *dst = vs + item * D + part * 16;
      const uint32_t wv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 a = e4m3x2_to_float2((uint16_t)(wv[k] & 0xFFFF));
        const float2 bb = e4m3x2_to_float2((uint16_t)(wv[k] >> 16));
        *reinterpret_cast<float4 *>(dst + 4 * k) = make_float4(a.x, a.y, bb.x, bb.y);
      }
    }
    __syncthreads();
    if (h < H) {
      // partial dot products for all chunk items
      float acc[kChunk];
#pragma unroll
      for (int j = 0; j < kChunk; ++j) {
        float a = 0.f;
        if (j < nc) {
          const float *v = vs + j * D + lane * 2;
#pragma unroll
          for (int k = 0; k < EPL / 2; ++k) {
            const float2 vv = *reinterpret_cast<const float2 *>(v + 64 * k);
            a = fmaf(qv[2 * k], vv.x, a);
            a = fmaf(qv[2 * k + 1], vv.y, a);
          }
        }
        acc[j] = a;
      }
      // transposing butterfly: lane l ends with the full sum of item l
#pragma unroll
      for (int s = 16; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < s; ++i) {
          const float send = upper ? acc[i] : acc[i + s];
          const float keep = upper ? acc[i + s] : acc[i];
          acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
      }
      const float sl = (lane < nc) ? acc[0] * iscale[lane] : -INFINITY;   // log2-domain logit
      const float mnew = fmaxf(mrun, warp_max(sl));
      const float p = (lane < nc) ? exp2f(sl - mnew) : 0.f;
      const float alpha = exp2f(mrun - mnew);                            // 0 on the first chunk
      lrun = lrun * alpha + warp_sum(p);
      mrun = mnew;
      ps[warp * kChunk + lane] = p * ((lane < nc) ? iscale[lane] : 0.f);
      __syncwarp();
#pragma unroll
      for (int k = 0; k < EPL; ++k) o[k] *= alpha;
      for (int j = 0; j < nc; ++j) {
        const float pj = ps[warp * kChunk + j];
        const float *v = vs + j * D + lane * 2;
#pragma unroll
        for (int k = 0; k < EPL / 2; ++k) {
          const float2 vv = *reinterpret_cast<const float2 *>(v + 64 * k);
          o[2 * k] = fmaf(pj, vv.x, o[2 * k]);
          o[2 * k + 1] = fmaf(pj, vv.y, o[2 * k + 1]);
        }
      }
      __syncwarp();
    }
  }
  if (h >= H) return;
  const float inv = 1.f / lrun;
  __nv_bfloat16 *orow = out + ((int64_t)row * H + h) * D;
#pragma unroll
  for (int k = 0; k < EPL / 2; ++k) {
    *reinterpret_cast<__nv_bfloat162 *>(orow + lane * 2 + 64 * k) =
        __floats2bfloat162_rn(o[2 * k] * inv, o[2 * k + 1] * inv);
  }
  if (lse && lane == 0) lse[(int64_t)row * H + h] = (mrun + log2f(lrun)) * 0.6931471805599453f;
}

template <int D>
int launch_generic(const __nv_bfloat16 *q, const uint8_t *codes, const float *scales,
                   const int32_t *idx, const uint8_t *wcodes, const float *wscales,
                   const int32_t *q_pos, const csa_dims *d, __nv_bfloat16 *out, float *lse,
                   cudaStream_t stream) {
  const int warps = d->H < 8 ? d->H : 8;
  const int rows = d->B * d->Tq;
  const size_t smem = sizeof(float) * (kChunk * D + 8 * kChunk) + sizeof(void *) * kChunk +
                      sizeof(float) * kChunk + sizeof(int) * kMaxSel;
  if (int rc = set_smem_once((const void *)attend_generic_kernel<D>, (int)smem, "attend_generic_kernel")) return rc;
  const dim3 grid((d->H + warps - 1) / warps, 1);
  // grid.y carries the row; split launches beyond 65535 rows
  for (int r0 = 0; r0 < rows; r0 += 65535) {
    const int r = rows - r0 < 65535 ? rows - r0 : 65535;
    attend_generic_kernel<D><<<dim3(grid.x, r), warps * 32, smem, stream>>>(
        q + (int64_t)r0 * d->H * D, codes, scales, idx ? idx + (int64_t)r0 * d->K : nullptr,
        wcodes, wscales, q_pos + r0, d->Tq, d->H, d->K, d->W, d->m, d->n_entries, d->entry_cap,
        d->win_cap, d->softmax_scale, out + (int64_t)r0 * d->H * D, lse ? lse + (int64_t)r0 * d->H : nullptr,
        status_word_device_ptr());
    count_launches(1);
  }
  return check_launch("attend_generic_kernel");
}

}  // namespace

bool attend_tc_supported(const csa_dims *d);
size_t attend_tc_workspace(const csa_dims *d, bool dense);
int launch_attend_tc(const uint16_t *q, const uint8_t *codes, const float *scales, const int32_t *idx,
                     const uint8_t *wcodes, const float *wscales, const int32_t *q_pos,
                     const csa_dims *d, uint16_t *out, float *lse, void *workspace,
                     cudaStream_t stream);

bool attend_prefill_supported(const csa_dims *d);
int launch_attend_prefill(const uint16_t *q, const uint8_t *codes, const float *scales, const int32_t *idx,
                          const uint8_t *wcodes, const float *wscales, const int32_t *q_pos,
                          const csa_dims *d, uint16_t *out, float *lse, cudaStream_t stream);

// 128 heads x 512-wide entries run on the tensor-core kernel with heads as
// the MMA rows; 64 heads x 512 (selected entries + window <= 640 items) on the
// one with items as the MMA rows; other shapes use the generic CUDA-core
// kernel above.
int launch_attend(const uint16_t *q, const uint8_t *codes, const float *scales, const int32_t *idx,
                  const uint8_t *wcodes, const float *wscales, const int32_t *q_pos,
                  const csa_dims *d, uint16_t *out, float *lse, void *workspace, size_t ws_bytes,
                  cudaStream_t stream) {
  (void)ws_bytes;
  if ((int64_t)d->B * d->Tq == 0) return CSA_OK;
  if (attend_tc_supported(d))
    return launch_attend_tc(q, codes, scales, idx, wcodes, wscales, q_pos, d, out, lse, workspace, stream);
  if (idx && attend_prefill_supported(d))
    return launch_attend_prefill(q, codes, scales, idx, wcodes, wscales, q_pos, d, out, lse, stream);
  const auto *qb = reinterpret_cast<const __nv_bfloat16 *>(q);
  auto *ob = reinterpret_cast<__nv_bfloat16 *>(out);
  switch (d->D) {
    case 64: return launch_generic<64>(qb, codes, scales, idx, wcodes, wscales, q_pos, d, ob, lse, stream);
    case 128: return launch_generic<128>(qb, codes, scales, idx, wcodes, wscales, q_pos, d, ob, lse, stream);
    case 256: return launch_generic<256>(qb, codes, scales, idx, wcodes, wscales, q_pos, d, ob, lse, stream);
    case 512: return launch_generic<512>(qb, codes, scales, idx, wcodes, wscales, q_pos, d, ob, lse, stream);
    default: return fail(CSA_ERR_UNSUPPORTED, "attend: D=%d not compiled", d->D);
  }
}

}  // namespace csa

namespace csa {
// The generic kernel keeps its whole softmax state on chip; the tensor-core
// kernel needs scratch for split partial outputs when a row is split.
size_t attend_workspace(const csa_dims *d, bool dense) {
  return attend_tc_supported(d) ? attend_tc_workspace(d, dense) : 0;
}
}  // namespace csa
