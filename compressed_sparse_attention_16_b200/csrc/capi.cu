// C ABI of libcsa: argument validation, error reporting, the device status
// word, and dispatch to the kernels.  See include/csa.h for the contract of
// every entry point.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace csa {

int launch_compress_ew(const float *x, const float *z, int B, int T, int D, int m, int64_t x_bstride, uint8_t *codes,
                       float *scales, int64_t dst_first, int64_t dst_bstride, int ring_cap, uint8_t *wcodes,
                       float *wscales, int64_t w_first, int64_t w_bstride, int w_ring, float *pooled,
                       cudaStream_t stream);
int launch_compress(const float *x, const float *z, int B, int T, int D, int m, int64_t x_bstride,
                    uint8_t *codes, float *scales, int64_t dst_first, int64_t dst_bstride,
                    int ring_cap, float *pooled, cudaStream_t stream);
size_t index_topk_workspace(const csa_dims *d);
int launch_index_topk(const uint8_t *qI, const float *w, const uint8_t *kI, const int32_t *q_pos,
                      const csa_dims *d, int32_t *idx_out, float *score_out, void *workspace,
                      cudaStream_t stream);
int launch_attend(const uint16_t *q, const uint8_t *codes, const float *scales, const int32_t *idx,
                  const uint8_t *wcodes, const float *wscales, const int32_t *q_pos,
                  const csa_dims *d, uint16_t *out, float *lse, void *workspace, size_t ws_bytes,
                  cudaStream_t stream);
size_t attend_workspace(const csa_dims *d, bool dense);
size_t decode_step_workspace(const csa_dims *d, int n_new);
int launch_decode_step(const float *x_new, const float *z_new, int n_new, const uint8_t *kI_new,
                       const uint16_t *q, const uint8_t *qI, const float *w, const int32_t *q_pos,
                       uint8_t *codes, float *scales, uint8_t *kI, uint8_t *win_codes, float *win_scales,
                       const csa_dims *d, int32_t *idx_out, float *score_out, uint16_t *out, float *lse,
                       void *workspace, size_t workspace_bytes, cudaStream_t stream);

// ---------------------------------------------------------------------------
// errors
// ---------------------------------------------------------------------------
static thread_local char g_err[512] = "";

int fail(int code, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return code;
}

void clear_error() { g_err[0] = '\0'; }

static std::atomic<uint64_t> g_launches{0};
void count_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

int check_launch(const char *what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return CSA_OK;
}

// ---------------------------------------------------------------------------
// device status word: one per device that loads the library
// ---------------------------------------------------------------------------
static __device__ unsigned g_status_word;

unsigned *status_word_device_ptr() {
  static std::mutex mu;
  static unsigned *ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!ptrs[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<unsigned *>(p);
  }
  return ptrs[dev];
}

bool encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType type, const void *base, uint64_t inner, uint64_t rows,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  if (((uintptr_t)base & 15u) != 0 || rows < 1) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode(map, type, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_3d(CUtensorMap *map, CUtensorMapDataType type, const void *base, const uint64_t dims[3],
                    const uint64_t strides[2], const uint32_t box[3]) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (!encode) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return false;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  if (((uintptr_t)base & 15u) != 0) return false;
  const cuuint64_t d[3] = {(cuuint64_t)dims[0], (cuuint64_t)dims[1], (cuuint64_t)dims[2]};
  const cuuint64_t st[2] = {(cuuint64_t)strides[0], (cuuint64_t)strides[1]};
  const cuuint32_t bx[3] = {box[0], box[1], box[2]};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode(map, type, 3, const_cast<void *>(base), d, st, bx, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int set_smem_once(const void *kernel, int bytes, const char *name) {
  // one slot per kernel instance that raises its limit (the generic
  // attention per D, the indexer paths per head count and shape, the
  // attention chunk shapes, the merges, the fused step and the long pooling
  // kernel): fewer than 40 in this library, so 64 slots per device suffice
  constexpr int kSlots = 64;
  static std::mutex mu;
  static const void *done[64][kSlots] = {{nullptr}};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return fail(CSA_ERR_CUDA, "%s: no device", name);
  std::lock_guard<std::mutex> lock(mu);
  for (int i = 0; i < kSlots; ++i) {
    if (done[dev][i] == kernel) return CSA_OK;
    if (done[dev][i] == nullptr) {
      const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
      if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "%s: cudaFuncSetAttribute: %s", name, cudaGetErrorString(e));
      done[dev][i] = kernel;
      return CSA_OK;
    }
  }
  return fail(CSA_ERR_CUDA, "%s: attribute table full", name);
}

// A bounded wait on a phase nothing completes: it gives up after limit_ns
// and reports STATUS_TIMEOUT, the path every pipeline wait takes on expiry.
__global__ void selftest_timeout_kernel(unsigned long long limit_ns, unsigned *status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(1u) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    uint64_t t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    for (;;) {
      uint32_t ok;
      asm volatile(
          "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
          "selp.u32 %0, 1, 0, p;\n\t}"
          : "=r"(ok)
          : "r"(a), "r"(0u)
          : "memory");
      if (ok) break;   // never: no thread arrives
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
      if (t - t0 > limit_ns) {
        raise_status(status, STATUS_TIMEOUT);
        break;
      }
    }
  }
}

}  // namespace csa

using namespace csa;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

int need_status() {
  if (!status_word_device_ptr())
    return fail(CSA_ERR_CUDA, "cannot resolve the device status word (no CUDA device?)");
  return CSA_OK;
}

int check_attend_dims(const char *fn, const csa_dims *d, bool dense) {
  if (!d) return fail(CSA_ERR_INVALID, "%s: dims is NULL", fn);
  if (d->B < 0 || d->Tq < 0 || d->H < 1 || d->W < 1 || d->m < 1 || d->n_entries < 0)
    return fail(CSA_ERR_INVALID, "%s: bad dims (B=%d Tq=%d H=%d W=%d m=%d n_entries=%d)", fn, d->B,
                d->Tq, d->H, d->W, d->m, d->n_entries);
  if (d->entry_cap < d->n_entries) return fail(CSA_ERR_INVALID, "%s: entry_cap < n_entries", fn);
  if (d->win_cap < d->W) return fail(CSA_ERR_INVALID, "%s: win_cap (%d) < W (%d)", fn, d->win_cap, d->W);
  if (d->D != 64 && d->D != 128 && d->D != 256 && d->D != 512)
    return fail(CSA_ERR_UNSUPPORTED, "%s: D=%d (supported 64, 128, 256, 512)", fn, d->D);
  if (!dense && (d->K < 1 || d->K > 2048))
    return fail(CSA_ERR_UNSUPPORTED, "%s: K=%d (supported 1..2048)", fn, d->K);
  if (!(d->softmax_scale == d->softmax_scale)) return fail(CSA_ERR_INVALID, "%s: softmax_scale is NaN", fn);
  return CSA_OK;
}

}  // namespace

namespace csa {
int check_index_dims(const char *fn, const csa_dims *d) {
  if (!d) return fail(CSA_ERR_INVALID, "%s: dims is NULL", fn);
  if (d->B < 0 || d->Tq < 0 || d->m < 1 || d->n_entries < 0 || d->entry_cap < d->n_entries)
    return fail(CSA_ERR_INVALID, "%s: bad dims (B=%d Tq=%d m=%d n_entries=%d entry_cap=%lld)", fn, d->B, d->Tq,
                d->m, d->n_entries, (long long)d->entry_cap);
  if (d->K < 1 || d->K > 2048) return fail(CSA_ERR_UNSUPPORTED, "%s: K=%d (1..2048)", fn, d->K);
  if ((d->dI != 32 && d->dI != 64) || d->HI < 1 || d->HI > 8)
    return fail(CSA_ERR_UNSUPPORTED, "%s: HI=%d dI=%d", fn, d->HI, d->dI);
  return CSA_OK;
}
// The CSA_CHECK build checks every top-k list the library writes; the
// default build does not.
static int debug_check_topk(const int32_t *idx, const float *score, const int32_t *q_pos, const csa_dims *d,
                            cudaStream_t stream) {
#ifdef CSA_CHECK
  return launch_check_topk(idx, score, q_pos, d, stream);
#else
  (void)idx; (void)score; (void)q_pos; (void)d; (void)stream;
  return CSA_OK;
#endif
}
}  // namespace csa

extern "C" {

int csa_check_build(void) {
#ifdef CSA_CHECK
  return 1;
#else
  return 0;
#endif
}

int csa_check_topk(const int32_t *idx, const float *score, const int32_t *q_pos, const csa_dims *d,
                   csa_stream_t stream) {
  clear_error();
  if (!d || !idx || !q_pos || d->B < 0 || d->Tq < 0 || d->m < 1 || d->K < 1 || d->n_entries < 0)
    return fail(CSA_ERR_INVALID, "csa_check_topk: bad arguments");
  if (((uintptr_t)idx & 3) || ((uintptr_t)score & 3) || ((uintptr_t)q_pos & 3))
    return fail(CSA_ERR_INVALID, "csa_check_topk: misaligned buffer");
  return launch_check_topk(idx, score, q_pos, d, reinterpret_cast<cudaStream_t>(stream));
}

int csa_version(void) { return 100; }

uint64_t csa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int csa_selftest_timeout(uint64_t limit_ns, csa_stream_t stream) {
  csa::clear_error();
  if (limit_ns < 1000ull) limit_ns = 1000ull;
  if (limit_ns > 100000000ull) limit_ns = 100000000ull;
  csa::selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns,
                                                                                 csa::status_word_device_ptr());
  csa::count_launches(1);
  return csa::check_launch("selftest_timeout_kernel");
}

const char *csa_last_error(void) { return g_err; }

int csa_compress(const float *x, const float *z, int32_t B, int32_t T, int32_t D, int32_t m,
                 int64_t x_batch_stride, uint8_t *codes, float *scales, int64_t dst_first,
                 int64_t dst_batch_stride, int32_t ring_cap, float *pooled,
                 csa_stream_t stream) {
  clear_error();
  if (B < 0 || T < 0 || m < 1) return fail(CSA_ERR_INVALID, "csa_compress: bad B/T/m (%d/%d/%d)", B, T, m);
  if (D < 4 || D > 1024 || D % 4 || !pow2(D / 4))
    return fail(CSA_ERR_UNSUPPORTED, "csa_compress: D=%d (needs D/4 a power of two, 4..1024)", D);
  if (B == 0 || T < m) return CSA_OK;
  if (!x || !z || !codes || !scales) return fail(CSA_ERR_INVALID, "csa_compress: NULL buffer");
  if (!aligned16(x) || !aligned16(z) || (pooled && !aligned16(pooled)) || ((uintptr_t)codes & 3))
    return fail(CSA_ERR_INVALID, "csa_compress: misaligned buffer");
  if (x_batch_stride % 4 || (B > 1 && x_batch_stride < (int64_t)T * D))
    return fail(CSA_ERR_INVALID, "csa_compress: x_batch_stride must be a multiple of 4 and >= T*D");
  if (dst_first < 0 || ring_cap < 0) return fail(CSA_ERR_INVALID, "csa_compress: negative dst_first/ring_cap");
  if (ring_cap == 0 && B > 1 && dst_batch_stride < dst_first + T / m)
    return fail(CSA_ERR_INVALID, "csa_compress: dst_batch_stride too small");
  if (ring_cap > 0 && B > 1 && dst_batch_stride < ring_cap)
    return fail(CSA_ERR_INVALID, "csa_compress: dst_batch_stride < ring_cap");
  return launch_compress(x, z, B, T, D, m, x_batch_stride, codes, scales, dst_first,
                         dst_batch_stride, ring_cap, pooled, reinterpret_cast<cudaStream_t>(stream));
}

int csa_compress_ew(const float *x, const float *z, int32_t B, int32_t T, int32_t D, int32_t m,
                    int64_t x_batch_stride, uint8_t *codes, float *scales, int64_t dst_first,
                    int64_t dst_batch_stride, int32_t ring_cap, uint8_t *win_codes, float *win_scales,
                    int64_t win_first, int64_t win_batch_stride, int32_t win_ring_cap, float *pooled,
                    csa_stream_t stream) {
  clear_error();
  if (B < 0 || T < 0 || m < 1) return fail(CSA_ERR_INVALID, "csa_compress_ew: bad B/T/m (%d/%d/%d)", B, T, m);
  if (D < 4 || D > 1024 || D % 4 || !pow2(D / 4))
    return fail(CSA_ERR_UNSUPPORTED, "csa_compress_ew: D=%d (needs D/4 a power of two, 4..1024)", D);
  if (B == 0 || T == 0) return CSA_OK;
  if (!x || !z || !codes || !scales || !win_codes || !win_scales)
    return fail(CSA_ERR_INVALID, "csa_compress_ew: NULL buffer");
  if (!aligned16(x) || !aligned16(z) || (pooled && !aligned16(pooled)) || ((uintptr_t)codes & 3) ||
      ((uintptr_t)win_codes & 3))
    return fail(CSA_ERR_INVALID, "csa_compress_ew: misaligned buffer");
  if (x_batch_stride % 4 || (B > 1 && x_batch_stride < (int64_t)T * D))
    return fail(CSA_ERR_INVALID, "csa_compress_ew: x_batch_stride must be a multiple of 4 and >= T*D");
  if (dst_first < 0 || ring_cap < 0 || win_first < 0 || win_ring_cap < 0)
    return fail(CSA_ERR_INVALID, "csa_compress_ew: negative first slot or ring capacity");
  if (ring_cap == 0 && B > 1 && dst_batch_stride < dst_first + T / m)
    return fail(CSA_ERR_INVALID, "csa_compress_ew: dst_batch_stride too small");
  if (ring_cap > 0 && B > 1 && dst_batch_stride < ring_cap)
    return fail(CSA_ERR_INVALID, "csa_compress_ew: dst_batch_stride < ring_cap");
  if (win_ring_cap == 0 && B > 1 && win_batch_stride < win_first + T)
    return fail(CSA_ERR_INVALID, "csa_compress_ew: win_batch_stride too small");
  if (win_ring_cap > 0 && B > 1 && win_batch_stride < win_ring_cap)
    return fail(CSA_ERR_INVALID, "csa_compress_ew: win_batch_stride < win_ring_cap");
  return launch_compress_ew(x, z, B, T, D, m, x_batch_stride, codes, scales, dst_first, dst_batch_stride, ring_cap,
                            win_codes, win_scales, win_first, win_batch_stride, win_ring_cap, pooled,
                            reinterpret_cast<cudaStream_t>(stream));
}

size_t csa_index_topk_workspace(const csa_dims *d) {
  if (!d || d->B < 0 || d->Tq < 0 || d->n_entries < 0) return 0;
  return index_topk_workspace(d);
}

int csa_index_topk(const uint8_t *qI, const float *w, const uint8_t *kI, const int32_t *q_pos,
                   const csa_dims *d, int32_t *idx_out, float *score_out, void *workspace,
                   size_t workspace_bytes, csa_stream_t stream) {
  clear_error();
  if (int rc = check_index_dims("csa_index_topk", d)) return rc;
  if ((int64_t)d->B * d->Tq == 0) return CSA_OK;
  if (!qI || !w || !kI || !q_pos || !idx_out) return fail(CSA_ERR_INVALID, "csa_index_topk: NULL buffer");
  if (!aligned16(kI) || !aligned16(qI) || ((uintptr_t)w & 3) || ((uintptr_t)q_pos & 3) ||
      ((uintptr_t)idx_out & 3) || ((uintptr_t)score_out & 3))
    return fail(CSA_ERR_INVALID, "csa_index_topk: misaligned buffer");
  const size_t need = index_topk_workspace(d);
  if (need && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(CSA_ERR_WORKSPACE, "csa_index_topk: workspace needs %zu bytes (got %zu)", need,
                workspace_bytes);
  if (int rc = need_status()) return rc;
  const int rc = launch_index_topk(qI, w, kI, q_pos, d, idx_out, score_out, workspace,
                                   reinterpret_cast<cudaStream_t>(stream));
  return rc ? rc : debug_check_topk(idx_out, score_out, q_pos, d, reinterpret_cast<cudaStream_t>(stream));
}

size_t csa_index_topk_mx_workspace(const csa_dims *d) {
  if (!d || d->B < 0 || d->Tq < 0 || d->n_entries < 0) return 0;
  return index_mx_workspace(d);
}

int csa_index_topk_mx(const uint8_t *qI, const uint8_t *qI_scales, const float *w, const uint8_t *kI,
                      const uint8_t *kI_scales, const int32_t *q_pos, const csa_dims *d, int32_t *idx_out,
                      float *score_out, void *workspace, size_t workspace_bytes, csa_stream_t stream) {
  clear_error();
  if (int rc = check_index_dims("csa_index_topk_mx", d)) return rc;
  if ((int64_t)d->B * d->Tq == 0) return CSA_OK;
  if (!qI || !qI_scales || !w || !kI || !kI_scales || !q_pos || !idx_out)
    return fail(CSA_ERR_INVALID, "csa_index_topk_mx: NULL buffer");
  if (!aligned16(kI) || !aligned16(qI) || ((uintptr_t)w & 3) || ((uintptr_t)q_pos & 3) ||
      ((uintptr_t)idx_out & 3) || ((uintptr_t)score_out & 3))
    return fail(CSA_ERR_INVALID, "csa_index_topk_mx: misaligned buffer");
  int splits, slice;
  if (!index_mx_plan(d, &splits, &slice))
    return fail(CSA_ERR_UNSUPPORTED, "csa_index_topk_mx: dI=%d HI=%d K=%d n_entries=%d (supported: dI 64, HI 1..8, "
                "at most 20,480 / K slices of 4,096 entries)", d->dI, d->HI, d->K, d->n_entries);
  const size_t need = index_mx_workspace(d);
  if (!workspace || workspace_bytes < need || !aligned16(workspace))
    return fail(CSA_ERR_WORKSPACE, "csa_index_topk_mx: workspace needs %zu bytes (got %zu)", need,
                workspace_bytes);
  if (int rc = need_status()) return rc;
  const int rc = launch_index_mx(qI, qI_scales, w, kI, kI_scales, q_pos, d, idx_out, score_out, workspace,
                                 reinterpret_cast<cudaStream_t>(stream));
  return rc ? rc : debug_check_topk(idx_out, score_out, q_pos, d, reinterpret_cast<cudaStream_t>(stream));
}

size_t csa_attend_workspace(const csa_dims *d) { return d ? attend_workspace(d, false) : 0; }
size_t hca_attend_workspace(const csa_dims *d) { return d ? attend_workspace(d, true) : 0; }

static int attend_common(const char *fn, const uint16_t *q, const uint8_t *codes,
                         const float *scales, const int32_t *idx, const uint8_t *win_codes,
                         const float *win_scales, const int32_t *q_pos, const csa_dims *d,
                         uint16_t *out, float *lse, void *workspace, size_t workspace_bytes,
                         csa_stream_t stream) {
  clear_error();
  const bool dense = idx == nullptr;
  if (int rc = check_attend_dims(fn, d, dense)) return rc;
  if ((int64_t)d->B * d->Tq == 0) return CSA_OK;
  if (!q || !win_codes || !win_scales || !q_pos || !out || (d->n_entries > 0 && (!codes || !scales)))
    return fail(CSA_ERR_INVALID, "%s: NULL buffer", fn);
  if (!aligned16(q) || !aligned16(out) || (codes && !aligned16(codes)) || !aligned16(win_codes) ||
      ((uintptr_t)q_pos & 3) || ((uintptr_t)idx & 3) || ((uintptr_t)lse & 3) ||
      ((uintptr_t)scales & 3) || ((uintptr_t)win_scales & 3))
    return fail(CSA_ERR_INVALID, "%s: misaligned buffer", fn);
  const size_t need = attend_workspace(d, dense);
  if (need && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(CSA_ERR_WORKSPACE, "%s: workspace needs %zu bytes (got %zu)", fn, need, workspace_bytes);
  if (int rc = need_status()) return rc;
  return launch_attend(q, codes, scales, idx, win_codes, win_scales, q_pos, d, out, lse, workspace,
                       workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
}

int csa_attend(const uint16_t *q, const uint8_t *codes, const float *scales, const int32_t *idx,
               const uint8_t *win_codes, const float *win_scales, const int32_t *q_pos,
               const csa_dims *d, uint16_t *out, float *lse, void *workspace,
               size_t workspace_bytes, csa_stream_t stream) {
  if (!idx) {
    clear_error();
    return fail(CSA_ERR_INVALID, "csa_attend: idx is NULL (use hca_attend for dense attention)");
  }
  return attend_common("csa_attend", q, codes, scales, idx, win_codes, win_scales, q_pos, d, out,
                       lse, workspace, workspace_bytes, stream);
}

int hca_attend(const uint16_t *q, const uint8_t *codes, const float *scales,
               const uint8_t *win_codes, const float *win_scales, const int32_t *q_pos,
               const csa_dims *d, uint16_t *out, float *lse, void *workspace,
               size_t workspace_bytes, csa_stream_t stream) {
  return attend_common("hca_attend", q, codes, scales, nullptr, win_codes, win_scales, q_pos, d,
                       out, lse, workspace, workspace_bytes, stream);
}

size_t csa_decode_step_workspace(const csa_dims *d, int32_t n_new) {
  if (!d) return 0;
  const size_t n = decode_step_workspace(d, n_new);
  clear_error();
  return n;
}

int csa_decode_step(const float *x_new, const float *z_new, int32_t n_new, const uint8_t *kI_new,
                    const uint16_t *q, const uint8_t *qI, const float *w, const int32_t *q_pos,
                    uint8_t *codes, float *scales, uint8_t *kI, uint8_t *win_codes, float *win_scales,
                    const csa_dims *d, int32_t *idx_out, float *score_out, uint16_t *out, float *lse,
                    void *workspace, size_t workspace_bytes, csa_stream_t stream) {
  clear_error();
  if (int rc = check_index_dims("csa_decode_step", d)) return rc;
  if (int rc = check_attend_dims("csa_decode_step", d, false)) return rc;
  if (d->B == 0) return CSA_OK;
  if (!x_new || !z_new || !q || !qI || !w || !q_pos || !codes || !scales || !kI || !win_codes || !win_scales ||
      !idx_out || !out)
    return fail(CSA_ERR_INVALID, "csa_decode_step: NULL buffer");
  if (!aligned16(x_new) || !aligned16(z_new) || !aligned16(q) || !aligned16(out) || !aligned16(codes) ||
      !aligned16(kI) || !aligned16(win_codes) || (kI_new && !aligned16(kI_new)) || ((uintptr_t)qI & 15) ||
      ((uintptr_t)w & 3) || ((uintptr_t)q_pos & 3) || ((uintptr_t)scales & 3) || ((uintptr_t)win_scales & 3) ||
      ((uintptr_t)idx_out & 3) || ((uintptr_t)score_out & 3) || ((uintptr_t)lse & 3) || !aligned16(workspace))
    return fail(CSA_ERR_INVALID, "csa_decode_step: misaligned buffer");
  if (int rc = need_status()) return rc;
  const int rc = launch_decode_step(x_new, z_new, n_new, kI_new, q, qI, w, q_pos, codes, scales, kI, win_codes, win_scales,
                            d, idx_out, score_out, out, lse, workspace, workspace_bytes,
                            reinterpret_cast<cudaStream_t>(stream));
  return rc ? rc : debug_check_topk(idx_out, score_out, q_pos, d, reinterpret_cast<cudaStream_t>(stream));
}

int csa_sync_status(csa_stream_t stream) {
  clear_error();
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "csa_sync_status: %s", cudaGetErrorString(e));
  unsigned *p = status_word_device_ptr();
  if (!p) return fail(CSA_ERR_CUDA, "csa_sync_status: no device status word");
  unsigned v = 0;
  e = cudaMemcpy(&v, p, sizeof(v), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemset(p, 0, sizeof(unsigned));
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail(CSA_ERR_CUDA, "csa_sync_status: %s", cudaGetErrorString(e));
  if (v & STATUS_TIMEOUT) return fail(CSA_ERR_TIMEOUT, "a device-side wait timed out (status 0x%x)", v);
  if (v & STATUS_CHECK) return fail(CSA_ERR_CHECK, "an output check failed: a top-k list out of order or range "
                                    "(status 0x%x)", v);
  if (v & (STATUS_BAD_WEIGHT | STATUS_BAD_INDEX | STATUS_BAD_POSITION))
    return fail(CSA_ERR_INVALID, "invalid device data: %s%s%s (status 0x%x)",
                (v & STATUS_BAD_WEIGHT) ? "indexer weight off its grid or a NaN block scale; " : "",
                (v & STATUS_BAD_INDEX) ? "attention index out of range; " : "",
                (v & STATUS_BAD_POSITION) ? "negative query position" : "", v);
  return CSA_OK;
}

}  // extern "C"
