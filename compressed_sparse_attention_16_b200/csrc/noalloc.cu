// csa_index_topk_noalloc: the indexer + top-k call for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code running inside a custom
// allocator's hooks, inference runtimes that forbid allocation after start-up
// (every byte is planned at load time), plug-ins that only receive the
// buffers of their inputs and outputs, and host threads that must not
// synchronise the device (cudaMalloc/cudaFree may).  csa_index_topk needs a
// caller-provided workspace for its per-entry score buffer; this variant uses
// instead a fixed scratch array that lives in the library's own device image.
//
// The scratch is a file-scope __device__ array of kScratchBytes.  Every GPU
// that loads the library holds this memory until the process exits.  Host
// code cannot use the array's name as a device address, so on the first call
// on each device the entry point asks the runtime for the array's address
// (cudaGetSymbolAddress with that device current), checks the result and
// caches it; later calls reuse the cached address.  The cache is per device
// ordinal for the life of the process: it does not survive cudaDeviceReset
// (or anything else that destroys and recreates the device's primary
// context), after which the cached address would be stale.
#include <mutex>

#include "common.cuh"

namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;   // 8 MiB

static __device__ __align__(256) unsigned char g_index_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[64] = {nullptr};

// Device address of the scratch array on the current device, or nullptr with
// the error recorded.
void *scratch_address() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    csa::fail(CSA_ERR_CUDA, "csa_index_topk_noalloc: no current CUDA device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_index_scratch);
    if (e != cudaSuccess || p == nullptr) {
      csa::fail(CSA_ERR_CUDA, "csa_index_topk_noalloc: cudaGetSymbolAddress failed: %s",
                cudaGetErrorString(e));
      return nullptr;
    }
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" {

int csa_index_topk_noalloc(const uint8_t *qI, const float *w, const uint8_t *kI,
                           const int32_t *q_pos, const csa_dims *d, int32_t *idx_out,
                           float *score_out, csa_stream_t stream) {
  csa::clear_error();
  // the shape is validated first, exactly as csa_index_topk does, so that the
  // scratch size below is only ever computed for a valid shape
  if (int rc = csa::check_index_dims("csa_index_topk_noalloc", d)) return rc;
  const size_t need = csa_index_topk_workspace(d);
  if (need > kScratchBytes)
    return csa::fail(CSA_ERR_UNSUPPORTED,
                     "csa_index_topk_noalloc: this shape needs %zu bytes of scratch; the "
                     "allocation-free variant holds at most %zu (use csa_index_topk with a workspace)",
                     need, kScratchBytes);
  void *scratch = scratch_address();
  if (!scratch) return CSA_ERR_CUDA;
  // The scores are written before they are read, so stale contents left by
  // an earlier call need no clearing.
  return csa_index_topk(qI, w, kI, q_pos, d, idx_out, score_out, scratch, kScratchBytes, stream);
}

}  // extern "C"
