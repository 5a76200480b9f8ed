// Output checks of the top-k lists, run after every index call in the
// CSA_CHECK build of the library (and callable in any build through
// csa_check_topk).  A violation sets STATUS_CHECK in the device status word;
// nothing traps, so the context stays usable.
//
// A row at position t lists min(k, n_vis) entries, n_vis = min(floor((t + 1)
// / m), n_entries) (jiwasawa.github.io DeepSeek-V4 article, "Compressed Sparse
// Attention (CSA)": the top-k selector over the visible compressed entries):
// every listed index in [0, n_vis), then -1 padding; with scores, each listed
// score finite and >= 0, the list in rank order (score descending, equal
// scores by ascending index, so no index repeats) and the padding scores 0.
#include "common.cuh"

namespace csa {
namespace {

constexpr int kCheckThreads = 256;

__global__ void __launch_bounds__(kCheckThreads)
check_topk_kernel(const int32_t *__restrict__ idx, const float *__restrict__ score, const int32_t *__restrict__ q_pos,
                  int m, int n_entries, int K, unsigned *status) {
  const int64_t row = blockIdx.x;
  const int64_t t = q_pos[row];
  const int nvis = t < 0 ? 0 : (int)min((t + 1) / m, (int64_t)n_entries);
  const int cnt = min(K, nvis);
  const int32_t *ri = idx + row * K;
  const float *rs = score ? score + row * K : nullptr;
  bool bad = false;
  for (int j = threadIdx.x; j < K; j += kCheckThreads) {
    const int32_t v = ri[j];
    if (j < cnt) {
      bad |= v < 0 || v >= nvis;
      if (rs) {
        const float s = rs[j];
        bad |= !(s >= 0.f && s <= 3.402823466e38f);
        if (j + 1 < cnt) {
          const float s2 = rs[j + 1];
          const int32_t v2 = ri[j + 1];
          bad |= !(s > s2 || (s == s2 && v < v2));
        }
      }
    } else {
      bad |= v != -1;
      if (rs) bad |= rs[j] != 0.f;
    }
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) raise_status(status, STATUS_CHECK);
}

}  // namespace

int launch_check_topk(const int32_t *idx, const float *score, const int32_t *q_pos, const csa_dims *d,
                      cudaStream_t stream) {
  const int64_t rows = (int64_t)d->B * d->Tq;
  if (rows == 0) return CSA_OK;
  if (rows >= (1ll << 31)) return fail(CSA_ERR_UNSUPPORTED, "csa_check_topk: too many rows");
  check_topk_kernel<<<(unsigned)rows, kCheckThreads, 0, stream>>>(idx, score, q_pos, d->m, d->n_entries, d->K,
                                                                  status_word_device_ptr());
  count_launches(1);
  return check_launch("check_topk_kernel");
}

}  // namespace csa
