/*
 * csa.h -- C ABI of the B200 hybrid compressed-attention library (libcsa.so).
 *
 * The library implements the data-parallel path of DeepSeek-V4-style hybrid
 * attention as four asynchronous GPU operations:
 *
 *   csa_compress    softmax-gated pooling of m-token blocks into FP8 entries
 *   csa_index_topk  FP4 Lightning-Indexer scores + per-query top-k selection
 *   csa_attend      shared-KV multi-query attention over selected entries and
 *                   a sliding window, one joint softmax
 *   hca_attend      the dense (heavily compressed) variant: every visible entry
 *
 * Sources (page title, section):
 *   - "DeepSeek V4とOpenCode" (hazakura.dev), "衝撃1：CSA + HCA": 4 tokens per
 *     CSA entry, FP4 Lightning Indexer picks the top-k, 128-token sliding
 *     window; HCA folds 128 tokens per entry and attends densely.
 *   - jiwasawa.github.io DeepSeek-V4 article, "Compressed Sparse Attention
 *     (CSA)" / "Heavily Compressed Attention (HCA)": sequence length becomes
 *     1/m, indexer scores + top-k selector (DSA), shared key-value MQA over
 *     the selected entries; HCA has m' >> m and no selection; a sliding-window
 *     branch over recent uncompressed tokens runs alongside.
 *   - "DeepSeek V4 Flash：知っておくべき284Bパラメータのオープンソースモデル"
 *     (studioglobal.ai), "アテンションのブレイクスルー：CSAとHCA": softmax-
 *     gated pooling, top 512 compressed blocks per query, HCA 128:1, window of
 *     the latest 128 tokens.
 *   - "DeepSeek V4 1M context window agent efficient inference"
 *     (ai-papers.net), "ハイブリッドアテンションの仕組み": KV entries in FP8,
 *     indexer in FP4.
 *
 * Conventions shared by every call
 * --------------------------------
 *   - All pointers are DEVICE pointers (cudaMalloc / torch CUDA tensors) unless
 *     stated otherwise.  Every buffer is owned by the caller; the library never
 *     allocates, frees or retains a pointer after the call returns.
 *   - Every call is asynchronous on `stream` (NULL = the legacy default
 *     stream); the library never synchronises except in csa_sync_status().
 *   - Buffers must be 16-byte aligned and densely packed in the layouts given
 *     (row-major, last index fastest).
 *   - Return value: CSA_OK (0) or a negative CSA_ERR_* code.  On error nothing
 *     was launched and csa_last_error() returns a message (thread-local).
 *   - Formats: E4M3 = OCP FP8 E4M3 ("FN": no infinities; 0x7F/0xFF are NaN and
 *     never written).  E2M1 = OCP MX FP4, two codes per byte, the even element
 *     in the low nibble.  bf16 values are passed as their uint16 bit patterns.
 */
#ifndef CSA_H
#define CSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st *csa_stream_t;

enum {
  CSA_OK = 0,
  CSA_ERR_INVALID = -1,     /* bad shape, pointer, alignment or argument     */
  CSA_ERR_UNSUPPORTED = -2, /* valid but outside the compiled shape set      */
  CSA_ERR_CUDA = -3,        /* a CUDA runtime call or launch failed          */
  CSA_ERR_TIMEOUT = -4,     /* a device-side bounded wait gave up            */
  CSA_ERR_WORKSPACE = -5,   /* workspace missing or smaller than required    */
  CSA_ERR_CHECK = -6        /* an output check (csa_check_topk, CSA_CHECK build) failed */
};

/*
 * Shapes of one attention / indexer call.
 *   B          sequences in the batch
 *   Tq         query rows per sequence
 *   H          attention query heads (shared K = V, multi-query)
 *   D          width of a KV entry; one of 64, 128, 256, 512
 *   HI, dI     indexer heads (1..8) and indexer width (32 or 64)
 *   K          top-k (1..2048)
 *   W          sliding-window length in tokens (1..win_cap)
 *   m          tokens per compressed entry (CSA: 4, HCA: 128; any m >= 1)
 *   n_entries  valid compressed entries per sequence (cache fill level)
 *   entry_cap  entry stride per sequence of the cache buffers (>= n_entries)
 *   win_cap    window-ring capacity; token p sits in slot p % win_cap
 *   softmax_scale  multiplies q . v before the softmax (1.0: folded into q)
 */
typedef struct csa_dims {
  int32_t B, Tq, H, D, HI, dI, K, W, m;
  int32_t n_entries;
  int64_t entry_cap;
  int32_t win_cap;
  float softmax_scale;
} csa_dims;

/*
 * csa_compress -- softmax-gated pooling into FP8 entries.
 * (studioglobal.ai "アテンションのブレイクスルー：CSAとHCA": softmax-gated
 *  pooling; hazakura.dev "衝撃1": m = 4 and m' = 128; ai-papers.net
 *  "ハイブリッドアテンションの仕組み": FP8 KV.)
 *
 * For every sequence b and every FULL block i (i < T / m; a partial tail is
 * not an entry) and channel c:
 *     C[c]  = sum_j softmax_j(z[b, i*m + j, c]) * x[b, i*m + j, c]   (fp32)
 *     s     = max_c |C[c]| / 448   (s = 1 if that is 0)
 *     code  = E4M3(C[c] / s), round-to-nearest-even, saturating at +-448
 * With m = 1 this stores single tokens (the sliding-window cache).
 *
 *   x, z       fp32 [B, *, D], token t of sequence b at x + b*x_batch_stride + t*D;
 *              the first T tokens are read.
 *   codes      u8   entry slot e of sequence b at codes + (b*dst_batch_stride + e)*D
 *   scales     fp32 scale of that entry at scales[b*dst_batch_stride + e]
 *   dst_first  slot of block 0; block i goes to slot dst_first + i, taken modulo
 *              ring_cap when ring_cap > 0 (ring buffer), else used as is.  With
 *              a ring, only the call's last ring_cap blocks are pooled and
 *              stored (earlier ones would be overwritten by them).
 *   pooled     optional fp32 [B, T/m, D] copy of C before quantisation (NULL = none)
 * Requires D % 4 == 0, 4 <= D <= 1024, m >= 1, T >= 0; T < m is a no-op.
 */
int csa_compress(const float *x, const float *z, int32_t B, int32_t T, int32_t D, int32_t m,
                 int64_t x_batch_stride, uint8_t *codes, float *scales, int64_t dst_first,
                 int64_t dst_batch_stride, int32_t ring_cap, float *pooled,
                 csa_stream_t stream);

/*
 * csa_compress_ew -- csa_compress for the entries and, in the same pass over
 * x, every one of the T tokens as a window entry (csa_compress with m = 1):
 * the block's tokens are read once.  Arguments as csa_compress, plus the
 * window's codes u8 [B, win_cap, D] and scales fp32 [B, win_cap] (batch
 * stride win_batch_stride entries), first slot win_first and ring capacity
 * win_ring_cap (0: no ring; with a ring only the call's last win_ring_cap
 * tokens are written, token p at slot (win_first + p) mod win_ring_cap).
 * Results are bit-identical to the two csa_compress calls.  Fused for
 * m = 2, 4 or 8 and D <= 1024; other m run the two passes.  Tokens past the
 * last full block enter the window only.
 */
int csa_compress_ew(const float *x, const float *z, int32_t B, int32_t T, int32_t D, int32_t m,
                    int64_t x_batch_stride, uint8_t *codes, float *scales, int64_t dst_first,
                    int64_t dst_batch_stride, int32_t ring_cap, uint8_t *win_codes, float *win_scales,
                    int64_t win_first, int64_t win_batch_stride, int32_t win_ring_cap, float *pooled,
                    csa_stream_t stream);

/*
 * csa_index_topk -- Lightning-Indexer scores and top-k.
 * (jiwasawa "Compressed Sparse Attention (CSA)": indexer scores per query and
 *  a top-k selector; hazakura.dev "衝撃1": FP4 indexer; studioglobal.ai
 *  "アテンションのブレイクスルー": top 512 blocks per query.)
 *
 * For query row (b, i) at position t = q_pos[b, i], entry s is visible iff
 * s < n_vis = min(floor((t + 1) / m), n_entries).  Its score is
 *     score = sum_h w[b,i,h] * max(0, sum_j qI[b,i,h,j] * kI[b,s,j])
 * computed exactly (E2M1 products are multiples of 1/4; w must be a multiple
 * of 1/16 in [0, 1], so 64*score is an integer below 2^24).  A weight off
 * that grid is not an argument error the host can see (w lives on the
 * device): the kernels round 16*w to the nearest integer, clamp it to
 * [0, 16] and set a status bit that the next csa_sync_status() reports as
 * CSA_ERR_INVALID; the row's results are then those of the clamped weights.  The row's output
 * lists the min(K, n_vis) best entries in rank order -- score descending, ties
 * to the lower index -- followed by -1 padding.
 *
 *   qI         u8   [B, Tq, HI, dI/2]   packed E2M1, 16-byte aligned
 *   w          fp32 [B, Tq, HI]
 *   kI         u8   [B, entry_cap, dI/2] packed E2M1
 *   q_pos      int32 [B, Tq]             (>= 0)
 *   idx_out    int32 [B, Tq, K]
 *   score_out  fp32 [B, Tq, K] scores of the listed entries (0 for padding), or NULL
 *   workspace  device scratch of at least csa_index_topk_workspace(d) bytes
 * Uses d->B, Tq, HI, dI, K, m, n_entries, entry_cap.
 */
size_t csa_index_topk_workspace(const csa_dims *d);
int csa_index_topk(const uint8_t *qI, const float *w, const uint8_t *kI, const int32_t *q_pos,
                   const csa_dims *d, int32_t *idx_out, float *score_out, void *workspace,
                   size_t workspace_bytes, csa_stream_t stream);

/*
 * csa_index_topk_mx -- the indexer and top-k on block-scaled FP4 (MXFP4)
 * queries and keys.
 * (jiwasawa "限界を押し広げるインフラストラクチャの最適化": FP4 on the
 *  indexer's QK path; studioglobal.ai "FP4/FP8混合精度": MXFP4, two values per
 *  byte; jiwasawa "Compressed Sparse Attention (CSA)": indexer + top-k.)
 *
 * Element j of a query head or key row is its E2M1 code times
 * 2^(s - 127), s the row's UE8M0 scale code for block j / 32 (the output of
 * csa_quantize_mxfp4).  For query row (b, i) at position t and visible entry
 * s (as csa_index_topk):
 *     score = sum_h w[b,i,h] * max(0, sum_j q[b,i,h,j] * k[b,s,j])
 * evaluated on the tensor cores with the block scales applied in the MMA and
 * fp32 accumulation: not exact.  The listed entries are the k best by the
 * computed fp32 score (ties to the lower index), in rank order, -1 padding;
 * entries whose exact scores lie within the evaluation's rounding of the
 * k-th may be listed in place of one another.
 *
 *   qI         u8 [B, Tq, HI, 32]  packed E2M1 (dI = 64), 16-byte aligned
 *   qI_scales  u8 [B, Tq, HI, 2]   UE8M0 codes (0xFF, NaN, is reported)
 *   w          fp32 [B, Tq, HI]    finite, >= 0 (else reported and taken as 0)
 *   kI         u8 [B, entry_cap, 32], 16-byte aligned
 *   kI_scales  u8 [B, entry_cap, 2]
 *   q_pos, idx_out as csa_index_topk; score_out fp32 [B, Tq, K] (the
 *   computed scores, 0 for padding) or NULL
 *   workspace  at least csa_index_topk_mx_workspace(d) bytes
 * Supported: dI = 64, HI 1..8, K 1..2048, and at most 20,480 / K slices of
 * 4,096 entries per row (n_entries <= 163,840 at K = 512); otherwise
 * CSA_ERR_UNSUPPORTED before any launch.  Negative weights, non-finite
 * weights and 0xFF scales set a status bit (csa_sync_status ->
 * CSA_ERR_INVALID).  The workspace query returns 0 for unsupported shapes.
 */
size_t csa_index_topk_mx_workspace(const csa_dims *d);
int csa_index_topk_mx(const uint8_t *qI, const uint8_t *qI_scales, const float *w, const uint8_t *kI,
                      const uint8_t *kI_scales, const int32_t *q_pos, const csa_dims *d,
                      int32_t *idx_out, float *score_out, void *workspace, size_t workspace_bytes,
                      csa_stream_t stream);

/*
 * csa_check_topk -- checks top-k lists on the device (the pages have no
 * counterpart: a debugging aid).  For each row at position t =
 * q_pos[row]: the first min(K, n_vis) indices in [0, n_vis), the rest -1;
 * with score (may be NULL) each listed score finite and >= 0, the list in
 * rank order (score descending, equal scores by ascending index) and padding
 * scores 0.  A violation sets a status bit: the next csa_sync_status()
 * returns CSA_ERR_CHECK.  Nothing traps.  Uses d->B, Tq, K, m, n_entries;
 * idx int32 [B, Tq, K], score fp32 [B, Tq, K], q_pos int32 [B, Tq].
 *
 * csa_check_build -- 1 in the CSA_CHECK build of the library (libcsa_check.so,
 * built by `python -m compressed_sparse_attention_16_b200.build --check`),
 * which runs csa_check_topk after every csa_index_topk, csa_index_topk_mx and
 * csa_decode_step; 0 otherwise.
 */
int csa_check_topk(const int32_t *idx, const float *score, const int32_t *q_pos, const csa_dims *d,
                   csa_stream_t stream);
int csa_check_build(void);

/*
 * csa_index_topk_noalloc -- csa_index_topk without a caller-provided workspace.
 * (The pages have no counterpart: this is a deployment convenience.)
 *
 * For callers that cannot allocate device memory -- code inside allocator
 * hooks, runtimes that plan every byte at load time and forbid cudaMalloc
 * afterwards, plug-ins that only receive their inputs' and outputs' buffers.
 * Same arguments, results and errors as csa_index_topk, minus the workspace:
 * the scratch is an 8 MiB array inside the library's device image, held by
 * every GPU that loads the library until the process exits.  The shape is
 * validated first, exactly as csa_index_topk does; a valid shape whose
 * csa_index_topk_workspace(d) exceeds 8 MiB is then rejected with
 * CSA_ERR_UNSUPPORTED before any launch.  What fits depends on the path the
 * shape takes: up to 64 query rows with >= 2,048 entries, 4 bytes per
 * (row, entry) plus 32 KiB per row (16 rows x 16,384 entries: 1.5 MiB;
 * 64 rows x 20,000 entries: 7.2 MiB); 65 to 148 decode rows, about 33 KiB
 * per row; the prefill path (> 64 rows, K <= 1,024), 16 bytes per
 * (row, K), i.e. up to 1,023 rows at K = 512.  The library allocates nothing
 * and calls no allocating routine.
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.  The cached address does not survive cudaDeviceReset
 *     (or any destruction of the device's primary context).
 *   - All calls share the one array: calls whose kernels overlap on the GPU
 *     (different streams, or different host threads) race and corrupt each
 *     other's results; serialise them.  Stale contents from an earlier call
 *     are harmless (every score is written before it is read, and the
 *     counters a path needs are cleared by the call itself).
 */
int csa_index_topk_noalloc(const uint8_t *qI, const float *w, const uint8_t *kI,
                           const int32_t *q_pos, const csa_dims *d, int32_t *idx_out,
                           float *score_out, csa_stream_t stream);

/*
 * csa_attend -- sparse shared-KV MQA over selected entries + window.
 * (jiwasawa "Compressed Sparse Attention (CSA)": shared key-value MQA over
 *  the selected entries; "Heavily Compressed Attention (HCA)": the sliding
 *  window branch; studioglobal.ai: the window is the latest 128 tokens.)
 *
 * For query row (b, i) at position t = q_pos[b, i] the key/value set is
 *     U = { entry idx[b,i,j] : idx >= 0 }  +  { window token p : max(0,t-W+1) <= p <= t }
 * (no de-duplication), each row dequantised as code * scale, K = V.  For every
 * head h: S_u = softmax_scale * q[b,i,h,:] . U_u,  out = sum_u softmax(S)_u U_u,
 * lse = max S + ln(sum exp(S - max S)).
 *
 *   q          bf16 [B, Tq, H, D]
 *   codes      u8   [B, entry_cap, D], scales fp32 [B, entry_cap]   (csa_compress output)
 *   idx        int32 [B, Tq, K]  (entries must be < n_entries; -1 = unused)
 *   win_codes  u8   [B, win_cap, D], win_scales fp32 [B, win_cap]   (m = 1 entries)
 *   q_pos      int32 [B, Tq]
 *   out        bf16 [B, Tq, H, D];  lse fp32 [B, Tq, H] or NULL
 *   workspace  device scratch of at least csa_attend_workspace(d) bytes
 * Requires W <= win_cap (every window token still resident in the ring).
 */
size_t csa_attend_workspace(const csa_dims *d);
int csa_attend(const uint16_t *q, const uint8_t *codes, const float *scales, const int32_t *idx,
               const uint8_t *win_codes, const float *win_scales, const int32_t *q_pos,
               const csa_dims *d, uint16_t *out, float *lse, void *workspace,
               size_t workspace_bytes, csa_stream_t stream);

/*
 * hca_attend -- dense attention over every visible entry + window.
 * (jiwasawa "Heavily Compressed Attention (HCA)": no sparse selection, dense
 *  attention over the compressed sequence; hazakura.dev "衝撃1": m' = 128.)
 * As csa_attend with the selection replaced by all entries s < n_vis(t) =
 * min(floor((t+1)/m), n_entries).  Same buffers minus idx.
 */
size_t hca_attend_workspace(const csa_dims *d);
int hca_attend(const uint16_t *q, const uint8_t *codes, const float *scales,
               const uint8_t *win_codes, const float *win_scales, const int32_t *q_pos,
               const csa_dims *d, uint16_t *out, float *lse, void *workspace,
               size_t workspace_bytes, csa_stream_t stream);

/*
 * csa_decode_step -- one whole CSA decode step in a single launch: append the
 * step's new tokens, then index, select and attend for one query per
 * sequence.
 * (jiwasawa.github.io DeepSeek-V4 article, "Compressed Sparse Attention
 *  (CSA)": indexer scores, top-k selector, shared key-value MQA over the
 *  selected entries; "Heavily Compressed Attention (HCA)": the sliding-window
 *  branch; hazakura.dev "衝撃1：CSA + HCA": 4 tokens per entry, FP4 indexer,
 *  128-token window, 1M-token contexts; studioglobal.ai "アテンションの
 *  ブレイクスルー": softmax-gated pooling, top 512 blocks.)
 *
 * Computes exactly what this sequence of calls computes, for every sequence
 * b with query position t = q_pos[b]:
 *   1. csa_compress of the n_new tokens x_new/z_new[b] (positions
 *      t - n_new + 1 .. t, which must end a block: (t + 1) % m == 0) into the
 *      entries (t + 1)/m - n_new/m .. (t + 1)/m - 1 of codes/scales, and with
 *      m = 1 into the window ring win_codes/win_scales (slot p % win_cap);
 *   2. if kI_new is not NULL, its rows are copied into kI at those entries;
 *   3. csa_index_topk (Tq = 1) -> idx_out, score_out;
 *   4. csa_attend -> out, lse.
 * The results are bit-identical to those calls' (the same arithmetic in the
 * same order).  A query position that does not end a block, or that has
 * fewer than n_new tokens before it, skips the append for that sequence and
 * sets a status bit (csa_sync_status -> CSA_ERR_INVALID).
 *
 *   x_new, z_new  fp32 [B, n_new, D]
 *   kI_new        u8 [B, n_new / m, dI / 2] packed E2M1, or NULL (keys already in kI)
 *   q             bf16 [B, 1, H, D];  qI u8 [B, 1, HI, dI/2] (16-byte aligned);  w fp32 [B, 1, HI]
 *   q_pos         int32 [B]
 *   codes, scales, kI, win_codes, win_scales: the caches of csa_compress /
 *                 csa_index_topk / csa_attend, updated in place
 *   d             the csa_index_topk / csa_attend shape: Tq = 1, n_entries =
 *                 the entry count after the append (visibility is capped by it)
 *   idx_out int32 [B, 1, K];  score_out fp32 [B, 1, K] or NULL
 *   out bf16 [B, 1, H, D];  lse fp32 [B, 1, H] or NULL
 *   workspace     at least csa_decode_step_workspace(d, n_new) bytes.  It must
 *                 be zero-filled before its first use (cudaMemset after
 *                 allocation); every call then leaves it in the state the next
 *                 call with the same shape expects.  Zero it again when B, K,
 *                 W or the GPU changes, and after a call that timed out
 *                 (csa_sync_status returns CSA_ERR_TIMEOUT).  Calls that share
 *                 a workspace must not overlap on the GPU.
 * Supported: H = 128, D = 512, dI = 64, HI <= 4, Tq = 1, K <= 2048, n_new a
 * multiple of m with n_new <= 16 and n_new <= win_cap, 4*B <= the GPU's SM
 * count, at most 8,192 visible entries per CTA (B sequences share the SMs).
 * Anything else returns CSA_ERR_UNSUPPORTED before any launch (use the
 * separate calls); csa_decode_step_workspace returns 0 for such shapes.
 * The launch is cooperative (one CTA per SM); it must not be issued while
 * another kernel occupies the GPU's SMs indefinitely.
 */
size_t csa_decode_step_workspace(const csa_dims *d, int32_t n_new);
int csa_decode_step(const float *x_new, const float *z_new, int32_t n_new, const uint8_t *kI_new,
                    const uint16_t *q, const uint8_t *qI, const float *w, const int32_t *q_pos,
                    uint8_t *codes, float *scales, uint8_t *kI, uint8_t *win_codes, float *win_scales,
                    const csa_dims *d, int32_t *idx_out, float *score_out, uint16_t *out, float *lse,
                    void *workspace, size_t workspace_bytes, csa_stream_t stream);

/* Message of the last failed call on this host thread ("" if none). */
const char *csa_last_error(void);

/*
 * csa_quantize_mxfp4 -- fp32 values to MXFP4 (E2M1 elements, one E8M0 scale
 * per 32 consecutive elements), the format the indexer consumes.
 * ("DeepSeek V4 Flash：知っておくべき284Bパラメータのオープンソースモデル"
 *  (studioglobal.ai), "FP4/FP8混合精度": FP4 values are MXFP4, two per byte;
 *  jiwasawa.github.io DeepSeek-V4 article, "限界を押し広げるインフラストラクチャ
 *  の最適化": FP4 on the indexer's QK path.)
 *
 * For every block of 32 consecutive elements v of a row:
 *     X     = max(floor(log2(max |v|)) - 2, -127)   (-127 for an all-zero block)
 *     scale = E8M0 code X + 127                     (the value 2^X)
 *     code  = E2M1(v / 2^X), round-to-nearest-even, saturating at +-6; the
 *             sign is kept (a negative value that rounds to zero is -0, 0x8)
 * v / 2^X is exact in fp32, so every code and scale is fully determined.
 *
 *   x        fp32 [rows, cols], finite values
 *   codes    u8   [rows, cols/2]   packed E2M1, the even element in the low nibble
 *   scales   u8   [rows, cols/32]  E8M0 codes
 * Requires cols a positive multiple of 32, rows >= 0 (0 is a no-op); x
 * 16-byte and codes 4-byte aligned.  CSA_ERR_INVALID for anything else.
 */
int csa_quantize_mxfp4(const float *x, int64_t rows, int32_t cols, uint8_t *codes, uint8_t *scales,
                       csa_stream_t stream);

/*
 * Waits for `stream`, then reads and clears the library's device status word,
 * which kernels set when a bounded device-side wait gives up.  Returns CSA_OK,
 * CSA_ERR_TIMEOUT, or CSA_ERR_CUDA if the stream itself reported an error.
 */
int csa_sync_status(csa_stream_t stream);

/* Diagnostic of the failure path (no counterpart on the pages): launches one
 * small kernel whose bounded wait is on an mbarrier phase that nothing
 * completes.  After `limit_ns` nanoseconds of wall time (clamped to
 * [1 us, 100 ms]) the wait gives up exactly as a stalled pipeline in the
 * other kernels does: it sets the timeout bit in the device status word and
 * the kernel returns, leaving the context usable.  The next
 * csa_sync_status(stream) therefore returns CSA_ERR_TIMEOUT (and clears the
 * bit).  Returns CSA_OK or CSA_ERR_CUDA if the launch fails. */
int csa_selftest_timeout(uint64_t limit_ns, csa_stream_t stream);

/* Library ABI version (major * 100 + minor). */
int csa_version(void);

/* Number of GPU kernels this library has launched in this process (all
 * devices, all threads) -- for accounting in benchmarks and tests. */
uint64_t csa_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* CSA_H */
