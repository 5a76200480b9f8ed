// Shared device helpers and host error plumbing for libcsa.
#pragma once

#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "csa.h"

namespace csa {

// ---------------------------------------------------------------------------
// host side: thread-local error message
// ---------------------------------------------------------------------------
int fail(int code, const char *fmt, ...);
int check_launch(const char *what);
void count_launches(unsigned n);   // bookkeeping for csa_launch_count()
void clear_error();
// Host checks of a csa_index_topk shape (CSA_OK or the error, message set).
int check_index_dims(const char *fn, const csa_dims *d);
// The K best of each row's splits x K candidate keys in rank order (scores
// as 64 * score integers, or fp32 bits when float_scores).
int launch_topk_merge(const uint64_t *cand, int splits, const csa_dims *d, const int32_t *q_pos, int32_t *idx_out,
                      float *score_out, bool float_scores, cudaStream_t stream);
// The block-scaled (MXFP4) indexer: plan, workspace bytes (0 when the shape
// is outside the plan), launch.
bool index_mx_plan(const csa_dims *d, int *splits, int *slice);
size_t index_mx_workspace(const csa_dims *d);
int launch_index_mx(const uint8_t *qI, const uint8_t *qs, const float *w, const uint8_t *kI, const uint8_t *ks,
                    const int32_t *q_pos, const csa_dims *d, int32_t *idx_out, float *score_out, void *workspace,
                    cudaStream_t stream);

// ---------------------------------------------------------------------------
// device status word (set by kernels, read + cleared by csa_sync_status)
// ---------------------------------------------------------------------------
enum : unsigned {
  STATUS_TIMEOUT = 1u,      // a bounded wait gave up
  STATUS_BAD_WEIGHT = 2u,   // indexer weight off its grid (1/16 steps in [0, 1]; block-scaled: negative or
                            // not finite, or an E8M0 scale of 0xFF)
  STATUS_BAD_INDEX = 4u,    // attention index outside [0, n_entries) other than -1
  STATUS_BAD_POSITION = 8u, // negative query position (treated as position 0 / no entries)
  STATUS_CHECK = 16u,       // an output check found a top-k list out of order or range
};
// Checks each row's top-k list (indices in range and rank order); a violation
// sets STATUS_CHECK.  Run after every index call in the CSA_CHECK build.
int launch_check_topk(const int32_t *idx, const float *score, const int32_t *q_pos, const csa_dims *d,
                      cudaStream_t stream);
unsigned *status_word_device_ptr();   // address of the status word, current device
// Raises a kernel's dynamic shared-memory limit once per (device, kernel), so
// that launches captured into CUDA graphs issue no attribute calls.
int set_smem_once(const void *kernel, int bytes, const char *name);
// 2-D tensor map for TMA loads: `rows` rows of `inner` elements, `row_bytes`
// apart; boxes of box_inner x box_rows.  False if the driver entry point is
// missing or the encoder rejects the arguments.
bool encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType type, const void *base, uint64_t inner, uint64_t rows,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows, CUtensorMapSwizzle swizzle);
// 3-D tensor map without swizzling: dims[0] is the contiguous dimension,
// strides[0..1] the byte strides of dims 1 and 2, box[0..2] the box.
bool encode_tmap_3d(CUtensorMap *map, CUtensorMapDataType type, const void *base, const uint64_t dims[3],
                    const uint64_t strides[2], const uint32_t box[3]);

__device__ __forceinline__ void raise_status(unsigned *status, unsigned bit) {
  atomicOr(status, bit);
}

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Two E4M3 codes (low byte first) -> two floats (exact).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t two) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
  return __half22float2(*reinterpret_cast<__half2 *>(&h));
}

// PTX prmt in its default mode: each selector nibble picks one of the 8 bytes
// of {b:a}; if the nibble's bit 3 is set, the picked byte's sign bit is
// replicated instead of copying it.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// Four E4M3 codes (low byte first) -> four bf16 (exact), as two bf16x2
// words.  Byte s eeee mmm is placed at bf16 bits s 0000eeee mmm0000: for
// e >= 1 that bf16 is 2^(e-127) (1 + m/8), for e = 0 the bf16 subnormal
// (m/8) 2^-126, in both cases the code's value (2^(e-7) (1 + m/8), resp.
// m 2^-9) times 2^-120; one bf16 multiply by 2^120 (bits 0x7B80) then
// restores it exactly.  Integer placement and one multiply per pair replace
// three conversion instructions.  The two NaN codes (0x7F, 0xFF), which
// the library's quantiser never writes, come out as +-480.
__device__ __forceinline__ void e4m3x4_to_bf16x4(uint32_t w, uint32_t &lo, uint32_t &hi) {
  // 16-bit lanes [sign byte : code]: bytes 0, 1 (resp. 2, 3) of w with their
  // sign bits replicated into the byte above
  const uint32_t t0 = prmt(w, 0u, 0x9180u), t1 = prmt(w, 0u, 0xB3A2u);
  const uint32_t y0 = ((t0 << 4) & 0x07F007F0u) | (t0 & 0x80008000u);
  const uint32_t y1 = ((t1 << 4) & 0x07F007F0u) | (t1 & 0x80008000u);
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(lo) : "r"(y0), "r"(0x7B807B80u));
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(hi) : "r"(y1), "r"(0x7B807B80u));
}

// 16 E4M3 codes -> 16 bf16 (exact), as two 16-byte words
__device__ __forceinline__ void e4m3x16_to_bf16x16(const uint4 &c, uint4 &lo, uint4 &hi) {
  e4m3x4_to_bf16x4(c.x, lo.x, lo.y);
  e4m3x4_to_bf16x4(c.y, lo.z, lo.w);
  e4m3x4_to_bf16x4(c.z, hi.x, hi.y);
  e4m3x4_to_bf16x4(c.w, hi.z, hi.w);
}

}  // namespace csa
