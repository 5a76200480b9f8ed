// fp32 -> MXFP4: E2M1 elements with one E8M0 (power-of-two) scale per block
// of 32 consecutive elements.
//
// Page: "DeepSeek V4 Flash：知っておくべき284Bパラメータのオープンソースモデル"
// (studioglobal.ai), section "FP4/FP8混合精度" -- FP4 values are MXFP4, two
// per byte; jiwasawa.github.io DeepSeek-V4 article, section "限界を押し広げる
// インフラストラクチャの最適化" -- FP4 on the indexer's QK path.  The block
// scale follows the microscaling rule: X = floor(log2(max|v|)) - 2 (the
// largest E2M1 value is 1.5 * 2^2), at least -127, so that max|v| / 2^X lies
// in [4, 8) and the elements round to E2M1 with saturation at 6.
//
// HBM-bound: each thread reads 8 consecutive values (two 16-byte loads) and
// writes 4 bytes of codes; four consecutive threads hold one 32-element
// block and agree on its maximum with two shuffles.  v * 2^-X is exact in
// fp32 (a power-of-two scaling that neither overflows nor loses a bit that
// E2M1 could keep), so the hardware conversion (round to nearest even,
// saturating) decides every code exactly.
#include "common.cuh"

namespace csa {
namespace {

constexpr int kQThreads = 256;

// Eight fp32 -> four bytes of E2M1 codes, element i in nibble i (the even
// element of each pair in the low nibble).  The conversion's first source
// goes to the high nibble.
__device__ __forceinline__ uint32_t e2m1x8(float4 a, float4 b) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(a.x), "f"(a.y), "f"(a.z), "f"(a.w), "f"(b.x), "f"(b.y), "f"(b.z), "f"(b.w));
  return r;
}

__global__ void __launch_bounds__(kQThreads) quantize_mxfp4_kernel(const float4 *__restrict__ x, int64_t groups,
                                                                   uint32_t *__restrict__ codes,
                                                                   uint8_t *__restrict__ scales) {
  const int64_t stride = (int64_t)gridDim.x * kQThreads;   // a multiple of 32: a warp keeps whole blocks
  // every lane runs the same number of iterations (the shuffles need all 32)
  const int64_t first = (int64_t)blockIdx.x * kQThreads + threadIdx.x;
  const int64_t base = first - (threadIdx.x & 31);
  for (int64_t g0 = base; g0 < groups; g0 += stride) {
    const int64_t g = g0 + (threadIdx.x & 31);
    const bool in = g < groups;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (in) {
      a = __ldg(x + 2 * g);
      b = __ldg(x + 2 * g + 1);
    }
    float m = fmaxf(fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))),
                    fmaxf(fmaxf(fabsf(b.x), fabsf(b.y)), fmaxf(fabsf(b.z), fabsf(b.w))));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    // biased exponent e of max|v| (0 for zero and subnormals): floor(log2) = e - 127
    const int e = (int)((__float_as_uint(m) >> 23) & 0xFFu);
    const int X = max(e - 129, -127);
    const float inv = __int_as_float((127 - X) << 23);   // 2^-X, X in [-127, 126]
    const uint32_t w = e2m1x8(make_float4(a.x * inv, a.y * inv, a.z * inv, a.w * inv),
                              make_float4(b.x * inv, b.y * inv, b.z * inv, b.w * inv));
    if (in) {
      codes[g] = w;
      if ((g & 3) == 0) scales[g >> 2] = (uint8_t)(X + 127);
    }
  }
}

}  // namespace
}  // namespace csa

extern "C" int csa_quantize_mxfp4(const float *x, int64_t rows, int32_t cols, uint8_t *codes, uint8_t *scales,
                                  csa_stream_t stream) {
  using namespace csa;
  clear_error();
  if (rows < 0 || cols <= 0 || cols % 32)
    return fail(CSA_ERR_INVALID, "csa_quantize_mxfp4: rows=%lld, cols=%d (cols must be a positive multiple of 32)",
                (long long)rows, cols);
  if (rows == 0) return CSA_OK;
  if (!x || !codes || !scales) return fail(CSA_ERR_INVALID, "csa_quantize_mxfp4: NULL buffer");
  if (((uintptr_t)x & 15) || ((uintptr_t)codes & 3)) return fail(CSA_ERR_INVALID, "csa_quantize_mxfp4: misaligned buffer");
  if (rows > ((int64_t)1 << 40) / cols) return fail(CSA_ERR_INVALID, "csa_quantize_mxfp4: too many elements");
  const int64_t groups = rows * cols / 8;
  static int sms_cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return fail(CSA_ERR_CUDA, "csa_quantize_mxfp4: no device");
  if (!sms_cache[dev] && cudaDeviceGetAttribute(&sms_cache[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return fail(CSA_ERR_CUDA, "csa_quantize_mxfp4: cannot query the SM count");
  const int64_t want = (groups + kQThreads - 1) / kQThreads;
  const int grid = (int)(want < (int64_t)sms_cache[dev] * 8 ? want : (int64_t)sms_cache[dev] * 8);
  quantize_mxfp4_kernel<<<grid, kQThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float4 *>(x), groups, reinterpret_cast<uint32_t *>(codes), scales);
  count_launches(1);
  return check_launch("quantize_mxfp4_kernel");
}
