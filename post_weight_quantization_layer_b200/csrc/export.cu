// Checkpoint export of one quantized linear: half-precision scales and packed zero points.
//
// Source: "AutoGPTQ 官方示例全解析" §1.4 and "OLMo 仓库中的 AutoGPTQ 快速上手" §四 第4步 —
// save_quantized writes the quantized weights (gptq_model-{bits}bit-{group_size}g, .bin or
// .safetensors) beside quantize_config.json.  The pages name the stored pieces only as
// "INT4 + scale + zero_point"; this library stores, per linear:
//   qweight [n_in*bits/32, n_out] int32 (the sweep's own packed codes, unchanged),
//   qzeros  [G, n_out*bits/32] int32: for each group the zero points of the output channels
//           form an LSB-first stream of bits-wide fields cut into 32-bit words (the same
//           packing as qweight, along n_out instead of n_in; 3-bit fields straddle words),
//   scales  [G, n_out] fp16 (round to nearest even from the fp32 scales),
//   g_idx   [n_in] int32 (unchanged).
#include <algorithm>

#include "common.cuh"

namespace gptq {
namespace {

// One thread per output word: word w of group g holds bits [32w, 32w + 32) of that group's
// stream of zero points.
__global__ void pack_zeros_kernel(const int32_t* __restrict__ zeros, int64_t G, int64_t n_out, int bits,
                                  int32_t* __restrict__ qzeros) {
  const int64_t nw = n_out * bits / 32;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t g = blockIdx.y;
  if (w >= nw || g >= G) return;
  const int64_t bit0 = w * 32;
  const int64_t ofirst = bit0 / bits, olast = (bit0 + 31) / bits;
  const uint32_t mask = (1u << bits) - 1u;
  uint32_t acc = 0u;
  for (int64_t o = ofirst; o <= olast && o < n_out; ++o) {
    const uint32_t v = static_cast<uint32_t>(zeros[g * n_out + o]) & mask;
    const int shift = static_cast<int>(o * bits - bit0);
    acc |= shift >= 0 ? (shift < 32 ? (v << shift) : 0u) : (v >> (-shift));
  }
  qzeros[g * nw + w] = static_cast<int32_t>(acc);
}

__global__ void scales_to_half_kernel(const float* __restrict__ s, int64_t count, __half* __restrict__ out) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = __float2half_rn(s[i]);
}

}  // namespace
}  // namespace gptq

using namespace gptq;

extern "C" int gptq_export_layer(const float* scales, const int32_t* zeros, int64_t groups, int64_t n_out, int bits,
                                 uint16_t* scales_f16, int32_t* qzeros, void* stream) {
  if (!scales || !zeros || !scales_f16 || !qzeros) return GPTQ_ERR_INVALID_ARG;
  if (groups <= 0 || n_out <= 0) return GPTQ_ERR_INVALID_ARG;
  if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return GPTQ_ERR_INVALID_ARG;
  if ((n_out * bits) % 32 != 0 || groups > 65535) return GPTQ_ERR_UNSUPPORTED;
  if (!aligned16(scales) || !aligned16(zeros) || !aligned16(scales_f16) || !aligned16(qzeros))
    return GPTQ_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t nw = n_out * bits / 32;
  const dim3 zgrid(static_cast<unsigned>((nw + 127) / 128), static_cast<unsigned>(groups));
  pack_zeros_kernel<<<zgrid, 128, 0, s>>>(zeros, groups, n_out, bits, qzeros);
  GPTQ_TRY(after_launch());
  const int64_t count = groups * n_out;
  const unsigned sgrid = static_cast<unsigned>(std::min<int64_t>((count + 255) / 256, 4 * 148));
  scales_to_half_kernel<<<sgrid, 256, 0, s>>>(scales, count, reinterpret_cast<__half*>(scales_f16));
  return after_launch();
}
