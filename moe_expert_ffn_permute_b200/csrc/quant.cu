// quant.cu -- the step before the layer: bf16 activations -> E4M3 codes with one
// UE8M0 scale per 1x128 block (the layer's input format).  Same rule as the
// FC1 epilogue's requantisation (TensorRT-LLM PR #16346 "DSV4 o_proj: fuse
// fp8/UE8M0 quantize ...", Description: BF16 -> FP8 + 1x128 UE8M0 from the
// block amax): n = smallest integer with max(amax, 1e-4) <= 448 * 2^n, codes =
// round-to-nearest-even, saturating E4M3 of x / 2^n, scale byte n + 127.
// HBM-bound: 2 bytes read + 1 + 1/128 bytes written per element.
#include <cuda_runtime.h>

#include "internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

// 16 lanes per 128-wide block, 8 elements (16 bytes) per lane.
__global__ void __launch_bounds__(256) quantize_kernel(const uint4* __restrict__ x,
                                                       long long blocks,
                                                       uint2* __restrict__ codes,
                                                       uint8_t* __restrict__ scales) {
  const long long gid = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  const long long blk = gid >> 4;
  const bool live = blk < blocks;
  uint4 v = make_uint4(0, 0, 0, 0);
  if (live) v = __ldcs(&x[gid]);
  float f[8];
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float amax = 0.0f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    f[2 * q] = __uint_as_float(w[q] << 16);
    f[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
    amax = fmaxf(amax, fmaxf(fabsf(f[2 * q]), fabsf(f[2 * q + 1])));
  }
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1)
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if (!live) return;
  const int n = ue8m0_exponent(amax);
  const float inv_scale = __uint_as_float(static_cast<uint32_t>(127 - n) << 23);
  uint32_t lo = 0, hi = 0;
  lo = cvt_e4m3x2(f[0] * inv_scale, f[1] * inv_scale) |
       (static_cast<uint32_t>(cvt_e4m3x2(f[2] * inv_scale, f[3] * inv_scale)) << 16);
  hi = cvt_e4m3x2(f[4] * inv_scale, f[5] * inv_scale) |
       (static_cast<uint32_t>(cvt_e4m3x2(f[6] * inv_scale, f[7] * inv_scale)) << 16);
  codes[gid] = make_uint2(lo, hi);
  if ((threadIdx.x & 15) == 0) scales[blk] = static_cast<uint8_t>(n + 127);
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_quantize_act(const void* x_bf16, int T, int H, uint8_t* x_codes,
                                       uint8_t* x_scales, moe_stream_t stream) {
  if (x_bf16 == nullptr || x_codes == nullptr || x_scales == nullptr) return MOE_ERR_INVALID_ARG;
  if (T < 1 || H < 1) return MOE_ERR_INVALID_ARG;
  if (H % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(x_bf16) % 16 != 0 || reinterpret_cast<uintptr_t>(x_codes) % 8 != 0)
    return MOE_ERR_ALIGNMENT;
  const long long blocks = static_cast<long long>(T) * (H / 128);
  const long long threads = blocks * 16;
  const int grid = static_cast<int>((threads + 255) / 256);
  const cudaError_t e = moe::launch_plain(
      moe::quantize_kernel, dim3(grid), dim3(256), 0, reinterpret_cast<cudaStream_t>(stream),
      static_cast<const uint4*>(x_bf16), blocks, reinterpret_cast<uint2*>(x_codes), x_scales);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
