// combine.cu -- step 4, the direct weighted top-k combine back to token order
// (DeepGEMM PR #386 "Optimize sm100 version with token-aware BM240 tiling,
// native UE8M0, and direct combine", title):
//   out[t, c] = bf16( sum_{j=0}^{k-1} topk_w[t, j] * y[t*k + j, c] )
// summed in fp32 with j ascending (deterministic).  A slot whose expert id was
// out of range (inv[s] < 0) contributes nothing.  HBM-bound: each thread reads
// 2k 16-byte vectors of y and writes two 16-byte vectors of out.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int kMaxK = 8;   // slots per group of loads (larger k loops over groups)
// Each thread owns two 16-byte chunks of the token's row, c and c + H/16 (one
// in each half of the row): twice the loads in flight per thread of a
// one-chunk thread (k rows x 2 x 16 bytes), which the streaming read of y
// needs to approach the copy bandwidth at large token counts.
constexpr int kCpt = 2;

__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y,
                                                      const float* __restrict__ topk_w,
                                                      const int32_t* __restrict__ inv, int T,
                                                      int H, int k, uint16_t* __restrict__ out) {
  griddep_launch_dependents();
  griddep_wait();
  const int vecs = H / 8;
  const int half = vecs / kCpt;
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (i >= static_cast<long long>(T) * half) return;
  const int t = static_cast<int>(i / half);
  const int c = static_cast<int>(i - static_cast<long long>(t) * half);
  float acc[kCpt][8];
#pragma unroll
  for (int h = 0; h < kCpt; ++h)
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[h][q] = 0.0f;
  for (int j0 = 0; j0 < k; j0 += kMaxK) {
    // Issue every load of this group before using any: the routing check, the
    // weight and the y vectors of a slot are independent loads (a slot that
    // was not routed has a y row too, of stale bytes, which are never used).
    int iv[kMaxK];
    float w[kMaxK];
    uint4 v[kMaxK][kCpt];
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      const long long s = static_cast<long long>(t) * k + j0 + j;
      const bool in = j0 + j < k;
      iv[j] = in ? __ldg(&inv[s]) : -1;
      w[j] = in ? __ldg(&topk_w[s]) : 0.0f;
#pragma unroll
      for (int h = 0; h < kCpt; ++h)
        v[j][h] = in ? __ldcs(reinterpret_cast<const uint4*>(y + s * H) + c + h * half)
                     : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j0 + j >= k) break;
      if (iv[j] < 0) continue;
#pragma unroll
      for (int h = 0; h < kCpt; ++h) {
        const uint32_t wv[4] = {v[j][h].x, v[j][h].y, v[j][h].z, v[j][h].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float lo = __uint_as_float(wv[q] << 16);
          const float hi = __uint_as_float(wv[q] & 0xFFFF0000u);
          acc[h][2 * q] = fmaf(w[j], lo, acc[h][2 * q]);
          acc[h][2 * q + 1] = fmaf(w[j], hi, acc[h][2 * q + 1]);
        }
      }
    }
  }
#pragma unroll
  for (int h = 0; h < kCpt; ++h) {
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __nv_bfloat162 b = __floats2bfloat162_rn(acc[h][2 * q], acc[h][2 * q + 1]);
      o[q] = *reinterpret_cast<uint32_t*>(&b);
    }
    reinterpret_cast<uint4*>(out + static_cast<long long>(t) * H)[c + h * half] =
        make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

cudaError_t launch_combine(const moe_plan_s* p, const float* topk_w, void* out, uint8_t* ws,
                           cudaStream_t st) {
  const long long n = static_cast<long long>(p->T) * (p->H / 8 / kCpt);
  const int blocks = static_cast<int>((n + 255) / 256);
  return launch_pdl(combine_kernel, dim3(blocks), dim3(256), 0, st,
                    reinterpret_cast<const uint16_t*>(ws + p->ws.y), topk_w,
                    reinterpret_cast<const int32_t*>(ws + p->ws.inv), p->T, p->H, p->k,
                    reinterpret_cast<uint16_t*>(out));
}

}  // namespace moe
