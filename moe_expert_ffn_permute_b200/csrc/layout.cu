// layout.cu -- conversions between row-major operands and the pre-swizzled
// tile layout the grouped GEMMs stream with linear bulk copies: a 128-row x
// 128-byte tile is 16 KB, tiles ordered [row block][k-block], and byte c of
// row r sits at r * 128 + (((c / 16) ^ (r % 8)) * 16) + c % 16.
#include <cuda_runtime.h>

#include "internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

// Row-major [rows, K] bytes -> tiles.  One thread per 16-byte chunk; reads are
// coalesced along rows.
__global__ void __launch_bounds__(256) prepack_kernel(const uint4* __restrict__ src, long long rows,
                                                      int K, uint8_t* __restrict__ dst) {
  const int vec = K / 16;
  const int kb_n = K / 128;
  const long long n = rows * vec;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / vec;
    const int c = static_cast<int>(i - row * vec);
    const long long rb = row / 128;
    const int r = static_cast<int>(row - rb * 128);
    uint8_t* d = dst + (rb * kb_n + (c >> 3)) * static_cast<long long>(kTileBytes) + swz128(r, c & 7);
    *reinterpret_cast<uint4*>(d) = __ldg(&src[i]);
  }
}

// Tiles -> row-major (inspection of the FC1 activation).
__global__ void __launch_bounds__(256) unpack_kernel(const uint8_t* __restrict__ src, long long rows,
                                                     int K, uint4* __restrict__ dst) {
  const int vec = K / 16;
  const int kb_n = K / 128;
  const long long n = rows * vec;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / vec;
    const int c = static_cast<int>(i - row * vec);
    const long long rb = row / 128;
    const int r = static_cast<int>(row - rb * 128);
    dst[i] = *reinterpret_cast<const uint4*>(
        src + (rb * kb_n + (c >> 3)) * static_cast<long long>(kTileBytes) + swz128(r, c & 7));
  }
}

int blocks_for(long long n) {
  const long long b = (n + 255) / 256;
  return static_cast<int>(b < 148 * 16 ? b : 148 * 16);
}

}  // namespace

cudaError_t launch_prepack(const uint8_t* src, long long rows, int K, uint8_t* dst,
                           cudaStream_t st) {
  const long long n = rows * (K / 16);
  prepack_kernel<<<blocks_for(n), 256, 0, st>>>(reinterpret_cast<const uint4*>(src), rows, K, dst);
  return cudaGetLastError();
}

cudaError_t launch_unpack_act(const moe_plan_s* p, const uint8_t* ws, uint8_t* dst,
                              cudaStream_t st) {
  const int row_bytes = p->I * (p->w_dtype == MOE_W_BF16 ? 2 : 1);
  const long long n = p->rows_cap * (row_bytes / 16);
  unpack_kernel<<<blocks_for(n), 256, 0, st>>>(ws + p->ws.act, p->rows_cap, row_bytes,
                                               reinterpret_cast<uint4*>(dst));
  return cudaGetLastError();
}

}  // namespace moe
