// layout.cu -- conversions between row-major operands and the layouts the
// grouped GEMMs stream with linear bulk copies: pre-swizzled tiles (a 128-row x
// 128-byte tile is 16 KB, tiles ordered [row block][k-block], and byte c of row
// r sits at r * 128 + (((c / 16) ^ (r % 8)) * 16) + c % 16), and MXFP4 weight
// scales in the tensor core's 512-byte scale chunks.
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

// Packed E2M1 weights [rows, row_bytes] -> tiles of 128 rows x 64 bytes (128
// codes of one k-block per row), 8 KB each, tile (b, kb) at (b * row_bytes/64 +
// kb) * 8192, row r of the tile at r * 64 -- contiguous in HBM, so that one
// k-block of 128 weight rows is a single 8 KB stream; the tensor map that
// reads it widens the codes into the tensor core's padded shared-memory
// layout.  One thread per 16-byte chunk.
__global__ void __launch_bounds__(256) prepack_fp4_kernel(const uint4* __restrict__ src,
                                                          long long rows, int row_bytes,
                                                          uint8_t* __restrict__ dst) {
  const int vec = row_bytes / 16;
  const int kb_n = row_bytes / 64;
  const long long n = rows * vec;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / vec;
    const int c = static_cast<int>(i - row * vec);
    const long long rb = row / 128;
    const int r = static_cast<int>(row - rb * 128);
    uint8_t* d = dst + (rb * kb_n + (c >> 2)) * 8192ll + r * 64 + (c & 3) * 16;
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

// MXFP4 weight scales [rows, K/32] (four bytes per row per 128-wide k-block)
// -> chunks: for row block b and k-block kb, 512 bytes at (b * K/128 + kb) * 512
// holding row r's four bytes at (r % 32) * 16 + (r / 32) * 4 -- the layout the
// tensor core's scale copy (32x128b.warpx4) reads.  One thread per 4-byte word.
__global__ void __launch_bounds__(256) prepack_fp4_scales_kernel(
    const uint32_t* __restrict__ src, long long rows, int kb_n, uint8_t* __restrict__ dst) {
  const long long n = rows * kb_n;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = i / kb_n;
    const int kb = static_cast<int>(i - row * kb_n);
    const long long b = row / 128;
    const int r = static_cast<int>(row - b * 128);
    *reinterpret_cast<uint32_t*>(dst + (b * kb_n + kb) * 512 + (r & 31) * 16 + (r >> 5) * 4) =
        __ldg(&src[i]);
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
  return launch_plain(prepack_kernel, dim3(blocks_for(n)), dim3(256), 0, st,
                      reinterpret_cast<const uint4*>(src), rows, K, dst);
}

cudaError_t launch_prepack_fp4(const uint8_t* src, long long rows, int row_bytes, uint8_t* dst,
                               cudaStream_t st) {
  const long long n = rows * (row_bytes / 16);
  return launch_plain(prepack_fp4_kernel, dim3(blocks_for(n)), dim3(256), 0, st,
                      reinterpret_cast<const uint4*>(src), rows, row_bytes, dst);
}

cudaError_t launch_prepack_fp4_scales(const uint8_t* src, long long rows, int K, uint8_t* dst,
                                      cudaStream_t st) {
  const int kb_n = K / 128;
  return launch_plain(prepack_fp4_scales_kernel, dim3(blocks_for(rows * kb_n)), dim3(256), 0, st,
                      reinterpret_cast<const uint32_t*>(src), rows, kb_n, dst);
}

cudaError_t launch_unpack_act(const moe_plan_s* p, const uint8_t* ws, uint8_t* dst,
                              cudaStream_t st) {
  const int row_bytes = p->I * (p->w_dtype == MOE_W_BF16 ? 2 : 1);
  const long long n = p->rows_cap * (row_bytes / 16);
  return launch_plain(unpack_kernel, dim3(blocks_for(n)), dim3(256), 0, st,
                      static_cast<const uint8_t*>(ws + p->ws.act), p->rows_cap, row_bytes,
                      reinterpret_cast<uint4*>(dst));
}

}  // namespace moe
