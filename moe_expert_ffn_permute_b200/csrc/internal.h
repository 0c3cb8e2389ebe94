// internal.h -- plan object, workspace layout and kernel launchers shared by the
// translation units of the MoE library (not part of the public ABI).
#pragma once
#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/moe.h"

namespace moe {

constexpr int kRouteChunk = 2048;   // slots per routing block
constexpr int kRouteThreads = 256;
constexpr int kTileM = 128;          // rows per m-tile (expert blocks are padded to it)

// Token scale chunks (the gathered x's and the FC1 activation's 1x128 UE8M0
// scales, laid out for tcgen05.cp ...32x128b.warpx4): one 512-byte chunk per
// 128-row tile and group of kSfGroup consecutive 128-wide k-blocks.  Row r's
// scale for k-block kb is the byte at chunk kb / kSfGroup, offset
// (r % 32) * 16 + (r / 32) * 4 + kb % kSfGroup.  A 1x128 scale is the same for
// the four 32-wide K steps of its k-block, so the MMAs of k-block kb all read
// byte kb % 4 (the scale-factor id) and one TMEM copy serves four k-blocks.
constexpr int kSfGroup = 4;
__host__ __device__ constexpr int sf_groups(int k_blocks) {
  return (k_blocks + kSfGroup - 1) / kSfGroup;
}
__host__ __device__ constexpr int sf_byte(int r, int kb) {
  return (kb / kSfGroup) * 512 + (r & 31) * 16 + (r >> 5) * 4 + kb % kSfGroup;
}

// Byte offsets of every buffer inside the caller's workspace (256-B aligned).
struct WorkspaceLayout {
  size_t err, counts, offsets, pad_off, tile_off, pair_off;
  size_t block_hist;
  size_t sched;             // fused-GEMM tile counter + per-m-tile FC1 completion counts
  size_t perm, inv;
  size_t row_token;         // padded row -> token index (-1 for padding rows)
  size_t xg, xg_sf;         // gathered x (expert order, padded) + its scale chunks
  size_t act, act_sf;       // FC1 output: FP8 activation + scale chunks
  size_t act_f32;           // debug capture (0 bytes when off)
  size_t y;                 // FC2 output, bf16, slot order
  size_t pair_sf1, pair_sf2;   // weight scales expanded for the CTA-pair GEMM (FP8 plans)
  // Two staging sets for the host-buffer entries (moe_forward_hostio uses set
  // 0; moe_forward_hostio_batches alternates between them): inputs and output.
  size_t in_x[2], in_xs[2], in_idx[2], in_w[2];
  size_t out_stage[2];
  size_t total;
};

}  // namespace moe

struct moe_plan_s {
  int T, H, I, E, k;
  int w_dtype;
  moe_act_params act;
  int debug_act_f32;
  int debug_fault;       // test hook: the fused GEMM's FC2 dependency can never be met
  int w_tiled;           // weights given as tiles (moe_prepack_weights): FP8 / BF16
                         // pre-swizzled 16 KB tiles, E2M1 plain 8 KB tiles
  int w_sf_chunked;      // MXFP4 scales given in 512-byte chunks (moe_prepack_weight_scales)
  int pair_mode;         // 2-SM GEMM: 0 automatic, 1 never, 2 always
  int swap_mode;         // token-major MMAs: 0 automatic, 1 never, 2 always
  int wide_mode;         // wide token-major tiles (two m-tiles): 0 automatic, 1 never, 2 always
  // Copy streams and events of moe_forward_hostio_batches, created on its
  // first call on a device (io_device = that device, -1 before).
  int io_device;
  cudaStream_t io_h2d, io_d2h;
  cudaEvent_t io_entry, io_in[2], io_done[2], io_out[2];
  long long S;           // T*k
  long long rows_cap;    // padded row capacity (multiple of 128)
  int route_blocks;
  moe::WorkspaceLayout ws;
};

namespace moe {

void compute_layout(moe_plan_s* p);
int use_swap(const moe_plan_s* p);    // token-major (swap-AB) MMAs: 0 never, 1 all, 2 by tile
int use_wide(const moe_plan_s* p);    // 1: the GEMM kernel with wide token-major tiles

// Launch with programmatic stream serialization: the kernel may start while its
// predecessor in the stream finishes; it must execute griddep_wait() before
// touching memory the predecessor writes or reads.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Launch without attributes.  Returns this launch's own status: unlike
// cudaGetLastError() after a <<<>>> launch, it neither reports nor clears an
// error left behind by some earlier, unrelated launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_plain(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                         cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = nullptr;
  cfg.numAttrs = 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Streaming multiprocessors of the current device (looked up once per device;
// thread-safe).
int sm_count();
// Raise a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per (kernel, device); thread-safe.
cudaError_t ensure_max_dynamic_smem(const void* kernel, int bytes);

// Kernel launchers (each returns the status of its own launches).
cudaError_t launch_route(const moe_plan_s* p, const int32_t* topk_idx, uint8_t* ws,
                         cudaStream_t st);
// Routing and gather fused in one launch (slot counts up to kFusedMaxSlots).
constexpr int kFusedMaxSlots = 4096;
cudaError_t launch_route_gather(const moe_plan_s* p, const int32_t* topk_idx, const uint8_t* x,
                                const uint8_t* xs, uint8_t* ws, cudaStream_t st);
// MXFP4 weight scales [rows, K/32] -> 512-byte tensor-core chunks.
cudaError_t launch_prepack_fp4_scales(const uint8_t* src, long long rows, int K, uint8_t* dst,
                                      cudaStream_t st);
cudaError_t launch_gather(const moe_plan_s* p, const uint8_t* x, const uint8_t* xs, uint8_t* ws,
                          cudaStream_t st);
cudaError_t launch_fc1(const moe_plan_s* p, const void* w1, const uint8_t* w1s, uint8_t* ws,
                       cudaStream_t st);
cudaError_t launch_fc2(const moe_plan_s* p, const void* w2, const uint8_t* w2s, uint8_t* ws,
                       cudaStream_t st);
// FC1 and FC2 in one persistent launch (dynamic tile scheduler).
cudaError_t launch_fc12(const moe_plan_s* p, const void* w1, const uint8_t* w1s, const void* w2,
                        const uint8_t* w2s, uint8_t* ws, cudaStream_t st);
// The same on CTA pairs with the 2-SM MMA (FP8, tiled weights only).
cudaError_t launch_fc12_pairs(const moe_plan_s* p, const void* w1, const uint8_t* w1s,
                              const void* w2, const uint8_t* w2s, uint8_t* ws, cudaStream_t st);
cudaError_t launch_combine(const moe_plan_s* p, const float* topk_w, void* out, uint8_t* ws,
                           cudaStream_t st);
cudaError_t launch_unpack_act(const moe_plan_s* p, const uint8_t* ws, uint8_t* dst,
                              cudaStream_t st);
cudaError_t launch_prepack(const uint8_t* src, long long rows, int K, uint8_t* dst,
                           cudaStream_t st);
// Packed E2M1 weights [rows, row_bytes] -> 8 KB tiles of 128 rows x 64 bytes.
cudaError_t launch_prepack_fp4(const uint8_t* src, long long rows, int row_bytes, uint8_t* dst,
                               cudaStream_t st);
cudaError_t launch_unpack_act_scales(const moe_plan_s* p, const uint8_t* ws, uint8_t* dst,
                                     cudaStream_t st);

}  // namespace moe
