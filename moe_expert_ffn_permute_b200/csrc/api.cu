// api.cu -- the C ABI (include/moe.h): plan construction and validation,
// workspace layout, and the stream-ordered launch sequence of the layer.
#include <cmath>
#include <cstring>
#include <mutex>
#include <new>
#include <utility>
#include <vector>

#include "internal.h"

namespace moe {

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_device_mu;
int g_sm_count[kMaxDevices] = {};
std::vector<std::pair<const void*, int>> g_smem_set;   // (kernel, device) done
}  // namespace

int sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lock(g_device_mu);
  if (g_sm_count[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

cudaError_t ensure_max_dynamic_smem(const void* kernel, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_device_mu);
  for (const auto& kd : g_smem_set)
    if (kd.first == kernel && kd.second == dev) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) g_smem_set.emplace_back(kernel, dev);
  return e;
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

void compute_layout(moe_plan_s* p) {
  WorkspaceLayout& L = p->ws;
  const size_t S = static_cast<size_t>(p->S);
  const size_t E = static_cast<size_t>(p->E);
  const size_t rows = static_cast<size_t>(p->rows_cap);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L.err = take(256);
  L.counts = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.pad_off = take((E + 1) * 4);
  L.tile_off = take((E + 1) * 4);
  L.pair_off = take((E + 1) * 4);
  L.block_hist = take(static_cast<size_t>(p->route_blocks) * E * 4);
  L.sched = take(256 + rows / kTileM * 4);
  L.perm = take(S * 4);
  L.inv = take(S * 4);
  L.row_token = take(rows * 4);
  // BF16 plans keep 2-byte activations and no scale chunks.
  const bool bf16 = p->w_dtype == MOE_W_BF16;
  const size_t elem = bf16 ? 2 : 1;
  L.xg = take(rows * p->H * elem);
  L.xg_sf = take(bf16 ? 0 : rows / kTileM * sf_groups(p->H / 128) * 512);
  L.act = take(rows * p->I * elem);
  L.act_sf = take(bf16 ? 0 : rows / kTileM * sf_groups(p->I / 128) * 512);
  L.y = take(S * p->H * 2);
  // One 1 KB record per (expert, n-tile, k-block) of each GEMM: the two 128-row
  // weight blocks of a 256-wide tile, each block's scale byte repeated 512 times.
  const bool fp8 = p->w_dtype == MOE_W_E4M3_UE8M0_128x128;
  L.pair_sf1 = take(fp8 ? E * (p->I / 128) * (p->H / 128) * 1024 : 0);
  L.pair_sf2 = take(fp8 ? E * (p->H / 256) * (p->I / 128) * 1024 : 0);
  for (int b = 0; b < 2; ++b) {
    L.in_x[b] = take(static_cast<size_t>(p->T) * p->H * elem);
    L.in_xs[b] = take(bf16 ? 0 : static_cast<size_t>(p->T) * (p->H / 128));
    L.in_idx[b] = take(S * 4);
    L.in_w[b] = take(S * 4);
    L.out_stage[b] = take(static_cast<size_t>(p->T) * p->H * 2);
  }
  // Debug capture last: switching it on or off moves no other buffer.
  L.act_f32 = take(p->debug_act_f32 ? rows * p->I * 4 : 0);
  L.total = off;
}

}  // namespace moe

using moe::kTileM;

static bool aligned(const void* p, size_t a) {
  return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

static moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// 2-SM GEMM: needs tiled FP8 weights and is used only when asked for (mode
// 2).  Automatic mode keeps the single-CTA kernel: at 8192 tokens of the
// 7168 x 2048 x 32-expert layer both run power-capped and the pair kernel
// measured no faster.
static bool use_pairs(const moe_plan_s* p) {
  if (!p->w_tiled || p->w_dtype != MOE_W_E4M3_UE8M0_128x128) return false;
  return p->pair_mode == 2;
}

namespace moe {
// Token-major (swap-AB) MMAs: the MMAs used here have M = 128, so a tile with
// few token rows computes mostly padding; with the weights as A and the tile's
// tokens as B (N = their count rounded up to 16) the tensor work follows the
// tokens.  Returns the kernel's mode: 0 never (mode 1, or CTA pairs), 1 every
// tile (mode 2), 2 tile by tile from its row count (mode 0, automatic).
int use_swap(const moe_plan_s* p) {
  if (use_pairs(p) || p->swap_mode == 1) return 0;
  return p->swap_mode == 2 ? 1 : 2;
}

// Wide token-major tiles (up to 240 tokens of two consecutive m-tiles of one
// expert in one tile): they need token-major MMAs and halve the weight stream
// of experts with 129..240 tokens.  Measured (same box, wide on vs off):
// MXFP4 weights gain 12% at 128 and 15% at 192 slots per expert and lose 7% at
// 96; FP8 and BF16 weights lose 7-14% at 128-192 (their pre-swizzled weight
// tiles are cheap bulk copies, so the wide kernel's three stages and longer
// epilogue outweigh the halved stream).  Automatic mode: MXFP4 weights with
// 96 < S/E <= 224 slots per expert.
int use_wide(const moe_plan_s* p) {
  if (use_swap(p) == 0 || p->wide_mode == 1) return 0;
  if (p->wide_mode == 2) return 1;
  if (p->w_dtype != MOE_W_E2M1_UE8M0_1x32) return 0;
  const long long per_expert = p->S / p->E;
  return per_expert > 96 && per_expert <= 224 ? 1 : 0;
}
}  // namespace moe

static moe_status check_ws(moe_plan_t plan, const void* workspace) {
  if (plan == nullptr) return MOE_ERR_INVALID_ARG;
  if (workspace == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

// x_scales is required except for BF16 plans (BF16 activations carry no scales).
static bool x_scales_ok(moe_plan_t plan, const uint8_t* x_scales) {
  return x_scales != nullptr || plan->w_dtype == MOE_W_BF16;
}

static moe_status check_weights(moe_plan_t plan, const void* w, const uint8_t* ws) {
  if (w == nullptr) return MOE_ERR_INVALID_ARG;
  if (ws == nullptr && plan->w_dtype != MOE_W_BF16) return MOE_ERR_INVALID_ARG;
  const size_t wa = plan->w_dtype == MOE_W_E2M1_UE8M0_1x32 ? 32 : 16;
  if (!aligned(w, wa)) return MOE_ERR_ALIGNMENT;
  if (plan->w_dtype == MOE_W_E2M1_UE8M0_1x32 && !aligned(ws, plan->w_sf_chunked ? 16 : 4))
    return MOE_ERR_ALIGNMENT;
  return MOE_OK;
}

extern "C" {

moe_status moe_plan(int T, int H, int I, int E, int k, moe_dtypes dtypes, moe_act_params act,
                    moe_plan_t* out) {
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (T < 1 || H < 1 || I < 1 || k < 1 || E < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (E > 256) return MOE_ERR_UNSUPPORTED;
  if (H % 128 != 0 || I % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (H % 256 != 0) return MOE_ERR_UNSUPPORTED;   // FC2 tiles are 256 columns wide
  if (static_cast<long long>(T) * k >= (1ll << 31)) return MOE_ERR_INVALID_ARG;
  if (dtypes.w_dtype != MOE_W_E4M3_UE8M0_128x128 && dtypes.w_dtype != MOE_W_E2M1_UE8M0_1x32 &&
      dtypes.w_dtype != MOE_W_BF16)
    return MOE_ERR_INVALID_ARG;
  if (act.kind != MOE_ACT_SWIGLU && act.kind != MOE_ACT_SWIGLU_OAI) return MOE_ERR_INVALID_ARG;
  if (act.kind == MOE_ACT_SWIGLU_OAI) {
    if (!(act.limit > 0.0f) || std::isnan(act.alpha) || std::isnan(act.up_bias) ||
        std::isinf(act.alpha) || std::isinf(act.up_bias))
      return MOE_ERR_INVALID_ARG;
  } else {
    act.alpha = 1.0f;
    act.up_bias = 0.0f;
    act.limit = INFINITY;
  }
  moe_plan_s* p = new (std::nothrow) moe_plan_s();
  if (p == nullptr) return MOE_ERR_INVALID_ARG;
  p->T = T;
  p->H = H;
  p->I = I;
  p->E = E;
  p->k = k;
  p->w_dtype = dtypes.w_dtype;
  p->act = act;
  p->debug_act_f32 = 0;
  p->debug_fault = 0;
  p->w_tiled = 0;
  p->w_sf_chunked = 0;
  p->pair_mode = 0;
  p->swap_mode = 0;
  p->wide_mode = 0;
  p->io_device = -1;
  p->S = static_cast<long long>(T) * k;
  // Sum over experts of ceil(n_e / 128) <= floor((S + 127 E) / 128).
  p->rows_cap = ((p->S + 127ll * E) / kTileM) * kTileM;
  if (p->rows_cap < kTileM) p->rows_cap = kTileM;
  p->route_blocks = static_cast<int>((p->S + moe::kRouteChunk - 1) / moe::kRouteChunk);
  moe::compute_layout(p);
  *out = p;
  return MOE_OK;
}

static void release_io(moe_plan_s* p);

void moe_plan_destroy(moe_plan_t plan) {
  if (plan == nullptr) return;
  release_io(plan);
  delete plan;
}

size_t moe_workspace_bytes(moe_plan_t plan) { return plan ? plan->ws.total : 0; }

moe_status moe_plan_set_weight_layout(moe_plan_t plan, int layout) {
  if (plan == nullptr) return MOE_ERR_INVALID_ARG;
  if (layout != MOE_WEIGHTS_ROW_MAJOR && layout != MOE_WEIGHTS_TILED &&
      layout != MOE_WEIGHTS_SCALES_CHUNKED && layout != MOE_WEIGHTS_TILED_SCALES_CHUNKED)
    return MOE_ERR_INVALID_ARG;
  const bool fp4 = plan->w_dtype == MOE_W_E2M1_UE8M0_1x32;
  if (layout == MOE_WEIGHTS_TILED && fp4) return MOE_ERR_UNSUPPORTED;
  if ((layout == MOE_WEIGHTS_SCALES_CHUNKED || layout == MOE_WEIGHTS_TILED_SCALES_CHUNKED) &&
      !fp4)
    return MOE_ERR_UNSUPPORTED;
  plan->w_tiled = (layout == MOE_WEIGHTS_TILED || layout == MOE_WEIGHTS_TILED_SCALES_CHUNKED);
  plan->w_sf_chunked =
      (layout == MOE_WEIGHTS_SCALES_CHUNKED || layout == MOE_WEIGHTS_TILED_SCALES_CHUNKED);
  return MOE_OK;
}

moe_status moe_prepack_weight_scales(moe_plan_t plan, const uint8_t* w1_scales,
                                     const uint8_t* w2_scales, uint8_t* w1_scales_chunked,
                                     uint8_t* w2_scales_chunked, moe_stream_t stream) {
  if (plan == nullptr || w1_scales == nullptr || w2_scales == nullptr ||
      w1_scales_chunked == nullptr || w2_scales_chunked == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (plan->w_dtype != MOE_W_E2M1_UE8M0_1x32) return MOE_ERR_UNSUPPORTED;
  if (!aligned(w1_scales, 4) || !aligned(w2_scales, 4) || !aligned(w1_scales_chunked, 16) ||
      !aligned(w2_scales_chunked, 16))
    return MOE_ERR_ALIGNMENT;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  const long long E = plan->E;
  if (moe::launch_prepack_fp4_scales(w1_scales, E * 2 * plan->I, plan->H, w1_scales_chunked,
                                     st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return cuda_status(
      moe::launch_prepack_fp4_scales(w2_scales, E * plan->H, plan->I, w2_scales_chunked, st));
}

moe_status moe_plan_set_cta_pairs(moe_plan_t plan, int mode) {
  if (plan == nullptr || mode < 0 || mode > 2) return MOE_ERR_INVALID_ARG;
  if (mode == 2 && (!plan->w_tiled || plan->w_dtype != MOE_W_E4M3_UE8M0_128x128))
    return MOE_ERR_UNSUPPORTED;
  plan->pair_mode = mode;
  return MOE_OK;
}

moe_status moe_prepack_weights(moe_plan_t plan, const void* w1, const void* w2, void* w1_tiled,
                               void* w2_tiled, moe_stream_t stream) {
  if (plan == nullptr || w1 == nullptr || w2 == nullptr || w1_tiled == nullptr ||
      w2_tiled == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(w1, 16) || !aligned(w2, 16) || !aligned(w1_tiled, 16) || !aligned(w2_tiled, 16))
    return MOE_ERR_ALIGNMENT;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  const long long E = plan->E;
  if (plan->w_dtype == MOE_W_E2M1_UE8M0_1x32) {
    // E2M1 codes: 64-byte (128-element) k-blocks, 8 KB tiles of 128 rows.
    if (moe::launch_prepack_fp4(static_cast<const uint8_t*>(w1), E * 2 * plan->I, plan->H / 2,
                                static_cast<uint8_t*>(w1_tiled), st) != cudaSuccess)
      return MOE_ERR_CUDA;
    return cuda_status(moe::launch_prepack_fp4(static_cast<const uint8_t*>(w2), E * plan->H,
                                               plan->I / 2, static_cast<uint8_t*>(w2_tiled), st));
  }
  const int elem = plan->w_dtype == MOE_W_BF16 ? 2 : 1;   // bytes per weight
  if (moe::launch_prepack(static_cast<const uint8_t*>(w1), E * 2 * plan->I, plan->H * elem,
                          static_cast<uint8_t*>(w1_tiled), st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return cuda_status(moe::launch_prepack(static_cast<const uint8_t*>(w2), E * plan->H,
                                         plan->I * elem, static_cast<uint8_t*>(w2_tiled), st));
}

moe_status moe_copy_act(moe_plan_t plan, const void* workspace, uint8_t* dst,
                        moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if (dst == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(dst, 16)) return MOE_ERR_ALIGNMENT;
  return cuda_status(moe::launch_unpack_act(plan, static_cast<const uint8_t*>(workspace), dst,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_plan_set_debug(moe_plan_t plan, int flags) {
  if (plan == nullptr) return MOE_ERR_INVALID_ARG;
  if (flags & ~3) return MOE_ERR_INVALID_ARG;
  plan->debug_act_f32 = flags & 1;
  plan->debug_fault = (flags >> 1) & 1;
  moe::compute_layout(plan);
  return MOE_OK;
}

moe_status moe_plan_set_swap_ab(moe_plan_t plan, int mode) {
  if (plan == nullptr || mode < 0 || mode > 2) return MOE_ERR_INVALID_ARG;
  plan->swap_mode = mode;
  return MOE_OK;
}

int moe_plan_swap_ab_active(moe_plan_t plan) {
  return plan == nullptr ? 0 : moe::use_swap(plan);
}

moe_status moe_plan_set_wide_tiles(moe_plan_t plan, int mode) {
  if (plan == nullptr || mode < 0 || mode > 2) return MOE_ERR_INVALID_ARG;
  plan->wide_mode = mode;
  return MOE_OK;
}

int moe_plan_wide_tiles_active(moe_plan_t plan) {
  return plan == nullptr ? 0 : moe::use_wide(plan);
}

int moe_plan_cta_pairs_active(moe_plan_t plan) {
  return plan != nullptr && use_pairs(plan) ? 1 : 0;
}

int moe_forward_launch_count(moe_plan_t plan) {
  if (plan == nullptr) return 0;
  // Routing + gather (one launch up to kFusedMaxSlots slots; else [route
  // histogram,] route scan+scatter, gather), [pair scale expansion,] FC1+FC2
  // (one launch), combine.
  const int front = plan->S <= moe::kFusedMaxSlots ? 1 : (plan->route_blocks > 1 ? 3 : 2);
  return front + (use_pairs(plan) ? 1 : 0) + 2;
}

moe_status moe_route(moe_plan_t plan, const int32_t* topk_idx, void* workspace,
                     moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if (topk_idx == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(topk_idx, 4)) return MOE_ERR_ALIGNMENT;
  return cuda_status(moe::launch_route(plan, topk_idx, static_cast<uint8_t*>(workspace),
                                       reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_gather(moe_plan_t plan, const void* x, const uint8_t* x_scales, void* workspace,
                      moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if (x == nullptr || !x_scales_ok(plan, x_scales)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16)) return MOE_ERR_ALIGNMENT;
  return cuda_status(moe::launch_gather(plan, static_cast<const uint8_t*>(x), x_scales,
                                        static_cast<uint8_t*>(workspace),
                                        reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_route_gather(moe_plan_t plan, const int32_t* topk_idx, const void* x,
                            const uint8_t* x_scales, void* workspace, moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if (topk_idx == nullptr || x == nullptr || !x_scales_ok(plan, x_scales))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(topk_idx, 4) || !aligned(x, 16)) return MOE_ERR_ALIGNMENT;
  if (plan->S > moe::kFusedMaxSlots) {
    if ((s = moe_route(plan, topk_idx, workspace, stream)) != MOE_OK) return s;
    return moe_gather(plan, x, x_scales, workspace, stream);
  }
  return cuda_status(moe::launch_route_gather(plan, topk_idx, static_cast<const uint8_t*>(x),
                                              x_scales, static_cast<uint8_t*>(workspace),
                                              reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_fc1(moe_plan_t plan, const void* w1, const uint8_t* w1_scales, void* workspace,
                   moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if ((s = check_weights(plan, w1, w1_scales)) != MOE_OK) return s;
  return cuda_status(moe::launch_fc1(plan, w1, w1_scales, static_cast<uint8_t*>(workspace),
                                     reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_fc2(moe_plan_t plan, const void* w2, const uint8_t* w2_scales, void* workspace,
                   moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if ((s = check_weights(plan, w2, w2_scales)) != MOE_OK) return s;
  return cuda_status(moe::launch_fc2(plan, w2, w2_scales, static_cast<uint8_t*>(workspace),
                                     reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_fc1_fc2(moe_plan_t plan, const void* w1, const uint8_t* w1_scales, const void* w2,
                       const uint8_t* w2_scales, void* workspace, moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if ((s = check_weights(plan, w1, w1_scales)) != MOE_OK) return s;
  if ((s = check_weights(plan, w2, w2_scales)) != MOE_OK) return s;
  auto ws = static_cast<uint8_t*>(workspace);
  auto st = reinterpret_cast<cudaStream_t>(stream);
  if (use_pairs(plan))
    return cuda_status(moe::launch_fc12_pairs(plan, w1, w1_scales, w2, w2_scales, ws, st));
  return cuda_status(moe::launch_fc12(plan, w1, w1_scales, w2, w2_scales, ws, st));
}

moe_status moe_combine(moe_plan_t plan, const float* topk_w, void* out, void* workspace,
                       moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if (topk_w == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  if (!aligned(topk_w, 4) || !aligned(out, 16)) return MOE_ERR_ALIGNMENT;
  return cuda_status(moe::launch_combine(plan, topk_w, out, static_cast<uint8_t*>(workspace),
                                         reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_forward(moe_plan_t plan, const void* x, const uint8_t* x_scales,
                       const int32_t* topk_idx, const float* topk_w, const void* w1,
                       const uint8_t* w1_scales, const void* w2, const uint8_t* w2_scales,
                       void* out, void* workspace, moe_stream_t stream) {
  // Validate everything before the first launch.
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if (x == nullptr || !x_scales_ok(plan, x_scales) || topk_idx == nullptr || topk_w == nullptr ||
      out == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(topk_idx, 4) || !aligned(topk_w, 4) || !aligned(out, 16))
    return MOE_ERR_ALIGNMENT;
  if ((s = check_weights(plan, w1, w1_scales)) != MOE_OK) return s;
  if ((s = check_weights(plan, w2, w2_scales)) != MOE_OK) return s;
  if ((s = moe_route_gather(plan, topk_idx, x, x_scales, workspace, stream)) != MOE_OK) return s;
  // FC1 and FC2 share one persistent launch: FC2 tiles of an m-tile start as
  // soon as that m-tile's FC1 tiles are done (no wave tail between the GEMMs).
  if ((s = moe_fc1_fc2(plan, w1, w1_scales, w2, w2_scales, workspace, stream)) != MOE_OK)
    return s;
  return moe_combine(plan, topk_w, out, workspace, stream);
}

moe_status moe_forward_hostio(moe_plan_t plan, const void* x_host, const uint8_t* x_scales_host,
                              const int32_t* topk_idx_host, const float* topk_w_host,
                              const void* w1, const uint8_t* w1_scales, const void* w2,
                              const uint8_t* w2_scales, void* out_host, void* workspace,
                              moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if (x_host == nullptr || !x_scales_ok(plan, x_scales_host) || topk_idx_host == nullptr ||
      topk_w_host == nullptr || out_host == nullptr)
    return MOE_ERR_INVALID_ARG;
  if ((s = check_weights(plan, w1, w1_scales)) != MOE_OK) return s;
  if ((s = check_weights(plan, w2, w2_scales)) != MOE_OK) return s;
  auto ws = static_cast<uint8_t*>(workspace);
  auto st = reinterpret_cast<cudaStream_t>(stream);
  const auto& L = plan->ws;
  const size_t T = plan->T, H = plan->H, S = static_cast<size_t>(plan->S);
  const bool bf16 = plan->w_dtype == MOE_W_BF16;
  if (cudaMemcpyAsync(ws + L.in_x[0], x_host, T * H * (bf16 ? 2 : 1), cudaMemcpyHostToDevice, st) !=
          cudaSuccess ||
      (!bf16 && cudaMemcpyAsync(ws + L.in_xs[0], x_scales_host, T * (H / 128),
                                cudaMemcpyHostToDevice, st) != cudaSuccess) ||
      cudaMemcpyAsync(ws + L.in_idx[0], topk_idx_host, S * 4, cudaMemcpyHostToDevice, st) !=
          cudaSuccess ||
      cudaMemcpyAsync(ws + L.in_w[0], topk_w_host, S * 4, cudaMemcpyHostToDevice, st) !=
          cudaSuccess)
    return MOE_ERR_CUDA;
  uint8_t* out_dev = ws + L.out_stage[0];
  s = moe_forward(plan, ws + L.in_x[0], bf16 ? nullptr : ws + L.in_xs[0],
                  reinterpret_cast<const int32_t*>(ws + L.in_idx[0]),
                  reinterpret_cast<const float*>(ws + L.in_w[0]), w1, w1_scales, w2, w2_scales,
                  out_dev, workspace, stream);
  if (s != MOE_OK) return s;
  if (cudaMemcpyAsync(out_host, out_dev, T * H * 2, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

// Copy streams and events of the batched host-buffer entry, created on the
// first call on a device (a plan moved to another device gets new ones).
static void release_io(moe_plan_s* p) {
  if (p->io_device < 0) return;
  int cur = 0;
  const bool restore = cudaGetDevice(&cur) == cudaSuccess && cur != p->io_device;
  if (restore) cudaSetDevice(p->io_device);
  cudaStreamDestroy(p->io_h2d);
  cudaStreamDestroy(p->io_d2h);
  cudaEventDestroy(p->io_entry);
  for (int b = 0; b < 2; ++b) {
    cudaEventDestroy(p->io_in[b]);
    cudaEventDestroy(p->io_done[b]);
    cudaEventDestroy(p->io_out[b]);
  }
  if (restore) cudaSetDevice(cur);
  p->io_device = -1;
}

static cudaError_t ensure_io(moe_plan_s* p) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (p->io_device == dev) return cudaSuccess;
  release_io(p);
  const unsigned ev_flags = cudaEventDisableTiming;
  if ((e = cudaStreamCreateWithFlags(&p->io_h2d, cudaStreamNonBlocking)) != cudaSuccess) return e;
  if ((e = cudaStreamCreateWithFlags(&p->io_d2h, cudaStreamNonBlocking)) != cudaSuccess) {
    cudaStreamDestroy(p->io_h2d);
    return e;
  }
  cudaEvent_t* evs[7] = {&p->io_entry, &p->io_in[0], &p->io_in[1], &p->io_done[0],
                         &p->io_done[1], &p->io_out[0], &p->io_out[1]};
  for (int i = 0; i < 7; ++i) {
    if ((e = cudaEventCreateWithFlags(evs[i], ev_flags)) != cudaSuccess) {
      for (int j = 0; j < i; ++j) cudaEventDestroy(*evs[j]);
      cudaStreamDestroy(p->io_h2d);
      cudaStreamDestroy(p->io_d2h);
      return e;
    }
  }
  p->io_device = dev;
  return cudaSuccess;
}

moe_status moe_forward_hostio_batches(moe_plan_t plan, int n_batches,
                                      const void* const* x_host,
                                      const uint8_t* const* x_scales_host,
                                      const int32_t* const* topk_idx_host,
                                      const float* const* topk_w_host, const void* w1,
                                      const uint8_t* w1_scales, const void* w2,
                                      const uint8_t* w2_scales, void* const* out_host,
                                      void* workspace, moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if (n_batches < 1 || x_host == nullptr || topk_idx_host == nullptr ||
      topk_w_host == nullptr || out_host == nullptr)
    return MOE_ERR_INVALID_ARG;
  const bool bf16 = plan->w_dtype == MOE_W_BF16;
  if (!bf16 && x_scales_host == nullptr) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n_batches; ++i)
    if (x_host[i] == nullptr || (!bf16 && x_scales_host[i] == nullptr) ||
        topk_idx_host[i] == nullptr || topk_w_host[i] == nullptr || out_host[i] == nullptr)
      return MOE_ERR_INVALID_ARG;
  if ((s = check_weights(plan, w1, w1_scales)) != MOE_OK) return s;
  if ((s = check_weights(plan, w2, w2_scales)) != MOE_OK) return s;
  if (ensure_io(plan) != cudaSuccess) return MOE_ERR_CUDA;
  auto ws = static_cast<uint8_t*>(workspace);
  auto st = reinterpret_cast<cudaStream_t>(stream);
  const auto& L = plan->ws;
  const size_t T = plan->T, H = plan->H, S = static_cast<size_t>(plan->S);
  const size_t x_bytes = T * H * (bf16 ? 2 : 1), out_bytes = T * H * 2;
  cudaStream_t h2d = plan->io_h2d, d2h = plan->io_d2h;
  // Everything enqueued on `stream` before this call comes first.
  if (cudaEventRecord(plan->io_entry, st) != cudaSuccess ||
      cudaStreamWaitEvent(h2d, plan->io_entry, 0) != cudaSuccess ||
      cudaStreamWaitEvent(d2h, plan->io_entry, 0) != cudaSuccess)
    return MOE_ERR_CUDA;
  for (int i = 0; i < n_batches; ++i) {
    const int b = i & 1;
    // Staging set b's inputs are free once the layer of batch i-2 is done.
    if (i >= 2 && cudaStreamWaitEvent(h2d, plan->io_done[b], 0) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (cudaMemcpyAsync(ws + L.in_x[b], x_host[i], x_bytes, cudaMemcpyHostToDevice, h2d) !=
            cudaSuccess ||
        (!bf16 && cudaMemcpyAsync(ws + L.in_xs[b], x_scales_host[i], T * (H / 128),
                                  cudaMemcpyHostToDevice, h2d) != cudaSuccess) ||
        cudaMemcpyAsync(ws + L.in_idx[b], topk_idx_host[i], S * 4, cudaMemcpyHostToDevice,
                        h2d) != cudaSuccess ||
        cudaMemcpyAsync(ws + L.in_w[b], topk_w_host[i], S * 4, cudaMemcpyHostToDevice, h2d) !=
            cudaSuccess ||
        cudaEventRecord(plan->io_in[b], h2d) != cudaSuccess)
      return MOE_ERR_CUDA;
    // The layer waits for its inputs and, for staging set b's output, for the
    // output copy of batch i-2.
    if (cudaStreamWaitEvent(st, plan->io_in[b], 0) != cudaSuccess ||
        (i >= 2 && cudaStreamWaitEvent(st, plan->io_out[b], 0) != cudaSuccess))
      return MOE_ERR_CUDA;
    s = moe_forward(plan, ws + L.in_x[b], bf16 ? nullptr : ws + L.in_xs[b],
                    reinterpret_cast<const int32_t*>(ws + L.in_idx[b]),
                    reinterpret_cast<const float*>(ws + L.in_w[b]), w1, w1_scales, w2,
                    w2_scales, ws + L.out_stage[b], workspace, stream);
    if (s != MOE_OK) return s;
    if (cudaEventRecord(plan->io_done[b], st) != cudaSuccess ||
        cudaStreamWaitEvent(d2h, plan->io_done[b], 0) != cudaSuccess ||
        cudaMemcpyAsync(out_host[i], ws + L.out_stage[b], out_bytes, cudaMemcpyDeviceToHost,
                        d2h) != cudaSuccess ||
        cudaEventRecord(plan->io_out[b], d2h) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  // `stream` completes only after every output copy has landed.
  for (int b = 0; b < 2 && b < n_batches; ++b)
    if (cudaStreamWaitEvent(st, plan->io_out[b], 0) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_workspace_view(moe_plan_t plan, void* workspace, moe_workspace_view_t* v) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if (v == nullptr) return MOE_ERR_INVALID_ARG;
  auto ws = static_cast<uint8_t*>(workspace);
  const auto& L = plan->ws;
  v->counts = reinterpret_cast<int32_t*>(ws + L.counts);
  v->offsets = reinterpret_cast<int32_t*>(ws + L.offsets);
  v->perm = reinterpret_cast<int32_t*>(ws + L.perm);
  v->inv = reinterpret_cast<int32_t*>(ws + L.inv);
  v->pad_offsets = reinterpret_cast<int32_t*>(ws + L.pad_off);
  v->act = ws + L.act;
  v->act_f32 = plan->debug_act_f32 ? reinterpret_cast<float*>(ws + L.act_f32) : nullptr;
  v->y = reinterpret_cast<uint16_t*>(ws + L.y);
  v->error_word = reinterpret_cast<uint32_t*>(ws + L.err);
  v->rows = plan->rows_cap;
  return MOE_OK;
}

moe_status moe_copy_act_scales(moe_plan_t plan, const void* workspace, uint8_t* dst,
                               moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  if (dst == nullptr) return MOE_ERR_INVALID_ARG;
  if (plan->w_dtype == MOE_W_BF16) return MOE_ERR_UNSUPPORTED;
  return cuda_status(moe::launch_unpack_act_scales(plan, static_cast<const uint8_t*>(workspace),
                                                   dst, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_clear_device_error(moe_plan_t plan, void* workspace, moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  return cuda_status(cudaMemsetAsync(static_cast<uint8_t*>(workspace) + plan->ws.err, 0, 4,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_check_device_error(moe_plan_t plan, const void* workspace, moe_stream_t stream) {
  moe_status s = check_ws(plan, workspace);
  if (s != MOE_OK) return s;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, static_cast<const uint8_t*>(workspace) + plan->ws.err, 4,
                      cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return MOE_ERR_CUDA;
  if (word & (1u << MOE_ERR_DEVICE_TIMEOUT)) return MOE_ERR_DEVICE_TIMEOUT;
  if (word & (1u << MOE_ERR_BAD_ROUTING)) return MOE_ERR_BAD_ROUTING;
  return MOE_OK;
}

const char* moe_status_str(moe_status status) {
  switch (status) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_ALIGNMENT: return "MOE_ERR_ALIGNMENT";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE_TIMEOUT: return "MOE_ERR_DEVICE_TIMEOUT";
    case MOE_ERR_BAD_ROUTING: return "MOE_ERR_BAD_ROUTING";
  }
  return "MOE_ERR_UNKNOWN";
}

}  // extern "C"
