// gemm.cu -- FC1 and FC2 grouped GEMMs on the 5th-generation tensor cores, in
// one persistent launch (FC2 tiles of an m-tile start as soon as that m-tile's
// FC1 tiles have published their rows) or as separate launches.
//
// One persistent CTA per SM computes tiles of one expert.  Token-row tiles are
// 128 tokens x 256 columns:
//   FC1: A = gathered x rows [128 x H], B = 128 gate rows + 128 up rows of W1[e],
//        D = fp32 [128 x 256] in tensor memory; the epilogue applies the
//        (OAI-)SwiGLU and requantises the 128-wide activation block to E4M3 +
//        one UE8M0 scale per row (BF16 weights: rounds it to bf16).
//   FC2: A = activation rows [128 x I], B = 256 rows of W2[e]; the epilogue
//        writes bf16 rows to their slot (t*k + j) for the combine.
// Token-major ("swap AB") tiles, used for tiles with few tokens, make each
// 128-row half of the weight tile the A operand and the tile's tokens B
// (N = their count rounded up to 16), so the tensor work follows the tokens;
// the epilogue then owns one feature per TMEM lane.
// Weights: E4M3 with 128x128 or E2M1 with 1x32 UE8M0 scales, applied by the
// MMA itself (tcgen05.mma.kind::mxf8f6f4.block_scale, one scale per 32-wide K
// sub-block; coarser blocks are replicated), with E4M3 activations; or BF16
// weights and activations (kind::f16, no scales).
//
// Warp roles (12 warps):
//   warp 0   operand producer: bulk copies of pre-swizzled A/B tiles (2-D TMA
//            for row-major and MXFP4 weights); a token-major tile copies only
//            the first round16(rows) rows of its token tile
//   warp 1   MMA issuer (one lane); owns the tensor-memory allocation
//   warp 2   tile scheduler: writes task infos into a ring of shared-memory slots
//   warp 3   scale-factor producer: A scale chunks and prepacked MXFP4 scale
//            chunks (bulk copies), FP8 B scales (shared-memory stores) or
//            unchunked MXFP4 scales (cp.async)
//   warps 4-11 epilogue: two warps per 32-lane TMEM sub-partition
// Every wait is bounded (mbarrier waits and the FC1->FC2 dependency): on expiry
// the error word gets MOE_ERR_DEVICE_TIMEOUT and the CTA winds down.
//
// Scheduler slot release (fw-ai/DeepGEMM PR #16 "Sync upstream through PR #441:
// fix Mega MoE scheduler ordering", Overview): a consumer copies the task info
// out of its slot, then executes fence.acq_rel.cta, and only then arrives on the
// slot's empty barrier, so the scheduler can never overwrite metadata that is
// still being read.
//
// Activation (DeepGEMM PR #445 "fix(sm90): support parameterized SwiGLU in FP8
// MegaMoE", Summary): gate = min(gate, limit), up = clamp(up, -limit, limit),
// a = gate * sigmoid(alpha * gate) * (up + up_bias); its swapAB variant (the
// same PR's calc_diff table) for the token-major tiles.
// Requantisation (TensorRT-LLM PR #16346 "DSV4 o_proj: fuse fp8/UE8M0 quantize
// ...", Description): per 1x128 block, amax -> UE8M0 exponent -> E4M3 codes,
// done in the producing GEMM's epilogue.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>

#include "internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

constexpr int BM = 128, BN = 256, BK = 128, SCHED_DEPTH = 4;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0, kSfSetStride = 16;
constexpr int kEpiWarps = 8;
constexpr int kSchedConsumers = 3 + kEpiWarps;   // 2 producers, MMA, epilogue warps
constexpr uint64_t kDepWaitLimitNs = 2000000000ull;
// Automatic swap-AB: a tile of r token rows costs 2 x 128 x round16(r) MMA
// work token-major against 128 x 256 token-row, but its FC1 epilogue does more
// (a cross-lane amax, a barrier, byte stores); token-major from this size down.
constexpr int kSwapRows = 96;
// Wide token-major tiles (token-aware tiling, DeepGEMM PR #386 "Optimize sm100
// version with token-aware BM240 tiling, native UE8M0, and direct combine",
// title): the tokens of two consecutive m-tiles of one expert, up to 240, are
// the MMA's N, so an expert with 129..240 tokens streams its weights once.  Two
// accumulators of 128 features x 240 tokens take TMEM columns 0..479; the scale
// sets take the last 32.
constexpr int kWideMaxRows = 240;

// Per-kernel layout: the wide kernel's stages hold two token tiles (32 KB of
// A), so it keeps three stages; its scale columns sit above both accumulators.
template <bool kWide>
struct Cfg {
  static constexpr int kStages = kWide ? 3 : 4;
  static constexpr int kARows = kWide ? 2 * BM : BM;        // token rows a stage holds
  static constexpr uint32_t kD1Col = kWide ? 240u : 128u;    // token-major: second half's D
  // TMEM scale sets, two of each kind used in turn (so that a copy never
  // lands in the set that MMAs issued just before it may still read): token
  // scales (up to 8 columns: two 128-row chunks) and weight scales (8 columns:
  // two 128-row halves).
  static constexpr uint32_t kSfaCol = kWide ? 480u : 256u;
  static constexpr uint32_t kSfbCol = kWide ? 488u : 264u;
  static constexpr int kSfaBytes = kWide ? 1024 : 512;       // token scale chunk(s) per stage
};

template <bool kWide>
struct __align__(1024) SmemT {
  static constexpr int STAGES = Cfg<kWide>::kStages;
  uint8_t a[STAGES][Cfg<kWide>::kARows * BK];
  uint8_t b[STAGES][BN * BK];
  uint8_t sfa[STAGES][Cfg<kWide>::kSfaBytes];
  uint8_t sfb[STAGES][1024];
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tmem_full;
  uint64_t tmem_empty;
  uint64_t drain;   // tensor-core completion before TMEM is freed
  uint64_t sched_full[SCHED_DEPTH];
  uint64_t sched_empty[SCHED_DEPTH];
  uint64_t pair[4];
  int4 task[SCHED_DEPTH];          // kind | reuse << 1 | expert << 2, m-tile, n-tile, rows
  int task_pos[SCHED_DEPTH];       // position (unpadded) of the tile's first row
  float amax[2][2][BM];            // [tile parity][half][row]
  float swap_red[2][4][64];        // token-major FC1: per-warp amax [half][sub-partition][token]
  uint64_t swap_bar[2];            // token-major FC1: the four warps of a half (bounded waits)
  float swap_inv[2][64];           // token-major FC1: 1 / 2^n per token [half][token]
  uint32_t tmem_base;
  int abort_flag;
};

// One GEMM "phase": FC1 (x rows x W1, SwiGLU + requant epilogue) or FC2
// (activation rows x W2, bf16 slot-order epilogue).
struct Phase {
  int n_tiles;               // per m-tile: I/128 (FC1) or H/256 (FC2)
  int k_blocks;              // K / 128
  int b_rows_per_expert;     // 2I (FC1) or H (FC2)
  const uint8_t* sfa_chunks; // token scales [m-tiles][sf_groups(k_blocks)][512]
  const uint8_t* w_sf;       // weight scales
  const uint8_t* a_tiles;    // A operand, pre-swizzled tiles [m-tiles][k_blocks][16 KB]
  const uint8_t* w_tiles;    // weights as pre-swizzled tiles [E * n-blocks][k_blocks][16 KB],
                             // or null: weights row-major, loaded by 2-D TMA
};

struct Params {
  int E, I, H;
  int phases;                // bit 0: FC1 tiles, bit 1: FC2 tiles
  int dynamic;               // tiles from a global counter (else round-robin)
  int swap;                  // token-major MMAs (weights as A, the tile's tokens as B):
                             // 0 never, 1 always, 2 for tiles of at most kSwapRows rows
  int dep_extra;             // test hook: FC2 waits for this many FC1 completions more
  int sf_chunked;            // MXFP4 weight scales prepacked into 512-byte chunks
  int fp4_tiled;             // MXFP4 codes prepacked into 8 KB tiles (one TMA box each)
  Phase ph[2];
  const int32_t* tile_off;
  const int32_t* pair_off;   // per expert: pairs of consecutive m-tiles (wide kernel)
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* perm;
  uint32_t* tile_counter;    // dynamic scheduling (zeroed by the routing kernel)
  uint32_t* fc1_done;        // per m-tile: FC1 epilogue warps finished (zeroed by routing)
  // FC1 epilogue
  uint8_t* act;
  uint8_t* act_sf_chunks;
  float* act_f32;
  int oai;
  float alpha, up_bias, limit;
  // FC2 epilogue
  uint16_t* y;
  uint32_t* err;
};

struct Task {
  int kind, e, mt, nt, rows, pos;
  int reuse;   // the expert has more than one m-tile: its weight tiles are read again
};

// Consumer side of the scheduler ring: copy the task info out of the slot,
// order those reads before the release (acquire/release fence at CTA scope),
// then arrive on the slot's empty barrier.
template <class Smem>
__device__ __forceinline__ bool get_task(Smem& sm, int& slot, uint32_t& phase, Task& t,
                                         uint32_t* err) {
  if (!mbar_wait(&sm.sched_full[slot], phase, err, &sm.abort_flag)) return false;
  const int4 v = sm.task[slot];
  t.kind = v.x & 1;
  t.reuse = (v.x >> 1) & 1;
  t.e = v.x >> 2;
  t.mt = v.y;
  t.nt = v.z;
  t.rows = v.w;
  t.pos = sm.task_pos[slot];
  __syncwarp();
  fence_acq_rel_cta();
  if (lane_id() == 0) mbar_arrive(&sm.sched_empty[slot]);
  if (++slot == SCHED_DEPTH) {
    slot = 0;
    phase ^= 1u;
  }
  return true;
}

// sigmoid(z) with the fast exponential and an approximate reciprocal (the
// epilogue's transcendental pipe is shared by the E4M3 / bf16 conversions).
// Single-thread variant of get_task for the MMA issuer, which runs its loop
// on one lane only.
template <class Smem>
__device__ __forceinline__ bool get_task_single(Smem& sm, int& slot, uint32_t& phase, Task& t,
                                                uint32_t* err) {
  if (!mbar_wait(&sm.sched_full[slot], phase, err, &sm.abort_flag)) return false;
  const int4 v = sm.task[slot];
  t.kind = v.x & 1;
  t.reuse = (v.x >> 1) & 1;
  t.e = v.x >> 2;
  t.mt = v.y;
  t.nt = v.z;
  t.rows = v.w;
  t.pos = sm.task_pos[slot];
  fence_acq_rel_cta();
  mbar_arrive(&sm.sched_empty[slot]);
  if (++slot == SCHED_DEPTH) {
    slot = 0;
    phase ^= 1u;
  }
  return true;
}

// Token-major tile?  In the wide kernel a tile of more than 128 rows (two
// m-tiles) is always token-major.
template <bool kWide>
__device__ __forceinline__ bool swap_tile(const Params& p, int rows) {
  return (kWide && rows > BM) || p.swap == 1 || (p.swap == 2 && rows <= kSwapRows);
}

// Token-major N: the tile's rows rounded up to 16 (the MMA's N granularity).
__device__ __forceinline__ uint32_t swap_n(int rows) {
  return static_cast<uint32_t>(max(16, (rows + 15) & ~15));
}

__device__ __forceinline__ float sigmoidf_fast(float z) {
  return __fdividef(1.0f, 1.0f + __expf(-z));
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Weight formats: E4M3 with 128x128 UE8M0 scales, E2M1 with 1x32 UE8M0 scales
// (both with E4M3 activations, block-scaled MMA), or BF16 (BF16 activations,
// kind::f16 MMA, no scales).
enum : int { kWFp8 = 0, kWFp4 = 1, kWBf16 = 2 };

template <int kW, bool kWide>
__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a1,
                    const __grid_constant__ CUtensorMap tmap_b1,
                    const __grid_constant__ CUtensorMap tmap_a2,
                    const __grid_constant__ CUtensorMap tmap_b2, const Params p) {
  constexpr bool kFp4 = kW == kWFp4;
  constexpr bool kBf16 = kW == kWBf16;
  using Smem = SmemT<kWide>;
  using C = Cfg<kWide>;
  constexpr int STAGES = Smem::STAGES;
  extern __shared__ uint8_t smem_raw[];
  griddep_launch_dependents();
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // The operand producer's expect-tx arrive, plus the scale warp's: one
      // arrive (lane 0, after the warp's shared-memory writes or bulk copies),
      // or one per lane when its lanes' cp.async copies arrive themselves
      // (unchunked MXFP4 scales); BF16 has no scales.
      mbar_init(&sm.full[s], kBf16 ? 1 : (kFp4 && !p.sf_chunked ? 33 : 2));
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.tmem_full, 1);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.tmem_empty, kEpiWarps);
    for (int r = 0; r < SCHED_DEPTH; ++r) {
      mbar_init(&sm.sched_full[r], 1);
      mbar_init(&sm.sched_empty[r], kSchedConsumers);
    }
    for (int q = 0; q < 4; ++q) mbar_init(&sm.pair[q], 2);
    for (int h = 0; h < 2; ++h) mbar_init(&sm.swap_bar[h], 4);
    sm.abort_flag = 0;
    fence_mbarrier_init();
    if ((p.phases & 1) && p.ph[0].w_tiles == nullptr) tma_prefetch_desc(&tmap_b1);
    if ((p.phases & 2) && p.ph[1].w_tiles == nullptr) tma_prefetch_desc(&tmap_b2);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  // Everything above is local set-up that overlaps the previous kernel's tail.
  griddep_wait();

  if (warp == 2) {
    // ------------------------------------------------------------ scheduler
    // Tile index space: [0, T1) FC1 tiles, [T1, T1 + T2) FC2 tiles, m-tile
    // major within a phase.  With dynamic scheduling every FC1 tile is handed
    // out before any FC2 tile, so an FC2 tile only ever waits for FC1 tiles
    // that running CTAs already own (no deadlock, even if not all CTAs are
    // resident).
    // Wide kernel: the index space runs over pairs of consecutive m-tiles of
    // one expert, two indices per (pair, n-tile): a pair of at most 240 rows is
    // one wide token-major task at the first index (the second is skipped); a
    // pair of more rows is two tasks, one per m-tile; a lone m-tile is one.
    if (lane == 0) {
      const int units = kWide ? 2 * p.pair_off[p.E] : p.tile_off[p.E];
      const int T1 = (p.phases & 1) ? units * p.ph[0].n_tiles : 0;
      const int T2 = (p.phases & 2) ? units * p.ph[1].n_tiles : 0;
      int slot = 0;
      uint32_t phase = 0;
      int e_cur[2] = {0, 0};
      for (int i = 0;; ++i) {
        const int tile = p.dynamic ? static_cast<int>(atomicAdd(p.tile_counter, 1u))
                                   : static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
        Task t{0, -1, 0, 0, 0, 0, 0};
        if (tile < T1 + T2) {
          const int kind = tile < T1 ? 0 : 1;
          const int local_tile = kind ? tile - T1 : tile;
          const int nt_n = p.ph[kind].n_tiles;
          t.kind = kind;
          int& e = e_cur[kind];
          if (kWide) {
            const int unit = local_tile >> 1, sub = local_tile & 1;
            const int pg = unit / nt_n;
            t.nt = unit - pg * nt_n;
            if (p.pair_off[e] > pg) e = 0;   // round-robin order is monotone per phase
            while (p.pair_off[e + 1] <= pg) ++e;
            const int mt0 = p.tile_off[e] + 2 * (pg - p.pair_off[e]);
            const int local0 = (mt0 - p.tile_off[e]) * BM;
            const int rows_all = min(2 * BM, p.counts[e] - local0);
            if (rows_all <= kWideMaxRows) {
              if (sub) continue;   // one task covers the pair (or the lone m-tile)
              t.mt = mt0;
              t.rows = rows_all;
              t.pos = p.offsets[e] + local0;
            } else {
              t.mt = mt0 + sub;
              t.rows = sub ? rows_all - BM : BM;
              t.pos = p.offsets[e] + local0 + sub * BM;
            }
            t.e = e;
            t.reuse = p.counts[e] > kWideMaxRows;
          } else {
            t.mt = local_tile / nt_n;
            t.nt = local_tile - t.mt * nt_n;
            if (p.tile_off[e] > t.mt) e = 0;   // round-robin order is monotone per phase
            while (p.tile_off[e + 1] <= t.mt) ++e;
            const int local = (t.mt - p.tile_off[e]) * BM;
            t.e = e;
            t.rows = min(BM, p.counts[e] - local);
            t.pos = p.offsets[e] + local;
            t.reuse = (p.tile_off[e + 1] - p.tile_off[e]) > 1;
          }
        }
        if (!mbar_wait(&sm.sched_empty[slot], phase ^ 1u, p.err, &sm.abort_flag)) break;
        sm.task[slot] = make_int4(t.kind | (t.reuse << 1) | (t.e << 2), t.mt, t.nt, t.rows);
        sm.task_pos[slot] = t.pos;
        mbar_arrive(&sm.sched_full[slot]);   // release: the slot's contents are visible
        if (++slot == SCHED_DEPTH) {
          slot = 0;
          phase ^= 1u;
        }
        if (t.e < 0) break;
      }
    }
  } else if (warp == 0 || warp == 3) {
    // ------------------------------------------------------------ producers
    // Warp 0 streams the operand tiles (its bulk copies wait on the copy
    // engine); warp 3 provides the stage's scale factors in parallel.
    const bool operands = warp == 0;
    int slot = 0, stage = 0;
    uint32_t sphase = 0, phase = 0;
    if (kBf16 && !operands) {
      // No scale factors: the scale warp only releases its task slots.
      Task t;
      while (get_task(sm, slot, sphase, t, p.err)) {
        if (t.e < 0) break;
      }
    } else {
    // A tiles are re-read by every n-tile of their m-tile: keep them in L2.
    // Weight tiles are re-read only when the expert has several m-tiles;
    // otherwise they stream through L2 once and go first.
    const uint64_t pol_a = l2_policy_evict_last();
    const uint64_t pol_b_once = l2_policy_evict_first();
    const uint64_t pol_b_reused = l2_policy_evict_normal();
    const uint32_t ab_bytes = BM * BK + (kFp4 ? BN * BK / 2 : BN * BK);
    const uint32_t fc1_target = static_cast<uint32_t>(kEpiWarps * p.ph[0].n_tiles + p.dep_extra);
    Task t;
    bool aborted = false;
    while (!aborted && get_task(sm, slot, sphase, t, p.err)) {
      if (t.e < 0) break;
      const Phase& ph = p.ph[t.kind];
      const uint64_t pol_b = t.reuse ? pol_b_reused : pol_b_once;
      const CUtensorMap* tb = t.kind ? &tmap_b2 : &tmap_b1;
      // A token-major tile's MMAs read only its first N = round16(rows) token
      // rows, which are the first N * 128 bytes of the pre-swizzled tile (the
      // swizzle permutes 16-byte chunks within a row): copy just those.  A wide
      // tile's rows continue into the next m-tile's tile, copied right behind
      // the first (row 128 + i keeps row i's swizzle phase).
      const bool wide = kWide && t.rows > BM;
      const uint32_t a_bytes =
          swap_tile<kWide>(p, t.rows)
              ? (wide ? kTileBytes + swap_n(t.rows - BM) * 128u : swap_n(t.rows) * 128u)
              : kTileBytes;
      // Rows of B for this tile: two 128-row halves.
      int brow0, brow1;
      if (t.kind == 0) {
        brow0 = t.e * ph.b_rows_per_expert + t.nt * 128;          // gate rows
        brow1 = brow0 + p.I;                                      // up rows
      } else {
        brow0 = t.e * ph.b_rows_per_expert + t.nt * 256;
        brow1 = brow0 + 128;
      }
      if (t.kind == 1 && (p.phases & 1)) {
        // FC2 after FC1 in the same launch: wait until every FC1 epilogue warp
        // of this m-tile has published its rows (activation tiles and their
        // scale chunks), then order those generic-proxy writes before this
        // thread's async-proxy (bulk copy) reads.
        if (lane == 0) {
          // A wide tile reads the activation rows of two m-tiles.
          for (int m = 0; m < (wide ? 2 : 1); ++m) {
            const uint32_t* flag = p.fc1_done + t.mt + m;
            if (ld_acquire_gpu(flag) < fc1_target) {
              const uint64_t t0 = globaltimer();
              while (ld_acquire_gpu(flag) < fc1_target) {
                if (sm.abort_flag) break;
                if (globaltimer() - t0 > kDepWaitLimitNs) {
                  atomicOr(p.err, kErrTimeoutBit);
                  sm.abort_flag = 1;
                  break;
                }
                __nanosleep(128);
              }
            }
          }
          fence_proxy_async_global();
        }
        __syncwarp();
        if (sm.abort_flag) break;
      }
      uint32_t sf0 = 0, sf1 = 0;   // FP8 weight scales for k-blocks kb = 32*c + lane
      for (int kb = 0; kb < ph.k_blocks; ++kb) {
        if (!operands && !kFp4 && (kb & 31) == 0) {
          const int kq = kb + lane;
          const int kbs = ph.k_blocks;
          if (kq < kbs) {
            sf0 = ph.w_sf[static_cast<size_t>(brow0 / 128) * kbs + kq];
            sf1 = ph.w_sf[static_cast<size_t>(brow1 / 128) * kbs + kq];
          }
        }
        if (!mbar_wait(&sm.empty[stage], phase ^ 1u, p.err, &sm.abort_flag)) {
          aborted = true;
          break;
        }
        if (operands) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&sm.full[stage], ab_bytes - kTileBytes + a_bytes);
            // Operand tiles are contiguous and pre-swizzled: one linear bulk
            // copy each (row-major weights fall back to 2-D TMA tiles).
            if (wide) {
              bulk_load_hint(
                  sm.a[stage],
                  ph.a_tiles + (static_cast<size_t>(t.mt) * ph.k_blocks + kb) * kTileBytes,
                  kTileBytes, &sm.full[stage], pol_a);
              bulk_load_hint(
                  sm.a[stage] + kTileBytes,
                  ph.a_tiles + (static_cast<size_t>(t.mt + 1) * ph.k_blocks + kb) * kTileBytes,
                  a_bytes - kTileBytes, &sm.full[stage], pol_a);
            } else {
              bulk_load_hint(
                  sm.a[stage],
                  ph.a_tiles + (static_cast<size_t>(t.mt) * ph.k_blocks + kb) * kTileBytes,
                  a_bytes, &sm.full[stage], pol_a);
            }
            if (ph.w_tiles != nullptr) {
              bulk_load_hint(
                  sm.b[stage],
                  ph.w_tiles + (static_cast<size_t>(brow0 / 128) * ph.k_blocks + kb) * kTileBytes,
                  kTileBytes, &sm.full[stage], pol_b);
              bulk_load_hint(
                  sm.b[stage] + 128 * BK,
                  ph.w_tiles + (static_cast<size_t>(brow1 / 128) * ph.k_blocks + kb) * kTileBytes,
                  kTileBytes, &sm.full[stage], pol_b);
            } else if (kFp4 && p.fp4_tiled) {
              // Tiled E2M1 codes: the k-block of a 128-row block is one
              // contiguous 8 KB tile, row (block * k_blocks + kb) * 128 of the map.
              tma_load_2d(sm.b[stage], tb, 0, (brow0 / 128 * ph.k_blocks + kb) * 128,
                          &sm.full[stage], pol_b);
              tma_load_2d(sm.b[stage] + 128 * BK, tb, 0, (brow1 / 128 * ph.k_blocks + kb) * 128,
                          &sm.full[stage], pol_b);
            } else if (t.kind == 0) {
              tma_load_2d(sm.b[stage], tb, kb * BK, brow0, &sm.full[stage], pol_b);
              tma_load_2d(sm.b[stage] + 128 * BK, tb, kb * BK, brow1, &sm.full[stage], pol_b);
            } else {
              tma_load_2d(sm.b[stage], tb, kb * BK, brow0, &sm.full[stage], pol_b);
            }
          }
          __syncwarp();
        } else {
          // A group's first k-block brings the token scales of the group's four
          // k-blocks (one chunk per m-tile; a wide tile's second m-tile too) and,
          // for FP8 weights, writes the group's weight scales: the MMA issuer
          // copies both into TMEM once per group.
          const bool group_start = kb % kSfGroup == 0;
          if (lane == 0 && group_start) {
            const int groups = sf_groups(ph.k_blocks), g = kb / kSfGroup;
            mbar_expect_tx(&sm.full[stage], wide ? 1024 : 512);
            bulk_load(sm.sfa[stage],
                      ph.sfa_chunks + (static_cast<size_t>(t.mt) * groups + g) * 512, 512,
                      &sm.full[stage]);
            if (wide)
              bulk_load(sm.sfa[stage] + 512,
                        ph.sfa_chunks + (static_cast<size_t>(t.mt + 1) * groups + g) * 512, 512,
                        &sm.full[stage]);
          }
          if (kFp4 && p.sf_chunked) {
            // Prepacked scales: the stage's two 512-byte chunks (128 weight rows
            // each) are contiguous, so two bulk copies replace 256 scattered
            // 4-byte reads.
            if (lane == 0) {
              mbar_expect_tx(&sm.full[stage], 1024);
              bulk_load(sm.sfb[stage],
                        ph.w_sf + (static_cast<size_t>(brow0 / 128) * ph.k_blocks + kb) * 512,
                        512, &sm.full[stage]);
              bulk_load(sm.sfb[stage] + 512,
                        ph.w_sf + (static_cast<size_t>(brow1 / 128) * ph.k_blocks + kb) * 512,
                        512, &sm.full[stage]);
              mbar_arrive(&sm.full[stage]);
            }
            __syncwarp();
          } else if (kFp4) {
            // One 32-bit word = the four 1x32 scales of this 128-wide k-block.
            const int kw = ph.k_blocks * 4;   // scale bytes per weight row
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const int rb = c ? brow1 : brow0;
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const int r = lane + 32 * q;
                cp_async_4(sm.sfb[stage] + c * 512 + lane * 16 + q * 4,
                           ph.w_sf + static_cast<size_t>(rb + r) * kw + kb * 4);
              }
            }
            cp_async_mbar_arrive_noinc(&sm.full[stage]);
          } else {
            if (group_start) {
              // One scale per 128 x 128 weight block: byte c of every row's word
              // is the block's scale for k-block kb + c (kb + c stays inside the
              // 32 k-blocks held in sf0 / sf1).
              uint32_t g = 0, u = 0;
#pragma unroll
              for (int c = 0; c < kSfGroup; ++c) {
                const uint32_t gc = __shfl_sync(0xffffffffu, sf0, (kb + c) & 31);
                const uint32_t uc = __shfl_sync(0xffffffffu, sf1, (kb + c) & 31);
                if (kb + c < ph.k_blocks) {
                  g |= (gc & 0xFFu) << (8 * c);
                  u |= (uc & 0xFFu) << (8 * c);
                }
              }
              reinterpret_cast<uint4*>(sm.sfb[stage])[lane] = make_uint4(g, g, g, g);
              reinterpret_cast<uint4*>(sm.sfb[stage] + 512)[lane] = make_uint4(u, u, u, u);
              // Every lane makes its writes visible to the tensor core (async
              // proxy); the warp barrier orders them before lane 0's release.
              fence_proxy_async_smem();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.full[stage]);
          }
        }
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    }   // BF16 scale warp / producers
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    // One lane issues everything: a warp-wide wait + fence + __syncwarp per
    // k-block leaves the tensor pipe idle between k-blocks.
    if (lane == 0) {
      int slot = 0, stage = 0;
      uint32_t sphase = 0, phase = 0, acc_phase = 0;
      // TMEM scale sets (two of each, alternating so that a copy never lands in
      // the set the MMAs just issued may still read): token scales switch per
      // group of four k-blocks, weight scales per k-block (MXFP4) or per group
      // (FP8).  The first copy goes to set 0.
      uint32_t tset = 1, wset = 1;
      // Shared-memory descriptors of stage 0, built once: a stage's descriptor
      // is stage 0's plus its byte offset >> 4, and each 32-byte K step of a
      // 128-byte k-block adds 2 (the 14-bit address field cannot carry: shared
      // addresses stay below 2^18 bytes).  The issuing lane then spends a
      // 64-bit add per operand instead of rebuilding every descriptor.
      const uint64_t a_desc0 = umma_desc_sw128(smem_u32(sm.a[0]));
      const uint64_t b_desc0 = umma_desc_sw128(smem_u32(sm.b[0]));
      const uint64_t sfa_desc0 = sf_desc(smem_u32(sm.sfa[0]));
      const uint64_t sfb_desc0 = sf_desc(smem_u32(sm.sfb[0]));
      constexpr uint64_t kAStage = (C::kARows * BK) >> 4, kBStage = (BN * BK) >> 4;
      constexpr uint64_t kBHalf = (128 * BK) >> 4, kKStep = 32 >> 4;
      constexpr uint64_t kSfaStage = C::kSfaBytes >> 4, kSfbStage = 1024 >> 4;
      constexpr uint64_t kSfHalf = 512 >> 4;   // the second 128-row chunk of a scale pair
      Task t;
      bool aborted = false;
      while (!aborted && get_task_single(sm, slot, sphase, t, p.err)) {
        if (t.e < 0) break;
        if (!mbar_wait(&sm.tmem_empty, acc_phase ^ 1u, p.err, &sm.abort_flag)) break;
        tc_fence_after();
        const int k_blocks = p.ph[t.kind].k_blocks;
        // Token-major tiles: N = the tile's tokens rounded up to 16.  The
        // instruction descriptor of K step ks is this one with scale id ks.
        const bool swap = swap_tile<kWide>(p, t.rows);
        const bool wide = kWide && t.rows > BM;   // tokens of two m-tiles, N up to 240
        const uint32_t n = swap ? swap_n(t.rows) : BN;
        const uint32_t idesc0 =
            kBf16 ? bf16_idesc(n)
                  : (swap ? mxf8f6f4_idesc_ab(kFp4 ? 5u : 0u, 0u, n, 0)
                          : mxf8f6f4_idesc(kFp4 ? 5u : 0u, BN, 0));
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, p.err, &sm.abort_flag)) {
            aborted = true;
            break;
          }
          const uint64_t ad = a_desc0 + static_cast<uint64_t>(stage) * kAStage;
          const uint64_t bd = b_desc0 + static_cast<uint64_t>(stage) * kBStage;
          if (kBf16) {
            // 128 bytes of K = 64 BF16 values: four MMAs of K = 16 (32 bytes each).
            if (swap) {
              // Token-major, as for the block-scaled formats below.
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const uint32_t acc = (kb > 0 || ks > 0) ? 1u : 0u;
                mma_bf16(tmem + kAccCol, bd + ks * kKStep, ad + ks * kKStep, idesc0, acc);
                mma_bf16(tmem + kAccCol + C::kD1Col, bd + kBHalf + ks * kKStep,
                         ad + ks * kKStep, idesc0, acc);
              }
            } else {
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_bf16(tmem + kAccCol, ad + ks * kKStep, bd + ks * kKStep, idesc0,
                         (kb > 0 || ks > 0) ? 1u : 0u);
            }
          } else {
            // Unchunked MXFP4 weight scales land by cp.async (generic proxy):
            // order them before the tensor core's (async proxy) reads.
            if (kFp4 && !p.sf_chunked) fence_proxy_async_smem();
            // Scale-factor ids: the token operand reads byte kc of its words (its
            // 1x128 scale for k-block kb); MXFP4 weights read byte ks (their four
            // 1x32 scales), FP8 weights byte kc (one scale per 128 x 128 block).
            const uint32_t kc = static_cast<uint32_t>(kb % kSfGroup);
            const bool group_start = kc == 0;
            const bool w_copy = kFp4 || group_start;
            if (group_start) tset ^= 1u;
            if (w_copy) wset ^= 1u;
            const uint32_t sft = tmem + C::kSfaCol + tset * kSfSetStride;   // token scales
            const uint32_t sfw = tmem + C::kSfbCol + wset * kSfSetStride;   // weight scales
            if (group_start) {
              // Token scales: rows 0..127 in columns 0..3, a wide tile's rows
              // 128.. in columns 4..7 (the layout N > 128 reads).
              const uint64_t sfad = sfa_desc0 + static_cast<uint64_t>(stage) * kSfaStage;
              tmem_cp_32x128b_warpx4(sft, sfad);
              if (wide) tmem_cp_32x128b_warpx4(sft + 4, sfad + kSfHalf);
            }
            if (w_copy) {
              const uint64_t sfbd = sfb_desc0 + static_cast<uint64_t>(stage) * kSfbStage;
              tmem_cp_32x128b_warpx4(sfw, sfbd);
              tmem_cp_32x128b_warpx4(sfw + 4, sfbd + kSfHalf);
            }
            const uint32_t tok_sf = sft | (kc << 30);
            if (swap) {
              // Token-major: each 128-row half of the weight tile is the A
              // operand (A scale id: the weights'), the tile's tokens are B with
              // N = their count rounded up to 16 (B scale id: kc).  D0 (columns
              // 0..) holds the first half, D1 (columns 128..) the second.
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const uint32_t wid = kFp4 ? static_cast<uint32_t>(ks) : kc;
                const uint32_t idesc = idesc0 | (kc << 4) | (wid << 29);
                const uint32_t acc = (kb > 0 || ks > 0) ? 1u : 0u;
                mma_mxf8f6f4(tmem + kAccCol, bd + ks * kKStep, ad + ks * kKStep, idesc,
                             sfw | (wid << 30), tok_sf, acc);
                mma_mxf8f6f4(tmem + kAccCol + C::kD1Col, bd + kBHalf + ks * kKStep,
                             ad + ks * kKStep, idesc, (sfw + 4) | (wid << 30), tok_sf, acc);
              }
            } else {
              // Token rows are A (A scale id kc), the weights B.
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const uint32_t wid = kFp4 ? static_cast<uint32_t>(ks) : kc;
                const uint32_t idesc = idesc0 | (wid << 4) | (kc << 29);
                mma_mxf8f6f4(tmem + kAccCol, ad + ks * kKStep, bd + ks * kKStep, idesc, tok_sf,
                             sfw | (wid << 30), (kb > 0 || ks > 0) ? 1u : 0u);
              }
            }
          }
          tc_commit(&sm.empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (aborted) break;
        tc_commit(&sm.tmem_full);
        acc_phase ^= 1u;
      }
      // Every MMA and TMEM copy issued above completes before the TMEM is
      // freed, on the abort path too.
      tc_commit(&sm.drain);
      if (!mbar_wait_limited(&sm.drain, 0, kWaitLimitNs)) atomicOr(p.err, kErrTimeoutBit);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------- epilogue
    const int q = warp & 3;            // TMEM sub-partition (lanes 32q .. 32q+31)
    const int half = (warp - 4) >> 2;  // which half of the tile's columns
    const int row = q * 32 + lane;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
    int slot = 0;
    uint32_t sphase = 0, acc_phase = 0, pair_phase = 0, swap_phase = 0;
    int tile_par = 0;
    Task t;
    // Token-major FC1: the four warps of this half meet on an mbarrier (a
    // bounded wait, so an aborting CTA cannot leave a warp waiting forever).
    auto half_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.swap_bar[half]);
      const bool ok = mbar_wait(&sm.swap_bar[half], swap_phase, p.err, &sm.abort_flag);
      swap_phase ^= 1u;
      return ok;
    };
    while (get_task(sm, slot, sphase, t, p.err)) {
      if (t.e < 0) break;
      if (!mbar_wait(&sm.tmem_full, acc_phase, p.err, &sm.abort_flag)) break;
      tc_fence_after();
      if (swap_tile<kWide>(p, t.rows)) {
        // Token-major tile: TMEM lane = feature, column = token.  This warp
        // owns feature f of the tile for the tokens of its half.  A wide tile
        // (more than 128 rows, tokens of m-tiles mt and mt + 1) takes two
        // rounds of 128 tokens; the accumulator is released after the last
        // round's loads.
        const int f = q * 32 + lane;
        const int rounds = (kWide && t.rows > BM) ? 2 : 1;
        bool ok = true;
        if (t.kind == 0) {
          for (int rho = 0; rho < rounds && ok; ++rho) {
          const int mt = t.mt + rho;                  // m-tile of this round's tokens
          const int tok0 = rho * BM + half * 64;      // first token (column) of this warp
          const int ntok = min(64, t.rows - tok0);    // uniform over the half's warps
          // (Loaded unconditionally: TMEM columns are always addressable, and a
          // conditional load would move the arrays to local memory.)
          uint32_t g[64], u[64];
          tmem_ld_32x32b_x32(t_row + kAccCol + tok0, *reinterpret_cast<uint32_t(*)[32]>(g));
          tmem_ld_32x32b_x32(t_row + kAccCol + tok0 + 32,
                             *reinterpret_cast<uint32_t(*)[32]>(g + 32));
          tmem_ld_32x32b_x32(t_row + kAccCol + C::kD1Col + tok0,
                             *reinterpret_cast<uint32_t(*)[32]>(u));
          tmem_ld_32x32b_x32(t_row + kAccCol + C::kD1Col + tok0 + 32,
                             *reinterpret_cast<uint32_t(*)[32]>(u + 32));
          tmem_ld_wait();
          if (rho == rounds - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.tmem_empty);
          }
          if (ntok > 0) {
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              float gv = __uint_as_float(g[j]);
              float uv = __uint_as_float(u[j]);
              float a;
              if (p.oai) {
                gv = fminf(gv, p.limit);
                uv = fminf(fmaxf(uv, -p.limit), p.limit);
                a = gv * sigmoidf_fast(p.alpha * gv) * (uv + p.up_bias);
              } else {
                a = gv * sigmoidf_fast(gv) * uv;
              }
              g[j] = __float_as_uint(j < ntok ? a : 0.0f);
            }
          }
          if (kBf16 && ntok > 0) {
            // BF16 activation, token-major: feature f of n-tile nt is column
            // 128 * nt + f, i.e. byte 2 * (f % 64) of a row of activation tile
            // (m-tile, 2 * nt + f / 64).
            uint8_t* tile = p.act + (static_cast<size_t>(mt) * (p.I / 64) + 2 * t.nt + (f >> 6)) *
                                        kTileBytes;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              if (j < ntok) {
                const float av = __uint_as_float(g[j]);
                const int rr = half * 64 + j;   // row of the m-tile
                *reinterpret_cast<uint16_t*>(tile + swz128(rr, (f & 63) >> 3) + (f & 7) * 2) =
                    static_cast<uint16_t>(pack_bf16x2(av, 0.0f) & 0xFFFFu);
                if (p.act_f32 != nullptr)
                  p.act_f32[(static_cast<size_t>(mt) * BM + rr) * p.I + t.nt * 128 + f] = av;
              }
            }
          } else if (ntok > 0) {
            // amax of every token over this warp's 32 features (lanes), then
            // over the half's four warps (128 features = one requant block).
            // Transpose-reduction per 32 tokens: at the step with lane offset o
            // a lane keeps the o tokens of its side of bit o and trades the
            // other o with its partner, so after 31 shuffles lane l holds the
            // maximum of token l.
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              if (32 * r < ntok) {
                float m[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) m[i] = fabsf(__uint_as_float(g[32 * r + i]));
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) {
                  const bool upper = (lane & o) != 0;
#pragma unroll
                  for (int i = 0; i < o; ++i) {
                    const float send = upper ? m[i] : m[i + o];
                    const float keep = upper ? m[i + o] : m[i];
                    m[i] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, o));
                  }
                }
                sm.swap_red[half][q][32 * r + lane] = m[0];
              }
            }
            if (!half_sync()) {
              ok = false;
              break;
            }
            const int nb = p.I / 128, groups = sf_groups(nb);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const int j = lane + 32 * c;
              if (j < ntok) {
                const float m = fmaxf(fmaxf(sm.swap_red[half][0][j], sm.swap_red[half][1][j]),
                                      fmaxf(sm.swap_red[half][2][j], sm.swap_red[half][3][j]));
                const int n = ue8m0_exponent(m);
                if (q == 0) sm.swap_inv[half][j] = __uint_as_float(static_cast<uint32_t>(127 - n) << 23);
                if (q == 0) {
                  const int rr = half * 64 + j;   // row of the m-tile
                  p.act_sf_chunks[static_cast<size_t>(mt) * groups * 512 + sf_byte(rr, t.nt)] =
                      static_cast<uint8_t>(n + 127);
                }
              }
            }
            if (!half_sync()) {
              ok = false;
              break;
            }
            uint8_t* tile = p.act + (static_cast<size_t>(mt) * nb + t.nt) * kTileBytes;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              if (j < ntok) {
                const float av = __uint_as_float(g[j]);
                const int rr = half * 64 + j;
                tile[swz128(rr, f >> 4) + (f & 15)] =
                    static_cast<uint8_t>(cvt_e4m3x2(av * sm.swap_inv[half][j], 0.0f) & 0xFFu);
                if (p.act_f32 != nullptr)
                  p.act_f32[(static_cast<size_t>(mt) * BM + rr) * p.I + t.nt * 128 + f] = av;
              }
            }
          }
          }   // rounds
          if (!ok) break;
          if (p.phases & 2) {
            // Publish this warp's rows of every m-tile the tile covers.
            __threadfence();
            __syncwarp();
            if (lane == 0)
              for (int rho = 0; rho < rounds; ++rho) atomicAdd(p.fc1_done + t.mt + rho, 1u);
          }
        } else {
          const uint32_t dcol = kAccCol + (half ? C::kD1Col : 0u);   // this half's features
          const int h = t.nt * 256 + half * 128 + f;   // output column
          for (int rho = 0; rho < rounds; ++rho) {
          uint32_t v[128];
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tmem_ld_32x32b_x32(t_row + dcol + rho * BM + c * 32,
                               *reinterpret_cast<uint32_t(*)[32]>(v + 32 * c));
          tmem_ld_wait();
          if (rho == rounds - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.tmem_empty);
          }
          const int base = rho * BM;   // first token of this round
          int pl[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int j = base + lane + 32 * c;
            pl[c] = j < t.rows ? p.perm[t.pos + j] : 0;
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) {
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) {
              const int sl = __shfl_sync(0xffffffffu, pl[c], jj);
              if (base + c * 32 + jj < t.rows)
                p.y[static_cast<size_t>(sl) * p.H + h] =
                    static_cast<uint16_t>(pack_bf16x2(__uint_as_float(v[c * 32 + jj]), 0.0f) & 0xFFFFu);
            }
          }
          }   // rounds
        }
        acc_phase ^= 1u;
        continue;
      }
      if (t.kind == 0) {
        uint32_t g[64], u[64];
        tmem_ld_32x32b_x32(t_row + kAccCol + half * 64, *reinterpret_cast<uint32_t(*)[32]>(g));
        tmem_ld_32x32b_x32(t_row + kAccCol + half * 64 + 32,
                           *reinterpret_cast<uint32_t(*)[32]>(g + 32));
        tmem_ld_32x32b_x32(t_row + kAccCol + 128 + half * 64,
                           *reinterpret_cast<uint32_t(*)[32]>(u));
        tmem_ld_32x32b_x32(t_row + kAccCol + 128 + half * 64 + 32,
                           *reinterpret_cast<uint32_t(*)[32]>(u + 32));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.tmem_empty);
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          float gv = __uint_as_float(g[i]);
          float uv = __uint_as_float(u[i]);
          float a;
          if (p.oai) {
            gv = fminf(gv, p.limit);
            uv = fminf(fmaxf(uv, -p.limit), p.limit);
            a = gv * sigmoidf_fast(p.alpha * gv) * (uv + p.up_bias);
          } else {
            a = gv * sigmoidf_fast(gv) * uv;
          }
          g[i] = __float_as_uint(a);
          amax = fmaxf(amax, fabsf(a));
        }
        if (kBf16) {
          // BF16 activation (round to nearest even): this warp's 64 columns are
          // exactly one 128-byte row of activation tile (m-tile, 2 * nt + half).
          uint8_t* tile = p.act + (static_cast<size_t>(t.mt) * (p.I / 64) + 2 * t.nt + half) *
                                      kTileBytes;
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const int i0 = v * 8;
            *reinterpret_cast<uint4*>(tile + swz128(row, v)) = make_uint4(
                pack_bf16x2(__uint_as_float(g[i0]), __uint_as_float(g[i0 + 1])),
                pack_bf16x2(__uint_as_float(g[i0 + 2]), __uint_as_float(g[i0 + 3])),
                pack_bf16x2(__uint_as_float(g[i0 + 4]), __uint_as_float(g[i0 + 5])),
                pack_bf16x2(__uint_as_float(g[i0 + 6]), __uint_as_float(g[i0 + 7])));
          }
          if (p.act_f32 != nullptr) {
            const size_t prow = static_cast<size_t>(t.mt) * BM + row;
            float4* fd =
                reinterpret_cast<float4*>(p.act_f32 + prow * p.I + t.nt * 128 + half * 64);
#pragma unroll
            for (int v = 0; v < 16; ++v)
              fd[v] = make_float4(__uint_as_float(g[4 * v]), __uint_as_float(g[4 * v + 1]),
                                  __uint_as_float(g[4 * v + 2]), __uint_as_float(g[4 * v + 3]));
          }
          if (p.phases & 2) {
            __threadfence();
            __syncwarp();
            if (lane == 0) atomicAdd(p.fc1_done + t.mt, 1u);
          }
          acc_phase ^= 1u;
          continue;
        }
        // Combine the two halves' amax of this row (the other warp of the pair).
        sm.amax[tile_par][half][row] = amax;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.pair[q]);
        if (!mbar_wait(&sm.pair[q], pair_phase, p.err, &sm.abort_flag)) break;
        pair_phase ^= 1u;
        amax = fmaxf(amax, sm.amax[tile_par][half ^ 1][row]);
        const int n = ue8m0_exponent(amax);
        const float inv_scale = __uint_as_float(static_cast<uint32_t>(127 - n) << 23);
        const size_t prow = static_cast<size_t>(t.mt) * BM + row;
        // The activation is stored as pre-swizzled 128 x 128 tiles (FC2's A).
        uint8_t* tile = p.act + (static_cast<size_t>(t.mt) * (p.I / 128) + t.nt) * kTileBytes;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint32_t w[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int i0 = v * 16 + j * 4;
            const uint32_t lo = cvt_e4m3x2(__uint_as_float(g[i0]) * inv_scale,
                                           __uint_as_float(g[i0 + 1]) * inv_scale);
            const uint32_t hi = cvt_e4m3x2(__uint_as_float(g[i0 + 2]) * inv_scale,
                                           __uint_as_float(g[i0 + 3]) * inv_scale);
            w[j] = lo | (hi << 16);
          }
          *reinterpret_cast<uint4*>(tile + swz128(row, half * 4 + v)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (half == 0)
          p.act_sf_chunks[static_cast<size_t>(t.mt) * sf_groups(p.I / 128) * 512 +
                          sf_byte(row, t.nt)] = static_cast<uint8_t>(n + 127);
        if (p.act_f32 != nullptr) {
          float4* fd = reinterpret_cast<float4*>(p.act_f32 + prow * p.I + t.nt * 128 + half * 64);
#pragma unroll
          for (int v = 0; v < 16; ++v)
            fd[v] = make_float4(__uint_as_float(g[4 * v]), __uint_as_float(g[4 * v + 1]),
                                __uint_as_float(g[4 * v + 2]), __uint_as_float(g[4 * v + 3]));
        }
        if (p.phases & 2) {
          // Publish this warp's rows to FC2 tiles of the same launch: make the
          // stores visible at GPU scope, then count this warp as done.
          __threadfence();
          __syncwarp();
          if (lane == 0) atomicAdd(p.fc1_done + t.mt, 1u);
        }
      } else {
        uint32_t v[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld_32x32b_x32(t_row + kAccCol + half * 128 + c * 32,
                             *reinterpret_cast<uint32_t(*)[32]>(v + 32 * c));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.tmem_empty);
        if (row < t.rows) {
          const int s = p.perm[t.pos + row];
          uint4* dst = reinterpret_cast<uint4*>(p.y + static_cast<size_t>(s) * p.H + t.nt * 256 +
                                                half * 128);
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const uint32_t w0 = pack_bf16x2(__uint_as_float(v[8 * c + 0]), __uint_as_float(v[8 * c + 1]));
            const uint32_t w1 = pack_bf16x2(__uint_as_float(v[8 * c + 2]), __uint_as_float(v[8 * c + 3]));
            const uint32_t w2 = pack_bf16x2(__uint_as_float(v[8 * c + 4]), __uint_as_float(v[8 * c + 5]));
            const uint32_t w3 = pack_bf16x2(__uint_as_float(v[8 * c + 6]), __uint_as_float(v[8 * c + 7]));
            dst[c] = make_uint4(w0, w1, w2, w3);
          }
        }
      }
      acc_phase ^= 1u;
      tile_par ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// --------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D K-major tensor map: inner dimension `inner` elements, `outer` rows, box
// 128 (K) x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_rows, bool fp4) {
  EncodeTiledFn enc = get_encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      enc(m, fp4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
          const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int kW, bool kWide>
cudaError_t launch_gemm(const moe_plan_s* pl, int phases, bool dynamic, const void* w1,
                        const uint8_t* w1s, const void* w2, const uint8_t* w2s, uint8_t* ws,
                        cudaStream_t st) {
  const auto& L = pl->ws;
  CUtensorMap maps[4];
  std::memset(maps, 0, sizeof(maps));
  Params p{};
  p.E = pl->E;
  p.I = pl->I;
  p.H = pl->H;
  p.phases = phases;
  p.dynamic = dynamic ? 1 : 0;
  p.swap = use_swap(pl);
  p.dep_extra = pl->debug_fault ? 1 : 0;
  p.sf_chunked = pl->w_sf_chunked;
  long long max_tiles = 0;
  constexpr bool kFp4 = kW == kWFp4;
  constexpr bool kBf16 = kW == kWBf16;
  // FP8 / BF16 tiles are pre-swizzled and bulk-copied; E2M1 tiles are read by a
  // tensor map over the tile array (the copy widens the codes).
  const bool tiled = pl->w_tiled != 0 && !kFp4;
  const bool fp4_tiled = pl->w_tiled != 0 && kFp4;
  p.fp4_tiled = fp4_tiled ? 1 : 0;
  // Bytes of one weight row of K elements, and the map's inner extent: FP4 maps
  // count 4-bit elements (the copy widens them), the others count bytes.
  auto row_bytes = [](int K) { return kFp4 ? K / 2 : (kBf16 ? 2 * K : K); };
  auto inner = [](int K) { return kBf16 ? 2 * K : K; };
  // K-blocks of 128 bytes in shared memory (128 elements for FP8/FP4, 64 BF16).
  auto k_blocks = [](int K) { return kBf16 ? K / 64 : K / 128; };
  if (phases & 1) {
    const int K = pl->H;
    const uint64_t rows = static_cast<uint64_t>(pl->E) * 2 * pl->I;
    if (fp4_tiled ? !make_map(&maps[1], w1, 128, rows * (K / 128), 64, 128, true)
                  : (!tiled && !make_map(&maps[1], w1, inner(K), rows, row_bytes(K), 128, kFp4)))
      return cudaErrorInvalidValue;
    p.ph[0] = Phase{pl->I / 128, k_blocks(K), 2 * pl->I, kBf16 ? nullptr : ws + L.xg_sf, w1s,
                    ws + L.xg, tiled ? static_cast<const uint8_t*>(w1) : nullptr};
    max_tiles += (pl->rows_cap / BM) * p.ph[0].n_tiles;
  }
  if (phases & 2) {
    const int K = pl->I;
    const uint64_t rows = static_cast<uint64_t>(pl->E) * pl->H;
    if (fp4_tiled ? !make_map(&maps[3], w2, 128, rows * (K / 128), 64, 128, true)
                  : (!tiled && !make_map(&maps[3], w2, inner(K), rows, row_bytes(K), 256, kFp4)))
      return cudaErrorInvalidValue;
    p.ph[1] = Phase{pl->H / 256, k_blocks(K), pl->H, kBf16 ? nullptr : ws + L.act_sf, w2s,
                    ws + L.act, tiled ? static_cast<const uint8_t*>(w2) : nullptr};
    max_tiles += (pl->rows_cap / BM) * p.ph[1].n_tiles;
  }
  p.tile_off = reinterpret_cast<const int32_t*>(ws + L.tile_off);
  p.pair_off = reinterpret_cast<const int32_t*>(ws + L.pair_off);
  p.counts = reinterpret_cast<const int32_t*>(ws + L.counts);
  p.offsets = reinterpret_cast<const int32_t*>(ws + L.offsets);
  p.perm = reinterpret_cast<const int32_t*>(ws + L.perm);
  p.tile_counter = reinterpret_cast<uint32_t*>(ws + L.sched);
  p.fc1_done = reinterpret_cast<uint32_t*>(ws + L.sched) + 64;
  p.act = ws + L.act;
  p.act_sf_chunks = ws + L.act_sf;
  p.act_f32 = pl->debug_act_f32 ? reinterpret_cast<float*>(ws + L.act_f32) : nullptr;
  p.oai = pl->act.kind == MOE_ACT_SWIGLU_OAI;
  p.alpha = pl->act.alpha;
  p.up_bias = pl->act.up_bias;
  p.limit = pl->act.limit;
  p.y = reinterpret_cast<uint16_t*>(ws + L.y);
  p.err = reinterpret_cast<uint32_t*>(ws + L.err);
  const size_t smem = sizeof(SmemT<kWide>) + 1024;
  auto kern = moe_gemm_kernel<kW, kWide>;
  cudaError_t e = ensure_max_dynamic_smem(reinterpret_cast<const void*>(kern),
                                          static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(std::min<long long>(sm_count(), max_tiles));
  return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, maps[0], maps[1], maps[2],
                    maps[3], p);
}

}  // namespace

size_t gemm_smem_bytes() { return sizeof(SmemT<false>) + 1024; }

// phases: 1 FC1 only, 2 FC2 only, 3 both in one launch (dynamic scheduling).
static cudaError_t launch_phases(const moe_plan_s* p, int phases, const void* w1,
                                 const uint8_t* w1s, const void* w2, const uint8_t* w2s,
                                 uint8_t* ws, cudaStream_t st) {
  const bool dyn = phases == 3;
  const bool wide = use_wide(p) != 0;
  switch (p->w_dtype) {
    case MOE_W_E2M1_UE8M0_1x32:
      return wide ? launch_gemm<kWFp4, true>(p, phases, dyn, w1, w1s, w2, w2s, ws, st)
                  : launch_gemm<kWFp4, false>(p, phases, dyn, w1, w1s, w2, w2s, ws, st);
    case MOE_W_BF16:
      return wide ? launch_gemm<kWBf16, true>(p, phases, dyn, w1, w1s, w2, w2s, ws, st)
                  : launch_gemm<kWBf16, false>(p, phases, dyn, w1, w1s, w2, w2s, ws, st);
    default:
      return wide ? launch_gemm<kWFp8, true>(p, phases, dyn, w1, w1s, w2, w2s, ws, st)
                  : launch_gemm<kWFp8, false>(p, phases, dyn, w1, w1s, w2, w2s, ws, st);
  }
}

cudaError_t launch_fc1(const moe_plan_s* p, const void* w1, const uint8_t* w1s, uint8_t* ws,
                       cudaStream_t st) {
  return launch_phases(p, 1, w1, w1s, nullptr, nullptr, ws, st);
}

cudaError_t launch_fc2(const moe_plan_s* p, const void* w2, const uint8_t* w2s, uint8_t* ws,
                       cudaStream_t st) {
  return launch_phases(p, 2, nullptr, nullptr, w2, w2s, ws, st);
}

cudaError_t launch_fc12(const moe_plan_s* p, const void* w1, const uint8_t* w1s, const void* w2,
                        const uint8_t* w2s, uint8_t* ws, cudaStream_t st) {
  return launch_phases(p, 3, w1, w1s, w2, w2s, ws, st);
}

}  // namespace moe
