// gemm2.cu -- FC1 and FC2 in one persistent launch on CTA pairs (clusters of
// two) with the 2-SM tensor-core MMA (tcgen05.mma.cta_group::2): each pair
// computes a 256 x 256 tile of one expert -- two 128-row m-tiles of the same
// expert, one per CTA -- so each SM loads its own A rows but only half of B.
// Per 128-wide k-block an SM then moves 32 KB instead of 48 KB, which is what
// bounds the single-CTA kernel at large token counts.
//
// Every shared-memory operand of a stage arrives by TMA with its completion
// counted on the pair leader's mbarrier: the pre-swizzled 16 KB tiles
// (gathered x, FP8 activation, prepacked FP8 weights), the activation scale
// chunks, and the weight scales as 1 KB records expanded once per call by a
// small kernel (a warp that wrote them to shared memory would have to signal
// the other CTA with a cluster-scope release every k-block, which costs more
// than the k-block's MMAs).  The leader copies the scales into both CTAs'
// TMEM (tcgen05.cp.cta_group::2).
//
// Roles (per CTA, 12 warps): warp 0 operand-tile producer, warp 1 MMA issuer
// (the leader's only; both own the pair's TMEM allocation), warp 2 tile
// scheduler (leader's only: it writes each task into both CTAs' slot rings),
// warp 3 scale producer, warps 4-11 epilogue (each CTA its own 128 rows).
//
// Barrier scopes: full, empty and tmem_full complete only through TMA bytes
// and tcgen05.commit, so their waits acquire at CTA scope; the task slots
// (written with st.shared::cluster) and tmem_empty (released by the other
// CTA's epilogue) are waited on at cluster scope.
//
// Scheduler slot release (fw-ai/DeepGEMM PR #16 "Sync upstream through PR #441:
// fix Mega MoE scheduler ordering", Overview): consumers copy the task info out
// of their slot, fence, then arrive on the leader's empty barrier for the slot.
// Activation and requantisation: as in gemm.cu (DeepGEMM PR #445 Summary;
// TensorRT-LLM PR #16346 Description).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>

#include "internal.h"
#include "sm100_pair.cuh"

namespace moe {
namespace {

constexpr int BM = 128, BN = 256, BK = 128, STAGES = 6, SCHED_DEPTH = 4;
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCol = 0, kSfaCol = 256, kSfbCol = 264, kSfSetStride = 16;
constexpr int kEpiWarps = 8;
constexpr int kLeaderConsumers = 3 + kEpiWarps;   // two producers, MMA, epilogue warps
constexpr int kPeerConsumers = 2 + kEpiWarps;     // two producers, epilogue warps
constexpr uint64_t kDepWaitLimitNs = 2000000000ull;
// Bytes landing on the leader's full barrier per stage: both CTAs' A tile,
// half B tile, A scale chunk and B scale record.
constexpr uint32_t kStageTx = 2 * (kTileBytes + kTileBytes + 512 + 1024);

// Tensor maps, per GEMM: A tiles, B tiles, A scale chunks, B scale records.
struct Maps {
  CUtensorMap a[2], b[2], sfa[2], sfb[2];
};

struct __align__(1024) Smem {
  uint8_t a[STAGES][BM * BK];
  uint8_t b[STAGES][(BN / 2) * BK];
  uint8_t sfa[STAGES][512];
  uint8_t sfb[STAGES][1024];
  uint64_t full[STAGES];    // leader only
  uint64_t empty[STAGES];   // each CTA
  uint64_t tmem_full;       // each CTA
  uint64_t tmem_empty;      // leader only
  uint64_t drain;           // leader only: MMA completion before TMEM is freed
  uint64_t sched_full[SCHED_DEPTH];
  uint64_t sched_empty[SCHED_DEPTH];   // leader only
  uint64_t pair[4];
  int4 task[SCHED_DEPTH];   // kind | reuse << 1 | expert << 2, m-tile, n-tile, rows (0: none)
  int task_pos[SCHED_DEPTH];
  float amax[2][2][BM];
  uint32_t tmem_base;
  int abort_flag;
};

struct Phase {
  int n_tiles, k_blocks, b_rows_per_expert;
};

struct Params {
  int E, I, H;
  Phase ph[2];
  const int32_t* tile_off;
  const int32_t* pair_off;
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* perm;
  uint32_t* tile_counter;
  uint32_t* fc1_done;
  uint8_t* act;
  uint8_t* act_sf_chunks;
  float* act_f32;
  int oai;
  float alpha, up_bias, limit;
  uint16_t* y;
  uint32_t* err;
};

struct Task {
  int kind, e, mt, nt, rows, pos, reuse;
};

__device__ __forceinline__ void unpack_task(const int4 v, int pos, Task& t) {
  t.kind = v.x & 1;
  t.reuse = (v.x >> 1) & 1;
  t.e = v.x >> 2;
  t.mt = v.y;
  t.nt = v.z;
  t.rows = v.w;
  t.pos = pos;
}

// Warp-wide consumer of the local slot ring; releases the slot on the
// leader's empty barrier (release at cluster scope).
__device__ __forceinline__ bool get_task(Smem& sm, int& slot, uint32_t& phase, Task& t,
                                         uint32_t* err, const uint32_t* lead_sched_empty) {
  if (!mbar_wait_cluster(&sm.sched_full[slot], phase, err, &sm.abort_flag)) return false;
  unpack_task(sm.task[slot], sm.task_pos[slot], t);
  __syncwarp();
  asm volatile("fence.acq_rel.cluster;" ::: "memory");
  if (lane_id() == 0) mbar_arrive_cluster(lead_sched_empty[slot]);
  if (++slot == SCHED_DEPTH) {
    slot = 0;
    phase ^= 1u;
  }
  return true;
}

__device__ __forceinline__ float sigmoidf_fast(float z) {
  return __fdividef(1.0f, 1.0f + __expf(-z));
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__global__ void __launch_bounds__(kThreads, 1)
    moe_gemm_pair_kernel(const __grid_constant__ Maps tm, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  griddep_launch_dependents();
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&sm.full[s], 1);   // the leader's expect-tx arrive; bytes from both CTAs
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.tmem_full, 1);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.tmem_empty, 2 * kEpiWarps);
    for (int r = 0; r < SCHED_DEPTH; ++r) {
      mbar_init(&sm.sched_full[r], 1);
      mbar_init(&sm.sched_empty[r], kLeaderConsumers + kPeerConsumers);
    }
    for (int q = 0; q < 4; ++q) mbar_init(&sm.pair[q], 2);
    sm.abort_flag = 0;
    fence_mbarrier_init();
    for (int g = 0; g < 2; ++g) {
      tma_prefetch_desc(&tm.a[g]);
      tma_prefetch_desc(&tm.b[g]);
      tma_prefetch_desc(&tm.sfa[g]);
      tma_prefetch_desc(&tm.sfb[g]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(&sm.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs' barriers exist before any remote operation
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  griddep_wait();

  // Cluster addresses of the leader's barriers that both CTAs signal.
  uint32_t lead_full[STAGES], lead_sched_empty[SCHED_DEPTH];
#pragma unroll
  for (int s = 0; s < STAGES; ++s) lead_full[s] = mapa_shared(smem_u32(&sm.full[s]), 0);
#pragma unroll
  for (int r = 0; r < SCHED_DEPTH; ++r)
    lead_sched_empty[r] = mapa_shared(smem_u32(&sm.sched_empty[r]), 0);
  const uint32_t lead_tmem_empty = mapa_shared(smem_u32(&sm.tmem_empty), 0);

  if (warp == 2) {
    // ------------------------------------------------------------ scheduler
    // Leader only.  Tiles: [0, T1) FC1 (pair, n-tile), [T1, T1 + T2) FC2, pair
    // major; all FC1 tiles are handed out before any FC2 tile.
    if (leader && lane == 0) {
      const int total_pairs = p.pair_off[p.E];
      const int T1 = total_pairs * p.ph[0].n_tiles;
      const int T2 = total_pairs * p.ph[1].n_tiles;
      const uint32_t peer_task0 = mapa_shared(smem_u32(&sm.task[0]), 1);
      const uint32_t peer_pos0 = mapa_shared(smem_u32(&sm.task_pos[0]), 1);
      const uint32_t peer_full0 = mapa_shared(smem_u32(&sm.sched_full[0]), 1);
      int slot = 0;
      uint32_t phase = 0;
      int e_cur[2] = {0, 0};
      while (true) {
        const int tile = static_cast<int>(atomicAdd(p.tile_counter, 1u));
        int4 v0 = make_int4(~3, 0, 0, 0), v1 = v0;   // expert -1: no more work
        int pos0 = 0, pos1 = 0;
        const bool live = tile < T1 + T2;
        if (live) {
          const int kind = tile < T1 ? 0 : 1;
          const int lt = kind ? tile - T1 : tile;
          const int nt_n = p.ph[kind].n_tiles;
          const int pg = lt / nt_n;
          const int nt = lt - pg * nt_n;
          int& e = e_cur[kind];
          if (p.pair_off[e] > pg) e = 0;
          while (p.pair_off[e + 1] <= pg) ++e;
          const int mt0 = p.tile_off[e] + 2 * (pg - p.pair_off[e]);
          const int mt1 = mt0 + 1;
          const bool has1 = mt1 < p.tile_off[e + 1];
          const int reuse = (p.tile_off[e + 1] - p.tile_off[e]) > 2;
          const int local0 = (mt0 - p.tile_off[e]) * BM;
          const int rows0 = min(BM, p.counts[e] - local0);
          const int rows1 = has1 ? min(BM, p.counts[e] - local0 - BM) : 0;
          const int code = kind | (reuse << 1) | (e << 2);
          v0 = make_int4(code, mt0, nt, rows0);
          // A CTA whose m-tile is missing (odd tile count) computes on mt0's
          // rows and stores nothing (rows = 0).
          v1 = make_int4(code, has1 ? mt1 : mt0, nt, rows1);
          pos0 = p.offsets[e] + local0;
          pos1 = pos0 + BM;
        }
        if (!mbar_wait_cluster(&sm.sched_empty[slot], phase ^ 1u, p.err, &sm.abort_flag)) break;
        sm.task[slot] = v0;
        sm.task_pos[slot] = pos0;
        st_cluster_v4(peer_task0 + slot * sizeof(int4), v1);
        st_cluster_s32(peer_pos0 + slot * sizeof(int), pos1);
        mbar_arrive(&sm.sched_full[slot]);
        mbar_arrive_cluster(peer_full0 + slot * sizeof(uint64_t));
        if (++slot == SCHED_DEPTH) {
          slot = 0;
          phase ^= 1u;
        }
        if (!live) break;
      }
    }
  } else if (warp == 0 || warp == 3) {
    // ------------------------------------------------------------ producers
    // Warp 0 loads the operand tiles, warp 3 the scales; only the leader's
    // warp 0 arrives (with the stage's byte count) on the full barrier.
    const bool tiles = warp == 0;
    int slot = 0, stage = 0;
    uint32_t sphase = 0, phase = 0;
    const uint64_t pol_a = l2_policy_evict_last();
    const uint64_t pol_b_once = l2_policy_evict_first();
    const uint64_t pol_b_reused = l2_policy_evict_normal();
    const uint32_t fc1_target = static_cast<uint32_t>(kEpiWarps * p.ph[0].n_tiles);
    Task t;
    bool aborted = false;
    while (!aborted && get_task(sm, slot, sphase, t, p.err, lead_sched_empty)) {
      if (t.e < 0) break;
      const Phase& ph = p.ph[t.kind];
      const uint64_t pol_b = t.reuse ? pol_b_reused : pol_b_once;
      // B rows of the pair's tile: 128 gate + 128 up rows (FC1) or 256
      // consecutive rows (FC2); this CTA loads the half `rank`.
      const int brow0 = t.kind == 0 ? t.e * ph.b_rows_per_expert + t.nt * 128
                                    : t.e * ph.b_rows_per_expert + t.nt * 256;
      const int my_brow = rank ? brow0 + (t.kind == 0 ? p.I : 128) : brow0;
      if (t.kind == 1 && t.rows > 0) {
        // FC2 in the same launch: wait for this m-tile's FC1 rows, then order
        // those generic-proxy writes before the async-proxy (TMA) reads.
        if (lane == 0) {
          const uint32_t* flag = p.fc1_done + t.mt;
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
          fence_proxy_async_global();
        }
        __syncwarp();
        if (sm.abort_flag) break;
      }
      const int g = t.kind;
      // Scale record of (expert, n-tile, k-block): 4 rows of 256 bytes.
      const int rec0 = (t.e * ph.n_tiles + t.nt) * ph.k_blocks;
      for (int kb = 0; kb < ph.k_blocks; ++kb) {
        if (!mbar_wait(&sm.empty[stage], phase ^ 1u, p.err, &sm.abort_flag)) {
          aborted = true;
          break;
        }
        if (lane == 0) {
          const int a_tile = t.mt * ph.k_blocks + kb;
          if (tiles) {
            if (leader) mbar_arrive_expect_tx(&sm.full[stage], kStageTx);
            // Tiles are rows of 128 bytes in these maps: tile index * 128.
            const int b_tile = (my_brow / 128) * ph.k_blocks + kb;
            tma_load_2d_pair(sm.a[stage], &tm.a[g], 0, a_tile * 128, lead_full[stage], pol_a);
            tma_load_2d_pair(sm.b[stage], &tm.b[g], 0, b_tile * 128, lead_full[stage], pol_b);
          } else {
            // Token scales: the chunk of the k-block's group (two 256-byte rows).
            const int a_chunk = t.mt * sf_groups(ph.k_blocks) + kb / kSfGroup;
            tma_load_2d_pair(sm.sfa[stage], &tm.sfa[g], 0, a_chunk * 2, lead_full[stage], pol_a);
            tma_load_2d_pair(sm.sfb[stage], &tm.sfb[g], 0, (rec0 + kb) * 4, lead_full[stage],
                             pol_b_reused);
          }
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (leader && lane == 0) {
      int slot = 0, stage = 0;
      uint32_t sphase = 0, phase = 0, acc_phase = 0, sfset = 0;
      // Stage-0 descriptors built once; a stage adds its byte offset >> 4 and
      // a 32-byte K step adds 2 (the 14-bit address field cannot carry).
      const uint64_t a_desc0 = umma_desc_sw128(smem_u32(sm.a[0]));
      const uint64_t b_desc0 = umma_desc_sw128(smem_u32(sm.b[0]));
      const uint64_t sfa_desc0 = sf_desc(smem_u32(sm.sfa[0]));
      const uint64_t sfb_desc0 = sf_desc(smem_u32(sm.sfb[0]));
      constexpr uint64_t kAStage = (BM * BK) >> 4, kBStage = ((BN / 2) * BK) >> 4;
      constexpr uint64_t kSfaStage = 512 >> 4, kSfbStage = 1024 >> 4, kKStep = 32 >> 4;
      Task t;
      bool aborted = false;
      while (!aborted) {
        if (!mbar_wait_cluster(&sm.sched_full[slot], sphase, p.err, &sm.abort_flag)) break;
        unpack_task(sm.task[slot], sm.task_pos[slot], t);
        asm volatile("fence.acq_rel.cluster;" ::: "memory");
        mbar_arrive(&sm.sched_empty[slot]);
        if (++slot == SCHED_DEPTH) {
          slot = 0;
          sphase ^= 1u;
        }
        if (t.e < 0) break;
        if (!mbar_wait_cluster(&sm.tmem_empty, acc_phase ^ 1u, p.err, &sm.abort_flag)) break;
        tc_fence_after();
        const int k_blocks = p.ph[t.kind].k_blocks;
        for (int kb = 0; kb < k_blocks; ++kb) {
          if (!mbar_wait(&sm.full[stage], phase, p.err, &sm.abort_flag)) {
            aborted = true;
            break;
          }
          const uint32_t sfa = tmem + kSfaCol + sfset * kSfSetStride;
          const uint32_t sfb = tmem + kSfbCol + sfset * kSfSetStride;
          const uint64_t sfbd = sfb_desc0 + static_cast<uint64_t>(stage) * kSfbStage;
          tmem_cp_pair_32x128b_warpx4(sfa, sfa_desc0 + static_cast<uint64_t>(stage) * kSfaStage);
          tmem_cp_pair_32x128b_warpx4(sfb, sfbd);
          tmem_cp_pair_32x128b_warpx4(sfb + 4, sfbd + (512 >> 4));
          const uint64_t ad = a_desc0 + static_cast<uint64_t>(stage) * kAStage;
          const uint64_t bd = b_desc0 + static_cast<uint64_t>(stage) * kBStage;
          // Token rows (A) read byte kb % 4 of their scale words (the k-block's
          // 1x128 scale); the weight records repeat one byte per block, read at
          // K step ks.
          const uint32_t kc = static_cast<uint32_t>(kb % kSfGroup);
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
            mma_mxf8f6f4_pair(tmem + kAccCol, ad + ks * kKStep, bd + ks * kKStep,
                              mxf8f6f4_idesc_m256(BN, 0) | (static_cast<uint32_t>(ks) << 4) |
                                  (kc << 29),
                              sfa | (kc << 30), sfb | (static_cast<uint32_t>(ks) << 30),
                              (kb > 0 || ks > 0) ? 1u : 0u);
          }
          tc_commit_pair_multicast(&sm.empty[stage], 0x3);
          sfset ^= 1u;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (aborted) break;
        tc_commit_pair_multicast(&sm.tmem_full, 0x3);
        acc_phase ^= 1u;
      }
      // Every MMA and TMEM copy issued above (into both CTAs' TMEM) completes
      // before the pair frees its TMEM, on the abort path too.
      tc_commit_pair_multicast(&sm.drain, 0x1);
      if (!mbar_wait_limited(&sm.drain, 0, kWaitLimitNs)) atomicOr(p.err, kErrTimeoutBit);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int half = (warp - 4) >> 2;
    const int row = q * 32 + lane;
    const uint32_t t_row = tmem + (static_cast<uint32_t>(q * 32) << 16);
    int slot = 0;
    uint32_t sphase = 0, acc_phase = 0, pair_phase = 0;
    int tile_par = 0;
    Task t;
    while (get_task(sm, slot, sphase, t, p.err, lead_sched_empty)) {
      if (t.e < 0) break;
      if (!mbar_wait(&sm.tmem_full, acc_phase, p.err, &sm.abort_flag)) break;
      tc_fence_after();
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
        if (lane == 0) mbar_arrive_cluster(lead_tmem_empty);
        if (t.rows > 0) {
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
          sm.amax[tile_par][half][row] = amax;
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.pair[q]);
          if (!mbar_wait(&sm.pair[q], pair_phase, p.err, &sm.abort_flag)) break;
          pair_phase ^= 1u;
          amax = fmaxf(amax, sm.amax[tile_par][half ^ 1][row]);
          const int n = ue8m0_exponent(amax);
          const float inv_scale = __uint_as_float(static_cast<uint32_t>(127 - n) << 23);
          const size_t prow = static_cast<size_t>(t.mt) * BM + row;
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
            float4* fd =
                reinterpret_cast<float4*>(p.act_f32 + prow * p.I + t.nt * 128 + half * 64);
#pragma unroll
            for (int v = 0; v < 16; ++v)
              fd[v] = make_float4(__uint_as_float(g[4 * v]), __uint_as_float(g[4 * v + 1]),
                                  __uint_as_float(g[4 * v + 2]), __uint_as_float(g[4 * v + 3]));
          }
          // Publish this warp's rows to FC2 tiles of the same launch.
          __threadfence();
          __syncwarp();
          if (lane == 0) atomicAdd(p.fc1_done + t.mt, 1u);
          tile_par ^= 1;
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
        if (lane == 0) mbar_arrive_cluster(lead_tmem_empty);
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
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();   // no remote operation targets a CTA that has left
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

// --------------------------------------------------------------- host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// A byte buffer viewed as rows of `width` bytes; boxes of `box_rows` rows, no
// swizzle (the tiles are stored pre-swizzled).
bool map_rows(CUtensorMap* m, const void* base, uint64_t bytes, uint32_t width,
              uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t dims[2] = {width, bytes / width};
  const cuuint64_t strides[1] = {width};
  const cuuint32_t box[2] = {width, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t gemm_pair_smem_bytes() { return sizeof(Smem) + 1024; }

namespace {

// Weight scales of both GEMMs as the CTA-pair kernel loads them: one 1 KB
// record per (expert, n-tile, k-block) holding, 512 times each, the scale
// byte of the tile's first 128-row weight block and then of its second (FC1:
// the gate and up blocks of n-tile nt; FC2: the two halves of the 256-row
// n-tile).  Source scales are [row block][k-block] bytes, one per 128 x 128
// weight block.
__global__ void __launch_bounds__(256)
    expand_pair_scales_kernel(const uint8_t* __restrict__ w1s, const uint8_t* __restrict__ w2s,
                              uint4* __restrict__ out1, uint4* __restrict__ out2, int E, int I,
                              int H) {
  // Complete only after the previous kernel of the stream has, so that the
  // GEMM's own dependency wait covers both.
  griddep_wait();
  griddep_launch_dependents();
  const int kb1 = H / 128, nt1 = I / 128, kb2 = I / 128, nt2 = H / 256;
  const size_t n1 = static_cast<size_t>(E) * nt1 * kb1 * 64;   // 16-byte units
  const size_t n2 = static_cast<size_t>(E) * nt2 * kb2 * 64;
  for (size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n1 + n2;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const bool fc2 = i >= n1;
    const size_t j = fc2 ? i - n1 : i;
    const size_t rec = j / 64;
    const int second = static_cast<int>((j % 64) / 32);
    uint32_t v;
    if (!fc2) {
      const int kb = static_cast<int>(rec % kb1);
      const size_t en = rec / kb1;
      const int nt = static_cast<int>(en % nt1);
      const size_t e = en / nt1;
      const size_t rb = e * (2 * nt1) + nt + (second ? nt1 : 0);
      v = w1s[rb * kb1 + kb];
    } else {
      const int kb = static_cast<int>(rec % kb2);
      const size_t en = rec / kb2;
      const int nt = static_cast<int>(en % nt2);
      const size_t e = en / nt2;
      const size_t rb = e * (H / 128) + 2 * nt + second;
      v = w2s[rb * kb2 + kb];
    }
    const uint32_t w = v * 0x01010101u;
    (fc2 ? out2 : out1)[j] = make_uint4(w, w, w, w);
  }
}

}  // namespace

cudaError_t launch_fc12_pairs(const moe_plan_s* pl, const void* w1, const uint8_t* w1s,
                              const void* w2, const uint8_t* w2s, uint8_t* ws, cudaStream_t st) {
  const auto& L = pl->ws;
  const uint64_t rows = static_cast<uint64_t>(pl->rows_cap);
  const uint64_t E = pl->E;
  const uint64_t xg_bytes = rows * pl->H, act_bytes = rows * pl->I;
  const uint64_t w1_bytes = E * 2 * pl->I * pl->H, w2_bytes = E * pl->H * pl->I;
  const uint64_t sfa1_bytes = rows / kTileM * sf_groups(pl->H / 128) * 512;
  const uint64_t sfa2_bytes = rows / kTileM * sf_groups(pl->I / 128) * 512;
  const uint64_t sfb1_bytes = E * (pl->I / 128) * (pl->H / 128) * 1024;
  const uint64_t sfb2_bytes = E * (pl->H / 256) * (pl->I / 128) * 1024;
  Maps m;
  std::memset(&m, 0, sizeof(m));
  if (!map_rows(&m.a[0], ws + L.xg, xg_bytes, 128, 128) ||
      !map_rows(&m.b[0], w1, w1_bytes, 128, 128) ||
      !map_rows(&m.sfa[0], ws + L.xg_sf, sfa1_bytes, 256, 2) ||
      !map_rows(&m.sfb[0], ws + L.pair_sf1, sfb1_bytes, 256, 4) ||
      !map_rows(&m.a[1], ws + L.act, act_bytes, 128, 128) ||
      !map_rows(&m.b[1], w2, w2_bytes, 128, 128) ||
      !map_rows(&m.sfa[1], ws + L.act_sf, sfa2_bytes, 256, 2) ||
      !map_rows(&m.sfb[1], ws + L.pair_sf2, sfb2_bytes, 256, 4))
    return cudaErrorInvalidValue;

  const uint64_t units = (sfb1_bytes + sfb2_bytes) / 16;
  const int xblocks = static_cast<int>(std::min<uint64_t>((units + 255) / 256, 4ull * static_cast<uint64_t>(sm_count())));
  cudaError_t e = launch_pdl(expand_pair_scales_kernel, dim3(xblocks), dim3(256), 0, st, w1s, w2s,
                             reinterpret_cast<uint4*>(ws + L.pair_sf1),
                             reinterpret_cast<uint4*>(ws + L.pair_sf2), pl->E, pl->I, pl->H);
  if (e != cudaSuccess) return e;

  Params p{};
  p.E = pl->E;
  p.I = pl->I;
  p.H = pl->H;
  p.ph[0] = Phase{pl->I / 128, pl->H / 128, 2 * pl->I};
  p.ph[1] = Phase{pl->H / 256, pl->I / 128, pl->H};
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
  const size_t smem = sizeof(Smem) + 1024;
  e = ensure_max_dynamic_smem(reinterpret_cast<const void*>(moe_gemm_pair_kernel),
                              static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long max_pairs = (pl->rows_cap / kTileM + 1) / 2 * (pl->H / 256 + pl->I / 128);
  const int clusters = static_cast<int>(std::min<long long>(sm_count() / 2, max_pairs));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, moe_gemm_pair_kernel, m, p);
}

}  // namespace moe
