// route.cu -- step 1 (routing) and the FC1 operand gather, as separate launches
// or, for up to 4096 slots, as one (route_gather_kernel).
//
// Routing groups the T*k slots (slot s = t*k + j holds expert topk_idx[t, j]) by
// expert: a per-expert histogram, an exclusive scan, and a stable scatter that
// keeps each expert's slots in ascending slot order (DeepGEMM PR #386 "Optimize
// sm100 version with token-aware BM240 tiling, native UE8M0, and direct
// combine", Description: tokens are grouped per expert before the grouped
// GEMMs).  The result is integer and deterministic: it does not depend on the
// order in which blocks run.
//
// Layout produced for the GEMMs: every expert's rows start at a multiple of 128
// (pad_off[e] = 128 * tile_off[e]), so an m-tile never straddles two experts and
// the scale chunks can be addressed per tile.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "sm100.cuh"

namespace moe {
namespace {

// An expert id of -1 marks a masked slot: it is skipped without an error (the
// masked / unmasked sweeps of DeepGEMM PR #386's Description); any other id
// outside [0, E) is skipped and reported as MOE_ERR_BAD_ROUTING.
constexpr int kMaskedSlot = -1;

// The UE8M0 bytes of k-blocks 4g .. 4g+3 of one row of scales (0 past the
// row's end), as the 32-bit word of group g in the token scale-chunk layout.
__device__ __forceinline__ uint32_t sf_group_word(const uint8_t* __restrict__ row_sf, int kb_n,
                                                  int g) {
  uint32_t w = 0;
#pragma unroll
  for (int c = 0; c < kSfGroup; ++c) {
    const int kb = g * kSfGroup + c;
    if (kb < kb_n) w |= static_cast<uint32_t>(__ldg(&row_sf[kb])) << (8 * c);
  }
  return w;
}

// Kernel 1: per-block histograms of the block's kRouteChunk slots.
__global__ void __launch_bounds__(kRouteThreads) route_hist_kernel(
    const int32_t* __restrict__ idx, int S, int E, int32_t* __restrict__ block_hist,
    uint32_t* err) {
  __shared__ int32_t hist[256];
  const int tid = threadIdx.x;
  griddep_launch_dependents();
  griddep_wait();
  for (int e = tid; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int base = blockIdx.x * kRouteChunk;
  // All of this thread's ids are loaded before any is counted (one round trip).
  constexpr int kPer = kRouteChunk / kRouteThreads;
  int v[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int s = base + tid + u * kRouteThreads;
    v[u] = s < S ? __ldg(&idx[s]) : kMaskedSlot;
  }
  bool bad = false;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int e = v[u];
    if (e >= 0 && e < E) {
      atomicAdd(&hist[e], 1);
    } else if (e != kMaskedSlot) {
      bad = true;
    }
  }
  if (bad) atomicOr(err, kErrRoutingBit);
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) block_hist[blockIdx.x * E + e] = hist[e];
}

// Block-wide exclusive scans over the experts: thread e holds expert e's
// routed-slot count (0 for e >= E) and gets the expert's slot offset, padded
// m-tile offset and m-tile-pair offset, plus the inclusive values (the totals,
// at thread E - 1).  `part` is shared scratch; contains one block barrier.
struct ExpertOffsets {
  int slot, tile, pair;            // exclusive
  int slot_end, tile_end, pair_end;   // inclusive
};
__device__ __forceinline__ ExpertOffsets expert_offsets(int count,
                                                        int32_t (*part)[kRouteThreads / 32]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tiles = (count + kTileM - 1) / kTileM;
  const int pairs = (tiles + 1) / 2;
  int a = count, b = tiles, c = pairs;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int a2 = __shfl_up_sync(0xffffffffu, a, off);
    const int b2 = __shfl_up_sync(0xffffffffu, b, off);
    const int c2 = __shfl_up_sync(0xffffffffu, c, off);
    if (lane >= off) {
      a += a2;
      b += b2;
      c += c2;
    }
  }
  if (lane == 31) {
    part[0][warp] = a;
    part[1][warp] = b;
    part[2][warp] = c;
  }
  __syncthreads();
  for (int w = 0; w < warp; ++w) {
    a += part[0][w];
    b += part[1][w];
    c += part[2][w];
  }
  return {a - count, b - tiles, c - pairs, a, b, c};
}

// Rank a warp's slots among equal experts.  The warp owns `groups` groups of
// 32 consecutive slots (ids in v, one per lane and group; -1 for a masked or
// absent slot, any other id outside [0, E) is reported through `bad`) and
// keeps its running count per expert in `count[e]` (its own row of shared
// memory, zeroed by the caller).  On return v[u] holds (rank << 9) | e for a
// routed slot -- its rank among the warp's slots of expert e, in slot order --
// and kUnrouted otherwise.
constexpr int kUnrouted = -1;
template <int kPer>
__device__ __forceinline__ void rank_in_warp(int (&v)[kPer], int groups, int E,
                                             int32_t* count, bool& bad) {
  const int lane = threadIdx.x & 31;
  const unsigned lower = (1u << lane) - 1u;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    if (u >= groups) break;   // warp-uniform
    int e = v[u];
    if (!(e >= 0 && e < E)) {
      if (e != kMaskedSlot) bad = true;
      e = -1;
    }
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int before = e >= 0 ? count[e] : 0;
    __syncwarp();   // every lane has read its count before the group's leader updates it
    if (e >= 0 && (peers & lower) == 0) count[e] = before + __popc(peers);
    __syncwarp();
    v[u] = e >= 0 ? ((before + __popc(peers & lower)) << 9) | e : kUnrouted;
  }
}

// Kernel 2: scan + stable scatter.  Every block re-derives, from the block
// histograms, the per-expert totals, the exclusive scans over experts and its
// own starting position per expert (the histograms are small, so this costs
// less than a separate scan launch); block 0 publishes counts / offsets and
// the padded tile offsets.  Inside the block, warp w owns 256 consecutive
// slots and ranks them with rank_in_warp; a slot's sorted position is the
// block's start for its expert + the expert's slots in lower warps + its rank
// in the warp, i.e. ascending slot order within every expert.
__global__ void __launch_bounds__(kRouteThreads) route_scatter_kernel(
    const int32_t* __restrict__ idx, int S, int E, int nblk,
    const int32_t* __restrict__ block_hist, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ tile_off, int32_t* __restrict__ pad_off,
    int32_t* __restrict__ pair_off,
    int32_t* __restrict__ perm, int32_t* __restrict__ inv, uint32_t* err,
    uint32_t* __restrict__ sched, int sched_words, int32_t* __restrict__ row_token, int k) {
  constexpr int kWarps = kRouteThreads / 32;
  constexpr int kPer = kRouteChunk / kRouteThreads;   // 32-slot groups per warp
  griddep_launch_dependents();
  griddep_wait();
  // Block 0 also zeroes the fused GEMM's tile counter and per-m-tile
  // completion counts (sched may be null when no GEMM follows).
  if (blockIdx.x == 0 && sched != nullptr)
    for (int i = threadIdx.x; i < sched_words; i += blockDim.x) sched[i] = 0u;
  __shared__ int32_t wpre[kWarps][256];   // per warp and expert: count, then lower warps' count
  __shared__ int32_t start[256];          // this block's first position per expert
  __shared__ int32_t total[257];
  __shared__ int32_t scan[257];
  __shared__ int32_t tscan[257];          // padded m-tile offsets
  __shared__ int32_t part[3][kWarps];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int base = blockIdx.x * kRouteChunk;
  const int wbase = base + warp * (kRouteChunk / kWarps);
  // The warp's ids, loaded once up front (their latency overlaps the
  // histogram sums below).
  int v[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int s = wbase + u * 32 + lane;
    v[u] = s < S ? __ldg(&idx[s]) : kMaskedSlot;
  }
  for (int e = lane; e < E; e += 32) wpre[warp][e] = 0;
  // Thread e: expert e's slots in earlier blocks and in all blocks.
  int before = 0, all = 0;
  if (nblk > 1 && tid < E) {
    for (int b = 0; b < nblk; ++b) {
      const int c = block_hist[b * E + tid];
      if (b < static_cast<int>(blockIdx.x)) before += c;
      all += c;
    }
  }
  __syncwarp();
  bool bad = false;
  rank_in_warp<kPer>(v, kPer, E, wpre[warp], bad);
  // With a single block nothing else has looked at the ids.
  if (nblk == 1 && bad) atomicOr(err, kErrRoutingBit);
  __syncthreads();
  int mine = 0;   // this block's slots of expert tid
  if (tid < E) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int c = wpre[w][tid];
      wpre[w][tid] = mine;
      mine += c;
    }
  }
  if (nblk == 1) all = mine;
  const ExpertOffsets o = expert_offsets(tid < E ? all : 0, part);
  if (tid < E) {
    total[tid] = all;
    scan[tid] = o.slot;
    tscan[tid] = o.tile;
    start[tid] = o.slot + before;
    if (blockIdx.x == 0) {
      offsets[tid] = o.slot;
      counts[tid] = all;
      tile_off[tid] = o.tile;
      pad_off[tid] = o.tile * kTileM;
      if (pair_off != nullptr) pair_off[tid] = o.pair;   // pairs of m-tiles of one expert
    }
    if (tid == E - 1) {
      scan[E] = o.slot_end;
      tscan[E] = o.tile_end;
      if (blockIdx.x == 0) {
        offsets[E] = o.slot_end;
        tile_off[E] = o.tile_end;
        pad_off[E] = o.tile_end * kTileM;
        if (pair_off != nullptr) pair_off[E] = o.pair_end;
      }
    }
  }
  __syncthreads();
  // Padding rows of the row -> token map read -1 (experts split over blocks).
  if (row_token != nullptr) {
    for (int e = blockIdx.x + warp * gridDim.x; e < E; e += kWarps * gridDim.x) {
      const int lo = tscan[e] * kTileM + total[e], hi = tscan[e + 1] * kTileM;
      for (int r = lo + lane; r < hi; r += 32) row_token[r] = -1;
    }
  }
  // Positions past the routed slots (left by out-of-range ids) read -1.
  const int routed = scan[E];
  for (int p = base + tid; p < base + kRouteChunk && p < S; p += blockDim.x)
    if (p >= routed) perm[p] = -1;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int s = wbase + u * 32 + lane;
    if (s >= S) continue;
    if (v[u] != kUnrouted) {
      const int e = v[u] & 511;
      const int pos = start[e] + wpre[warp][e] + (v[u] >> 9);
      if (pos >= 0 && pos < S) {   // always true; guards the store
        perm[pos] = s;
        inv[s] = pos;
        if (row_token != nullptr) row_token[tscan[e] * kTileM + (pos - scan[e])] = s / k;
      } else {
        atomicOr(err, kErrRoutingBit);
        inv[s] = -1;
      }
    } else {
      inv[s] = -1;
    }
  }
}

// Gather, token-major: one warp per token.  The token's x row is read once
// (in chunks of 8 x 16 bytes per lane) and written to the padded row of each
// of its routed slots: slot s = t*k + j at sorted position inv[s] of expert e
// (the e with offsets[e] <= inv[s] < offsets[e+1]) goes to padded row
// pad_off[e] + inv[s] - offsets[e] (m-tile P / 128, row P % 128), in the
// pre-swizzled tile layout the FC1 producer bulk-copies.  Its scale bytes go
// to the token scale-chunk layout (sf_byte: one 512-byte chunk per tile and
// group of four k-blocks, row r's four bytes at (r % 32) * 16 + (r / 32) * 4).
// Padding rows are left untouched (their results are never stored).  Reading
// x once per token instead of once per slot matters when x does not fit in L2.
constexpr int kGatherWarps = 8;
constexpr int kGatherBatch = 8;   // 16-byte vectors per lane per chunk

__global__ void __launch_bounds__(kGatherWarps * 32) gather_kernel(
    const uint8_t* __restrict__ x, const uint8_t* __restrict__ xs, int row_bytes, int T, int k,
    int E, const int32_t* __restrict__ offsets, const int32_t* __restrict__ pad_off,
    const int32_t* __restrict__ inv, uint8_t* __restrict__ xg, uint8_t* __restrict__ xg_sf) {
  __shared__ int32_t s_off[257];
  __shared__ int32_t s_pad[257];
  griddep_launch_dependents();
  griddep_wait();
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    s_off[e] = __ldg(&offsets[e]);
    s_pad[e] = __ldg(&pad_off[e]);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kGatherWarps + warp;
  if (t >= T) return;
  const int vec = row_bytes / 16;
  const int kb_n = row_bytes / 128;
  const uint4* __restrict__ src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * row_bytes);
  for (int j0 = 0; j0 < k; j0 += 32) {
    // Lane l resolves slot j0 + l's padded row (-1: not routed).
    int prow = -1;
    if (j0 + lane < k) {
      const int pos = __ldg(&inv[static_cast<size_t>(t) * k + j0 + lane]);
      if (pos >= 0) {
        int lo = 0, hi = E - 1;   // largest e with offsets[e] <= pos
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (s_off[mid] <= pos) lo = mid; else hi = mid - 1;
        }
        prow = s_pad[lo] + (pos - s_off[lo]);
      }
    }
    const int nj = min(32, k - j0);
    for (int c0 = 0; c0 < vec; c0 += 32 * kGatherBatch) {
      uint4 v[kGatherBatch];
#pragma unroll
      for (int u = 0; u < kGatherBatch; ++u) {
        const int c = c0 + lane + 32 * u;
        if (c < vec) v[u] = __ldg(&src[c]);
      }
      for (int jj = 0; jj < nj; ++jj) {
        const int P = __shfl_sync(0xffffffffu, prow, jj);
        if (P < 0) continue;
        uint8_t* __restrict__ dst =
            xg + static_cast<size_t>(P / kTileM) * kb_n * kTileBytes;
        const int r = P % kTileM;
#pragma unroll
        for (int u = 0; u < kGatherBatch; ++u) {
          const int c = c0 + lane + 32 * u;
          if (c < vec)
            *reinterpret_cast<uint4*>(dst + static_cast<size_t>(c >> 3) * kTileBytes +
                                      swz128(r, c & 7)) = v[u];
        }
      }
    }
    if (xs == nullptr) continue;   // BF16 activations: no scales
    for (int jj = 0; jj < nj; ++jj) {
      const int P = __shfl_sync(0xffffffffu, prow, jj);
      if (P < 0) continue;
      const int r = P % kTileM;
      const int groups = sf_groups(kb_n);
      uint8_t* chunk = xg_sf + static_cast<size_t>(P / kTileM) * groups * 512 + sf_byte(r, 0);
      for (int g = lane; g < groups; g += 32)
        *reinterpret_cast<uint32_t*>(chunk + static_cast<size_t>(g) * 512) =
            sf_group_word(xs + static_cast<size_t>(t) * kb_n, kb_n, g);
    }
  }
}

// Routing and gather in one launch, for small slot counts (S <= kFusedMaxSlots):
// every block repeats the counting sort for all S slots, so no block waits for
// another; block 0 also publishes what the separate routing launch writes
// (counts, offsets, tile / pad / pair offsets, perm, inv, the row -> token map,
// the zeroed GEMM counters, the error bit).  Then each warp copies routed rows:
// sorted position pos of expert e goes to padded row 128 * tile_off[e] + pos -
// offsets[e], from token perm[pos] / k, in the same tiled layout and scale
// chunks as gather_kernel.  The bytes written equal those of the two separate
// launches.
//
// The sort is warp-local until one block-wide scan: warp w owns the contiguous
// slots [w * C, (w + 1) * C) and walks them 32 at a time, ranking each slot
// among the group's equal experts with __match_any_sync and keeping a running
// count per expert in its own row of shared memory (warp-synchronous, no block
// barrier per group).  A slot's sorted position is then the expert's offset,
// plus the slots of that expert in lower warps, plus its rank inside the warp:
// ascending slot order within each expert, as the stable scatter requires.
// Thread e computes expert e's totals, and the exclusive scans over experts
// (slots, padded m-tiles, m-tile pairs) are block scans over those threads.
__global__ void __launch_bounds__(kRouteThreads) route_gather_kernel(
    const int32_t* __restrict__ idx, int S, int E, int k, const uint8_t* __restrict__ x,
    const uint8_t* __restrict__ xs, int row_bytes, int32_t* __restrict__ counts,
    int32_t* __restrict__ offsets, int32_t* __restrict__ tile_off, int32_t* __restrict__ pad_off,
    int32_t* __restrict__ pair_off, int32_t* __restrict__ perm, int32_t* __restrict__ inv,
    uint32_t* err, uint32_t* __restrict__ sched, int sched_words,
    int32_t* __restrict__ row_token, uint8_t* __restrict__ xg, uint8_t* __restrict__ xg_sf) {
  constexpr int kWarps = kRouteThreads / 32;
  constexpr int kPer = kFusedMaxSlots / kRouteThreads;   // 32-slot groups per warp, at most
  extern __shared__ int32_t sorted[];   // [S] slot at each sorted position
  __shared__ int32_t wpre[kWarps][256];  // per warp and expert: count, then lower warps' count
  __shared__ int32_t total[257];
  __shared__ int32_t scan[257];
  __shared__ int32_t tscan[257];        // padded m-tile offsets
  __shared__ int32_t part[3][kWarps];   // per-warp sums for the block scans
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool lead = blockIdx.x == 0;
  const int chunk = (S + 32 * kWarps - 1) / (32 * kWarps) * 32;   // slots per warp
  griddep_launch_dependents();
  griddep_wait();
  if (lead && sched != nullptr)
    for (int i = tid; i < sched_words; i += blockDim.x) sched[i] = 0u;
  for (int e = lane; e < E; e += 32) wpre[warp][e] = 0;
  // This warp's ids, all loaded before any is used (one round trip).
  int v[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int s = warp * chunk + u * 32 + lane;
    v[u] = u * 32 < chunk && s < S ? __ldg(&idx[s]) : kMaskedSlot;
  }
  __syncwarp();
  bool bad = false;
  rank_in_warp<kPer>(v, chunk / 32, E, wpre[warp], bad);
  if (lead && bad) atomicOr(err, kErrRoutingBit);
  __syncthreads();
  // Thread e: expert e's total, and its per-warp counts turned into the count
  // of expert e in lower warps.
  int tot = 0;
  if (tid < E) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const int c = wpre[w][tid];
      wpre[w][tid] = tot;
      tot += c;
    }
    total[tid] = tot;
  }
  const ExpertOffsets o = expert_offsets(tot, part);
  if (tid < E) {
    scan[tid] = o.slot;
    tscan[tid] = o.tile;
    if (lead) {
      offsets[tid] = o.slot;
      counts[tid] = tot;
      tile_off[tid] = o.tile;
      pad_off[tid] = o.tile * kTileM;
      pair_off[tid] = o.pair;
    }
    if (tid == E - 1) {
      scan[E] = o.slot_end;
      tscan[E] = o.tile_end;
      if (lead) {
        offsets[E] = o.slot_end;
        tile_off[E] = o.tile_end;
        pad_off[E] = o.tile_end * kTileM;
        pair_off[E] = o.pair_end;
      }
    }
  }
  __syncthreads();
  const int routed = scan[E];
  if (lead) {
    // Padding rows of the row -> token map read -1; so do positions past the
    // routed slots (left by masked or out-of-range ids).
    for (int e = warp; e < E; e += kWarps) {
      const int lo = tscan[e] * kTileM + total[e], hi = tscan[e + 1] * kTileM;
      for (int r = lo + lane; r < hi; r += 32) row_token[r] = -1;
    }
    for (int q = routed + tid; q < S; q += blockDim.x) perm[q] = -1;
  }
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    if (u * 32 >= chunk) break;
    const int s = warp * chunk + u * 32 + lane;
    if (s >= S) continue;
    if (v[u] != kUnrouted) {
      const int e = v[u] & 511;
      const int q = scan[e] + wpre[warp][e] + (v[u] >> 9);
      sorted[q] = s;   // q < routed <= S: the counts above bound it
      if (lead) {
        perm[q] = s;
        inv[s] = q;
        row_token[tscan[e] * kTileM + (q - scan[e])] = s / k;
      }
    } else if (lead) {
      inv[s] = -1;
    }
  }
  __syncthreads();
  // Gather: one warp per routed row; all loads of a row are issued before its
  // stores.
  const int kb_n = row_bytes / 128;   // 128-byte k-blocks per row (scale blocks when FP8)
  const int vec = row_bytes / 16;
  const bool scales = xs != nullptr;  // BF16 activations carry none
  for (int q = blockIdx.x * kWarps + warp; q < routed; q += gridDim.x * kWarps) {
    int lo = 0, hi = E - 1;   // expert of sorted position q: largest e with scan[e] <= q
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (scan[mid] <= q) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const long long P = static_cast<long long>(tscan[e]) * kTileM + (q - scan[e]);
    const int t = sorted[q] / k;
    const int tile = static_cast<int>(P / kTileM);
    const int r = static_cast<int>(P % kTileM);
    const uint4* __restrict__ src =
        reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * row_bytes);
    uint8_t* __restrict__ dst = xg + static_cast<size_t>(tile) * kb_n * kTileBytes;
    // Rows of up to 8192 bytes move in one batch of loads; the scale words of
    // up to 64 groups (256 k-blocks) are loaded with them.
    constexpr int kBatch = 16;
    const int groups = sf_groups(kb_n);
    uint8_t* chunk = xg_sf + static_cast<size_t>(tile) * groups * 512 + sf_byte(r, 0);
    const uint8_t* row_sf = scales ? xs + static_cast<size_t>(t) * kb_n : nullptr;
    for (int c0 = lane; c0 < vec; c0 += 32 * kBatch) {
      uint4 xv[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int c = c0 + 32 * u;
        if (c < vec) xv[u] = __ldg(&src[c]);
      }
      uint32_t sb[2] = {0u, 0u};
      if (scales && c0 == lane) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int g = lane + 32 * u;
          if (g < groups) sb[u] = sf_group_word(row_sf, kb_n, g);
        }
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int c = c0 + 32 * u;
        if (c < vec)
          *reinterpret_cast<uint4*>(dst + static_cast<size_t>(c >> 3) * kTileBytes +
                                    swz128(r, c & 7)) = xv[u];
      }
      if (scales && c0 == lane) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int g = lane + 32 * u;
          if (g < groups)
            *reinterpret_cast<uint32_t*>(chunk + static_cast<size_t>(g) * 512) = sb[u];
        }
      }
    }
    for (int g = lane + 64; scales && g < groups; g += 32)   // rows of more than 256 k-blocks
      *reinterpret_cast<uint32_t*>(chunk + static_cast<size_t>(g) * 512) =
          sf_group_word(row_sf, kb_n, g);
  }
}

// Unpack the FC1 activation's scale chunks to a plain u8 [rows, I/128] array.
__global__ void unpack_act_scales_kernel(const uint8_t* __restrict__ chunks, int nb,
                                         long long rows, uint8_t* __restrict__ dst) {
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (i >= rows * nb) return;
  const long long r = i / nb;
  const int b = static_cast<int>(i - r * nb);
  const long long tile = r / kTileM;
  const int rr = static_cast<int>(r - tile * kTileM);
  dst[i] = chunks[tile * sf_groups(nb) * 512 + sf_byte(rr, b)];
}

}  // namespace

cudaError_t launch_route(const moe_plan_s* p, const int32_t* topk_idx, uint8_t* ws,
                         cudaStream_t st) {
  const auto& L = p->ws;
  const int S = static_cast<int>(p->S);
  if (p->route_blocks > 1) {
    cudaError_t e = launch_pdl(route_hist_kernel, dim3(p->route_blocks), dim3(kRouteThreads), 0,
                               st, topk_idx, S, p->E,
                               reinterpret_cast<int32_t*>(ws + L.block_hist),
                               reinterpret_cast<uint32_t*>(ws + L.err));
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(
      route_scatter_kernel, dim3(p->route_blocks), dim3(kRouteThreads), 0, st, topk_idx, S,
      p->E, p->route_blocks, reinterpret_cast<const int32_t*>(ws + L.block_hist),
      reinterpret_cast<int32_t*>(ws + L.counts), reinterpret_cast<int32_t*>(ws + L.offsets),
      reinterpret_cast<int32_t*>(ws + L.tile_off), reinterpret_cast<int32_t*>(ws + L.pad_off),
      reinterpret_cast<int32_t*>(ws + L.pair_off), reinterpret_cast<int32_t*>(ws + L.perm),
      reinterpret_cast<int32_t*>(ws + L.inv),
      reinterpret_cast<uint32_t*>(ws + L.err), reinterpret_cast<uint32_t*>(ws + L.sched),
      static_cast<int>(64 + p->rows_cap / kTileM), reinterpret_cast<int32_t*>(ws + L.row_token),
      p->k);
}

cudaError_t launch_gather(const moe_plan_s* p, const uint8_t* x, const uint8_t* xs, uint8_t* ws,
                          cudaStream_t st) {
  const auto& L = p->ws;
  const int blocks = (p->T + kGatherWarps - 1) / kGatherWarps;   // one warp per token
  const bool bf16 = p->w_dtype == MOE_W_BF16;   // 2-byte activations, no scales
  return launch_pdl(gather_kernel, dim3(blocks), dim3(kGatherWarps * 32), 0, st, x,
                    bf16 ? nullptr : xs, p->H * (bf16 ? 2 : 1), p->T, p->k, p->E,
                    reinterpret_cast<const int32_t*>(ws + L.offsets),
                    reinterpret_cast<const int32_t*>(ws + L.pad_off),
                    reinterpret_cast<const int32_t*>(ws + L.inv), ws + L.xg, ws + L.xg_sf);
}

cudaError_t launch_route_gather(const moe_plan_s* p, const int32_t* topk_idx, const uint8_t* x,
                                const uint8_t* xs, uint8_t* ws, cudaStream_t st) {
  const auto& L = p->ws;
  const int S = static_cast<int>(p->S);
  // One warp per routed row (at most S), two blocks per SM at most.
  const int sms = sm_count();
  const bool bf16 = p->w_dtype == MOE_W_BF16;   // 2-byte activations, no scales
  const int want = (S + kRouteThreads / 32 - 1) / (kRouteThreads / 32);
  const int blocks = std::max(1, std::min(want, 2 * sms));
  const int dyn = S * static_cast<int>(sizeof(int32_t));   // the sorted slot list
  if (dyn > 48 * 1024) {
    const cudaError_t a = ensure_max_dynamic_smem(
        reinterpret_cast<const void*>(route_gather_kernel),
        kFusedMaxSlots * static_cast<int>(sizeof(int32_t)));
    if (a != cudaSuccess) return a;
  }
  return launch_pdl(
      route_gather_kernel, dim3(blocks), dim3(kRouteThreads), dyn, st,
      topk_idx, S, p->E, p->k, x, bf16 ? nullptr : xs, p->H * (bf16 ? 2 : 1),
      reinterpret_cast<int32_t*>(ws + L.counts),
      reinterpret_cast<int32_t*>(ws + L.offsets), reinterpret_cast<int32_t*>(ws + L.tile_off),
      reinterpret_cast<int32_t*>(ws + L.pad_off), reinterpret_cast<int32_t*>(ws + L.pair_off),
      reinterpret_cast<int32_t*>(ws + L.perm), reinterpret_cast<int32_t*>(ws + L.inv),
      reinterpret_cast<uint32_t*>(ws + L.err), reinterpret_cast<uint32_t*>(ws + L.sched),
      static_cast<int>(64 + p->rows_cap / kTileM), reinterpret_cast<int32_t*>(ws + L.row_token),
      ws + L.xg, ws + L.xg_sf);
}

cudaError_t launch_unpack_act_scales(const moe_plan_s* p, const uint8_t* ws, uint8_t* dst,
                                     cudaStream_t st) {
  const long long n = p->rows_cap * (p->I / 128);
  const int blocks = static_cast<int>((n + 255) / 256);
  return launch_plain(unpack_act_scales_kernel, dim3(blocks), dim3(256), 0, st,
                      static_cast<const uint8_t*>(ws + p->ws.act_sf), p->I / 128, p->rows_cap, dst);
}

}  // namespace moe

// ---------------------------------------------------------------------------
// Allocation-free routing (moe_route_static in include/moe.h).
//
// Some callers cannot allocate device memory at the point where they route: a
// serving runtime whose pooled allocator owns the whole device budget, or a
// latency-critical loop in which a device allocation could synchronise the
// device.  For them the routing step can take its scratch (the per-block
// histograms, the padded tile offsets and the error word) from a buffer that
// lives in this module's static device memory, sized once for at most
// MOE_ROUTE_STATIC_MAX_SLOTS slots and kept by every GPU that loads the library
// until the process exits.  The routing kernels themselves are the ones above;
// only where their scratch lives differs.
namespace moe {
namespace {

constexpr long long kStaticMaxSlots = MOE_ROUTE_STATIC_MAX_SLOTS;
constexpr size_t kStaticErrOff = 0;
constexpr size_t kStaticTileOff = 256;
constexpr size_t kStaticPadOff = kStaticTileOff + 257 * 4 + 252;   // 256-B aligned
constexpr size_t kStaticHistOff = kStaticPadOff + 257 * 4 + 252;
constexpr size_t kStaticHistBytes =
    static_cast<size_t>((kStaticMaxSlots + kRouteChunk - 1) / kRouteChunk) * 256 * 4;
constexpr size_t kStaticScratchBytes = kStaticHistOff + kStaticHistBytes;   // ~515 KiB

// Host code must not hand this name to a kernel: on the host it is only a
// stand-in for the symbol.  Its device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_route_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
uint8_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of the static scratch on the current device, looked up once
// per device (with that device current) and cached.
cudaError_t static_scratch(uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_route_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<uint8_t*>(ptr);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_route_static(const int32_t* topk_idx, int T, int k, int E,
                                       int32_t* counts, int32_t* offsets, int32_t* perm,
                                       int32_t* inv, moe_stream_t stream) {
  using namespace moe;
  if (topk_idx == nullptr || counts == nullptr || offsets == nullptr || perm == nullptr ||
      inv == nullptr)
    return MOE_ERR_INVALID_ARG;
  if (T < 1 || k < 1 || E < 1 || k > E) return MOE_ERR_INVALID_ARG;
  if (E > 256) return MOE_ERR_UNSUPPORTED;
  const long long S = static_cast<long long>(T) * k;
  if (S > kStaticMaxSlots) return MOE_ERR_UNSUPPORTED;   // beyond the static scratch
  for (const void* p : {static_cast<const void*>(topk_idx), static_cast<const void*>(counts),
                        static_cast<const void*>(offsets), static_cast<const void*>(perm),
                        static_cast<const void*>(inv)})
    if (reinterpret_cast<uintptr_t>(p) % 4 != 0) return MOE_ERR_ALIGNMENT;
  uint8_t* scratch = nullptr;
  if (static_scratch(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  auto st = reinterpret_cast<cudaStream_t>(stream);
  const int nblk = static_cast<int>((S + kRouteChunk - 1) / kRouteChunk);
  // The error word keeps the previous call's bits: clear it first.
  if (cudaMemsetAsync(scratch + kStaticErrOff, 0, 4, st) != cudaSuccess) return MOE_ERR_CUDA;
  auto err = reinterpret_cast<uint32_t*>(scratch + kStaticErrOff);
  auto hist = reinterpret_cast<int32_t*>(scratch + kStaticHistOff);
  // Each launch's own status is checked (an earlier, unrelated launch error is
  // neither reported here nor cleared).
  if (nblk > 1 &&
      launch_plain(route_hist_kernel, dim3(nblk), dim3(kRouteThreads), 0, st, topk_idx,
                   static_cast<int>(S), E, hist, err) != cudaSuccess)
    return MOE_ERR_CUDA;
  const cudaError_t e = launch_plain(
      route_scatter_kernel, dim3(nblk), dim3(kRouteThreads), 0, st, topk_idx,
      static_cast<int>(S), E, nblk, static_cast<const int32_t*>(hist), counts, offsets,
      reinterpret_cast<int32_t*>(scratch + kStaticTileOff),
      reinterpret_cast<int32_t*>(scratch + kStaticPadOff), static_cast<int32_t*>(nullptr), perm,
      inv, err, static_cast<uint32_t*>(nullptr), 0, static_cast<int32_t*>(nullptr), k);
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
