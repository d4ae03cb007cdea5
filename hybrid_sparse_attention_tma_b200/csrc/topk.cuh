// topk.cuh -- per-(tile, KV head) top-k selection over importance scores.
//
// TopK over the full layer's block scores (HySparse explainer, techwalker.com)
// or token scores with k = 1024 (HySparse2 release note; demingchina
// commentary section 03). Candidates of a tile are the blocks b with
// b*B <= last query position of the tile, or (window-exclusive reading) only
// those starting before the last query's forced window, b*B <= last - w.
// Rule: score descending, ties to the lower index; the kept set is written in
// ascending index order, padded -1.
//
// Method: scores are >= 0, so their fp32 bit patterns order like the values.
// A 4-pass MSB-first radix select (8 bits per pass, per-warp histograms in
// shared memory) finds the k-th largest bit pattern tau and how many of the
// k slots go to entries equal to tau. A final compaction over the row in
// index order (each thread a contiguous segment, one block scan) keeps every
// entry > tau plus the first (k - #greater) entries == tau. Index order both
// breaks ties toward the lower index and emits the result already sorted.
//
// Two shapes of the same kernel: rows of up to kStageMax candidates are
// staged once in shared memory by a 256-thread CTA (block-level selection,
// short rows, many CTAs per SM); longer rows (token level) are streamed from
// global memory / L2 by a 1024-thread CTA.
#pragma once

#include "hs_common.cuh"
#include "seqtable.cuh"

namespace hs {
namespace topk {

constexpr int kStageMax = 8192;  // candidates staged in shared memory (32 KB)

struct Params {
  const float* scores;  // [n_tiles, Hkv, nblk]
  int* idx;             // [n_tiles, Hkv, k]
  int* cnt;             // [n_tiles, Hkv]
  int Hkv, nblk, B, k;
  int w, exclusive;  // forced window; 1 = candidates stop before the last query's window
};

// Block-wide exclusive scan of one int per thread; returns the total.
template <int THREADS>
__device__ __forceinline__ int block_excl_scan(int v, int* warp_sums, int& total) {
  constexpr int kWarps = THREADS / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int s = lane < kWarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += y;
    }
    if (lane < kWarps) warp_sums[lane] = s;  // inclusive
  }
  __syncthreads();
  total = warp_sums[kWarps - 1];
  const int base = warp > 0 ? warp_sums[warp - 1] : 0;
  __syncthreads();
  return base + x - v;
}

template <int THREADS, bool STAGED>
__global__ void __launch_bounds__(THREADS)
    topk_kernel(const Params p, const __grid_constant__ SeqTable st) {
  constexpr int kWarps = THREADS / 32;
  __shared__ int hist[kWarps][256];
  __shared__ int warp_sums[32];
  __shared__ uint32_t s_prefix;
  __shared__ int s_krem;
  __shared__ uint32_t staged[STAGED ? kStageMax : 1];

  const int row = blockIdx.x;  // tile * Hkv + g
  const int tile = row / p.Hkv;
  const TileInfo ti = tile_info(st, tile);
  const int last_pos = ti.pos0 + ti.n - 1;
  const int lim = p.exclusive ? last_pos - p.w : last_pos;  // candidates: b * B <= lim
  const int n = lim < 0 ? 0 : min(p.nblk, lim / p.B + 1);
  const uint32_t* gkeys = reinterpret_cast<const uint32_t*>(p.scores + size_t(row) * p.nblk);
  int* out = p.idx + size_t(row) * p.k;
  const int k = p.k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  if (n <= k) {
    // every candidate is kept
    for (int j = threadIdx.x; j < k; j += THREADS) out[j] = j < n ? j : -1;
    if (threadIdx.x == 0) p.cnt[row] = n;
    return;
  }
  if (k == 0) {
    if (threadIdx.x == 0) p.cnt[row] = 0;
    return;
  }
  if constexpr (STAGED) {
    for (int j = threadIdx.x; j < n; j += THREADS) staged[j] = __ldg(gkeys + j);
    __syncthreads();
  }
  auto key_at = [&](int j) -> uint32_t {
    if constexpr (STAGED) return staged[j];
    else return __ldg(gkeys + j);
  };

  // ---- radix select of the k-th largest bit pattern ----
  uint32_t prefix = 0;  // fixed high bits of tau
  int krem = k;         // how many of the k still to place at/below the prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int b = lane; b < 256; b += 32) hist[warp][b] = 0;
    __syncwarp();
    for (int j = threadIdx.x; j < n; j += THREADS) {
      const uint32_t key = key_at(j);
      if ((key & hi_mask) == prefix) atomicAdd(&hist[warp][(key >> shift) & 0xFF], 1);
    }
    __syncthreads();
    // bins reduced across warps; warp 0 finds the bucket holding the krem-th largest
    if (warp == 0) {
      int cnt8[8];
      int tot = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {  // lane handles bins 255 - (lane*8 + e), descending
        const int b = 255 - (lane * 8 + e);
        int s = 0;
        for (int w = 0; w < kWarps; ++w) s += hist[w][b];
        cnt8[e] = s;
        tot += s;
      }
      // inclusive prefix of the per-lane totals (descending bin order)
      int inc = tot;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += y;
      }
      const int excl = inc - tot;
      // the lane whose range crosses krem owns the bucket
      const bool mine = excl < krem && inc >= krem;
      if (mine) {
        int acc = excl, e = 0;
        for (; e < 7; ++e) {
          if (acc + cnt8[e] >= krem) break;
          acc += cnt8[e];
        }
        const int b = 255 - (lane * 8 + e);
        s_prefix = prefix | (uint32_t(b) << shift);
        s_krem = krem - acc;
      }
    }
    __syncthreads();
    prefix = s_prefix;
    krem = s_krem;
  }
  const uint32_t tau = prefix;
  const int take_eq = krem;  // entries equal to tau to keep (lowest indices)

  // ---- ordered compaction ----
  // Thread t owns the contiguous segment [t*L, t*L + L) of the row: it counts
  // its entries > tau and == tau, one pair of block scans gives every thread
  // its output offset and the number of tau-entries before it, and a second
  // walk writes the kept indices. Segments are in index order, so the output
  // is ascending and ties go to the lowest indices.
  const int L = (n + THREADS - 1) / THREADS;
  const int j0 = min(n, threadIdx.x * L), j1 = min(n, j0 + L);
  int gt = 0, eq = 0;
  {
    // counting may go in any order: start each lane at a different offset so
    // staged (shared-memory) segments whose length is a multiple of 32 do not
    // put a warp's accesses in one bank
    const int len = j1 - j0;
    int off = len > 0 ? lane % len : 0;
    for (int c = 0; c < len; ++c) {
      const uint32_t key = key_at(j0 + off);
      gt += key > tau ? 1 : 0;
      eq += key == tau ? 1 : 0;
      off = off + 1 == len ? 0 : off + 1;
    }
  }
  int gt_total, eq_total;
  const int gt_before = block_excl_scan<THREADS>(gt, warp_sums, gt_total);
  const int eq_before = block_excl_scan<THREADS>(eq, warp_sums, eq_total);
  int pos = gt_before + min(eq_before, take_eq);
  int eq_seen = eq_before;
  if (gt > 0 || (eq > 0 && eq_before < take_eq)) {
    for (int j = j0; j < j1; ++j) {
      const uint32_t key = key_at(j);
      if (key > tau) {
        out[pos++] = j;
      } else if (key == tau) {
        if (eq_seen < take_eq) out[pos++] = j;
        ++eq_seen;
      }
    }
  }
  const int out_base = gt_total + min(eq_total, take_eq);
  for (int j = out_base + threadIdx.x; j < k; j += THREADS) out[j] = -1;
  if (threadIdx.x == 0) p.cnt[row] = out_base;
}

}  // namespace topk
}  // namespace hs
