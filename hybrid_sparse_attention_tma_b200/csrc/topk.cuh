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
// index order (each warp a contiguous range walked 32 keys at a time, one
// scan over the warps, ballots inside a warp) keeps every entry > tau plus
// the first (k - #greater) entries == tau. Index order both breaks ties
// toward the lower index and emits the result already sorted.
//
// The row selection is a device function over any number of whole warps and
// any barrier: the kernel below runs it per CTA, and the token-score pass
// runs it on two of its warps for the fused top-k.
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

// Shared scratch of one row selection (kWarps per-warp histograms).
template <int THREADS>
struct SelScratch {
  int hist[THREADS / 32][256];
  int warp_sums[32];
  uint32_t prefix;
  int krem;
};

// Exclusive scan of one int per thread over THREADS threads (t = 0 ..
// THREADS - 1, whole warps) with `sync()` as their barrier; returns the total.
template <int THREADS, typename Sync>
__device__ __forceinline__ int group_excl_scan(int v, int t, int* warp_sums, int& total, Sync sync) {
  constexpr int kWarps = THREADS / 32;
  const int lane = t & 31, warp = t >> 5;
  int x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  sync();
  if (warp == 0) {
    int s = lane < kWarps ? warp_sums[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += y;
    }
    if (lane < kWarps) warp_sums[lane] = s;  // inclusive
  }
  sync();
  total = warp_sums[kWarps - 1];
  const int base = warp > 0 ? warp_sums[warp - 1] : 0;
  sync();
  return base + x - v;
}

// Top-k of one row of n candidates, run by THREADS threads (t = 0 .. THREADS
// - 1, whole warps) with `sync()` as their barrier; key(j) is the fp32 bit
// pattern of candidate j (scores are >= 0, so bit order is value order).
// Writes out[0 .. k) (kept indices ascending, padded -1) and *cnt_out.
template <int THREADS, int kU = 8, typename Key, typename Sync>
__device__ void select_row(int n, int k, int t, Key key_at, Sync sync, SelScratch<THREADS>& sc, int* out,
                           int* cnt_out) {
  constexpr int kWarps = THREADS / 32;
  const int lane = t & 31, warp = t >> 5;
  if (n <= k) {
    // every candidate is kept
    for (int j = t; j < k; j += THREADS) out[j] = j < n ? j : -1;
    if (t == 0) *cnt_out = n;
    return;
  }
  if (k == 0) {
    if (t == 0) *cnt_out = 0;
    return;
  }
  // ---- radix select of the k-th largest bit pattern ----
  uint32_t prefix = 0;  // fixed high bits of tau
  int krem = k;         // how many of the k still to place at/below the prefix
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + 8));
    for (int b = lane; b < 256; b += 32) sc.hist[warp][b] = 0;
    __syncwarp();
    // kU loads in flight per thread before their histogram updates (rows read
    // from L2 are latency-bound); consecutive threads read consecutive keys
    for (int j0 = t; j0 < n; j0 += kU * THREADS) {
      uint32_t kk[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) kk[u] = j0 + u * THREADS < n ? key_at(j0 + u * THREADS) : 0u;
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (j0 + u * THREADS < n && (kk[u] & hi_mask) == prefix) atomicAdd(&sc.hist[warp][(kk[u] >> shift) & 0xFF], 1);
    }
    sync();
    // bins reduced across warps; warp 0 finds the bucket holding the krem-th largest
    if (warp == 0) {
      int cnt8[8];
      int tot = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) {  // lane handles bins 255 - (lane*8 + e), descending
        const int b = 255 - (lane * 8 + e);
        int s = 0;
        for (int w = 0; w < kWarps; ++w) s += sc.hist[w][b];
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
        sc.prefix = prefix | (uint32_t(b) << shift);
        sc.krem = krem - acc;
      }
    }
    sync();
    prefix = sc.prefix;
    krem = sc.krem;
    sync();  // every thread has read them before the next pass overwrites
  }
  const uint32_t tau = prefix;
  const int take_eq = krem;  // entries equal to tau to keep (lowest indices)

  // ---- ordered compaction ----
  // Warp w owns the contiguous range [w*Lw, w*Lw + Lw) of the row (Lw a
  // multiple of 32) and walks it 32 keys at a time, lane l reading key
  // base + l (coalesced). A first walk counts the entries > tau and == tau
  // of each warp; a scan over the warps gives each warp its output offset and
  // the number of tau-entries before its range; the second walk writes the
  // kept indices, each lane finding its place among the 32 by ballots. Ranges
  // and lanes follow index order, so the output is ascending and ties go to
  // the lowest indices.
  const int Lw = ((n + kWarps - 1) / kWarps + 31) & ~31;
  const int w0 = min(n, warp * Lw), w1 = min(n, w0 + Lw);
  int gt = 0, eq = 0;
  for (int c0 = w0; c0 < w1; c0 += 32 * kU) {
    uint32_t kk[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) kk[u] = c0 + u * 32 + lane < w1 ? key_at(c0 + u * 32 + lane) : 0u;
#pragma unroll
    for (int u = 0; u < kU; ++u)
      if (c0 + u * 32 + lane < w1) {
        gt += kk[u] > tau ? 1 : 0;
        eq += kk[u] == tau ? 1 : 0;
      }
  }
  gt = __reduce_add_sync(0xffffffffu, gt);
  eq = __reduce_add_sync(0xffffffffu, eq);
  int gt_total, eq_total;
  const int gt_before = __shfl_sync(
      0xffffffffu, group_excl_scan<THREADS>(lane == 0 ? gt : 0, t, sc.warp_sums, gt_total, sync), 0);
  const int eq_before = __shfl_sync(
      0xffffffffu, group_excl_scan<THREADS>(lane == 0 ? eq : 0, t, sc.warp_sums, eq_total, sync), 0);
  if (gt > 0 || (eq > 0 && eq_before < take_eq)) {
    const uint32_t lt = (1u << lane) - 1u;
    int pos_run = gt_before + min(eq_before, take_eq);  // output slots before this chunk
    int eq_run = eq_before;                             // tau-entries before this chunk
    for (int c0 = w0; c0 < w1; c0 += 32 * kU) {
      uint32_t kk[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) kk[u] = c0 + u * 32 + lane < w1 ? key_at(c0 + u * 32 + lane) : 0u;
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int j = c0 + u * 32 + lane;
        const bool valid = j < w1;
        const bool e = valid && kk[u] == tau;
        const uint32_t be = __ballot_sync(0xffffffffu, e);
        const bool keep = (valid && kk[u] > tau) || (e && eq_run + __popc(be & lt) < take_eq);
        const uint32_t bk = __ballot_sync(0xffffffffu, keep);
        // pos < k always holds for a consistent selection; the bound keeps a
        // selection whose group barrier gave up (kernel aborting) inside out[]
        const int pos = pos_run + __popc(bk & lt);
        if (keep && pos < k) out[pos] = j;
        pos_run += __popc(bk);
        eq_run += __popc(be);
      }
    }
  }
  const int out_base = min(k, gt_total + min(eq_total, take_eq));
  for (int j = max(0, out_base) + t; j < k; j += THREADS) out[j] = -1;
  if (t == 0) *cnt_out = out_base;
}

// Candidates of selection tile `tile`: blocks b with b * B <= the tile's last
// query position (window-exclusive reading: <= last - w).
__device__ __forceinline__ int n_candidates(const TileInfo& ti, int nblk, int B, int w, int exclusive) {
  const int last_pos = ti.pos0 + ti.n - 1;
  const int lim = exclusive ? last_pos - w : last_pos;
  return lim < 0 ? 0 : min(nblk, lim / B + 1);
}

template <int THREADS, bool STAGED>
__global__ void __launch_bounds__(THREADS)
    topk_kernel(const Params p, const __grid_constant__ SeqTable st) {
  __shared__ SelScratch<THREADS> sc;
  __shared__ uint32_t staged[STAGED ? kStageMax : 1];
  const int row = blockIdx.x;  // tile * Hkv + g
  const TileInfo ti = tile_info(st, row / p.Hkv);
  const int n = n_candidates(ti, p.nblk, p.B, p.w, p.exclusive);
  const uint32_t* gkeys = reinterpret_cast<const uint32_t*>(p.scores + size_t(row) * p.nblk);
  if constexpr (STAGED) {
    if (n > p.k && p.k > 0) {
      for (int j = threadIdx.x; j < n; j += THREADS) staged[j] = __ldg(gkeys + j);
      __syncthreads();
    }
  }
  auto key_at = [&](int j) -> uint32_t {
    if constexpr (STAGED) return staged[j];
    else return __ldg(gkeys + j);
  };
  select_row<THREADS>(n, p.k, int(threadIdx.x), key_at, [] { __syncthreads(); }, sc, p.idx + size_t(row) * p.k,
                      p.cnt + row);
}

}  // namespace topk
}  // namespace hs
