// token_scores.cuh -- token-level importance scores of the full layer.
//
// score(t, g, j) = max over queries q of tile t, heads h of KV group g with
// j <= pos(q) of exp(s_{q,h,j} - lse_{q,h}) (token-level selection of
// HySparse2: the full layer's attention scores drive a top-1024 token choice,
// HySparse2 release note on airebao.com; the score formula is the reading
// used throughout this library). lse is final only after the forward pass,
// so the per-key maximum needs the logits again: this kernel recomputes
// S^T = K_blk * Q_tile^T with the KEYS on the MMA's M dimension. A thread then
// owns one key (one TMEM lane) and reduces over the row columns with one
// FFMA + one MAX per element -- no exponentials, no cross-lane traffic; a
// single exp2 per (tile, key) at the end.
//
// CTA: warp 0-3 reducers (thread = key), warp 4 TMA producer, warp 5 UMMA
// issuer. A work item is (tile, KV head, 256 keys): its 2 key blocks (128
// keys each) stay in shared memory while the tile's T*G query rows stream
// through a ring of 256-row chunks (with their lse), each block taking one
// M = 128, N = 256 MMA per K step: per FLOP that reads a quarter fewer
// operand bytes from shared memory than N = 128, whose port the operand
// reads alone would fill. TMEM holds one 128 x 256 fp32 accumulator per key
// block (2 x 256 columns).
//
// Fused top-k (SELECT): the top-k of a (tile, KV head) plane is taken inside
// this kernel (HySparse2 release note: the selection is a free by-product of
// the full layer). Items stay spread over all CTAs. The reducers of the item
// that completes a plane (a per-plane arrival counter) append the plane to a
// global queue of completed planes; two selector warps in every CTA take the
// next queue slot whenever they are free, wait for it to be filled, and run
// the row selection of topk.cuh on that plane's scores while they are still
// in L2, then drop those L2 lines without write-back, so the scores neither
// return from nor reach HBM. (Handing each plane to the CTA that completed it
// instead piles the selections onto the slowest CTA: every CTA holds items of
// every long plane, so the slowest one completes them all.) Tiles run longest
// first across all sequences, so the planes completed last, whose selection
// is not hidden behind other items, are the shortest.
#pragma once

#include "hs_common.cuh"
#include "seqtable.cuh"
#include "topk.cuh"

namespace hs {
namespace tscore {

constexpr int kThreads = 192;     // reducers (4 warps), producer, issuer
constexpr int kSelThreads = 64;   // selector warps of the fused top-k (8 warps in all: no register cap below 255)
template <bool SELECT>
constexpr int threads() { return SELECT ? kThreads + kSelThreads : kThreads; }
constexpr int kBlocks = 2;   // key blocks per item
constexpr int kRows = 256;   // query rows per chunk (the MMA's N)
constexpr int kQStagesMax = 3;
template <int D>
constexpr int q_stages() { return D == 128 ? 2 : 3; }  // 2 at d = 128 to fit the augmentation tiles
constexpr int kSlabBytes = 128 * 128;     // a 128-row x 64-column swizzled slab (K block)
constexpr int kQSlabBytes = kRows * 128;  // a kRows-row x 64-column slab (Q chunk)

struct Params {
  const float* lse;  // [Hq, Tq] natural log (from the forward pass)
  float* scores;     // [n_tiles, Hkv, nblk] (nblk = max_kv)
  int G, Hq, Hkv, Tq, nblk;
  float scale_log2;
  int n_items;
  WaitCtl wc;
  // fused top-k only (the work areas are set up by item_prefix_kernel)
  int* arrive;       // [n_tiles * Hkv] items finished per plane (zeroed)
  int* queue;        // [n_tiles * Hkv] completed planes in completion order (-1 = slot not filled yet)
  int* qctr;         // [0] slots handed out to selectors, [1] slots filled
  int* idx;          // [n_tiles, Hkv, k]
  int* cnt;          // [n_tiles, Hkv]
  int k, w, exclusive;
  int discard;       // 1: drop each selected plane's score lines from L2 (scores are scratch)
  const int* order;  // [n_tiles] tile at each position of the item order (longest first), or null
};

// The row's lse enters the MMA as one extra K step of 16 columns: K rows get
// [1, 1, 0 ...], Q rows get [hi, lo, 0 ...] with hi + lo = -lse2 / c (bf16
// pair, c = scale * log2 e > 0), so the accumulator holds s + (-lse2 / c) and
// score = exp2(c * max) needs only a max per element from the reducers.
// The augmentation tiles use the unswizzled K-major layout: 8-row x 16-byte
// core matrices, the two K halves 128 bytes apart, 8-row groups 256 apart.
template <int D>
struct Layout {
  static constexpr int kTile = (D / 64) * kSlabBytes;    // K block: 128 rows x D bf16
  static constexpr int kQTile = (D / 64) * kQSlabBytes;  // Q chunk: kRows rows x D bf16
  static constexpr int kQStages = q_stages<D>();
  static constexpr int kAug = 128 * 16 * 2;              // K augmentation: 128 rows x 16 bf16
  static constexpr int kQAug = kRows * 16 * 2;           // Q augmentation: kRows rows x 16 bf16
  static constexpr int kOffK = 0;
  static constexpr int kOffQ = kBlocks * kTile;
  static constexpr int kOffQa = kOffQ + kQStages * kQTile;
  static constexpr int kOffKa = kOffQa + kQStages * kQAug;
  static constexpr int kOffCtl = kOffKa + kAug;
  static constexpr int kOffSel = kOffCtl + 512;  // selector scratch (fused top-k)
};

struct Ctl {
  uint64_t k_full, k_empty;
  uint64_t q_full[kQStagesMax], q_empty[kQStagesMax];
  uint64_t acc_full[kBlocks], acc_free[kBlocks];
  uint64_t teardown;
  uint64_t sel_bar;
  int sel_plane;  // plane handed from the polling selector thread to the group (-1: stop)
  int sel_round;  // hand-overs so far
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Ctl) <= 512, "control block over its slot");

template <int D, bool SELECT = false>
constexpr int smem_bytes() {
  return Layout<D>::kOffSel + (SELECT ? int(sizeof(topk::SelScratch<kSelThreads>)) : 0) + 1024;
}
static_assert(smem_bytes<128, true>() <= 232448 && smem_bytes<64, true>() <= 232448, "smem over 227 KB");

// unswizzled K-major descriptor (layout type 0)
__device__ __forceinline__ uint64_t sdesc_noswz(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= uint64_t((smem_addr >> 4) & 0x3FFF);
  d |= uint64_t((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;
  return d;
}
// byte offset of 16-byte chunk `half` (K columns 8*half .. 8*half+7) of row r
__device__ __forceinline__ uint32_t aug_off(int r, int half) {
  return uint32_t((r >> 3) * 256 + half * 128 + (r & 7) * 16);
}

// item -> (tile, g, first key); items are enumerated tile by tile, KV head by
// KV head, in 256-key ranges (kBlocks x 128) up to the tile's last query position.
struct Item {
  int tile, g, key0, nkeys;  // keys [key0, key0 + nkeys)
  TileInfo ti;
  int nchunks;               // kRows-row chunks of the tile (rows = n * G)
};

__device__ __forceinline__ int ranges_of(const TileInfo& ti) {
  return (ti.pos0 + ti.n - 1) / (kBlocks * 128) + 1;
}

// Last query position of tile i of sequence b (the tile's longest plane).
__device__ __forceinline__ int tile_last(const SeqTable& st, int b, int i) {
  const int n_b = st.cu_q[b + 1] - st.cu_q[b];
  const int ctx = st.cu_kv[b + 1] - st.cu_kv[b] - n_b;
  return ctx + min((i + 1) * st.T, n_b) - 1;
}

// Position of `tile` in the longest-first order: tiles by last position
// descending, ties to the lower sequence. Inside one sequence the last
// position rises with the tile index, so each sequence contributes the count
// of its tiles that come first, found by binary search.
__device__ int longest_first_rank(const SeqTable& st, int tile) {
  int b = 0;
  {
    int lo = 0, hi = st.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (st.tile_base[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    b = lo;
  }
  const int i = tile - st.tile_base[b];
  const int x = tile_last(st, b, i);
  int rank = st.tile_base[b + 1] - st.tile_base[b] - 1 - i;  // own sequence: its later tiles
  for (int c = 0; c < st.batch; ++c) {
    if (c == b) continue;
    const int nt = st.tile_base[c + 1] - st.tile_base[c];
    // first tile of c that comes before `tile`: last > x (or >= x for c < b)
    int lo = 0, hi = nt;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      const int y = tile_last(st, c, mid);
      if (y > x || (c < b && y == x)) hi = mid; else lo = mid + 1;
    }
    rank += nt - lo;
  }
  return rank;
}

__device__ __forceinline__ int order_tile(const int* order, int v) { return order ? order[v] : v; }

// items are laid out tile-major: item = tile_item_base(tile) + g * ranges + r.
// The prefix of items per tile is computed on the fly by a binary search over
// tiles using the closed form of ranges per tile inside one sequence.
__device__ __forceinline__ Item get_item(const SeqTable& st, const Params& p, const int* tile_items_prefix, int w) {
  int lo = 0, hi = st.n_tiles - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_items_prefix[mid] <= w) lo = mid; else hi = mid - 1;
  }
  Item it;
  it.tile = order_tile(p.order, lo);
  it.ti = tile_info(st, it.tile);
  const int nr = ranges_of(it.ti);
  const int local = w - tile_items_prefix[lo];
  it.g = local / nr;
  const int r = local % nr;
  it.key0 = r * kBlocks * 128;
  const int last = it.ti.pos0 + it.ti.n - 1;  // candidate keys are <= last
  it.nkeys = min(kBlocks * 128, last + 1 - it.key0);
  it.nchunks = (it.ti.n * p.G + kRows - 1) / kRows;
  return it;
}

// Prefix sums of items per tile in item order (Hkv * 256-key ranges), one CTA
// of 1024 threads. With `order` (fused top-k) the item order is longest tile
// first, written to order[], and the top-k's per-plane arrival counters, its
// queue of completed planes and the queue's two counters are reset.
__global__ void __launch_bounds__(1024) item_prefix_kernel(const __grid_constant__ SeqTable st, int Hkv, int* out,
                                                           int* order, int* arrive, int* queue, int* qctr) {
  __shared__ int part[1024];
  const int n = st.n_tiles;
  if (order) {
    for (int t = threadIdx.x; t < n; t += 1024) order[longest_first_rank(st, t)] = t;
    for (int i = threadIdx.x; i < n * Hkv; i += 1024) {
      arrive[i] = 0;
      queue[i] = -1;
    }
    if (threadIdx.x < 2) qctr[threadIdx.x] = 0;
    __syncthreads();  // order[] complete before the prefix reads it
  }
  const int per = (n + 1023) / 1024;
  const int t0 = threadIdx.x * per, t1 = min(n, t0 + per);
  int sum = 0;
  for (int t = t0; t < t1; ++t) sum += Hkv * ranges_of(tile_info(st, order_tile(order, t)));
  part[threadIdx.x] = sum;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {  // inclusive scan (Hillis-Steele)
    const int v = threadIdx.x >= off ? part[threadIdx.x - off] : 0;
    __syncthreads();
    part[threadIdx.x] += v;
    __syncthreads();
  }
  int acc = threadIdx.x > 0 ? part[threadIdx.x - 1] : 0;
  for (int t = t0; t < t1; ++t) {
    out[t] = acc;
    acc += Hkv * ranges_of(tile_info(st, order_tile(order, t)));
  }
  if (threadIdx.x == 1023) out[n] = part[1023];
}

// Drop the L2 lines that lie wholly inside [base, base + bytes) without
// writing them back (their content becomes undefined). Lines shared with
// neighbouring data are left alone.
__device__ __forceinline__ void discard_lines(const void* base, size_t bytes, int t, int nthreads) {
  const uintptr_t b = reinterpret_cast<uintptr_t>(base);
  const uintptr_t first = (b + 127) & ~uintptr_t(127), end = (b + bytes) & ~uintptr_t(127);
  for (uintptr_t a = first + uintptr_t(t) * 128; a < end; a += uintptr_t(nthreads) * 128)
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(a) : "memory");
}

// A selector's wait for a word to reach `want` (a queue slot to be filled,
// want = 0; the group's hand-over count) may last as long as the whole pass:
// it gives up only when no plane at all was completed (the queue's filled
// count stood still) for the time limit. Returns the word's value, or -1.
__device__ __noinline__ int wait_at_least(const volatile int* word, int want, const int* filled,
                                          volatile int* abort_flag, const WaitCtl& wc, int site, int ctx) {
  unsigned long long t0 = global_ns();
  long long c0 = clock64();
  int seen = -1;
  for (int it = 0;; ++it) {
    const int v = *word;
    if (v >= want) return v;
    if (*abort_flag) return -1;
    if ((it & 15) == 0) {  // the progress signal is a global read: not on every poll
      const int now = *reinterpret_cast<const volatile int*>(filled);
      if (now != seen) {
        seen = now;
        t0 = global_ns();
        c0 = clock64();
      } else if (wait_expired(t0, c0, wc.timeout_ns)) {
        *abort_flag = 1;
        record_failure(wc, site, ctx);
        return -1;
      }
    }
    __nanosleep(2048);
  }
}

template <int D, bool SELECT>
__global__ void __launch_bounds__(threads<SELECT>(), 1)
    token_scores_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                        const Params p, const __grid_constant__ SeqTable st, const int* __restrict__ tile_items_prefix) {
  using L = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl& c = *reinterpret_cast<Ctl*>(smem + L::kOffCtl);
  constexpr int kQStages = L::kQStages;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // constant K-side augmentation: every key row [1, 1, 0, ..., 0]
  if (threadIdx.x < 128) {
    *reinterpret_cast<uint4*>(smem + L::kOffKa + aug_off(threadIdx.x, 0)) = make_uint4(pack_bf16(1.f, 1.f), 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(smem + L::kOffKa + aug_off(threadIdx.x, 1)) = make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();  // read by the tensor cores (async proxy)

  if (threadIdx.x == 0) {
    mbar_init(&c.k_full, 1);
    mbar_init(&c.k_empty, 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&c.q_full[s], 1);
      mbar_init(&c.q_empty[s], 1);  // MMA done with Q and its augmentation
    }
    for (int b = 0; b < kBlocks; ++b) {
      mbar_init(&c.acc_full[b], 1);
      mbar_init(&c.acc_free[b], 4);
    }
    mbar_init(&c.teardown, 1);
    if constexpr (SELECT) mbar_init(&c.sel_bar, kSelThreads / 32);  // selector group barrier
    c.abort = 0;
    c.sel_round = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&c.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  volatile int* abort_flag = &c.abort;

  if (warp == 4) {
    // ===================== producer: K blocks, Q chunks + their lse =====================
    int qctr = 0, items = 0;
    int last_q[kQStagesMax] = {-1, -1, -1};
    int k_loads = 0;
    bool ok = true;
    for (int wi = blockIdx.x; wi < p.n_items && ok; wi += gridDim.x) {
      const Item it = get_item(st, p, tile_items_prefix, wi);
      if (lane == 0) {
        if (items > 0 && !mbar_wait(&c.k_empty, (items - 1) & 1, abort_flag, p.wc, 101, wi << 12)) ok = false;
        if (ok) {
          mbar_expect_tx(&c.k_full, kBlocks * L::kTile);
          for (int b = 0; b < kBlocks; ++b)
            for (int sl = 0; sl < D / 64; ++sl)
              tma_load_3d(smem + L::kOffK + b * L::kTile + sl * kSlabBytes, &map_k, &c.k_full, sl * 64, it.g,
                          it.ti.kv0 + it.key0 + b * 128);
          ++k_loads;
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      ++items;
      // the chunk's lse values (rows lane + 32 k, row = query * G + head-in-group)
      // are loaded one chunk ahead, so their latency overlaps the ring wait
      constexpr int kRowsPerLane = kRows / 32;
      const int qpc = kRows / p.G;
      const float inv_c = 1.f / p.scale_log2;
      auto load_lse = [&](int qc, float (&x)[kRowsPerLane]) {
#pragma unroll
        for (int k = 0; k < kRowsPerLane; ++k) {
          const int rr = lane + 32 * k;
          const int ql = qc * qpc + rr / p.G;
          const int h = it.g * p.G + rr % p.G;
          x[k] = ql < it.ti.n ? __ldg(p.lse + size_t(h) * p.Tq + it.ti.qrow0 + ql) : 0.f;
        }
      };
      float lse_nx[kRowsPerLane];
      load_lse(0, lse_nx);
      for (int qc = 0; qc < it.nchunks && ok; ++qc) {
        const int s = qctr % kQStages;
        float lse_cur[kRowsPerLane];
#pragma unroll
        for (int k = 0; k < kRowsPerLane; ++k) lse_cur[k] = lse_nx[k];
        if (qc + 1 < it.nchunks) load_lse(qc + 1, lse_nx);
        int okw = 1;
        if (lane == 0) okw = mbar_wait(&c.q_empty[s], ((qctr / kQStages) & 1) ^ 1, abort_flag, p.wc, 102, (wi << 12) | qc);
        okw = __shfl_sync(0xffffffffu, okw, 0);
        if (!okw) { ok = false; break; }
        // augmentation of the chunk's kRows rows: [hi, lo] = -lse2 / c as a bf16
        // pair; rows past the tile get a huge negative hi so they never win a maximum
        uint8_t* qa = smem + L::kOffQa + s * L::kQAug;
#pragma unroll
        for (int k = 0; k < kRowsPerLane; ++k) {
          const int rr = lane + 32 * k;
          const int ql = qc * qpc + rr / p.G;
          uint32_t hl = pack_bf16(-3.0e38f, 0.f);
          if (ql < it.ti.n) {
            const float x = -(lse_cur[k] * 1.4426950408889634f) * inv_c;
            const float hi = __bfloat162float(__float2bfloat16_rn(x));
            hl = pack_bf16(hi, x - hi);
          }
          *reinterpret_cast<uint4*>(qa + aug_off(rr, 0)) = make_uint4(hl, 0u, 0u, 0u);
          *reinterpret_cast<uint4*>(qa + aug_off(rr, 1)) = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_expect_tx(&c.q_full[s], L::kQTile);
          for (int sl = 0; sl < D / 64; ++sl)
            tma_load_3d(smem + L::kOffQ + s * L::kQTile + sl * kQSlabBytes, &map_q, &c.q_full[s], sl * 64,
                        it.g * p.G, it.ti.qrow0 + qc * qpc);
          last_q[s] = qctr;
        }
        ++qctr;
      }
    }
    if (lane == 0 && *abort_flag) {
      for (int s = 0; s < kQStages; ++s)
        if (last_q[s] >= 0) mbar_wait_drain(&c.q_full[s], (last_q[s] / kQStages) & 1, p.wc, 190);
      if (k_loads > 0) mbar_wait_drain(&c.k_full, (k_loads - 1) & 1, p.wc, 191);
    }
  } else if (warp == 5) {
    // ===================== UMMA issuer: S^T[key, row] = K_blk . Q_chunk^T =====================
    if (lane == 0) {
      constexpr uint32_t kId = idesc_bf16_f32(128, kRows, false, false);
      int qctr = 0, items = 0;
      int acc_cnt[kBlocks] = {};
      bool ok = true;
      // descriptors built once; a K step adds its offset / 16 to the start field
      const uint64_t k_desc0 = sdesc_sw128(smem_u32(smem + L::kOffK), 16, 1024);
      const uint64_t q_desc0 = sdesc_sw128(smem_u32(smem + L::kOffQ), 16, 1024);
      const uint64_t ka_desc = sdesc_noswz(smem_u32(smem + L::kOffKa), 128, 256);
      const uint64_t qa_desc0 = sdesc_noswz(smem_u32(smem + L::kOffQa), 128, 256);
      for (int wi = blockIdx.x; wi < p.n_items && ok; wi += gridDim.x) {
        const Item it = get_item(st, p, tile_items_prefix, wi);
        const int nb = (it.nkeys + 127) / 128;
        if (!mbar_wait(&c.k_full, items & 1, abort_flag, p.wc, 110, wi << 12)) { ok = false; break; }
        ++items;
        for (int qc = 0; qc < it.nchunks && ok; ++qc) {
          const int s = qctr % kQStages;
          if (!mbar_wait(&c.q_full[s], (qctr / kQStages) & 1, abort_flag, p.wc, 111, (wi << 12) | qc)) { ok = false; break; }
          tc_fence_after();
          for (int b = 0; b < nb; ++b) {
            if (acc_cnt[b] > 0 &&
                !mbar_wait(&c.acc_free[b], (acc_cnt[b] - 1) & 1, abort_flag, p.wc, 112, (wi << 12) | qc)) { ok = false; break; }
            ++acc_cnt[b];
            tc_fence_after();
            const uint64_t ka = k_desc0 + uint64_t((b * L::kTile) >> 4);
            const uint64_t qb = q_desc0 + uint64_t((s * L::kQTile) >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t koff = uint64_t(((kk >> 2) * kSlabBytes + (kk & 3) * 32) >> 4);
              const uint64_t qoff = uint64_t(((kk >> 2) * kQSlabBytes + (kk & 3) * 32) >> 4);
              umma_bf16(tmem + b * kRows, ka + koff, qb + qoff, kId, kk > 0 ? 1u : 0u);
            }
            // + 1 * hi + 1 * lo = -lse2 / c per row
            umma_bf16(tmem + b * kRows, ka_desc, qa_desc0 + uint64_t((s * L::kQAug) >> 4), kId, 1u);
            umma_commit(&c.acc_full[b]);
          }
          if (!ok) break;
          umma_commit(&c.q_empty[s]);
          ++qctr;
        }
        if (!ok) break;
        umma_commit(&c.k_empty);
      }
      umma_commit(&c.teardown);
      mbar_wait_drain(&c.teardown, 0, p.wc, 192);
    }
  } else if (warp < 4) {
    // ===================== reducers: thread = key lane =====================
    const int kl = warp * 32 + lane;  // key within each 128-key block
    int acc_cnt[kBlocks] = {};
    bool ok = true;
    const float cs = p.scale_log2;
    for (int wi = blockIdx.x; wi < p.n_items; wi += gridDim.x) {
      const Item it = get_item(st, p, tile_items_prefix, wi);
      const int nb = (it.nkeys + 127) / 128;
      const int qpc = kRows / p.G;
      float best[kBlocks];
#pragma unroll
      for (int b = 0; b < kBlocks; ++b) best[b] = -INFINITY;
      for (int qc = 0; qc < it.nchunks && ok; ++qc) {
        // valid columns of this chunk: rows of queries inside the tile
        const int c_max = min(kRows, (it.ti.n - qc * qpc) * p.G);
        const int pos_first = it.ti.pos0 + qc * qpc;  // position of the chunk's first query
#pragma unroll
        for (int b = 0; b < kBlocks; ++b) {
          if (b >= nb) break;
          if (!mbar_wait_warp(&c.acc_full[b], acc_cnt[b] & 1, abort_flag, p.wc, 120, (wi << 12) | qc)) { ok = false; break; }
          ++acc_cnt[b];
          tc_fence_after();
          const int key = it.key0 + b * 128 + kl;
          // causal: column c (query pos_first + c / G) sees key iff c >= G * (key - pos_first)
          const int c_min = max(0, (key - pos_first) * p.G);
          const bool full = (c_min == 0) && (c_max == kRows);
          const uint32_t taddr = tmem + b * kRows + (uint32_t(warp * 32) << 16);
          float m = best[b];  // max over rows of s - lse2 / c
          // the accumulator's kRows columns, 128 at a time: four loads, one wait
#pragma unroll
          for (int h = 0; h < kRows / 128; ++h) {
            uint32_t v[4][32];
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) tmem_ld32(taddr + h * 128 + ch * 32, v[ch]);
            tmem_ld_wait();
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              if (full) {
#pragma unroll
                for (int e = 0; e < 32; e += 2) m = max3f(m, __uint_as_float(v[ch][e]), __uint_as_float(v[ch][e + 1]));
              } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                  const int col = h * 128 + ch * 32 + e;
                  if (col >= c_min && col < c_max) m = fmaxf(m, __uint_as_float(v[ch][e]));
                }
              }
            }
          }
          best[b] = m;
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.acc_free[b]);
        }
        if (!ok) break;
      }
      if (ok) {
        float* out = p.scores + (size_t(it.tile) * p.Hkv + it.g) * p.nblk;
#pragma unroll
        for (int b = 0; b < kBlocks; ++b) {
          const int key = it.key0 + b * 128 + kl;
          if (b < nb && key < it.key0 + it.nkeys) out[key] = best[b] > -1.0e30f ? ex2(best[b] * cs) : 0.f;
        }
      }
      if constexpr (SELECT) {
        // Count the item on its plane once all four warps' scores are visible
        // device-wide: the barrier orders the four warps' stores before
        // thread 0's gpu-scope fence, which is cumulative, so one fence
        // publishes them all. The CTA that brings the count to the plane's
        // item total appends the plane to the queue of completed planes.
        // Every reducer thread takes this barrier once per item, whatever its `ok`.
        named_bar_sync(1, 128);
        if (threadIdx.x == 0 && ok && !*abort_flag) {
          const int plane = it.tile * p.Hkv + it.g;
          __threadfence();
          if (atomicAdd(p.arrive + plane, 1) == ranges_of(it.ti) - 1) {
            __threadfence();  // the other CTAs' scores of the plane are seen before the slot is
            const int slot = atomicAdd(p.qctr + 1, 1);
            atomicExch(p.queue + slot, plane);
          }
        }
      }
    }
  } else if constexpr (SELECT) {
    // ===================== selectors: top-k of each completed plane =====================
    const int t = threadIdx.x - kThreads;
    topk::SelScratch<kSelThreads>& ss = *reinterpret_cast<topk::SelScratch<kSelThreads>*>(smem + L::kOffSel);
    bool ok = true;
    uint32_t ph = 0;
    // bounded group barrier of the selector warps (release / acquire at CTA scope)
    auto gsync = [&]() {
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.sel_bar);
      if (ok && !mbar_wait_warp(&c.sel_bar, ph, abort_flag, p.wc, 140)) ok = false;
      ph ^= 1;
    };
    const int n_planes = st.n_tiles * p.Hkv;
    for (int round = 1; ok; ++round) {
      // one thread takes the next queue slot and waits (sleeping between
      // polls of one word) for it to be filled; the other warp sleeps on the
      // hand-over count in shared memory
      int plane = -1;
      if (t == 0) {
        const int h = atomicAdd(p.qctr, 1);
        if (h < n_planes) plane = wait_at_least(p.queue + h, 0, p.qctr + 1, abort_flag, p.wc, 141, h);
        *reinterpret_cast<volatile int*>(&c.sel_plane) = plane;
        __threadfence_block();
        *reinterpret_cast<volatile int*>(&c.sel_round) = round;
      } else if (t == 32) {
        if (wait_at_least(&c.sel_round, round, p.qctr + 1, abort_flag, p.wc, 142, round) >= round) {
          __threadfence_block();  // the plane is read after the count that announced it
          plane = *reinterpret_cast<volatile int*>(&c.sel_plane);
        }
      }
      plane = __shfl_sync(0xffffffffu, plane, 0);
      if (plane < 0 || plane >= n_planes) break;
      __threadfence();
      const TileInfo ti = tile_info(st, plane / p.Hkv);
      const int n = topk::n_candidates(ti, p.nblk, 1, p.w, p.exclusive);
      const float* row = p.scores + size_t(plane) * p.nblk;
      // written by other CTAs during this kernel: read at L2, the point of
      // coherence (a line of this SM's L1 could hold an older copy of a
      // neighbouring plane's edge); 32 loads in flight per lane
      auto key_at = [&](int j) -> uint32_t { return __float_as_uint(__ldcg(row + j)); };
      topk::select_row<kSelThreads, 32>(n, p.k, t, key_at, gsync, ss, p.idx + size_t(plane) * p.k,
                                        p.cnt + plane);
      gsync();  // every read of the plane is done before its lines are dropped
      if (p.discard) discard_lines(row, size_t(ti.pos0 + ti.n) * sizeof(float), t, kSelThreads);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tscore
}  // namespace hs
