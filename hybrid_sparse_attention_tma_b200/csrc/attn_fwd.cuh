// attn_fwd.cuh -- tcgen05 attention forward shared by the full layer (causal
// attention + block-score by-product) and the sparse layers (attention over
// the reused KV cache at the selected blocks plus the forced recent window).
//
// Full layer: "standard scaled dot-product attention" whose FlashAttention
// kernel is lightly modified to emit block-level maximum scores from the
// online-softmax row maximum (HySparse explainer, techwalker.com, paragraphs
// on the master layer and on the implementation). Sparse layer: attention over
// the selected KV blocks of the shared cache (QbitAI repost, block-sparse
// branch) with the most recent tokens forced into the set (HySparse2 release
// note, airebao.com).
//
// CTA organisation (one CTA per SM, persistent over a host-ordered schedule):
//   warps 0-3  softmax warpgroup for Q-tile 0 (128 rows = TMEM lanes)
//   warps 4-7  softmax warpgroup for Q-tile 1
//   warp  8    TMA producer (Q tiles, K/V tiles or gathered blocks)
//   warp  9    UMMA issuer (one thread) + TMEM owner; the gated window-only
//              call issues Q-tile 1's MMAs from warp 10
//   warps 10-11 score warps (full layer with block scores only)
// A work item is up to 256 "rows" of one sequence and one KV head g; row
// r = query * G + head-in-group, so every Q-tile holds whole queries and the
// group's heads share each K/V tile (GQA/MQA packing into the MMA M dim).
// TMEM (512 columns): S_t at t*256, O_t at t*256+128 (fp32, 128 lanes); the
// softmax writes P_t (bf16, two per column) over the first 64 columns of S_t
// and the PV MMA reads its A operand from there.
// SMEM: Q[2] | K/V ring[5] | control. All operand tiles use the 128-byte
// swizzle (8-row x 128-byte atoms), K-major except V (MN-major). The gated
// sliding-window instantiation and the fused sparse layer run a 3-stage ring
// and spend the freed space on a 256-row output buffer that holds the other
// branch's output (TMA-loaded when an item starts, or written at the fused
// layer's switch to its window branch); the epilogue mixes in place and
// TMA-stores it.
#pragma once

#include "hs_common.cuh"

namespace hs {
namespace attn {

// Warps 0-7 softmax, 8 TMA producer, 9 UMMA issuer. The window-only gated
// call (two tiles and an epilogue per item) gives each Q-tile its own issuer
// (warps 9, 10) so that one tile's wait never delays the other's MMAs at item
// boundaries; with longer items one issuer in the order PV_0 QK_0 PV_1 QK_1
// keeps the two softmax warpgroups out of phase, which overlaps one's softmax
// with the other's MMAs (measured: the full, plain sparse and fused sparse
// layers are faster with one issuer, the window call with two). The full
// layer with block scores adds warps 10-11, which reduce each work item's
// spilled block maxima while the softmax warps move on.
template <int MODE, int SB>
constexpr bool two_issuers() {
  return MODE == 1 && SB == 0;
}
template <int MODE, int SB>
constexpr int threads_for() {
  return (MODE == 0 && SB > 0) ? 384 : two_issuers<MODE, SB>() ? 352 : 320;
}
constexpr int kStages = 5;
constexpr int kSlabBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kMaxItemRows = 256;
// Of the 4 exp2 pairs in each 8-key chunk of P, how many run on the FMA pipe
// (polynomial) instead of the MUFU unit; balances the two pipes.
#ifndef HS_EXP2_POLY_PAIRS
#define HS_EXP2_POLY_PAIRS 1
#endif
constexpr int kPolyPairs = HS_EXP2_POLY_PAIRS;

// kFused: a whole HySparse sparse layer in one pass -- the selected blocks /
// tokens (+ forced window) of the shared cache, then the sliding-window branch
// over the layer's own K_swa / V_swa, then the sigmoid gate.
enum Mode : int { kFull = 0, kSparse = 1, kFused = 2 };

// One work item: up to 256 rows (whole queries x the KV head's group) of one
// sequence and one KV head.
struct Item {
  int qrow0;   // packed query row of the item's first query
  int nq;      // queries in the item (rows = nq * G <= 256); <= 0 means empty
  int pos0;    // position of the first query in its sequence
  int kv0;     // packed key row of the sequence's first key
  int kv_len;  // keys of the sequence
  int g;       // KV head
  int tile0;   // global selection tile of the first query
  int qoff;    // index of the first query inside tile0
};

// Host-computed schedule, passed by value in the kernel parameters.
// Items are enumerated sequence by sequence in `seq` order; the full layer
// lists sequences longest first and each sequence's chunks last-to-first
// (decreasing causal cost), so the persistent CTAs start with the heaviest
// work (dealt in snake order, see snake_item).
constexpr int kMaxSched = 256;
struct Sched {
  int n_seq;
  int n_items;
  int seq[kMaxSched];             // processing order -> sequence id
  int first_item[kMaxSched + 1];  // prefix of item counts in processing order
  int cu_q[kMaxSched + 1];        // natural order
  int cu_kv[kMaxSched + 1];
  int tile_base[kMaxSched];       // first global selection tile of each sequence
};

struct Params {
  int G, Hq, Hkv, Tq;
  float scale_log2;  // softmax scale * log2(e)
  __nv_bfloat16* o;
  float* lse;  // [Hq, Tq] natural log, may be null
  // block-score by-product (full mode with SB = B > 1)
  float* scores;  // [n_tiles, Hkv, nblk]
  float* spill;   // [gridDim.x][2][spill_tiles][256 rows][128 / B] (double-buffered per CTA)
  int spill_tiles;  // 128-key tiles of the longest sequence
  int nblk;
  int T, B;
  int chunks_per_tile;  // sparse mode: ceil(T*G / 256)
  // sparse mode
  const int* idx;  // [n_tiles, Hkv, topk]
  const int* cnt;  // [n_tiles, Hkv]
  int topk;
  int w;
  int gathered;    // token level: map_kb / map_vb view buffers of the selected rows, [n_tiles * Hkv][topk][D]
  // gate epilogue (sliding-window branch): o = sig(gamma) * o_other + (1 - sig(gamma)) * o_this
  const float* gamma;                // [Tq, Hq] or null
  const __nv_bfloat16* o_other;      // [Tq, Hq, D] sparse-branch output
  int o_tma;                         // gated call: o_other / o move through smem by TMA (64 % G == 0)
  // fused sparse layer: SWA window over K_swa / V_swa, optional o_sparse output
  int ws;
  __nv_bfloat16* o_mid;              // [Tq, Hq, D] sparse-branch output or null (lse_sparse goes to lse)
  WaitCtl wc;
};

template <int D, bool GATE>
struct Layout {
  static constexpr int kSlabs = D / 64;
  static constexpr int kTileBytes = kSlabs * kSlabBytes;  // Q tile / K tile / V tile
  static constexpr int kNStages = GATE ? 3 : kStages;     // K/V ring depth
  static constexpr int kRound = 64 * D * 2;  // 64 output rows (bf16) as 128-byte swizzled 64-column slabs
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffO = kOffKV + kNStages * kTileBytes;  // [2 warpgroups][2 rounds] (GATE only)
  static constexpr int kOffCtl = kOffO + (GATE ? 4 * kRound : 0);
};

struct Ctl {
  uint64_t q_full, q_empty;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], p_full[2], o_ready[2], o_free[2];
  uint64_t teardown[2];  // per UMMA issuer
  uint64_t wg_bar[2];   // per softmax warpgroup: bounded barrier of its 4 warps
  uint64_t g_full[2];   // per softmax warpgroup: other-branch output landed (gated call)
  uint64_t sc_ready;    // softmax warps: item's spill + lse2 written (count 8)
  uint64_t lse_taken;   // score warps: lse2 copied to registers (count 2)
  uint64_t sc_free[2];  // score warps: spill buffer [parity] consumed (count 2)
  uint32_t tmem_base;
  int abort;
  float lse2[kMaxItemRows];
};

template <int D, bool GATE>
constexpr int smem_bytes() {
  // + 1024 for manual 1024-byte alignment of the dynamic smem base
  return Layout<D, GATE>::kOffCtl + int(sizeof(Ctl)) + 1024;
}
static_assert(smem_bytes<128, true>() <= 232448 && smem_bytes<128, false>() <= 232448, "smem over 227 KB");


template <int MODE>
__device__ __forceinline__ Item get_item(const Params& p, const Sched& sc, int w) {
  int lo = 0, hi = sc.n_seq - 1;  // entry e with first_item[e] <= w < first_item[e+1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sc.first_item[mid] <= w) lo = mid; else hi = mid - 1;
  }
  const int b = sc.seq[lo];
  const int local = w - sc.first_item[lo];
  const int n_b = sc.cu_q[b + 1] - sc.cu_q[b];
  const int kv_b = sc.cu_kv[b + 1] - sc.cu_kv[b];
  const int c_b = kv_b - n_b;
  const int qpc = kMaxItemRows / p.G;  // queries per 256-row chunk
  Item it;
  it.g = local % p.Hkv;
  int qloc0, nq;
  if (MODE == kFull) {
    const int n_chunks = (n_b + qpc - 1) / qpc;
    const int chunk = n_chunks - 1 - local / p.Hkv;
    qloc0 = chunk * qpc;
    nq = min(qpc, n_b - qloc0);
  } else {
    const int per_tile = p.chunks_per_tile * p.Hkv;
    const int ti = local / per_tile;
    const int chunk = (local / p.Hkv) % p.chunks_per_tile;
    const int tile_nq = min(p.T, n_b - ti * p.T);
    qloc0 = ti * p.T + chunk * qpc;
    nq = min(qpc, tile_nq - chunk * qpc);
  }
  it.qrow0 = sc.cu_q[b] + qloc0;
  it.nq = nq;
  it.pos0 = c_b + qloc0;
  it.kv0 = sc.cu_kv[b];
  it.kv_len = kv_b;
  it.tile0 = sc.tile_base[b] + qloc0 / p.T;
  it.qoff = qloc0 % p.T;
  return it;
}

// The k-th work item of this CTA. Items are listed heaviest first; dealing
// them to the persistent CTAs in alternating direction each round (0..n-1,
// then n-1..0) balances the per-CTA totals of a decreasing cost list far
// better than plain round-robin (causal full layer at 32768 tokens: max/mean
// 1.0005 instead of 1.035). Strictly increasing in k for every CTA.
__device__ __forceinline__ int snake_item(int k) {
  return k * int(gridDim.x) + ((k & 1) ? int(gridDim.x) - 1 - int(blockIdx.x) : int(blockIdx.x));
}

// Number of 128-key tiles an item iterates over, and the sparse-mode split.
struct KvPlan {
  int n_sel;  // tiles of selected keys (sparse) or causal tiles (full)
  int n_win;  // window tiles (sparse, w > 0)
  int win_lo; // first window key (position)
  int cnt;    // selected blocks
  int n_swa;  // fused sparse layer: tiles of the own-cache sliding window
  int swa_lo; // its first key (position)
  __device__ __forceinline__ int n1() const { return n_sel + n_win; }  // tiles of the shared cache
  __device__ __forceinline__ int total() const { return n_sel + n_win + n_swa; }
};

__device__ __forceinline__ KvPlan kv_plan(const Params& p, const Item& it, int mode) {
  KvPlan k{};
  const int last_pos = it.pos0 + it.nq - 1;
  if (mode == kFull) {
    k.n_sel = last_pos / 128 + 1;
    k.n_win = 0;
  } else {
    const int c = p.cnt ? __ldg(p.cnt + it.tile0 * p.Hkv + it.g) : 0;
    k.cnt = c;
    k.n_sel = (c * p.B + 127) / 128;
    if (p.w > 0) {
      k.win_lo = max(0, it.pos0 - p.w + 1);
      k.n_win = (last_pos - k.win_lo + 1 + 127) / 128;
    }
    if (mode == kFused) {
      k.swa_lo = max(0, it.pos0 - p.ws + 1);
      k.n_swa = (last_pos - k.swa_lo + 1 + 127) / 128;
    }
  }
  return k;
}

// ------------------------------------------------------------------------
// The kernel
// ------------------------------------------------------------------------
template <int D, int MODE, int SB>
__global__ void __launch_bounds__(threads_for<MODE, SB>(), 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_kb,
                    const __grid_constant__ CUtensorMap map_vb, const __grid_constant__ CUtensorMap map_g,
                    const __grid_constant__ CUtensorMap map_o, const __grid_constant__ CUtensorMap map_ks,
                    const __grid_constant__ CUtensorMap map_vs, const Params p,
                    const __grid_constant__ Sched sc) {
  // the window-only instantiation serves the gated sliding-window call; the
  // fused sparse layer computes its gate input itself
  constexpr bool kGate = (MODE == kSparse && SB == 0);
  constexpr bool kFuse = (MODE == kFused);
  constexpr bool kBuf = kGate || kFuse;  // 256-row output buffer + gate epilogue
  constexpr bool kSp = (MODE != kFull);
  constexpr int kIssuers = two_issuers<MODE, SB>() ? 2 : 1;
  using L = Layout<D, kBuf>;
  constexpr int kNS = L::kNStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl& c = *reinterpret_cast<Ctl*>(smem + L::kOffCtl);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&c.q_full, 1);
    mbar_init(&c.q_empty, kIssuers);  // released by every UMMA issuer
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&c.kv_full[s], 1);
      mbar_init(&c.kv_empty[s], kIssuers);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&c.s_full[t], 1);
      mbar_init(&c.p_full[t], 4);
      mbar_init(&c.o_ready[t], 1);
      mbar_init(&c.o_free[t], 4);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&c.teardown[t], 1);
      mbar_init(&c.wg_bar[t], 4);
      mbar_init(&c.g_full[t], 1);
    }
    mbar_init(&c.sc_ready, 8);
    mbar_init(&c.lse_taken, 2);
    mbar_init(&c.sc_free[0], 2);
    mbar_init(&c.sc_free[1], 2);
    c.abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&c.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 8 && lane == 0) {
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
    if (kSp) {
      prefetch_tensormap(&map_kb);
      prefetch_tensormap(&map_vb);
    }
    if (kBuf && p.o_tma) {
      prefetch_tensormap(&map_g);
      prefetch_tensormap(&map_o);
    }
    if (kFuse) {
      prefetch_tensormap(&map_ks);
      prefetch_tensormap(&map_vs);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  volatile int* abort_flag = &c.abort;

  if (warp == 8) {
    // ===================== TMA producer =====================
    // Lane 0 owns the barriers and issues the tile loads; for token-level
    // gathers all 32 lanes fetch indices and issue gather4 loads in parallel.
    int ctr = 0;        // K/V ring uses
    int q_uses = 0;     // Q loads issued
    int last_use[kNS];
#pragma unroll
    for (int s = 0; s < kNS; ++s) last_use[s] = -1;
    bool ok = true;
    auto wait0 = [&](uint64_t* bar, uint32_t parity, int site, int ctx) -> bool {
      int r = 1;
      if (lane == 0) r = mbar_wait(bar, parity, abort_flag, p.wc, site, ctx) ? 1 : 0;
      return __shfl_sync(0xffffffffu, r, 0) != 0;
    };
    for (int k = 0, wi = snake_item(0); wi < sc.n_items && ok; wi = snake_item(++k)) {
      const Item it = get_item<MODE>(p, sc, wi);
      if (it.nq <= 0) continue;
      const KvPlan kp = kv_plan(p, it, MODE);
      const int n = kp.total();
      if (n == 0) continue;
      const int rows = it.nq * p.G;
      const int n_qt = rows > 128 ? 2 : 1;
      if (q_uses > 0 && !wait0(&c.q_empty, (q_uses - 1) & 1, 1, wi << 12)) { ok = false; break; }
      if (lane == 0) {
        mbar_expect_tx(&c.q_full, n_qt * L::kTileBytes);
        for (int t = 0; t < n_qt; ++t)
          for (int s = 0; s < L::kSlabs; ++s)
            tma_load_3d(smem + L::kOffQ + t * L::kTileBytes + s * kSlabBytes, &map_q, &c.q_full, s * 64,
                        it.g * p.G, it.qrow0 + t * (128 / p.G));
      }
      ++q_uses;
      const int* idx_row = kSp ? p.idx + (size_t(it.tile0) * p.Hkv + it.g) * p.topk : nullptr;
      for (int i = 0; i < n && ok; ++i) {
        for (int kind = 0; kind < 2; ++kind) {
          const int s = ctr % kNS;
          if (!wait0(&c.kv_empty[s], ((ctr / kNS) & 1) ^ 1, 2, (wi << 12) | i)) { ok = false; break; }
          if (lane == 0) mbar_expect_tx(&c.kv_full[s], L::kTileBytes);
          __syncwarp();
          uint8_t* dst = smem + L::kOffKV + s * L::kTileBytes;
          const CUtensorMap* mt = kind == 0 ? &map_k : &map_v;
          if (MODE == kFull || i >= kp.n_sel) {
            // contiguous 128-key tiles: causal (full), forced window, or the
            // fused layer's own-cache sliding window
            const bool own = kFuse && i >= kp.n1();
            const int key0 = (MODE == kFull) ? i * 128
                             : own ? kp.swa_lo + (i - kp.n1()) * 128
                                   : kp.win_lo + (i - kp.n_sel) * 128;
            const CUtensorMap* mc = own ? (kind == 0 ? &map_ks : &map_vs) : mt;
            if (lane == 0)
              for (int sl = 0; sl < L::kSlabs; ++sl)
                tma_load_3d(dst + sl * kSlabBytes, mc, &c.kv_full[s], sl * 64, it.g, it.kv0 + key0);
          } else {
            const CUtensorMap* mb = kind == 0 ? &map_kb : &map_vb;
            if (SB == 1 && p.gathered) {
              // token level, rows gathered once per block: slots i*128 .. i*128+127
              // of the (tile, kv head) plane are one tile load
              if (lane == 0)
                for (int sl = 0; sl < L::kSlabs; ++sl)
                  tma_load_3d(dst + sl * kSlabBytes, mb, &c.kv_full[s], sl * 64, i * 128, it.tile0 * p.Hkv + it.g);
            } else if constexpr (SB == 1) {
              // token level: lane l gathers selected rows 4l..4l+3 of the tile
              // from the 2-D row view (row = token * H_kv + kv head); padded
              // slots re-read the first selected row and are masked
              const int r4 = lane * 4;
              int rws[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int slot = i * 128 + r4 + e;
                const int key = __ldg(idx_row + (slot < kp.cnt ? slot : 0));
                rws[e] = (it.kv0 + key) * p.Hkv + it.g;
              }
              for (int sl = 0; sl < L::kSlabs; ++sl)
                tma_load_2d_gather4(dst + sl * kSlabBytes + r4 * 128, mb, &c.kv_full[s], sl * 64, rws[0], rws[1],
                                    rws[2], rws[3]);
            } else if (lane == 0) {
              constexpr int sbk = SB > 0 ? SB : 128;
              constexpr int nb = 128 / sbk;
              for (int bi = 0; bi < nb; ++bi) {
                const int slot = i * nb + bi;
                const int blk = __ldg(idx_row + (slot < kp.cnt ? slot : 0));
                for (int sl = 0; sl < L::kSlabs; ++sl)
                  tma_load_3d(dst + sl * kSlabBytes + bi * sbk * 128, mb, &c.kv_full[s], sl * 64, it.g,
                              it.kv0 + blk * sbk);
              }
            }
          }
          last_use[s] = ctr;
          ++ctr;
        }
      }
    }
    // drain: never leave the CTA with TMA writes in flight
    if (lane == 0 && *abort_flag) {
      for (int s = 0; s < kNS; ++s)
        if (last_use[s] >= 0) mbar_wait_drain(&c.kv_full[s], (last_use[s] / kNS) & 1, p.wc, 90);
      if (q_uses > 0) mbar_wait_drain(&c.q_full, (q_uses - 1) & 1, p.wc, 91);
    }
  } else if (warp == 9 || (kIssuers == 2 && warp == 10)) {
    // ===================== UMMA issuer(s) =====================
    // One issuer walks both Q-tiles (t = 0, 1) or, with two issuers, warp
    // 9 + t owns Q-tile t. Every issuer walks the same K/V ring and releases
    // each stage and Q with its own commit (barrier count = issuers); an
    // issuer whose Q-tile has no rows in an item only waits for the loads and
    // arrives, so the ring phases stay in step.
    const int t_lo = kIssuers == 2 ? warp - 9 : 0;
    const int t_hi = kIssuers == 2 ? warp - 9 : 1;
    if (lane == 0) {
      constexpr uint32_t kIdQK = idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdPV = idesc_bf16_f32(128, D, false, true);
      int ctr = 0, q_uses = 0;
      int uses[2] = {0, 0};     // S/P/O phases per Q-tile
      int items_t[2] = {0, 0};  // items in which tile t took part (o_free phase)
      bool ok = true;
      // Descriptors are built once; a K step only adds its byte offset / 16
      // to the 14-bit start-address field (no carry: smem < 256 KB).
      const uint64_t q_desc0 = sdesc_sw128(smem_u32(smem + L::kOffQ), 16, 1024);
      const uint64_t k_desc0 = sdesc_sw128(smem_u32(smem + L::kOffKV), 16, 1024);
      const uint64_t v_desc0 = sdesc_sw128(smem_u32(smem + L::kOffKV), kSlabBytes, 1024);
      auto issue_qk = [&](int t, int stage) {
        const uint32_t d_tmem = tmem + t * 256;
        const uint64_t qd = q_desc0 + uint64_t((t * L::kTileBytes) >> 4);
        const uint64_t kd = k_desc0 + uint64_t((stage * L::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = uint64_t(((kk >> 2) * kSlabBytes + (kk & 3) * 32) >> 4);
          umma_bf16(d_tmem, qd + off, kd + off, kIdQK, kk > 0 ? 1u : 0u);
        }
        umma_commit(&c.s_full[t]);
      };
      auto issue_pv = [&](int t, int stage, bool acc) {
        const uint32_t d_tmem = tmem + t * 256 + 128;
        const uint32_t pa = tmem + t * 256;  // P_t over the first 64 columns of S_t
        const uint64_t vd = v_desc0 + uint64_t((stage * L::kTileBytes) >> 4);
        umma_bf16_ts(d_tmem, pa, vd, kIdPV, acc ? 1u : 0u);
#pragma unroll
        for (int kk = 1; kk < 8; ++kk) umma_bf16_ts(d_tmem, pa + kk * 8, vd + uint64_t(kk * (2048 >> 4)), kIdPV, 1u);
        umma_commit(&c.o_ready[t]);
      };
      // release a K/V stage / Q: by commit after this issuer's MMAs, or at once
      auto release = [&](uint64_t* bar, bool issued) {
        if (issued) umma_commit(bar);
        else mbar_arrive(bar);
      };
      auto wait_kv = [&](int site, int ctx) -> int {
        const int s = ctr % kNS;
        if (!mbar_wait(&c.kv_full[s], (ctr / kNS) & 1, abort_flag, p.wc, site, ctx)) return -1;
        ++ctr;
        return s;
      };
      for (int k = 0, wi = snake_item(0); wi < sc.n_items && ok; wi = snake_item(++k)) {
        const Item it = get_item<MODE>(p, sc, wi);
        if (it.nq <= 0) continue;
        const KvPlan kp = kv_plan(p, it, MODE);
        const int n = kp.total();
        if (n == 0) continue;
        const int n_qt = it.nq * p.G > 128 ? 2 : 1;
        const int t_end = min(t_hi, n_qt - 1);  // last Q-tile of this issuer with rows in the item
        const bool mine = t_lo <= t_end;
        if (!mbar_wait(&c.q_full, q_uses & 1, abort_flag, p.wc, 10, wi << 12)) { ok = false; break; }
        ++q_uses;
        tc_fence_after();
        // prologue: S_t(0)
        const int sk = wait_kv(11, wi << 12);
        if (sk < 0) { ok = false; break; }
        tc_fence_after();
        for (int t = t_lo; t <= t_end; ++t) issue_qk(t, sk);
        release(&c.kv_empty[sk], mine);
        if (n == 1) release(&c.q_empty, mine);  // Q is only read by QK: free it early
        for (int i = 0; i < n && ok; ++i) {
          const int sv = wait_kv(12, (wi << 12) | i);
          if (sv < 0) { ok = false; break; }
          int sk_next = -1;
          for (int t = t_lo; t <= t_end; ++t) {
            if (!mbar_wait(&c.p_full[t], (uses[t] + i) & 1, abort_flag, p.wc, 13, (wi << 12) | i)) { ok = false; break; }
            if (i == 0 && items_t[t] > 0 &&
                !mbar_wait(&c.o_free[t], (items_t[t] - 1) & 1, abort_flag, p.wc, 14)) { ok = false; break; }
            tc_fence_after();
            issue_pv(t, sv, i > 0 && !(kFuse && i == kp.n1()));  // fused: the SWA branch starts a fresh O
            if (i + 1 < n) {
              if (sk_next < 0) {
                sk_next = wait_kv(15, (wi << 12) | i);
                if (sk_next < 0) { ok = false; break; }
                tc_fence_after();
              }
              issue_qk(t, sk_next);
            }
          }
          if (!ok) break;
          if (i + 1 < n && sk_next < 0) {  // an issuer without rows still takes the next K stage
            sk_next = wait_kv(15, (wi << 12) | i);
            if (sk_next < 0) { ok = false; break; }
          }
          release(&c.kv_empty[sv], mine);
          if (sk_next >= 0) release(&c.kv_empty[sk_next], mine);
          if (i + 2 == n) release(&c.q_empty, mine);  // last QK of the item issued
        }
        if (!ok) break;
        for (int t = t_lo; t <= t_end; ++t) {
          uses[t] += n;
          items_t[t] += 1;
        }
      }
      // make sure no tensor-core op of this issuer is still writing TMEM before teardown
      umma_commit(&c.teardown[t_lo]);
      mbar_wait_drain(&c.teardown[t_lo], 0, p.wc, 92);
    }
  } else if (warp < 8) {
    // ===================== softmax warpgroups =====================
    const int t = warp >> 2;       // Q-tile
    const int quad = warp & 3;     // TMEM lane quadrant
    const int r = quad * 32 + lane;  // row inside the Q-tile
    const int vr = t * 128 + r;      // row inside the item
    const uint32_t t_s = tmem + t * 256 + (uint32_t(quad * 32) << 16);
    const uint32_t t_o = t_s + 128;
    int uses = 0, items_t = 0, sc_items = 0;
    bool ok = true;
    // gated call: this warpgroup's two 64-row rounds of the output buffer, the
    // phase of its bounded barrier and of g_full, and the loads it issued
    uint8_t* o_buf = smem + L::kOffO + t * 2 * L::kRound;
    int wg_phase = 0, g_uses = 0, g_issued = 0;
    auto wg_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.wg_bar[t]);
      const bool r = mbar_wait_warp(&c.wg_bar[t], wg_phase & 1, abort_flag, p.wc, 33);
      ++wg_phase;
      return r;
    };
    for (int k = 0, wi = snake_item(0); wi < sc.n_items; wi = snake_item(++k)) {
      const Item it = get_item<MODE>(p, sc, wi);
      if (it.nq <= 0) continue;
      const KvPlan kp = kv_plan(p, it, MODE);
      const int n = kp.total();
      const int rows = it.nq * p.G;
      const bool active = (t == 0) || rows > 128;
      const bool valid = vr < rows;
      const int ql = vr / p.G;
      const int h = it.g * p.G + (vr % p.G);
      const int pos = it.pos0 + ql;
      const int qrow = it.qrow0 + ql;
      float m_used = -INFINITY, l = 0.f;
      const int par = sc_items & 1;  // spill buffer of this item (full mode with scores)
      float sg = 0.f;                // gate of this row (gated call)
      if constexpr (kBuf) {
        if (p.gamma && valid) sg = 1.f / (1.f + __expf(-__ldg(p.gamma + size_t(qrow) * p.Hq + h)));
      }
      if constexpr (MODE == kFull && SB > 0) {
        if (sc_items >= 2 && ok &&
            !mbar_wait_warp(&c.sc_free[par], ((sc_items >> 1) - 1) & 1, abort_flag, p.wc, 31, wi << 12))
          ok = false;
      }
      if (active && n > 0 && ok) {
        if constexpr (kGate) {
          // the other branch's output does not depend on this item: load its
          // rows now, behind the whole softmax loop (the buffer's previous
          // store was read out before this thread left the last epilogue)
          if (p.o_tma && p.gamma && quad == 0 && lane == 0) {
            const int nr = min(2, (rows - t * 128 + 63) / 64);
            mbar_expect_tx(&c.g_full[t], nr * L::kRound);
            for (int rd = 0; rd < nr; ++rd)
              for (int sl = 0; sl < L::kSlabs; ++sl)
                tma_load_3d(o_buf + rd * L::kRound + sl * (64 * 128), &map_g, &c.g_full[t], sl * 64, it.g * p.G,
                            it.qrow0 + (t * 128 + rd * 64) / p.G);
            ++g_issued;
          }
        }
        const int* idx_row =
            kSp ? p.idx + (size_t(it.tile0) * p.Hkv + it.g) * p.topk : nullptr;
        for (int i = 0; i < n; ++i) {
          if (!mbar_wait_warp(&c.s_full[t], (uses + i) & 1, abort_flag, p.wc, 20, (wi << 12) | i)) { ok = false; break; }
          tc_fence_after();
          if constexpr (kFuse) {
            if (i == kp.n1()) {
              // The shared-cache phase is complete: this S was committed after
              // its last PV. o_sparse = O / l goes to this row's slot of the
              // output buffer (and to o_mid if asked), lse_sparse to lse; the
              // sliding-window branch then starts from an empty softmax state
              // (its first PV overwrites O).
              const float inv = l > 0.f ? 1.f / l : 0.f;
              const int rr = vr - (t * 128 + (quad >> 1) * 64);
              uint8_t* rbuf = o_buf + (quad >> 1) * L::kRound + rr * 128;
              uint4* mid = (p.o_mid && valid) ? reinterpret_cast<uint4*>(p.o_mid + (size_t(qrow) * p.Hq + h) * D)
                                              : nullptr;
#pragma unroll
              for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t ov[32];
                if (i > 0) {
                  tmem_ld32(t_o + ch * 32, ov);
                  tmem_ld_wait();
                } else {
#pragma unroll
                  for (int j = 0; j < 32; ++j) ov[j] = 0u;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const uint4 res = make_uint4(
                      pack_bf16(__uint_as_float(ov[8 * j + 0]) * inv, __uint_as_float(ov[8 * j + 1]) * inv),
                      pack_bf16(__uint_as_float(ov[8 * j + 2]) * inv, __uint_as_float(ov[8 * j + 3]) * inv),
                      pack_bf16(__uint_as_float(ov[8 * j + 4]) * inv, __uint_as_float(ov[8 * j + 5]) * inv),
                      pack_bf16(__uint_as_float(ov[8 * j + 6]) * inv, __uint_as_float(ov[8 * j + 7]) * inv));
                  *reinterpret_cast<uint4*>(rbuf + (ch >> 1) * (64 * 128) + ((((ch & 1) * 4 + j) ^ (rr & 7)) << 4)) =
                      res;
                  if (mid) mid[ch * 4 + j] = res;
                }
              }
              if (valid && p.lse)
                p.lse[size_t(h) * p.Tq + qrow] = (l > 0.f ? m_used + __log2f(l) : -INFINITY) * 0.69314718055994531f;
              m_used = -INFINITY;
              l = 0.f;
            }
          }
          uint32_t u[128];
          tmem_ld32(t_s + 0, *reinterpret_cast<uint32_t(*)[32]>(&u[0]));
          tmem_ld32(t_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&u[32]));
          tmem_ld32(t_s + 64, *reinterpret_cast<uint32_t(*)[32]>(&u[64]));
          tmem_ld32(t_s + 96, *reinterpret_cast<uint32_t(*)[32]>(&u[96]));
          tmem_ld_wait();
          // raw logits (the softmax scale is folded into one FFMA per element below)
          float x[128];
#pragma unroll
          for (int j = 0; j < 128; ++j) x[j] = __uint_as_float(u[j]);
          const float cs = p.scale_log2;
          // ---- masks ----
          if (MODE == kFull) {
            const int key0 = i * 128;
            if (key0 + 127 > pos) {
#pragma unroll
              for (int j = 0; j < 128; ++j)
                if (key0 + j > pos) x[j] = -INFINITY;
            }
          } else if (i < kp.n_sel) {
            if constexpr (SB == 1) {
              // selected tokens are ascending: those with key <= pos - w form a
              // prefix of the tile's slots; find its length by binary search
              const int lim = pos - p.w;
              const int s0 = i * 128, s1 = min(kp.cnt, s0 + 128);
              if (s1 - s0 < 128 || __ldg(idx_row + s1 - 1) > lim) {
                int lo = s0, hi = s1;  // first slot in [s0, s1) with key > lim
                while (lo < hi) {
                  const int mid = (lo + hi) >> 1;
                  if (__ldg(idx_row + mid) <= lim) lo = mid + 1; else hi = mid;
                }
                const int nvis = lo - s0;
#pragma unroll
                for (int j = 0; j < 128; ++j)
                  if (j >= nvis) x[j] = -INFINITY;
              }
            } else if constexpr (SB > 1) {
              // selected keys must satisfy key <= pos - w; keys of a block are
              // consecutive, so each block gives one threshold on j % SB
              constexpr int nb = 128 / SB;
              const int lim = pos - p.w;
              const int slot_last = min(kp.cnt, (i + 1) * nb) - 1;
              const int maxkey = __ldg(idx_row + slot_last) * SB + SB - 1;
              if (maxkey > lim || (i + 1) * nb > kp.cnt) {
                int thr[nb];
#pragma unroll
                for (int b = 0; b < nb; ++b) {
                  const int slot = i * nb + b;
                  thr[b] = slot < kp.cnt ? lim - __ldg(idx_row + slot) * SB : -1;
                }
#pragma unroll
                for (int j = 0; j < 128; ++j)
                  if ((j % SB) > thr[j / SB]) x[j] = -INFINITY;
              }
            }
          } else {
            // forced window of the shared cache, or the fused layer's own window
            const bool own = kFuse && i >= kp.n1();
            const int key0 = own ? kp.swa_lo + (i - kp.n1()) * 128 : kp.win_lo + (i - kp.n_sel) * 128;
            const int lo = pos - (own ? p.ws : p.w) + 1;
#pragma unroll
            for (int j = 0; j < 128; ++j) {
              const int key = key0 + j;
              if (key < lo || key > pos) x[j] = -INFINITY;
            }
          }
          // ---- row max; block maxima for the scores ----
          float mt = -INFINITY;
          if constexpr (MODE == kFull && SB > 0) {
            // this row's maxima of the tile's nb blocks, one vector store
            // ([tile][row][block] layout; blocks past the sequence are never read)
            constexpr int nb = 128 / SB;
            float* sp = p.spill + ((size_t(blockIdx.x) * 2 + par) * p.spill_tiles + i) * kMaxItemRows * nb +
                        size_t(vr) * nb;
            float mb[nb];
#pragma unroll
            for (int b = 0; b < nb; ++b) mb[b] = max_n<SB>(x + b * SB);
            if constexpr (nb == 1) {
              sp[0] = mb[0] * cs;  // log2 units
            } else if constexpr (nb == 2) {
              *reinterpret_cast<float2*>(sp) = make_float2(mb[0] * cs, mb[1] * cs);
            } else {
#pragma unroll
              for (int q4 = 0; q4 < nb / 4; ++q4)
                reinterpret_cast<float4*>(sp)[q4] =
                    make_float4(mb[4 * q4] * cs, mb[4 * q4 + 1] * cs, mb[4 * q4 + 2] * cs, mb[4 * q4 + 3] * cs);
            }
            mt = max_n<nb>(mb);
          } else {
            mt = max_n<128>(x);
          }
          mt *= cs;  // log2 units
          // ---- online softmax with lazy rescaling (exact: O and l share m_used) ----
          float factor = 1.f;
          bool rescale = false;
          if (mt > m_used + 8.f) {
            factor = (m_used == -INFINITY) ? 0.f : ex2(m_used - mt);
            m_used = mt;
            rescale = true;
          }
          const float nmu = (m_used == -INFINITY) ? 0.f : -m_used;
          const uint64_t cs2 = f2(cs, cs), nmu2 = f2(nmu, nmu);
          uint64_t rs2[2] = {f2(0.f, 0.f), f2(0.f, 0.f)};
          // S_t is already in registers: P_t overwrites its first 64 columns
#pragma unroll
          for (int cq = 0; cq < 4; ++cq) {  // 4 x 32 keys = 4 x 16 columns of packed bf16
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int j = cq * 32 + 2 * e;
              float t0, t1, a0, a1;
              f2_split(f2_fma(f2(x[j], x[j + 1]), cs2, nmu2), t0, t1);
              if ((e & 3) >= 4 - kPolyPairs) {
                exp2_poly_pair(t0, t1, a0, a1);
              } else {
                a0 = ex2(t0);
                a1 = ex2(t1);
              }
              rs2[e & 1] = f2_add(rs2[e & 1], f2(a0, a1));
              pk[e] = pack_bf16(a0, a1);
            }
            tmem_st16(t_s + cq * 16, pk);
          }
          float rs[4];
          f2_split(rs2[0], rs[0], rs[1]);
          f2_split(rs2[1], rs[2], rs[3]);
          l = l * factor + ((rs[0] + rs[1]) + (rs[2] + rs[3]));
          // S_t(i) was committed after PV_t(i-1), and a commit tracks every
          // earlier tensor-core op of the issuing thread: PV_t(i-1) is done, so
          // the P buffer and O may be touched without waiting on o_ready.
          // tcgen05.ld/st are warp-collective: rescale the whole warp's rows
          // together (rows that keep their max use factor 1).
          const int i0 = (kFuse && i >= kp.n1()) ? kp.n1() : 0;  // first tile of this softmax
          if (__any_sync(0xffffffffu, rescale && i > i0)) {
            const float f = (rescale && i > i0) ? factor : 1.f;
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
              uint32_t ov[32];
              tmem_ld32(t_o + ch * 32, ov);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * f);
              tmem_st32(t_o + ch * 32, ov);
            }
            tmem_st_wait();
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.p_full[t]);
        }
        // ---- epilogue: O / l, lse ----
        if (ok && mbar_wait_warp(&c.o_ready[t], (uses + n - 1) & 1, abort_flag, p.wc, 22)) {
          tc_fence_after();
          const float inv = l > 0.f ? 1.f / l : 0.f;
          __nv_bfloat16* orow = p.o + (size_t(qrow) * p.Hq + h) * D;
          if constexpr (kBuf) {
            // o = sig(gamma) o_other + (1 - sig(gamma)) o_this. The other
            // branch's rows sit in this warpgroup's buffer in the TMA box
            // layout (gated call with o_tma: loaded by TMA at item start; fused
            // layer: written by this thread at the phase switch); each thread
            // overwrites its row in place and one thread stores the full
            // 64-row rounds (partial ones go direct).
            const bool gate = p.gamma != nullptr;
            if (kGate && p.o_tma && gate && ok) {
              if (mbar_wait_warp(&c.g_full[t], g_uses & 1, abort_flag, p.wc, 23, wi << 12)) ++g_uses;
              else ok = false;
            }
            const int rnd = quad >> 1;
            const int row_base = t * 128 + rnd * 64;
            const bool tma_round = p.o_tma && row_base + 64 <= rows;
            const int rr = vr - row_base;  // 0..63
            uint8_t* rbuf = o_buf + rnd * L::kRound + rr * 128;
            const uint4* src = reinterpret_cast<const uint4*>(p.o_other + (size_t(qrow) * p.Hq + h) * D);
            uint4* dst = reinterpret_cast<uint4*>(orow);
            if (ok) {
#pragma unroll
              for (int ch = 0; ch < D / 32; ++ch) {
                uint32_t ov[32];
                tmem_ld32(t_o + ch * 32, ov);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  uint4* chunk = reinterpret_cast<uint4*>(rbuf + (ch >> 1) * (64 * 128) +
                                                          ((((ch & 1) * 4 + j) ^ (rr & 7)) << 4));
                  float of[8];
#pragma unroll
                  for (int e = 0; e < 8; ++e) of[e] = __uint_as_float(ov[8 * j + e]) * inv;
                  if (gate && valid) {
                    const uint4 u4 = (kFuse || p.o_tma) ? *chunk : __ldg(src + ch * 4 + j);
                    const uint32_t w4[4] = {u4.x, u4.y, u4.z, u4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                      const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
                      of[2 * e] = sg * f2.x + (1.f - sg) * of[2 * e];
                      of[2 * e + 1] = sg * f2.y + (1.f - sg) * of[2 * e + 1];
                    }
                  }
                  const uint4 res = make_uint4(pack_bf16(of[0], of[1]), pack_bf16(of[2], of[3]),
                                               pack_bf16(of[4], of[5]), pack_bf16(of[6], of[7]));
                  if (tma_round) *chunk = res;
                  else if (valid) dst[ch * 4 + j] = res;
                }
              }
            }
            if (p.o_tma) {
              fence_proxy_async_smem();
              if (!wg_sync()) {
                ok = false;
              } else if (quad == 0 && lane == 0 && ok) {
                for (int rd = 0; rd < 2; ++rd) {
                  const int rb = t * 128 + rd * 64;
                  if (rb + 64 <= rows)
                    for (int sl = 0; sl < L::kSlabs; ++sl)
                      tma_store_3d(&map_o, o_buf + rd * L::kRound + sl * (64 * 128), sl * 64, it.g * p.G,
                                   it.qrow0 + rb / p.G);
                }
                bulk_commit();
                bulk_wait_read0();  // the buffer may be refilled once the stores have read it
              }
              // fused layer: the whole warpgroup refills the buffer at the next
              // phase switch, so every warp waits for the stores' reads
              if (kFuse && !wg_sync()) ok = false;
            }
          } else {
#pragma unroll
            for (int ch = 0; ch < D / 32; ++ch) {
              uint32_t ov[32];
              tmem_ld32(t_o + ch * 32, ov);
              tmem_ld_wait();
              if (valid) {
                uint32_t pk2[16];
#pragma unroll
                for (int j = 0; j < 16; ++j)
                  pk2[j] = pack_bf16(__uint_as_float(ov[2 * j]) * inv, __uint_as_float(ov[2 * j + 1]) * inv);
                uint4* dst = reinterpret_cast<uint4*>(orow + ch * 32);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  dst[j] = make_uint4(pk2[4 * j], pk2[4 * j + 1], pk2[4 * j + 2], pk2[4 * j + 3]);
              }
            }
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.o_free[t]);
        } else {
          ok = false;
        }
        uses += n;
        items_t += 1;
      } else if (valid && (n == 0 || !active)) {
        // no visible key at all (sparse, k = 0 and w = 0): o = 0, lse = -inf
        if (n == 0) {
          uint4* dst = reinterpret_cast<uint4*>(p.o + (size_t(qrow) * p.Hq + h) * D);
          for (int j = 0; j < D / 8; ++j) dst[j] = make_uint4(0, 0, 0, 0);
        }
      }
      const float lse2 = (l > 0.f) ? m_used + __log2f(l) : -INFINITY;
      // (the fused layer reports the sparse branch's lse, written at its phase switch)
      if (!kFuse && valid && active && p.lse) p.lse[size_t(h) * p.Tq + qrow] = lse2 * 0.69314718055994531f;
      if (valid && n == 0 && p.lse) p.lse[size_t(h) * p.Tq + qrow] = -INFINITY;
      // ---- hand the item's lse to the score warp (full mode, B > 1) ----
      if constexpr (MODE == kFull && SB > 0) {
        if (sc_items >= 1 && ok &&
            !mbar_wait_warp(&c.lse_taken, (sc_items - 1) & 1, abort_flag, p.wc, 32, wi << 12))
          ok = false;
        c.lse2[vr] = lse2;
        __threadfence_block();  // spill stores and lse2 visible before the arrive
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.sc_ready);
        ++sc_items;
      }
    }
    if constexpr (kBuf) {
      // never leave with TMA traffic on this warpgroup's buffer in flight
      if (quad == 0 && lane == 0) {
        if (g_issued > g_uses) mbar_wait_drain(&c.g_full[t], (g_issued - 1) & 1, p.wc, 93);
        bulk_wait0();
      }
    }
  } else {
    // ===================== score warps (10, 11) =====================
    // score(t, g, b) = max over the tile's rows r of exp2(m_{r,b} - lse2_r):
    // the per-row block maxima m were spilled during the main loop; with the
    // final lse2 known they are reduced here, off the softmax critical path.
    // Warp 10 + wq owns the item's rows [128 wq, 128 wq + 128); lane l owns
    // rows 4l..4l+3 of that half.
    const int wq = warp - 10;
    int sc_items = 0;
    if constexpr (MODE == kFull && SB > 0)
    for (int k = 0, wi = snake_item(0); wi < sc.n_items; wi = snake_item(++k)) {
      const Item it = get_item<MODE>(p, sc, wi);
      if (it.nq <= 0) continue;
      const KvPlan kp = kv_plan(p, it, MODE);
      const int n = kp.total();
      if (!mbar_wait_warp(&c.sc_ready, sc_items & 1, abort_flag, p.wc, 40, wi << 12)) break;
      float l2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) l2[e] = c.lse2[wq * 128 + lane * 4 + e];
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.lse_taken);
      const int par = sc_items & 1;
      const int rows = it.nq * p.G;
      constexpr int nb = SB > 0 ? 128 / SB : 1;
      // this lane's 4 rows of a tile: 4 * nb consecutive floats ([tile][row][block])
      const float* sp = p.spill + (size_t(blockIdx.x) * 2 + par) * p.spill_tiles * kMaxItemRows * nb +
                        size_t(wq * 128 + lane * 4) * nb;
      const int nblk_item = min(p.nblk, (n * 128) / SB);
      const int ntile_item = (nblk_item + nb - 1) / nb;
      // selection tiles of the item's queries (row = query * G + head)
      const int t_first = it.qoff / p.T, t_last = (it.qoff + it.nq - 1) / p.T;
      // several tiles per round, their loads in flight before any use
      constexpr int kU = nb >= 8 ? 1 : 8 / nb;
      for (int i0 = 0; i0 < ntile_item; i0 += kU) {
        float4 v4[kU][nb];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          const float4* src = reinterpret_cast<const float4*>(sp + size_t(min(i0 + u, ntile_item - 1)) * kMaxItemRows * nb);
#pragma unroll
          for (int q = 0; q < nb; ++q) v4[u][q] = src[q];
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
          if (i0 + u >= ntile_item) break;
          const float* f = reinterpret_cast<const float*>(&v4[u][0]);  // row e, block j at f[e * nb + j]
#pragma unroll
          for (int j = 0; j < nb; ++j) {
            const int b = (i0 + u) * nb + j;
            if (b >= nblk_item) break;
            const float vv[4] = {f[j] - l2[0], f[nb + j] - l2[1], f[2 * nb + j] - l2[2], f[3 * nb + j] - l2[3]};
            for (int tt = t_first; tt <= t_last; ++tt) {
              // rows of tile tt inside the item: queries [tt*T - qoff, (tt+1)*T - qoff)
              const int ra = max(wq * 128, (tt * p.T - it.qoff) * p.G);
              const int rb = min(min(rows, wq * 128 + 128), ((tt + 1) * p.T - it.qoff) * p.G);
              if (ra >= rb) continue;  // the tile has no rows in this half
              const int tile_last = min(it.pos0 - it.qoff + (tt + 1) * p.T - 1, it.kv_len - 1);
              if (b * SB > tile_last) continue;  // not a candidate of this tile
              float v = -INFINITY;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int r = wq * 128 + lane * 4 + e;
                if (r >= ra && r < rb) v = fmaxf(v, vv[e]);
              }
#pragma unroll
              for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
              if (lane == 0 && v > -INFINITY)
                atomicMax(reinterpret_cast<unsigned int*>(p.scores + (size_t(it.tile0 + tt) * p.Hkv + it.g) * p.nblk + b),
                          __float_as_uint(ex2(v)));
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.sc_free[par]);
      ++sc_items;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn
}  // namespace hs
