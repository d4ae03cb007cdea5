// decode_tc.cuh -- the full layer of a hybrid block for one new token per
// sequence, on tcgen05 tensor cores: causal attention of the token over all
// its keys plus the exact token scores that drive the top-k selection
// (HySparse2 release note on airebao.com: the sparse layers reuse the full
// layer's token choice, made from its attention scores; the score of key j is
// max over the KV group's heads h of exp(s_hj - lse_h)).
//
// The scores need each head's final lse, so the layer takes two passes over
// the keys of a (sequence, KV head) "unit": pass 1 reduces (m, l) per head,
// pass 2 recomputes the logits with lse known, so P = exp(s - lse) is final,
// writes the scores and accumulates P.V. Both passes run in ONE persistent
// kernel whose work items (pass, unit, key chunk) are taken from an atomic
// counter. Pass-1 items form one stream and pass-2 items another, both in
// unit order; the kernel takes the first D pass-1 items, then alternates
// pass-2 and pass-1 items. D exceeds the items in flight plus one unit's
// chunks, so a pass-2 item almost never finds its unit's pass 1 unfinished,
// and a unit's keys are read the second time about 2D items after the first:
// pass 1 loads K with an evict-last hint and pass 2 reads it back from L2
// (pass 2 loads with evict-first). Items are taken in increasing order and a
// pass-2 item waits only for pass-1 items of smaller index, which are held by
// running CTAs that never wait on anything, so the waits always end.
//
// Pass 1 (heads on the MMA's M): S = Q K^T with M = 128 rows = two copies of
// the G <= 64 heads, N = 128 keys; the copy c rows reduce key columns
// [64c, 64c + 64), so all four compute warps work; the copies' (m, l) are
// merged in shared memory into one pair per (chunk, head) that the completion
// warp folds into the unit's running pair.
// Pass 2 (keys on M): S^T = K Q^T (M = 128 keys, N = 64 head columns) with
// the row's -lse2 / c folded in as one extra K step (key rows [1, 1, 1, 0...],
// head rows a three-term bf16 split of -lse2 / c), so a thread (= one key)
// reads x_h = s_h - lse2_h / c and gets P_h = exp2(c x_h) and the score
// exp2(c max_h x_h) from its own registers. P^T goes to shared memory as the
// MN-major B operand of O^T += V^T P^T (M = d = 128, N = 64 heads, K = keys);
// each item adds its O^T into an fp32 accumulator with red.add.
//
// CTA: warps 0-3 compute (thread = TMEM lane), warp 4 producer (work counter,
// TMA loads, lse augmentation), warp 5 UMMA issuer and TMEM owner, warp 6
// completion: it takes each finished item off the compute warps' path --
// adds a pass-1 chunk's sum l * 2^m (log2 units) to its unit's per-head fp64
// total with red.add (exact to fp64 rounding for |logit * log2 e| < ~1000, no
// reference maximum needed, no contention retries), counts the unit's
// finished items and, for the last one, writes lse2 = log2(total) and raises
// the ready flag, or (pass 2) converts the unit's O accumulator to bf16.
#pragma once

#include "hs_common.cuh"

namespace hs {
namespace dtc {

constexpr int kD = 128;
constexpr int kSlab = 128 * 128;        // 128 rows x 64 bf16, 128-byte swizzle
constexpr int kTileBytes = 2 * kSlab;   // 128 rows x 128 bf16
constexpr int kStages = 3;              // K / V ring
constexpr int kItemRing = 4;
constexpr int kThreads = 224;
constexpr int kMaxUnits = 256;
constexpr int kAugBytes = 128 * 16 * 2;  // 128 rows x 16 bf16, unswizzled K-major
constexpr int kQAugBytes = 64 * 16 * 2;

struct Layout {
  static constexpr int kOffQ = 0;                                 // 2 x 32 KB
  static constexpr int kOffKV = kOffQ + 2 * kTileBytes;           // 3 x 32 KB
  static constexpr int kOffP = kOffKV + kStages * kTileBytes;     // 2 x 16 KB (P^T, 128 keys x 64 heads)
  static constexpr int kOffKa = kOffP + 2 * 128 * 128;            // key-side augmentation
  static constexpr int kOffQa = kOffKa + kAugBytes;               // 2 x head-side augmentation
  static constexpr int kOffCtl = kOffQa + 2 * kQAugBytes;
};

struct Ctl {
  uint64_t item_full[kItemRing], item_empty[kItemRing];
  uint64_t q_full[2], q_empty[2];
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_free[2];                 // pass 1
  uint64_t st_full[2], st_free[2], p_full[2], p_free[2], o_full, o_free;  // pass 2
  uint64_t teardown;
  uint64_t cbar;  // bounded barrier of the four compute warps
  uint64_t part_full[kItemRing];  // compute warps -> completion warp: item's results are out
  int item_id[kItemRing];
  uint32_t tmem_base;
  int abort;
  float cm[kItemRing][64], cl[kItemRing][64];  // pass 1: copy 1's (m, l), merged by copy 0
  float2 ml[kItemRing][64];                    // pass 1: the chunk's (m, l) per head
};

constexpr int smem_bytes() { return Layout::kOffCtl + int(sizeof(Ctl)) + 1024; }
static_assert(smem_bytes() <= 232448, "smem over 227 KB");

// TMEM columns
constexpr uint32_t kColS = 0;     // pass 1: S[2], 128 columns each
constexpr uint32_t kColST = 256;  // pass 2: S^T[2], 64 columns each
constexpr uint32_t kColO = 384;   // pass 2: O^T, 64 columns

struct Sched {
  int n_units, n_items, Hkv, chunk_keys;
  int n1;     // items per pass (= chunks of all units)
  int delay;  // D: pass-1 items taken before the first pass-2 item
  int cu_kv[kMaxUnits + 1];       // per sequence (batch <= kMaxUnits)
  int chunk_base[kMaxUnits + 1];  // prefix of chunks per unit
};

struct Params {
  const __nv_bfloat16* q;  // [batch, Hq, 128]
  int G, Hq, Hkv, Tq, nblk;
  float scale_log2;        // c = softmax scale * log2(e)
  double* unit_l;          // [units][64] pass-1 totals sum_j 2^(c s_j), fp64, zero on entry
  float* lse2;             // [units][64]
  float* o_acc;            // [units][64][128] fp32, zero on entry
  int* sync;               // [0] work counter, [1 + u] p1 done, [1 + U + u] ready, [1 + 2U + u] p2 done
  float* scores;           // [batch, Hkv, nblk]
  __nv_bfloat16* o;        // [batch, Hq, 128]
  float* lse;              // [Hq, Tq] natural log, may be null
  WaitCtl wc;
};

struct ItemInfo {
  int pass;   // 1 or 2
  int u, b, g, chunk;
  int key0, nkeys, ntiles;
  int kv0, kv_len;
};

__device__ __forceinline__ ItemInfo item_info(const Sched& sc, int id) {
  // merged order: pass-1 items 0..D-1, then pass-2 item j and pass-1 item D + j
  // alternately, then the remaining pass-2 items
  const int D = sc.delay, n1 = sc.n1;
  int pass, k;
  if (id < D) { pass = 1; k = id; }
  else {
    const int j = id - D;
    if (j < 2 * (n1 - D)) { pass = (j & 1) ? 1 : 2; k = (j & 1) ? D + (j >> 1) : (j >> 1); }
    else { pass = 2; k = j - (n1 - D); }
  }
  int lo = 0, hi = sc.n_units - 1;  // unit u with chunk_base[u] <= k < chunk_base[u + 1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sc.chunk_base[mid] <= k) lo = mid; else hi = mid - 1;
  }
  ItemInfo it;
  it.pass = pass;
  it.u = lo;
  it.b = it.u / sc.Hkv;
  it.g = it.u % sc.Hkv;
  it.chunk = k - sc.chunk_base[lo];
  it.kv0 = sc.cu_kv[it.b];
  it.kv_len = sc.cu_kv[it.b + 1] - it.kv0;
  it.key0 = it.chunk * sc.chunk_keys;
  it.nkeys = min(sc.chunk_keys, it.kv_len - it.key0);
  it.ntiles = (it.nkeys + 127) / 128;
  return it;
}

// L2 eviction priorities for the TMA loads
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ void tma_load_3d_hint(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                                 int c2, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5}], [%2], %6;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "l"(pol)
      : "memory");
}

// unswizzled K-major descriptor (8-row x 16-byte core matrices)
__device__ __forceinline__ uint64_t sdesc_noswz(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= uint64_t((smem_addr >> 4) & 0x3FFF);
  d |= uint64_t((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= uint64_t((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;
  return d;
}
__device__ __forceinline__ uint32_t aug_off(int r, int half) {
  return uint32_t((r >> 3) * 256 + half * 128 + (r & 7) * 16);
}

// Bounded spin on a flag another CTA raises; false (and a recorded failure)
// if it does not come up within the limit or the CTA aborted.
__device__ __noinline__ bool wait_flag(const int* flag, volatile int* abort_flag, const WaitCtl& wc, int site,
                                       int ctx) {
  const unsigned long long t0 = global_ns();
  const long long c0 = clock64();
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v != 0) return true;
    if (*abort_flag) return false;
    if (wait_expired(t0, c0, wc.timeout_ns)) {
      *abort_flag = 1;
      record_failure(wc, site, ctx);
      return false;
    }
    __nanosleep(256);
  }
}

__device__ __forceinline__ void red_add_f64(double* p, double v) {
  asm volatile("red.relaxed.gpu.global.add.f64 [%0], %1;" ::"l"(p), "d"(v) : "memory");
}

__device__ __forceinline__ void red_add_f32(float* p, float v) {
  asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    full_decode_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                          const __grid_constant__ CUtensorMap map_v, const Params p, const __grid_constant__ Sched sc) {
  using L = Layout;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl& c = *reinterpret_cast<Ctl*>(smem + L::kOffCtl);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int U = sc.n_units;
  int* work = p.sync;
  int* p1_done = p.sync + 1;
  int* ready = p.sync + 1 + U;
  int* p2_done = p.sync + 1 + 2 * U;

  // Q rows of absent heads (G < 64) stay zero: TMA writes rows < G only.
  // Key-side augmentation rows [1, 1, 1, 0, ...]; head-side upper halves zero.
  for (int i = threadIdx.x; i < 2 * kTileBytes / 16; i += kThreads)
    reinterpret_cast<uint4*>(smem + L::kOffQ)[i] = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x < 128) {
    *reinterpret_cast<uint4*>(smem + L::kOffKa + aug_off(threadIdx.x, 0)) =
        make_uint4(pack_bf16(1.f, 1.f), pack_bf16(1.f, 0.f), 0u, 0u);
    *reinterpret_cast<uint4*>(smem + L::kOffKa + aug_off(threadIdx.x, 1)) = make_uint4(0u, 0u, 0u, 0u);
    const int qb = threadIdx.x >> 6, r = threadIdx.x & 63;
    *reinterpret_cast<uint4*>(smem + L::kOffQa + qb * kQAugBytes + aug_off(r, 0)) = make_uint4(0u, 0u, 0u, 0u);
    *reinterpret_cast<uint4*>(smem + L::kOffQa + qb * kQAugBytes + aug_off(r, 1)) = make_uint4(0u, 0u, 0u, 0u);
  }
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kItemRing; ++i) {
      mbar_init(&c.item_full[i], 1);
      mbar_init(&c.item_empty[i], 6);  // 4 compute warps, the issuer, the completion warp
      mbar_init(&c.part_full[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.q_full[i], 1);
      mbar_init(&c.q_empty[i], 1);
      mbar_init(&c.s_full[i], 1);
      mbar_init(&c.s_free[i], 4);
      mbar_init(&c.st_full[i], 1);
      mbar_init(&c.st_free[i], 4);
      mbar_init(&c.p_full[i], 4);
      mbar_init(&c.p_free[i], 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&c.kv_full[s], 1);
      mbar_init(&c.kv_empty[s], 1);
    }
    mbar_init(&c.o_full, 1);
    mbar_init(&c.o_free, 4);
    mbar_init(&c.teardown, 1);
    mbar_init(&c.cbar, 4);
    c.abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&c.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_k);
    prefetch_tensormap(&map_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  volatile int* abort_flag = &c.abort;
  const float cs = p.scale_log2;

  if (warp == 4) {
    // ============================ producer ============================
    const uint64_t pol_keep = policy_evict_last(), pol_stream = policy_evict_first();
    int ctr = 0, q_uses = 0;
    int last_use[kStages] = {-1, -1, -1};
    int last_q[2] = {-1, -1};
    bool ok = true;
    auto wait0 = [&](uint64_t* bar, uint32_t parity, int site, int ctx) -> bool {
      int r = 1;
      if (lane == 0) r = mbar_wait(bar, parity, abort_flag, p.wc, site, ctx) ? 1 : 0;
      return __shfl_sync(0xffffffffu, r, 0) != 0;
    };
    // one K or V tile of the item into the next ring stage
    auto load_tile = [&](const ItemInfo& it, int tile, bool is_v, uint64_t pol, int ctx) -> bool {
      const int s = ctr % kStages;
      if (!wait0(&c.kv_empty[s], ((ctr / kStages) & 1) ^ 1, 202, ctx)) return false;
      if (lane == 0) {
        mbar_expect_tx(&c.kv_full[s], kTileBytes);
        uint8_t* dst = smem + L::kOffKV + s * kTileBytes;
        for (int sl = 0; sl < 2; ++sl)
          tma_load_3d_hint(dst + sl * kSlab, is_v ? &map_v : &map_k, &c.kv_full[s], sl * 64, it.g,
                           it.kv0 + it.key0 + tile * 128, pol);
      }
      last_use[s] = ctr;
      ++ctr;
      return true;
    };
    for (int n = 0; ok; ++n) {
      const int slot = n % kItemRing;
      if (n >= kItemRing && !wait0(&c.item_empty[slot], ((n / kItemRing) - 1) & 1, 200, n)) { ok = false; break; }
      int id = 0;
      if (lane == 0) {
        id = atomicAdd(work, 1);
        c.item_id[slot] = id < sc.n_items ? id : -1;
        mbar_arrive(&c.item_full[slot]);
      }
      id = __shfl_sync(0xffffffffu, id, 0);
      if (id >= sc.n_items) break;
      const ItemInfo it = item_info(sc, id);
      const int qb = q_uses & 1;
      if (q_uses >= 2 && !wait0(&c.q_empty[qb], ((q_uses >> 1) - 1) & 1, 201, id << 8)) { ok = false; break; }
      uint8_t* qdst = smem + L::kOffQ + qb * kTileBytes;
      if (it.pass == 1) {
        if (lane == 0) {
          mbar_expect_tx(&c.q_full[qb], 4 * 128 * p.G);
          for (int cp = 0; cp < 2; ++cp)
            for (int sl = 0; sl < 2; ++sl)
              tma_load_3d(qdst + sl * kSlab + cp * 64 * 128, &map_q, &c.q_full[qb], sl * 64, it.g * p.G, it.b);
        }
        last_q[qb] = q_uses++;
        for (int i = 0; i < it.ntiles && ok; ++i)
          if (!load_tile(it, i, false, pol_keep, (id << 8) | i)) ok = false;
      } else {
        // K(0) does not depend on lse: start it before waiting for the unit's pass 1
        if (!load_tile(it, 0, false, pol_stream, id << 8)) { ok = false; break; }
        int okf = 1;
        if (lane == 0) okf = wait_flag(ready + it.u, abort_flag, p.wc, 203, id) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, okf, 0)) { ok = false; break; }
        // head rows of the augmentation: -lse2 / c as hi + mid + lo (bf16)
        uint8_t* qa = smem + L::kOffQa + qb * kQAugBytes;
        for (int h = lane; h < 64; h += 32) {
          uint4 v = make_uint4(pack_bf16(-3.0e38f, 0.f), 0u, 0u, 0u);
          if (h < p.G) {
            const float x = -__ldcg(p.lse2 + it.u * 64 + h) / cs;
            const float hi = __bfloat162float(__float2bfloat16_rn(x));
            const float mid = __bfloat162float(__float2bfloat16_rn(x - hi));
            const float lo = x - hi - mid;
            v = make_uint4(pack_bf16(hi, mid), pack_bf16(lo, 0.f), 0u, 0u);
          }
          *reinterpret_cast<uint4*>(qa + aug_off(h, 0)) = v;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_expect_tx(&c.q_full[qb], 2 * 128 * p.G);
          for (int sl = 0; sl < 2; ++sl)
            tma_load_3d(qdst + sl * kSlab, &map_q, &c.q_full[qb], sl * 64, it.g * p.G, it.b);
        }
        last_q[qb] = q_uses++;
        // the issuer's order: K(0), then per tile i: K(i + 1), V(i)
        for (int i = 0; i < it.ntiles && ok; ++i) {
          if (i + 1 < it.ntiles && !load_tile(it, i + 1, false, pol_stream, (id << 8) | (i + 1))) { ok = false; break; }
          if (!load_tile(it, i, true, pol_stream, (id << 8) | i)) ok = false;
        }
      }
    }
    // never leave with TMA writes in flight
    if (lane == 0 && *abort_flag) {
      for (int s = 0; s < kStages; ++s)
        if (last_use[s] >= 0) mbar_wait_drain(&c.kv_full[s], (last_use[s] / kStages) & 1, p.wc, 290);
      for (int b = 0; b < 2; ++b)
        if (last_q[b] >= 0) mbar_wait_drain(&c.q_full[b], (last_q[b] >> 1) & 1, p.wc, 291);
    }
  } else if (warp == 5) {
    // ============================ UMMA issuer ============================
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16_f32(128, 128, false, false);   // S = Q K^T
      constexpr uint32_t kIdST = idesc_bf16_f32(128, 64, false, false);   // S^T = K Q^T
      constexpr uint32_t kIdPV = idesc_bf16_f32(128, 64, true, true);     // O^T += V^T P^T
      int ctr = 0, q_uses = 0, s_tiles = 0, st_tiles = 0, p2_items = 0;
      bool ok = true;
      const uint64_t q_desc0 = sdesc_sw128(smem_u32(smem + L::kOffQ), 16, 1024);
      const uint64_t k_desc0 = sdesc_sw128(smem_u32(smem + L::kOffKV), 16, 1024);
      const uint64_t v_desc0 = sdesc_sw128(smem_u32(smem + L::kOffKV), kSlab, 1024);
      const uint64_t p_desc0 = sdesc_sw128(smem_u32(smem + L::kOffP), kSlab, 1024);
      const uint64_t ka_desc = sdesc_noswz(smem_u32(smem + L::kOffKa), 128, 256);
      const uint64_t qa_desc0 = sdesc_noswz(smem_u32(smem + L::kOffQa), 128, 256);
      auto kstep = [](int kk) { return uint64_t(((kk >> 2) * kSlab + (kk & 3) * 32) >> 4); };
      auto wait_kv = [&](int site, int ctx) -> int {
        const int s = ctr % kStages;
        if (!mbar_wait(&c.kv_full[s], (ctr / kStages) & 1, abort_flag, p.wc, site, ctx)) return -1;
        ++ctr;
        return s;
      };
      // S^T(tile) of a pass-2 item into buffer st_tiles % 2
      auto issue_st = [&](int qb, int ctx) -> bool {
        const int buf = st_tiles & 1;
        const int s = wait_kv(212, ctx);
        if (s < 0) return false;
        if (st_tiles >= 2 && !mbar_wait(&c.st_free[buf], ((st_tiles >> 1) - 1) & 1, abort_flag, p.wc, 213, ctx))
          return false;
        tc_fence_after();
        const uint32_t d = tmem + kColST + buf * 64;
        const uint64_t kd = k_desc0 + uint64_t((s * kTileBytes) >> 4);
        const uint64_t qd = q_desc0 + uint64_t((qb * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) umma_bf16(d, kd + kstep(kk), qd + kstep(kk), kIdST, kk > 0 ? 1u : 0u);
        umma_bf16(d, ka_desc, qa_desc0 + uint64_t((qb * kQAugBytes) >> 4), kIdST, 1u);
        umma_commit(&c.st_full[buf]);
        umma_commit(&c.kv_empty[s]);
        ++st_tiles;
        return true;
      };
      for (int n = 0; ok; ++n) {
        const int slot = n % kItemRing;
        if (!mbar_wait(&c.item_full[slot], (n / kItemRing) & 1, abort_flag, p.wc, 210, n)) { ok = false; break; }
        const int id = c.item_id[slot];
        if (id < 0) break;
        const ItemInfo it = item_info(sc, id);
        const int qb = q_uses & 1;
        if (!mbar_wait(&c.q_full[qb], (q_uses >> 1) & 1, abort_flag, p.wc, 211, id << 8)) { ok = false; break; }
        ++q_uses;
        tc_fence_after();
        if (it.pass == 1) {
          const uint64_t qd = q_desc0 + uint64_t((qb * kTileBytes) >> 4);
          for (int i = 0; i < it.ntiles && ok; ++i) {
            const int buf = s_tiles & 1;
            const int s = wait_kv(214, (id << 8) | i);
            if (s < 0) { ok = false; break; }
            if (s_tiles >= 2 &&
                !mbar_wait(&c.s_free[buf], ((s_tiles >> 1) - 1) & 1, abort_flag, p.wc, 215, (id << 8) | i)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t kd = k_desc0 + uint64_t((s * kTileBytes) >> 4);
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk)
              umma_bf16(tmem + kColS + buf * 128, qd + kstep(kk), kd + kstep(kk), kIdS, kk > 0 ? 1u : 0u);
            umma_commit(&c.s_full[buf]);
            umma_commit(&c.kv_empty[s]);
            ++s_tiles;
          }
          if (!ok) break;
          umma_commit(&c.q_empty[qb]);
        } else {
          const int st0 = st_tiles;  // tile i of this item uses S^T buffer (st0 + i) % 2
          if (!issue_st(qb, id << 8)) { ok = false; break; }
          for (int i = 0; i < it.ntiles && ok; ++i) {
            if (i + 1 < it.ntiles && !issue_st(qb, (id << 8) | (i + 1))) { ok = false; break; }
            const int pbuf = (st0 + i) & 1;
            const int pn = st0 + i;  // P^T buffer uses so far
            if (!mbar_wait(&c.p_full[pbuf], (pn >> 1) & 1, abort_flag, p.wc, 216, (id << 8) | i)) { ok = false; break; }
            const int sv = wait_kv(217, (id << 8) | i);
            if (sv < 0) { ok = false; break; }
            if (i == 0 && p2_items > 0 &&
                !mbar_wait(&c.o_free, (p2_items - 1) & 1, abort_flag, p.wc, 218, id << 8)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t vd = v_desc0 + uint64_t((sv * kTileBytes) >> 4);
            const uint64_t pd = p_desc0 + uint64_t((pbuf * 128 * 128) >> 4);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_bf16(tmem + kColO, vd + uint64_t(kk * (2048 >> 4)), pd + uint64_t(kk * (2048 >> 4)), kIdPV,
                        (i > 0 || kk > 0) ? 1u : 0u);
            umma_commit(&c.p_free[pbuf]);
            umma_commit(&c.kv_empty[sv]);
          }
          if (!ok) break;
          umma_commit(&c.o_full);
          umma_commit(&c.q_empty[qb]);
          ++p2_items;
        }
        mbar_arrive(&c.item_empty[slot]);
      }
      umma_commit(&c.teardown);
      mbar_wait_drain(&c.teardown, 0, p.wc, 292);
    }
  } else if (warp < 4) {
    // ============================ compute warps ============================
    const int r = warp * 32 + lane;  // TMEM lane
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    int s_tiles = 0, st_tiles = 0, p2_items = 0, cb_phase = 0;
    bool ok = true;
    uint8_t* pbuf_base = smem + L::kOffP;
    // all four compute warps meet (bounded: a warp that gave up makes the
    // others give up too instead of waiting forever)
    auto cbar = [&](int ctx) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.cbar);
      const bool r2 = mbar_wait_warp(&c.cbar, cb_phase & 1, abort_flag, p.wc, 225, ctx);
      ++cb_phase;
      return r2;
    };
    for (int n = 0; ok; ++n) {
      const int slot = n % kItemRing;
      if (!mbar_wait_warp(&c.item_full[slot], (n / kItemRing) & 1, abort_flag, p.wc, 220, n)) { ok = false; break; }
      const int id = c.item_id[slot];
      if (id < 0) break;
      const ItemInfo it = item_info(sc, id);
      const int key_end = it.key0 + it.nkeys;
      if (it.pass == 1) {
        // ---------------- pass 1: (m, l) of head h over this copy's columns ----------------
        const int cp = r >> 6, h = r & 63;
        float m = -INFINITY, l = 0.f;
        for (int i = 0; i < it.ntiles; ++i) {
          const int buf = s_tiles & 1;
          if (!mbar_wait_warp(&c.s_full[buf], (s_tiles >> 1) & 1, abort_flag, p.wc, 221, (id << 8) | i)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t u32[64];
          tmem_ld32(tmem + kColS + buf * 128 + cp * 64 + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&u32[0]));
          tmem_ld32(tmem + kColS + buf * 128 + cp * 64 + 32 + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&u32[32]));
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.s_free[buf]);
          ++s_tiles;
          const int kbase = it.key0 + i * 128 + cp * 64;
          float x[64];
#pragma unroll
          for (int j = 0; j < 64; ++j) x[j] = (kbase + j < key_end) ? __uint_as_float(u32[j]) * cs : -INFINITY;
          const float mt = max_n<64>(x);
          if (mt > m) {
            l *= (m == -INFINITY) ? 0.f : ex2(m - mt);
            m = mt;
          }
          if (m > -INFINITY) {
            float a0 = 0.f, a1 = 0.f;
#pragma unroll
            for (int j = 0; j < 64; j += 4) {
              float e0, e1;
              exp2_poly_pair(x[j] - m, x[j + 1] - m, e0, e1);
              a0 += ex2(x[j + 2] - m) + e0;
              a1 += ex2(x[j + 3] - m) + e1;
            }
            l += a0 + a1;
          }
        }
        if (!ok) break;
        // copy 1 hands its (m, l) to copy 0, which leaves the chunk's pair for
        // the completion warp
        if (cp == 1) {
          c.cm[slot][h] = m;
          c.cl[slot][h] = l;
        }
        if (!cbar(id)) { ok = false; break; }
        if (cp == 0) {
          const float m1 = c.cm[slot][h], l1 = c.cl[slot][h];
          const float M = fmaxf(m, m1);
          const float Lm = (M == -INFINITY) ? 0.f : l * ex2(m - M) + l1 * ex2(m1 - M);
          c.ml[slot][h] = make_float2(M, Lm);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.part_full[slot]);
      } else {
        // ---------------- pass 2: scores, P^T, O^T ----------------
        float* srow = p.scores + size_t(it.u) * p.nblk;
        for (int i = 0; i < it.ntiles; ++i) {
          const int buf = st_tiles & 1;
          if (!mbar_wait_warp(&c.st_full[buf], (st_tiles >> 1) & 1, abort_flag, p.wc, 222, (id << 8) | i)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t u32[64];
          tmem_ld32(tmem + kColST + buf * 64 + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&u32[0]));
          tmem_ld32(tmem + kColST + buf * 64 + 32 + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&u32[32]));
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.st_free[buf]);
          const int key = it.key0 + i * 128 + r;
          const bool valid = key < key_end;
          float mx = -INFINITY;
          uint32_t pk[32];
#pragma unroll
          for (int j = 0; j < 64; j += 2) {
            float a = __uint_as_float(u32[j]) * cs, b2 = __uint_as_float(u32[j + 1]) * cs;
            if (j >= p.G || !valid) a = -INFINITY;
            if (j + 1 >= p.G || !valid) b2 = -INFINITY;
            mx = max3f(mx, a, b2);
            float e0, e1;
            if (j & 2) exp2_poly_pair(a, b2, e0, e1);
            else { e0 = ex2(a); e1 = ex2(b2); }
            pk[j >> 1] = pack_bf16(a == -INFINITY ? 0.f : e0, b2 == -INFINITY ? 0.f : e1);
          }
          if (valid) srow[key] = ex2(mx);
          // P^T row of this key: 64 heads = 128 bytes, 16-byte chunks swizzled
          if (st_tiles >= 2 &&
              !mbar_wait_warp(&c.p_free[buf], ((st_tiles >> 1) - 1) & 1, abort_flag, p.wc, 223, (id << 8) | i)) {
            ok = false;
            break;
          }
          uint8_t* prow = pbuf_base + buf * (128 * 128) + r * 128;
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)
            *reinterpret_cast<uint4*>(prow + ((q4 ^ (r & 7)) << 4)) =
                make_uint4(pk[4 * q4], pk[4 * q4 + 1], pk[4 * q4 + 2], pk[4 * q4 + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.p_full[buf]);
          ++st_tiles;
        }
        if (!ok) break;
        // O^T of this item: thread = d lane, columns = heads
        if (!mbar_wait_warp(&c.o_full, p2_items & 1, abort_flag, p.wc, 224, id << 8)) { ok = false; break; }
        tc_fence_after();
        uint32_t ov[64];
        tmem_ld32(tmem + kColO + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&ov[0]));
        tmem_ld32(tmem + kColO + 32 + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&ov[32]));
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.o_free);
        ++p2_items;
        float* acc = p.o_acc + size_t(it.u) * 64 * kD + r;
#pragma unroll
        for (int h = 0; h < 64; ++h)
          if (h < p.G) red_add_f32(acc + h * kD, __uint_as_float(ov[h]));
        __threadfence();  // the accumulator adds reach L2 before the completion warp counts the item
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.part_full[slot]);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.item_empty[slot]);
    }
  } else {
    // ============================ completion warp ============================
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int slot = n % kItemRing;
      if (!mbar_wait_warp(&c.item_full[slot], (n / kItemRing) & 1, abort_flag, p.wc, 226, n)) break;
      const int id = c.item_id[slot];
      if (id < 0) break;
      const ItemInfo it = item_info(sc, id);
      if (!mbar_wait_warp(&c.part_full[slot], (n / kItemRing) & 1, abort_flag, p.wc, 227, id)) break;
      const int nu = sc.chunk_base[it.u + 1] - sc.chunk_base[it.u];
      if (it.pass == 1) {
        for (int h = lane; h < p.G; h += 32) {
          const float2 v = c.ml[slot][h];
          if (v.y > 0.f) red_add_f64(p.unit_l + it.u * 64 + h, double(v.y) * exp2(double(v.x)));
        }
        __syncwarp();
        int last = 0;
        if (lane == 0) {
          __threadfence();
          last = atomicAdd(p1_done + it.u, 1) == nu - 1;
        }
        if (__shfl_sync(0xffffffffu, last, 0)) {
          __threadfence();
          for (int h = lane; h < p.G; h += 32) {
            const double tot = __ldcg(p.unit_l + it.u * 64 + h);
            p.lse2[it.u * 64 + h] = tot > 0.0 ? float(log2(tot)) : -INFINITY;
          }
          __threadfence();
          __syncwarp();
          if (lane == 0) asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(ready + it.u), "r"(1) : "memory");
        }
      } else {
        int last = 0;
        if (lane == 0) {
          __threadfence();
          last = atomicAdd(p2_done + it.u, 1) == nu - 1;
        }
        if (__shfl_sync(0xffffffffu, last, 0)) {
          // the unit's O: accumulator -> bf16, lane = 4 consecutive d
          __threadfence();
          const float4* acc = reinterpret_cast<const float4*>(p.o_acc + size_t(it.u) * 64 * kD) + lane;
          const int hq0 = it.g * p.G;
          for (int h0 = 0; h0 < p.G; h0 += 8) {
            float4 v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = h0 + e < p.G ? __ldcg(acc + (h0 + e) * (kD / 4)) : make_float4(0, 0, 0, 0);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if (h0 + e < p.G)
                *reinterpret_cast<uint2*>(p.o + (size_t(it.b) * p.Hq + hq0 + h0 + e) * kD + lane * 4) =
                    make_uint2(pack_bf16(v[e].x, v[e].y), pack_bf16(v[e].z, v[e].w));
          }
          if (p.lse)
            for (int h = lane; h < p.G; h += 32)
              p.lse[size_t(hq0 + h) * p.Tq + it.b] = __ldcg(p.lse2 + it.u * 64 + h) * 0.69314718055994531f;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.item_empty[slot]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}


// ============================================================================
// Sparse-layer decode on the tensor cores
// ============================================================================
// One new token per sequence attends over V_q = {j in idx : j <= pos - w} U
// [pos - w + 1, pos] of the full layer's KV cache (HySparse2 release note on
// airebao.com: the sparse layers reuse the full layer's cache and its top-k
// tokens, with the most recent tokens forced in; its key-data table sizes an
// FP8 KV cache). Slots of a (sequence, KV head) unit: the window first
// (slot s < min(w, pos + 1) holds key pos - w + 1 + s, or s when the window
// reaches back to 0), then selected token j at slot w + j when
// idx[j] <= pos - w; other slots are empty and masked. The unit's 128-slot
// tiles are cut into `nsplit` contiguous ranges, one work item each; with
// more than one range, the unit's last item merges the ranges' partials.
//
// Rows of the MMA tile are two copies of the G <= 64 heads; copy c reduces
// key columns [64c, 64c + 64) of each 128-key tile with its own online softmax
// (lazy rescale, P kept in tensor memory over S) and writes zeros for the
// other half, so O rows of copy c sum over that copy's keys only. At the end
// of an item copy 1 hands its (m, l, O) to copy 0 through shared memory (the
// Q buffer, free once the item's last QK is done).
// The producer warp lists each tile's rows: it loads an item's sequence
// bounds, selection count and first candidate indices in one round trip, and
// the indices of several tiles per round trip after that (FP8: then their
// scales). Two loader warps copy the listed rows with 16-byte cp.async, every
// thread keeping several tiles' copies in flight: the rows are scattered
// 256-byte (bf16) or 128-byte (FP8) pieces, and the number of bytes in flight
// per SM is what bounds their rate. bf16 KV lands in the ring tile in the
// 128-byte swizzle the MMA reads. FP8 KV lands in a staging tile; the thread
// that copied a piece expands it to fp16 into the ring tile (every e4m3 value
// is an fp16 value), Q is converted to fp16 in shared memory, and the MMAs run
// with fp16 operands. The K scale multiplies the logits, the V scale the
// probabilities before PV. The issuer thread loads Q (TMA) when the previous
// item has released the buffer, so the slot lists and copies of the next item
// run ahead across item boundaries.
namespace sdec {

template <bool FP8>
constexpr int stages() { return FP8 ? 4 : 5; }  // 32 KB K or V ring tiles, in the order K0 V0 K1 V1 ...
constexpr int kMaxStages = 5;
template <bool FP8>
constexpr int lag() { return FP8 ? 2 : 3; }     // copy groups a loader thread keeps in flight behind the newest
constexpr int kRaw = 3;                          // FP8 staging tiles (e4m3, 128 rows x 128 bytes) = lag + 1
constexpr int kRawBytes = 128 * 128;
constexpr int kMeta = 6;                         // per-tile slot metadata ring
constexpr int kBatch = 8;                        // tiles whose candidate indices are fetched per round trip
constexpr int kMaxUnits = 1 << 20;
constexpr int kMaxSplit = 8;                     // a unit's ranges are one thread-block cluster (portable size)
constexpr int kLoadWarps = 4;
constexpr int kLoadThreads = 32 * kLoadWarps;
// warps 0-3 softmax, 4 slot lists, 5 MMA issuer, 6-9 loaders
constexpr int kThreads = 192 + kLoadThreads;
static_assert(lag<true>() + 1 == kRaw, "FP8 staging ring = copy groups in flight");

struct Meta {
  int row[128];       // packed row (token * Hkv + g) to load for each slot
  uint32_t valid[4];  // bit (4l + e) of word e: slot 4l + e holds a visible key
  float ks[128], vs[128];  // FP8: the rows' scales, copied by the loaders with the tile's K
};

template <bool FP8>
struct Layout {
  static constexpr int kOffQ = 0;                                      // 32 KB (Q, then copy 1's O at item end)
  static constexpr int kOffKV = kTileBytes;                            // ring of 32 KB tiles
  static constexpr int kOffRaw = kOffKV + stages<FP8>() * kTileBytes;  // FP8 staging
  static constexpr int kOffMeta = kOffRaw + (FP8 ? kRaw * kRawBytes : 0);
  static constexpr int kOffCtl = kOffMeta + kMeta * int(sizeof(Meta));
  // at the end of a range (cluster launch): the range's (m, l) and unnormalised O, in the ring
  static constexpr int kOffPartO = kOffKV;                 // [64 heads][32 float4], float4 j of head h at j ^ (h & 7)
  static constexpr int kOffPartML = kOffKV + 64 * 128 * 4;  // [64] float2 (m, l), log2 units
};

struct Ctl {
  uint64_t q_full, q_ready, q_empty;
  uint64_t kv_full[kMaxStages], kv_empty[kMaxStages];
  uint64_t meta_full[kMeta], meta_empty[kMeta], sc_full[kMeta];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t o_full, o_free, cbar, teardown;
  uint32_t tmem_base;
  int abort;
  float cm[64], cl[64];  // copy 1's (m, l) at item end
};

template <bool FP8>
constexpr int smem_bytes() { return Layout<FP8>::kOffCtl + int(sizeof(Ctl)) + 1024; }
static_assert(smem_bytes<false>() <= 232448 && smem_bytes<true>() <= 232448, "smem over 227 KB");
static_assert(Layout<true>::kOffPartML + 64 * 8 <= Layout<true>::kOffRaw, "partials fit in the ring");

struct Params {
  const int* idx;     // [units, topk] (tile = sequence for decode)
  const int* cnt;     // [units]
  const int* cu_kv;   // device prefix sums
  const uint8_t* k;   // cache rows [T_kv * Hkv]: 128 bf16 (256 bytes) or 128 e4m3 codes
  const uint8_t* v;
  const float* k_scale;  // [T_kv, Hkv]
  const float* v_scale;
  int topk, w, G, Hq, Hkv, Tq;
  int log2_block;  // selected blocks of 2^log2_block keys (0: token level)
  int n_units, nsplit, tiles_per_split, unit_tiles, n_items;
  float scale_log2;
  __nv_bfloat16* o;
  float* lse;
  WaitCtl wc;
};

// FP16 operands (FP8 KV): kind::f16 with a/b format F16 (0), fp32 accumulate
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (uint32_t(a_mn_major) << 15) | (uint32_t(b_mn_major) << 16) | (uint32_t(N >> 3) << 17) |
         (uint32_t(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Launch: nsplit == 1 -> grid min(SMs, items), each CTA loops over items;
// nsplit > 1 -> one CTA per item, clusters of nsplit CTAs (a unit's ranges),
// merged through distributed shared memory at the end.
template <bool FP8>
__global__ void __launch_bounds__(kThreads, 1)
    sparse_decode_tc_kernel(const __grid_constant__ CUtensorMap map_q, const Params p) {
  using L = Layout<FP8>;
  constexpr int kSt = stages<FP8>();
  constexpr int kLag = lag<FP8>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctl& c = *reinterpret_cast<Ctl*>(smem + L::kOffCtl);
  Meta* meta = reinterpret_cast<Meta*>(smem + L::kOffMeta);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // the first item's sequence bounds, count and first candidate indices head
  // for L2 while the CTA sets up (kBatch tiles = 32 lanes x 128 bytes)
  if (warp == 4 && int(blockIdx.x) < p.n_items) {
    const int u = blockIdx.x / p.nsplit;
    const int j0 = ((blockIdx.x % p.nsplit) * p.tiles_per_split * 128 - p.w + lane * 32) >> p.log2_block;
    if (lane == 0) {
      prefetch_l2(p.cu_kv + u / p.Hkv);
      if (p.cnt) prefetch_l2(p.cnt + u);
    }
    if (p.cnt && j0 + 31 >= 0 && j0 < p.topk) prefetch_l2(p.idx + size_t(u) * p.topk + max(j0, 0));
  }
  for (int i = threadIdx.x; i < kTileBytes / 16; i += kThreads)
    reinterpret_cast<uint4*>(smem + L::kOffQ)[i] = make_uint4(0u, 0u, 0u, 0u);  // Q rows of absent heads
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(&c.q_full, 1);
    mbar_init(&c.q_ready, kLoadWarps);  // FP8: the loader warps turned Q into fp16
    mbar_init(&c.q_empty, 4);           // the softmax warps are done with the buffer (Q, then the copy merge)
    for (int s = 0; s < kSt; ++s) {
      mbar_init(&c.kv_full[s], kLoadWarps);
      mbar_init(&c.kv_empty[s], 1);
    }
    for (int m = 0; m < kMeta; ++m) {
      mbar_init(&c.meta_full[m], 1);
      mbar_init(&c.meta_empty[m], 4 + kLoadWarps);  // softmax warps and loader warps
      mbar_init(&c.sc_full[m], kLoadWarps);         // FP8: the tile's scales have landed
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.s_full[i], 1);
      mbar_init(&c.p_full[i], 4);
      mbar_init(&c.pv_done[i], 1);
    }
    mbar_init(&c.o_full, 1);
    mbar_init(&c.o_free, 4);
    mbar_init(&c.cbar, 4);
    mbar_init(&c.teardown, 1);
    c.abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&c.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 5 && lane == 0) prefetch_tensormap(&map_q);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  volatile int* abort_flag = &c.abort;
  const float cs = p.scale_log2;
  // item -> unit u, tiles [t0, t1) of its slot space
  auto item_tiles = [&](int it, int& u, int& t0, int& t1) {
    u = it / p.nsplit;
    t0 = (it % p.nsplit) * p.tiles_per_split;
    t1 = min(p.unit_tiles, t0 + p.tiles_per_split);
  };

  if (warp == 4) {
    // ============================ producer: slot lists ============================
    int mctr = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x) {
      int u, t0, t1;
      item_tiles(it, u, t0, t1);
      const int n = t1 - t0;
      const int b = u / p.Hkv, g = u % p.Hkv;
      // the sequence bounds, the selection count and the first batch of
      // candidate indices do not depend on one another: one round trip
      const int kv0 = __ldg(p.cu_kv + b);
      const int kv1 = __ldg(p.cu_kv + b + 1);
      const int cnt = p.cnt ? __ldg(p.cnt + u) : 0;
      for (int tb = 0; tb < n && ok; tb += kBatch) {
        // slot keys of tiles tb .. tb + kBatch - 1 (lane: slots 4 lane .. 4 lane + 3 of each)
        int key[kBatch][4];
#pragma unroll
        for (int bi = 0; bi < kBatch; ++bi)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // selected part: slot w + j holds key idx[j >> log2 B] * B + (j mod B)
            const int jsel = (t0 + tb + bi) * 128 + lane * 4 + e - p.w;
            const int jb = jsel >> p.log2_block;
            key[bi][e] = (p.cnt && tb + bi < n && jsel >= 0 && jb < p.topk)
                             ? (__ldg(p.idx + size_t(u) * p.topk + jb) << p.log2_block) +
                                   (jsel & ((1 << p.log2_block) - 1))
                             : -1;
          }
        const int pos = kv1 - kv0 - 1;
        const int win_lo = max(0, pos - p.w + 1);
        const int n_win = p.w > 0 ? pos - win_lo + 1 : 0;
#pragma unroll
        for (int bi = 0; bi < kBatch; ++bi)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int slot = (t0 + tb + bi) * 128 + lane * 4 + e;
            const int jsel = slot - p.w;
            if (slot < n_win) key[bi][e] = win_lo + slot;
            else if (jsel < 0 || (jsel >> p.log2_block) >= cnt || key[bi][e] > pos - p.w) key[bi][e] = -1;
          }
#pragma unroll
        for (int bi = 0; bi < kBatch; ++bi) {
          const int i = tb + bi;
          if (i < n && ok) {
            const int m = mctr % kMeta;
            bool got = true;
            if (mctr >= kMeta) {
              int r = 1;
              if (lane == 0)
                r = mbar_wait(&c.meta_empty[m], ((mctr / kMeta) - 1) & 1, abort_flag, p.wc, 302, (it << 8) | i) ? 1 : 0;
              got = __shfl_sync(0xffffffffu, r, 0) != 0;
            }
            if (!got) {
              ok = false;
              continue;
            }
            Meta& mt = meta[m];
            uint32_t vbits = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int k2 = key[bi][e];
              mt.row[lane * 4 + e] = (kv0 + (k2 >= 0 ? k2 : 0)) * p.Hkv + g;
              vbits |= uint32_t(k2 >= 0) << e;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint32_t bl = __ballot_sync(0xffffffffu, (vbits >> e) & 1u);
              if (lane == 0) mt.valid[e] = bl;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&c.meta_full[m]);
            ++mctr;
          }
        }
      }
    }
  } else if (warp == 5) {
    // ============================ UMMA issuer ============================
    if (lane == 0) {
      constexpr uint32_t kIdQK = FP8 ? idesc_f16_f32(128, 128, false, false) : idesc_bf16_f32(128, 128, false, false);
      constexpr uint32_t kIdPV = FP8 ? idesc_f16_f32(128, 128, false, true) : idesc_bf16_f32(128, 128, false, true);
      int ctr = 0, q_uses = 0, tiles = 0, items = 0;
      bool ok = true;
      const uint64_t q_desc = sdesc_sw128(smem_u32(smem + L::kOffQ), 16, 1024);
      const uint64_t k_desc0 = sdesc_sw128(smem_u32(smem + L::kOffKV), 16, 1024);
      const uint64_t v_desc0 = sdesc_sw128(smem_u32(smem + L::kOffKV), kSlab, 1024);
      auto kstep = [](int kk) { return uint64_t(((kk >> 2) * kSlab + (kk & 3) * 32) >> 4); };
      auto wait_kv = [&](int site, int ctx) -> int {
        const int s = ctr % kSt;
        if (!mbar_wait(&c.kv_full[s], (ctr / kSt) & 1, abort_flag, p.wc, site, ctx)) return -1;
        ++ctr;
        return s;
      };
      auto issue_qk = [&](int buf, int ctx) -> bool {
        const int s = wait_kv(311, ctx);
        if (s < 0) return false;
        tc_fence_after();
        const uint64_t kd = k_desc0 + uint64_t((s * kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk)
          umma_bf16(tmem + buf * 128, q_desc + kstep(kk), kd + kstep(kk), kIdQK, kk > 0 ? 1u : 0u);
        umma_commit(&c.s_full[buf]);
        umma_commit(&c.kv_empty[s]);
        return true;
      };
      for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x) {
        int u, t0, t1;
        item_tiles(it, u, t0, t1);
        const int n = t1 - t0;
        const int b = u / p.Hkv, g = u % p.Hkv;
        // Q of the item (two copies of its G heads) once the buffer is free
        if (q_uses > 0 && !mbar_wait(&c.q_empty, (q_uses - 1) & 1, abort_flag, p.wc, 301, it << 8)) { ok = false; break; }
        mbar_expect_tx(&c.q_full, 4 * 128 * p.G);
        for (int cp = 0; cp < 2; ++cp)
          for (int sl = 0; sl < 2; ++sl)
            tma_load_3d(smem + L::kOffQ + sl * kSlab + cp * 64 * 128, &map_q, &c.q_full, sl * 64, g * p.G, b);
        if (!mbar_wait(&c.q_full, q_uses & 1, abort_flag, p.wc, 310, it << 8)) {
          mbar_wait_drain(&c.q_full, q_uses & 1, p.wc, 391);  // no copy outlives the kernel
          ok = false;
          break;
        }
        if (FP8 && !mbar_wait(&c.q_ready, q_uses & 1, abort_flag, p.wc, 316, it << 8)) { ok = false; break; }
        ++q_uses;
        tc_fence_after();
        // ring order K0 V0 K1 V1 ...: QK(i + 1) is issued while V(i) is held,
        // before PV(i), so the tensor core computes S(i + 1) during softmax(i);
        // PV(i) precedes QK(i + 2) into the same S buffer (in-order execution)
        if (!issue_qk(tiles & 1, it << 8)) { ok = false; break; }
        int sv = wait_kv(313, it << 8);
        if (sv < 0) { ok = false; break; }
        for (int i = 0; i < n && ok; ++i) {
          const int buf = (tiles + i) & 1;
          if (i + 1 < n && !issue_qk(buf ^ 1, (it << 8) | (i + 1))) { ok = false; break; }
          if (!mbar_wait(&c.p_full[buf], ((tiles + i) >> 1) & 1, abort_flag, p.wc, 312, (it << 8) | i)) { ok = false; break; }
          if (i == 0 && items > 0 && !mbar_wait(&c.o_free, (items - 1) & 1, abort_flag, p.wc, 314, it << 8)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t vd = v_desc0 + uint64_t((sv * kTileBytes) >> 4);
          const uint32_t pa = tmem + buf * 128;  // P over the first 64 columns of S
          umma_bf16_ts(tmem + 256, pa, vd, kIdPV, i > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 1; kk < 8; ++kk) umma_bf16_ts(tmem + 256, pa + kk * 8, vd + uint64_t(kk * (2048 >> 4)), kIdPV, 1u);
          umma_commit(&c.pv_done[buf]);
          umma_commit(&c.kv_empty[sv]);
          if (i + 1 < n && (sv = wait_kv(313, (it << 8) | (i + 1))) < 0) { ok = false; break; }
        }
        if (!ok) break;
        tiles += n;
        ++items;
        umma_commit(&c.o_full);
      }
      umma_commit(&c.teardown);
      mbar_wait_drain(&c.teardown, 0, p.wc, 392);
    }
  } else if (warp < 4) {
    // ============================ softmax warps ============================
    const int r = warp * 32 + lane;
    const int cp = r >> 6, h = r & 63;
    const uint32_t lane_base = uint32_t(warp * 32) << 16;
    int tiles = 0, items = 0, cb_phase = 0, mctr = 0;
    bool ok = true;
    auto cbar = [&](int ctx) -> bool {
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.cbar);
      const bool r2 = mbar_wait_warp(&c.cbar, cb_phase & 1, abort_flag, p.wc, 325, ctx);
      ++cb_phase;
      return r2;
    };
    float* scratch = reinterpret_cast<float*>(smem + L::kOffQ);  // [64 heads][128] at item end
    for (int it = blockIdx.x; it < p.n_items && ok; it += gridDim.x) {
      int u, t0, t1;
      item_tiles(it, u, t0, t1);
      const int n = t1 - t0;
      float m_used = -INFINITY, l = 0.f;
      for (int i = 0; i < n; ++i) {
        const int buf = (tiles + i) & 1;
        const int mm = mctr % kMeta;
        if (!mbar_wait_warp(&c.meta_full[mm], (mctr / kMeta) & 1, abort_flag, p.wc, 320, (it << 8) | i) ||
            (FP8 && !mbar_wait_warp(&c.sc_full[mm], (mctr / kMeta) & 1, abort_flag, p.wc, 324, (it << 8) | i)) ||
            !mbar_wait_warp(&c.s_full[buf], ((tiles + i) >> 1) & 1, abort_flag, p.wc, 321, (it << 8) | i)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const Meta& mt = meta[mm];
        uint32_t u32[64];
        tmem_ld32(tmem + buf * 128 + cp * 64 + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&u32[0]));
        tmem_ld32(tmem + buf * 128 + cp * 64 + 32 + lane_base, *reinterpret_cast<uint32_t(*)[32]>(&u32[32]));
        tmem_ld_wait();
        float x[64];
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const int col = cp * 64 + j;
          float v = __uint_as_float(u32[j]) * cs;
          if (FP8) v *= mt.ks[col];
          x[j] = ((mt.valid[col & 3] >> (col >> 2)) & 1u) ? v : -INFINITY;
        }
        const float mt_max = max_n<64>(x);
        float factor = 1.f;
        bool rescale = false;
        if (mt_max > m_used + 8.f) {
          factor = (m_used == -INFINITY) ? 0.f : ex2(m_used - mt_max);
          m_used = mt_max;
          rescale = true;
        }
        const float nmu = (m_used == -INFINITY) ? 0.f : -m_used;
        float rs0 = 0.f, rs1 = 0.f;
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          float e0, e1;
          if (j & 2) exp2_poly_pair(x[j] + nmu, x[j + 1] + nmu, e0, e1);
          else { e0 = ex2(x[j] + nmu); e1 = ex2(x[j + 1] + nmu); }
          if (x[j] == -INFINITY) e0 = 0.f;
          if (x[j + 1] == -INFINITY) e1 = 0.f;
          rs0 += e0;
          rs1 += e1;
          if (FP8) pk[j >> 1] = pack_f16(e0 * mt.vs[cp * 64 + j], e1 * mt.vs[cp * 64 + j + 1]);
          else pk[j >> 1] = pack_bf16(e0, e1);
        }
        l = l * factor + (rs0 + rs1);
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.meta_empty[mm]);
        ++mctr;
        // P of this copy's 64 keys into its 32 columns, zeros into the other 32
        uint32_t zero[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) zero[j] = 0u;
        if (cp == 0) {
          tmem_st32(tmem + buf * 128 + lane_base, pk);
          tmem_st32(tmem + buf * 128 + 32 + lane_base, zero);
        } else {
          tmem_st32(tmem + buf * 128 + lane_base, zero);
          tmem_st32(tmem + buf * 128 + 32 + lane_base, pk);
        }
        // O rescale: PV(i - 1) must be complete first (it is not implied here)
        if (__any_sync(0xffffffffu, rescale && i > 0)) {
          if (!mbar_wait_warp(&c.pv_done[buf ^ 1], ((tiles + i - 1) >> 1) & 1, abort_flag, p.wc, 322, (it << 8) | i)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float f = (rescale && i > 0) ? factor : 1.f;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t ov[32];
            tmem_ld32(tmem + 256 + ch * 32 + lane_base, ov);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) ov[j] = __float_as_uint(__uint_as_float(ov[j]) * f);
            tmem_st32(tmem + 256 + ch * 32 + lane_base, ov);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.p_full[buf]);
      }
      if (!ok) break;
      tiles += n;
      // ---- item end: copy 1 hands (m, l, O) to copy 0 through the Q buffer ----
      if (!mbar_wait_warp(&c.o_full, items & 1, abort_flag, p.wc, 323, it << 8)) { ok = false; break; }
      tc_fence_after();
      if (cp == 1) {
        float* dst = scratch + h * kD;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t ov[32];
          tmem_ld32(tmem + 256 + ch * 32 + lane_base, ov);
          tmem_ld_wait();
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4)  // float4 slot q4 of row h at q4 ^ (h & 7): conflict-free banks
            reinterpret_cast<float4*>(dst + ch * 32)[q4 ^ (h & 7)] =
                make_float4(__uint_as_float(ov[4 * q4]), __uint_as_float(ov[4 * q4 + 1]),
                            __uint_as_float(ov[4 * q4 + 2]), __uint_as_float(ov[4 * q4 + 3]));
        }
        c.cm[h] = m_used;
        c.cl[h] = l;
      }
      if (!cbar(it)) { ok = false; break; }
      const int b = u / p.Hkv, g = u % p.Hkv;
      if (cp == 0) {
        // every lane of warps 0-1 takes part in the (warp-collective) TMEM
        // loads; rows of absent heads (h >= G) only skip the stores
        const bool has_head = h < p.G;
        const float m1 = c.cm[h], l1 = c.cl[h];
        const float M = fmaxf(m_used, m1);
        const float w0 = (M == -INFINITY) ? 0.f : ex2(m_used - M), w1 = (M == -INFINITY) ? 0.f : ex2(m1 - M);
        const float Lm = l * w0 + l1 * w1;
        const bool direct = p.nsplit == 1;  // the item is the whole unit: write O and lse
        const float inv = direct ? (Lm > 0.f ? 1.f / Lm : 0.f) : 1.f;
        const float* src = scratch + h * kD;
        // a range's partial stays in this CTA's ring for the cluster merge
        float4* po = reinterpret_cast<float4*>(smem + L::kOffPartO) + h * 32;
        uint2* dst = reinterpret_cast<uint2*>(p.o + (size_t(b) * p.Hq + g * p.G + min(h, p.G - 1)) * kD);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t ov[32];
          tmem_ld32(tmem + 256 + ch * 32 + lane_base, ov);
          tmem_ld_wait();
#pragma unroll
          for (int q4 = 0; q4 < 8; ++q4) {
            const float4 o1 = reinterpret_cast<const float4*>(src + ch * 32)[q4 ^ (h & 7)];  // as written
            const float4 v = make_float4((__uint_as_float(ov[4 * q4]) * w0 + o1.x * w1) * inv,
                                         (__uint_as_float(ov[4 * q4 + 1]) * w0 + o1.y * w1) * inv,
                                         (__uint_as_float(ov[4 * q4 + 2]) * w0 + o1.z * w1) * inv,
                                         (__uint_as_float(ov[4 * q4 + 3]) * w0 + o1.w * w1) * inv);
            if (has_head) {
              if (direct) dst[ch * 8 + q4] = make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
              else po[(ch * 8 + q4) ^ (h & 7)] = v;
            }
          }
        }
        if (has_head) {
          if (direct) {
            if (p.lse) p.lse[size_t(g * p.G + h) * p.Tq + b] = (Lm > 0.f ? M + __log2f(Lm) : -INFINITY) * 0.69314718055994531f;
          } else {
            reinterpret_cast<float2*>(smem + L::kOffPartML)[h] = make_float2(M, Lm);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&c.o_free);
        mbar_arrive(&c.q_empty);
      }
      ++items;
    }
  } else {
    // ============================ loader warps ============================
    // Steps K0 V0 K1 V1 ... of the CTA's items, each 128 listed rows. Issue:
    // 16-byte cp.async of every row piece (bf16: into ring tile `step % kSt`
    // in the 128-byte swizzle; FP8: into staging tile `step % kRaw`, and with
    // a K step the rows' K and V scales into the tile's metadata), one commit
    // group per step. Completion, kLag steps later: wait for the thread's
    // group (FP8: signal the scales, then expand the thread's own pieces to
    // fp16 into the ring tile), fence for the tensor core, arrive on the
    // tile's barrier. The ring tile is claimed at issue (bf16) or at
    // completion (FP8); either way the issuer can always release enough
    // tiles for the loaders to move on (it holds at most V(i) and K(i + 1)
    // while waiting). Each warp issues its own copies: the number of warps
    // issuing scattered copies is what sets the rate.
    const int t = threadIdx.x - 192;  // 0 .. kLoadThreads - 1
    int issued = 0, completed = 0, mi = 0, cmi = 0, q_uses = 0;
    bool ok = true;
    // cursors over (item, step within the item)
    int iss_it = blockIdx.x, iss_n = 0, iss_i2 = 0, cmp_it = blockIdx.x, cmp_n = 0, cmp_i2 = 0;
    auto item_len = [&](int it) {
      int u, t0, t1;
      item_tiles(it, u, t0, t1);
      return t1 - t0;
    };
    if (iss_it < p.n_items) iss_n = cmp_n = item_len(iss_it);
    while (ok) {
      if (iss_it < p.n_items) {
        const bool is_v = iss_i2 & 1;
        const int mm = mi % kMeta;
        const int ctx = (iss_it << 8) | (iss_i2 >> 1);
        if (!is_v && !mbar_wait_warp(&c.meta_full[mm], (mi / kMeta) & 1, abort_flag, p.wc, 331, ctx)) {
          ok = false;
          break;
        }
        const int* rows = meta[mm].row;
        const uint8_t* src = is_v ? p.v : p.k;
        if constexpr (!FP8) {
          const int s = issued % kSt;
          if (!mbar_wait_warp(&c.kv_empty[s], ((issued / kSt) & 1) ^ 1, abort_flag, p.wc, 332, ctx)) {
            ok = false;
            break;
          }
          uint8_t* dst = smem + L::kOffKV + s * kTileBytes;
          const int ch = t & 15;  // 16-byte piece of the 256-byte row
#pragma unroll
          for (int j = 0; j < 2048 / kLoadThreads; ++j) {
            const int row = (t >> 4) + (kLoadThreads / 16) * j;
            cp_async16(dst + (ch >> 3) * kSlab + row * 128 + (((ch & 7) ^ (row & 7)) << 4),
                       src + size_t(rows[row]) * 256 + ch * 16);
          }
        } else {
          uint8_t* dst = smem + L::kOffRaw + (issued % kRaw) * kRawBytes;
          const int sub = t & 7;  // 16-code piece of the 128-byte row
#pragma unroll
          for (int j = 0; j < 1024 / kLoadThreads; ++j) {
            const int row = (t >> 3) + (kLoadThreads / 8) * j;
            cp_async16(dst + row * 128 + sub * 16, src + size_t(rows[row]) * 128 + sub * 16);
          }
          if (!is_v) {
            static_assert(kLoadThreads == 128, "one scale pair per loader thread");
            cp_async4(&meta[mm].ks[t], p.k_scale + rows[t]);
            cp_async4(&meta[mm].vs[t], p.v_scale + rows[t]);
          }
        }
        cp_async_commit();
        if (is_v) {  // the loaders are done with the tile's row list
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.meta_empty[mm]);
          ++mi;
        }
        ++issued;
        if (++iss_i2 == 2 * iss_n) {
          iss_i2 = 0;
          iss_it += gridDim.x;
          if (iss_it < p.n_items) iss_n = item_len(iss_it);
        }
      }
      if (completed == issued) break;
      const bool tail = iss_it >= p.n_items;
      if (!tail && issued - completed <= kLag) continue;
      if (tail) cp_async_wait<0>();
      else cp_async_wait<kLag>();
      // ---- completion of step `completed` ----
      const int s = completed % kSt;
      const int ctx = (cmp_it << 8) | (cmp_i2 >> 1);
      if constexpr (FP8) {
        if (!(cmp_i2 & 1)) {  // a K step: the tile's scales are in place
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.sc_full[cmi % kMeta]);
        } else {
          ++cmi;
        }
        if (cmp_i2 == 0) {
          // the item's first step: its Q (row t) to fp16 for the issuer
          if (!mbar_wait_warp(&c.q_full, q_uses & 1, abort_flag, p.wc, 330, ctx)) {
            ok = false;
            break;
          }
          static_assert(kLoadThreads == 128, "one Q row per loader thread");
#pragma unroll 4
          for (int chn = 0; chn < 16; ++chn) {
            uint8_t* ptr = smem + L::kOffQ + (chn >> 3) * kSlab + t * 128 + (((chn & 7) ^ (t & 7)) << 4);
            uint4 v = *reinterpret_cast<uint4*>(ptr);
            uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[e]));
              w4[e] = pack_f16(f.x, f.y);
            }
            *reinterpret_cast<uint4*>(ptr) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&c.q_ready);
          ++q_uses;
        }
        if (!mbar_wait_warp(&c.kv_empty[s], ((completed / kSt) & 1) ^ 1, abort_flag, p.wc, 332, ctx)) {
          ok = false;
          break;
        }
        const uint8_t* raw = smem + L::kOffRaw + (completed % kRaw) * kRawBytes;
        uint8_t* dst = smem + L::kOffKV + s * kTileBytes;
        const int sub = t & 7;
#pragma unroll 4
        for (int j = 0; j < 1024 / kLoadThreads; ++j) {
          const int row = (t >> 3) + (kLoadThreads / 8) * j;
          const uint4 r4 = *reinterpret_cast<const uint4*>(raw + row * 128 + sub * 16);  // this thread's copy
          const uint32_t w4[4] = {r4.x, r4.y, r4.z, r4.w};
          uint32_t hv[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hv[2 * e]) : "h"(uint16_t(w4[e] & 0xFFFFu)));
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(hv[2 * e + 1]) : "h"(uint16_t(w4[e] >> 16)));
          }
          // codes 16 sub .. 16 sub + 15 = fp16 elements -> chunks 2 sub, 2 sub + 1 of the row
#pragma unroll
          for (int hc = 0; hc < 2; ++hc) {
            const int chn = 2 * sub + hc;
            *reinterpret_cast<uint4*>(dst + (chn >> 3) * kSlab + row * 128 + (((chn & 7) ^ (row & 7)) << 4)) =
                make_uint4(hv[4 * hc], hv[4 * hc + 1], hv[4 * hc + 2], hv[4 * hc + 3]);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.kv_full[s]);
      ++completed;
      if (++cmp_i2 == 2 * cmp_n) {
        cmp_i2 = 0;
        cmp_it += gridDim.x;
        if (cmp_it < p.n_items) cmp_n = item_len(cmp_it);
      }
    }
    cp_async_wait<0>();  // no copy outlives the loaders (abort paths included)
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (p.nsplit > 1) {
    // ---- the unit's ranges are the CTAs of this cluster: merge their partials ----
    // CTA rank r writes heads r, r + nsplit, ...; thread = (head, quarter of d).
    // Every thread of every CTA passes both cluster barriers (abort paths too):
    // the second keeps each CTA's shared memory alive while its peers read it.
    cluster_sync_all();
    const int rank = int(cluster_ctarank());
    const int t = threadIdx.x;
    const int hh = rank + p.nsplit * (t >> 2), part = t & 3;
    if (t < 128 && hh < p.G) {
      const int u = blockIdx.x / p.nsplit, b = u / p.Hkv, g = u % p.Hkv;
      const float2* ml_local = reinterpret_cast<const float2*>(smem + L::kOffPartML) + hh;
      const float4* o_local = reinterpret_cast<const float4*>(smem + L::kOffPartO) + hh * 32;
      float M = -INFINITY;
      for (int q = 0; q < p.nsplit; ++q) M = fmaxf(M, ld_dsmem_f2(dsmem_addr(ml_local, q)).x);
      float Lsum = 0.f;
      float4 acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int q = 0; q < p.nsplit; ++q) {
        const float2 ml = ld_dsmem_f2(dsmem_addr(ml_local, q));
        const float wq = ml.x == -INFINITY ? 0.f : ex2(ml.x - M);
        Lsum += wq * ml.y;
        float4 v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = ld_dsmem_f4(dsmem_addr(o_local + ((part * 8 + e) ^ (hh & 7)), q));
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          acc[e].x = fmaf(wq, v[e].x, acc[e].x);
          acc[e].y = fmaf(wq, v[e].y, acc[e].y);
          acc[e].z = fmaf(wq, v[e].z, acc[e].z);
          acc[e].w = fmaf(wq, v[e].w, acc[e].w);
        }
      }
      const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
      uint4* dst = reinterpret_cast<uint4*>(p.o + (size_t(b) * p.Hq + g * p.G + hh) * kD + part * 32);
#pragma unroll
      for (int e = 0; e < 8; e += 2)
        dst[e >> 1] = make_uint4(pack_bf16(acc[e].x * inv, acc[e].y * inv), pack_bf16(acc[e].z * inv, acc[e].w * inv),
                                 pack_bf16(acc[e + 1].x * inv, acc[e + 1].y * inv),
                                 pack_bf16(acc[e + 1].z * inv, acc[e + 1].w * inv));
      if (p.lse && part == 0)
        p.lse[size_t(g * p.G + hh) * p.Tq + b] = (Lsum > 0.f ? M + __log2f(Lsum) : -INFINITY) * 0.69314718055994531f;
    }
    cluster_sync_all();
  }
}

}  // namespace sdec

}  // namespace dtc
}  // namespace hs
