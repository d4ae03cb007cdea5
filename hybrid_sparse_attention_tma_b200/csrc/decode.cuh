// decode.cuh -- one new token per sequence: sparse-layer decode (split-K over
// the selected set plus the forced window, bf16 or FP8-e4m3 KV) and the full
// layer's decode with its exact token scores.
//
// Decode reads each selected K/V row once and is bound by HBM bandwidth; the
// KV head's G query heads (64 under MQA) share every K/V row, so the math is
// a small dense contraction done with warp-level bf16 MMAs (4 warps x 16
// heads): Q stays in registers, K/V rows are gathered with cp.async into
// XOR-swizzled shared memory, S and O accumulate in registers.
//
// Sparse decode (HySparse2 release note: sparse layers reuse the full layer's
// KV cache and top-k tokens, with the latest 128 forced in; its key-data table
// sizes an FP8 KV cache): V_q = {j in idx : j <= pos - w} U [pos-w+1, pos],
// split into 128-key chunks, one CTA per (sequence, KV head, chunk); the
// chunks' partial (m, l, O) are merged by log-sum-exp. FP8 rows decode as
// x = scale[token] * e4m3(code): e4m3 -> bf16 is exact, the K scale multiplies
// the logits and the V scale multiplies P before the PV product.
//
// Full-layer decode: causal attention of the new token over all its keys plus
// token scores score(j) = max_h exp(s_hj - lse_h). The scores need the final
// lse, so the layer runs in two exact passes: (1) lse per head from split-K
// (m, l) partials over K; (2) with lse known, P = exp(s - lse) is final: each
// CTA writes its keys' scores directly and sums P.V into an fp32 partial;
// a last kernel adds the partials.
#pragma once

#include "hs_common.cuh"

namespace hs {
namespace dec {

constexpr int kThreads = 128;  // 4 warps x 16 heads = 64 heads
constexpr int kHeads = 64;
constexpr int kChunk = 128;    // keys per sparse-decode CTA
constexpr int kFullChunk = 64; // keys per pipeline step of the full-layer decode

// ----------------------------------------------------------------------------
// warp MMA helpers (m16n8k16, bf16 in, fp32 accumulate)
// ----------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// two e4m3 codes (low byte first) -> bf16x2, exactly (e4m3 values are bf16 values)
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint16_t two) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(two));
  const __half2 hh = *reinterpret_cast<const __half2*>(&h2);
  const float2 f = __half22float2(hh);
  return pack_bf16(f.x, f.y);
}

// Row r of a [rows][128 bf16] tile: 16-byte chunk c lives at chunk c ^ (r & 7)
__device__ __forceinline__ uint32_t swz(int r, int c) { return uint32_t(r * 256 + ((c ^ (r & 7)) * 16)); }

// ----------------------------------------------------------------------------
// Shared pieces
// ----------------------------------------------------------------------------
struct SparseParams {
  const __nv_bfloat16* q;  // [batch, Hq, 128]
  const void* k;           // [T_kv, Hkv, 128] bf16 or e4m3
  const void* v;
  const float* k_scale;    // [T_kv, Hkv] (FP8)
  const float* v_scale;
  const int* idx;          // [batch, Hkv, topk]
  const int* cnt;          // [batch, Hkv]
  const int* cu_kv;        // device prefix sums of kv_b
  int topk, w, Hq, Hkv, G, n_chunks;
  float scale_log2;
  float* part_o;           // [batch*Hkv, n_chunks, 64, 128]
  float* part_ml;          // [batch*Hkv, n_chunks, 64, 2]  (m, l) in log2 units
};

// Load the KV head's 64 query rows (G valid, rest zero) into shared memory.
__device__ __forceinline__ void load_q_tile(uint8_t* sq, const __nv_bfloat16* q, int b, int g, int Hq, int G) {
  for (int i = threadIdx.x; i < kHeads * 16; i += kThreads) {  // 64 rows x 16 chunks of 16 B
    const int r = i >> 4, c = i & 15;
    const bool valid = r < G;
    const __nv_bfloat16* src = q + (size_t(b) * Hq + g * G + (valid ? r : 0)) * 128 + c * 8;
    cp_async16(smem_u32(sq) + swz(r, c), src, valid);
  }
}

// Q fragments (A operand) of this warp's 16 heads, all 8 k-steps.
__device__ __forceinline__ void q_fragments(const uint8_t* sq, uint32_t (&qa)[8][4]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = warp * 16 + (lane & 15);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks) {
    const int c = ks * 2 + (lane >> 4);
    ldsm_x4(smem_u32(sq) + swz(r, c), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
  }
}

// S[16 heads x NK keys] += Q . K^T for keys stored bf16 in a swizzled tile.
template <int NK>
__device__ __forceinline__ void qk_bf16(const uint32_t (&qa)[8][4], const uint8_t* sk, float (&s)[NK / 8][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int nt = 0; nt < NK / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
  for (int np = 0; np < NK / 16; ++np) {  // pairs of 8-key n-tiles
    const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int c = ks * 2 + ((lane >> 3) & 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(smem_u32(sk) + swz(key, c), b0, b1, b2, b3);
      mma16816(s[2 * np], qa[ks], b0, b1);
      mma16816(s[2 * np + 1], qa[ks], b2, b3);
    }
  }
}

// O[16 heads x 128] += P[16 x NK] . V[NK x 128], V bf16 swizzled.
template <int NK>
__device__ __forceinline__ void pv_bf16(const uint32_t (&pa)[NK / 16][4], const uint8_t* sv, float (&o)[16][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int ks = 0; ks < NK / 16; ++ks) {
    const int key = ks * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
    for (int dp = 0; dp < 8; ++dp) {  // pairs of 8-wide d tiles
      const int c = dp * 2 + (lane >> 4);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(sv) + swz(key, c), b0, b1, b2, b3);
      mma16816(o[2 * dp], pa[ks], b0, b1);
      mma16816(o[2 * dp + 1], pa[ks], b2, b3);
    }
  }
}

// ----------------------------------------------------------------------------
// A6: sparse decode, one CTA per (sequence, KV head, 128-key chunk)
// ----------------------------------------------------------------------------
// Q | K, V tiles (bf16, swizzled; FP8 codes are gathered into their upper
// halves and expanded in place) | scales, keys.
template <bool FP8>
constexpr int sparse_smem_bytes() {
  return kHeads * 256 + 2 * kChunk * 256 + 3 * kChunk * 4 + 1024;
}

template <bool FP8>
__global__ void __launch_bounds__(kThreads) sparse_decode_kernel(const SparseParams p) {
  constexpr int kRowBytes = FP8 ? 128 : 256;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = base;
  uint8_t* sk = sq + kHeads * 256;   // bf16 tiles the MMAs read
  uint8_t* sv = sk + kChunk * 256;
  // gather target: the bf16 tiles, or (FP8) the upper half of each tile
  uint8_t* gk = FP8 ? sk + kChunk * 128 : sk;
  uint8_t* gv = FP8 ? sv + kChunk * 128 : sv;
  float* sks = reinterpret_cast<float*>(sv + kChunk * 256);
  float* svs = sks + kChunk;
  int* skey = reinterpret_cast<int*>(svs + kChunk);

  const int chunk = blockIdx.x;
  const int bg = blockIdx.y;  // sequence * Hkv + g
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  static_assert(kChunk == kThreads, "one slot of the chunk per thread");
  __shared__ uint32_t s_valid[kChunk / 32];

  // Slot order of V_q: the window [pos-w+1, pos] first, then the selected
  // tokens <= pos - w. The index list is ascending, so its visible part is a
  // prefix and slot w + j holds idx[j] exactly when idx[j] <= pos - w: every
  // slot decides its own membership from one index, loaded together with the
  // sequence bounds, and no pass over the whole list precedes the gather.
  const int slot = chunk * kChunk + threadIdx.x;
  const int jsel = slot - p.w;  // position in the index list of a selected slot
  const int kv0 = __ldg(p.cu_kv + b);
  const int kv1 = __ldg(p.cu_kv + b + 1);
  const int cnt = p.cnt ? __ldg(p.cnt + bg) : 0;
  const int cand = (jsel >= 0 && jsel < p.topk) ? __ldg(p.idx + size_t(bg) * p.topk + jsel) : -1;
  const int pos = kv1 - kv0 - 1;  // the new token is the sequence's last position
  const int win_lo = max(0, pos - p.w + 1);
  const int n_win = p.w > 0 ? pos - win_lo + 1 : 0;
  int key = -1;
  if (slot < n_win) key = win_lo + slot;
  else if (jsel >= 0 && jsel < cnt && cand >= 0 && cand <= pos - p.w) key = cand;
  skey[threadIdx.x] = key;
  const uint32_t bal = __ballot_sync(0xffffffffu, key >= 0);
  if (lane == 0) s_valid[warp] = bal;
  __syncthreads();
  uint32_t vmask[kChunk / 32];
#pragma unroll
  for (int w = 0; w < kChunk / 32; ++w) vmask[w] = s_valid[w];
  float* pml = p.part_ml + (size_t(bg) * p.n_chunks + chunk) * kHeads * 2;
  if ((vmask[0] | vmask[1] | vmask[2] | vmask[3]) == 0) {
    if (threadIdx.x < kHeads) {
      pml[2 * threadIdx.x] = -INFINITY;
      pml[2 * threadIdx.x + 1] = 0.f;
    }
    return;
  }
  // gather: Q and K in one cp.async group, V in the next, so the QK product
  // starts while V is still in flight; empty slots are zero-filled, not read
  load_q_tile(sq, p.q, b, g, p.Hq, p.G);
  constexpr int kChunks16 = kRowBytes / 16;
  auto gather = [&](const void* src_base, uint8_t* dst) {
    for (int i = threadIdx.x; i < kChunk * kChunks16; i += kThreads) {
      const int r = i / kChunks16, c = i % kChunks16;
      const int kr = skey[r];
      const size_t row = (size_t(kv0) + (kr >= 0 ? kr : 0)) * p.Hkv + g;
      const uint8_t* src = reinterpret_cast<const uint8_t*>(src_base) + row * kRowBytes + c * 16;
      const uint32_t off = FP8 ? uint32_t(r * 128 + ((c ^ (r & 7)) << 4)) : swz(r, c);
      cp_async16(smem_u32(dst) + off, src, kr >= 0);
    }
    cp_async_commit();
  };
  gather(p.k, gk);
  gather(p.v, gv);
  if (FP8) {
    const size_t row = (size_t(kv0) + (key >= 0 ? key : 0)) * p.Hkv + g;
    sks[threadIdx.x] = key >= 0 ? __ldg(p.k_scale + row) : 0.f;
    svs[threadIdx.x] = key >= 0 ? __ldg(p.v_scale + row) : 0.f;
  }
  if constexpr (FP8) cp_async_wait<0>();
  else cp_async_wait<1>();
  __syncthreads();
  if constexpr (FP8) {
    // e4m3 -> bf16 is exact: expand both tiles in place into the swizzled
    // bf16 layout, then the same ldmatrix / mma path as bf16 KV serves FP8.
    // The codes of row r sit at byte 128 * (128 + r) of the tile; rows 0-63
    // expand into bytes [0, 16 KB), below every code; rows 64-127 overwrite
    // codes, so they are read into registers before anything is written.
    constexpr int kItems = kChunk * 8;                    // (row, 16-code chunk) per tile
    constexpr int kPer = kItems / kThreads;               // per thread and tile, per half
    auto expand = [&](uint4 u, uint8_t* dst, int r, int c) {
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
      uint32_t b[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        b[2 * j] = e4m3x2_to_bf16x2(uint16_t(w4[j] & 0xFFFFu));
        b[2 * j + 1] = e4m3x2_to_bf16x2(uint16_t(w4[j] >> 16));
      }
      *reinterpret_cast<uint4*>(dst + swz(r, 2 * c)) = make_uint4(b[0], b[1], b[2], b[3]);
      *reinterpret_cast<uint4*>(dst + swz(r, 2 * c + 1)) = make_uint4(b[4], b[5], b[6], b[7]);
    };
    static_assert(kItems % (2 * kThreads) == 0, "even split of the expansion");
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      uint4 u[2][kPer / 2];
#pragma unroll
      for (int tv = 0; tv < 2; ++tv)
#pragma unroll
        for (int j = 0; j < kPer / 2; ++j) {
          const int rc = half * (kItems / 2) + j * kThreads + threadIdx.x;
          const int r = rc >> 3, c = rc & 7;
          u[tv][j] = *reinterpret_cast<const uint4*>((tv ? gv : gk) + r * 128 + ((c ^ (r & 7)) << 4));
        }
      if (half == 1) __syncthreads();  // every code of rows 64-127 is in registers
#pragma unroll
      for (int tv = 0; tv < 2; ++tv)
#pragma unroll
        for (int j = 0; j < kPer / 2; ++j) {
          const int rc = half * (kItems / 2) + j * kThreads + threadIdx.x;
          expand(u[tv][j], tv ? sv : sk, rc >> 3, rc & 7);
        }
      __syncthreads();
    }
  }

  uint32_t qa[8][4];
  q_fragments(sq, qa);
  float s[kChunk / 8][4];
  qk_bf16<kChunk>(qa, sk, s);

  // softmax partial per head row (rows lane/4 and lane/4 + 8 of this warp)
  const float cs = p.scale_log2;
  float m[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int nt = 0; nt < kChunk / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int col = nt * 8 + 2 * (lane & 3) + (e & 1);
      float x = s[nt][e] * cs;
      if (FP8) x *= sks[col];
      if (!((vmask[nt >> 2] >> (col & 31)) & 1u)) x = -INFINITY;
      s[nt][e] = x;
      m[e >> 1] = fmaxf(m[e >> 1], x);
    }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    m[r] = fmaxf(m[r], __shfl_xor_sync(0xffffffffu, m[r], 1));
    m[r] = fmaxf(m[r], __shfl_xor_sync(0xffffffffu, m[r], 2));
  }
  float l[2] = {0.f, 0.f};
  uint32_t pa[kChunk / 16][4];
#pragma unroll
  for (int nt = 0; nt < kChunk / 8; ++nt) {
    float pe[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      pe[e] = ex2(s[nt][e] - m[e >> 1]);
      l[e >> 1] += pe[e];
      if (FP8) pe[e] *= svs[nt * 8 + 2 * (lane & 3) + (e & 1)];
    }
    const int ks = nt >> 1, hi8 = nt & 1;
    pa[ks][0 + 2 * hi8] = pack_bf16(pe[0], pe[1]);
    pa[ks][1 + 2 * hi8] = pack_bf16(pe[2], pe[3]);
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
    l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
  }
  float o[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
  if constexpr (!FP8) {
    cp_async_wait<0>();  // V
    __syncthreads();
  }
  pv_bf16<kChunk>(pa, sv, o);

  // partials: unnormalised O and (m, l) per head
  float* po = p.part_o + (size_t(bg) * p.n_chunks + chunk) * kHeads * 128;
  const int h0 = warp * 16 + (lane >> 2);
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    const int dcol = nt * 8 + 2 * (lane & 3);
    *reinterpret_cast<float2*>(po + size_t(h0) * 128 + dcol) = make_float2(o[nt][0], o[nt][1]);
    *reinterpret_cast<float2*>(po + size_t(h0 + 8) * 128 + dcol) = make_float2(o[nt][2], o[nt][3]);
  }
  if ((lane & 3) == 0) {
    pml[2 * h0] = m[0];
    pml[2 * h0 + 1] = l[0];
    pml[2 * (h0 + 8)] = m[1];
    pml[2 * (h0 + 8) + 1] = l[1];
  }
}

// Merge the chunk partials of one (sequence, KV head) by log-sum-exp. CTA
// (bg, quarter) covers 16 heads: one warp per head, each lane 4 of the 128
// dims. The lanes read the (m, l) of up to 32 chunks at once and the partial-O
// loads of 8 chunks are issued before any of them is used (empty chunks are
// not read), so the merge takes a few memory round trips however many chunks
// there are.
constexpr int kCombineHeads = 16;

struct CombineParams {
  const float* part_o;
  const float* part_ml;
  int n_chunks, Hq, Hkv, G, Tq;
  bool normalised;        // partial O already divided by the final l (full-layer pass 2)
  const float* lse2_in;   // [batch*Hkv, 64] log2 units (normalised case)
  __nv_bfloat16* o;       // [batch, Hq, 128]
  float* lse;             // [Hq, Tq] natural log
};

__global__ void __launch_bounds__(32 * kCombineHeads) combine_kernel(const CombineParams p) {
  const int bg = blockIdx.x;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y * kCombineHeads + (threadIdx.x >> 5);
  if (h >= p.G) return;  // whole warps
  const int n = p.n_chunks;
  const float* ml = p.part_ml + size_t(bg) * n * kHeads * 2;
  // this lane's float4 of chunk c: po[c * kHeads * 32]
  const float4* po = reinterpret_cast<const float4*>(p.part_o) + (size_t(bg) * n * kHeads + h) * 32 + lane;
  float M = -INFINITY;
  if (!p.normalised) {
    for (int c = lane; c < n; c += 32) M = fmaxf(M, ml[(size_t(c) * kHeads + h) * 2]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  }
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = 0.f;  // this lane's chunks
  auto add = [&](float wk, const float4& v) {
    // a chunk without keys has weight 0 and an unwritten partial: skip it
    if (wk != 0.f) {
      acc.x = fmaf(wk, v.x, acc.x);
      acc.y = fmaf(wk, v.y, acc.y);
      acc.z = fmaf(wk, v.z, acc.z);
      acc.w = fmaf(wk, v.w, acc.w);
    }
  };
  for (int c0 = 0; c0 < n; c0 += 32) {
    float wl = 1.f;  // weight of chunk c0 + lane
    if (!p.normalised) {
      wl = 0.f;
      const int c = c0 + lane;
      if (c < n) {
        const float mc = ml[(size_t(c) * kHeads + h) * 2];
        if (mc != -INFINITY) {
          wl = ex2(mc - M);
          L += wl * ml[(size_t(c) * kHeads + h) * 2 + 1];
        }
      }
    }
    const int nc = min(32, n - c0);
    int k = 0;
    const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
    for (; k + 8 <= nc; k += 8) {
      float wk[8];
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        wk[u] = __shfl_sync(0xffffffffu, wl, k + u);
        v[u] = wk[u] != 0.f ? po[size_t(c0 + k + u) * kHeads * 32] : zero;  // empty chunks are not read
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) add(wk[u], v[u]);
    }
    for (; k < nc; ++k) {
      const float wk = __shfl_sync(0xffffffffu, wl, k);
      if (wk != 0.f) add(wk, po[size_t(c0 + k) * kHeads * 32]);
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  const float inv = p.normalised ? 1.f : (L > 0.f ? 1.f / L : 0.f);
  const int hq = g * p.G + h;
  *reinterpret_cast<uint2*>(p.o + (size_t(b) * p.Hq + hq) * 128 + lane * 4) =
      make_uint2(pack_bf16(acc.x * inv, acc.y * inv), pack_bf16(acc.z * inv, acc.w * inv));
  if (lane == 0 && p.lse) {
    float lse2;
    if (p.normalised) lse2 = p.lse2_in[size_t(bg) * kHeads + h];
    else lse2 = L > 0.f ? M + __log2f(L) : -INFINITY;
    p.lse[size_t(hq) * p.Tq + b] = lse2 * 0.69314718055994531f;
  }
}

// ----------------------------------------------------------------------------
// A7: full-layer decode -- pass 1 (per-head lse) and pass 2 (P.V + scores)
// ----------------------------------------------------------------------------
struct FullParams {
  const __nv_bfloat16* q;  // [batch, Hq, 128]
  const __nv_bfloat16* k;  // [T_kv, Hkv, 128]
  const __nv_bfloat16* v;
  const int* cu_kv;
  int Hq, Hkv, G, n_split, max_kv;
  float scale_log2;
  float* part_ml;   // pass 1: [batch*Hkv, n_split, 64, 2]
  float* lse2;      // [batch*Hkv, 64] (written by the lse combine, read by pass 2)
  float* part_o;    // pass 2: [batch*Hkv, n_split, 64, 128], already normalised
  float* scores;    // [batch, Hkv, nblk = max_kv]
  int nblk;
};

// keys of split s of a sequence with kv_len keys: [s*len, min((s+1)*len, kv_len))
__device__ __forceinline__ void split_range(int kv_len, int n_split, int s, int& k0, int& k1) {
  const int per = ((kv_len + n_split - 1) / n_split + kFullChunk - 1) / kFullChunk * kFullChunk;
  k0 = min(kv_len, s * per);
  k1 = min(kv_len, k0 + per);
}

template <bool PASS2>
constexpr int full_smem_bytes() {
  return kHeads * 256 + (PASS2 ? 4 : 2) * kFullChunk * 256 + 1024;
}

template <bool PASS2>
__global__ void __launch_bounds__(kThreads) full_decode_kernel(const FullParams p) {
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sq = base;
  uint8_t* sk[2] = {sq + kHeads * 256, sq + kHeads * 256 + kFullChunk * 256};
  uint8_t* sv[2] = {sk[1] + kFullChunk * 256, sk[1] + 2 * kFullChunk * 256};
  __shared__ float red[4][kFullChunk];
  __shared__ float slse[kHeads];

  const int s = blockIdx.x;
  const int bg = blockIdx.y;
  const int b = bg / p.Hkv, g = bg % p.Hkv;
  const int kv0 = __ldg(p.cu_kv + b);
  const int kv_len = __ldg(p.cu_kv + b + 1) - kv0;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int k0, k1;
  split_range(kv_len, p.n_split, s, k0, k1);
  const int n_steps = (k1 - k0 + kFullChunk - 1) / kFullChunk;

  if (PASS2 && threadIdx.x < kHeads) slse[threadIdx.x] = p.lse2[size_t(bg) * kHeads + threadIdx.x];
  load_q_tile(sq, p.q, b, g, p.Hq, p.G);
  cp_async_commit();
  auto issue = [&](int step, int buf) {
    const int kb = k0 + step * kFullChunk;
    for (int i = threadIdx.x; i < kFullChunk * 16; i += kThreads) {
      const int r = i >> 4, c = i & 15;
      const int key = min(kb + r, kv_len - 1);
      const size_t row = (size_t(kv0) + key) * p.Hkv + g;
      cp_async16(smem_u32(sk[buf]) + swz(r, c), p.k + row * 128 + c * 8, true);
      if (PASS2) cp_async16(smem_u32(sv[buf]) + swz(r, c), p.v + row * 128 + c * 8, true);
    }
    cp_async_commit();
  };
  if (n_steps > 0) issue(0, 0);
  cp_async_wait<0>();
  __syncthreads();
  uint32_t qa[8][4];
  q_fragments(sq, qa);
  const float cs = p.scale_log2;
  const int h0 = warp * 16 + (lane >> 2);
  float lse_r[2] = {0.f, 0.f};
  if (PASS2) {
    lse_r[0] = slse[h0];
    lse_r[1] = slse[h0 + 8];
  }
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  float o[PASS2 ? 16 : 1][4];
#pragma unroll
  for (int nt = 0; nt < (PASS2 ? 16 : 1); ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
  const bool row_valid[2] = {h0 < p.G, h0 + 8 < p.G};

  for (int st = 0; st < n_steps; ++st) {
    const int buf = st & 1;
    if (st + 1 < n_steps) issue(st + 1, buf ^ 1);
    if (st + 1 < n_steps) cp_async_wait<1>(); else cp_async_wait<0>();
    __syncthreads();
    const int kb = k0 + st * kFullChunk;
    const int nk = min(kFullChunk, k1 - kb);
    float sacc[kFullChunk / 8][4];
    qk_bf16<kFullChunk>(qa, sk[buf], sacc);
    if constexpr (!PASS2) {
      // running (m, l) per head row
      float mt[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < kFullChunk / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = nt * 8 + 2 * (lane & 3) + (e & 1);
          const float x = col < nk ? sacc[nt][e] * cs : -INFINITY;
          sacc[nt][e] = x;
          mt[e >> 1] = fmaxf(mt[e >> 1], x);
        }
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mt[r] = fmaxf(mt[r], __shfl_xor_sync(0xffffffffu, mt[r], 1));
        mt[r] = fmaxf(mt[r], __shfl_xor_sync(0xffffffffu, mt[r], 2));
        const float mn = fmaxf(m[r], mt[r]);
        l[r] *= (m[r] == -INFINITY) ? 0.f : ex2(m[r] - mn);
        m[r] = mn;
      }
#pragma unroll
      for (int nt = 0; nt < kFullChunk / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) l[e >> 1] += ex2(sacc[nt][e] - m[e >> 1]);
    } else {
      // exact probabilities: P = exp2(s*c - lse2); token score = max over heads
      uint32_t pa[kFullChunk / 16][4];
      float colmax[kFullChunk / 8][2];
#pragma unroll
      for (int nt = 0; nt < kFullChunk / 8; ++nt) {
        float pe[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = nt * 8 + 2 * (lane & 3) + (e & 1);
          const bool ok = col < nk && row_valid[e >> 1];
          pe[e] = ok ? ex2(fmaf(sacc[nt][e], cs, -lse_r[e >> 1])) : 0.f;
        }
        colmax[nt][0] = fmaxf(pe[0], pe[2]);
        colmax[nt][1] = fmaxf(pe[1], pe[3]);
        const int ks = nt >> 1, hi8 = nt & 1;
        pa[ks][0 + 2 * hi8] = pack_bf16(pe[0], pe[1]);
        pa[ks][1 + 2 * hi8] = pack_bf16(pe[2], pe[3]);
      }
      // max over the warp's 16 heads: lanes sharing lane & 3 hold the same columns
#pragma unroll
      for (int nt = 0; nt < kFullChunk / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float v = colmax[nt][e];
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
          if (lane < 4) red[warp][nt * 8 + 2 * lane + e] = v;
        }
      pv_bf16<kFullChunk>(pa, sv[buf], o);
      __syncthreads();
      if (threadIdx.x < kFullChunk && threadIdx.x < nk) {
        const float sc = fmaxf(fmaxf(red[0][threadIdx.x], red[1][threadIdx.x]),
                               fmaxf(red[2][threadIdx.x], red[3][threadIdx.x]));
        p.scores[size_t(bg) * p.nblk + kb + threadIdx.x] = sc;
      }
    }
    __syncthreads();  // buffer `buf` is refilled by the next iteration's issue
  }
  if constexpr (!PASS2) {
    // each of the 4 lanes sharing a head row summed a quarter of the columns
    // (with the same, quad-uniform running max): add them up
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      l[r] += __shfl_xor_sync(0xffffffffu, l[r], 1);
      l[r] += __shfl_xor_sync(0xffffffffu, l[r], 2);
    }
    if ((lane & 3) == 0) {
      float* pml = p.part_ml + (size_t(bg) * p.n_split + s) * kHeads * 2;
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        pml[2 * (h0 + 8 * r)] = m[r];
        pml[2 * (h0 + 8 * r) + 1] = l[r];
      }
    }
  } else {
    float* po = p.part_o + (size_t(bg) * p.n_split + s) * kHeads * 128;
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      const int dcol = nt * 8 + 2 * (lane & 3);
      *reinterpret_cast<float2*>(po + size_t(h0) * 128 + dcol) = make_float2(o[nt][0], o[nt][1]);
      *reinterpret_cast<float2*>(po + size_t(h0 + 8) * 128 + dcol) = make_float2(o[nt][2], o[nt][3]);
    }
  }
}

// lse2 per (sequence, KV head, head) from the pass-1 partials: CTA (bg,
// quarter), one warp per head, the lanes strided over the splits.
__global__ void __launch_bounds__(32 * kCombineHeads) lse_combine_kernel(const float* part_ml, int n_split,
                                                                         float* lse2) {
  const int bg = blockIdx.x, lane = threadIdx.x & 31;
  const int h = blockIdx.y * kCombineHeads + (threadIdx.x >> 5);
  const float* ml = part_ml + size_t(bg) * n_split * kHeads * 2;
  float M = -INFINITY;
  for (int s = lane; s < n_split; s += 32) M = fmaxf(M, ml[(size_t(s) * kHeads + h) * 2]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
  float L = 0.f;
  for (int s = lane; s < n_split; s += 32) {
    const float m = ml[(size_t(s) * kHeads + h) * 2];
    if (m > -INFINITY) L += ex2(m - M) * ml[(size_t(s) * kHeads + h) * 2 + 1];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
  if (lane == 0) lse2[size_t(bg) * kHeads + h] = L > 0.f ? M + __log2f(L) : -INFINITY;
}

}  // namespace dec
}  // namespace hs
