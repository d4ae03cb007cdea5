// swa_decode.cuh -- the HySparse sliding-window branch at decode time.
//
// The SWA branch keeps its own small K/V cache (QbitAI repost, two-branch
// paragraph; techwalker.com explainer: the window branch must not share the
// full layer's KV), and only the last `window` (128) positions of it are ever
// read. Here that cache is a ring of R >= window slots per sequence: position
// p of sequence b lives at slot p mod R of ring[b][R][H_kv][d]. The new token
// (position pos = kv_b - 1) attends over positions [max(0, pos - window + 1),
// pos] and the branch output is mixed with the sparse branch by the sigmoid
// gate o = sig(gamma) o_sparse + (1 - sig(gamma)) o_swa (both pages' gate).
//
// The work per (sequence, KV head) is G x window x d multiply-adds over 64 KB
// of K/V: small and bound by reading the window, so it runs on the CUDA cores.
#pragma once

#include "hs_common.cuh"

namespace hs {
namespace swad {

constexpr int kMaxWindow = 128;
constexpr int kMaxG = 64;
constexpr int kThreads = 128;

// Sequence of a packed new-token row (binary search of the device prefix sums).
__device__ __forceinline__ int seq_of_row(const int* __restrict__ cu_q, int batch, long long row) {
  int lo = 0, hi = batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(cu_q + mid) <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ring[b][p mod R] = x[row of the new token at position p], for the new tokens
// of each sequence that are among its last R positions (an earlier new token
// of the same call would be overwritten by a later one in the same slot).
// Thread = one 16-byte piece of a [H_kv][d] row.
__global__ void __launch_bounds__(256) ring_write_kernel(const int* __restrict__ cu_q, const int* __restrict__ cu_kv,
                                                         int batch, long long rows, int row_pieces, int R,
                                                         const uint4* __restrict__ k_new,
                                                         const uint4* __restrict__ v_new, uint4* __restrict__ k_ring,
                                                         uint4* __restrict__ v_ring) {
  const long long n = rows * row_pieces;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long row = e / row_pieces;
    const int pc = int(e - row * row_pieces);
    const int b = seq_of_row(cu_q, batch, row);
    const int q0 = __ldg(cu_q + b), n_b = __ldg(cu_q + b + 1) - q0;
    const int i = int(row - q0);
    if (i < n_b - R) continue;
    const int pos = (__ldg(cu_kv + b + 1) - __ldg(cu_kv + b)) - n_b + i;
    const size_t dst = (size_t(b) * R + pos % R) * row_pieces + pc;
    k_ring[dst] = __ldg(k_new + e);
    v_ring[dst] = __ldg(v_new + e);
  }
}

// Shared memory of one CTA (G heads, W <= kMaxWindow keys, d = D), in 32-bit
// words: Q [G][D] fp32 | K [W][D/2 + 1] bf16 pairs (odd row stride: the score
// loop's threads read different rows at the same column without bank
// conflicts), padded to 16 bytes | V [W][D/2] bf16 pairs | P [G][W] fp32.
__host__ __device__ constexpr int k_words(int D, int W) { return (W * (D / 2 + 1) + 3) & ~3; }
template <int D>
__host__ __device__ constexpr int smem_words(int G, int W) {
  return G * D + k_words(D, W) + W * (D / 2) + G * W;
}

// One CTA per (sequence b, KV head g); one query per sequence (q row cu_q[b]).
template <int D>
__global__ void __launch_bounds__(kThreads) swa_gated_decode_kernel(
    const int* __restrict__ cu_q, const int* __restrict__ cu_kv, int Hq, int Hkv, int G, int window, int R,
    float scale_log2, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_ring,
    const __nv_bfloat16* __restrict__ v_ring, const float* __restrict__ gamma,
    const __nv_bfloat16* __restrict__ o_sparse, __nv_bfloat16* __restrict__ o) {
  extern __shared__ uint32_t sm[];
  constexpr int KW = D / 2 + 1, VW = D / 2;
  const int b = blockIdx.x / Hkv, g = blockIdx.x % Hkv;
  const int t = threadIdx.x;
  const int qrow = __ldg(cu_q + b);
  const int pos = __ldg(cu_kv + b + 1) - __ldg(cu_kv + b) - 1;
  const int lo = max(0, pos - window + 1);
  const int nk = pos - lo + 1;  // 1 .. window
  float* qs = reinterpret_cast<float*>(sm);
  uint32_t* ks = sm + G * D;
  uint32_t* vs = ks + k_words(D, nk);
  float* ps = reinterpret_cast<float*>(vs + nk * VW);
  // stage the window's K / V rows (16-byte pieces, 16 threads per 256-byte row,
  // four loads in flight per thread before any store) and the G query rows
  constexpr int PP = D / 8;  // pieces per row
  const uint4* kr = reinterpret_cast<const uint4*>(k_ring);
  const uint4* vr = reinterpret_cast<const uint4*>(v_ring);
  for (int e0 = t; e0 < nk * PP; e0 += 4 * kThreads) {
    uint4 kv[4], vv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e0 + u * kThreads;
      if (e < nk * PP) {
        const int j = e / PP, pc = e - j * PP;
        const size_t src = ((size_t(b) * R + (lo + j) % R) * Hkv + g) * PP + pc;
        kv[u] = __ldg(kr + src);
        vv[u] = __ldg(vr + src);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int e = e0 + u * kThreads;
      if (e < nk * PP) {
        const int j = e / PP, pc = e - j * PP;
        uint32_t* kd = ks + j * KW + pc * 4;  // odd row stride: four word stores
        kd[0] = kv[u].x;
        kd[1] = kv[u].y;
        kd[2] = kv[u].z;
        kd[3] = kv[u].w;
        reinterpret_cast<uint4*>(vs + j * VW)[pc] = vv[u];
      }
    }
  }
  for (int e = t; e < G * D; e += kThreads) {
    const int hh = e / D, dd = e - hh * D;
    qs[e] = __bfloat162float(q[(size_t(qrow) * Hq + g * G + hh) * D + dd]);
  }
  __syncthreads();
  // logits, log2 units: thread = (head, key) pairs, keys fastest
  for (int e = t; e < G * nk; e += kThreads) {
    const int hh = e / nk, j = e - hh * nk;
    const float* qh = qs + hh * D;
    const uint32_t* kj = ks + j * KW;
    float acc = 0.f;
#pragma unroll 8
    for (int w = 0; w < VW; ++w) {
      const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kj + w));
      acc = fmaf(qh[2 * w], kf.x, fmaf(qh[2 * w + 1], kf.y, acc));
    }
    ps[hh * nk + j] = acc * scale_log2;
  }
  __syncthreads();
  // softmax of each head's row: warp per head, lane = keys lane, lane + 32, ...
  const int warp = t >> 5, lane = t & 31;
  for (int hh = warp; hh < G; hh += kThreads / 32) {
    float* ph = ps + hh * nk;
    float m = -INFINITY;
    for (int j = lane; j < nk; j += 32) m = fmaxf(m, ph[j]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float sum = 0.f;
    for (int j = lane; j < nk; j += 32) {
      const float e = exp2f(ph[j] - m);
      ph[j] = e;
      sum += e;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    const float inv = 1.f / sum;  // nk >= 1: the new token sees itself
    for (int j = lane; j < nk; j += 32) ph[j] *= inv;
  }
  __syncthreads();
  // o_swa[h][d] = sum_j p[h][j] v[j][d] (thread = column d), then the gate
  if (t < D) {
    const __nv_bfloat16* vb = reinterpret_cast<const __nv_bfloat16*>(vs);
    for (int hh = 0; hh < G; ++hh) {
      const float* ph = ps + hh * nk;
      float acc = 0.f;
      for (int j = 0; j < nk; ++j) acc = fmaf(ph[j], __bfloat162float(vb[j * D + t]), acc);
      const int h = g * G + hh;
      const size_t oi = (size_t(qrow) * Hq + h) * D + t;
      const float sg = 1.f / (1.f + __expf(-__ldg(gamma + size_t(qrow) * Hq + h)));
      o[oi] = __float2bfloat16_rn(sg * __bfloat162float(o_sparse[oi]) + (1.f - sg) * acc);
    }
  }
}

}  // namespace swad
}  // namespace hs
