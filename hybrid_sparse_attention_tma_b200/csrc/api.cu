// api.cu -- the libhs C ABI: argument validation, workspace sizing, tensor
// maps, schedules and kernel launches. No call allocates device memory.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <numeric>
#include <vector>

#include "../../include/hs.h"
#include "attn_fwd.cuh"
#include "hs_common.cuh"
#include "seqtable.cuh"
#include "decode_tc.cuh"
#include "swa_decode.cuh"
#include "token_scores.cuh"
#include "topk.cuh"

using namespace hs;

namespace {

constexpr size_t kHeaderBytes = 256;
constexpr unsigned long long kDefaultTimeoutNs = 4000000000ull;  // 4 s
unsigned long long g_timeout_ns = kDefaultTimeoutNs;

inline cudaStream_t S(hs_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 3-D bf16 tensor [outer][mid][d] viewed as dims {d, mid, outer}; box {64, box_mid, box_outer};
// 128-byte swizzle; out-of-range rows read as zero.
bool make_map_3d(CUtensorMap* m, const void* base, int d, int mid, long long outer, int box_mid, int box_outer) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(mid), cuuint64_t(outer)};
  cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(d) * 2 * cuuint64_t(mid)};
  cuuint32_t box[3] = {64, cuuint32_t(box_mid), cuuint32_t(box_outer)};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D row view of a [T][H][d] bf16 tensor (row = t * H + h) for tile::gather4
// loads: box {64 columns, 1 row}, 128-byte swizzle.
bool make_map_rows(CUtensorMap* m, const void* base, int d, long long rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cuuint64_t(d), cuuint64_t(rows)};
  cuuint64_t strides[1] = {cuuint64_t(d) * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------- validation ----------------
struct Shape {
  int batch, Hq, Hkv, G, d;
  long long Tq, Tkv;
  int max_q, max_kv;
  float scale;
};

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

hs_status check_varlen(const hs_varlen* vl, Shape* sh, bool need_device_cu = true) {
  if (!vl) return HS_ERR_INVALID_ARG;
  if (vl->batch < 1 || vl->n_q_heads < 1 || vl->n_kv_heads < 1) return HS_ERR_INVALID_ARG;
  if (vl->n_q_heads % vl->n_kv_heads) return HS_ERR_INVALID_ARG;
  if (!vl->cu_q_host || !vl->cu_kv_host) return HS_ERR_INVALID_ARG;
  if (need_device_cu && (!vl->cu_q || !vl->cu_kv)) return HS_ERR_INVALID_ARG;
  if (vl->cu_q_host[0] != 0 || vl->cu_kv_host[0] != 0) return HS_ERR_INVALID_ARG;
  sh->batch = vl->batch;
  sh->Hq = vl->n_q_heads;
  sh->Hkv = vl->n_kv_heads;
  sh->G = sh->Hq / sh->Hkv;
  sh->d = vl->head_dim;
  sh->max_q = 0;
  sh->max_kv = 0;
  for (int b = 0; b < vl->batch; ++b) {
    const int nq = vl->cu_q_host[b + 1] - vl->cu_q_host[b];
    const int nkv = vl->cu_kv_host[b + 1] - vl->cu_kv_host[b];
    if (nq < 0 || nkv < nq) return HS_ERR_INVALID_ARG;
    sh->max_q = std::max(sh->max_q, nq);
    sh->max_kv = std::max(sh->max_kv, nkv);
  }
  sh->Tq = vl->cu_q_host[vl->batch];
  sh->Tkv = vl->cu_kv_host[vl->batch];
  if (sh->Tkv > (1LL << 31) - 1 || sh->Tq > (1LL << 31) - 1) return HS_ERR_UNSUPPORTED;
  if (!(vl->softmax_scale >= 0.f) || std::isinf(vl->softmax_scale)) return HS_ERR_INVALID_ARG;
  sh->scale = vl->softmax_scale > 0.f ? vl->softmax_scale : 1.f / std::sqrt(float(sh->d));
  if (sh->d != 64 && sh->d != 128) return HS_ERR_UNSUPPORTED;
  return HS_OK;
}

hs_status check_sel(const hs_sel* sel) {
  if (!sel) return HS_ERR_INVALID_ARG;
  if (sel->q_tile < 1 || sel->block < 1 || sel->topk < 0 || sel->window < 0) return HS_ERR_INVALID_ARG;
  if (sel->topk > 4096) return HS_ERR_UNSUPPORTED;
  if (!is_pow2(sel->block) || sel->block > 128 || (sel->block > 1 && sel->block < 8)) return HS_ERR_UNSUPPORTED;
  if (sel->flags & ~HS_SEL_WINDOW_EXCLUSIVE) return HS_ERR_INVALID_ARG;
  return HS_OK;
}

int n_tiles_of(const hs_varlen* vl, int T) {
  long long n = 0;
  for (int b = 0; b < vl->batch; ++b) n += (vl->cu_q_host[b + 1] - vl->cu_q_host[b] + T - 1) / T;
  return int(n);
}

bool fill_seqtable(const hs_varlen* vl, int T, SeqTable* st) {
  if (vl->batch > kMaxSeq) return false;
  st->batch = vl->batch;
  st->T = T;
  st->tile_base[0] = 0;
  for (int b = 0; b <= vl->batch; ++b) {
    st->cu_q[b] = vl->cu_q_host[b];
    st->cu_kv[b] = vl->cu_kv_host[b];
  }
  for (int b = 0; b < vl->batch; ++b)
    st->tile_base[b + 1] = st->tile_base[b] + (vl->cu_q_host[b + 1] - vl->cu_q_host[b] + T - 1) / T;
  st->n_tiles = st->tile_base[vl->batch];
  return true;
}

// Selection tiles of a batch: sum over sequences of ceil(n_b / T).
long long n_sel_tiles(const hs_varlen* vl, int T) {
  long long n = 0;
  for (int b = 0; b < vl->batch; ++b) n += (vl->cu_q_host[b + 1] - vl->cu_q_host[b] + T - 1) / T;
  return n;
}

// Schedule of the tcgen05 attention kernel (see attn::Sched).
bool fill_sched(const hs_varlen* vl, const Shape& sh, int mode, int T, int chunks_per_tile, attn::Sched* sc) {
  if (vl->batch > attn::kMaxSched) return false;
  const int B = vl->batch;
  std::vector<int> order(B);
  std::iota(order.begin(), order.end(), 0);
  if (mode == attn::kFull) {
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
      return (vl->cu_kv_host[a + 1] - vl->cu_kv_host[a]) > (vl->cu_kv_host[b + 1] - vl->cu_kv_host[b]);
    });
  }
  const int qpc = attn::kMaxItemRows / sh.G;
  sc->n_seq = B;
  sc->first_item[0] = 0;
  int tb = 0;
  for (int b = 0; b < B; ++b) {
    sc->cu_q[b] = vl->cu_q_host[b];
    sc->cu_kv[b] = vl->cu_kv_host[b];
    sc->tile_base[b] = tb;
    tb += (vl->cu_q_host[b + 1] - vl->cu_q_host[b] + T - 1) / T;
  }
  sc->cu_q[B] = vl->cu_q_host[B];
  sc->cu_kv[B] = vl->cu_kv_host[B];
  long long acc = 0;
  for (int e = 0; e < B; ++e) {
    const int b = order[e];
    sc->seq[e] = b;
    const int n_b = vl->cu_q_host[b + 1] - vl->cu_q_host[b];
    long long items;
    if (mode == attn::kFull)
      items = (long long)((n_b + qpc - 1) / qpc) * sh.Hkv;
    else
      items = (long long)((n_b + T - 1) / T) * chunks_per_tile * sh.Hkv;
    acc += items;
    if (acc > (1LL << 30)) return false;
    sc->first_item[e + 1] = int(acc);
  }
  sc->n_items = int(acc);
  return true;
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

// A kernel's dynamic shared-memory limit is a per-device attribute: each call
// site keeps one of these and raises the limit once on every device it
// launches on (devices beyond the mask get the call on every launch).
struct PerDeviceOnce {
  std::mutex mu;
  uint64_t done[2] = {0, 0};  // devices 0..127
};

template <typename K>
cudaError_t set_smem_once(PerDeviceOnce& once, K kernel, int bytes) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 128) return set_smem(kernel, bytes);
  std::lock_guard<std::mutex> lock(once.mu);
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (once.done[dev >> 6] & bit) return cudaSuccess;
  const cudaError_t e = set_smem(kernel, bytes);
  if (e == cudaSuccess) once.done[dev >> 6] |= bit;
  return e;
}

// Tensor maps of one attention launch. g / o (the other branch's output and
// this call's output, boxes of 64 rows = 64/G queries x G heads) are used by
// the gated sliding-window call only; the other calls pass copies of q.
struct Maps {
  CUtensorMap q, k, v, kb, vb, g, o, ks, vs;  // ks / vs: the fused sparse layer's own window cache
};

// Launch the tcgen05 attention kernel.
template <int D, int MODE, int SB>
hs_status launch_attn(const Maps& m, const attn::Params& p, const attn::Sched& sc, int grid, cudaStream_t st) {
  auto kern = attn::attn_fwd_kernel<D, MODE, SB>;
  constexpr int need = attn::smem_bytes<D, (MODE == attn::kSparse && SB == 0) || MODE == attn::kFused>();
  constexpr int smem = need > 116 * 1024 ? need : 116 * 1024;
  static PerDeviceOnce once;
  if (set_smem_once(once, kern, smem) != cudaSuccess) return HS_ERR_CUDA;
  kern<<<grid, attn::threads_for<MODE, SB>(), smem, st>>>(m.q, m.k, m.v, m.kb, m.vb, m.g, m.o, m.ks, m.vs, p, sc);
  return cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}

template <int MODE, int SB>
hs_status dispatch_attn_d(int d, const Maps& m, const attn::Params& p, const attn::Sched& sc, int grid,
                          cudaStream_t st) {
  if (d == 64) return launch_attn<64, MODE, SB>(m, p, sc, grid, st);
  return launch_attn<128, MODE, SB>(m, p, sc, grid, st);
}

hs_status dispatch_full(int d, int B, const Maps& m, const attn::Params& p, const attn::Sched& sc, int grid,
                        cudaStream_t st) {
  switch (B) {
    case 8: return dispatch_attn_d<attn::kFull, 8>(d, m, p, sc, grid, st);
    case 16: return dispatch_attn_d<attn::kFull, 16>(d, m, p, sc, grid, st);
    case 32: return dispatch_attn_d<attn::kFull, 32>(d, m, p, sc, grid, st);
    case 64: return dispatch_attn_d<attn::kFull, 64>(d, m, p, sc, grid, st);
    case 128: return dispatch_attn_d<attn::kFull, 128>(d, m, p, sc, grid, st);
    default: return dispatch_attn_d<attn::kFull, 0>(d, m, p, sc, grid, st);
  }
}

WaitCtl wait_ctl(void* ws) { return WaitCtl{reinterpret_cast<ErrWord*>(ws), g_timeout_ns}; }

size_t full_decode_ws_bytes(const hs_varlen* vl, const Shape& sh);
bool is_decode(const hs_varlen* vl, const hs_sel* sel);

// Block-maximum spill of one CTA (double-buffered): per 128-key tile of the
// longest sequence, 256 rows x (128 / B) blocks.
size_t spill_floats_per_cta(int max_kv, int B) {
  return 2 * size_t((max_kv + 127) / 128) * size_t(128 / B) * attn::kMaxItemRows;
}

// Workspace of the token-level score pass after the header: the item prefix
// (n_tiles + 1 ints), then for the fused top-k the item order (n_tiles ints),
// the per-plane arrival counters, the queue of completed planes (one int per
// plane each) and the queue's two counters.
size_t token_prefix_bytes(int n_tiles) { return align_up(sizeof(int) * (size_t(n_tiles) + 1), 256); }
size_t token_arrive_bytes(int n_tiles, int Hkv) {
  return align_up(sizeof(int) * (size_t(n_tiles) + 2 * size_t(n_tiles) * Hkv + 2), 256);
}

size_t full_ws_bytes(const hs_varlen* vl, const Shape& sh, const hs_sel* sel) {
  if (is_decode(vl, sel) && sh.d == 128 && sh.G <= 64) return full_decode_ws_bytes(vl, sh);
  size_t b = kHeaderBytes;
  if (sel->block > 1) {
    b += size_t(num_sms()) * spill_floats_per_cta(sh.max_kv, sel->block) * sizeof(float);
  } else {
    const int nt = n_tiles_of(vl, sel->q_tile);
    b += token_prefix_bytes(nt) + token_arrive_bytes(nt, sh.Hkv);  // token-score items, fused top-k counters
  }
  return align_up(b, 256);
}

// Decode: one new query per sequence, selection tile 1, token level.
bool is_decode(const hs_varlen* vl, const hs_sel* sel) {
  if (sel->q_tile != 1 || sel->block != 1) return false;
  for (int b = 0; b < vl->batch; ++b)
    if (vl->cu_q_host[b + 1] - vl->cu_q_host[b] != 1) return false;
  return true;
}

// One query per sequence and single-query tiles, any selection block (the
// sparse decode; the token-level full-layer decode kernel needs block 1).
bool is_decode_batch(const hs_varlen* vl, const hs_sel* sel) {
  if (sel->q_tile != 1) return false;
  for (int b = 0; b < vl->batch; ++b)
    if (vl->cu_q_host[b + 1] - vl->cu_q_host[b] != 1) return false;
  return true;
}

// Full-layer decode on the tensor cores (decode_tc.cuh): keys per work item.
// Pass 2 re-reads a unit's K about D = (one unit's chunks + two grids of
// items) pass-1 items after pass 1 read it. Each item costs a few
// microseconds of hand-offs besides its tiles, so items are long (up to 32
// tiles of 128 keys, as long as every CTA gets two items per pass); an L2
// budget (HS_DEC_L2_BUDGET_MB, off by default) can shorten them so that K
// stays in L2 between the passes. Measured at 64 x 131072 keys: 1.28 ms with
// 32-tile items against 1.62 / 2.04 ms with 8 / 4 tiles.
#ifndef HS_DEC_MAX_TILES
#define HS_DEC_MAX_TILES 32
#endif
#ifndef HS_DEC_L2_BUDGET_MB
#define HS_DEC_L2_BUDGET_MB (1LL << 40)
#endif
#ifndef HS_DEC_DELAY_GRIDS
#define HS_DEC_DELAY_GRIDS 2
#endif
int full_decode_chunk_keys(const hs_varlen* vl, const Shape& sh) {
  long long tiles = 0, unit_tiles = 0;
  for (int b = 0; b < vl->batch; ++b) {
    const long long t = (vl->cu_kv_host[b + 1] - vl->cu_kv_host[b] + 127) / 128;
    tiles += t;
    unit_tiles = std::max(unit_tiles, t);
  }
  tiles *= sh.Hkv;
  const long long grid = num_sms();
  long long T = HS_DEC_MAX_TILES;
  while (T > 1 && (2 * T * grid + unit_tiles) * 32768LL > (HS_DEC_L2_BUDGET_MB << 20)) --T;
  while (T > 1 && tiles / T < 2 * grid) --T;
  return int(T) * 128;
}

// Workspace: header | sync words (work counter + 3 per unit) | O accumulators
// [units][64][128] fp32 | pass-1 fp64 totals [units][64] (these three are
// zeroed together before each launch) | lse2 [units][64].
struct FullDecodeWs {
  size_t sync, o_acc, unit_l, lse2, total;
};

FullDecodeWs full_decode_layout(const hs_varlen* vl, const Shape& sh) {
  (void)vl;
  const size_t U = size_t(sh.batch) * sh.Hkv;
  FullDecodeWs w;
  w.sync = kHeaderBytes;
  w.o_acc = align_up(w.sync + (1 + 3 * U) * sizeof(int), 256);
  w.unit_l = align_up(w.o_acc + U * 64 * 128 * sizeof(float), 256);
  w.lse2 = align_up(w.unit_l + U * 64 * sizeof(double), 256);
  w.total = align_up(w.lse2 + U * 64 * sizeof(float), 256);
  return w;
}

size_t full_decode_ws_bytes(const hs_varlen* vl, const Shape& sh) { return full_decode_layout(vl, sh).total; }

// Sparse decode on the tensor cores (decode_tc.cuh, namespace sdec): each
// (sequence, KV head) unit's slot space (window w + k selected tokens) is cut
// into 128-slot tiles and those into `nsplit` <= 8 ranges, one work item each;
// with more than one range, a unit's items are one thread-block cluster.
struct SparseDecodePlan {
  int unit_tiles, nsplit, tiles_per_split, n_items;
};

SparseDecodePlan sparse_decode_plan(const Shape& sh, const hs_sel* sel, int split_k) {
  SparseDecodePlan pl;
  const int U = sh.batch * sh.Hkv;
  // ranges of equal slot counts (not whole tiles): the ranges of a unit finish together
  pl.unit_tiles = std::max(1, (sel->topk * sel->block + sel->window + 127) / 128);
  int want = split_k > 0 ? split_k : std::max(1, num_sms() / std::max(1, U));
  want = std::min({want, pl.unit_tiles, dtc::sdec::kMaxSplit});
  pl.tiles_per_split = (pl.unit_tiles + want - 1) / want;
  pl.nsplit = (pl.unit_tiles + pl.tiles_per_split - 1) / pl.tiles_per_split;
  pl.n_items = U * pl.nsplit;
  return pl;
}

// Workspace: the header only (the ranges of a unit merge in shared memory).
size_t sparse_decode_ws_bytes(const Shape&, const hs_sel*) { return kHeaderBytes; }

// Token-level scores: items are (tile, KV head, 256-key range) up to the
// tile's last query position.
long long token_score_items(const hs_varlen* vl, int T, int Hkv) {
  long long n = 0;
  for (int b = 0; b < vl->batch; ++b) {
    const int n_b = vl->cu_q_host[b + 1] - vl->cu_q_host[b];
    const int c_b = vl->cu_kv_host[b + 1] - vl->cu_kv_host[b] - n_b;
    for (int i = 0; i * T < n_b; ++i) {
      const int last = c_b + std::min((i + 1) * T, n_b) - 1;
      n += (long long)Hkv * (last / (tscore::kBlocks * 128) + 1);
    }
  }
  return n;
}

// Waits on an mbarrier that nothing ever arrives at; the bounded wait gives up
// after wc.timeout_ns, records the failure in the error word and returns.
__global__ void debug_wait_kernel(WaitCtl wc) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, wc, 99);
}

// FP8-e4m3 KV rows -> bf16: thread = 16 codes of one row (one 16-byte load,
// two 16-byte stores); exact e4m3 -> f16 conversion, fp32 product with the
// row's scale, bf16 round-to-nearest-even. HBM-bound: 3 bytes per element.
__global__ void __launch_bounds__(256) kv_dequant_kernel(const uint4* __restrict__ codes, const float* __restrict__ scale,
                                                         uint4* __restrict__ out, long long rows, int chunks_per_row) {
  const long long n = rows * chunks_per_row;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float sc = __ldg(scale + i / chunks_per_row);
    const uint4 c = __ldg(codes + i);
    const uint32_t w4[4] = {c.x, c.y, c.z, c.w};
    uint32_t o8[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        uint32_t h2;
        asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(uint16_t(hlf ? (w4[e] >> 16) : (w4[e] & 0xFFFFu))));
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
        o8[2 * e + hlf] = pack_bf16(f.x * sc, f.y * sc);
      }
    }
    out[2 * i] = make_uint4(o8[0], o8[1], o8[2], o8[3]);
    out[2 * i + 1] = make_uint4(o8[4], o8[5], o8[6], o8[7]);
  }
}

// 2^x on the FMA pipe, as the softmax uses it, over an array (self test).
__global__ void debug_exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, long long n) {
  const long long stride = 2LL * gridDim.x * blockDim.x;
  for (long long i = 2LL * (blockIdx.x * (long long)blockDim.x + threadIdx.x); i < n; i += stride) {
    const bool two = i + 1 < n;
    float a, b;
    exp2_poly_pair(x[i], two ? x[i + 1] : 0.f, a, b);
    y[i] = a;
    if (two) y[i + 1] = b;
  }
}

template <int D, bool SELECT>
hs_status launch_token_scores(const Maps& m, const tscore::Params& p, const SeqTable& st, const int* prefix,
                              int grid, cudaStream_t s) {
  auto kern = tscore::token_scores_kernel<D, SELECT>;
  constexpr int smem =
      tscore::smem_bytes<D, SELECT>() > 116 * 1024 ? tscore::smem_bytes<D, SELECT>() : 116 * 1024;
  static PerDeviceOnce once;
  if (set_smem_once(once, kern, smem) != cudaSuccess) return HS_ERR_CUDA;
  kern<<<grid, tscore::threads<SELECT>(), smem, s>>>(m.q, m.k, p, st, prefix);
  return cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}

// Top-k taken inside the score pass (token level).
struct FusedTopk {
  const hs_sel* sel;
  int32_t* idx;
  int32_t* cnt;
};

// The token-level score pass: a second QK pass reduces max(s - lse) per key
// (see token_scores.cuh); with `top`, each plane's top-k is selected in the
// same kernel and the scores are left as scratch.
hs_status token_pass(const hs_varlen* vl, const Shape& sh, int T, const void* q, const Maps& fwd_maps,
                     const float* lse, float* scores, int nblk, float scale_log2, void* ws, cudaStream_t s,
                     const FusedTopk* top) {
  // Q chunks of tscore::kRows rows (query * G + head): a box of kRows / G queries
  Maps m = fwd_maps;
  if (!make_map_3d(&m.q, q, sh.d, sh.Hq, sh.Tq, sh.G, tscore::kRows / sh.G)) return HS_ERR_CUDA;
  SeqTable table;
  if (!fill_seqtable(vl, T, &table)) return HS_ERR_UNSUPPORTED;
  const long long items = token_score_items(vl, T, sh.Hkv);
  if (items > (1LL << 30)) return HS_ERR_UNSUPPORTED;
  char* w = reinterpret_cast<char*>(ws) + kHeaderBytes;
  int* prefix = reinterpret_cast<int*>(w);
  int* order = top ? reinterpret_cast<int*>(w + token_prefix_bytes(table.n_tiles)) : nullptr;
  const size_t n_planes = size_t(table.n_tiles) * sh.Hkv;
  int* arrive = top ? order + table.n_tiles : nullptr;
  int* queue = top ? arrive + n_planes : nullptr;
  int* qctr = top ? queue + n_planes : nullptr;
  tscore::item_prefix_kernel<<<1, 1024, 0, s>>>(table, sh.Hkv, prefix, order, arrive, queue, qctr);
  if (cudaGetLastError() != cudaSuccess) return HS_ERR_CUDA;
  tscore::Params tp{};
  tp.lse = lse;
  tp.scores = scores;
  tp.G = sh.G;
  tp.Hq = sh.Hq;
  tp.Hkv = sh.Hkv;
  tp.Tq = int(sh.Tq);
  tp.nblk = nblk;
  tp.scale_log2 = scale_log2;
  tp.n_items = int(items);
  tp.wc = wait_ctl(ws);
  if (top) {
    tp.arrive = arrive;
    tp.queue = queue;
    tp.qctr = qctr;
    tp.idx = top->idx;
    tp.cnt = top->cnt;
    tp.k = top->sel->topk;
    tp.w = top->sel->window;
    tp.exclusive = (top->sel->flags & HS_SEL_WINDOW_EXCLUSIVE) ? 1 : 0;
    tp.discard = 1;
    tp.order = order;
  }
  const int tgrid = int(std::min<long long>(num_sms(), std::max<long long>(1, items)));
  if (top)
    return sh.d == 64 ? launch_token_scores<64, true>(m, tp, table, prefix, tgrid, s)
                      : launch_token_scores<128, true>(m, tp, table, prefix, tgrid, s);
  return sh.d == 64 ? launch_token_scores<64, false>(m, tp, table, prefix, tgrid, s)
                    : launch_token_scores<128, false>(m, tp, table, prefix, tgrid, s);
}

}  // namespace

// ----------------------------------------------------------------------------
// Scratch for hs_full_attn_select_noalloc: callers that cannot allocate device
// memory get this fixed array instead of a workspace. It is resident on every
// GPU that loads the library until the process exits. Layout: the 256-byte
// error header, then the per-CTA block-maximum spill.
// ----------------------------------------------------------------------------
static constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kNoAllocMaxDevices = 128;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of the scratch array on the current device. In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device (with that device current) and cached.
hs_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return HS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr) return HS_ERR_CUDA;
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return HS_OK;
}
}  // namespace

// ============================================================================
template <int D>
hs_status launch_swa_gated_decode(const hs_varlen* vl, const Shape& sh, int window, int ring_len,
                                         const void* q, const void* k_ring, const void* v_ring, const float* gamma,
                                         const void* o_sparse, void* o, cudaStream_t s) {
  const int smem = 4 * swad::smem_words<D>(sh.G, window);
  static PerDeviceOnce once;
  if (set_smem_once(once, swad::swa_gated_decode_kernel<D>, 4 * swad::smem_words<D>(swad::kMaxG, swad::kMaxWindow)) !=
      cudaSuccess)
    return HS_ERR_CUDA;
  swad::swa_gated_decode_kernel<D><<<vl->batch * sh.Hkv, swad::kThreads, smem, s>>>(
      vl->cu_q, vl->cu_kv, sh.Hq, sh.Hkv, sh.G, window, ring_len, sh.scale * 1.4426950408889634f,
      reinterpret_cast<const __nv_bfloat16*>(q), reinterpret_cast<const __nv_bfloat16*>(k_ring),
      reinterpret_cast<const __nv_bfloat16*>(v_ring), gamma, reinterpret_cast<const __nv_bfloat16*>(o_sparse),
      reinterpret_cast<__nv_bfloat16*>(o));
  return cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}

extern "C" {

const char* hs_status_string(hs_status s) {
  switch (s) {
    case HS_OK: return "ok";
    case HS_ERR_INVALID_ARG: return "invalid argument";
    case HS_ERR_UNSUPPORTED: return "unsupported configuration";
    case HS_ERR_WORKSPACE: return "workspace missing or too small";
    case HS_ERR_CUDA: return "CUDA error";
    case HS_ERR_TIMEOUT: return "device-side bounded wait timed out";
  }
  return "unknown status";
}

size_t hs_workspace_size(int op, const hs_varlen* vl, const hs_sel* sel) {
  Shape sh;
  if (check_varlen(vl, &sh, false) != HS_OK) return 0;
  switch (op) {
    case HS_OP_FULL_ATTN_SELECT:
      if (!sel || check_sel(sel) != HS_OK) return 0;
      return full_ws_bytes(vl, sh, sel);
    case HS_OP_TOPK_SELECT:
    case HS_OP_SPARSE_ATTN_PREFILL:
    case HS_OP_SWA_GATED:
    case HS_OP_SPARSE_SWA_GATED_PREFILL:
      return kHeaderBytes;
    case HS_OP_SPARSE_ATTN_DECODE:
      if (!sel || check_sel(sel) != HS_OK) return 0;
      return sparse_decode_ws_bytes(sh, sel);
    default:
      return 0;
  }
}

hs_status hs_workspace_init(void* ws, size_t ws_bytes, hs_stream_t stream) {
  if (!ws || ws_bytes < kHeaderBytes) return HS_ERR_WORKSPACE;
  return cudaMemsetAsync(ws, 0, kHeaderBytes, S(stream)) == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}

static ErrWord last_err{};

hs_status hs_check_error(void* ws, hs_stream_t stream) {
  if (!ws) return HS_ERR_WORKSPACE;
  if (cudaStreamSynchronize(S(stream)) != cudaSuccess) return HS_ERR_CUDA;
  ErrWord e{};
  if (cudaMemcpy(&e, ws, sizeof(e), cudaMemcpyDeviceToHost) != cudaSuccess) return HS_ERR_CUDA;
  if (e.flag != 0) {
    last_err = e;
    if (cudaMemset(ws, 0, sizeof(ErrWord)) != cudaSuccess) return HS_ERR_CUDA;
    return HS_ERR_TIMEOUT;
  }
  return HS_OK;
}

// The full layer; with `top` (token-level prefill only) the top-k is taken
// inside the score pass and `scores` is scratch.
static hs_status full_attn_select_impl(const hs_varlen* vl, const hs_sel* sel, const void* q, const void* k,
                                       const void* v, void* o, float* lse, float* scores, void* ws,
                                       size_t ws_bytes, hs_stream_t stream, const FusedTopk* top) {
  Shape sh;
  hs_status st = check_varlen(vl, &sh);
  if (st != HS_OK) return st;
  if ((st = check_sel(sel)) != HS_OK) return st;
  if (sh.Tq == 0) return HS_OK;  // nothing to read or write (pointers may be null)
  if (!q || !k || !v || !o || !scores) return HS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return HS_ERR_INVALID_ARG;
  if (!ws || ws_bytes < full_ws_bytes(vl, sh, sel)) return HS_ERR_WORKSPACE;
  if (!is_pow2(sh.G) || sh.G > 128) return HS_ERR_UNSUPPORTED;
  if (vl->batch > attn::kMaxSched) return HS_ERR_UNSUPPORTED;
  const int T = sel->q_tile, B = sel->block;
  const int n_tiles = n_tiles_of(vl, T);
  const int nblk = (sh.max_kv + B - 1) / B;
  cudaStream_t s = S(stream);
  // the fused top-k reads only keys the score pass wrote: no zero fill
  if (!top && cudaMemsetAsync(scores, 0, size_t(n_tiles) * sh.Hkv * nblk * sizeof(float), s) != cudaSuccess)
    return HS_ERR_CUDA;
  if (is_decode(vl, sel) && sh.d == 128 && sh.G <= 64) {
    if (top) return HS_ERR_UNSUPPORTED;
    // one query per sequence: both exact passes in one persistent tcgen05 kernel
    const int U = sh.batch * sh.Hkv;
    if (U > dtc::kMaxUnits) return HS_ERR_UNSUPPORTED;
    static dtc::Sched dsc;  // large; filled under the lock
    static std::mutex dmu;
    std::lock_guard<std::mutex> lock(dmu);
    const int chunk_keys = full_decode_chunk_keys(vl, sh);
    dsc.n_units = U;
    dsc.Hkv = sh.Hkv;
    dsc.chunk_keys = chunk_keys;
    for (int b = 0; b <= sh.batch; ++b) dsc.cu_kv[b] = vl->cu_kv_host[b];
    std::vector<int> nch(U);
    dsc.chunk_base[0] = 0;
    for (int u = 0; u < U; ++u) {
      const int b = u / sh.Hkv;
      nch[u] = (vl->cu_kv_host[b + 1] - vl->cu_kv_host[b] + chunk_keys - 1) / chunk_keys;
      dsc.chunk_base[u + 1] = dsc.chunk_base[u] + nch[u];
    }
    // pass-2 items trail the pass-1 stream by D items (see decode_tc.cuh)
    int s_max = 0;
    for (int u = 0; u < U; ++u) s_max = std::max(s_max, nch[u]);
    dsc.n1 = dsc.chunk_base[U];
    dsc.delay = std::min(dsc.n1, s_max + HS_DEC_DELAY_GRIDS * num_sms());
    dsc.n_items = 2 * dsc.n1;
    const FullDecodeWs lay = full_decode_layout(vl, sh);
    char* w = reinterpret_cast<char*>(ws);
    dtc::Params dp{};
    dp.q = reinterpret_cast<const __nv_bfloat16*>(q);
    dp.G = sh.G;
    dp.Hq = sh.Hq;
    dp.Hkv = sh.Hkv;
    dp.Tq = int(sh.Tq);
    dp.nblk = nblk;
    dp.scale_log2 = sh.scale * 1.4426950408889634f;
    dp.sync = reinterpret_cast<int*>(w + lay.sync);
    dp.o_acc = reinterpret_cast<float*>(w + lay.o_acc);
    dp.lse2 = reinterpret_cast<float*>(w + lay.lse2);
    dp.unit_l = reinterpret_cast<double*>(w + lay.unit_l);
    dp.scores = scores;
    dp.o = reinterpret_cast<__nv_bfloat16*>(o);
    dp.lse = lse;
    dp.wc = wait_ctl(ws);
    if (cudaMemsetAsync(w + lay.sync, 0, lay.lse2 - lay.sync, s) != cudaSuccess) return HS_ERR_CUDA;
    Maps m;
    if (!make_map_3d(&m.q, q, sh.d, sh.Hq, sh.Tq, sh.G, 1) || !make_map_3d(&m.k, k, sh.d, sh.Hkv, sh.Tkv, 1, 128) ||
        !make_map_3d(&m.v, v, sh.d, sh.Hkv, sh.Tkv, 1, 128))
      return HS_ERR_CUDA;
    static PerDeviceOnce once;
    if (set_smem_once(once, dtc::full_decode_tc_kernel, dtc::smem_bytes()) != cudaSuccess) return HS_ERR_CUDA;
    const int grid = std::min(num_sms(), std::max(1, dsc.n_items));
    dtc::full_decode_tc_kernel<<<grid, dtc::kThreads, dtc::smem_bytes(), s>>>(m.q, m.k, m.v, dp, dsc);
    return cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
  }

  Maps m;
  if (!make_map_3d(&m.q, q, sh.d, sh.Hq, sh.Tq, sh.G, 128 / sh.G) ||
      !make_map_3d(&m.k, k, sh.d, sh.Hkv, sh.Tkv, 1, 128) || !make_map_3d(&m.v, v, sh.d, sh.Hkv, sh.Tkv, 1, 128))
    return HS_ERR_CUDA;
  m.kb = m.k;
  m.vb = m.v;
  m.g = m.o = m.ks = m.vs = m.q;
  static attn::Sched sc;  // large; filled per call under the host lock below
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (!fill_sched(vl, sh, attn::kFull, T, 1, &sc)) return HS_ERR_UNSUPPORTED;
  attn::Params p{};
  p.G = sh.G;
  p.Hq = sh.Hq;
  p.Hkv = sh.Hkv;
  p.Tq = int(sh.Tq);
  p.scale_log2 = sh.scale * 1.4426950408889634f;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.scores = scores;
  p.spill = reinterpret_cast<float*>(reinterpret_cast<char*>(ws) + kHeaderBytes);
  p.spill_tiles = (sh.max_kv + 127) / 128;
  p.nblk = nblk;
  p.T = T;
  p.B = B;
  p.chunks_per_tile = 1;
  p.wc = wait_ctl(ws);
  const int grid = std::min(num_sms(), std::max(1, sc.n_items));
  hs_status rc = dispatch_full(sh.d, B, m, p, sc, grid, s);
  if (rc != HS_OK || B > 1) return rc;
  // token level: the second QK pass (see token_scores.cuh), with the top-k fused when asked
  if (!lse) return HS_ERR_INVALID_ARG;
  return token_pass(vl, sh, T, q, m, lse, scores, nblk, p.scale_log2, ws, s, top);
}

hs_status hs_full_attn_select(const hs_varlen* vl, const hs_sel* sel, const void* q, const void* k,
                              const void* v, void* o, float* lse, float* scores, void* ws, size_t ws_bytes,
                              hs_stream_t stream) {
  return full_attn_select_impl(vl, sel, q, k, v, o, lse, scores, ws, ws_bytes, stream, nullptr);
}

hs_status hs_full_attn_select_topk(const hs_varlen* vl, const hs_sel* sel, const void* q, const void* k,
                                   const void* v, void* o, float* lse, float* scores, int32_t* idx,
                                   int32_t* cnt, void* ws, size_t ws_bytes, hs_stream_t stream) {
  Shape sh;
  hs_status st = check_varlen(vl, &sh);
  if (st != HS_OK) return st;
  if ((st = check_sel(sel)) != HS_OK) return st;
  if (sh.Tq == 0) return HS_OK;  // nothing to read or write (pointers may be null)
  if (!idx || !cnt) return HS_ERR_INVALID_ARG;
  if (vl->batch > kMaxSeq) return HS_ERR_UNSUPPORTED;
  const bool fused = sel->block == 1 && !(is_decode(vl, sel) && sh.d == 128 && sh.G <= 64);
  if (fused) {
    const FusedTopk top{sel, idx, cnt};
    return full_attn_select_impl(vl, sel, q, k, v, o, lse, scores, ws, ws_bytes, stream, &top);
  }
  // block-level scores and the decode kernel: the two calls back to back
  st = full_attn_select_impl(vl, sel, q, k, v, o, lse, scores, ws, ws_bytes, stream, nullptr);
  if (st != HS_OK) return st;
  return hs_topk_select(vl, sel, scores, idx, cnt, ws, ws_bytes, stream);
}

hs_status hs_topk_select(const hs_varlen* vl, const hs_sel* sel, const float* scores, int32_t* idx, int32_t* cnt,
                         void* ws, size_t ws_bytes, hs_stream_t stream) {
  Shape sh;
  hs_status st = check_varlen(vl, &sh, false);
  if (st != HS_OK) return st;
  if ((st = check_sel(sel)) != HS_OK) return st;
  if (sh.Tq == 0) return HS_OK;  // nothing to read or write (pointers may be null)
  if (!scores || !idx || !cnt) return HS_ERR_INVALID_ARG;
  if (!ws || ws_bytes < kHeaderBytes) return HS_ERR_WORKSPACE;
  if (vl->batch > kMaxSeq) return HS_ERR_UNSUPPORTED;
  SeqTable table;
  fill_seqtable(vl, sel->q_tile, &table);
  topk::Params p{};
  p.scores = scores;
  p.idx = idx;
  p.cnt = cnt;
  p.Hkv = sh.Hkv;
  p.nblk = (sh.max_kv + sel->block - 1) / sel->block;
  p.B = sel->block;
  p.k = sel->topk;
  p.w = sel->window;
  p.exclusive = (sel->flags & HS_SEL_WINDOW_EXCLUSIVE) ? 1 : 0;
  const long long rows = (long long)table.n_tiles * sh.Hkv;
  if (rows > (1LL << 31) - 1) return HS_ERR_UNSUPPORTED;
  if (p.nblk <= topk::kStageMax)
    topk::topk_kernel<256, true><<<unsigned(rows), 256, 0, S(stream)>>>(p, table);
  else
    topk::topk_kernel<1024, false><<<unsigned(rows), 1024, 0, S(stream)>>>(p, table);
  return cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}

// One sparse layer: the plain sparse branch, or (swa != null) the fused layer
// with the sliding-window branch and the gate.
struct SwaArgs {
  int32_t window;
  const void* k_swa;
  const void* v_swa;
  const float* gamma;
  void* o_sparse;  // optional
};

// Selected rows gathered once per block (token level): kg / vg [n_tiles][Hkv][topk][d].
struct GatheredKV {
  const void* kg;
  const void* vg;
};

static hs_status sparse_layer(const hs_varlen* vl, const hs_sel* sel, const void* q, const void* k, const void* v,
                              const int32_t* idx, const int32_t* cnt, void* o, float* lse, const SwaArgs* swa,
                              void* ws, size_t ws_bytes, hs_stream_t stream, const GatheredKV* gkv = nullptr) {
  Shape sh;
  hs_status st = check_varlen(vl, &sh);
  if (st != HS_OK) return st;
  if ((st = check_sel(sel)) != HS_OK) return st;
  if (sh.Tq == 0) return HS_OK;  // nothing to read or write (pointers may be null)
  if (!q || !k || !v || !o || (sel->topk > 0 && (!idx || !cnt))) return HS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return HS_ERR_INVALID_ARG;
  if (swa) {
    if (swa->window < 1 || !swa->k_swa || !swa->v_swa || !swa->gamma) return HS_ERR_INVALID_ARG;
    if (!aligned16(swa->k_swa) || !aligned16(swa->v_swa) || (swa->o_sparse && !aligned16(swa->o_sparse)))
      return HS_ERR_INVALID_ARG;
  }
  if (!ws || ws_bytes < kHeaderBytes) return HS_ERR_WORKSPACE;
  if (!is_pow2(sh.G) || sh.G > 128) return HS_ERR_UNSUPPORTED;
  if (vl->batch > attn::kMaxSched) return HS_ERR_UNSUPPORTED;
  const int T = sel->q_tile, B = sel->block;
  if (gkv && (B != 1 || swa || !gkv->kg || !gkv->vg || !aligned16(gkv->kg) || !aligned16(gkv->vg)))
    return HS_ERR_INVALID_ARG;
  Maps m;
  if (!make_map_3d(&m.q, q, sh.d, sh.Hq, sh.Tq, sh.G, 128 / sh.G) ||
      !make_map_3d(&m.k, k, sh.d, sh.Hkv, sh.Tkv, 1, 128) || !make_map_3d(&m.v, v, sh.d, sh.Hkv, sh.Tkv, 1, 128))
    return HS_ERR_CUDA;
  if (gkv) {
    // planes of topk slots, one per (selection tile, KV head); 128-slot boxes
    const long long planes = (long long)n_sel_tiles(vl, T) * sh.Hkv;
    if (sel->topk > 0 && (!make_map_3d(&m.kb, gkv->kg, sh.d, sel->topk, planes, 128, 1) ||
                          !make_map_3d(&m.vb, gkv->vg, sh.d, sel->topk, planes, 128, 1)))
      return HS_ERR_CUDA;
    if (sel->topk == 0) m.kb = m.vb = m.k;
  } else if (B == 1) {
    if (!make_map_rows(&m.kb, k, sh.d, sh.Tkv * sh.Hkv) || !make_map_rows(&m.vb, v, sh.d, sh.Tkv * sh.Hkv))
      return HS_ERR_CUDA;
  } else if (!make_map_3d(&m.kb, k, sh.d, sh.Hkv, sh.Tkv, 1, B) || !make_map_3d(&m.vb, v, sh.d, sh.Hkv, sh.Tkv, 1, B)) {
    return HS_ERR_CUDA;
  }
  m.g = m.o = m.ks = m.vs = m.q;
  if (swa && (!make_map_3d(&m.ks, swa->k_swa, sh.d, sh.Hkv, sh.Tkv, 1, 128) ||
              !make_map_3d(&m.vs, swa->v_swa, sh.d, sh.Hkv, sh.Tkv, 1, 128)))
    return HS_ERR_CUDA;
  static attn::Sched sc;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  const int cpt = (T * sh.G + attn::kMaxItemRows - 1) / attn::kMaxItemRows;
  if (!fill_sched(vl, sh, attn::kSparse, T, cpt, &sc)) return HS_ERR_UNSUPPORTED;
  attn::Params p{};
  p.G = sh.G;
  p.Hq = sh.Hq;
  p.Hkv = sh.Hkv;
  p.Tq = int(sh.Tq);
  p.scale_log2 = sh.scale * 1.4426950408889634f;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.T = T;
  p.B = B;
  p.chunks_per_tile = cpt;
  p.idx = idx;
  p.cnt = cnt;
  p.topk = sel->topk;
  p.w = sel->window;
  p.gathered = gkv ? 1 : 0;
  p.wc = wait_ctl(ws);
  if (swa) {
    p.ws = swa->window;
    p.gamma = swa->gamma;
    p.o_mid = reinterpret_cast<__nv_bfloat16*>(swa->o_sparse);
    // the final output goes through the smem buffer by TMA in 64-row rounds of whole queries (G | 64)
    p.o_tma = sh.G <= 64 && make_map_3d(&m.o, o, sh.d, sh.Hq, sh.Tq, sh.G, 64 / sh.G);
  }
  const int grid = std::min(num_sms(), std::max(1, sc.n_items));
  if (swa) {
    switch (B) {
      case 1: return dispatch_attn_d<attn::kFused, 1>(sh.d, m, p, sc, grid, S(stream));
      case 8: return dispatch_attn_d<attn::kFused, 8>(sh.d, m, p, sc, grid, S(stream));
      case 16: return dispatch_attn_d<attn::kFused, 16>(sh.d, m, p, sc, grid, S(stream));
      case 32: return dispatch_attn_d<attn::kFused, 32>(sh.d, m, p, sc, grid, S(stream));
      case 64: return dispatch_attn_d<attn::kFused, 64>(sh.d, m, p, sc, grid, S(stream));
      case 128: return dispatch_attn_d<attn::kFused, 128>(sh.d, m, p, sc, grid, S(stream));
      default: return HS_ERR_UNSUPPORTED;
    }
  }
  switch (B) {
    case 1: return dispatch_attn_d<attn::kSparse, 1>(sh.d, m, p, sc, grid, S(stream));
    case 8: return dispatch_attn_d<attn::kSparse, 8>(sh.d, m, p, sc, grid, S(stream));
    case 16: return dispatch_attn_d<attn::kSparse, 16>(sh.d, m, p, sc, grid, S(stream));
    case 32: return dispatch_attn_d<attn::kSparse, 32>(sh.d, m, p, sc, grid, S(stream));
    case 64: return dispatch_attn_d<attn::kSparse, 64>(sh.d, m, p, sc, grid, S(stream));
    case 128: return dispatch_attn_d<attn::kSparse, 128>(sh.d, m, p, sc, grid, S(stream));
    default: return HS_ERR_UNSUPPORTED;
  }
}

hs_status hs_sparse_attn_prefill(const hs_varlen* vl, const hs_sel* sel, const void* q, const void* k,
                                 const void* v, const int32_t* idx, const int32_t* cnt, void* o, float* lse,
                                 void* ws, size_t ws_bytes, hs_stream_t stream) {
  return sparse_layer(vl, sel, q, k, v, idx, cnt, o, lse, nullptr, ws, ws_bytes, stream);
}

hs_status hs_sparse_attn_prefill_gathered(const hs_varlen* vl, const hs_sel* sel, const void* q, const void* k,
                                          const void* v, const void* kg, const void* vg, const int32_t* idx,
                                          const int32_t* cnt, void* o, float* lse, void* ws, size_t ws_bytes,
                                          hs_stream_t stream) {
  const GatheredKV gkv{kg, vg};
  return sparse_layer(vl, sel, q, k, v, idx, cnt, o, lse, nullptr, ws, ws_bytes, stream, &gkv);
}

// One CTA per (selection tile, KV head) plane; thread = 16-byte piece of a
// slot row (16 consecutive threads read one 256-byte row and write it out
// contiguously). Slots past cnt are zero. HBM-bound: 2 x (topk rows read +
// topk rows written) per plane.
__global__ void __launch_bounds__(256) gather_selected_kernel(const __grid_constant__ SeqTable st, int Hkv, int topk,
                                                              int pieces, const uint4* __restrict__ k,
                                                              const uint4* __restrict__ v, const int* __restrict__ idx,
                                                              const int* __restrict__ cnt, uint4* __restrict__ kg,
                                                              uint4* __restrict__ vg) {
  const int plane = blockIdx.x;  // tile * Hkv + g
  const int tile = plane / Hkv, g = plane % Hkv;
  const TileInfo ti = tile_info(st, tile);
  const int c = __ldg(cnt + plane);
  const int* ip = idx + size_t(plane) * topk;
  const size_t base = size_t(plane) * topk * pieces;
  const int n = topk * pieces;
#pragma unroll 4
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int s = e / pieces, pc = e - s * pieces;
    uint4 kv = make_uint4(0u, 0u, 0u, 0u), vv = kv;
    if (s < c) {
      const size_t row = (size_t(ti.kv0) + __ldg(ip + s)) * Hkv + g;
      kv = __ldg(k + row * pieces + pc);
      vv = __ldg(v + row * pieces + pc);
    }
    kg[base + e] = kv;
    vg[base + e] = vv;
  }
}

hs_status hs_gather_selected_kv(const hs_varlen* vl, const hs_sel* sel, const void* k, const void* v,
                                const int32_t* idx, const int32_t* cnt, void* kg, void* vg, hs_stream_t stream) {
  Shape sh;
  hs_status st = check_varlen(vl, &sh);
  if (st != HS_OK) return st;
  if ((st = check_sel(sel)) != HS_OK) return st;
  if (sel->block != 1) return HS_ERR_INVALID_ARG;
  if (sh.Tq == 0 || sel->topk == 0) return HS_OK;
  if (!k || !v || !idx || !cnt || !kg || !vg || !aligned16(k) || !aligned16(v) || !aligned16(kg) || !aligned16(vg))
    return HS_ERR_INVALID_ARG;
  if (sh.d % 8) return HS_ERR_UNSUPPORTED;
  SeqTable table;
  if (!fill_seqtable(vl, sel->q_tile, &table)) return HS_ERR_UNSUPPORTED;
  const long long planes = (long long)table.n_tiles * sh.Hkv;
  if (planes == 0) return HS_OK;
  if (planes > INT32_MAX) return HS_ERR_UNSUPPORTED;
  gather_selected_kernel<<<unsigned(planes), 256, 0, S(stream)>>>(
      table, sh.Hkv, sel->topk, sh.d / 8, reinterpret_cast<const uint4*>(k), reinterpret_cast<const uint4*>(v), idx,
      cnt, reinterpret_cast<uint4*>(kg), reinterpret_cast<uint4*>(vg));
  return cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}

hs_status hs_sparse_swa_gated_prefill(const hs_varlen* vl, const hs_sel* sel, const void* q, const void* k,
                                      const void* v, const int32_t* idx, const int32_t* cnt, int32_t swa_window,
                                      const void* k_swa, const void* v_swa, const float* gamma, void* o,
                                      void* o_sparse, float* lse_sparse, void* ws, size_t ws_bytes,
                                      hs_stream_t stream) {
  const SwaArgs swa{swa_window, k_swa, v_swa, gamma, o_sparse};
  return sparse_layer(vl, sel, q, k, v, idx, cnt, o, lse_sparse, &swa, ws, ws_bytes, stream);
}

hs_status hs_sparse_attn_decode(const hs_varlen* vl, const hs_sel* sel, const void* q, hs_kv_dtype kv_dtype,
                                const void* k, const void* v, const float* k_scale, const float* v_scale,
                                const int32_t* idx, const int32_t* cnt, int32_t split_k, void* o, float* lse,
                                void* ws, size_t ws_bytes, hs_stream_t stream) {
  Shape sh;
  hs_status st = check_varlen(vl, &sh);
  if (st != HS_OK) return st;
  if ((st = check_sel(sel)) != HS_OK) return st;
  if (sh.Tq == 0) return HS_OK;  // nothing to read or write (pointers may be null)
  if (!is_decode_batch(vl, sel)) return HS_ERR_INVALID_ARG;  // one query per sequence, q_tile = 1
  if (sh.d != 128 || sh.G > 64) return HS_ERR_UNSUPPORTED;
  if (kv_dtype != HS_KV_BF16 && kv_dtype != HS_KV_FP8_E4M3) return HS_ERR_INVALID_ARG;
  const bool fp8 = kv_dtype == HS_KV_FP8_E4M3;
  if (!q || !k || !v || !o || (sel->topk > 0 && (!idx || !cnt)) || (fp8 && (!k_scale || !v_scale)))
    return HS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return HS_ERR_INVALID_ARG;
  if (split_k < 0) return HS_ERR_INVALID_ARG;
  if (sel->topk + sel->window == 0) return HS_ERR_INVALID_ARG;  // empty visible set
  if (!ws || ws_bytes < sparse_decode_ws_bytes(sh, sel)) return HS_ERR_WORKSPACE;
  const int U = sh.batch * sh.Hkv;
  if (U > dtc::sdec::kMaxUnits) return HS_ERR_UNSUPPORTED;
  const SparseDecodePlan pl = sparse_decode_plan(sh, sel, split_k);
  cudaStream_t s = S(stream);
  dtc::sdec::Params p{};
  p.idx = idx;
  p.cnt = sel->topk > 0 ? cnt : nullptr;
  p.cu_kv = vl->cu_kv;
  p.k = reinterpret_cast<const uint8_t*>(k);
  p.v = reinterpret_cast<const uint8_t*>(v);
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  p.topk = sel->topk;
  p.w = sel->window;
  p.log2_block = __builtin_ctz(unsigned(sel->block));  // a power of two (check_sel)
  p.G = sh.G;
  p.Hq = sh.Hq;
  p.Hkv = sh.Hkv;
  p.Tq = int(sh.Tq);
  p.n_units = U;
  p.nsplit = pl.nsplit;
  p.tiles_per_split = pl.tiles_per_split;
  p.unit_tiles = pl.unit_tiles;
  p.n_items = pl.n_items;
  p.scale_log2 = sh.scale * 1.4426950408889634f;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.wc = wait_ctl(ws);
  CUtensorMap map_q;
  if (!make_map_3d(&map_q, q, sh.d, sh.Hq, sh.Tq, sh.G, 1)) return HS_ERR_CUDA;
  // one range per unit: a persistent grid over the units; several: one CTA
  // per range, a unit's ranges in one cluster
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  cfg.gridDim = dim3(pl.nsplit > 1 ? pl.n_items : std::min(num_sms(), pl.n_items));
  cfg.blockDim = dim3(dtc::sdec::kThreads);
  cfg.stream = s;
  if (pl.nsplit > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(pl.nsplit);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  cudaError_t e;
  if (fp8) {
    cfg.dynamicSmemBytes = dtc::sdec::smem_bytes<true>();
    static PerDeviceOnce once;
    if (set_smem_once(once, dtc::sdec::sparse_decode_tc_kernel<true>, int(cfg.dynamicSmemBytes)) != cudaSuccess)
      return HS_ERR_CUDA;
    e = cudaLaunchKernelEx(&cfg, dtc::sdec::sparse_decode_tc_kernel<true>, map_q, p);
  } else {
    cfg.dynamicSmemBytes = dtc::sdec::smem_bytes<false>();
    static PerDeviceOnce once;
    if (set_smem_once(once, dtc::sdec::sparse_decode_tc_kernel<false>, int(cfg.dynamicSmemBytes)) != cudaSuccess)
      return HS_ERR_CUDA;
    e = cudaLaunchKernelEx(&cfg, dtc::sdec::sparse_decode_tc_kernel<false>, map_q, p);
  }
  return e == cudaSuccess && cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}

hs_status hs_swa_ring_write(const hs_varlen* vl, int32_t ring_len, const void* k_new, const void* v_new,
                            void* k_ring, void* v_ring, hs_stream_t stream) {
  Shape sh;
  hs_status st = check_varlen(vl, &sh);
  if (st != HS_OK) return st;
  if (ring_len < 1) return HS_ERR_INVALID_ARG;
  if (sh.Tq == 0) return HS_OK;
  if (!k_new || !v_new || !k_ring || !v_ring || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_ring) ||
      !aligned16(v_ring))
    return HS_ERR_INVALID_ARG;
  const int row_pieces = sh.Hkv * sh.d / 8;
  const long long n = sh.Tq * row_pieces;
  const int grid = int(std::min<long long>(8LL * num_sms(), (n + 255) / 256));
  swad::ring_write_kernel<<<grid, 256, 0, S(stream)>>>(
      vl->cu_q, vl->cu_kv, vl->batch, sh.Tq, row_pieces, ring_len, reinterpret_cast<const uint4*>(k_new),
      reinterpret_cast<const uint4*>(v_new), reinterpret_cast<uint4*>(k_ring), reinterpret_cast<uint4*>(v_ring));
  return cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}

hs_status hs_swa_gated_decode(const hs_varlen* vl, int32_t window, int32_t ring_len, const void* q,
                              const void* k_ring, const void* v_ring, const float* gamma, const void* o_sparse,
                              void* o, hs_stream_t stream) {
  Shape sh;
  hs_status st = check_varlen(vl, &sh);
  if (st != HS_OK) return st;
  if (window < 1 || ring_len < window) return HS_ERR_INVALID_ARG;
  if (sh.Tq == 0) return HS_OK;
  for (int b = 0; b < vl->batch; ++b)  // one new token per sequence, which sees itself
    if (vl->cu_q_host[b + 1] - vl->cu_q_host[b] != 1 || vl->cu_kv_host[b + 1] - vl->cu_kv_host[b] < 1)
      return HS_ERR_INVALID_ARG;
  if (window > swad::kMaxWindow || sh.G > swad::kMaxG) return HS_ERR_UNSUPPORTED;
  if (!q || !k_ring || !v_ring || !gamma || !o_sparse || !o || !aligned16(k_ring) || !aligned16(v_ring) ||
      (reinterpret_cast<uintptr_t>(gamma) & 3) || (reinterpret_cast<uintptr_t>(q) & 3) ||
      (reinterpret_cast<uintptr_t>(o) & 3) || (reinterpret_cast<uintptr_t>(o_sparse) & 3))
    return HS_ERR_INVALID_ARG;
  if (sh.d == 64) return launch_swa_gated_decode<64>(vl, sh, window, ring_len, q, k_ring, v_ring, gamma, o_sparse, o, S(stream));
  return launch_swa_gated_decode<128>(vl, sh, window, ring_len, q, k_ring, v_ring, gamma, o_sparse, o, S(stream));
}

hs_status hs_swa_gated(const hs_varlen* vl, int32_t window, const void* q, const void* k_swa, const void* v_swa,
                       const float* gamma, const void* o_sparse, void* o, void* ws, size_t ws_bytes,
                       hs_stream_t stream) {
  Shape sh;
  hs_status st = check_varlen(vl, &sh);
  if (st != HS_OK) return st;
  if (sh.Tq == 0) return HS_OK;  // nothing to read or write (pointers may be null)
  if (window < 1) return HS_ERR_INVALID_ARG;
  if (!q || !k_swa || !v_swa || !gamma || !o_sparse || !o) return HS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_swa) || !aligned16(v_swa) || !aligned16(o) || !aligned16(o_sparse))
    return HS_ERR_INVALID_ARG;
  if (!ws || ws_bytes < kHeaderBytes) return HS_ERR_WORKSPACE;
  if (!is_pow2(sh.G) || sh.G > 128) return HS_ERR_UNSUPPORTED;
  if (vl->batch > attn::kMaxSched) return HS_ERR_UNSUPPORTED;
  Maps m;
  if (!make_map_3d(&m.q, q, sh.d, sh.Hq, sh.Tq, sh.G, 128 / sh.G) ||
      !make_map_3d(&m.k, k_swa, sh.d, sh.Hkv, sh.Tkv, 1, 128) ||
      !make_map_3d(&m.v, v_swa, sh.d, sh.Hkv, sh.Tkv, 1, 128))
    return HS_ERR_CUDA;
  m.kb = m.k;
  m.vb = m.v;
  m.g = m.o = m.ks = m.vs = m.q;
  static attn::Sched sc;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  const int T = attn::kMaxItemRows / sh.G;  // one 256-row chunk per schedule tile
  if (!fill_sched(vl, sh, attn::kSparse, T, 1, &sc)) return HS_ERR_UNSUPPORTED;
  attn::Params p{};
  p.G = sh.G;
  p.Hq = sh.Hq;
  p.Hkv = sh.Hkv;
  p.Tq = int(sh.Tq);
  p.scale_log2 = sh.scale * 1.4426950408889634f;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = nullptr;
  p.T = T;
  p.B = 1;
  p.chunks_per_tile = 1;
  p.idx = nullptr;
  p.cnt = nullptr;
  p.topk = 0;
  p.w = window;
  p.gamma = gamma;
  p.o_other = reinterpret_cast<const __nv_bfloat16*>(o_sparse);
  // 64-row rounds of whole queries need G | 64; G = 128 mixes with direct loads/stores
  p.o_tma = sh.G <= 64 && make_map_3d(&m.g, o_sparse, sh.d, sh.Hq, sh.Tq, sh.G, 64 / sh.G) &&
            make_map_3d(&m.o, o, sh.d, sh.Hq, sh.Tq, sh.G, 64 / sh.G);
  p.wc = wait_ctl(ws);
  const int grid = std::min(num_sms(), std::max(1, sc.n_items));
  return dispatch_attn_d<attn::kSparse, 0>(sh.d, m, p, sc, grid, S(stream));
}

hs_status hs_full_attn_select_noalloc(const hs_varlen* vl, const hs_sel* sel, const void* q, const void* k,
                                      const void* v, void* o, float* lse, float* scores, int32_t check,
                                      hs_stream_t stream) {
  Shape sh;
  hs_status st = check_varlen(vl, &sh);
  if (st != HS_OK) return st;
  if ((st = check_sel(sel)) != HS_OK) return st;
  if (sh.Tq == 0) return HS_OK;  // nothing to read or write (pointers may be null)
  if (!q || !k || !v || !o || !scores) return HS_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return HS_ERR_INVALID_ARG;
  if (!is_pow2(sh.G) || sh.G > 128) return HS_ERR_UNSUPPORTED;
  if (vl->batch > attn::kMaxSched) return HS_ERR_UNSUPPORTED;
  if (sel->block == 1) return HS_ERR_UNSUPPORTED;
  const int T = sel->q_tile, B = sel->block;
  const int nblk = (sh.max_kv + B - 1) / B;
  // one CTA's spill (double-buffered, whole 128-key tiles); the fixed scratch
  // bounds the grid
  const size_t per_cta = spill_floats_per_cta(sh.max_kv, B) * sizeof(float);
  const size_t cap = (kNoAllocScratchBytes - kHeaderBytes) / per_cta;
  if (cap < 1) return HS_ERR_WORKSPACE;  // sequence longer than the fixed scratch can serve
  cudaStream_t s = S(stream);
  void* scratch = nullptr;
  if ((st = noalloc_scratch(&scratch)) != HS_OK) return st;
  // every call starts from a clear error header (stream-ordered), so a wait
  // that gave up in an earlier unchecked call is not reported by this one
  if (cudaMemsetAsync(scratch, 0, kHeaderBytes, s) != cudaSuccess) return HS_ERR_CUDA;
  const int n_tiles = n_tiles_of(vl, T);
  if (cudaMemsetAsync(scores, 0, size_t(n_tiles) * sh.Hkv * nblk * sizeof(float), s) != cudaSuccess)
    return HS_ERR_CUDA;
  Maps m;
  if (!make_map_3d(&m.q, q, sh.d, sh.Hq, sh.Tq, sh.G, 128 / sh.G) ||
      !make_map_3d(&m.k, k, sh.d, sh.Hkv, sh.Tkv, 1, 128) || !make_map_3d(&m.v, v, sh.d, sh.Hkv, sh.Tkv, 1, 128))
    return HS_ERR_CUDA;
  m.kb = m.k;
  m.vb = m.v;
  m.g = m.o = m.ks = m.vs = m.q;
  static attn::Sched sc;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (!fill_sched(vl, sh, attn::kFull, T, 1, &sc)) return HS_ERR_UNSUPPORTED;
  attn::Params p{};
  p.G = sh.G;
  p.Hq = sh.Hq;
  p.Hkv = sh.Hkv;
  p.Tq = int(sh.Tq);
  p.scale_log2 = sh.scale * 1.4426950408889634f;
  p.o = reinterpret_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.scores = scores;
  p.spill = reinterpret_cast<float*>(reinterpret_cast<char*>(scratch) + kHeaderBytes);
  p.spill_tiles = (sh.max_kv + 127) / 128;
  p.nblk = nblk;
  p.T = T;
  p.B = B;
  p.chunks_per_tile = 1;
  p.wc = WaitCtl{reinterpret_cast<ErrWord*>(scratch), g_timeout_ns};
  const int grid = int(std::min<size_t>(cap, size_t(std::min(num_sms(), std::max(1, sc.n_items)))));
  if ((st = dispatch_full(sh.d, B, m, p, sc, grid, s)) != HS_OK) return st;
  if (check) {
    if (cudaStreamSynchronize(s) != cudaSuccess) return HS_ERR_CUDA;
    ErrWord e{};
    if (cudaMemcpy(&e, scratch, sizeof(e), cudaMemcpyDeviceToHost) != cudaSuccess) return HS_ERR_CUDA;
    if (e.flag != 0) {
      last_err = e;
      return HS_ERR_TIMEOUT;
    }
  }
  return HS_OK;
}

hs_status hs_last_error_detail(int32_t* site, int32_t* block, int32_t* ctx) {
  if (!site || !block || !ctx) return HS_ERR_INVALID_ARG;
  *site = last_err.site;
  *block = last_err.block;
  *ctx = last_err.ctx;
  return HS_OK;
}

hs_status hs_debug_wait_timeout(void* ws, size_t ws_bytes, uint64_t timeout_ns, hs_stream_t stream) {
  if (!ws || ws_bytes < kHeaderBytes) return HS_ERR_WORKSPACE;
  if (timeout_ns == 0 || timeout_ns > 2000000000ull) return HS_ERR_INVALID_ARG;
  WaitCtl wc{reinterpret_cast<ErrWord*>(ws), timeout_ns};
  debug_wait_kernel<<<1, 32, 0, S(stream)>>>(wc);
  return cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}

hs_status hs_kv_dequantize(const void* codes, const float* scale, int64_t rows, int32_t head_dim, void* out,
                           hs_stream_t stream) {
  if (rows < 0 || head_dim <= 0 || head_dim % 16) return HS_ERR_INVALID_ARG;
  if (rows == 0) return HS_OK;
  if (!codes || !scale || !out || !aligned16(codes) || !aligned16(out) || (reinterpret_cast<uintptr_t>(scale) & 3))
    return HS_ERR_INVALID_ARG;
  const int cpr = head_dim / 16;
  const long long n = rows * cpr;
  const int grid = int(std::min<long long>(8LL * num_sms(), (n + 255) / 256));
  kv_dequant_kernel<<<grid, 256, 0, S(stream)>>>(reinterpret_cast<const uint4*>(codes), scale,
                                                 reinterpret_cast<uint4*>(out), rows, cpr);
  return cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}

hs_status hs_debug_exp2_poly(const float* x, float* y, int64_t n, hs_stream_t stream) {
  if (n < 0) return HS_ERR_INVALID_ARG;
  if (n == 0) return HS_OK;
  if (!x || !y || (reinterpret_cast<uintptr_t>(x) & 3) || (reinterpret_cast<uintptr_t>(y) & 3))
    return HS_ERR_INVALID_ARG;
  const long long pairs = (n + 1) / 2;
  const int grid = int(std::min<long long>(4LL * num_sms(), (pairs + 255) / 256));
  debug_exp2_poly_kernel<<<grid, 256, 0, S(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? HS_OK : HS_ERR_CUDA;
}

}  // extern "C"
