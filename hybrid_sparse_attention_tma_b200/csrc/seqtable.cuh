// seqtable.cuh -- varlen bookkeeping passed to kernels by value (host copy of
// the prefix sums), so a CTA can map a selection tile back to its sequence.
#pragma once

namespace hs {

constexpr int kMaxSeq = 256;

struct SeqTable {
  int batch;
  int n_tiles;
  int T;
  int cu_q[kMaxSeq + 1];
  int cu_kv[kMaxSeq + 1];
  int tile_base[kMaxSeq + 1];  // prefix of ceil(n_b / T)
};

struct TileInfo {
  int seq;
  int pos0;      // position of the tile's first query
  int n;         // queries in the tile
  int kv0;       // first packed key row of the sequence
  int kv_len;
  int qrow0;     // first packed query row
};

__device__ __forceinline__ TileInfo tile_info(const SeqTable& st, int tile) {
  int lo = 0, hi = st.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (st.tile_base[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  TileInfo ti;
  const int b = lo;
  const int n_b = st.cu_q[b + 1] - st.cu_q[b];
  const int kv_b = st.cu_kv[b + 1] - st.cu_kv[b];
  const int i = tile - st.tile_base[b];
  ti.seq = b;
  ti.pos0 = kv_b - n_b + i * st.T;
  ti.n = min(st.T, n_b - i * st.T);
  ti.kv0 = st.cu_kv[b];
  ti.kv_len = kv_b;
  ti.qrow0 = st.cu_q[b] + i * st.T;
  return ti;
}

}  // namespace hs
