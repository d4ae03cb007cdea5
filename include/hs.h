/*
 * hs.h -- C ABI of libhs, the hybrid-block sparse attention hot path
 * (HySparse / HySparse2) for NVIDIA B200 (sm_100a).
 *
 * A hybrid block is one full causal attention layer followed by N sparse
 * attention layers that reuse the full layer's KV cache and its per-tile
 * top-k key selection (QbitAI repost of HySparse, "hybrid block" paragraphs;
 * HySparse2 release note on airebao.com, "KV Reuse").
 *
 * Conventions shared by every call
 * --------------------------------
 * Pointers: every tensor argument is a DEVICE pointer owned by the caller,
 *   except hs_varlen.cu_q_host / cu_kv_host, which are HOST pointers.
 *   The library never allocates or frees memory. Calls that need scratch take
 *   a caller-owned device workspace `ws` of at least hs_workspace_size(op, ...)
 *   bytes; call hs_workspace_init() once on a new workspace.
 * Streams: every call only enqueues work on `stream` and returns; nothing
 *   synchronises except hs_check_error().
 * Varlen packing: sequence b has n_b new queries and kv_b = c_b + n_b keys
 *   (c_b cached tokens; the new tokens' K/V are already appended). Query rows
 *   of all sequences are packed along one token axis with prefix sums cu_q;
 *   keys likewise with cu_kv. Query i of sequence b sits at position
 *   c_b + i of that sequence.
 * Layouts (row-major, token-major, contiguous):
 *   Q, O      [T_q,  H_q,  d]   bf16
 *   K, V      [T_kv, H_kv, d]   bf16 (or e4m3 bytes for FP8 decode)
 *   lse       [H_q, T_q]        fp32, natural log
 *   gamma     [T_q, H_q]        fp32
 *   scores    [n_tiles, H_kv, n_blk]  fp32, n_blk = ceil(max_kv / B)
 *   idx       [n_tiles, H_kv, k] int32 ascending, padded with -1
 *   cnt       [n_tiles, H_kv]   int32
 *   Query head h reads KV head h / (H_q / H_kv). Selection tile i of sequence
 *   b covers its new queries [i*T, min((i+1)*T, n_b)); tiles are numbered
 *   sequence after sequence; n_tiles = sum_b ceil(n_b / T).
 * Errors: each call validates its arguments on the host before launching
 *   anything and returns a status. Device-side failures (a bounded wait that
 *   gave up) are recorded in the workspace and reported by hs_check_error().
 * Limits: at most 256 sequences per call (batch <= 256); a larger batch is
 *   HS_ERR_UNSUPPORTED (split it into several calls). Per call the packed
 *   token axes hold at most 2^31 - 1 rows.
 * Devices: calls may target any device; each kernel's shared-memory limit is
 *   raised once per device it runs on. Calls on one device that share a
 *   workspace must be ordered (one stream, or events between streams).
 */
#ifndef HS_H_
#define HS_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HS_API __attribute__((visibility("default")))
#else
#define HS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* hs_stream_t; /* same object as cudaStream_t; NULL = legacy default stream */

typedef enum {
  HS_OK = 0,
  HS_ERR_INVALID_ARG = 1,  /* null pointer, bad size, inconsistent prefix sums */
  HS_ERR_UNSUPPORTED = 2,  /* valid but not implemented (e.g. head_dim not 64/128) */
  HS_ERR_WORKSPACE = 3,    /* workspace missing or smaller than hs_workspace_size() */
  HS_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed */
  HS_ERR_TIMEOUT = 5       /* a device-side bounded wait gave up (see hs_check_error) */
} hs_status;

typedef struct {
  int32_t batch;           /* number of sequences, >= 1 */
  int32_t n_q_heads;       /* H_q */
  int32_t n_kv_heads;      /* H_kv; H_q % H_kv == 0 */
  int32_t head_dim;        /* d: 64 or 128 */
  const int32_t* cu_q;     /* device [batch+1] prefix sums of n_b */
  const int32_t* cu_kv;    /* device [batch+1] prefix sums of kv_b */
  const int32_t* cu_q_host;  /* host copy of cu_q (same values) */
  const int32_t* cu_kv_host; /* host copy of cu_kv (same values) */
  float softmax_scale;     /* 0 => 1/sqrt(d) */
} hs_varlen;

typedef struct {
  int32_t q_tile;  /* T: queries per selection tile (1 for decode) */
  int32_t block;   /* B: keys per selectable block; 1 = token-level selection */
  int32_t topk;    /* k: blocks kept per (tile, KV head); 0 <= k <= 4096 */
  int32_t window;  /* w: forced recent window (tokens) unioned into the sparse set */
  int32_t flags;   /* 0, or HS_SEL_WINDOW_EXCLUSIVE (zero-initialise the struct) */
} hs_sel;

/* hs_sel.flags: which blocks compete for the top-k (used by hs_topk_select).
 * 0 (union reading): every causal block, b * B <= last query position of the
 *   tile; the forced window is then added per query and may overlap the kept
 *   blocks (HySparse2 release note on airebao.com: the latest tokens are
 *   forced into the selected set).
 * HS_SEL_WINDOW_EXCLUSIVE: only blocks that start before the forced window of
 *   the tile's last query, b * B <= last_pos - w, so the k kept blocks are
 *   "global" and the w recent tokens come on top (demingchina
 *   commentary on HySparse2, section 03: 1024 global tokens plus the latest
 *   128). Identical to the union reading when w = 0. The sparse-attention
 *   calls need no flag: their visible set is the same rule for both readings.
 * Other bits are HS_ERR_INVALID_ARG. */
#define HS_SEL_WINDOW_EXCLUSIVE 1

typedef enum { HS_KV_BF16 = 0, HS_KV_FP8_E4M3 = 1 } hs_kv_dtype;

typedef enum {
  HS_OP_FULL_ATTN_SELECT = 0,
  HS_OP_TOPK_SELECT = 1,
  HS_OP_SPARSE_ATTN_PREFILL = 2,
  HS_OP_SPARSE_ATTN_DECODE = 3,
  HS_OP_SWA_GATED = 4,
  HS_OP_SPARSE_SWA_GATED_PREFILL = 5
} hs_op;

/* Bytes of workspace that `op` needs for these shapes (0 on invalid input).
 * The first 256 bytes of every workspace hold the device error word. */
HS_API size_t hs_workspace_size(int op, const hs_varlen* vl, const hs_sel* sel);

/* Zero the workspace header (error word). Call once on a new workspace. */
HS_API hs_status hs_workspace_init(void* ws, size_t ws_bytes, hs_stream_t stream);

/* Synchronise `stream`, read and clear the workspace error word.
 * Returns HS_ERR_TIMEOUT if a kernel's bounded wait gave up since the last
 * check, HS_ERR_CUDA if the stream reports an error, else HS_OK. */
HS_API hs_status hs_check_error(void* ws, hs_stream_t stream);

/* Where the last failure seen by hs_check_error() happened: the wait site
 * code, the CTA index and a kernel-specific context word (work item << 12 |
 * pipeline step for the attention kernels). For diagnostics only. */
HS_API hs_status hs_last_error_detail(int32_t* site, int32_t* block, int32_t* ctx);

/* Static description of a status code. */
HS_API const char* hs_status_string(hs_status s);

/*
 * hs_full_attn_select -- the full attention layer of a hybrid block.
 *
 * Computes causal scaled dot-product attention (HySparse explainer on
 * techwalker.com: the master layer runs standard scaled dot-product
 * attention) and, as a by-product, the key-importance scores that drive the
 * selection (same page: a lightly modified FlashAttention kernel emits
 * block-level maximum attention scores reusing the online-softmax row max;
 * HySparse2 release note: top-k selection is a free by-product):
 *   s_{q,h,j} = (q_{q,h} . k_{j,g}) * scale,           j <= pos(q)
 *   o_{q,h}   = sum_j softmax_j(s) v_{j,g},   lse_{q,h} = ln sum_j exp(s)
 *   score(t, g, b) = max over q in tile t, h in group g, j in block b,
 *                    j <= pos(q), of exp(s_{q,h,j} - lse_{q,h}).
 * Blocks with b*B > last position of t are not candidates; their score is 0.
 * In:  q [T_q,H_q,d], k/v [T_kv,H_kv,d] bf16. Out: o bf16, lse fp32, scores fp32.
 * Supported: d in {64,128}; G = H_q/H_kv a power of two <= 128; B = 1 or a
 * power of two <= 128 (B = 1 adds a second QK pass for token-level scores).
 * Decode (n_b = 1 for every sequence, T = 1) is dispatched to a split-K path.
 * Errors: HS_ERR_INVALID_ARG / UNSUPPORTED / WORKSPACE before any launch.
 */
HS_API hs_status hs_full_attn_select(const hs_varlen* vl, const hs_sel* sel,
                              const void* q, const void* k, const void* v,
                              void* o, float* lse, float* scores,
                              void* ws, size_t ws_bytes, hs_stream_t stream);

/*
 * hs_topk_select -- keep the k best candidate blocks per (tile, KV head).
 *
 * HySparse explainer (techwalker.com): TopK over the block scores picks the
 * key blocks; HySparse2 release note and demingchina commentary section 03:
 * token-level selection of 1024 tokens. Candidates of tile t are blocks
 * b <= floor(last_pos(t) / B). Order: score descending, ties to the lower
 * index. Output idx ascending, padded with -1; cnt = min(k, #candidates).
 * With sel->flags = HS_SEL_WINDOW_EXCLUSIVE the candidates stop before the
 * forced window of the tile's last query: b * B <= last_pos(t) - w.
 * The forced recent window itself is not applied here: the sparse attention
 * calls union it per query.
 * In: scores [n_tiles,H_kv,n_blk] fp32 (>= 0). Out: idx [n_tiles,H_kv,k], cnt.
 */
HS_API hs_status hs_topk_select(const hs_varlen* vl, const hs_sel* sel, const float* scores,
                         int32_t* idx, int32_t* cnt,
                         void* ws, size_t ws_bytes, hs_stream_t stream);

/*
 * hs_full_attn_select_topk -- hs_full_attn_select followed by hs_topk_select,
 * with the top-k taken inside the score pass where the selection is token
 * level (HySparse2 release note on airebao.com: the top-k choice comes free
 * with the full layer).
 *
 * Outputs o, lse, idx and cnt are exactly those of the two calls in sequence
 * (same selection rule, ties and -1 padding). Token-level prefill (B = 1,
 * not the one-query decode shape): the CTA that finishes a (tile, KV head)'s
 * last score range queues it, and two selector warps of whichever CTA is
 * free select it while its scores are in L2, then drop those cache lines
 * without write-back; no separate top-k launch runs, and the scores reach
 * HBM only where a long context's K stream evicted them first. `scores` is
 * scratch of the usual [n_tiles, H_kv, n_blk] shape and
 * its content on return is undefined. The kernels wait across CTAs for
 * queued planes (bounded: an error, not a hang, if a plane never comes), so
 * they assume all CTAs of the launch are resident, as they are on an idle
 * GPU. HybridBlock keeps the two calls by default: on B200 the selection
 * beside the score pass costs more than the separate launch. Other shapes (block-level selection, decode) run the
 * two calls back to back and `scores` holds the scores as documented there.
 * In: as hs_full_attn_select (lse required at token level). Out: o, lse,
 * idx [n_tiles,H_kv,k], cnt [n_tiles,H_kv] (both required).
 * Workspace: hs_workspace_size(HS_OP_FULL_ATTN_SELECT, ...).
 * Errors: as hs_full_attn_select; HS_ERR_INVALID_ARG for null idx / cnt.
 */
HS_API hs_status hs_full_attn_select_topk(const hs_varlen* vl, const hs_sel* sel,
                                   const void* q, const void* k, const void* v,
                                   void* o, float* lse, float* scores,
                                   int32_t* idx, int32_t* cnt,
                                   void* ws, size_t ws_bytes, hs_stream_t stream);

/*
 * hs_sparse_attn_prefill -- one sparse layer of a hybrid block.
 *
 * This layer's own queries attend over the full layer's K/V (KV Reuse) at
 * the keys selected for their tile, plus the forced recent window
 * (QbitAI repost: block-sparse global branch over the TopK blocks of the
 * shared KV cache; HySparse2 release note: the latest 128 tokens are forced
 * into the selected set):
 *   V_q = { j in blocks(idx_t) : j <= pos(q) - w }  U  [max(0, pos(q)-w+1), pos(q)]
 *   o_{q,h} = sum_{j in V_q} softmax_j(s) v_{j,g};  lse as above.
 * An empty V_q (only possible with w = 0) yields o = 0 and lse = -inf.
 * In: q [T_q,H_q,d], k/v (full layer's) [T_kv,H_kv,d], idx/cnt from
 * hs_topk_select. Out: o bf16, lse fp32 (lse may be NULL).
 */
HS_API hs_status hs_sparse_attn_prefill(const hs_varlen* vl, const hs_sel* sel,
                                 const void* q, const void* k, const void* v,
                                 const int32_t* idx, const int32_t* cnt,
                                 void* o, float* lse,
                                 void* ws, size_t ws_bytes, hs_stream_t stream);

/*
 * hs_gather_selected_kv -- token-level selection (sel->block = 1): copy the
 * selected tokens' K and V rows of every (selection tile, KV head) into
 * contiguous buffers, once per hybrid block. All sparse layers of a block
 * reuse the full layer's cache and its selected tokens (KV Reuse: QbitAI
 * repost; HySparse2 release note), so the gather is paid once and every
 * sparse prefill layer then reads whole 128-slot tiles
 * (hs_sparse_attn_prefill_gathered).
 *   kg[tile][g][s] = k[cu_kv[b(tile)] + idx[tile][g][s]][g]   for s < cnt[tile][g]
 *   kg[tile][g][s] = 0                                          for cnt <= s < topk
 * and the same for vg from v (b(tile): the tile's sequence).
 * In: k/v [T_kv, H_kv, d] bf16; idx/cnt from hs_topk_select for the same
 * (vl, sel). Out: kg/vg [n_tiles, H_kv, topk, d] bf16, n_tiles = sum over
 * sequences of ceil(n_b / q_tile) (device, caller-owned, 16-byte aligned, not
 * overlapping the inputs). topk = 0 or T_q = 0 is a no-op; block != 1, null or
 * misaligned pointers are HS_ERR_INVALID_ARG.
 */
HS_API hs_status hs_gather_selected_kv(const hs_varlen* vl, const hs_sel* sel,
                                const void* k, const void* v,
                                const int32_t* idx, const int32_t* cnt,
                                void* kg, void* vg, hs_stream_t stream);

/*
 * hs_sparse_attn_prefill_gathered -- hs_sparse_attn_prefill for token-level
 * selection (sel->block = 1) reading the selected tokens from kg/vg, filled
 * by hs_gather_selected_kv for the same (vl, sel, idx, cnt); k and v are still
 * read for the forced window and idx for the visibility mask. Same V_q, same
 * arithmetic in the same order as hs_sparse_attn_prefill, so o and lse are
 * identical. Argument rules as hs_sparse_attn_prefill, plus kg/vg non-null
 * and 16-byte aligned.
 */
HS_API hs_status hs_sparse_attn_prefill_gathered(const hs_varlen* vl, const hs_sel* sel,
                                 const void* q, const void* k, const void* v,
                                 const void* kg, const void* vg,
                                 const int32_t* idx, const int32_t* cnt,
                                 void* o, float* lse,
                                 void* ws, size_t ws_bytes, hs_stream_t stream);

/*
 * hs_sparse_attn_decode -- sparse layer for one new token per sequence.
 *
 * Same set V_q as the prefill call with T = 1, computed split-K over the
 * selected keys and merged by their log-sum-exp. The KV cache may be bf16 or
 * FP8 e4m3 (the HySparse2 key-data table sizes an FP8 KV cache); FP8 values
 * decode as x = scale[token, kv_head] * e4m3(code), with separate fp32 scale
 * arrays for K and V ([T_kv, H_kv]; NULL for bf16).
 * The slots of each (sequence, KV head) -- the window, then the tokens of
 * the selected blocks (block B = sel->block: token-level selection with B = 1;
 * HySparse's 64-token blocks with B = 64) -- form ceil((k B + w) / 128) tiles
 * of 128 keys, cut into split_k
 * contiguous ranges of whole tiles, one tensor-core work item each; the
 * ranges of a unit run as one thread-block cluster and their partial results
 * are merged by log-sum-exp through the cluster's shared memory, inside the
 * same launch (the workspace holds only the error header).
 * split_k: 0 = automatic (about one range per SM over all units); a value
 * above the tile count or above 8 (the portable cluster size) is clamped;
 * negative values are rejected.
 * An empty batch (T_q = 0) returns HS_OK without touching any pointer.
 * Requires n_b = 1 for every sequence and sel->q_tile = 1 (any block).
 */
HS_API hs_status hs_sparse_attn_decode(const hs_varlen* vl, const hs_sel* sel,
                                const void* q, hs_kv_dtype kv_dtype,
                                const void* k, const void* v,
                                const float* k_scale, const float* v_scale,
                                const int32_t* idx, const int32_t* cnt, int32_t split_k,
                                void* o, float* lse,
                                void* ws, size_t ws_bytes, hs_stream_t stream);

/*
 * hs_swa_gated -- HySparse's local branch and the gate that fuses it.
 *
 * The sliding-window branch uses the same queries over the layer's OWN small
 * KV cache (QbitAI repost: window of 128 by default; HySparse explainer: the
 * window branch must not share the full layer's KV), keys
 * [max(0, pos(q)-window+1), pos(q)], and the two branch outputs are fused by
 * a sigmoid gate (both pages). Reading of the gate:
 *   o = sigmoid(gamma) * o_sparse + (1 - sigmoid(gamma)) * o_swa,
 * gamma given per (token, query head).
 * In: q [T_q,H_q,d], k_swa/v_swa [T_kv,H_kv,d] bf16, gamma [T_q,H_q] fp32,
 * o_sparse [T_q,H_q,d] bf16. Out: o [T_q,H_q,d] bf16 (may alias o_sparse).
 */
HS_API hs_status hs_swa_gated(const hs_varlen* vl, int32_t window,
                       const void* q, const void* k_swa, const void* v_swa,
                       const float* gamma, const void* o_sparse, void* o,
                       void* ws, size_t ws_bytes, hs_stream_t stream);

/*
 * hs_sparse_swa_gated_prefill -- a whole HySparse sparse layer in one launch:
 * the block-sparse global branch of hs_sparse_attn_prefill, the sliding-window
 * branch of hs_swa_gated over the layer's own K_swa / V_swa, and the sigmoid
 * gate (QbitAI repost: each sparse layer has the two branches, fused by a
 * sigmoid gate; HySparse explainer: the window branch keeps its own cache):
 *   o = sigmoid(gamma) * o_sparse + (1 - sigmoid(gamma)) * o_swa.
 * Results equal hs_sparse_attn_prefill followed by hs_swa_gated, except that
 * the gate mixes the fp32 window output with o_sparse rounded to bf16 once
 * (as the two-call path does) without o_sparse passing through HBM.
 * In: q [T_q,H_q,d]; k/v (full layer's) [T_kv,H_kv,d]; idx/cnt from
 * hs_topk_select; swa_window >= 1; k_swa/v_swa [T_kv,H_kv,d] bf16;
 * gamma [T_q,H_q] fp32.
 * Out: o [T_q,H_q,d] bf16; o_sparse [T_q,H_q,d] bf16 and lse_sparse [H_q,T_q]
 * fp32 of the sparse branch, each optional (NULL skips the write).
 */
HS_API hs_status hs_sparse_swa_gated_prefill(const hs_varlen* vl, const hs_sel* sel,
                                      const void* q, const void* k, const void* v,
                                      const int32_t* idx, const int32_t* cnt,
                                      int32_t swa_window, const void* k_swa, const void* v_swa,
                                      const float* gamma, void* o, void* o_sparse, float* lse_sparse,
                                      void* ws, size_t ws_bytes, hs_stream_t stream);

/*
 * hs_kv_dequantize -- expand an FP8-e4m3 KV cache to bf16 for the prefill
 * calls of a block (the HySparse2 key-data table on airebao.com sizes an FP8
 * KV cache; the block's full layer and its sparse layers all read that one
 * cache, KV Reuse).
 *   out[r][i] = bf16_rn(scale[r] * e4m3(codes[r][i])),  r < rows, i < head_dim
 * with one fp32 scale per (token, KV head) row (rows = T_kv * H_kv; the
 * product is formed in fp32). Prefill attention is bound by the tensor cores,
 * so one pass over the cache (1 + 2 bytes per element) per block, shared by
 * the full layer and every sparse layer, stands in for expanding the codes
 * inside each attention kernel; decode reads the codes directly
 * (hs_sparse_attn_decode with HS_KV_FP8_E4M3).
 * In: codes [rows, head_dim] uint8, scale [rows] fp32. Out: out [rows, head_dim]
 * bf16 (device, caller-owned, must not overlap the inputs). head_dim a
 * multiple of 16; pointers 16-byte aligned (scale 4-byte). rows = 0 is a
 * no-op; negative sizes, null or misaligned pointers are HS_ERR_INVALID_ARG.
 */
/*
 * hs_swa_ring_write -- keep a layer's own sliding-window K/V cache as a ring
 * buffer (the SWA branch of HySparse reads only the last `window` positions
 * of its own small cache: QbitAI repost, two-branch paragraph; techwalker.com
 * explainer, the window branch must not share the full layer's KV).
 *   k_ring[b][p mod R][g] = k_new[row of the new token of sequence b at position p][g]
 * for the new tokens of each sequence (positions kv_b - n_b .. kv_b - 1) that
 * are among its last R positions; the same for v. R = ring_len >= the window.
 * In: k_new / v_new [T_q, H_kv, d] bf16 (rows in cu_q order). Out (device,
 * caller-owned, updated in place): k_ring / v_ring [batch, R, H_kv, d] bf16.
 * Pointers 16-byte aligned. T_q = 0 is a no-op; ring_len < 1, null or
 * misaligned pointers are HS_ERR_INVALID_ARG.
 */
HS_API hs_status hs_swa_ring_write(const hs_varlen* vl, int32_t ring_len,
                                   const void* k_new, const void* v_new,
                                   void* k_ring, void* v_ring, hs_stream_t stream);

/*
 * hs_swa_gated_decode -- the HySparse sliding-window branch and its gate for
 * one new token per sequence, over the layer's own K/V in a ring (written by
 * hs_swa_ring_write, the new token's row included):
 *   o_swa[b, h] = sum_{p = max(0, pos - window + 1)}^{pos} softmax_p(s) v_ring[b][p mod R][g(h)]
 *   o[b, h]     = sig(gamma[b, h]) o_sparse[b, h] + (1 - sig(gamma[b, h])) o_swa[b, h]
 * with pos = kv_b - 1 and the same scale as the other calls (the gate as in
 * hs_swa_gated). In: q [batch, H_q, d] bf16, gamma [batch, H_q] fp32,
 * o_sparse [batch, H_q, d] bf16 (the sparse decode layer's output). Out: o
 * [batch, H_q, d] bf16. Requires one new token per sequence (kv_b >= 1),
 * 1 <= window <= ring_len; window <= 128 and G <= 64 (else
 * HS_ERR_UNSUPPORTED). Null or misaligned pointers are HS_ERR_INVALID_ARG.
 */
HS_API hs_status hs_swa_gated_decode(const hs_varlen* vl, int32_t window, int32_t ring_len,
                                     const void* q, const void* k_ring, const void* v_ring,
                                     const float* gamma, const void* o_sparse, void* o,
                                     hs_stream_t stream);

HS_API hs_status hs_kv_dequantize(const void* codes, const float* scale, int64_t rows, int32_t head_dim,
                                  void* out, hs_stream_t stream);

/*
 * hs_full_attn_select_noalloc -- hs_full_attn_select for callers that cannot
 * allocate device memory. The pages have no counterpart to this entry point.
 *
 * Who needs it: code that runs where cudaMalloc (or a caching allocator such
 * as torch's) is unavailable or forbidden -- e.g. a plugin inside another
 * runtime that owns all device memory, or a latency-critical path that must
 * not allocate (cudaMalloc can synchronise the device). Such callers cannot
 * provide the workspace that hs_full_attn_select needs for its block-maximum
 * spill, so this variant uses a fixed array inside the library instead.
 *
 * Scratch: a file-scope device array of 64 MiB, resident on every GPU that
 * loads the library until the process exits. The caller still passes inputs
 * and outputs exactly as for hs_full_attn_select. No call allocates or frees
 * memory (no cudaMalloc/cudaFree or allocating library routine).
 * First call per device: looks up the array's device address with the device
 * current (cudaGetSymbolAddress) and caches it; make that first call before
 * any stream capture on that device.
 * Every call first zeroes the array's 256-byte error header with an async
 * memset on `stream`, so a bounded wait that gave up during an earlier call
 * made with check = 0 is never reported by a later call; such a failure is
 * visible only to a check != 0 call on the same launch.
 * Sharing: every call on a device uses the same array and leaves its contents
 * behind. Calls whose kernels overlap on the GPU (e.g. on two streams without
 * ordering) race on it and give wrong results; order them.
 * Limits: block-level selection only (B >= 8). A CTA's share is
 * 2 * ceil(max_kv / 128) * (128 / B) KB (whole 128-key tiles); the grid is
 * capped so that grid shares fit in the array; if a single share does not
 * fit -- more than ~32767 blocks, i.e. max_kv above ~2.1M tokens at B = 64 --
 * the call returns HS_ERR_WORKSPACE before launching. Smaller caps only mean
 * fewer CTAs, not different results.
 * check != 0: synchronise `stream` after the launch and return HS_ERR_TIMEOUT
 * if a device-side bounded wait gave up (details via hs_last_error_detail).
 */
HS_API hs_status hs_full_attn_select_noalloc(const hs_varlen* vl, const hs_sel* sel,
                                             const void* q, const void* k, const void* v,
                                             void* o, float* lse, float* scores,
                                             int32_t check, hs_stream_t stream);

/*
 * hs_debug_wait_timeout -- failure-detection self test (no counterpart on the
 * pages). Launches one tiny kernel that waits on a barrier nothing arrives
 * at; its bounded wait gives up after `timeout_ns` (1 .. 2e9), records the
 * failure in the workspace error word and returns, leaving the context
 * usable. hs_check_error() then reports HS_ERR_TIMEOUT and clears the word.
 * This is the same bounded wait every pipelined kernel uses.
 */
HS_API hs_status hs_debug_wait_timeout(void* ws, size_t ws_bytes, uint64_t timeout_ns, hs_stream_t stream);

/*
 * hs_debug_exp2_poly -- self test of the softmax's FMA-pipe exponential (no
 * counterpart on the pages). Writes y[i] = 2^x[i] as the attention kernels
 * compute one in four of their exponentials: a Cody-Waite split 2^x = 2^j * 2^f
 * (j = nearest integer, |f| <= 1/2) with a degree-3 minimax polynomial for
 * 2^f (relative error 7.5e-5), inputs clamped to >= -125 (so x < -125 gives
 * about 2^-125). x, y: device arrays of n fp32 values (4-byte aligned); n = 0
 * is a no-op; n < 0 or a null / misaligned pointer is HS_ERR_INVALID_ARG.
 */
HS_API hs_status hs_debug_exp2_poly(const float* x, float* y, int64_t n, hs_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HS_H_ */
