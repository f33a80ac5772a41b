/*
 * fbk.h - C ABI of the cached block attention library (libfbk.so).
 *
 * One attention layer of one denoising step of block (semi-autoregressive)
 * diffusion decoding. The current block of B query tokens of sequence b sits
 * at absolute positions L_b .. L_b+B-1, after a cached prefix of L_b tokens
 * (LaCache, "Exact Caching and Precision-Adaptive Inference for Diffusion Large
 * Language Models", §3.3.1 Notation, App. B.1). The block attends
 * bidirectionally to the prefix and to itself. The prefix contribution is kept
 * as the FlashAttention online-softmax state (O~, m, l) of LaCache §3.3.3
 * (FACache, Eq. 2-6), computed once per block and reused at every denoising
 * step of the block (FlashBlock, "Attention Caching for Efficient Long-Context
 * Block Diffusion", Abstract), where it is merged by log-sum-exp with a fresh
 * in-block state. When the block is final, its K is rotated (RoPE) and K/V are
 * appended to the cache (LaCache §3.3.2 RoPECache, Eq. 1).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Memory. Every pointer argument is DEVICE memory owned by the caller,
 *    except the structs themselves (fbk_shape, fbk_kv_cache, fbk_partial,
 *    fbk_layer_block), which are host structs read during the call only. The library allocates
 *    nothing and never synchronises. Apart from fbk_prefix_partial_static_scratch
 *    (last below), it keeps no state between calls.
 *  - Streams. `cuda_stream` is a cudaStream_t (NULL = legacy default stream).
 *    Every call only enqueues work on it and returns.
 *  - Errors. Argument errors are detected on the host and returned before any
 *    launch. A launch failure returns FBK_ERR_CUDA. Conditions that depend on
 *    device-resident values (prefix lengths, page ids) are checked on the
 *    device: the offending sequence is skipped and a bit is OR-ed into
 *    cache->error_flags (FBK_DEVERR_*), when that pointer is not NULL.
 *  - Types. bf16 is IEEE bfloat16 (uint16 storage). fp32 state is IEEE float.
 *  - Element order. Row-major; the last index is contiguous.
 *
 * Notation: b batch, Hq query heads, Hkv kv-heads (G = Hq/Hkv query heads per
 * kv-head, head h reads kv-head floor(h*Hkv/Hq)), d head_dim, B block_len,
 * L_b prefix length of sequence b, tau softmax scale.
 */
#ifndef FBK_H_
#define FBK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fbk_status {
  FBK_OK = 0,
  FBK_ERR_INVALID_ARG = -1,  /* NULL pointer, non-positive size, bad struct field */
  FBK_ERR_UNSUPPORTED = -2,  /* d not in {64,128}, Hq % Hkv != 0, G*B > 256, B > 64, b > 1024 ... */
  FBK_ERR_CAPACITY = -3,     /* cache geometry cannot hold the request */
  FBK_ERR_WORKSPACE = -4,    /* workspace NULL or smaller than fbk_prefix_workspace_bytes */
  FBK_ERR_CUDA = -5,         /* a CUDA runtime call or launch failed */
  FBK_ERR_SCRATCH_LIMIT = -6 /* fbk_prefix_partial_static_scratch: the call needs more than
                                FBK_STATIC_SCRATCH_BYTES of scratch */
} fbk_status;

/* Arithmetic of a call.
 *  FBK_BF16: production path. Block Q and the prefix P~ enter the tensor-core
 *    products as bf16 (fp32 accumulation); the output O is bf16.
 *  FBK_FP32_CHECK: the same operations on CUDA cores in fp32 from the same
 *    bf16 inputs (no bf16 rounding of Q^ or P~); the output O is fp32. */
typedef enum fbk_mode { FBK_BF16 = 0, FBK_FP32_CHECK = 1 } fbk_mode;

/* Device error bits OR-ed into fbk_kv_cache.error_flags. */
#define FBK_DEVERR_PREFIX_LEN 1u /* prefix_lens[b] < 0 or beyond the cache capacity: b skipped */
#define FBK_DEVERR_PAGE_ID 2u    /* a page-table entry outside [0, num_pages) was needed */
#define FBK_DEVERR_COMMIT 4u     /* commit would write past the capacity: block not appended */
#define FBK_DEVERR_TIMEOUT 8u    /* a bounded device-side wait gave up (kernel returned early) */

typedef struct fbk_shape {
  int32_t batch;       /* 1 <= b <= 1024 */
  int32_t n_q_heads;   /* Hq >= 1 */
  int32_t n_kv_heads;  /* Hkv >= 1, Hq % Hkv == 0 */
  int32_t head_dim;    /* d in {64, 128} */
  int32_t block_len;   /* B in [1, 64]; G*B <= 256 */
  float softmax_scale; /* tau > 0: scores are tau * <RoPE(q), k> (the pages write S = Q K^T: tau = 1) */
  double rope_base;    /* theta_i = rope_base^(-2i/d), rotate-half pairs (i, i + d/2) */
  int32_t mode;        /* fbk_mode */
} fbk_shape;

/* The KV cache: post-RoPE K and V of every committed token (RoPECache).
 * Contiguous: k, v are bf16 [b, Hkv, capacity_tokens, d]; token p of sequence
 *   b, kv-head g is row (b*Hkv + g)*capacity_tokens + p.
 * Paged (paged != 0): k, v are bf16 [num_pages, Hkv, page_size, d]; token p of
 *   sequence b lives in page page_table[b*max_pages_per_seq + p/page_size] at
 *   offset p % page_size. page_size is a power of two >= 16.
 * prefix_lens: int32 [b], the committed length L_b of each sequence. It is
 *   read by every call and advanced by B by fbk_commit_block_rope_append.
 * error_flags: int32 [1] or NULL; FBK_DEVERR_* bits are OR-ed in, never cleared. */
typedef struct fbk_kv_cache {
  void *k;
  void *v;
  int32_t paged;
  int32_t page_size;
  int32_t max_pages_per_seq;
  int64_t capacity_tokens; /* contiguous layout only */
  int64_t num_pages;       /* paged layout only */
  const int32_t *page_table;
  int32_t *prefix_lens;
  int32_t *error_flags;
} fbk_kv_cache;

/* An online-softmax state per (sequence, query head, block row), LaCache §3.3.3:
 * o_unnorm = O~ fp32 [b, Hq, B, d]; m fp32 [b, Hq, B] (the running max of the
 * scaled scores, natural-log units); l fp32 [b, Hq, B] (sum of exp(s - m)).
 * O~ and l are relative to that m. A row with no keys holds (0, -inf, 0). */
typedef struct fbk_partial {
  float *o_unnorm;
  float *m;
  float *l;
} fbk_partial;

/* Bytes of scratch fbk_prefix_partial needs for `num_splits` work shares
 * (0 = one share per SM of the current device): (shares + b*Hkv) * G*B * (d+2)
 * fp32 for the per-share states plus b*Hkv * 128*ceil(G*B/128) * d bf16 for the
 * rotated query rows, each region rounded up to 256 bytes. Depends only on b,
 * Hkv, G*B, d and the share count, not on the prefix lengths. Returns 0 for an
 * invalid shape; B up to 256 is valid here (fbk_prefix_partial_at's blocks). */
size_t fbk_prefix_workspace_bytes(const fbk_shape *shape, const fbk_kv_cache *cache,
                                  int32_t num_splits);

/* The share count that num_splits = 0 selects on the current device. */
int32_t fbk_default_num_splits(void);

/* Prefix state of the block queries over the cached prefix (FACache's cached
 * state, LaCache §3.3.3, Eq. 2-6, restricted to keys 0..L_b-1; FlashBlock's
 * cached block-external attention).
 *  q_blk: bf16 [b, B, Hq, d], PRE-RoPE; row t of sequence b is rotated at
 *         position prefix_lens[b] + t inside the kernel.
 *  out:   the state, written in full (every row of every head); o_unnorm
 *         16-byte aligned (FBK_ERR_UNSUPPORTED otherwise), like q_blk.
 *  ws:    device scratch of at least fbk_prefix_workspace_bytes(...) bytes,
 *         256-byte aligned (FBK_ERR_UNSUPPORTED otherwise), caller-owned,
 *         contents irrelevant on entry. It holds the per-share states and the
 *         RoPE-rotated block queries that the tensor-core kernel reads by TMA.
 *  num_splits: number of equal shares of the flattened (sequence, kv-head,
 *         64-key tile) work list, one CTA each (0 = one per SM).
 * Launches (FBK_BF16): the query rotation into ws, the tensor-core share
 * kernel, then a fixed-order LSE reduction of the per-share states
 * (deterministic run to run). FBK_FP32_CHECK: the fp32 share kernel (which
 * rotates the queries itself) and the same reduction. */
fbk_status fbk_prefix_partial(const fbk_shape *shape, const void *q_blk, const fbk_kv_cache *cache,
                              const fbk_partial *out, void *ws, size_t ws_bytes,
                              int32_t num_splits, void *cuda_stream);

/* One denoising step: in-block bidirectional attention (no mask) of the block
 * queries over the block keys, LSE-merged with the cached prefix state and
 * normalised: O = (e^(m1-m) O~1 + e^(m2-m) O~2) / (e^(m1-m) l1 + e^(m2-m) l2),
 * m = max(m1, m2), lse = m + log l (LaCache App. J, initialise with cache,
 * final normalisation and logsumexp).
 *  q_blk: bf16 [b, B, Hq, d] pre-RoPE; k_blk, v_blk: bf16 [b, B, Hkv, d], K pre-RoPE.
 *  prefix_lens: int32 [b] device (positions are prefix_lens[b] + t). In
 *         FBK_BF16 mode the in-block scores depend on positions only through
 *         their differences (RoPE), so the kernel rotates at t and does not
 *         read prefix_lens; FBK_FP32_CHECK rotates at prefix_lens[b] + t.
 *  prefix: a state from fbk_prefix_partial (read only).
 *  out: [b, B, Hq, d], bf16 (FBK_BF16) or fp32 (FBK_FP32_CHECK).
 *  lse: fp32 [b, Hq, B] or NULL. */
fbk_status fbk_block_attn_merge(const fbk_shape *shape, const void *q_blk, const void *k_blk,
                                const void *v_blk, const int32_t *prefix_lens,
                                const fbk_partial *prefix, void *out, float *lse,
                                void *cuda_stream);

/* Commit a finished block: K^ = RoPE(k_blk, L_b + t) computed in fp64 and
 * rounded once to bf16 (nearest even), V copied bit for bit, both written to
 * cache slots L_b .. L_b+B-1; then prefix_lens[b] += B (RoPECache,
 * LaCache §3.3.2, Eq. 1). A sequence whose block does not fit is left
 * unchanged and FBK_DEVERR_COMMIT is flagged. Two launches: the rows (one
 * CTA per sequence, block token and group of up to 16 kv-heads), then the
 * length update. */
fbk_status fbk_commit_block_rope_append(const fbk_shape *shape, const void *k_blk,
                                        const void *v_blk, fbk_kv_cache *cache,
                                        void *cuda_stream);

/* Uncached reference: softmax attention of the block queries over
 * [prefix keys 0..L_b-1 ; RoPE(k_blk)] in one fp32 pass on CUDA cores, with
 * no cached state (the computation FACache must reproduce exactly, LaCache
 * §3.1). Independent device code, used as a GPU cross-check. Output as in
 * fbk_block_attn_merge. */
fbk_status fbk_full_ref_attn(const fbk_shape *shape, const void *q_blk, const void *k_blk,
                             const void *v_blk, const fbk_kv_cache *cache, void *out,
                             float *lse, void *cuda_stream);

/* fbk_prefix_partial with the block's query rows rotated at q_pos[b] + t
 * instead of prefix_lens[b] + t (q_pos: int32 [b] on the device, required).
 * The cached keys are still rows 0 .. prefix_lens[b]-1 of the cache, stored
 * after RoPE at whatever positions they hold. This lets the block's rows meet
 * keys that lie after the block, such as a masked suffix in full-sequence
 * decoding (LaCache §3.3.1: U holds the prompt and the masked suffix). It also
 * lets any run of rows with consecutive positions stand in as the "block",
 * for instance a chunk of U's rows when FACache's cached state of U over U's
 * keys is computed (LaCache §3.3.3). The block length may exceed 64 here: B is
 * limited only by G*B <= 256. Otherwise as fbk_prefix_partial. */
fbk_status fbk_prefix_partial_at(const fbk_shape *shape, const void *q_blk, const int32_t *q_pos,
                                 const fbk_kv_cache *cache, const fbk_partial *out, void *ws, size_t ws_bytes,
                                 int32_t num_splits, void *cuda_stream);

/* Size of the library's built-in scratch array (per device) used by
 * fbk_prefix_partial_static_scratch: 32 MiB. */
#define FBK_STATIC_SCRATCH_BYTES (32u << 20)

/* fbk_prefix_partial without a caller-supplied workspace. The pages have no
 * counterpart to this call: it is an interface convenience only, and it
 * computes exactly what fbk_prefix_partial computes, with the same kernels
 * and the same results.
 *
 * Who it is for. Some callers cannot hand over scratch memory. Examples are a
 * plain C host with no device allocator of its own, or a plug-in inside another
 * runtime whose memory pool owns the device and forbids outside allocations.
 * Another is code that must not call cudaMalloc/cudaFree, because those
 * calls can synchronise the device and stall other streams. This entry point
 * allocates nothing either: its scratch is a fixed array of
 * FBK_STATIC_SCRATCH_BYTES bytes in the library's own device image, one per
 * device, created when the CUDA module is loaded.
 *
 * Footprint. The array lives in a device module of its own (it holds no
 * kernel), and a device that loads that module holds the 32 MiB until the
 * process exits. With lazy module loading (the CUDA default,
 * CUDA_MODULE_LOADING=LAZY) only the address lookup of this entry point's
 * first call loads it, so a process that never calls it pays nothing; with
 * CUDA_MODULE_LOADING=EAGER every device the process initialises pays it when
 * the library loads, whether or not this entry point is ever called.
 *
 * Arguments are those of fbk_prefix_partial minus ws and ws_bytes.
 *
 * Set-up. The first call on each device looks up the array's address with
 * cudaGetSymbolAddress, with that device current, and caches it for the rest of
 * the process. Make that first call before any stream capture begins on that
 * device. The cached address does not survive cudaDeviceReset.
 *
 * Limit. A call whose workspace, fbk_prefix_workspace_bytes(shape, cache,
 * num_splits), exceeds FBK_STATIC_SCRATCH_BYTES returns FBK_ERR_SCRATCH_LIMIT
 * before any launch. Lower num_splits, or use fbk_prefix_partial.
 *
 * Zeroing. No part of the array has to start at zero. Every scratch slot the
 * reduction reads is written by the share kernel of the same call.
 *
 * Concurrency. There is one array per device, shared by every caller. Calls
 * that overlap on one device race on it and corrupt each other's results:
 * calls from different streams or host threads must be ordered (one stream, or
 * events).
 *
 * Errors are otherwise those of fbk_prefix_partial. */
fbk_status fbk_prefix_partial_static_scratch(const fbk_shape *shape, const void *q_blk,
                                             const fbk_kv_cache *cache, const fbk_partial *out,
                                             int32_t num_splits, void *cuda_stream);

/* One layer's buffers for fbk_decode_block. The inputs of every denoising
 * step of the block are stored step-major: step s of q starts s*b*B*Hq*d
 * elements after q, step s of k and v s*b*B*Hkv*d elements after k and v. */
typedef struct fbk_layer_block {
  const void *q;            /* bf16 [steps, b, B, Hq, d], pre-RoPE block queries, 16-byte aligned */
  const void *k;            /* bf16 [steps, b, B, Hkv, d], pre-RoPE block keys, 16-byte aligned */
  const void *v;            /* bf16 [steps, b, B, Hkv, d], block values, 16-byte aligned */
  fbk_kv_cache cache;       /* this layer's cache and prefix lengths */
  fbk_partial prefix;       /* this layer's prefix state (rewritten at every refresh) */
  void *out;                /* [steps, b, B, Hq, d]: bf16 (FBK_BF16) or fp32 (FBK_FP32_CHECK) */
  float *lse;               /* fp32 [steps, b, Hq, B], or NULL */
  int32_t refresh_interval; /* r >= 1, see fbk_decode_block */
} fbk_layer_block;

/* Every denoising step of one block for n_layers attention layers, in one
 * call, with a cache update interval per layer (LaCache App. C: the longer
 * the interval, the faster the decoding and the larger the error).
 *
 * For step s = 0 .. steps-1, and within a step for layer l = 0 .. n_layers-1:
 *   if s % r_l == 0, the layer's prefix state is recomputed from step s's block
 *   queries (the launches of fbk_prefix_partial, same workspace rules);
 *   then the step output of layer l (fbk_block_attn_merge), into out[s] and lse[s].
 * Then, if commit != 0, each layer commits the K and V of the last step
 * (fbk_commit_block_rope_append), which advances its prefix_lens by B.
 *
 * r_l = 1 is the recompute-every-step schedule: every step is exact full
 * attention over prefix and block. r_l >= steps computes the state once per
 * block from step 0's queries (FlashBlock's reuse of the block-external
 * attention). Intervals may differ between layers, for instance to refresh
 * deeper layers more often.
 *
 *  layers: host array of n_layers structs, read during the call only.
 *  ws, ws_bytes, num_splits: as for fbk_prefix_partial; one workspace serves
 *         every layer, since all launches are ordered on the one stream.
 *  commit: with commit != 0 no two layers may share a prefix_lens array
 *         (FBK_ERR_INVALID_ARG), since each layer's commit advances its own.
 *
 * Every argument of every layer is checked before the first launch, with
 * the codes of the single calls. If a launch fails, FBK_ERR_CUDA is returned
 * and the launches before it stay enqueued. Like every call here, this one
 * only enqueues work, so a whole block can be captured as one CUDA graph. The
 * pages have no counterpart to the call itself: it is the loop over steps and
 * layers that a decoder runs, moved into the library so that the launches are
 * issued from native code. */
fbk_status fbk_decode_block(const fbk_shape *shape, const fbk_layer_block *layers, int32_t n_layers,
                            int32_t steps, int32_t commit, void *ws, size_t ws_bytes,
                            int32_t num_splits, void *cuda_stream);

/* Scratch and outputs of fbk_decode_block_adaptive, all device memory owned
 * by the caller; the call initialises every array itself.
 *  threshold:    theta >= 0 (may be +inf; FBK_ERR_INVALID_ARG for NaN or < 0).
 *  flags:        int32 [2, n_layers] scratch: refresh requests for the even
 *                and the odd steps.
 *  last_refresh: int32 [n_layers] scratch: each layer's last refresh step.
 *  drift:        fp32 [steps, n_layers] out: delta_s of every layer-step (the
 *                last step's row is 0: it decides nothing).
 *  refreshed:    int32 [steps, n_layers] out: 1 where the layer recomputed its
 *                prefix state at that step. */
typedef struct fbk_drift_policy {
  float threshold;
  int32_t *flags;
  int32_t *last_refresh;
  float *drift;
  int32_t *refreshed;
} fbk_drift_policy;

/* fbk_decode_block with an adaptive, depth-aware refresh in place of the
 * fixed intervals (Elastic-Cache, Abstract: an attention-aware drift test
 * decides when to refresh, and the refresh recomputes from the triggering
 * layer onward; the rule below is this library's reading of it). The layers'
 * refresh_interval fields are ignored.
 *
 * Step 0 computes every layer's prefix state. At every step s < steps - 1 the
 * step kernel of layer l computes
 *   delta_s = max over the block's query rows of
 *             pi_ext * (1 - cos(q_{s+1}, q_ref)),
 * pi_ext the share of the row's softmax mass on the prefix at step s, q_{s+1}
 * the row's pre-RoPE queries of step s + 1 (in the layer's step-major q) and
 * q_ref those of the step the layer's state was computed from; 1 - cos is
 * |q/|q| - r/|r||^2 / 2 (0 for equal rows and for zero rows). When
 * delta_s > threshold, layer l and every deeper layer recompute their state at
 * step s + 1. threshold = 0 refreshes every layer whose next queries differ
 * from its state's; threshold = +inf is FlashBlock's reuse of step 0's state.
 *
 * The decisions are taken on the device, so the whole block is still only
 * enqueued (one CUDA graph can hold it): every layer-step enqueues the prefix
 * launches, which return at once when no refresh is due. FBK_BF16 mode only
 * (FBK_ERR_UNSUPPORTED otherwise). Other arguments and errors as for
 * fbk_decode_block. */
fbk_status fbk_decode_block_adaptive(const fbk_shape *shape, const fbk_layer_block *layers, int32_t n_layers,
                                     int32_t steps, int32_t commit, const fbk_drift_policy *policy, void *ws,
                                     size_t ws_bytes, int32_t num_splits, void *cuda_stream);

/* Elements per quantisation group of fbk_fp8_group_quant (1 x 128). */
#define FBK_FP8_GROUP 128

/* Per-group FP8 quantisation of activations (LaCache §3.4, Mixed precision
 * strategy, Eq. 7-8): the FFN input is cut into groups of 1 x FBK_FP8_GROUP
 * consecutive elements of a row, and for each group g
 *   scale_g = max_{i in g} |x_i| / 448                          (Eq. 8)
 *   x'_i    = E4M3(clip(x_i / scale_g, -448, 448)),  i in g     (Eq. 7)
 * so that x_i ~ x'_i * scale_g. E4M3 is the OCP FP8 format with 4 exponent
 * bits (bias 7) and 3 mantissa bits, largest finite value 448. Both divisions
 * are IEEE fp32 divisions; the quotient is rounded to E4M3 to nearest, ties
 * to even. A group whose elements are all zero gets scale 0 and keeps its
 * zeros (with their signs) as codes. Inputs must be finite.
 *  x:      bf16 [rows, cols], row-major, 16-byte aligned.
 *  rows, cols: rows >= 0, cols >= 0 and a multiple of FBK_FP8_GROUP
 *          (FBK_ERR_INVALID_ARG otherwise); rows * cols <= 2^40
 *          (FBK_ERR_CAPACITY). rows == 0 or cols == 0 enqueues nothing.
 *  codes:  uint8 [rows, cols] E4M3 codes, 8-byte aligned.
 *  scales: fp32 [rows, cols / FBK_FP8_GROUP], 4-byte aligned; group j of row r
 *          at r * cols / FBK_FP8_GROUP + j.
 * One launch. Misaligned pointers return FBK_ERR_UNSUPPORTED. */
fbk_status fbk_fp8_group_quant(const void *x, int64_t rows, int64_t cols, void *codes, float *scales,
                               void *cuda_stream);

/* FACache step for the unchanged rows of a whole sequence (LaCache §3.3.3
 * FACache, Eq. 2-6, and App. J). The sequence's rows outside the current
 * block (the set U: prompt, earlier blocks and the masked suffix, n_rows per
 * sequence, in sequence order with the block removed) keep their
 * online-softmax state over U's keys for the whole block. This call streams
 * only the block's B keys for every row of U and every query head, merges
 * with that state and normalises:
 *   O = (e^(m1-m) O~1 + e^(m2-m) O~2) / (e^(m1-m) l1 + e^(m2-m) l2),
 * (O~1, m1, l1) the cached state and (O~2, m2, l2) the row's state over the
 * block's keys. The block's own rows are the other half of a step: they attend
 * to U's keys and the block's.
 *  q_u:   bf16 [b, n_rows, Hq, d], AFTER RoPE at the rows' own positions
 *         (RoPECache); 16-byte aligned.
 *  state: the cached state of U's rows over U's keys: o_unnorm fp32
 *         [b, Hq, n_rows, d] (16-byte aligned), m and l fp32 [b, Hq, n_rows].
 *  k_blk, v_blk: bf16 [b, B, Hkv, d], K before RoPE; 16-byte aligned.
 *  block_pos: int32 [b] on the device: c0, the block's first position. The
 *         block's keys are rotated at c0 + t. Any value is safe: it only
 *         selects rotation angles.
 *  out:   bf16 [b, n_rows, Hq, d]; lse: fp32 [b, Hq, n_rows] or NULL.
 * FBK_BF16 mode only (FBK_ERR_UNSUPPORTED otherwise). The shape rules are
 * those of fbk_shape except G*B <= 256, which does not apply here (B <= 64
 * still does). n_rows = 0 enqueues nothing; b * n_rows * Hq must stay below
 * 2^31 (FBK_ERR_CAPACITY). One launch. */
fbk_status fbk_facache_unchanged_rows(const fbk_shape *shape, int32_t n_rows, const void *q_u,
                                      const fbk_partial *state, const void *k_blk, const void *v_blk,
                                      const int32_t *block_pos, void *out, float *lse, void *cuda_stream);

/* FACache over a whole sequence as two calls (LaCache §3.3.1-§3.3.3, App. J).
 * The sequence's rows outside the current block (U: prompt, earlier blocks,
 * masked suffix; n_rows per sequence, in sequence order with the block
 * removed) keep their state over U's keys for the whole block:
 * fbk_facache_refresh computes it once per block, and fbk_facache_step uses it
 * at every denoising step. A step's outputs equal attention over the whole
 * sequence. Both calls use a workspace of fbk_facache_workspace_bytes(shape,
 * n_rows, num_splits) bytes (256-byte aligned, contents irrelevant on entry).
 * The shape rules are those of the block path (B <= 64, G*B <= 256).
 *
 * u_cache: U's K (after RoPE, at the rows' own positions) and V, contiguous
 *   [b, Hkv, capacity >= n_rows, d], with prefix_lens[b] = n_rows on the device.
 *
 * fbk_facache_refresh:
 *  q_u_raw: bf16 [b, n_rows, Hq, d], U's queries BEFORE RoPE.
 *  block_pos_host: int32 [b] on the HOST: c0, 0 <= c0 <= n_rows. Row i of U
 *           sits at position i (i < c0) or i + B.
 *  state:   the output, o_unnorm fp32 [b, Hq, n_rows, d] (16-byte aligned),
 *           m and l fp32 [b, Hq, n_rows].
 *  The rows are processed in chunks of up to 256/G rows that do not cross the
 *  block, one prefix computation each, whose states are copied into place.
 *
 * fbk_facache_step (FBK_BF16 only):
 *  q_u_rot: bf16 [b, n_rows, Hq, d], U's queries AFTER RoPE (RoPECache).
 *  state:   from fbk_facache_refresh.
 *  q_blk, k_blk, v_blk: the block, bf16 [b, B, Hq|Hkv, d], Q and K before RoPE.
 *  block_pos: int32 [b] on the device: c0.
 *  out_u: bf16 [b, n_rows, Hq, d]; lse_u fp32 [b, Hq, n_rows] or NULL.
 *  out_blk: bf16 [b, B, Hq, d]; lse_blk fp32 [b, Hq, B] or NULL.
 *  Launches: fbk_facache_unchanged_rows's kernel for U's rows; for the block's
 *  rows, the prefix computation over U's keys with the rows rotated at c0 + t,
 *  then fbk_block_attn_merge's kernel.
 * Errors, before any launch: the shape and cache codes of fbk_prefix_partial
 * (u_cache must be contiguous, else FBK_ERR_UNSUPPORTED); FBK_ERR_INVALID_ARG
 * for n_rows < 0, num_splits < 0, a missing pointer or (refresh) a host c0
 * outside [0, n_rows]; FBK_ERR_CAPACITY when (step) b * n_rows * Hq reaches
 * 2^31 or (refresh) the cache's capacity is below n_rows;
 * FBK_ERR_UNSUPPORTED for misaligned pointers (16 bytes) or a workspace not
 * 256-byte aligned; FBK_ERR_WORKSPACE for a missing or short workspace. */
size_t fbk_facache_workspace_bytes(const fbk_shape *shape, int32_t n_rows, int32_t num_splits);
fbk_status fbk_facache_refresh(const fbk_shape *shape, int32_t n_rows, const void *q_u_raw,
                               const int32_t *block_pos_host, const fbk_kv_cache *u_cache,
                               const fbk_partial *state, void *ws, size_t ws_bytes, int32_t num_splits,
                               void *cuda_stream);
fbk_status fbk_facache_step(const fbk_shape *shape, int32_t n_rows, const void *q_u_rot, const fbk_partial *state,
                            const void *q_blk, const void *k_blk, const void *v_blk, const int32_t *block_pos,
                            const fbk_kv_cache *u_cache, void *out_u, float *lse_u, void *out_blk, float *lse_blk,
                            void *ws, size_t ws_bytes, int32_t num_splits, void *cuda_stream);

/* Sparse block-external attention with a cached residual (FlashBlock,
 * Abstract: cached block-external attention combined with sparse attention as
 * residual reuse). Reading: pages of the prefix (the paged cache's pages) are
 * scored by the largest tau <RoPE(q_t, L_b + t), kbar> over the block's rows
 * and query heads, kbar the page's mean key; the top k pages per sequence form
 * a page table of their own for fbk_prefix_partial_at (queries rotated at the
 * true L_b + t); at a dense step the residual (O~/l, lse) dense minus sparse
 * is captured; at later steps the sparse state plus the residual becomes the
 * state fbk_block_attn_merge merges. Paged caches only.
 *
 * fbk_page_means: means fp32 [b, max_pages_per_seq, Hkv, d], the mean key of
 *   every logical page of the prefix (pages past prefix_lens untouched).
 * fbk_select_pages: q_blk bf16 [b, B, Hq, d] before RoPE; means as written by
 *   fbk_page_means (16-byte aligned, else FBK_ERR_UNSUPPORTED); k >= 1 pages kept;
 *   kept_table int32 [b, k] (physical page ids in increasing logical order,
 *   -1 past the kept count) and kept_lens int32 [b] (their token count, the
 *   partial last page included), both on the device; workspace of
 *   fbk_select_pages_workspace_bytes bytes, 256-byte aligned.
 * fbk_residual_capture: r_o fp32 [b, Hq, B, d] and r_lse fp32 [b, Hq, B] from
 *   the dense and the sparse state of the same queries (r_lse = -inf marks a
 *   row with no prefix).
 * fbk_residual_apply: ext = ((O~/l)_sparse + r_o, lse_sparse + r_lse, 1).
 * Errors, before any launch: FBK_ERR_INVALID_ARG for a missing pointer or
 * k < 1; FBK_ERR_UNSUPPORTED for a contiguous cache, misaligned means or
 * max_pages_per_seq above 25,600 (the selection holds a sequence's scores in
 * shared memory); FBK_ERR_WORKSPACE for a missing or short workspace; the
 * shape and cache codes of fbk_prefix_partial otherwise (the residual calls
 * accept B up to 256, with G*B <= 256). On the device, a page id outside
 * [0, num_pages) raises FBK_DEVERR_PAGE_ID and that page is skipped, and a bad
 * prefix length FBK_DEVERR_PREFIX_LEN (the sequence then counts as empty). */
fbk_status fbk_page_means(const fbk_shape *shape, const fbk_kv_cache *cache, float *means, void *cuda_stream);
size_t fbk_select_pages_workspace_bytes(const fbk_shape *shape, const fbk_kv_cache *cache);
fbk_status fbk_select_pages(const fbk_shape *shape, const void *q_blk, const fbk_kv_cache *cache, const float *means,
                            int32_t k, int32_t *kept_table, int32_t *kept_lens, void *ws, size_t ws_bytes,
                            void *cuda_stream);
fbk_status fbk_residual_capture(const fbk_shape *shape, const fbk_partial *dense, const fbk_partial *sparse,
                                float *r_o, float *r_lse, void *cuda_stream);
fbk_status fbk_residual_apply(const fbk_shape *shape, const fbk_partial *sparse, const float *r_o,
                              const float *r_lse, const fbk_partial *ext, void *cuda_stream);

/* Static text for a status code. */
const char *fbk_status_string(fbk_status status);

#ifdef __cplusplus
}
#endif

#endif /* FBK_H_ */
