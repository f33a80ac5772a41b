// extern "C" entry points of libfbk.so (declared in include/fbk.h): host-side
// argument checks, the kernel-side Geometry, workspace carving and dispatch.
// No entry point allocates, synchronises or keeps state.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <initializer_list>
#include <mutex>
#include <vector>

#include "facache_rows.h"
#include "launch.h"
#include "prefix_at.h"
#include "sparse_prefix.h"

namespace fbk {

// Per-group FP8 quantisation (fp8_quant.cu).
cudaError_t launch_fp8_group_quant(const __nv_bfloat16 *x, long long groups, uint8_t *codes, float *scales,
                                   int sms, cudaStream_t st);


namespace {

bool is_pow2(long long x) { return x > 0 && (x & (x - 1)) == 0; }

// rows_limit: the block path keeps a kv-head's G*B query rows in at most two
// 128-row tiles; entry points whose rows are not the block's skip that limit.
fbk_status check_shape(const fbk_shape *s, bool rows_limit = true, int max_block = 64) {
  if (!s) return FBK_ERR_INVALID_ARG;
  if (s->batch < 1 || s->n_q_heads < 1 || s->n_kv_heads < 1 || s->block_len < 1 || s->head_dim < 1)
    return FBK_ERR_INVALID_ARG;
  if (s->mode != FBK_BF16 && s->mode != FBK_FP32_CHECK) return FBK_ERR_INVALID_ARG;
  if (!isfinite(s->softmax_scale) || !(s->softmax_scale > 0.f) || !isfinite(s->rope_base) ||
      !(s->rope_base > 0.0))
    return FBK_ERR_INVALID_ARG;
  if (s->head_dim != 64 && s->head_dim != 128) return FBK_ERR_UNSUPPORTED;
  if (s->n_q_heads % s->n_kv_heads != 0) return FBK_ERR_UNSUPPORTED;
  if (s->block_len > max_block) return FBK_ERR_UNSUPPORTED;
  if (rows_limit && (long long)(s->n_q_heads / s->n_kv_heads) * s->block_len > 256) return FBK_ERR_UNSUPPORTED;
  if (s->batch > MAX_BATCH) return FBK_ERR_UNSUPPORTED;
  return FBK_OK;
}

fbk_status check_cache(const fbk_shape *s, const fbk_kv_cache *c) {
  if (!c || !c->k || !c->v || !c->prefix_lens) return FBK_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(c->k) | reinterpret_cast<uintptr_t>(c->v)) & 15u)
    return FBK_ERR_UNSUPPORTED;  // tensor-map and 16-byte vector access need 16-byte alignment
  long long rows;
  if (c->paged) {
    if (!c->page_table || c->max_pages_per_seq < 1 || c->num_pages < 1) return FBK_ERR_INVALID_ARG;
    if (!is_pow2(c->page_size) || c->page_size < 16) return FBK_ERR_UNSUPPORTED;
    rows = c->num_pages * s->n_kv_heads * (long long)c->page_size;
    if ((long long)c->max_pages_per_seq * c->page_size > 0x7fffffffll) return FBK_ERR_CAPACITY;
  } else {
    if (c->capacity_tokens < 1) return FBK_ERR_INVALID_ARG;
    if (c->capacity_tokens > 0x7fffffffll) return FBK_ERR_CAPACITY;
    rows = (long long)s->batch * s->n_kv_heads * c->capacity_tokens;
  }
  if (rows > 0x7fffffffll) return FBK_ERR_CAPACITY;  // TMA row coordinates are int32
  // the prefix kernels' work list (tiles plus UNIT_LEAD per unit) must stay below 2^31 entries
  const long long per_seq = c->paged ? (long long)c->max_pages_per_seq * c->page_size : c->capacity_tokens;
  if ((long long)s->batch * s->n_kv_heads * ((per_seq + KV_TILE - 1) / KV_TILE + UNIT_LEAD) > 0x7fffffffll)
    return FBK_ERR_CAPACITY;
  return FBK_OK;
}

Geometry make_geometry(const fbk_shape *s, const fbk_kv_cache *c) {
  Geometry g;
  memset(&g, 0, sizeof(g));
  g.batch = s->batch;
  g.hq = s->n_q_heads;
  g.hkv = s->n_kv_heads;
  g.group = s->n_q_heads / s->n_kv_heads;
  g.d = s->head_dim;
  g.blk = s->block_len;
  g.rows = g.group * g.blk;
  g.tau = s->softmax_scale;
  g.log2_base = log2(s->rope_base);
  for (int i = 0; i < g.d / 2; ++i)
    g.inv_freq_over_pi[i] = pow(s->rope_base, -2.0 * i / g.d) / M_PI;
  if (c) {
    g.kc = static_cast<const __nv_bfloat16 *>(c->k);
    g.vc = static_cast<const __nv_bfloat16 *>(c->v);
    g.paged = c->paged ? 1 : 0;
    g.page_size = c->paged ? c->page_size : 0;
    g.page_shift = 0;
    while (c->paged && (1 << g.page_shift) < c->page_size) ++g.page_shift;
    g.max_pages = c->paged ? c->max_pages_per_seq : 0;
    g.cap = c->paged ? 0 : c->capacity_tokens;
    g.num_pages = c->paged ? c->num_pages : 0;
    g.page_table = c->page_table;
    g.lens = c->prefix_lens;
    g.err = c->error_flags;
  }
  return g;
}

int default_shares() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return sms;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace layout: per-share states for P + b*Hkv - 1 slots (share + unit),
// O~ then m then l, followed by the rotated block queries of every unit in
// the tensor-core kernel's M-tile order ([b*Hkv][MT*128][d] bf16). Every
// region starts on a 256-byte boundary.
struct WsLayout {
  size_t o, m, l, qrot, total;
  long long slots;
};

WsLayout ws_layout(const fbk_shape *s, int shares) {
  const long long rows = (long long)(s->n_q_heads / s->n_kv_heads) * s->block_len;
  const long long units = (long long)s->batch * s->n_kv_heads, mt = rows > 128 ? 2 : 1;
  WsLayout w;
  w.slots = (long long)shares + units;
  w.o = 0;
  w.m = w.o + align256((size_t)(w.slots * rows * s->head_dim) * sizeof(float));
  w.l = w.m + align256((size_t)(w.slots * rows) * sizeof(float));
  w.qrot = w.l + align256((size_t)(w.slots * rows) * sizeof(float));
  w.total = w.qrot + align256((size_t)(units * mt * 128 * s->head_dim) * 2);
  return w;
}

Workspace carve(const WsLayout &l, void *base) {
  char *p = static_cast<char *>(base);
  Workspace w;
  w.o = reinterpret_cast<float *>(p + l.o);
  w.m = reinterpret_cast<float *>(p + l.m);
  w.l = reinterpret_cast<float *>(p + l.l);
  w.qrot = reinterpret_cast<__nv_bfloat16 *>(p + l.qrot);
  w.slots = l.slots;
  return w;
}

fbk_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FBK_OK : FBK_ERR_CUDA; }

// Workspace of FACache over a whole sequence: a prefix workspace big enough
// for a chunk of U's rows (b = 1, cmax rows per query head) and for the
// block's rows (the step), one state buffer for either, and the chunks'
// rotation bases.
struct FacSeqLayout {
  int cmax;
  long long nchunks;  // per sequence
  size_t part_o, part_m, part_l, pos, total;
};

FacSeqLayout fac_layout(const fbk_shape *s, int n_rows, int shares) {
  FacSeqLayout L;
  const int G = s->n_q_heads / s->n_kv_heads;
  L.cmax = 256 / G;
  fbk_shape chunk = *s;
  chunk.batch = 1;
  chunk.block_len = L.cmax;
  const size_t pfx = std::max(ws_layout(&chunk, shares).total, ws_layout(s, shares).total);
  const size_t rows = std::max((size_t)s->n_q_heads * L.cmax, (size_t)s->batch * s->n_q_heads * s->block_len);
  size_t off = align256(pfx);
  L.part_o = off;
  off = align256(off + rows * s->head_dim * sizeof(float));
  L.part_m = off;
  off = align256(off + rows * sizeof(float));
  L.part_l = off;
  off = align256(off + rows * sizeof(float));
  L.nchunks = ((long long)n_rows + L.cmax - 1) / L.cmax + 1;  // the block may cut one chunk in two
  L.pos = off;
  L.total = align256(off + (size_t)L.nchunks * sizeof(int));
  return L;
}

fbk_partial fac_part(const FacSeqLayout &L, void *ws) {
  char *p = static_cast<char *>(ws);
  return fbk_partial{reinterpret_cast<float *>(p + L.part_o), reinterpret_cast<float *>(p + L.part_m),
                     reinterpret_cast<float *>(p + L.part_l)};
}

bool misaligned16(std::initializer_list<const void *> ptrs) {
  uintptr_t bits = 0;
  for (const void *p : ptrs) bits |= reinterpret_cast<uintptr_t>(p);
  return (bits & 15u) != 0;
}

// Host checks of fbk_prefix_partial's pointers (after check_shape and check_cache).
fbk_status check_prefix_ptrs(const void *q_blk, const fbk_partial *out) {
  if (!q_blk || !out || !out->o_unnorm || !out->m || !out->l) return FBK_ERR_INVALID_ARG;
  if (misaligned16({q_blk, out->o_unnorm})) return FBK_ERR_UNSUPPORTED;
  return FBK_OK;
}

// Host checks of fbk_block_attn_merge's pointers (after check_shape).
fbk_status check_merge_ptrs(const void *q_blk, const void *k_blk, const void *v_blk,
                            const int32_t *prefix_lens, const fbk_partial *prefix, const void *out) {
  if (!q_blk || !k_blk || !v_blk || !prefix_lens || !prefix || !prefix->o_unnorm || !prefix->m ||
      !prefix->l || !out)
    return FBK_ERR_INVALID_ARG;
  if (misaligned16({q_blk, k_blk, v_blk, out, prefix->o_unnorm})) return FBK_ERR_UNSUPPORTED;
  return FBK_OK;
}

// Host checks of the commit's block pointers (after check_shape and check_cache).
fbk_status check_commit_ptrs(const void *k_blk, const void *v_blk) {
  if (!k_blk || !v_blk) return FBK_ERR_INVALID_ARG;
  if (misaligned16({k_blk, v_blk})) return FBK_ERR_UNSUPPORTED;
  return FBK_OK;
}

// Share count and workspace checks of a prefix computation.
fbk_status check_workspace(const fbk_shape *shape, int32_t num_splits, const void *ws, size_t ws_bytes,
                           int *shares, WsLayout *lay) {
  *shares = num_splits ? num_splits : default_shares();
  if (*shares < 1) return FBK_ERR_CUDA;
  *lay = ws_layout(shape, *shares);
  if (!ws || ws_bytes < lay->total) return FBK_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return FBK_ERR_UNSUPPORTED;  // TMA reads the query rows
  return FBK_OK;
}

// The launches of one prefix computation: query rotation and share kernel (or
// the fp32 share kernel), then the fixed-order split reduction. qpos: NULL, or
// the rotation base of the block's rows per sequence.
cudaError_t enqueue_prefix(const fbk_shape *shape, const Geometry &g, const void *q_blk, const Workspace &w,
                           int shares, const fbk_partial &out, cudaStream_t s, const int *qpos = nullptr,
                           const PrefixGate *gate = nullptr) {
  const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(q_blk);
  if (gate && shape->mode != FBK_BF16) return cudaErrorInvalidValue;  // gated launches: bf16 path only
  cudaError_t e = shape->mode == FBK_BF16 ? launch_prefix_tc_at(g, q, qpos, w, shares, s, gate)
                                          : launch_prefix_fp32_at(g, q, qpos, w, shares, s);
  if (e != cudaSuccess) return e;
  return launch_split_reduce(g, w, shares, out, s, gate ? gate->gate : nullptr);
}

// Geometry of the step kernel: no cache, only the prefix lengths.
Geometry merge_geometry(const fbk_shape *shape, const int32_t *prefix_lens) {
  Geometry g = make_geometry(shape, nullptr);
  g.lens = prefix_lens;
  return g;
}

cudaError_t enqueue_merge(const fbk_shape *shape, const Geometry &g, const void *q_blk, const void *k_blk,
                          const void *v_blk, const fbk_partial &prefix, void *out, float *lse, cudaStream_t s) {
  return launch_block_merge(g, static_cast<const __nv_bfloat16 *>(q_blk), static_cast<const __nv_bfloat16 *>(k_blk),
                            static_cast<const __nv_bfloat16 *>(v_blk), prefix, out, lse,
                            shape->mode == FBK_FP32_CHECK, s);
}

cudaError_t enqueue_commit(const Geometry &g, const void *k_blk, const void *v_blk, const fbk_kv_cache *cache,
                           cudaStream_t s) {
  return launch_commit(g, static_cast<const __nv_bfloat16 *>(k_blk), static_cast<const __nv_bfloat16 *>(v_blk),
                       static_cast<__nv_bfloat16 *>(cache->k), static_cast<__nv_bfloat16 *>(cache->v),
                       cache->prefix_lens, s);
}

// Built-in scratch of fbk_prefix_partial_static_scratch: one array per device,
// part of this file's device image, so using it allocates nothing.
static __device__ __align__(256) unsigned char g_static_scratch[FBK_STATIC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_static_scratch_mu;
void *g_static_scratch_addr[MAX_DEVICES];  // per device, looked up on first use

// Device address of g_static_scratch on the current device. The first call
// on a device asks the runtime (with that device current) and caches it.
fbk_status static_scratch_address(void **ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FBK_ERR_CUDA;
  if (dev < 0 || dev >= MAX_DEVICES) return FBK_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (!g_static_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return FBK_ERR_CUDA;
    g_static_scratch_addr[dev] = p;
  }
  *ptr = g_static_scratch_addr[dev];
  return FBK_OK;
}

}  // namespace
}  // namespace fbk

using namespace fbk;

extern "C" {

int32_t fbk_default_num_splits(void) { return default_shares(); }

size_t fbk_prefix_workspace_bytes(const fbk_shape *shape, const fbk_kv_cache *cache, int32_t num_splits) {
  (void)cache;
  // any shape a prefix computation accepts (fbk_prefix_partial_at allows B > 64)
  if (check_shape(shape, true, 256) != FBK_OK || num_splits < 0) return 0;
  const int shares = num_splits ? num_splits : default_shares();
  if (shares < 1) return 0;
  return ws_layout(shape, shares).total;
}

fbk_status fbk_prefix_partial(const fbk_shape *shape, const void *q_blk, const fbk_kv_cache *cache,
                              const fbk_partial *out, void *ws, size_t ws_bytes, int32_t num_splits,
                              void *cuda_stream) {
  fbk_status st = check_shape(shape);
  if (st != FBK_OK) return st;
  if ((st = check_cache(shape, cache)) != FBK_OK) return st;
  if (num_splits < 0) return FBK_ERR_INVALID_ARG;
  if ((st = check_prefix_ptrs(q_blk, out)) != FBK_OK) return st;
  int shares;
  WsLayout lay;
  if ((st = check_workspace(shape, num_splits, ws, ws_bytes, &shares, &lay)) != FBK_OK) return st;
  return from_cuda(enqueue_prefix(shape, make_geometry(shape, cache), q_blk, carve(lay, ws), shares, *out,
                                  static_cast<cudaStream_t>(cuda_stream)));
}

fbk_status fbk_block_attn_merge(const fbk_shape *shape, const void *q_blk, const void *k_blk,
                                const void *v_blk, const int32_t *prefix_lens,
                                const fbk_partial *prefix, void *out, float *lse, void *cuda_stream) {
  fbk_status st = check_shape(shape);
  if (st != FBK_OK) return st;
  if ((st = check_merge_ptrs(q_blk, k_blk, v_blk, prefix_lens, prefix, out)) != FBK_OK) return st;
  return from_cuda(enqueue_merge(shape, merge_geometry(shape, prefix_lens), q_blk, k_blk, v_blk, *prefix, out,
                                 lse, static_cast<cudaStream_t>(cuda_stream)));
}

fbk_status fbk_commit_block_rope_append(const fbk_shape *shape, const void *k_blk, const void *v_blk,
                                        fbk_kv_cache *cache, void *cuda_stream) {
  fbk_status st = check_shape(shape);
  if (st != FBK_OK) return st;
  if ((st = check_cache(shape, cache)) != FBK_OK) return st;
  if ((st = check_commit_ptrs(k_blk, v_blk)) != FBK_OK) return st;
  return from_cuda(enqueue_commit(make_geometry(shape, cache), k_blk, v_blk, cache,
                                  static_cast<cudaStream_t>(cuda_stream)));
}

fbk_status fbk_full_ref_attn(const fbk_shape *shape, const void *q_blk, const void *k_blk,
                             const void *v_blk, const fbk_kv_cache *cache, void *out, float *lse,
                             void *cuda_stream) {
  fbk_status st = check_shape(shape);
  if (st != FBK_OK) return st;
  if ((st = check_cache(shape, cache)) != FBK_OK) return st;
  if (!q_blk || !k_blk || !v_blk || !out) return FBK_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(k_blk) | reinterpret_cast<uintptr_t>(v_blk) |
       reinterpret_cast<uintptr_t>(q_blk)) & 3u)
    return FBK_ERR_UNSUPPORTED;
  const Geometry g = make_geometry(shape, cache);
  return from_cuda(launch_full_ref(g, static_cast<const __nv_bfloat16 *>(q_blk),
                                   static_cast<const __nv_bfloat16 *>(k_blk),
                                   static_cast<const __nv_bfloat16 *>(v_blk), out, lse,
                                   shape->mode == FBK_FP32_CHECK, static_cast<cudaStream_t>(cuda_stream)));
}

fbk_status fbk_prefix_partial_at(const fbk_shape *shape, const void *q_blk, const int32_t *q_pos,
                                 const fbk_kv_cache *cache, const fbk_partial *out, void *ws, size_t ws_bytes,
                                 int32_t num_splits, void *cuda_stream) {
  fbk_status st = check_shape(shape, true, 256);  // G*B <= 256 rows per kv-head, B up to 256
  if (st != FBK_OK) return st;
  if ((st = check_cache(shape, cache)) != FBK_OK) return st;
  if (num_splits < 0 || !q_pos) return FBK_ERR_INVALID_ARG;
  if ((st = check_prefix_ptrs(q_blk, out)) != FBK_OK) return st;
  int shares;
  WsLayout lay;
  if ((st = check_workspace(shape, num_splits, ws, ws_bytes, &shares, &lay)) != FBK_OK) return st;
  return from_cuda(enqueue_prefix(shape, make_geometry(shape, cache), q_blk, carve(lay, ws), shares, *out,
                                  static_cast<cudaStream_t>(cuda_stream), q_pos));
}

fbk_status fbk_prefix_partial_static_scratch(const fbk_shape *shape, const void *q_blk,
                                             const fbk_kv_cache *cache, const fbk_partial *out,
                                             int32_t num_splits, void *cuda_stream) {
  fbk_status st = check_shape(shape);
  if (st != FBK_OK) return st;
  if ((st = check_cache(shape, cache)) != FBK_OK) return st;
  if (num_splits < 0) return FBK_ERR_INVALID_ARG;
  if ((st = check_prefix_ptrs(q_blk, out)) != FBK_OK) return st;
  const int shares = num_splits ? num_splits : default_shares();
  if (shares < 1) return FBK_ERR_CUDA;
  const WsLayout lay = ws_layout(shape, shares);
  if (lay.total > (size_t)FBK_STATIC_SCRATCH_BYTES) return FBK_ERR_SCRATCH_LIMIT;
  void *scratch = nullptr;
  if ((st = static_scratch_address(&scratch)) != FBK_OK) return st;
  return from_cuda(enqueue_prefix(shape, make_geometry(shape, cache), q_blk, carve(lay, scratch), shares, *out,
                                  static_cast<cudaStream_t>(cuda_stream)));
}

fbk_status fbk_decode_block(const fbk_shape *shape, const fbk_layer_block *layers, int32_t n_layers,
                            int32_t steps, int32_t commit, void *ws, size_t ws_bytes, int32_t num_splits,
                            void *cuda_stream) {
  fbk_status st = check_shape(shape);
  if (st != FBK_OK) return st;
  if (!layers || n_layers < 1 || steps < 1 || num_splits < 0) return FBK_ERR_INVALID_ARG;
  // every layer is checked before the first launch
  for (int32_t l = 0; l < n_layers; ++l) {
    const fbk_layer_block &L = layers[l];
    if ((st = check_cache(shape, &L.cache)) != FBK_OK) return st;
    if (L.refresh_interval < 1) return FBK_ERR_INVALID_ARG;
    if ((st = check_prefix_ptrs(L.q, &L.prefix)) != FBK_OK) return st;
    if ((st = check_merge_ptrs(L.q, L.k, L.v, L.cache.prefix_lens, &L.prefix, L.out)) != FBK_OK) return st;
    if (commit) {
      for (int32_t j = 0; j < l; ++j)  // a shared length array would be advanced once per layer
        if (layers[j].cache.prefix_lens == L.cache.prefix_lens) return FBK_ERR_INVALID_ARG;
    }
  }
  // element strides of one step inside each layer's step-major arrays
  const size_t b = shape->batch, B = shape->block_len, d = shape->head_dim;
  const size_t q_step = b * B * shape->n_q_heads * d, kv_step = b * B * shape->n_kv_heads * d;
  const size_t out_step_bytes = q_step * (shape->mode == FBK_FP32_CHECK ? 4 : 2);
  const size_t lse_step = b * shape->n_q_heads * B;
  if ((size_t)steps > ((size_t)1 << 62) / (out_step_bytes * 2)) return FBK_ERR_CAPACITY;
  int shares;
  WsLayout lay;
  if ((st = check_workspace(shape, num_splits, ws, ws_bytes, &shares, &lay)) != FBK_OK) return st;
  const Workspace w = carve(lay, ws);
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);

  std::vector<Geometry> geo(n_layers);  // prefix and commit geometry of each layer
  for (int32_t l = 0; l < n_layers; ++l) geo[l] = make_geometry(shape, &layers[l].cache);
  Geometry gm = make_geometry(shape, nullptr);
  auto at = [](const void *p, size_t bytes) { return static_cast<const char *>(p) + bytes; };

  for (int32_t step = 0; step < steps; ++step) {
    for (int32_t l = 0; l < n_layers; ++l) {
      const fbk_layer_block &L = layers[l];
      const void *q = at(L.q, step * q_step * 2);
      if (step % L.refresh_interval == 0) {
        if (enqueue_prefix(shape, geo[l], q, w, shares, L.prefix, s) != cudaSuccess) return FBK_ERR_CUDA;
      }
      gm.lens = L.cache.prefix_lens;
      void *out = static_cast<char *>(L.out) + step * out_step_bytes;
      float *lse = L.lse ? L.lse + step * lse_step : nullptr;
      if (enqueue_merge(shape, gm, q, at(L.k, step * kv_step * 2), at(L.v, step * kv_step * 2), L.prefix, out, lse,
                        s) != cudaSuccess)
        return FBK_ERR_CUDA;
    }
  }
  if (commit) {
    for (int32_t l = 0; l < n_layers; ++l) {
      const fbk_layer_block &L = layers[l];
      const size_t last = (size_t)(steps - 1) * kv_step * 2;
      if (enqueue_commit(geo[l], at(L.k, last), at(L.v, last), &L.cache, s) != cudaSuccess) return FBK_ERR_CUDA;
    }
  }
  return FBK_OK;
}

fbk_status fbk_decode_block_adaptive(const fbk_shape *shape, const fbk_layer_block *layers, int32_t n_layers,
                                     int32_t steps, int32_t commit, const fbk_drift_policy *policy, void *ws,
                                     size_t ws_bytes, int32_t num_splits, void *cuda_stream) {
  fbk_status st = check_shape(shape);
  if (st != FBK_OK) return st;
  if (!layers || n_layers < 1 || steps < 1 || num_splits < 0 || !policy) return FBK_ERR_INVALID_ARG;
  if (shape->mode != FBK_BF16) return FBK_ERR_UNSUPPORTED;
  if (!(policy->threshold >= 0.f) || !policy->flags || !policy->last_refresh || !policy->drift ||
      !policy->refreshed)  // (a NaN threshold fails the first test)
    return FBK_ERR_INVALID_ARG;
  if ((long long)n_layers * steps > 0x7fffffffll) return FBK_ERR_CAPACITY;
  for (int32_t l = 0; l < n_layers; ++l) {
    const fbk_layer_block &L = layers[l];
    if ((st = check_cache(shape, &L.cache)) != FBK_OK) return st;
    if ((st = check_prefix_ptrs(L.q, &L.prefix)) != FBK_OK) return st;
    if ((st = check_merge_ptrs(L.q, L.k, L.v, L.cache.prefix_lens, &L.prefix, L.out)) != FBK_OK) return st;
    if (commit) {
      for (int32_t j = 0; j < l; ++j)
        if (layers[j].cache.prefix_lens == L.cache.prefix_lens) return FBK_ERR_INVALID_ARG;
    }
  }
  const size_t b = shape->batch, B = shape->block_len, d = shape->head_dim;
  const size_t q_step = b * B * shape->n_q_heads * d, kv_step = b * B * shape->n_kv_heads * d;
  const size_t out_step_bytes = q_step * 2;
  const size_t lse_step = b * shape->n_q_heads * B;
  if ((size_t)steps > ((size_t)1 << 62) / (out_step_bytes * 2)) return FBK_ERR_CAPACITY;
  int shares;
  WsLayout lay;
  if ((st = check_workspace(shape, num_splits, ws, ws_bytes, &shares, &lay)) != FBK_OK) return st;
  const Workspace w = carve(lay, ws);
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  std::vector<Geometry> geo(n_layers);
  for (int32_t l = 0; l < n_layers; ++l) geo[l] = make_geometry(shape, &layers[l].cache);
  Geometry gm = make_geometry(shape, nullptr);
  auto at = [](const void *p, size_t bytes) { return static_cast<const char *>(p) + bytes; };
  int32_t *flags = policy->flags;  // [2][n_layers]: requests for even and odd steps

  if (launch_adaptive_init(flags, policy->last_refresh, policy->drift, policy->refreshed, n_layers, steps, s) !=
      cudaSuccess)
    return FBK_ERR_CUDA;
  for (int32_t step = 0; step < steps; ++step) {
    int32_t *cur = flags + (step & 1) * n_layers, *nxt = flags + ((step + 1) & 1) * n_layers;
    for (int32_t l = 0; l < n_layers; ++l) {
      const fbk_layer_block &L = layers[l];
      const void *q = at(L.q, step * q_step * 2);
      const size_t cell = (size_t)step * n_layers + l;
      const PrefixGate gate{cur + l, policy->refreshed + cell, policy->last_refresh + l, step};
      if (enqueue_prefix(shape, geo[l], q, w, shares, L.prefix, s, nullptr, &gate) != cudaSuccess)
        return FBK_ERR_CUDA;
      const DriftArgs dr{static_cast<const __nv_bfloat16 *>(L.q), (long long)q_step, policy->last_refresh + l,
                         step + 1 < steps ? step + 1 : -1, cur + l, nxt + l, n_layers - l, policy->threshold,
                         policy->drift + cell};
      gm.lens = L.cache.prefix_lens;
      void *out = static_cast<char *>(L.out) + step * out_step_bytes;
      float *lse = L.lse ? L.lse + step * lse_step : nullptr;
      if (launch_block_merge(gm, static_cast<const __nv_bfloat16 *>(q),
                             reinterpret_cast<const __nv_bfloat16 *>(at(L.k, step * kv_step * 2)),
                             reinterpret_cast<const __nv_bfloat16 *>(at(L.v, step * kv_step * 2)), L.prefix, out, lse,
                             false, s, &dr) != cudaSuccess)
        return FBK_ERR_CUDA;
    }
  }
  if (commit) {
    for (int32_t l = 0; l < n_layers; ++l) {
      const fbk_layer_block &L = layers[l];
      const size_t last = (size_t)(steps - 1) * kv_step * 2;
      if (enqueue_commit(geo[l], at(L.k, last), at(L.v, last), &L.cache, s) != cudaSuccess) return FBK_ERR_CUDA;
    }
  }
  return FBK_OK;
}

fbk_status fbk_fp8_group_quant(const void *x, int64_t rows, int64_t cols, void *codes, float *scales,
                               void *cuda_stream) {
  if (rows < 0 || cols < 0 || cols % FBK_FP8_GROUP != 0) return FBK_ERR_INVALID_ARG;
  if (rows == 0 || cols == 0) return FBK_OK;  // nothing to quantise, nothing enqueued
  if (rows > ((int64_t)1 << 40) / cols) return FBK_ERR_CAPACITY;
  if (!x || !codes || !scales) return FBK_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(x) & 15u) || (reinterpret_cast<uintptr_t>(codes) & 7u) ||
      (reinterpret_cast<uintptr_t>(scales) & 3u))
    return FBK_ERR_UNSUPPORTED;
  const int sms = default_shares();
  if (sms < 1) return FBK_ERR_CUDA;
  return from_cuda(launch_fp8_group_quant(static_cast<const __nv_bfloat16 *>(x), rows * cols / FBK_FP8_GROUP,
                                          static_cast<uint8_t *>(codes), scales, sms,
                                          static_cast<cudaStream_t>(cuda_stream)));
}

fbk_status fbk_facache_unchanged_rows(const fbk_shape *shape, int32_t n_rows, const void *q_u,
                                      const fbk_partial *state, const void *k_blk, const void *v_blk,
                                      const int32_t *block_pos, void *out, float *lse, void *cuda_stream) {
  fbk_status st = check_shape(shape, false);
  if (st != FBK_OK) return st;
  if (shape->mode != FBK_BF16) return FBK_ERR_UNSUPPORTED;
  if (n_rows < 0) return FBK_ERR_INVALID_ARG;
  if (n_rows == 0) return FBK_OK;  // no unchanged rows, nothing enqueued
  if ((long long)shape->batch * n_rows * shape->n_q_heads > 0x7fffffffll) return FBK_ERR_CAPACITY;
  if ((st = check_merge_ptrs(q_u, k_blk, v_blk, block_pos, state, out)) != FBK_OK) return st;
  const int sms = default_shares();
  if (sms < 1) return FBK_ERR_CUDA;
  FacRowsArgs a;
  a.q = static_cast<const __nv_bfloat16 *>(q_u);
  a.state = *state;
  a.kb = static_cast<const __nv_bfloat16 *>(k_blk);
  a.vb = static_cast<const __nv_bfloat16 *>(v_blk);
  a.block_pos = block_pos;
  a.out = static_cast<__nv_bfloat16 *>(out);
  a.lse = lse;
  a.n_rows = n_rows;
  a.ctas_per_unit = 1;
  return from_cuda(launch_facache_rows(make_geometry(shape, nullptr), a, sms, static_cast<cudaStream_t>(cuda_stream)));
}

size_t fbk_facache_workspace_bytes(const fbk_shape *shape, int32_t n_rows, int32_t num_splits) {
  if (check_shape(shape) != FBK_OK || n_rows < 0 || num_splits < 0) return 0;
  const int shares = num_splits ? num_splits : default_shares();
  if (shares < 1) return 0;
  return fac_layout(shape, n_rows, shares).total;
}

fbk_status fbk_facache_refresh(const fbk_shape *shape, int32_t n_rows, const void *q_u_raw,
                               const int32_t *block_pos_host, const fbk_kv_cache *u_cache,
                               const fbk_partial *state, void *ws, size_t ws_bytes, int32_t num_splits,
                               void *cuda_stream) {
  fbk_status st = check_shape(shape);
  if (st != FBK_OK) return st;
  if ((st = check_cache(shape, u_cache)) != FBK_OK) return st;
  if (u_cache->paged) return FBK_ERR_UNSUPPORTED;
  if (n_rows < 0 || num_splits < 0 || !block_pos_host) return FBK_ERR_INVALID_ARG;
  if (n_rows == 0) return FBK_OK;
  if (u_cache->capacity_tokens < n_rows) return FBK_ERR_CAPACITY;
  if ((st = check_prefix_ptrs(q_u_raw, state)) != FBK_OK) return st;
  for (int32_t bi = 0; bi < shape->batch; ++bi)
    if (block_pos_host[bi] < 0 || block_pos_host[bi] > n_rows) return FBK_ERR_INVALID_ARG;
  const int shares = num_splits ? num_splits : default_shares();
  if (shares < 1) return FBK_ERR_CUDA;
  const FacSeqLayout L = fac_layout(shape, n_rows, shares);
  if (!ws || ws_bytes < L.total) return FBK_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return FBK_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const fbk_partial part = fac_part(L, ws);
  int *pos = reinterpret_cast<int *>(static_cast<char *>(ws) + L.pos);
  const size_t hq = shape->n_q_heads, d = shape->head_dim, U = n_rows;
  for (int32_t bi = 0; bi < shape->batch; ++bi) {
    const int c0 = block_pos_host[bi];
    const int n_before = (c0 + L.cmax - 1) / L.cmax, n_after = (n_rows - c0 + L.cmax - 1) / L.cmax;
    if (launch_chunk_positions(pos, n_before, n_after, c0, L.cmax, shape->block_len, s) != cudaSuccess)
      return FBK_ERR_CUDA;
    fbk_kv_cache one = *u_cache;  // this sequence's keys
    const size_t seq_elems = (size_t)shape->n_kv_heads * u_cache->capacity_tokens * d;
    one.k = static_cast<char *>(u_cache->k) + bi * seq_elems * 2;
    one.v = static_cast<char *>(u_cache->v) + bi * seq_elems * 2;
    one.prefix_lens = u_cache->prefix_lens + bi;
    int k = 0;
    const int bounds[3] = {0, c0, n_rows};
    for (int side = 0; side < 2; ++side) {
      for (int i0 = bounds[side]; i0 < bounds[side + 1]; i0 += L.cmax, ++k) {
        fbk_shape cs = *shape;
        cs.batch = 1;
        cs.block_len = std::min(L.cmax, bounds[side + 1] - i0);
        const Geometry g = make_geometry(&cs, &one);
        const Workspace w = carve(ws_layout(&cs, shares), ws);
        const void *q = static_cast<const char *>(q_u_raw) + ((size_t)bi * U + i0) * hq * d * 2;
        if (enqueue_prefix(&cs, g, q, w, shares, part, s, pos + k) != cudaSuccess) return FBK_ERR_CUDA;
        // the chunk's rows into the state: [Hq, rows, d] -> [b, Hq, U, d] at row i0
        const size_t rows = cs.block_len;
        float *o_dst = state->o_unnorm + ((size_t)bi * hq * U + i0) * d;
        if (cudaMemcpy2DAsync(o_dst, U * d * 4, part.o_unnorm, rows * d * 4, rows * d * 4, hq,
                              cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
            cudaMemcpy2DAsync(state->m + (size_t)bi * hq * U + i0, U * 4, part.m, rows * 4, rows * 4, hq,
                              cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
            cudaMemcpy2DAsync(state->l + (size_t)bi * hq * U + i0, U * 4, part.l, rows * 4, rows * 4, hq,
                              cudaMemcpyDeviceToDevice, s) != cudaSuccess)
          return FBK_ERR_CUDA;
      }
    }
  }
  return FBK_OK;
}

fbk_status fbk_facache_step(const fbk_shape *shape, int32_t n_rows, const void *q_u_rot, const fbk_partial *state,
                            const void *q_blk, const void *k_blk, const void *v_blk, const int32_t *block_pos,
                            const fbk_kv_cache *u_cache, void *out_u, float *lse_u, void *out_blk, float *lse_blk,
                            void *ws, size_t ws_bytes, int32_t num_splits, void *cuda_stream) {
  fbk_status st = check_shape(shape);
  if (st != FBK_OK) return st;
  if (shape->mode != FBK_BF16) return FBK_ERR_UNSUPPORTED;
  if ((st = check_cache(shape, u_cache)) != FBK_OK) return st;
  if (n_rows < 0 || num_splits < 0) return FBK_ERR_INVALID_ARG;
  if ((long long)shape->batch * n_rows * shape->n_q_heads > 0x7fffffffll) return FBK_ERR_CAPACITY;
  if ((st = check_merge_ptrs(q_blk, k_blk, v_blk, block_pos, state, out_blk)) != FBK_OK) return st;
  if (n_rows > 0 && (st = check_merge_ptrs(q_u_rot, k_blk, v_blk, block_pos, state, out_u)) != FBK_OK) return st;
  const int shares = num_splits ? num_splits : default_shares();
  if (shares < 1) return FBK_ERR_CUDA;
  const FacSeqLayout L = fac_layout(shape, n_rows, shares);
  if (!ws || ws_bytes < L.total) return FBK_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return FBK_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  if (n_rows > 0) {  // U's rows: their cached state merged with the block's keys
    FacRowsArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(q_u_rot);
    a.state = *state;
    a.kb = static_cast<const __nv_bfloat16 *>(k_blk);
    a.vb = static_cast<const __nv_bfloat16 *>(v_blk);
    a.block_pos = block_pos;
    a.out = static_cast<__nv_bfloat16 *>(out_u);
    a.lse = lse_u;
    a.n_rows = n_rows;
    a.ctas_per_unit = 1;
    const int sms = default_shares();
    if (sms < 1) return FBK_ERR_CUDA;
    if (launch_facache_rows(make_geometry(shape, nullptr), a, sms, s) != cudaSuccess) return FBK_ERR_CUDA;
  }
  // the block's rows: their state over U's keys (rotated at c0 + t), then the step kernel
  const fbk_partial part = fac_part(L, ws);
  if (enqueue_prefix(shape, make_geometry(shape, u_cache), q_blk, carve(ws_layout(shape, shares), ws), shares, part,
                     s, block_pos) != cudaSuccess)
    return FBK_ERR_CUDA;
  return from_cuda(enqueue_merge(shape, merge_geometry(shape, block_pos), q_blk, k_blk, v_blk, part, out_blk,
                                 lse_blk, s));
}

fbk_status fbk_page_means(const fbk_shape *shape, const fbk_kv_cache *cache, float *means, void *cuda_stream) {
  fbk_status st = check_shape(shape);
  if (st != FBK_OK) return st;
  if ((st = check_cache(shape, cache)) != FBK_OK) return st;
  if (!cache->paged) return FBK_ERR_UNSUPPORTED;
  if (!means) return FBK_ERR_INVALID_ARG;
  return from_cuda(launch_page_means(make_geometry(shape, cache), means, static_cast<cudaStream_t>(cuda_stream)));
}

size_t fbk_select_pages_workspace_bytes(const fbk_shape *shape, const fbk_kv_cache *cache) {
  if (check_shape(shape) != FBK_OK || !cache || !cache->paged || cache->max_pages_per_seq < 1) return 0;
  const size_t qrot = (size_t)shape->batch * shape->block_len * shape->n_q_heads * shape->head_dim * 4;
  return align256(qrot) + align256((size_t)shape->batch * shape->n_kv_heads * cache->max_pages_per_seq * 4);
}

fbk_status fbk_select_pages(const fbk_shape *shape, const void *q_blk, const fbk_kv_cache *cache, const float *means,
                            int32_t k, int32_t *kept_table, int32_t *kept_lens, void *ws, size_t ws_bytes,
                            void *cuda_stream) {
  fbk_status st = check_shape(shape);
  if (st != FBK_OK) return st;
  if ((st = check_cache(shape, cache)) != FBK_OK) return st;
  if (!cache->paged) return FBK_ERR_UNSUPPORTED;
  if (!q_blk || !means || !kept_table || !kept_lens || k < 1) return FBK_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(means) & 15u) return FBK_ERR_UNSUPPORTED;  // 16-byte vector loads
  if ((size_t)cache->max_pages_per_seq * 8 > 200 * 1024) return FBK_ERR_UNSUPPORTED;  // scores + flags in smem
  const size_t need = fbk_select_pages_workspace_bytes(shape, cache);
  if (!ws || ws_bytes < need) return FBK_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return FBK_ERR_UNSUPPORTED;
  const int sms = default_shares();
  if (sms < 1) return FBK_ERR_CUDA;
  float *qrot = static_cast<float *>(ws);
  float *scores = reinterpret_cast<float *>(static_cast<char *>(ws) +
                                            align256((size_t)shape->batch * shape->block_len * shape->n_q_heads *
                                                     shape->head_dim * 4));
  return from_cuda(launch_select_pages(make_geometry(shape, cache), static_cast<const __nv_bfloat16 *>(q_blk), means,
                                       k, qrot, scores, kept_table, kept_lens, sms,
                                       static_cast<cudaStream_t>(cuda_stream)));
}

fbk_status fbk_residual_capture(const fbk_shape *shape, const fbk_partial *dense, const fbk_partial *sparse,
                                float *r_o, float *r_lse, void *cuda_stream) {
  fbk_status st = check_shape(shape, true, 256);
  if (st != FBK_OK) return st;
  if (!dense || !sparse || !dense->o_unnorm || !dense->m || !dense->l || !sparse->o_unnorm || !sparse->m ||
      !sparse->l || !r_o || !r_lse)
    return FBK_ERR_INVALID_ARG;
  const int sms = default_shares();
  if (sms < 1) return FBK_ERR_CUDA;
  const int rows = shape->batch * shape->n_q_heads * shape->block_len;
  return from_cuda(launch_residual_capture(rows, shape->head_dim, *dense, *sparse, r_o, r_lse, sms,
                                           static_cast<cudaStream_t>(cuda_stream)));
}

fbk_status fbk_residual_apply(const fbk_shape *shape, const fbk_partial *sparse, const float *r_o,
                              const float *r_lse, const fbk_partial *ext, void *cuda_stream) {
  fbk_status st = check_shape(shape, true, 256);
  if (st != FBK_OK) return st;
  if (!sparse || !ext || !sparse->o_unnorm || !sparse->m || !sparse->l || !ext->o_unnorm || !ext->m || !ext->l ||
      !r_o || !r_lse)
    return FBK_ERR_INVALID_ARG;
  const int sms = default_shares();
  if (sms < 1) return FBK_ERR_CUDA;
  const int rows = shape->batch * shape->n_q_heads * shape->block_len;
  return from_cuda(launch_residual_apply(rows, shape->head_dim, *sparse, r_o, r_lse, *ext, sms,
                                         static_cast<cudaStream_t>(cuda_stream)));
}

const char *fbk_status_string(fbk_status status) {
  switch (status) {
    case FBK_OK: return "ok";
    case FBK_ERR_INVALID_ARG: return "invalid argument";
    case FBK_ERR_UNSUPPORTED: return "unsupported shape or alignment";
    case FBK_ERR_CAPACITY: return "cache geometry exceeds the supported size";
    case FBK_ERR_WORKSPACE: return "workspace missing or too small";
    case FBK_ERR_CUDA: return "CUDA error";
    case FBK_ERR_SCRATCH_LIMIT: return "call needs more scratch than the built-in 32 MiB array";
  }
  return "unknown status";
}

}  // extern "C"
