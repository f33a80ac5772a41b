// Sparse block-external attention with a cached residual (FlashBlock,
// "Attention Caching for Efficient Long-Context Block Diffusion", Abstract:
// cached block-external attention combined with sparse attention as residual
// reuse). The reading implemented here:
//  * pages of the prefix (P tokens, the cache's page size) are summarised by
//    their mean key per kv-head;
//  * a page's score is the largest tau <RoPE(q_t, L + t), kbar> over the
//    block's rows and query heads; the k best pages of each sequence are kept
//    (ties to the lower page index), in increasing page order, as a page table
//    of their own, so that the paged prefix path computes the sparse state;
//  * at a dense step the residual between the dense and the sparse state is
//    taken in normalised-output space, (O~/l)_dense - (O~/l)_sparse and
//    lse_dense - lse_sparse; at later steps the sparse state plus that
//    residual is turned into a state (O, lse, 1) that the step kernel merges
//    with the fresh in-block attention.
//
// The mean keys read every K byte of the prefix once (a committed block only
// changes its own pages, so a decoder needs them once per page); the scores
// read the means and the block's queries; the residual kernels touch one
// state.
#include "launch.h"
#include "sparse_prefix.h"

namespace fbk {
namespace {

// Mean key of every logical page (b, lp) of every kv-head: [b, max_pages, Hkv, d]
// fp32. One CTA per (b, lp); pages past the prefix are left untouched. The
// page's keys of one kv-head are P rows of d bf16 in one run; the CTA reads a
// kv-head's run in 16-byte chunks (thread: chunk c of rows s, s + NS, ...),
// then sums the NS partial sums of each column in a fixed order.
constexpr int MEAN_THREADS = 256;

template <int D>
__global__ void __launch_bounds__(MEAN_THREADS) page_means_kernel(Geometry g, float *__restrict__ means) {
  constexpr int CPR = D / 8, NS = MEAN_THREADS / CPR;  // 16-byte chunks per row, row slots
  __shared__ float part[NS][D + 4];
  const int b = blockIdx.x / g.max_pages, lp = blockIdx.x % g.max_pages;
  const int c = threadIdx.x % CPR, slot = threadIdx.x / CPR;
  pdl_wait();
  pdl_release();
  const int L = prefix_len(g, b);
  const int t0 = lp * g.page_size, n = min(g.page_size, L - t0);
  if (n <= 0) return;
  const int pid = g.page_table[(long long)b * g.max_pages + lp];
  if (pid < 0 || (long long)pid >= g.num_pages) {
    if (threadIdx.x == 0) raise_flag(g, FBK_DEVERR_PAGE_ID);
    return;
  }
  const float inv_n = 1.f / (float)n;
  for (int kvh = 0; kvh < g.hkv; ++kvh) {
    const uint4 *src = reinterpret_cast<const uint4 *>(g.kc + ((long long)pid * g.hkv + kvh) * g.page_size * D) + c;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int t = slot; t < n; t += NS) {
      const uint4 v = __ldg(src + (long long)t * CPR);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[2 * e] += __uint_as_float(w[e] << 16);
        acc[2 * e + 1] += __uint_as_float(w[e] & 0xffff0000u);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) part[slot][8 * c + e] = acc[e];
    __syncthreads();
    for (int i = threadIdx.x; i < D; i += MEAN_THREADS) {
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < NS; ++k) s += part[k][i];
      means[(((long long)b * g.max_pages + lp) * g.hkv + kvh) * D + i] = s * inv_n;
    }
    __syncthreads();  // part is rewritten by the next kv-head
  }
}

// The block's queries rotated at L + t, fp32 [b, B, Hq, d].
__global__ void __launch_bounds__(256) rotate_queries_kernel(Geometry g, const __nv_bfloat16 *__restrict__ q,
                                                             float *__restrict__ qrot) {
  pdl_wait();
  pdl_release();
  const int half = g.d / 2;
  const long long n = (long long)g.batch * g.blk * g.hq * half;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int i = (int)(idx % half);
    const long long row = idx / half;  // (b, t, h)
    const int t = (int)((row / g.hq) % g.blk), b = (int)(row / ((long long)g.hq * g.blk));
    const int L = prefix_len(g, b);
    const float2 cs = rope_cs_fast(L + t, g.inv_freq_over_pi[i]);
    const float x1 = __bfloat162float(q[row * g.d + i]), x2 = __bfloat162float(q[row * g.d + i + half]);
    qrot[row * g.d + i] = x1 * cs.x - x2 * cs.y;
    qrot[row * g.d + i + half] = x2 * cs.x + x1 * cs.y;
  }
}

// Score of every logical page per kv-head: scores [b, Hkv, max_pages], the
// largest tau <qrot[b, t, h], kbar[b, lp, kvh]> over the block's tokens t and
// the query heads h of kv-head kvh (the page's score is the largest over the
// kv-heads, taken by the selection). One CTA per (b, kvh, 64 pages): the mean
// keys of its pages and then 64 query rows at a time are staged transposed in
// shared memory ([d][64] each), and each thread forms a 4 x 4 block of dot
// products in fp32 (rows 4rg.., pages 4pg..), 16 multiply-adds per two
// 16-byte shared loads. Pages past the prefix are not written.
constexpr int SCORE_PAGES = 64, SCORE_ROWS = 64, SCORE_THREADS = 256;

constexpr int score_smem_bytes(int d) { return (d * (SCORE_PAGES + SCORE_ROWS) + SCORE_THREADS / 16 * SCORE_PAGES) * 4; }

template <int D>
__global__ void __launch_bounds__(SCORE_THREADS) page_scores_kernel(Geometry g, const float *__restrict__ qrot,
                                                                    const float *__restrict__ means,
                                                                    float *__restrict__ scores, int tiles) {
  extern __shared__ float4 score_smem[];
  float(*Kt)[SCORE_PAGES] = reinterpret_cast<float(*)[SCORE_PAGES]>(score_smem);
  float(*Qt)[SCORE_ROWS] = reinterpret_cast<float(*)[SCORE_ROWS]>(&Kt[D][0]);
  float(*red)[SCORE_PAGES] = reinterpret_cast<float(*)[SCORE_PAGES]>(&Qt[D][0]);
  const int tile = blockIdx.x % tiles, u = blockIdx.x / tiles, b = u / g.hkv, kvh = u % g.hkv;
  const int tid = threadIdx.x, pg = tid % 16, rg = tid / 16;
  pdl_wait();
  pdl_release();
  const int L = prefix_len(g, b);
  const int n_pages = (L + g.page_size - 1) / g.page_size, p0 = tile * SCORE_PAGES;
  if (p0 >= n_pages) return;
  const int np = min(SCORE_PAGES, n_pages - p0), R = g.group * g.blk;  // rows of the kv-head: (head, token)
  for (int idx = tid; idx < SCORE_PAGES * (D / 4); idx += SCORE_THREADS) {
    const int p = idx % SCORE_PAGES, i4 = idx / SCORE_PAGES;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (p < np)
      v = __ldg(reinterpret_cast<const float4 *>(means + (((long long)b * g.max_pages + p0 + p) * g.hkv + kvh) * D) + i4);
    Kt[4 * i4][p] = v.x;
    Kt[4 * i4 + 1][p] = v.y;
    Kt[4 * i4 + 2][p] = v.z;
    Kt[4 * i4 + 3][p] = v.w;
  }
  float best[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
  for (int r0 = 0; r0 < R; r0 += SCORE_ROWS) {
    __syncthreads();  // the previous rows are consumed
    for (int idx = tid; idx < SCORE_ROWS * (D / 4); idx += SCORE_THREADS) {
      const int rr = idx % SCORE_ROWS, i4 = idx / SCORE_ROWS, r = r0 + rr;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < R) {
        const int hl = r / g.blk, t = r % g.blk;
        v = __ldg(reinterpret_cast<const float4 *>(qrot + (((long long)b * g.blk + t) * g.hq + kvh * g.group + hl) * D) + i4);
      }
      Qt[4 * i4][rr] = v.x;
      Qt[4 * i4 + 1][rr] = v.y;
      Qt[4 * i4 + 2][rr] = v.z;
      Qt[4 * i4 + 3][rr] = v.w;
    }
    __syncthreads();
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
    for (int i = 0; i < D; ++i) {
      const float4 kv = *reinterpret_cast<const float4 *>(&Kt[i][4 * pg]);
      const float4 qv = *reinterpret_cast<const float4 *>(&Qt[i][4 * rg]);
      const float qa[4] = {qv.x, qv.y, qv.z, qv.w}, ka[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(qa[x], ka[y], acc[x][y]);
    }
#pragma unroll
    for (int x = 0; x < 4; ++x)
      if (r0 + 4 * rg + x < R)
#pragma unroll
        for (int y = 0; y < 4; ++y) best[y] = fmaxf(best[y], g.tau * acc[x][y]);
  }
#pragma unroll
  for (int y = 0; y < 4; ++y) red[rg][4 * pg + y] = best[y];
  __syncthreads();
  if (tid < np) {
    float m = -CUDART_INF_F;
#pragma unroll
    for (int k = 0; k < SCORE_THREADS / 16; ++k) m = fmaxf(m, red[k][tid]);
    scores[((long long)b * g.hkv + kvh) * g.max_pages + p0 + tid] = m;
  }
}

// Top-k pages of each sequence (one CTA per sequence). A page's score is the
// largest of its kv-heads' scores; the k best pages are kept, ties to the
// lower page index. The k-th largest score is found by a radix select over the
// scores' order-preserving 32-bit keys (four 8-bit digits, most significant
// first, one shared-memory histogram each, the lanes of a warp that share a
// bin adding once: scores cluster, so their top digits do); the pages above
// it are kept, and
// of the pages equal to it the lowest-indexed ones that complete the k. The
// kept pages' physical ids go to kept_table in increasing logical order (their
// positions from a block-wide scan of the keep flags, each thread owning a run
// of consecutive pages), with their token count (a partial last page counts
// its tokens; being the highest page, it is last when kept).
constexpr int SEL_THREADS = 1024;

__device__ __forceinline__ unsigned order_key(float f) {  // a < b  <=>  order_key(a) < order_key(b)
  const unsigned u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum of v over the CTA's threads in thread order; *total
// gets the sum. Every thread of the CTA calls it.
__device__ int block_exclusive_scan(int v, int *wsum, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int t = lane < SEL_THREADS / 32 ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    wsum[lane] = t;
  }
  __syncthreads();
  const int before = warp > 0 ? wsum[warp - 1] : 0;
  *total = wsum[SEL_THREADS / 32 - 1];
  __syncthreads();  // wsum is reused by the next call
  return before + x - v;
}

__global__ void __launch_bounds__(SEL_THREADS) select_pages_kernel(Geometry g, const float *__restrict__ scores, int k,
                                                                   int *__restrict__ kept_table,
                                                                   int *__restrict__ kept_lens) {
  extern __shared__ unsigned sel_key[];  // [max_pages]
  __shared__ int hist[256];
  __shared__ int wsum[32];
  __shared__ unsigned s_prefix;
  __shared__ int s_rem;
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_release();
  const int L = prefix_len(g, b);
  const int n_pages = (L + g.page_size - 1) / g.page_size;
  for (int p = tid; p < n_pages; p += SEL_THREADS) {
    float m = -CUDART_INF_F;
    for (int kvh = 0; kvh < g.hkv; ++kvh) m = fmaxf(m, scores[((long long)b * g.hkv + kvh) * g.max_pages + p]);
    sel_key[p] = order_key(m);
  }
  const bool keep_all = k >= n_pages;
  unsigned prefix = 0u, mask = 0u;
  int rem = keep_all ? n_pages : k;  // pages still to take among those matching prefix under mask
  for (int shift = 24; shift >= 0 && !keep_all; shift -= 8) {
    for (int i = tid; i < 256; i += SEL_THREADS) hist[i] = 0;
    __syncthreads();  // keys written (first pass), histogram cleared
    for (int p0 = warp * 32; p0 < n_pages; p0 += SEL_THREADS) {  // whole warps: the lanes of a bin add once
      const int p = p0 + lane;
      const unsigned key = p < n_pages ? sel_key[p] : 0u;
      const bool in = p < n_pages && (key & mask) == prefix;
      const int bin = in ? (int)((key >> shift) & 255u) : -1;
      const unsigned same = __match_any_sync(0xffffffffu, bin);
      if (in && lane == __ffs(same) - 1) atomicAdd(&hist[bin], __popc(same));
    }
    __syncthreads();
    if (warp == 0) {  // lane l holds digits 255 - 8l down to 248 - 8l
      int c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - 8 * lane - j];
        sum += c[j];
      }
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= rem);  // non-empty: the counts add up to >= rem
      if (lane == __ffs(hit) - 1) {
        int cum = incl - sum;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (cum + c[j] >= rem) {
            s_prefix = prefix | ((unsigned)(255 - 8 * lane - j) << shift);
            s_rem = rem - cum;
            break;
          }
          cum += c[j];
        }
      }
    }
    __syncthreads();
    prefix = s_prefix;
    rem = s_rem;
    mask |= 255u << shift;
  }
  __syncthreads();  // keys visible (keep_all skipped the passes)
  // prefix is now the k-th largest key; the rem lowest-indexed pages equal to it are kept
  const int C = (n_pages + SEL_THREADS - 1) / SEL_THREADS, lo = min(tid * C, n_pages), hi = min(lo + C, n_pages);
  int n_eq = 0;
  for (int p = lo; p < hi && !keep_all; ++p) n_eq += sel_key[p] == prefix;
  int total;
  int eq_rank = block_exclusive_scan(n_eq, wsum, &total);
  int n_keep = 0, tokens = 0;
  for (int p = lo; p < hi; ++p) {
    const unsigned key = sel_key[p];
    bool keep = keep_all || key > prefix;
    if (!keep_all && key == prefix) keep = eq_rank++ < rem;
    if (keep) {
      ++n_keep;
      tokens += min(g.page_size, L - p * g.page_size);
    }
  }
  int kept_total;
  int pos = block_exclusive_scan(n_keep, wsum, &kept_total);
  int tok_total;
  block_exclusive_scan(tokens, wsum, &tok_total);
  eq_rank -= n_eq;  // this run's first rank among the equal pages, again
  for (int p = lo; p < hi; ++p) {
    const unsigned key = sel_key[p];
    bool keep = keep_all || key > prefix;
    if (!keep_all && key == prefix) keep = eq_rank++ < rem;
    if (keep) kept_table[(long long)b * k + pos++] = g.page_table[(long long)b * g.max_pages + p];
  }
  for (int j = kept_total + tid; j < k; j += SEL_THREADS) kept_table[(long long)b * k + j] = -1;
  if (tid == 0) kept_lens[b] = tok_total;
}

// Residual at a dense step, per row of [b, Hq, B]: R_O = (O~/l)_dense -
// (O~/l)_sparse, R_lse = lse_dense - lse_sparse; a row with no prefix keys
// stores R_lse = -inf (no block-external part).
__global__ void __launch_bounds__(256) residual_capture_kernel(int rows, int d, fbk_partial dense, fbk_partial sparse,
                                                               float *__restrict__ r_o, float *__restrict__ r_lse) {
  pdl_wait();
  pdl_release();
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < (long long)rows * d;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long r = idx / d;
    const bool empty = dense.m[r] == -CUDART_INF_F;
    r_o[idx] = empty ? 0.f : dense.o_unnorm[idx] / dense.l[r] - sparse.o_unnorm[idx] / sparse.l[r];
    if (idx % d == 0)
      r_lse[r] = empty ? -CUDART_INF_F
                       : (dense.m[r] + logf(dense.l[r])) - (sparse.m[r] + logf(sparse.l[r]));
  }
}

// The block-external state at a later step: (O~/l)_sparse + R_O with
// m = lse_sparse + R_lse and l = 1; rows with R_lse = -inf get (0, -inf, 0).
__global__ void __launch_bounds__(256) residual_apply_kernel(int rows, int d, fbk_partial sparse,
                                                             const float *__restrict__ r_o,
                                                             const float *__restrict__ r_lse, fbk_partial ext) {
  pdl_wait();
  pdl_release();
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < (long long)rows * d;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long r = idx / d;
    const bool empty = r_lse[r] == -CUDART_INF_F;
    ext.o_unnorm[idx] = empty ? 0.f : sparse.o_unnorm[idx] / sparse.l[r] + r_o[idx];
    if (idx % d == 0) {
      ext.m[r] = empty ? -CUDART_INF_F : sparse.m[r] + logf(sparse.l[r]) + r_lse[r];
      ext.l[r] = empty ? 0.f : 1.f;
    }
  }
}

unsigned grid_for(long long n, int sms) {
  const long long want = (n + 255) / 256, cap = 8ll * sms;
  return (unsigned)std::max<long long>(1, std::min(want, cap));
}

}  // namespace

cudaError_t launch_page_means(const Geometry &g, float *means, cudaStream_t st) {
  const long long ctas = (long long)g.batch * g.max_pages;
  if (ctas > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  if (g.d == 128) return launch_pdl(page_means_kernel<128>, dim3((unsigned)ctas), dim3(MEAN_THREADS), 0, st, g, means);
  return launch_pdl(page_means_kernel<64>, dim3((unsigned)ctas), dim3(MEAN_THREADS), 0, st, g, means);
}

cudaError_t launch_select_pages(const Geometry &g, const __nv_bfloat16 *q, const float *means, int k, float *qrot,
                                float *scores, int *kept_table, int *kept_lens, int sms, cudaStream_t st) {
  const long long nrot = (long long)g.batch * g.blk * g.hq * (g.d / 2);
  cudaError_t e = launch_pdl(rotate_queries_kernel, dim3(grid_for(nrot, sms)), dim3(256), 0, st, g, q, qrot);
  if (e != cudaSuccess) return e;
  const int tiles = (g.max_pages + SCORE_PAGES - 1) / SCORE_PAGES;
  const long long ctas = (long long)g.batch * g.hkv * tiles;
  if (ctas > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  if (g.d == 128) {
    e = cudaFuncSetAttribute(page_scores_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, score_smem_bytes(128));
    if (e == cudaSuccess)
      e = launch_pdl(page_scores_kernel<128>, dim3((unsigned)ctas), dim3(SCORE_THREADS), score_smem_bytes(128), st, g,
                     (const float *)qrot, means, scores, tiles);
  } else {
    e = cudaFuncSetAttribute(page_scores_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, score_smem_bytes(64));
    if (e == cudaSuccess)
      e = launch_pdl(page_scores_kernel<64>, dim3((unsigned)ctas), dim3(SCORE_THREADS), score_smem_bytes(64), st, g,
                     (const float *)qrot, means, scores, tiles);
  }
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)g.max_pages * sizeof(unsigned);
  if (smem > 40 * 1024) {
    e = cudaFuncSetAttribute(select_pages_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(select_pages_kernel, dim3(g.batch), dim3(SEL_THREADS), smem, st, g, (const float *)scores, k,
                    kept_table, kept_lens);
}

cudaError_t launch_residual_capture(int rows, int d, const fbk_partial &dense, const fbk_partial &sparse, float *r_o,
                                    float *r_lse, int sms, cudaStream_t st) {
  return launch_pdl(residual_capture_kernel, dim3(grid_for((long long)rows * d, sms)), dim3(256), 0, st, rows, d,
                    dense, sparse, r_o, r_lse);
}

cudaError_t launch_residual_apply(int rows, int d, const fbk_partial &sparse, const float *r_o, const float *r_lse,
                                  const fbk_partial &ext, int sms, cudaStream_t st) {
  return launch_pdl(residual_apply_kernel, dim3(grid_for((long long)rows * d, sms)), dim3(256), 0, st, rows, d,
                    sparse, r_o, r_lse, ext);
}

}  // namespace fbk
