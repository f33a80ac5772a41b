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
// All of it is small next to the prefix itself: the mean keys read the cache
// once per committed block, the scores read the means and the block's queries,
// and the residual kernels touch one state.
#include "launch.h"
#include "sparse_prefix.h"

namespace fbk {
namespace {

// Mean key of every logical page (b, lp) of every kv-head: [b, max_pages, Hkv, d]
// fp32. One CTA per (b, lp); pages past the prefix are left untouched.
__global__ void __launch_bounds__(256) page_means_kernel(Geometry g, float *__restrict__ means) {
  const int b = blockIdx.x / g.max_pages, lp = blockIdx.x % g.max_pages;
  pdl_wait();
  pdl_release();
  const int L = prefix_len(g, b);
  const int t0 = lp * g.page_size, n = min(g.page_size, L - t0);
  if (n <= 0) return;
  const int pid = g.page_table[(long long)b * g.max_pages + lp];
  if (pid < 0 || (long long)pid >= g.num_pages) {
    raise_flag(g, FBK_DEVERR_PAGE_ID);
    return;
  }
  const int cols = g.hkv * g.d;
  for (int c = threadIdx.x; c < cols; c += blockDim.x) {
    const int kvh = c / g.d, i = c % g.d;
    const __nv_bfloat16 *src = g.kc + (((long long)pid * g.hkv + kvh) * g.page_size) * g.d + i;
    float s = 0.f;
    for (int t = 0; t < n; ++t) s += __bfloat162float(src[(long long)t * g.d]);
    means[(((long long)b * g.max_pages + lp) * g.hkv + kvh) * g.d + i] = s / (float)n;
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

// Score of every logical page: one warp per (b, lp), the largest
// tau <qrot[b, t, h], kbar[b, lp, kv(h)]> over t and h. Pages past the prefix
// score -inf.
__global__ void __launch_bounds__(256) page_scores_kernel(Geometry g, const float *__restrict__ qrot,
                                                          const float *__restrict__ means,
                                                          float *__restrict__ scores) {
  pdl_wait();
  pdl_release();
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= (long long)g.batch * g.max_pages) return;
  const int b = (int)(warp / g.max_pages), lp = (int)(warp % g.max_pages);
  const int L = prefix_len(g, b);
  float best = -CUDART_INF_F;
  if (lp * g.page_size < L) {
    for (int h = 0; h < g.hq; ++h) {
      const float *kbar = means + (((long long)b * g.max_pages + lp) * g.hkv + h / g.group) * g.d;
      for (int t = 0; t < g.blk; ++t) {
        const float *qv = qrot + (((long long)b * g.blk + t) * g.hq + h) * g.d;
        float s = 0.f;
        for (int i = lane; i < g.d; i += 32) s += qv[i] * kbar[i];
        s = warp_sum(s);
        best = fmaxf(best, g.tau * s);
      }
    }
  }
  if (lane == 0) scores[warp] = best;
}

// Top-k pages of each sequence (one CTA per sequence): a page is kept when
// fewer than k pages beat it (higher score, or equal score and lower index).
// Writes the kept physical pages in increasing logical order and their token
// count (a partial last page counts its tokens; being the highest page, it
// is last when kept).
__global__ void __launch_bounds__(1024) select_pages_kernel(Geometry g, const float *__restrict__ scores, int k,
                                                            int *__restrict__ kept_table, int *__restrict__ kept_lens) {
  extern __shared__ float sel_smem[];
  float *sc = sel_smem;
  int *keep = reinterpret_cast<int *>(sc + g.max_pages);
  const int b = blockIdx.x;
  pdl_wait();
  pdl_release();
  const int L = prefix_len(g, b);
  const int n_pages = (L + g.page_size - 1) / g.page_size;
  for (int p = threadIdx.x; p < n_pages; p += blockDim.x) sc[p] = scores[(long long)b * g.max_pages + p];
  __syncthreads();
  for (int p = threadIdx.x; p < n_pages; p += blockDim.x) {
    int beaten = 0;
    for (int o = 0; o < n_pages; ++o) beaten += (sc[o] > sc[p]) || (sc[o] == sc[p] && o < p);
    keep[p] = beaten < k ? 1 : 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // n_pages is at most max_pages: a serial pass is short
    int pos = 0, tokens = 0;
    for (int p = 0; p < n_pages; ++p) {
      if (!keep[p]) continue;
      kept_table[(long long)b * k + pos++] = g.page_table[(long long)b * g.max_pages + p];
      tokens += min(g.page_size, L - p * g.page_size);
    }
    for (; pos < k; ++pos) kept_table[(long long)b * k + pos] = -1;
    kept_lens[b] = tokens;
  }
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
  return launch_pdl(page_means_kernel, dim3((unsigned)ctas), dim3(256), 0, st, g, means);
}

cudaError_t launch_select_pages(const Geometry &g, const __nv_bfloat16 *q, const float *means, int k, float *qrot,
                                float *scores, int *kept_table, int *kept_lens, int sms, cudaStream_t st) {
  const long long nrot = (long long)g.batch * g.blk * g.hq * (g.d / 2);
  cudaError_t e = launch_pdl(rotate_queries_kernel, dim3(grid_for(nrot, sms)), dim3(256), 0, st, g, q, qrot);
  if (e != cudaSuccess) return e;
  const long long warps = (long long)g.batch * g.max_pages;
  e = launch_pdl(page_scores_kernel, dim3((unsigned)((warps + 7) / 8)), dim3(256), 0, st, g,
                 (const float *)qrot, means, scores);
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)g.max_pages * (sizeof(float) + sizeof(int));
  if (smem > 48 * 1024) {
    e = cudaFuncSetAttribute(select_pages_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  return launch_pdl(select_pages_kernel, dim3(g.batch), dim3(1024), smem, st, g, (const float *)scores, k,
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
