// Commit a finished block: RoPECache append (LaCache §3.3.2, Eq. 1).
//
// For sequence b with committed length L: K^[t] = RoPE(k_blk[t], L + t) in
// fp64, rounded once to bf16 (nearest even); V copied bit for bit; both stored
// at cache slots L .. L+B-1 (contiguous rows or pages); then prefix_lens[b]
// becomes L + B. One CTA per sequence, so the length is read before and
// written after every slot of that sequence, with no race between CTAs.
#include "launch.h"

namespace fbk {
namespace {

constexpr int THREADS = 256;

template <int D>
__global__ void __launch_bounds__(THREADS) commit_kernel(Geometry g,
                                                         const __nv_bfloat16 *__restrict__ kb,
                                                         const __nv_bfloat16 *__restrict__ vb,
                                                         __nv_bfloat16 *__restrict__ kc,
                                                         __nv_bfloat16 *__restrict__ vc, int *lens) {
  constexpr int HALF = D / 2;
  __shared__ int s_ok, s_L;
  const int b = blockIdx.x, blk = g.blk;
  if (threadIdx.x == 0) {
    const int L = lens[b];
    bool ok = L >= 0 && (long long)L + blk <= seq_capacity(g);
    if (ok && g.paged) {
      for (long long pg = (long long)L >> g.page_shift; pg <= ((long long)L + blk - 1) >> g.page_shift; ++pg) {
        const int id = g.page_table[(long long)b * g.max_pages + pg];
        if (id < 0 || (long long)id >= g.num_pages) {
          raise_flag(g, FBK_DEVERR_PAGE_ID);
          ok = false;
        }
      }
    }
    if (!ok) raise_flag(g, FBK_DEVERR_COMMIT);
    s_ok = ok;
    s_L = L;
  }
  __syncthreads();
  if (!s_ok) return;
  const int L = s_L;

  for (int idx = threadIdx.x; idx < blk * g.hkv * HALF; idx += THREADS) {
    const int i = idx % HALF, rowi = idx / HALF, kvh = rowi % g.hkv, t = rowi / g.hkv;
    const __nv_bfloat16 *src = kb + (((long long)b * blk + t) * g.hkv + kvh) * D;
    const double x1 = (double)__bfloat162float(src[i]);
    const double x2 = (double)__bfloat162float(src[i + HALF]);
    double c, s;
    rope_cs_f64(L + t, g.inv_freq_over_pi[i], &c, &s);
    // plain rounded products and differences (no fused multiply-add)
    const double y1 = __dsub_rn(__dmul_rn(x1, c), __dmul_rn(x2, s));
    const double y2 = __dadd_rn(__dmul_rn(x2, c), __dmul_rn(x1, s));
    const long long row = cache_row(g, b, kvh, (long long)L + t);
    kc[row * D + i] = __ushort_as_bfloat16(f64_to_bf16_rne(y1));
    kc[row * D + i + HALF] = __ushort_as_bfloat16(f64_to_bf16_rne(y2));
  }
  for (int idx = threadIdx.x; idx < blk * g.hkv * (D / 8); idx += THREADS) {
    const int ch = idx % (D / 8), rowi = idx / (D / 8), kvh = rowi % g.hkv, t = rowi / g.hkv;
    const long long row = cache_row(g, b, kvh, (long long)L + t);
    *reinterpret_cast<uint4 *>(vc + row * D + ch * 8) =
        *reinterpret_cast<const uint4 *>(vb + (((long long)b * blk + t) * g.hkv + kvh) * D + ch * 8);
  }
  __syncthreads();
  if (threadIdx.x == 0) lens[b] = L + blk;
}

}  // namespace

cudaError_t launch_commit(const Geometry &g, const __nv_bfloat16 *kb, const __nv_bfloat16 *vb,
                          __nv_bfloat16 *kc, __nv_bfloat16 *vc, int *lens, cudaStream_t st) {
  if (g.d == 128)
    commit_kernel<128><<<g.batch, THREADS, 0, st>>>(g, kb, vb, kc, vc, lens);
  else
    commit_kernel<64><<<g.batch, THREADS, 0, st>>>(g, kb, vb, kc, vc, lens);
  return cudaGetLastError();
}

}  // namespace fbk
