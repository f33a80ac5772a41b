// Commit a finished block: RoPECache append (LaCache §3.3.2, Eq. 1).
//
// For sequence b with committed length L: K^[t] = RoPE(k_blk[t], L + t) in
// fp64, rounded once to bf16 (nearest even); V copied bit for bit; both stored
// at cache slots L .. L+B-1 (contiguous rows or pages); then prefix_lens[b]
// becomes L + B.
//
// Two kernels, chained by programmatic dependent launch:
//  * commit_rows_kernel: one CTA per (sequence, block token, group of up to
//    16 kv-heads). It reads prefix_lens[b] but never writes it, so no CTA can
//    see a length another CTA already advanced. The block K/V loads do not
//    depend on L and are issued first; the fp64 cos/sin of the token's
//    position is computed once per CTA while they fly.
//  * commit_lens_kernel: one CTA. Its wait returns only once every CTA of the
//    first kernel has completed, so all reads of prefix_lens are done; it then
//    advances prefix_lens[b] for the sequences whose block fit and raises the
//    flags for the others.
// Both kernels decide "fits" from the same inputs with the same test.
#include "launch.h"

namespace fbk {
namespace {

constexpr int THREADS = 128;
constexpr int HG = 16;  // kv-heads per CTA

// L + B fits in the sequence's capacity and every page it touches is valid.
__device__ __forceinline__ bool block_fits(const Geometry &g, int b, int L, bool *bad_page) {
  *bad_page = false;
  if (L < 0 || (long long)L + g.blk > seq_capacity(g)) return false;
  if (g.paged) {
    for (long long pg = (long long)L >> g.page_shift; pg <= ((long long)L + g.blk - 1) >> g.page_shift; ++pg) {
      const int id = g.page_table[(long long)b * g.max_pages + pg];
      if (id < 0 || (long long)id >= g.num_pages) *bad_page = true;
    }
  }
  return !*bad_page;
}

template <int D>
__global__ void __launch_bounds__(THREADS) commit_rows_kernel(Geometry g, const __nv_bfloat16 *__restrict__ kb,
                                                             const __nv_bfloat16 *__restrict__ vb,
                                                             __nv_bfloat16 *__restrict__ kc,
                                                             __nv_bfloat16 *__restrict__ vc, int ngroups) {
  constexpr int HALF = D / 2, KI = D / 16, VI = D / 8;
  constexpr int KB = (HG * KI + THREADS - 1) / THREADS, VB = (HG * VI + THREADS - 1) / THREADS;
  __shared__ double2 tab[HALF];  // pair i = 8c + e at e * KI + c (conflict-free reads)
  __shared__ int s_ok;
  const int gi = blockIdx.x % ngroups, bt = blockIdx.x / ngroups, t = bt % g.blk, b = bt / g.blk;
  const int h0 = gi * HG, nh = min(HG, g.hkv - h0);
  const int nk = nh * KI, nv = nh * VI;
  pdl_wait();
  pdl_release();

  // block K and V of token t, heads h0 .. h0+nh-1 (independent of L)
  const long long row0 = ((long long)b * g.blk + t) * g.hkv + h0;
  uint4 xa[KB], xb[KB], xv[VB];
#pragma unroll
  for (int k = 0; k < KB; ++k) {
    const int item = threadIdx.x + THREADS * k;
    if (item < nk) {
      const uint4 *src = reinterpret_cast<const uint4 *>(kb + (row0 + item / KI) * D);
      xa[k] = src[item % KI];
      xb[k] = src[item % KI + KI];
    }
  }
#pragma unroll
  for (int k = 0; k < VB; ++k) {
    const int item = threadIdx.x + THREADS * k;
    if (item < nv) xv[k] = reinterpret_cast<const uint4 *>(vb + (row0 + item / VI) * D)[item % VI];
  }
  const int L = g.lens[b];
  if (threadIdx.x == 0) {
    bool bad_page;
    s_ok = block_fits(g, b, L, &bad_page);
  }
  for (int i = threadIdx.x; i < HALF; i += THREADS) {
    double c, s;
    rope_cs_f64(L + t, g.inv_freq_over_pi[i], &c, &s);
    tab[(i & 7) * KI + (i >> 3)] = make_double2(c, s);
  }
  __syncthreads();
  if (!s_ok) return;

  // K: an item is 8 rotation pairs, the 16-byte chunk c of each half of a row
#pragma unroll
  for (int k = 0; k < KB; ++k) {
    const int item = threadIdx.x + THREADS * k;
    if (item < nk) {
      const int c = item % KI, kvh = h0 + item / KI;
      const uint32_t aw[4] = {xa[k].x, xa[k].y, xa[k].z, xa[k].w};
      const uint32_t bw[4] = {xb[k].x, xb[k].y, xb[k].z, xb[k].w};
      uint32_t y1[4], y2[4];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t ha = (e & 1) ? (aw[e >> 1] >> 16) : (aw[e >> 1] & 0xffffu);
        const uint32_t hb = (e & 1) ? (bw[e >> 1] >> 16) : (bw[e >> 1] & 0xffffu);
        const double x1 = (double)bf16_bits_to_f32((uint16_t)ha), x2 = (double)bf16_bits_to_f32((uint16_t)hb);
        const double2 cs = tab[e * KI + c];
        // plain rounded products and differences (no fused multiply-add)
        const uint32_t r1 = f64_to_bf16_rne(__dsub_rn(__dmul_rn(x1, cs.x), __dmul_rn(x2, cs.y)));
        const uint32_t r2 = f64_to_bf16_rne(__dadd_rn(__dmul_rn(x2, cs.x), __dmul_rn(x1, cs.y)));
        if (e & 1) {
          y1[e >> 1] |= r1 << 16;
          y2[e >> 1] |= r2 << 16;
        } else {
          y1[e >> 1] = r1;
          y2[e >> 1] = r2;
        }
      }
      uint4 *dst = reinterpret_cast<uint4 *>(kc + cache_row(g, b, kvh, (long long)L + t) * D);
      dst[c] = make_uint4(y1[0], y1[1], y1[2], y1[3]);
      dst[c + KI] = make_uint4(y2[0], y2[1], y2[2], y2[3]);
    }
  }
  // V: bit-exact 16-byte copies
#pragma unroll
  for (int k = 0; k < VB; ++k) {
    const int item = threadIdx.x + THREADS * k;
    if (item < nv)
      reinterpret_cast<uint4 *>(vc + cache_row(g, b, h0 + item / VI, (long long)L + t) * D)[item % VI] = xv[k];
  }
}

__global__ void __launch_bounds__(1024) commit_lens_kernel(Geometry g, int *lens) {
  pdl_wait();  // every CTA of commit_rows_kernel has completed: no read of prefix_lens is pending
  pdl_release();
  for (int b = threadIdx.x; b < g.batch; b += blockDim.x) {
    const int L = lens[b];
    bool bad_page;
    if (block_fits(g, b, L, &bad_page)) {
      lens[b] = L + g.blk;
    } else {
      if (bad_page) raise_flag(g, FBK_DEVERR_PAGE_ID);
      raise_flag(g, FBK_DEVERR_COMMIT);
    }
  }
}

}  // namespace

cudaError_t launch_commit(const Geometry &g, const __nv_bfloat16 *kb, const __nv_bfloat16 *vb,
                          __nv_bfloat16 *kc, __nv_bfloat16 *vc, int *lens, cudaStream_t st) {
  const int ngroups = (g.hkv + HG - 1) / HG;
  const long long ctas = (long long)g.batch * g.blk * ngroups;
  if (ctas > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  cudaError_t e = g.d == 128
                      ? launch_pdl(commit_rows_kernel<128>, dim3((unsigned)ctas), dim3(THREADS), 0, st, g, kb,
                                   vb, kc, vc, ngroups)
                      : launch_pdl(commit_rows_kernel<64>, dim3((unsigned)ctas), dim3(THREADS), 0, st, g, kb,
                                   vb, kc, vc, ngroups);
  if (e != cudaSuccess) return e;
  const int nthreads = g.batch < 1024 ? ((g.batch + 31) / 32) * 32 : 1024;
  return launch_pdl(commit_lens_kernel, dim3(1), dim3(nthreads), 0, st, g, lens);
}

}  // namespace fbk
