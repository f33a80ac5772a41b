// Commit a finished block: RoPECache append (LaCache §3.3.2, Eq. 1).
//
// For sequence b with committed length L: K^[t] = RoPE(k_blk[t], L + t) in
// fp64, rounded once to bf16 (nearest even); V copied bit for bit; both stored
// at cache slots L .. L+B-1 (contiguous rows or pages); then prefix_lens[b]
// becomes L + B.
//
// Each sequence is handled by one cluster of 8 CTAs, CTA c taking block tokens
// [c*B/8, (c+1)*B/8) of every kv-head. Every CTA reads L, the cluster barrier
// (hardware, no spinning) guarantees all reads happened, and only then does
// CTA 0 advance prefix_lens[b]. The fp64 cos/sin of each (position, pair)
// are computed once per CTA into shared memory and reused by all kv-heads.
// The block K/V loads of the first batch are issued before the length is
// read, so the two memory round trips overlap.
#include <cooperative_groups.h>

#include "launch.h"

namespace fbk {
namespace {

namespace cg = cooperative_groups;

constexpr int THREADS = 512;
constexpr int CLUSTER = 8;
constexpr int MAX_TOK = 64 / CLUSTER;  // block_len <= 64
constexpr int KB = 2;                  // K items (8 rotation pairs) per thread per batch
constexpr int VB = 4;                  // V 16-byte chunks per thread per batch

template <int D>
__global__ void __cluster_dims__(CLUSTER, 1, 1) __launch_bounds__(THREADS)
    commit_kernel(Geometry g, const __nv_bfloat16 *__restrict__ kb, const __nv_bfloat16 *__restrict__ vb,
                  __nv_bfloat16 *__restrict__ kc, __nv_bfloat16 *__restrict__ vc, int *lens) {
  constexpr int HALF = D / 2, KI = D / 16, VI = D / 8;
  __shared__ int s_ok, s_L;
  __shared__ double2 tab[MAX_TOK * HALF];
  const int b = blockIdx.y, crank = blockIdx.x, blk = g.blk;
  const int t0 = crank * blk / CLUSTER, t1 = (crank + 1) * blk / CLUSTER, nt = t1 - t0;
  const int nk = nt * g.hkv * KI, nv = nt * g.hkv * VI;
  pdl_release();
  pdl_wait();

  int L = 0;
  bool first = true;
  for (int kbase = 0, vbase = 0; first || kbase < nk || vbase < nv; kbase += THREADS * KB, vbase += THREADS * VB) {
    // block K and V do not depend on L: the first batch is requested before the
    // length is known, so both round trips overlap
    uint4 xa[KB], xb[KB], xv[VB];
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      const int item = kbase + threadIdx.x + THREADS * k;
      if (item < nk) {
        const int c = item % KI, rowi = item / KI, kvh = rowi % g.hkv, t = t0 + rowi / g.hkv;
        const uint4 *src = reinterpret_cast<const uint4 *>(kb + (((long long)b * blk + t) * g.hkv + kvh) * D);
        xa[k] = src[c];
        xb[k] = src[c + KI];
      }
    }
#pragma unroll
    for (int k = 0; k < VB; ++k) {
      const int item = vbase + threadIdx.x + THREADS * k;
      if (item < nv) {
        const int ch = item % VI, rowi = item / VI, kvh = rowi % g.hkv, t = t0 + rowi / g.hkv;
        xv[k] = reinterpret_cast<const uint4 *>(vb + (((long long)b * blk + t) * g.hkv + kvh) * D)[ch];
      }
    }
    if (first) {
      first = false;
      if (threadIdx.x == 0) {
        const int Lb = lens[b];
        bool ok = Lb >= 0 && (long long)Lb + blk <= seq_capacity(g);
        if (ok && g.paged) {
          for (long long pg = (long long)Lb >> g.page_shift; pg <= ((long long)Lb + blk - 1) >> g.page_shift; ++pg) {
            const int id = g.page_table[(long long)b * g.max_pages + pg];
            if (id < 0 || (long long)id >= g.num_pages) ok = false;
          }
          if (!ok && crank == 0) raise_flag(g, FBK_DEVERR_PAGE_ID);
        }
        if (!ok && crank == 0) raise_flag(g, FBK_DEVERR_COMMIT);
        s_ok = ok;
        s_L = Lb;
      }
      cg::this_cluster().sync();  // every CTA of this sequence has read prefix_lens[b]
      L = s_L;
      if (!s_ok) return;
      if (crank == 0 && threadIdx.x == 0) lens[b] = L + blk;
      if (nt == 0) return;
      // entry of pair i = 8c + e sits at e * KI + c: the 8 lanes that rotate
      // chunks c = 0..7 of one row read 8 consecutive entries (no bank conflict)
      for (int idx = threadIdx.x; idx < nt * HALF; idx += THREADS) {
        const int tl = idx / HALF, i = idx % HALF;
        double c, sn;
        rope_cs_f64(L + t0 + tl, g.inv_freq_over_pi[i], &c, &sn);
        tab[tl * HALF + (i & 7) * KI + (i >> 3)] = make_double2(c, sn);
      }
      __syncthreads();
    }
    // K: an item is 8 rotation pairs, the 16-byte chunk c of each half of a row
#pragma unroll
    for (int k = 0; k < KB; ++k) {
      const int item = kbase + threadIdx.x + THREADS * k;
      if (item < nk) {
        const int c = item % KI, rowi = item / KI, kvh = rowi % g.hkv, tl = rowi / g.hkv;
        const uint32_t aw[4] = {xa[k].x, xa[k].y, xa[k].z, xa[k].w};
        const uint32_t bw[4] = {xb[k].x, xb[k].y, xb[k].z, xb[k].w};
        uint32_t y1[4], y2[4];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const uint32_t ha = (e & 1) ? (aw[e >> 1] >> 16) : (aw[e >> 1] & 0xffffu);
          const uint32_t hb = (e & 1) ? (bw[e >> 1] >> 16) : (bw[e >> 1] & 0xffffu);
          const double x1 = (double)bf16_bits_to_f32((uint16_t)ha), x2 = (double)bf16_bits_to_f32((uint16_t)hb);
          const double2 cs = tab[tl * HALF + e * KI + c];
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
        uint4 *dst = reinterpret_cast<uint4 *>(kc + cache_row(g, b, kvh, (long long)L + t0 + tl) * D);
        dst[c] = make_uint4(y1[0], y1[1], y1[2], y1[3]);
        dst[c + KI] = make_uint4(y2[0], y2[1], y2[2], y2[3]);
      }
    }
    // V: bit-exact 16-byte copies
#pragma unroll
    for (int k = 0; k < VB; ++k) {
      const int item = vbase + threadIdx.x + THREADS * k;
      if (item < nv) {
        const int ch = item % VI, rowi = item / VI, kvh = rowi % g.hkv, t = t0 + rowi / g.hkv;
        reinterpret_cast<uint4 *>(vc + cache_row(g, b, kvh, (long long)L + t) * D)[ch] = xv[k];
      }
    }
  }
}

}  // namespace

cudaError_t launch_commit(const Geometry &g, const __nv_bfloat16 *kb, const __nv_bfloat16 *vb,
                          __nv_bfloat16 *kc, __nv_bfloat16 *vc, int *lens, cudaStream_t st) {
  dim3 grid(CLUSTER, g.batch);
  if (g.d == 128) return launch_pdl(commit_kernel<128>, grid, dim3(THREADS), 0, st, g, kb, vb, kc, vc, lens);
  return launch_pdl(commit_kernel<64>, grid, dim3(THREADS), 0, st, g, kb, vb, kc, vc, lens);
}

}  // namespace fbk
