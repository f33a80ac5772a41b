// Uncached reference attention on CUDA cores (fp32), independent of the
// cached-state kernels: block query row t of (b, h) at position L_b + t
// attends to [cache rows 0..L_b-1 ; RoPE(k_blk)] with one online-softmax pass
// (LaCache App. B.2: FlashAttention over all key blocks, no cache). It is the
// computation FACache must reproduce (LaCache §3.1).
//
// One warp per query row. The rotated query row sits in shared memory; lane j
// scores key c0 + j of each 32-key chunk, the chunk's max and sum are warp
// reductions, and each lane accumulates d/32 output columns.
#include "launch.h"

namespace fbk {
namespace {

constexpr int WARPS = 8;

template <int D, bool F32OUT>
__global__ void __launch_bounds__(WARPS * 32) full_ref_kernel(
    Geometry g, const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ kb,
    const __nv_bfloat16 *__restrict__ vb, void *__restrict__ out, float *__restrict__ lse) {
  constexpr int HALF = D / 2, CPL = D / 32;
  __shared__ float qs[WARPS][D];
  const int bh = blockIdx.y, b = bh / g.hq, h = bh % g.hq;
  const int kvh = (int)(((long long)h * g.hkv) / g.hq);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * WARPS + warp;
  if (t >= g.blk) return;
  const int L = prefix_len(g, b);
  const int pos = L + t;

  const __nv_bfloat16 *qsrc = q + (((long long)b * g.blk + t) * g.hq + h) * D;
  for (int i = lane; i < HALF; i += 32) {
    const float x1 = __bfloat162float(qsrc[i]), x2 = __bfloat162float(qsrc[i + HALF]);
    const float2 c = rope_cs_f32(pos, g.inv_freq_over_pi[i]);
    qs[warp][i] = x1 * c.x - x2 * c.y;
    qs[warp][i + HALF] = x2 * c.x + x1 * c.y;
  }
  __syncwarp();

  float m = -CUDART_INF_F, l = 0.f, o[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) o[c] = 0.f;
  const int n_keys = L + g.blk;
  for (int c0 = 0; c0 < n_keys; c0 += 32) {
    const int j = c0 + lane;
    float s = -CUDART_INF_F;
    const __nv_bfloat16 *vrow = nullptr;
    if (j < L) {
      const long long row = cache_row(g, b, kvh, j);
      if (row >= 0) {
        const __nv_bfloat16 *krow = g.kc + row * D;
        float acc = 0.f;
        for (int k = 0; k < D; k += 2) {
          const float2 kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(krow + k));
          acc += qs[warp][k] * kv.x + qs[warp][k + 1] * kv.y;
        }
        s = acc * g.tau;
        vrow = g.vc + row * D;
      }
    } else if (j < n_keys) {
      const int tj = j - L;
      const __nv_bfloat16 *krow = kb + (((long long)b * g.blk + tj) * g.hkv + kvh) * D;
      float acc = 0.f;
      for (int i = 0; i < HALF; ++i) {
        const float x1 = __bfloat162float(krow[i]), x2 = __bfloat162float(krow[i + HALF]);
        const float2 c = rope_cs_f32(L + tj, g.inv_freq_over_pi[i]);
        acc += qs[warp][i] * (x1 * c.x - x2 * c.y) + qs[warp][i + HALF] * (x2 * c.x + x1 * c.y);
      }
      s = acc * g.tau;
      vrow = vb + (((long long)b * g.blk + tj) * g.hkv + kvh) * D;
    }
    const float mn = fmaxf(m, warp_max(s));
    const float alpha = lse_weight(m, mn);
    const float p = vrow ? expf(s - mn) : 0.f;
    l = alpha * l + warp_sum(p);
    m = mn;
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[c] *= alpha;
    for (int jj = 0; jj < 32; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const unsigned long long vp = __shfl_sync(0xffffffffu, (unsigned long long)vrow, jj);
      if (pj != 0.f) {
        const __nv_bfloat16 *vr = reinterpret_cast<const __nv_bfloat16 *>(vp);
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[c] += pj * __bfloat162float(vr[lane * CPL + c]);
      }
    }
  }
  const float inv = 1.f / l;
  const long long orow = (((long long)b * g.blk + t) * g.hq + h) * D + lane * CPL;
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    if (F32OUT)
      reinterpret_cast<float *>(out)[orow + c] = o[c] * inv;
    else
      reinterpret_cast<__nv_bfloat16 *>(out)[orow + c] = __float2bfloat16_rn(o[c] * inv);
  }
  if (lse && lane == 0) lse[((long long)b * g.hq + h) * g.blk + t] = m + logf(l);
}

}  // namespace

cudaError_t launch_full_ref(const Geometry &g, const __nv_bfloat16 *q, const __nv_bfloat16 *kb,
                            const __nv_bfloat16 *vb, void *out, float *lse, bool f32_out,
                            cudaStream_t st) {
  dim3 grid((g.blk + WARPS - 1) / WARPS, g.batch * g.hq);
  if (g.d == 128) {
    if (f32_out)
      full_ref_kernel<128, true><<<grid, WARPS * 32, 0, st>>>(g, q, kb, vb, out, lse);
    else
      full_ref_kernel<128, false><<<grid, WARPS * 32, 0, st>>>(g, q, kb, vb, out, lse);
  } else {
    if (f32_out)
      full_ref_kernel<64, true><<<grid, WARPS * 32, 0, st>>>(g, q, kb, vb, out, lse);
    else
      full_ref_kernel<64, false><<<grid, WARPS * 32, 0, st>>>(g, q, kb, vb, out, lse);
  }
  return cudaGetLastError();
}

}  // namespace fbk
