// One denoising step: in-block attention fused with the merge of the cached
// prefix state.
//
// For every block query row (sequence b, head h, token t) at position L_b + t:
//   S_j = tau <RoPE(q_t), RoPE(k_j)>, j < B (bidirectional, no mask),
//   block state m2 = max_j S_j, l2 = sum_j e^(S_j - m2), O~2 = sum_j e^(S_j - m2) v_j,
//   merged with the prefix state (O~1, m1, l1): m = max(m1, m2),
//   O = (e^(m1-m) O~1 + e^(m2-m) O~2) / (e^(m1-m) l1 + e^(m2-m) l2), lse = m + log l.
// This is FACache's "initialise from cache, process only the tiles that
// overlap the current block" (LaCache §3.3.3 and App. J) for the block's own
// query rows, i.e. FlashBlock's reuse of block-external attention with fresh
// block-internal attention (FlashBlock, Abstract).
//
// One CTA per (unit, chunk of 4*RPW query rows); everything in fp32 on CUDA
// cores (B <= 64 keys per row). Row max / sum are warp-shuffle reductions with
// lane j holding keys j and j+32.
#include "launch.h"

namespace fbk {
namespace {

constexpr int WARPS = 4;

struct Layout {
  int kp, k_off, v_off, q_off, p_off, cs_off, floats;
  __host__ __device__ Layout(int d, int blk, int rc) {
    kp = d + 4;
    k_off = 0;
    v_off = k_off + blk * kp;
    q_off = v_off + blk * d;
    p_off = q_off + rc * d;
    cs_off = p_off + rc * 64;
    cs_off = (cs_off + 1) & ~1;  // float2 alignment
    floats = cs_off + 2 * blk * (d / 2);
  }
};

template <int D, int RPW, bool F32OUT>
__global__ void __launch_bounds__(WARPS * 32) block_merge_kernel(
    Geometry g, const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ kb,
    const __nv_bfloat16 *__restrict__ vb, fbk_partial pfx, void *__restrict__ out,
    float *__restrict__ lse) {
  constexpr int RC = WARPS * RPW, CPL = D / 32, HALF = D / 2;
  extern __shared__ float4 smem_f4[];
  float *sm = reinterpret_cast<float *>(smem_f4);
  const Layout lay(D, g.blk, RC);
  float *Kf = sm + lay.k_off;
  float *Vf = sm + lay.v_off;
  float *Qf = sm + lay.q_off;
  float *Ps = sm + lay.p_off;
  float2 *cs = reinterpret_cast<float2 *>(sm + lay.cs_off);

  const int u = blockIdx.y, b = u / g.hkv, kvh = u % g.hkv;
  const int r0 = blockIdx.x * RC;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int L = g.lens[b];
  if (L < 0) {
    raise_flag(g, FBK_DEVERR_PREFIX_LEN);
    L = 0;
  }
  const int blk = g.blk;

  for (int idx = tid; idx < blk * HALF; idx += WARPS * 32)
    cs[idx] = rope_cs_f32(L + idx / HALF, g.inv_freq_over_pi[idx % HALF]);
  __syncthreads();

  for (int idx = tid; idx < blk * HALF; idx += WARPS * 32) {
    const int t = idx / HALF, i = idx % HALF;
    const __nv_bfloat16 *src = kb + (((long long)b * blk + t) * g.hkv + kvh) * D;
    const float x1 = __bfloat162float(src[i]), x2 = __bfloat162float(src[i + HALF]);
    const float2 c = cs[idx];
    Kf[t * lay.kp + i] = x1 * c.x - x2 * c.y;
    Kf[t * lay.kp + i + HALF] = x2 * c.x + x1 * c.y;
    const __nv_bfloat162 v2 = *reinterpret_cast<const __nv_bfloat162 *>(
        vb + (((long long)b * blk + t) * g.hkv + kvh) * D + 2 * i);
    const float2 vf = __bfloat1622float2(v2);
    Vf[t * D + 2 * i] = vf.x;
    Vf[t * D + 2 * i + 1] = vf.y;
  }
  for (int idx = tid; idx < RC * HALF; idx += WARPS * 32) {
    const int rr = idx / HALF, i = idx % HALF, r = r0 + rr;
    float y1 = 0.f, y2 = 0.f;
    if (r < g.rows) {
      const int hl = r / blk, t = r % blk, h = kvh * g.group + hl;
      const __nv_bfloat16 *src = q + (((long long)b * blk + t) * g.hq + h) * D;
      const float x1 = __bfloat162float(src[i]), x2 = __bfloat162float(src[i + HALF]);
      const float2 c = cs[t * HALF + i];
      y1 = x1 * c.x - x2 * c.y;
      y2 = x2 * c.x + x1 * c.y;
    }
    Qf[rr * D + i] = y1;
    Qf[rr * D + i + HALF] = y2;
  }
  __syncthreads();

#pragma unroll 1
  for (int rr = 0; rr < RPW; ++rr) {
    const int rl = warp * RPW + rr, r = r0 + rl;
    if (r >= g.rows) break;
    const int hl = r / blk, t = r % blk, h = kvh * g.group + hl;
    const float *qrow = Qf + rl * D;
    const int j0 = lane < blk ? lane : 0, j1 = lane + 32 < blk ? lane + 32 : 0;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
    for (int k = 0; k < D; k += 4) {
      const float4 qv = *reinterpret_cast<const float4 *>(qrow + k);
      const float4 a = *reinterpret_cast<const float4 *>(Kf + j0 * lay.kp + k);
      const float4 c = *reinterpret_cast<const float4 *>(Kf + j1 * lay.kp + k);
      s0 += qv.x * a.x + qv.y * a.y + qv.z * a.z + qv.w * a.w;
      s1 += qv.x * c.x + qv.y * c.y + qv.z * c.z + qv.w * c.w;
    }
    s0 = lane < blk ? s0 * g.tau : -CUDART_INF_F;
    s1 = lane + 32 < blk ? s1 * g.tau : -CUDART_INF_F;
    const float m2 = warp_max(fmaxf(s0, s1));
    const float p0 = expf(s0 - m2), p1 = expf(s1 - m2);
    const float l2 = warp_sum(p0 + p1);
    Ps[rl * 64 + lane] = p0;
    Ps[rl * 64 + lane + 32] = p1;
    __syncwarp();
    float ob[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) ob[c] = 0.f;
    for (int j = 0; j < blk; ++j) {
      const float pj = Ps[rl * 64 + j];
#pragma unroll
      for (int c = 0; c < CPL; ++c) ob[c] += pj * Vf[j * D + lane * CPL + c];
    }
    const long long prow = ((long long)b * g.hq + h) * blk + t;
    const float m1 = pfx.m[prow], l1 = pfx.l[prow];
    const float *o1 = pfx.o_unnorm + prow * D + lane * CPL;
    const float mm = fmaxf(m1, m2);
    const float w1 = lse_weight(m1, mm), w2 = expf(m2 - mm);
    const float lt = w1 * l1 + w2 * l2;
    const float inv = 1.f / lt;
    const long long orow = (((long long)b * blk + t) * g.hq + h) * D + lane * CPL;
    float res[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) res[c] = (w1 * o1[c] + w2 * ob[c]) * inv;
    if (F32OUT) {
      float *dst = reinterpret_cast<float *>(out) + orow;
#pragma unroll
      for (int c = 0; c < CPL; ++c) dst[c] = res[c];
    } else {
      __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(out) + orow;
#pragma unroll
      for (int c = 0; c < CPL; c += 2)
        *reinterpret_cast<__nv_bfloat162 *>(dst + c) = __floats2bfloat162_rn(res[c], res[c + 1]);
    }
    if (lse && lane == 0) lse[prow] = mm + logf(lt);
    __syncwarp();
  }
}

template <int D, int RPW, bool F32OUT>
cudaError_t launch_cfg(const Geometry &g, const __nv_bfloat16 *q, const __nv_bfloat16 *kb,
                       const __nv_bfloat16 *vb, const fbk_partial &pfx, void *out, float *lse,
                       cudaStream_t st) {
  constexpr int RC = WARPS * RPW;
  const Layout lay(D, g.blk, RC);
  const size_t bytes = sizeof(float) * lay.floats;
  auto kern = block_merge_kernel<D, RPW, F32OUT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  dim3 grid((g.rows + RC - 1) / RC, g.batch * g.hkv);
  kern<<<grid, WARPS * 32, bytes, st>>>(g, q, kb, vb, pfx, out, lse);
  return cudaGetLastError();
}

template <int D, bool F32OUT>
cudaError_t launch_d(const Geometry &g, const __nv_bfloat16 *q, const __nv_bfloat16 *kb,
                     const __nv_bfloat16 *vb, const fbk_partial &pfx, void *out, float *lse,
                     cudaStream_t st) {
  // Few rows per CTA when there are few units, so the grid still covers the SMs.
  const long long units = (long long)g.batch * g.hkv;
  if (units * ((g.rows + 7) / 8) <= 512)
    return launch_cfg<D, 2, F32OUT>(g, q, kb, vb, pfx, out, lse, st);
  return launch_cfg<D, 8, F32OUT>(g, q, kb, vb, pfx, out, lse, st);
}

}  // namespace

cudaError_t launch_block_merge(const Geometry &g, const __nv_bfloat16 *q,
                               const __nv_bfloat16 *kb, const __nv_bfloat16 *vb,
                               const fbk_partial &pfx, void *out, float *lse, bool f32_out,
                               cudaStream_t st) {
  if (g.d == 128)
    return f32_out ? launch_d<128, true>(g, q, kb, vb, pfx, out, lse, st)
                   : launch_d<128, false>(g, q, kb, vb, pfx, out, lse, st);
  return f32_out ? launch_d<64, true>(g, q, kb, vb, pfx, out, lse, st)
                 : launch_d<64, false>(g, q, kb, vb, pfx, out, lse, st);
}

}  // namespace fbk
