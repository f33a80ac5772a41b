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
// The step is latency-bound (a few MB), so the kernel is built around a single
// DRAM round trip: every input of the CTA (block K and V of its kv-head, its
// query rows, their prefix-state rows) is requested at once with cp.async,
// the RoPE cos/sin table is computed while those copies fly, and everything
// after that runs from shared memory in fp32 on CUDA cores (B <= 64 keys per
// row). Row max and sum are warp-shuffle reductions, lane j holding keys j and
// j + 32. One CTA per (unit, chunk of 4*RPW query rows).
#include "launch.h"

namespace fbk {
namespace {

constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;

struct Layout {  // byte offsets, all 16-byte aligned
  int kraw, vraw, qraw, opart, ml, kf, qf, cs, ps, bytes, kp;
  __host__ __device__ Layout(int d, int blk, int rc) {
    kp = d + 4;
    kraw = 0;
    vraw = kraw + blk * d * 2;
    qraw = vraw + blk * d * 2;
    opart = qraw + rc * d * 2;
    ml = opart + rc * d * 4;
    kf = ml + ((2 * rc * 4 + 15) & ~15);
    qf = kf + blk * kp * 4;
    cs = qf + rc * d * 4;
    ps = cs + blk * (d / 2) * 8;
    bytes = ps + rc * 64 * 4;
  }
};

template <int D, int RPW, bool F32OUT>
__global__ void __launch_bounds__(THREADS) block_merge_kernel(
    Geometry g, const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ kb,
    const __nv_bfloat16 *__restrict__ vb, fbk_partial pfx, void *__restrict__ out,
    float *__restrict__ lse) {
  constexpr int RC = WARPS * RPW, CPL = D / 32, HALF = D / 2, CH = D / 8, CHF = D / 4;
  extern __shared__ float4 smem_f4[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(smem_f4);
  const int blk = g.blk;
  const Layout lay(D, blk, RC);
  __nv_bfloat16 *Kraw = reinterpret_cast<__nv_bfloat16 *>(sm + lay.kraw);
  __nv_bfloat16 *Vraw = reinterpret_cast<__nv_bfloat16 *>(sm + lay.vraw);
  __nv_bfloat16 *Qraw = reinterpret_cast<__nv_bfloat16 *>(sm + lay.qraw);
  float *Opart = reinterpret_cast<float *>(sm + lay.opart);
  float *Mpart = reinterpret_cast<float *>(sm + lay.ml);
  float *Lpart = Mpart + RC;
  float *Kf = reinterpret_cast<float *>(sm + lay.kf);
  float *Qf = reinterpret_cast<float *>(sm + lay.qf);
  float2 *cs = reinterpret_cast<float2 *>(sm + lay.cs);
  float *Ps = reinterpret_cast<float *>(sm + lay.ps);

  const int u = blockIdx.y, b = u / g.hkv, kvh = u % g.hkv;
  const int r0 = blockIdx.x * RC;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int L = g.lens[b];
  if (L < 0) {
    raise_flag(g, FBK_DEVERR_PREFIX_LEN);
    L = 0;
  }

  // ---- one round of asynchronous copies for everything this CTA reads
  const long long kv_row0 = ((long long)b * blk) * g.hkv + kvh;  // row of token t: kv_row0 + t*hkv
  for (int idx = tid; idx < blk * CH; idx += THREADS) {
    const int t = idx / CH, c = idx % CH;
    const long long src = (kv_row0 + (long long)t * g.hkv) * D + c * 8;
    cp_async16(Kraw + t * D + c * 8, kb + src);
    cp_async16(Vraw + t * D + c * 8, vb + src);
  }
  for (int idx = tid; idx < RC * CH; idx += THREADS) {
    const int rr = idx / CH, c = idx % CH, r = r0 + rr;
    if (r < g.rows) {
      const int t = r % blk, h = kvh * g.group + r / blk;
      cp_async16(Qraw + rr * D + c * 8, q + (((long long)b * blk + t) * g.hq + h) * D + c * 8);
    }
  }
  for (int idx = tid; idx < RC * CHF; idx += THREADS) {
    const int rr = idx / CHF, c = idx % CHF, r = r0 + rr;
    if (r < g.rows) {
      const int t = r % blk, h = kvh * g.group + r / blk;
      cp_async16(Opart + rr * D + c * 4, pfx.o_unnorm + (((long long)b * g.hq + h) * blk + t) * D + c * 4);
    }
  }
  for (int rr = tid; rr < RC; rr += THREADS) {
    const int r = r0 + rr;
    if (r < g.rows) {
      const int t = r % blk, h = kvh * g.group + r / blk;
      const long long prow = ((long long)b * g.hq + h) * blk + t;
      cp_async4(Mpart + rr, pfx.m + prow);
      cp_async4(Lpart + rr, pfx.l + prow);
    }
  }
  // ---- RoPE table of positions L .. L+B-1 while the copies are in flight
  for (int idx = tid; idx < blk * HALF; idx += THREADS)
    cs[idx] = rope_cs_fast(L + idx / HALF, g.inv_freq_over_pi[idx % HALF]);
  cp_async_wait_all();
  __syncthreads();

  // ---- rotate block K and the CTA's query rows into fp32
  for (int idx = tid; idx < blk * HALF; idx += THREADS) {
    const int t = idx / HALF, i = idx % HALF;
    const float x1 = __bfloat162float(Kraw[t * D + i]), x2 = __bfloat162float(Kraw[t * D + i + HALF]);
    const float2 c = cs[idx];
    Kf[t * lay.kp + i] = x1 * c.x - x2 * c.y;
    Kf[t * lay.kp + i + HALF] = x2 * c.x + x1 * c.y;
  }
  for (int idx = tid; idx < RC * HALF; idx += THREADS) {
    const int rr = idx / HALF, i = idx % HALF, r = r0 + rr;
    if (r < g.rows) {
      const float x1 = __bfloat162float(Qraw[rr * D + i]), x2 = __bfloat162float(Qraw[rr * D + i + HALF]);
      const float2 c = cs[(r % blk) * HALF + i];
      Qf[rr * D + i] = x1 * c.x - x2 * c.y;
      Qf[rr * D + i + HALF] = x2 * c.x + x1 * c.y;
    }
  }
  __syncthreads();

  // ---- per query row: block scores, softmax, P V, merge, normalise, store
#pragma unroll 1
  for (int rr = 0; rr < RPW; ++rr) {
    const int rl = warp * RPW + rr, r = r0 + rl;
    if (r >= g.rows) break;
    const int t = r % blk, h = kvh * g.group + r / blk;
    const float *qrow = Qf + rl * D;
    const int j0 = lane < blk ? lane : 0, j1 = lane + 32 < blk ? lane + 32 : 0;
    float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
    for (int k = 0; k < D; k += 4) {
      const float4 qv = *reinterpret_cast<const float4 *>(qrow + k);
      const float4 a = *reinterpret_cast<const float4 *>(Kf + j0 * lay.kp + k);
      s0 += qv.x * a.x + qv.y * a.y + qv.z * a.z + qv.w * a.w;
      if (blk > 32) {
        const float4 c = *reinterpret_cast<const float4 *>(Kf + j1 * lay.kp + k);
        s1 += qv.x * c.x + qv.y * c.y + qv.z * c.z + qv.w * c.w;
      }
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
#pragma unroll 4
    for (int j = 0; j < blk; ++j) {
      const float pj = Ps[rl * 64 + j];
      const __nv_bfloat16 *vr = Vraw + j * D + lane * CPL;
#pragma unroll
      for (int c = 0; c < CPL; c += 2) {
        const float2 v2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(vr + c));
        ob[c] += pj * v2.x;
        ob[c + 1] += pj * v2.y;
      }
    }
    const float m1 = Mpart[rl], l1 = Lpart[rl];
    const float mm = fmaxf(m1, m2);
    const float w1 = lse_weight(m1, mm), w2 = expf(m2 - mm);
    const float lt = w1 * l1 + w2 * l2;
    const float inv = 1.f / lt;
    const float *o1 = Opart + rl * D + lane * CPL;
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
    if (lse && lane == 0) lse[((long long)b * g.hq + h) * blk + t] = mm + logf(lt);
    __syncwarp();
  }
}

template <int D, int RPW, bool F32OUT>
cudaError_t launch_cfg(const Geometry &g, const __nv_bfloat16 *q, const __nv_bfloat16 *kb,
                       const __nv_bfloat16 *vb, const fbk_partial &pfx, void *out, float *lse,
                       cudaStream_t st) {
  constexpr int RC = WARPS * RPW;
  const Layout lay(D, g.blk, RC);
  auto kern = block_merge_kernel<D, RPW, F32OUT>;
  if (lay.bytes > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.bytes);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((g.rows + RC - 1) / RC, g.batch * g.hkv);
  kern<<<grid, THREADS, lay.bytes, st>>>(g, q, kb, vb, pfx, out, lse);
  return cudaGetLastError();
}

template <int D, bool F32OUT>
cudaError_t launch_d(const Geometry &g, const __nv_bfloat16 *q, const __nv_bfloat16 *kb,
                     const __nv_bfloat16 *vb, const fbk_partial &pfx, void *out, float *lse,
                     cudaStream_t st) {
  // Few rows per CTA when there are few units, so the grid still covers the SMs.
  const long long units = (long long)g.batch * g.hkv;
  if (units * ((g.rows + 7) / 8) <= 512) return launch_cfg<D, 2, F32OUT>(g, q, kb, vb, pfx, out, lse, st);
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
