// Split-L reduction: merge the per-share states of every (sequence, kv-head)
// unit into its prefix state, in increasing share order (deterministic).
//
// Each share's state is the recurrence of LaCache §3.3.3 (Eq. 2-6) over its
// own run of tiles; by associativity of that recurrence, the state over all
// tiles is the LSE merge m = max_c m_c, l = sum_c e^(m_c - m) l_c,
// O~ = sum_c e^(m_c - m) O~_c. One warp per query row: lane j fetches m and l
// of the j-th share of a batch of 32 (one round trip for all of them), the
// weights are broadcast by shuffle, and the O~ rows are read with the loop
// unrolled so that several loads are in flight at once.
#include "launch.h"

namespace fbk {
namespace {

constexpr int WARPS = 8;

template <int D>
__global__ void __launch_bounds__(WARPS * 32, 1) split_reduce_kernel(Geometry g, Workspace ws,
                                                                   int shares, fbk_partial out) {
  constexpr int CPL = D / 32;
  const int u = blockIdx.x, b = u / g.hkv, kvh = u % g.hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * WARPS + warp;
  pdl_wait();
  pdl_release();

  // tiles before sequence b and in total: parallel loads, block reduction
  __shared__ long long red[2][WARPS];
  long long before = 0, T = 0;
  for (int bb = threadIdx.x; bb < g.batch; bb += WARPS * 32) {
    const long long n = (long long)g.hkv * tiles_of(prefix_len(g, bb));
    if (bb < b) before += n;
    T += n;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, o);
    T += __shfl_xor_sync(0xffffffffu, T, o);
  }
  if (lane == 0) {
    red[0][warp] = before;
    red[1][warp] = T;
  }
  __syncthreads();
  before = T = 0;
#pragma unroll
  for (int w = 0; w < WARPS; ++w) {
    before += red[0][w];
    T += red[1][w];
  }
  if (r >= g.rows) return;
  const int tb = tiles_of(prefix_len(g, b));
  const long long A = before + (long long)kvh * tb, E = A + tb;

  const int hl = r / g.blk, t = r % g.blk, h = kvh * g.group + hl;
  const long long orow = ((long long)b * g.hq + h) * g.blk + t;
  float acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = 0.f;
  float M = -CUDART_INF_F, Lsum = 0.f;
  if (tb > 0) {
    const long long c_lo = share_of(A, T, shares), c_hi = share_of(E - 1, T, shares);
    const long long first_row = (c_lo + u) * g.rows + r;  // share c_lo always holds a piece of u
    for (long long base = c_lo; base <= c_hi; base += 32) {
      const long long c = base + lane;
      bool valid = false;
      if (c <= c_hi) {
        const long long lo = max(share_begin(c, T, shares), A);
        const long long hi = min(share_begin(c + 1, T, shares), E);
        valid = lo < hi;
      }
      const long long row = valid ? (c + u) * g.rows + r : first_row;
      const float mc = valid ? ws.m[row] : -CUDART_INF_F;
      const float lc = valid ? ws.l[row] : 0.f;
      const float Mn = fmaxf(M, warp_max(mc));
      const float keep = lse_weight(M, Mn);
      const float wc = valid ? expf(mc - Mn) : 0.f;
      Lsum = Lsum * keep + warp_sum(wc * lc);
#pragma unroll
      for (int cc = 0; cc < CPL; ++cc) acc[cc] *= keep;
      const int n = (int)min(32ll, c_hi - base + 1);
#pragma unroll 4
      for (int j = 0; j < n; ++j) {
        const float w = __shfl_sync(0xffffffffu, wc, j);
        const long long rj = __shfl_sync(0xffffffffu, row, j);
        const float *src = ws.o + rj * D + lane * CPL;  // empty shares read share c_lo's row, weight 0
        if constexpr (CPL == 4) {
          const float4 v = *reinterpret_cast<const float4 *>(src);  // 16-byte aligned: D*4 and the slot base are
          acc[0] += w * v.x;
          acc[1] += w * v.y;
          acc[2] += w * v.z;
          acc[3] += w * v.w;
        } else {
#pragma unroll
          for (int cc = 0; cc < CPL; cc += 2) {
            const float2 v = *reinterpret_cast<const float2 *>(src + cc);
            acc[cc] += w * v.x;
            acc[cc + 1] += w * v.y;
          }
        }
      }
      M = Mn;
    }
  }
  float *dst = out.o_unnorm + orow * D + lane * CPL;
  if constexpr (CPL == 4) {
    *reinterpret_cast<float4 *>(dst) = make_float4(acc[0], acc[1], acc[2], acc[3]);
  } else {
#pragma unroll
    for (int c = 0; c < CPL; c += 2) *reinterpret_cast<float2 *>(dst + c) = make_float2(acc[c], acc[c + 1]);
  }
  if (lane == 0) {
    out.m[orow] = M;
    out.l[orow] = Lsum;
  }
}

}  // namespace

cudaError_t launch_split_reduce(const Geometry &g, const Workspace &ws, int shares,
                                const fbk_partial &out, cudaStream_t st) {
  dim3 grid(g.batch * g.hkv, (g.rows + WARPS - 1) / WARPS);
  if (g.d == 128) return launch_pdl(split_reduce_kernel<128>, grid, dim3(WARPS * 32), 0, st, g, ws, shares, out);
  return launch_pdl(split_reduce_kernel<64>, grid, dim3(WARPS * 32), 0, st, g, ws, shares, out);
}

}  // namespace fbk
