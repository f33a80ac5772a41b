// Split-L reduction: merge the per-share states of every (sequence, kv-head)
// unit into its prefix state, in increasing share order (deterministic).
//
// Each share's state is the recurrence of LaCache §3.3.3 (Eq. 2-6) over its
// own run of tiles; by associativity of that recurrence, the state over all
// tiles is the LSE merge m = max_c m_c, l = sum_c e^(m_c - m) l_c,
// O~ = sum_c e^(m_c - m) O~_c. One warp per query row; lanes hold d/32 columns.
#include "launch.h"

namespace fbk {
namespace {

constexpr int WARPS = 8;

template <int D>
__global__ void __launch_bounds__(WARPS * 32) split_reduce_kernel(Geometry g, Workspace ws,
                                                                   int shares, fbk_partial out) {
  constexpr int CPL = D / 32;
  const int u = blockIdx.x, b = u / g.hkv, kvh = u % g.hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = blockIdx.y * WARPS + warp;
  if (r >= g.rows) return;

  long long before = 0, T = 0;
  for (int bb = 0; bb < g.batch; ++bb) {
    const long long n = (long long)g.hkv * tiles_of(prefix_len(g, bb));
    if (bb < b) before += n;
    T += n;
  }
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
    for (long long c = c_lo; c <= c_hi; ++c) {
      const long long lo = max(share_begin(c, T, shares), A);
      const long long hi = min(share_begin(c + 1, T, shares), E);
      if (lo < hi) M = fmaxf(M, ws.m[(c + u) * g.rows + r]);
    }
    for (long long c = c_lo; c <= c_hi; ++c) {
      const long long lo = max(share_begin(c, T, shares), A);
      const long long hi = min(share_begin(c + 1, T, shares), E);
      if (lo >= hi) continue;
      const long long row = (c + u) * g.rows + r;
      const float w = expf(ws.m[row] - M);
      Lsum += w * ws.l[row];
      const float *src = ws.o + row * D + lane * CPL;
#pragma unroll
      for (int cc = 0; cc < CPL; ++cc) acc[cc] += w * src[cc];
    }
  }
  float *dst = out.o_unnorm + orow * D + lane * CPL;
#pragma unroll
  for (int c = 0; c < CPL; ++c) dst[c] = acc[c];
  if (lane == 0) {
    out.m[orow] = M;
    out.l[orow] = Lsum;
  }
}

}  // namespace

cudaError_t launch_split_reduce(const Geometry &g, const Workspace &ws, int shares,
                                const fbk_partial &out, cudaStream_t st) {
  dim3 grid(g.batch * g.hkv, (g.rows + WARPS - 1) / WARPS);
  if (g.d == 128)
    split_reduce_kernel<128><<<grid, WARPS * 32, 0, st>>>(g, ws, shares, out);
  else
    split_reduce_kernel<64><<<grid, WARPS * 32, 0, st>>>(g, ws, shares, out);
  return cudaGetLastError();
}

}  // namespace fbk
