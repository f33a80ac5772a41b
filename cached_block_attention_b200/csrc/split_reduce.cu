// Split-L reduction: merge the per-share states of every (sequence, kv-head)
// unit into its prefix state, in increasing share order (deterministic).
//
// Each share's state is the recurrence of LaCache §3.3.3 (Eq. 2-6) over its
// own run of tiles; by associativity of that recurrence, the state over all
// tiles is the LSE merge m = max_c m_c, l = sum_c e^(m_c - m) l_c,
// O~ = sum_c e^(m_c - m) O~_c. One CTA per (unit, 32 query rows): warp 0
// lists the unit's pieces (their workspace slots) once in shared memory; each
// warp then reduces 4 rows, pieces in chunks of 8: lane j fetches m and l of
// the chunk's j-th piece while every lane fetches its columns of all the
// chunk's O~ rows (one round trip per chunk); the weights are broadcast by
// shuffle.
#include "launch.h"

namespace fbk {
namespace {

constexpr int WARPS = 8;
constexpr int MAX_PIECES = 1024;  // pieces of one unit handled per pass of the piece list
constexpr int NCH = 8;            // pieces whose O~ rows are in flight at once

template <int D, int ROWS_PER_WARP>
__global__ void __launch_bounds__(WARPS * 32) split_reduce_kernel(Geometry g, Workspace ws, int shares,
                                                                 fbk_partial out, const int *gate) {
  constexpr int CPL = D / 32, CTA_ROWS = WARPS * ROWS_PER_WARP;
  const int u = blockIdx.x, b = u / g.hkv, kvh = u % g.hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ long long red[2][WARPS];
  __shared__ int s_slot[MAX_PIECES];  // workspace slot of each piece of this unit
  __shared__ int s_n;
  pdl_wait();
  pdl_release();
  if (gate && *gate == 0) return;  // no refresh of this state at this step

  // list positions before sequence b and in total: parallel loads, block reduction
  long long before = 0, T = 0;
  for (int bb = threadIdx.x; bb < g.batch; bb += WARPS * 32) {
    const long long n = (long long)g.hkv * span_of(prefix_len(g, bb));
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
  // the unit's tiles in the work list: after its UNIT_LEAD lead positions
  const int tb = tiles_of(prefix_len(g, b));
  const long long A = before + (long long)kvh * span_of(prefix_len(g, b)) + UNIT_LEAD, E = A + tb;

  // the unit's pieces: shares c_lo .. c_hi, each non-empty one holding the
  // piece's state in slot c + u (computed once per CTA, in increasing share order)
  long long c_lo = 0, c_hi = -1;
  if (tb > 0) {
    c_lo = share_of(A, T, shares);
    c_hi = share_of(E - 1, T, shares);
  }
  const long long n_all = c_hi - c_lo + 1;
  const int r0 = blockIdx.y * CTA_ROWS;
  float acc[ROWS_PER_WARP][CPL], M[ROWS_PER_WARP], Lsum[ROWS_PER_WARP];
#pragma unroll
  for (int k = 0; k < ROWS_PER_WARP; ++k) {
    M[k] = -CUDART_INF_F;
    Lsum[k] = 0.f;
#pragma unroll
    for (int cc = 0; cc < CPL; ++cc) acc[k][cc] = 0.f;
  }
  for (long long pass = 0; pass < n_all; pass += MAX_PIECES) {
    const int np = (int)min((long long)MAX_PIECES, n_all - pass);
    __syncthreads();  // the previous pass's list is consumed
    if (warp == 0) {
      int kept = 0;
      for (int j0 = 0; j0 < np; j0 += 32) {
        const long long c = c_lo + pass + j0 + lane;
        bool valid = false;
        if (j0 + lane < np) {
          const long long lo = max(share_begin(c, T, shares), A);
          const long long hi = min(share_begin(c + 1, T, shares), E);
          valid = lo < hi;
        }
        const unsigned mask = __ballot_sync(0xffffffffu, valid);
        if (valid) s_slot[kept + __popc(mask & ((1u << lane) - 1))] = (int)(c + u);
        kept += __popc(mask);
      }
      if (lane == 0) s_n = kept;
    }
    __syncthreads();
    const int n = s_n;
#pragma unroll
    for (int k = 0; k < ROWS_PER_WARP; ++k) {
      const int r = r0 + warp * ROWS_PER_WARP + k;
      if (r >= g.rows) break;
      for (int base = 0; base < n; base += NCH) {
        const int nc = min(NCH, n - base);
        // lane j < nc: (m, l) of piece base + j; every lane: its columns of the chunk's O~ rows
        const long long my_row = (long long)s_slot[base + (lane < nc ? lane : 0)] * g.rows + r;
        const float mc = lane < nc ? ws.m[my_row] : -CUDART_INF_F;
        const float lc = lane < nc ? ws.l[my_row] : 0.f;
        float v[NCH][CPL];
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
          if (j < nc) {
            const float *src = ws.o + ((long long)s_slot[base + j] * g.rows + r) * D + lane * CPL;
            if constexpr (CPL == 4) {  // 16-byte aligned: D*4 and the region base are
              const float4 t4 = *reinterpret_cast<const float4 *>(src);
              v[j][0] = t4.x; v[j][1] = t4.y; v[j][2] = t4.z; v[j][3] = t4.w;
            } else {
#pragma unroll
              for (int cc = 0; cc < CPL; cc += 2) {
                const float2 t2 = *reinterpret_cast<const float2 *>(src + cc);
                v[j][cc] = t2.x; v[j][cc + 1] = t2.y;
              }
            }
          }
        }
        const float Mn = fmaxf(M[k], warp_max(mc));
        const float keep = lse_weight(M[k], Mn);
        const float wc = lane < nc ? expf(mc - Mn) : 0.f;
        Lsum[k] = Lsum[k] * keep + warp_sum(wc * lc);
#pragma unroll
        for (int cc = 0; cc < CPL; ++cc) acc[k][cc] *= keep;
#pragma unroll
        for (int j = 0; j < NCH; ++j) {
          const float w = __shfl_sync(0xffffffffu, wc, j);
          if (j < nc) {
#pragma unroll
            for (int cc = 0; cc < CPL; ++cc) acc[k][cc] += w * v[j][cc];
          }
        }
        M[k] = Mn;
      }
    }
  }
#pragma unroll
  for (int k = 0; k < ROWS_PER_WARP; ++k) {
    const int r = r0 + warp * ROWS_PER_WARP + k;
    if (r >= g.rows) break;
    const int hl = r / g.blk, t = r % g.blk, h = kvh * g.group + hl;
    const long long orow = ((long long)b * g.hq + h) * g.blk + t;
    float *dst = out.o_unnorm + orow * D + lane * CPL;
    if constexpr (CPL == 4) {
      *reinterpret_cast<float4 *>(dst) = make_float4(acc[k][0], acc[k][1], acc[k][2], acc[k][3]);
    } else {
#pragma unroll
      for (int c = 0; c < CPL; c += 2) *reinterpret_cast<float2 *>(dst + c) = make_float2(acc[k][c], acc[k][c + 1]);
    }
    if (lane == 0) {
      out.m[orow] = M[k];
      out.l[orow] = Lsum[k];
    }
  }
}

// Rows per warp: 4 when there are enough rows to keep several warps per SM
// busy (the unit's piece list is then shared by 32 rows), else 1 (more CTAs,
// shorter chains).
template <int D, int RPW>
cudaError_t launch_rpw(const Geometry &g, const Workspace &ws, int shares, const fbk_partial &out,
                       cudaStream_t st, const int *gate) {
  dim3 grid(g.batch * g.hkv, (g.rows + WARPS * RPW - 1) / (WARPS * RPW));
  return launch_pdl(split_reduce_kernel<D, RPW>, grid, dim3(WARPS * 32), 0, st, g, ws, shares, out, gate);
}

}  // namespace

cudaError_t launch_split_reduce(const Geometry &g, const Workspace &ws, int shares,
                                const fbk_partial &out, cudaStream_t st, const int *gate) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const bool four = (long long)g.batch * g.hkv * g.rows >= 4ll * WARPS * sms;
  if (g.d == 128)
    return four ? launch_rpw<128, 4>(g, ws, shares, out, st, gate) : launch_rpw<128, 1>(g, ws, shares, out, st, gate);
  return four ? launch_rpw<64, 4>(g, ws, shares, out, st, gate) : launch_rpw<64, 1>(g, ws, shares, out, st, gate);
}

}  // namespace fbk
