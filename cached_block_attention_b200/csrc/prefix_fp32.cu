// Prefix state on CUDA cores in fp32 (FBK_FP32_CHECK).
//
// Same work list as the tensor-core kernel: CTA c walks the pieces of share c
// and, for every piece, streams its 64-key tiles through the FlashAttention
// recurrence of LaCache §3.3.3 (Eq. 2-6): running max m, rescale alpha,
// P~ = exp(S - m), l and O~ updated per tile. The block queries are rotated at
// L_b + t and kept in fp32 (no bf16 rounding), so this kernel isolates the
// indexing and merge logic from tensor-core rounding. Query rows are handled
// 32 at a time; each 32-row chunk re-reads the piece's tiles (from L2).
#include "launch.h"
#include "prefix_at.h"

namespace fbk {
namespace {

constexpr int THREADS = 256;
constexpr int ROWS_PER_PASS = 32;  // 8 warps x 4 rows

template <int D>
struct Smem {
  static constexpr int KP = D + 4;  // padded K row: float4 reads by 32 lanes hit distinct banks
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + KV_TILE * KP;
  static constexpr int Q_OFF = V_OFF + KV_TILE * D;
  static constexpr int P_OFF = Q_OFF + ROWS_PER_PASS * D;
  static constexpr int LEN_OFF = P_OFF + ROWS_PER_PASS * KV_TILE;  // [MAX_BATCH] int
  static constexpr int SCAN_OFF = LEN_OFF + MAX_BATCH;               // [MAX_BATCH] int
  static constexpr int FLOATS = SCAN_OFF + MAX_BATCH;
};

template <int D>
__global__ void __launch_bounds__(THREADS) prefix_fp32_kernel(Geometry g,
                                                              const __nv_bfloat16 *__restrict__ q,
                                                              Workspace ws, int shares,
                                                              const int *__restrict__ qpos) {
  extern __shared__ float4 smem_f4[];
  float *sm = reinterpret_cast<float *>(smem_f4);
  using S = Smem<D>;
  float *Kf = sm + S::K_OFF;
  float *Vf = sm + S::V_OFF;
  float *Qf = sm + S::Q_OFF;
  float *Ps = sm + S::P_OFF;
  constexpr int CPL = D / 32;  // output columns per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int *s_len = reinterpret_cast<int *>(sm + S::LEN_OFF);
  int *s_scan = reinterpret_cast<int *>(sm + S::SCAN_OFF);
  pdl_wait();
  pdl_release();
  const long long T = load_tile_scan(g, s_len, s_scan);
  if (T == 0) return;
  PieceWalker walk;
  walk.init(g, s_len, s_scan, blockIdx.x, T, shares);
  Piece p;
  while (walk.next(g, p)) {
    const long long slot = (long long)blockIdx.x + p.u;
    const int pos0 = qpos ? qpos[p.b] : p.L;  // rotation base of the block's rows
    for (int r0 = 0; r0 < g.rows; r0 += ROWS_PER_PASS) {
      __syncthreads();  // previous users of Qf are done
      for (int idx = threadIdx.x; idx < ROWS_PER_PASS * (D / 2); idx += THREADS) {
        const int rr = idx / (D / 2), i = idx % (D / 2), r = r0 + rr;
        float y1 = 0.f, y2 = 0.f;
        if (r < g.rows) {
          const int hl = r / g.blk, t = r % g.blk, h = p.kvh * g.group + hl;
          const __nv_bfloat16 *src = q + (((long long)p.b * g.blk + t) * g.hq + h) * D;
          const float x1 = __bfloat162float(src[i]), x2 = __bfloat162float(src[i + D / 2]);
          const float2 cs = rope_cs_f32(pos0 + t, freq_over_pi(i, D, g.log2_base));
          y1 = x1 * cs.x - x2 * cs.y;
          y2 = x2 * cs.x + x1 * cs.y;
        }
        Qf[rr * D + i] = y1;
        Qf[rr * D + i + D / 2] = y2;
      }
      float m[4], l[4], o[4][CPL];
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        m[rr] = -CUDART_INF_F;
        l[rr] = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) o[rr][c] = 0.f;
      }
      for (int j = p.tile_begin; j < p.tile_end; ++j) {
        __syncthreads();  // Qf written / previous tile consumed
        for (int idx = threadIdx.x; idx < KV_TILE * (D / 8); idx += THREADS) {
          const int key = idx / (D / 8), ch = idx % (D / 8);
          const long long pos = (long long)j * KV_TILE + key;
          uint4 kraw = make_uint4(0, 0, 0, 0), vraw = make_uint4(0, 0, 0, 0);
          if (pos < p.L) {
            const long long row = cache_row(g, p.b, p.kvh, pos);
            if (row >= 0) {
              kraw = *reinterpret_cast<const uint4 *>(g.kc + row * D + ch * 8);
              vraw = *reinterpret_cast<const uint4 *>(g.vc + row * D + ch * 8);
            }
          }
          const uint32_t kw[4] = {kraw.x, kraw.y, kraw.z, kraw.w};
          const uint32_t vw[4] = {vraw.x, vraw.y, vraw.z, vraw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            Kf[key * S::KP + ch * 8 + 2 * e] = __uint_as_float(kw[e] << 16);
            Kf[key * S::KP + ch * 8 + 2 * e + 1] = __uint_as_float(kw[e] & 0xffff0000u);
            Vf[key * D + ch * 8 + 2 * e] = __uint_as_float(vw[e] << 16);
            Vf[key * D + ch * 8 + 2 * e + 1] = __uint_as_float(vw[e] & 0xffff0000u);
          }
        }
        __syncthreads();
        const long long key0 = (long long)j * KV_TILE + lane;
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const int rl = warp * 4 + rr;
          const float *qrow = Qf + rl * D;
          float s0 = 0.f, s1 = 0.f;
#pragma unroll 8
          for (int k = 0; k < D; k += 4) {
            const float4 qv = *reinterpret_cast<const float4 *>(qrow + k);
            const float4 a = *reinterpret_cast<const float4 *>(Kf + lane * S::KP + k);
            const float4 b = *reinterpret_cast<const float4 *>(Kf + (lane + 32) * S::KP + k);
            s0 += qv.x * a.x + qv.y * a.y + qv.z * a.z + qv.w * a.w;
            s1 += qv.x * b.x + qv.y * b.y + qv.z * b.z + qv.w * b.w;
          }
          s0 = key0 < p.L ? s0 * g.tau : -CUDART_INF_F;
          s1 = key0 + 32 < p.L ? s1 * g.tau : -CUDART_INF_F;
          const float mn = fmaxf(m[rr], warp_max(fmaxf(s0, s1)));  // Eq. 2
          const float alpha = lse_weight(m[rr], mn);              // Eq. 3
          const float p0 = expf(s0 - mn), p1 = expf(s1 - mn);     // Eq. 4
          l[rr] = alpha * l[rr] + warp_sum(p0 + p1);              // Eq. 5
          m[rr] = mn;
          Ps[rl * KV_TILE + lane] = p0;
          Ps[rl * KV_TILE + lane + 32] = p1;
          __syncwarp();
#pragma unroll
          for (int c = 0; c < CPL; ++c) o[rr][c] *= alpha;        // Eq. 6
          for (int key = 0; key < KV_TILE; ++key) {
            const float pk = Ps[rl * KV_TILE + key];
#pragma unroll
            for (int c = 0; c < CPL; ++c) o[rr][c] += pk * Vf[key * D + lane * CPL + c];
          }
          __syncwarp();
        }
      }
#pragma unroll
      for (int rr = 0; rr < 4; ++rr) {
        const int r = r0 + warp * 4 + rr;
        if (r < g.rows) {
          const long long row = slot * g.rows + r;
#pragma unroll
          for (int c = 0; c < CPL; ++c) ws.o[row * D + lane * CPL + c] = o[rr][c];
          if (lane == 0) {
            ws.m[row] = m[rr];
            ws.l[row] = l[rr];
          }
        }
      }
    }
  }
}

template <int D>
cudaError_t launch_d(const Geometry &g, const __nv_bfloat16 *q, const int *qpos, const Workspace &ws, int shares,
                     cudaStream_t st) {
  const size_t bytes = sizeof(float) * Smem<D>::FLOATS;
  cudaError_t e = cudaFuncSetAttribute(prefix_fp32_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(prefix_fp32_kernel<D>, dim3(shares), dim3(THREADS), bytes, st, g, q, ws, shares, qpos);
}

}  // namespace

cudaError_t launch_prefix_fp32_at(const Geometry &g, const __nv_bfloat16 *q, const int *qpos, const Workspace &ws,
                                  int shares, cudaStream_t st) {
  return g.d == 128 ? launch_d<128>(g, q, qpos, ws, shares, st) : launch_d<64>(g, q, qpos, ws, shares, st);
}

cudaError_t launch_prefix_fp32(const Geometry &g, const __nv_bfloat16 *q, const Workspace &ws,
                               int shares, cudaStream_t st) {
  return launch_prefix_fp32_at(g, q, nullptr, ws, shares, st);
}

}  // namespace fbk
