// FACache step for the unchanged rows of a whole sequence (LaCache §3.3.3,
// FACache, Eq. 2-6, and App. J: initialise from the cached state, stream only
// the KV tiles that overlap the current block).
//
// The sequence's rows outside the current block C (the set U: prompt, earlier
// blocks and the masked suffix) keep their online-softmax state over U's keys
// for the whole block. At each denoising step a row i of U, head h, starts
// from that state (O~1, m1, l1) and streams only the block's B keys:
//   S_t = tau <q_i, RoPE(k_t, c0 + t)>,  t < B
//   m2 = max_t S_t, l2 = sum_t e^(S_t - m2), O~2 = sum_t e^(S_t - m2) v_t
//   O_i = (e^(m1-m) O~1 + e^(m2-m) O~2) / (e^(m1-m) l1 + e^(m2-m) l2),
//   m = max(m1, m2), lse_i = m + log(e^(m1-m) l1 + e^(m2-m) l2).
// q_i is stored after RoPE at its own position (RoPECache, §3.3.2 Eq. 1), so
// the block's keys are rotated at their absolute positions c0 + t, with the
// angle reduced in fp64 before the fast sine and cosine.
//
// Per row and head the step reads q (2d bytes) and the state (4(d+2) bytes)
// and writes O (2d bytes), so it is bound by HBM bandwidth; the block's K and
// V are a few KB per kv-head. A CTA owns a slice of one (sequence, kv-head)
// unit: it stages the block's K (rotated in place) and V once, then its warps
// stride over the unit's tiles of 16 rows (one head, 16 consecutive rows of
// U). A warp loads its tile's queries into shared memory with cp.async and
// the state fragments into registers, computes S = Q K^T and O~2 = P~ V with
// bf16 tensor-core MMAs (mma.sync m16n8k16, fp32 accumulation), the row
// softmax on the accumulator fragments, and the merge.
#include "facache_rows.h"
#include "launch.h"
#include "tc.cuh"

namespace fbk {
namespace {

constexpr int FR_WARPS = 8;
constexpr int FR_ROWS = 16;  // rows of one tile: one m16 MMA tile

__device__ __forceinline__ void fr_ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void fr_ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                             uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void fr_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t fr_pack2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

// Shared memory: K^ and V of the block (bpad rows each), then one 16-row query
// tile per warp. Rows are padded by 16 bytes so that the 8 rows of an
// ldmatrix hit distinct banks.
template <int D>
struct FacRowsLayout {
  static constexpr int RS = D * 2 + 16;
  int bpad, ks, vs, qs, bytes;
  __host__ __device__ explicit FacRowsLayout(int blk) {
    bpad = (blk + 15) & ~15;
    ks = 0;
    vs = ks + bpad * RS;
    qs = vs + bpad * RS;
    bytes = qs + FR_WARPS * FR_ROWS * RS;
  }
};

template <int D>
__global__ void __launch_bounds__(FR_WARPS * 32) facache_rows_kernel(Geometry g, FacRowsArgs a) {
  using L = FacRowsLayout<D>;
  constexpr int RS = L::RS, CH = D / 8, NTW = D / 8, NTHREADS = FR_WARPS * 32;
  extern __shared__ float4 fr_smem[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(fr_smem);
  const int blk = g.blk, U = a.n_rows;
  const L lay(blk);
  const int bpad = lay.bpad;
  uint8_t *Ks = sm + lay.ks, *Vs = sm + lay.vs;
  const int unit = blockIdx.x / a.ctas_per_unit, part = blockIdx.x % a.ctas_per_unit;
  const int b = unit / g.hkv, kvh = unit % g.hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_release();

  // ---- 1. the block's K and V for this kv-head; padding rows are zeros
  const long long kv_row0 = (long long)b * blk * g.hkv + kvh;  // token t: row kv_row0 + t * hkv
  for (int idx = tid; idx < blk * CH; idx += NTHREADS) {
    const int t = idx / CH, c = idx % CH;
    const long long src = (kv_row0 + (long long)t * g.hkv) * D + c * 8;
    cp_async16(Ks + t * RS + c * 16, a.kb + src);
    cp_async16(Vs + t * RS + c * 16, a.vb + src);
  }
  for (int idx = tid; idx < (bpad - blk) * CH; idx += NTHREADS) {
    const int t = blk + idx / CH, c = idx % CH;
    *reinterpret_cast<uint4 *>(Ks + t * RS + c * 16) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(Vs + t * RS + c * 16) = make_uint4(0, 0, 0, 0);
  }
  cp_async_wait_all();
  __syncthreads();

  // ---- 2. rotate K at its absolute positions c0 + t (rotate-half pairs i, i + D/2)
  const int c0 = a.block_pos[b];
  for (int idx = tid; idx < blk * (D / 2); idx += NTHREADS) {
    const int t = idx / (D / 2), i = idx % (D / 2);
    __nv_bfloat16 *row = reinterpret_cast<__nv_bfloat16 *>(Ks + t * RS);
    // the position in 64 bits (c0 may be any int32), the angle in turns reduced in fp64
    const double turns = (double)((long long)c0 + t) * g.inv_freq_over_pi[i];
    float2 cs;
    __sincosf((float)((turns - 2.0 * rint(0.5 * turns)) * CUDART_PI), &cs.y, &cs.x);
    const float x1 = __bfloat162float(row[i]), x2 = __bfloat162float(row[i + D / 2]);
    row[i] = __float2bfloat16_rn(x1 * cs.x - x2 * cs.y);
    row[i + D / 2] = __float2bfloat16_rn(x2 * cs.x + x1 * cs.y);
  }
  __syncthreads();

  // ---- 3. the unit's tiles: head h = kvh * G + hh, rows i0 .. i0 + 15 of U
  uint8_t *Qw = sm + lay.qs + warp * FR_ROWS * RS;
  const uint32_t qs_a = (uint32_t)__cvta_generic_to_shared(Qw), ks_a = (uint32_t)__cvta_generic_to_shared(Ks),
                 vs_a = (uint32_t)__cvta_generic_to_shared(Vs);
  const int a_row = (lane & 7) + 8 * ((lane >> 3) & 1), a_col = 8 * (lane >> 4);
  const int b_row = (lane & 7) + 8 * (lane >> 4), b_col = 8 * ((lane >> 3) & 1);
  const int v_row = (lane & 7) + 8 * ((lane >> 3) & 1), v_col = 8 * (lane >> 4);
  const int lr = lane >> 2, lc = (lane & 3) * 2;
  const float sl2 = g.tau * 1.4426950408889634f, LN2 = 0.6931471805599453f;
  const int tiles_per_head = (U + FR_ROWS - 1) / FR_ROWS;
  const int tiles = g.group * tiles_per_head;
  for (int tile = part * FR_WARPS + warp; tile < tiles; tile += a.ctas_per_unit * FR_WARPS) {
    const int h = kvh * g.group + tile / tiles_per_head, i0 = (tile % tiles_per_head) * FR_ROWS;
    const int nrows = min(FR_ROWS, U - i0);
    __syncwarp();  // the previous tile's ldmatrix reads of Qw are done
    for (int idx = lane; idx < FR_ROWS * CH; idx += 32) {
      const int rr = idx / CH, c = idx % CH;
      if (rr < nrows)
        cp_async16(Qw + rr * RS + c * 16, a.q + (((long long)b * U + i0 + rr) * g.hq + h) * D + c * 8);
      else
        *reinterpret_cast<uint4 *>(Qw + rr * RS + c * 16) = make_uint4(0, 0, 0, 0);
    }
    // this thread's rows lr and lr + 8 of the tile: their cached state
    const bool va = lr < nrows, vbr = lr + 8 < nrows;
    const long long pa = ((long long)b * g.hq + h) * U + i0 + lr, pb = pa + 8;
    float2 o1a[NTW], o1b[NTW];
#pragma unroll
    for (int j = 0; j < NTW; ++j) {
      o1a[j] = va ? __ldg(reinterpret_cast<const float2 *>(a.state.o_unnorm + pa * D + 8 * j + lc))
                  : make_float2(0.f, 0.f);
      o1b[j] = vbr ? __ldg(reinterpret_cast<const float2 *>(a.state.o_unnorm + pb * D + 8 * j + lc))
                   : make_float2(0.f, 0.f);
    }
    const float m1a = va ? __ldg(a.state.m + pa) : -CUDART_INF_F, l1a = va ? __ldg(a.state.l + pa) : 0.f;
    const float m1b = vbr ? __ldg(a.state.m + pb) : -CUDART_INF_F, l1b = vbr ? __ldg(a.state.l + pb) : 0.f;
    cp_async_wait_all();
    __syncwarp();

    // S = Q K^T over the block's keys (up to 64)
    float sacc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      fr_ldsm_x4(qs_a + a_row * RS + (16 * kk + a_col) * 2, a0, a1, a2, a3);
#pragma unroll
      for (int jp = 0; jp < 4; ++jp) {
        if (16 * jp < bpad) {
          uint32_t b0, b1, b2, b3;
          fr_ldsm_x4(ks_a + (16 * jp + b_row) * RS + (16 * kk + b_col) * 2, b0, b1, b2, b3);
          fr_mma(sacc[2 * jp], a0, a1, a2, a3, b0, b1);
          fr_mma(sacc[2 * jp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    // softmax over the keys, rows lr and lr + 8, log2 units
    float mxa = -CUDART_INF_F, mxb = -CUDART_INF_F, sa = 0.f, sb = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = 8 * j + lc + e < blk;
        sacc[j][e] = ok ? sacc[j][e] * sl2 : -CUDART_INF_F;
        sacc[j][2 + e] = ok ? sacc[j][2 + e] * sl2 : -CUDART_INF_F;
        mxa = fmaxf(mxa, sacc[j][e]);
        mxb = fmaxf(mxb, sacc[j][2 + e]);
      }
    }
    mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
    mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
    mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
    mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
    uint32_t pa_frag[8], pb_frag[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float p0 = tc::ex2(sacc[j][0] - mxa), p1 = tc::ex2(sacc[j][1] - mxa);
      const float p2 = tc::ex2(sacc[j][2] - mxb), p3 = tc::ex2(sacc[j][3] - mxb);
      sa += p0 + p1;
      sb += p2 + p3;
      pa_frag[j] = fr_pack2(p0, p1);
      pb_frag[j] = fr_pack2(p2, p3);
    }
    sa += __shfl_xor_sync(0xffffffffu, sa, 1);
    sa += __shfl_xor_sync(0xffffffffu, sa, 2);
    sb += __shfl_xor_sync(0xffffffffu, sb, 1);
    sb += __shfl_xor_sync(0xffffffffu, sb, 2);
    // O~2 = P~ V, all D columns
    float oacc[NTW][4];
#pragma unroll
    for (int j = 0; j < NTW; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      if (16 * kk < bpad) {
        const uint32_t a0 = pa_frag[2 * kk], a1 = pb_frag[2 * kk], a2 = pa_frag[2 * kk + 1],
                       a3 = pb_frag[2 * kk + 1];
#pragma unroll
        for (int jp = 0; jp < NTW / 2; ++jp) {
          uint32_t b0, b1, b2, b3;
          fr_ldsm_x4_t(vs_a + (16 * kk + v_row) * RS + (16 * jp + v_col) * 2, b0, b1, b2, b3);
          fr_mma(oacc[2 * jp], a0, a1, a2, a3, b0, b1);
          fr_mma(oacc[2 * jp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    // merge with the cached state, normalise, store
    const float m2a = mxa * LN2, m2b = mxb * LN2;
    const float Ma = fmaxf(m1a, m2a), Mb = fmaxf(m1b, m2b);
    const float w1a = lse_weight(m1a, Ma), w2a = expf(m2a - Ma);
    const float w1b = lse_weight(m1b, Mb), w2b = expf(m2b - Mb);
    const float lta = w1a * l1a + w2a * sa, ltb = w1b * l1b + w2b * sb;
    const float ia = 1.f / lta, ib = 1.f / ltb;
    __nv_bfloat16 *da = a.out + (((long long)b * U + i0 + lr) * g.hq + h) * D + lc;
    __nv_bfloat16 *db = da + 8ll * g.hq * D;
#pragma unroll
    for (int j = 0; j < NTW; ++j) {
      if (va)
        *reinterpret_cast<uint32_t *>(da + 8 * j) = fr_pack2((w1a * o1a[j].x + w2a * oacc[j][0]) * ia,
                                                             (w1a * o1a[j].y + w2a * oacc[j][1]) * ia);
      if (vbr)
        *reinterpret_cast<uint32_t *>(db + 8 * j) = fr_pack2((w1b * o1b[j].x + w2b * oacc[j][2]) * ib,
                                                             (w1b * o1b[j].y + w2b * oacc[j][3]) * ib);
    }
    if (a.lse && (lane & 3) == 0) {
      if (va) a.lse[pa] = Ma + logf(lta);
      if (vbr) a.lse[pb] = Mb + logf(ltb);
    }
  }
}

template <int D>
cudaError_t launch_d(const Geometry &g, const FacRowsArgs &a0, int sms, cudaStream_t st) {
  const FacRowsLayout<D> lay(g.blk);
  auto kern = facache_rows_kernel<D>;
  if (lay.bytes > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.bytes);
    if (e != cudaSuccess) return e;
  }
  // one wave of resident CTAs spread over the units (each CTA's warps then
  // stride over equal shares of its unit's tiles), never more CTAs per unit
  // than it has tiles for whole warps
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, FR_WARPS * 32, lay.bytes);
  if (e != cudaSuccess) return e;
  FacRowsArgs a = a0;
  const long long units = (long long)g.batch * g.hkv;
  const long long tiles = (long long)g.group * ((a.n_rows + FR_ROWS - 1) / FR_ROWS);
  long long per_unit = (long long)sms * (per_sm > 0 ? per_sm : 1) / units;
  per_unit = per_unit < 1 ? 1 : per_unit;
  const long long max_per_unit = (tiles + FR_WARPS - 1) / FR_WARPS;
  a.ctas_per_unit = (int)(per_unit < max_per_unit ? per_unit : max_per_unit);
  const long long ctas = units * a.ctas_per_unit;
  if (ctas > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  return launch_pdl(kern, dim3((unsigned)ctas), dim3(FR_WARPS * 32), lay.bytes, st, g, a);
}

// Rotation base of every chunk of U's rows for one sequence: the chunks before
// the block start at positions 0, cmax, 2 cmax, ...; those after it at
// c0 + B + j cmax (U's row c0 + j cmax sits at that position).
__global__ void chunk_positions_kernel(int *pos, int n_before, int n_after, int c0, int cmax, int blk) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < n_before) pos[k] = k * cmax;
  else if (k < n_before + n_after) pos[k] = c0 + (k - n_before) * cmax + blk;
}

}  // namespace

cudaError_t launch_chunk_positions(int *pos, int n_before, int n_after, int c0, int cmax, int blk, cudaStream_t st) {
  const int n = n_before + n_after;
  if (n == 0) return cudaSuccess;
  chunk_positions_kernel<<<(n + 255) / 256, 256, 0, st>>>(pos, n_before, n_after, c0, cmax, blk);
  return cudaGetLastError();
}

cudaError_t launch_facache_rows(const Geometry &g, const FacRowsArgs &a, int sms, cudaStream_t st) {
  return g.d == 128 ? launch_d<128>(g, a, sms, st) : launch_d<64>(g, a, sms, st);
}

}  // namespace fbk
