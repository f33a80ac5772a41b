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
// The step moves a few MB and is latency-bound, so both variants are built
// around one DRAM round trip: every input of the CTA is requested up front
// (cp.async for block V, register loads for block K, the query rows and the
// prefix state; K and Q are rotated in registers as they arrive and stored
// once), and the rest runs from shared memory and registers.
//  * FBK_BF16: a CTA holds RT tiles of 16 query rows of one (sequence,
//    kv-head) unit and that unit's block K/V. S = Q^ K^T and O = P~ V are
//    warp-level bf16 tensor-core MMAs (mma.sync m16n8k16, fp32 accumulation;
//    at 16 x B x d these products are far too small for the TMEM/tcgen05
//    machinery to pay off). With few row tiles, 4 warps per tile split the
//    keys of S and the columns of O, keeping each warp's chain of dependent
//    steps short (what a step's latency is made of); with many, one warp per
//    tile does the fewest instructions. The RoPE table depends on kernel
//    parameters only (rotation at block offsets, see the kernel) and is built
//    before the kernel waits for its predecessor.
//  * FBK_FP32_CHECK: the same steps on CUDA cores in fp32 (no bf16 rounding of
//    Q^, K^ or P~): lane j scores keys j and j + 32, warp-shuffle row max/sum.
#include "launch.h"
#include "tc.cuh"

namespace fbk {
namespace {

// ====================================================================== bf16 (tensor cores)

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D (16x8 fp32) += A (16x16 bf16, row) * B (16x8 bf16, col)
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr));
}

constexpr int STEP_ROWS = 16;  // query rows of one row tile: one m16 MMA tile

// WPT warps per row tile (1: one warp does the whole tile; 4: the warps split
// the keys of S and the columns of O), RT row tiles per CTA.
template <int D, int WPT, int RT>
struct StepLayout {  // byte offsets in shared memory, all 16-byte aligned
  static constexpr int RS = D * 2 + 16;  // padded bf16 row: the 8 rows of an ldmatrix hit distinct banks
  int bpad, ps_stride, ks, vs, qs, ps, red, cs, dq, dc, rq, bytes;
  __host__ __device__ StepLayout(int blk, bool drift = false) {
    bpad = (blk + 15) & ~15;
    ps_stride = bpad * 2 + 16;
    ks = 0;
    vs = ks + bpad * RS;
    qs = vs + bpad * RS;
    ps = qs + RT * STEP_ROWS * RS;
    red = ps + (WPT > 1 ? RT * STEP_ROWS * ps_stride : 0);     // P~ of each row tile (bf16)
    cs = red + (WPT > 1 ? 2 * RT * WPT * STEP_ROWS * 4 : 0);   // [2][RT][WPT][16] fp32 max, sum
    dq = cs + blk * (D / 2) * 8;                              // [blk][D/2] (cos, sin)
    // adaptive refresh only: the query rows of the next step and of the
    // state's step ([2][rows][RS]), then 1 - cos per row (fp32)
    dc = dq + (drift ? 2 * RT * STEP_ROWS * RS : 0);
    rq = dc + (drift ? RT * STEP_ROWS * 4 : 0);
    bytes = rq + RT * STEP_ROWS * 16;  // per query row: its offset in q (8 bytes) and token (4 bytes)
  }
};

// bf16 step kernel: one CTA per (unit, RT tiles of 16 query rows); the CTA
// stages the unit's block K/V and RoPE table once for all its row tiles.
//
// RoPE at block offsets. The block's queries and keys sit at L_b + t. A score
// depends on the two positions only through their difference (RoPE's
// rotation matrices compose: R(a)^T R(b) = R(b - a)), so rotating Q and K at t
// alone gives the same scores exactly in real arithmetic; only the rounding
// of the rotated bf16 operands differs. The cos/sin table then depends on the
// kernel parameters only and is built before the kernel waits for its
// predecessor; prefix_lens is not needed on this path.
//
// WPT = 4: warp w of a row tile computes S for the key n-tiles w and w + 4
// (8 keys each), the row max and sum are combined across the tile's warps
// through shared memory, P~ goes to shared memory as bf16, and warp w then
// forms O~2 = P~ V and the merged output for its D/4 columns. Short chains
// per warp: the choice when there are few row tiles.
// WPT = 1: one warp computes all of S, the softmax on the accumulator
// fragments (quad shuffles), O~2 = P~ V with P~ re-packed in registers as the
// A operand, and all D columns. Fewest instructions per row: the choice when
// there are many row tiles.
template <int D, int WPT, int RT>
__global__ void __launch_bounds__(RT * WPT * 32) block_merge_mma_kernel(
    Geometry g, const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ kb,
    const __nv_bfloat16 *__restrict__ vb, fbk_partial pfx, __nv_bfloat16 *__restrict__ out,
    float *__restrict__ lse, int tiles, DriftArgs dr) {
  using L = StepLayout<D, WPT, RT>;
  constexpr int CTA_ROWS = RT * STEP_ROWS, NTHREADS = RT * WPT * 32;
  constexpr int HALF = D / 2, CH = D / 8, RS = L::RS;
  constexpr int COLS_W = D / WPT, NTW = COLS_W / 8;  // output columns (n-tiles) per warp
  extern __shared__ float4 smem_f4[];
  uint8_t *sm = reinterpret_cast<uint8_t *>(smem_f4);
  const int blk = g.blk;
  const bool drift = dr.q_base != nullptr && dr.next_step >= 0;
  const L lay(blk, dr.q_base != nullptr);
  const int bpad = lay.bpad, NT = bpad / 8, PSS = lay.ps_stride;
  uint8_t *Ks = sm + lay.ks, *Vs = sm + lay.vs, *Qs = sm + lay.qs, *Ps = sm + lay.ps;
  float *red_max = reinterpret_cast<float *>(sm + lay.red);
  float *red_sum = red_max + RT * WPT * STEP_ROWS;
  float2 *cs = reinterpret_cast<float2 *>(sm + lay.cs);
  long long *s_qoff = reinterpret_cast<long long *>(sm + lay.rq);
  int *s_tq = reinterpret_cast<int *>(sm + lay.rq + CTA_ROWS * 8);

  const int u = blockIdx.x / tiles, r0 = (blockIdx.x % tiles) * CTA_ROWS;
  const int b = u / g.hkv, kvh = u % g.hkv;
  const int rows_cta = min(CTA_ROWS, g.rows - r0);
  const int tid = threadIdx.x, lane = tid & 31;
  const int grp = tid / (WPT * 32), warp = (tid >> 5) % WPT;  // row tile of the CTA, warp inside the tile

  // ---- 0. cos/sin of t * theta_i, t < B (kernel parameters only), in fp32:
  // the angle in turns, reduced to [-1, 1], then the fast sine/cosine. At
  // t <= 63 the absolute error stays near 1e-5 rad, far below the bf16
  // rounding of the rotated operands.
  for (int idx = tid; idx < blk * HALF; idx += NTHREADS) {
    const int t = idx / HALF, i = idx % HALF;
    const float f = exp2f(-2.0f * (float)i / (float)D * (float)g.log2_base) * (float)(1.0 / CUDART_PI);
    float x = (float)t * f;
    x -= 2.0f * rintf(0.5f * x);
    float sn, c;
    __sincosf(x * (float)CUDART_PI, &sn, &c);
    // pair i = 8c + 2e + h sits at float2 (t, e, c, h): the 8 lanes that rotate
    // chunks c = 0..7 of one row read 8 consecutive float4 (no bank conflict)
    cs[t * HALF + ((i >> 1) & 3) * (D / 8) + (i >> 3) * 2 + (i & 1)] = make_float2(c, sn);
  }
  // each query row's token and the offset of its row in q (kernel parameters only)
  for (int rr = tid; rr < rows_cta; rr += NTHREADS) {
    const int r = r0 + rr, t = r % blk, h = kvh * g.group + r / blk;
    s_tq[rr] = t;
    s_qoff[rr] = (((long long)b * blk + t) * g.hq + h) * D;
  }
  __syncthreads();
  pdl_wait();
  pdl_release();
  if (dr.clear && blockIdx.x == 0 && tid == 0) *dr.clear = 0;  // this step's refresh request is used up

  // ---- 1. every global read of the CTA, issued at once: block V by cp.async
  // into shared memory; block K and the query rows into registers, in pairs of
  // 16-byte chunks (c, c + D/16) that hold the RoPE pairs (i, i + D/2), to be
  // rotated there; the prefix state into registers (below)
  const long long kv_row0 = (long long)b * blk * g.hkv + kvh;  // token t: row kv_row0 + t*hkv
  for (int idx = tid; idx < blk * CH; idx += NTHREADS) {
    const int t = idx / CH, c = idx % CH;
    cp_async16(Vs + t * RS + c * 16, vb + (kv_row0 + (long long)t * g.hkv) * D + c * 8);
  }
  // B <= 64 (the C ABI rejects longer blocks): MAXI items per thread cover every row
  constexpr int PAIRS = D / 16, MAXI = ((64 + CTA_ROWS) * PAIRS + NTHREADS - 1) / NTHREADS;
  const int nrot = (blk + rows_cta) * PAIRS;
  uint4 xa[MAXI], xb[MAXI];
#pragma unroll
  for (int i = 0; i < MAXI; ++i) {
    const int idx = tid + i * NTHREADS;
    if (idx < nrot) {
      const int rowi = idx / PAIRS, c = idx % PAIRS;
      const __nv_bfloat16 *row = rowi < blk ? kb + (kv_row0 + (long long)rowi * g.hkv) * D : q + s_qoff[rowi - blk];
      xa[i] = __ldg(reinterpret_cast<const uint4 *>(row) + c);
      xb[i] = __ldg(reinterpret_cast<const uint4 *>(row + HALF) + c);
    }
  }
  if (drift) {  // the rows of the next step's queries and of the state's queries
    const __nv_bfloat16 *qn = dr.q_base + (long long)dr.next_step * dr.q_stride;
    const __nv_bfloat16 *qr = dr.q_base + (long long)(*dr.last_refresh) * dr.q_stride;
    for (int idx = tid; idx < rows_cta * CH; idx += NTHREADS) {
      const int rr = idx / CH, c = idx % CH, r = r0 + rr;
      const int t = r % blk, h = kvh * g.group + r / blk;
      const long long off = (((long long)b * blk + t) * g.hq + h) * D + c * 8;
      cp_async16(sm + lay.dq + rr * RS + c * 16, qn + off);
      cp_async16(sm + lay.dq + (CTA_ROWS + rr) * RS + c * 16, qr + off);
    }
  }
  // padding key rows and query rows must be finite zeros
  for (int idx = tid; idx < (bpad - blk) * CH; idx += NTHREADS) {
    const int t = blk + idx / CH, c = idx % CH;
    *reinterpret_cast<uint4 *>(Ks + t * RS + c * 16) = make_uint4(0, 0, 0, 0);
    *reinterpret_cast<uint4 *>(Vs + t * RS + c * 16) = make_uint4(0, 0, 0, 0);
  }
  for (int idx = tid; idx < (CTA_ROWS - rows_cta) * CH; idx += NTHREADS) {
    const int rr = rows_cta + idx / CH, c = idx % CH;
    *reinterpret_cast<uint4 *>(Qs + rr * RS + c * 16) = make_uint4(0, 0, 0, 0);
  }
  // this thread's outputs: rows lr and lr + 8 of its row tile, columns col0 + 8j + lc (+1)
  const int lr = lane >> 2, lc = (lane & 3) * 2, col0 = warp * COLS_W, tr0 = grp * STEP_ROWS;
  const int ra = r0 + tr0 + lr, rb = ra + 8;
  const bool va = tr0 + lr < rows_cta, vbr = tr0 + lr + 8 < rows_cta;
  const int ta = va ? ra % blk : 0, ha = va ? kvh * g.group + ra / blk : 0;
  const int tb_ = vbr ? rb % blk : 0, hb = vbr ? kvh * g.group + rb / blk : 0;
  const long long pa = ((long long)b * g.hq + ha) * blk + ta, pb = ((long long)b * g.hq + hb) * blk + tb_;
  float2 o1a[NTW], o1b[NTW];
  float m1a = -CUDART_INF_F, l1a = 0.f, m1b = -CUDART_INF_F, l1b = 0.f;
#pragma unroll
  for (int j = 0; j < NTW; ++j) {
    o1a[j] = va ? __ldg(reinterpret_cast<const float2 *>(pfx.o_unnorm + pa * D + col0 + 8 * j + lc))
                : make_float2(0.f, 0.f);
    o1b[j] = vbr ? __ldg(reinterpret_cast<const float2 *>(pfx.o_unnorm + pb * D + col0 + 8 * j + lc))
                 : make_float2(0.f, 0.f);
  }
  if (va) { m1a = __ldg(pfx.m + pa); l1a = __ldg(pfx.l + pa); }
  if (vbr) { m1b = __ldg(pfx.m + pb); l1b = __ldg(pfx.l + pb); }
  // ---- 2. rotate block K and the query rows at their block offsets, 8 pairs per item, and store them
#pragma unroll
  for (int i = 0; i < MAXI; ++i) {
    const int idx = tid + i * NTHREADS;
    if (idx < nrot) {
      const int rowi = idx / PAIRS, c = idx % PAIRS;
      const bool is_k = rowi < blk;
      const int t = is_k ? rowi : s_tq[rowi - blk];
      uint8_t *row = is_k ? Ks + rowi * RS : Qs + (rowi - blk) * RS;
      const uint4 a = xa[i], bq = xb[i];
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {bq.x, bq.y, bq.z, bq.w};
      const float4 *cp = reinterpret_cast<const float4 *>(cs + t * HALF + 2 * c);  // + e * (D / 8) float2
      uint32_t y1[4], y2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float4 c2 = cp[e * (D / 16)];  // (cos, sin) of pairs 8c + 2e and 8c + 2e + 1
        const float x1l = __uint_as_float(aw[e] << 16), x1h = __uint_as_float(aw[e] & 0xffff0000u);
        const float x2l = __uint_as_float(bw[e] << 16), x2h = __uint_as_float(bw[e] & 0xffff0000u);
        y1[e] = pack2(x1l * c2.x - x2l * c2.y, x1h * c2.z - x2h * c2.w);
        y2[e] = pack2(x2l * c2.x + x1l * c2.y, x2h * c2.z + x1h * c2.w);
      }
      *reinterpret_cast<uint4 *>(row + c * 16) = make_uint4(y1[0], y1[1], y1[2], y1[3]);
      *reinterpret_cast<uint4 *>(row + D + c * 16) = make_uint4(y2[0], y2[1], y2[2], y2[3]);
    }
  }
  cp_async_wait_all();
  __syncthreads();

  if (drift) {
    // 1 - cos between the next step's and the state's query row, as
    // |q/|q| - r/|r||^2 / 2 (exactly 0 for equal rows; 0 if a row is zero):
    // one warp per row, lanes over the columns
    float *dcos = reinterpret_cast<float *>(sm + lay.dc);
    for (int rr = tid >> 5; rr < rows_cta; rr += NTHREADS / 32) {
      const uint8_t *rq = sm + lay.dq + rr * RS, *rf = sm + lay.dq + (CTA_ROWS + rr) * RS;
      float x[D / 32], y[D / 32], nx = 0.f, ny = 0.f;
#pragma unroll
      for (int e = 0; e < D / 32; ++e) {
        const int col = lane + 32 * e;
        x[e] = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(rq)[col]);
        y[e] = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(rf)[col]);
        nx += x[e] * x[e];
        ny += y[e] * y[e];
      }
      nx = warp_sum(nx);
      ny = warp_sum(ny);
      float dd = 0.f;
      if (nx > 0.f && ny > 0.f) {
        const float ix = rsqrtf(nx), iy = rsqrtf(ny);
#pragma unroll
        for (int e = 0; e < D / 32; ++e) {
          // rounded products (no fused multiply-add), so equal rows give exactly 0
          const float t = __fsub_rn(__fmul_rn(x[e], ix), __fmul_rn(y[e], iy));
          dd += t * t;
        }
      }
      dd = warp_sum(dd);
      if (lane == 0) dcos[rr] = 0.5f * dd;
    }
  }

  const uint32_t qs_a = (uint32_t)__cvta_generic_to_shared(Qs + tr0 * RS),
                 ks_a = (uint32_t)__cvta_generic_to_shared(Ks), vs_a = (uint32_t)__cvta_generic_to_shared(Vs);
  const int a_row = (lane & 7) + 8 * ((lane >> 3) & 1), a_col = 8 * (lane >> 4);  // A fragments (16x16)
  const int v_row = (lane & 7) + 8 * ((lane >> 3) & 1), v_col = 8 * (lane >> 4);  // V (transposed)
  const float sl2 = g.tau * 1.4426950408889634f;
  float mxa = -CUDART_INF_F, mxb = -CUDART_INF_F, sa = 0.f, sbs = 0.f;
  float oacc[NTW][4];
#pragma unroll
  for (int j = 0; j < NTW; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;

  if constexpr (WPT == 1) {
    // ---- 3. S = Q^ K^T, all key n-tiles (up to 64 keys)
    const int b_row = (lane & 7) + 8 * (lane >> 4), b_col = 8 * ((lane >> 3) & 1);
    float sacc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(qs_a + a_row * RS + (16 * kk + a_col) * 2, a0, a1, a2, a3);
#pragma unroll
      for (int jp = 0; jp < 4; ++jp) {
        if (16 * jp < bpad) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(ks_a + (16 * jp + b_row) * RS + (16 * kk + b_col) * 2, b0, b1, b2, b3);
          mma16816(sacc[2 * jp], a0, a1, a2, a3, b0, b1);
          mma16816(sacc[2 * jp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    // ---- 4. softmax on the fragments (rows lr and lr + 8), log2 units
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
    uint32_t pa_frag[8], pb_frag[8];  // P~ as bf16 pairs: [n-tile] for rows lr and lr + 8
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float p0 = tc::ex2(sacc[j][0] - mxa), p1 = tc::ex2(sacc[j][1] - mxa);
      const float p2 = tc::ex2(sacc[j][2] - mxb), p3 = tc::ex2(sacc[j][3] - mxb);
      sa += p0 + p1;
      sbs += p2 + p3;
      pa_frag[j] = pack2(p0, p1);
      pb_frag[j] = pack2(p2, p3);
    }
    sa += __shfl_xor_sync(0xffffffffu, sa, 1);
    sa += __shfl_xor_sync(0xffffffffu, sa, 2);
    sbs += __shfl_xor_sync(0xffffffffu, sbs, 1);
    sbs += __shfl_xor_sync(0xffffffffu, sbs, 2);
    // ---- 5. O~2 = P~ V, all D columns
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      if (16 * kk < bpad) {
        const uint32_t a0 = pa_frag[2 * kk], a1 = pb_frag[2 * kk], a2 = pa_frag[2 * kk + 1],
                       a3 = pb_frag[2 * kk + 1];
#pragma unroll
        for (int jp = 0; jp < NTW / 2; ++jp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vs_a + (16 * kk + v_row) * RS + (16 * jp + v_col) * 2, b0, b1, b2, b3);
          mma16816(oacc[2 * jp], a0, a1, a2, a3, b0, b1);
          mma16816(oacc[2 * jp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
  } else {
    const uint32_t ps_a = (uint32_t)__cvta_generic_to_shared(Ps + tr0 * PSS);
    uint8_t *Pt = Ps + tr0 * PSS;  // this row tile's P~
    float *rmax = red_max + grp * WPT * STEP_ROWS, *rsum = red_sum + grp * WPT * STEP_ROWS;
    // ---- 3. S = Q^ K^T for key n-tiles warp and warp + 4 (16 rows x 8 keys each)
    const int b_row = lane & 7, b_col = 8 * ((lane >> 3) & 1);  // B fragment (k16 x n8)
    float sacc[2][4], sacc2[2][4];  // even and odd kk: two chains of dependent MMAs
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int x = 0; x < 4; ++x) sacc[e][x] = sacc2[e][x] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a0, a1, a2, a3;
      ldsm_x4(qs_a + a_row * RS + (16 * kk + a_col) * 2, a0, a1, a2, a3);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int nt = warp + WPT * e;
        if (nt < NT) {
          uint32_t b0, b1;
          ldsm_x2(ks_a + (8 * nt + b_row) * RS + (16 * kk + b_col) * 2, b0, b1);
          if (kk & 1) mma16816(sacc2[e], a0, a1, a2, a3, b0, b1);
          else mma16816(sacc[e], a0, a1, a2, a3, b0, b1);
        }
      }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int x = 0; x < 4; ++x) sacc[e][x] += sacc2[e][x];
    // ---- 4. block softmax across the tile's warps (log2 units)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int nt = warp + WPT * e;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const bool ok = nt < NT && 8 * nt + lc + c < blk;
        sacc[e][c] = ok ? sacc[e][c] * sl2 : -CUDART_INF_F;
        sacc[e][2 + c] = ok ? sacc[e][2 + c] * sl2 : -CUDART_INF_F;
        mxa = fmaxf(mxa, sacc[e][c]);
        mxb = fmaxf(mxb, sacc[e][2 + c]);
      }
    }
    mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 1));
    mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, 2));
    mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 1));
    mxb = fmaxf(mxb, __shfl_xor_sync(0xffffffffu, mxb, 2));
    if ((lane & 3) == 0) {
      rmax[warp * STEP_ROWS + lr] = mxa;
      rmax[warp * STEP_ROWS + lr + 8] = mxb;
    }
    __syncthreads();
    mxa = mxb = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < WPT; ++w) {
      mxa = fmaxf(mxa, rmax[w * STEP_ROWS + lr]);
      mxb = fmaxf(mxb, rmax[w * STEP_ROWS + lr + 8]);
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int nt = warp + WPT * e;
      if (nt < NT) {
        const float p0 = tc::ex2(sacc[e][0] - mxa), p1 = tc::ex2(sacc[e][1] - mxa);
        const float p2 = tc::ex2(sacc[e][2] - mxb), p3 = tc::ex2(sacc[e][3] - mxb);
        sa += p0 + p1;
        sbs += p2 + p3;
        *reinterpret_cast<uint32_t *>(Pt + lr * PSS + (8 * nt + lc) * 2) = pack2(p0, p1);
        *reinterpret_cast<uint32_t *>(Pt + (lr + 8) * PSS + (8 * nt + lc) * 2) = pack2(p2, p3);
      }
    }
    sa += __shfl_xor_sync(0xffffffffu, sa, 1);
    sa += __shfl_xor_sync(0xffffffffu, sa, 2);
    sbs += __shfl_xor_sync(0xffffffffu, sbs, 1);
    sbs += __shfl_xor_sync(0xffffffffu, sbs, 2);
    if ((lane & 3) == 0) {
      rsum[warp * STEP_ROWS + lr] = sa;
      rsum[warp * STEP_ROWS + lr + 8] = sbs;
    }
    __syncthreads();
    sa = sbs = 0.f;
#pragma unroll
    for (int w = 0; w < WPT; ++w) {
      sa += rsum[w * STEP_ROWS + lr];
      sbs += rsum[w * STEP_ROWS + lr + 8];
    }
    // ---- 5. O~2 = P~ V for this warp's columns
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      if (16 * kk < bpad) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(ps_a + a_row * PSS + (16 * kk + a_col) * 2, a0, a1, a2, a3);
#pragma unroll
        for (int jp = 0; jp < NTW / 2; ++jp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(vs_a + (16 * kk + v_row) * RS + (col0 + 16 * jp + v_col) * 2, b0, b1, b2, b3);
          mma16816(oacc[2 * jp], a0, a1, a2, a3, b0, b1);
          mma16816(oacc[2 * jp + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
  }

  // ---- 6. merge with the prefix state, normalise, store
  const float LN2 = 0.6931471805599453f;
  const float m2a = mxa * LN2, m2b = mxb * LN2;
  const float Ma = fmaxf(m1a, m2a), Mb = fmaxf(m1b, m2b);
  const float w1a = lse_weight(m1a, Ma), w2a = expf(m2a - Ma);
  const float w1b = lse_weight(m1b, Mb), w2b = expf(m2b - Mb);
  const float lta = w1a * l1a + w2a * sa, ltb = w1b * l1b + w2b * sbs;
  const float ia = 1.f / lta, ib = 1.f / ltb;
  __nv_bfloat16 *da = out + (((long long)b * blk + ta) * g.hq + ha) * D + col0 + lc;
  __nv_bfloat16 *db = out + (((long long)b * blk + tb_) * g.hq + hb) * D + col0 + lc;
#pragma unroll
  for (int j = 0; j < NTW; ++j) {
    if (va)
      *reinterpret_cast<uint32_t *>(da + 8 * j) = pack2((w1a * o1a[j].x + w2a * oacc[j][0]) * ia,
                                                        (w1a * o1a[j].y + w2a * oacc[j][1]) * ia);
    if (vbr)
      *reinterpret_cast<uint32_t *>(db + 8 * j) = pack2((w1b * o1b[j].x + w2b * oacc[j][2]) * ib,
                                                        (w1b * o1b[j].y + w2b * oacc[j][3]) * ib);
  }
  if (lse && warp == 0 && (lane & 3) == 0) {
    if (va) lse[pa] = Ma + logf(lta);
    if (vbr) lse[pb] = Mb + logf(ltb);
  }
  if (drift) {
    // drift statistic: the prefix's share of the row's softmax mass times the
    // row's 1 - cos; the maximum over the CTA's rows, then over the grid
    const float *dcos = reinterpret_cast<const float *>(sm + lay.dc);
    float dm = 0.f;
    if (va) dm = fmaxf(dm, w1a * l1a / lta * dcos[tr0 + lr]);
    if (vbr) dm = fmaxf(dm, w1b * l1b / ltb * dcos[tr0 + lr + 8]);
    dm = warp_max(dm);
    if (lane == 0 && dm > 0.f) {
      atomicMax(reinterpret_cast<int *>(dr.drift_out), __float_as_int(dm));  // non-negative floats order as ints
      if (dm > dr.theta)
        for (int j = 0; j < dr.n_next; ++j) dr.next_flags[j] = 1;  // this layer and every deeper one
    }
  }
}

template <int D, int WPT, int RT>
cudaError_t launch_mma_cfg(const Geometry &g, const __nv_bfloat16 *q, const __nv_bfloat16 *kb,
                           const __nv_bfloat16 *vb, const fbk_partial &pfx, void *out, float *lse,
                           cudaStream_t st, const DriftArgs &da) {
  const StepLayout<D, WPT, RT> lay(g.blk, da.q_base != nullptr);
  auto kern = block_merge_mma_kernel<D, WPT, RT>;
  if (lay.bytes > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.bytes);
    if (e != cudaSuccess) return e;
  }
  const int tiles = (g.rows + RT * STEP_ROWS - 1) / (RT * STEP_ROWS);
  const long long ctas = (long long)g.batch * g.hkv * tiles;
  if (ctas > 0x7fffffffll) return cudaErrorInvalidConfiguration;
  return launch_pdl(kern, dim3((unsigned)ctas), dim3(RT * WPT * 32), lay.bytes, st, g, q, kb, vb, pfx,
                    static_cast<__nv_bfloat16 *>(out), lse, tiles, da);
}

// Layout choice from the number of 16-row tiles n = units * ceil(G*B / 16),
// fitted to measurements on the five workload shapes: with n at least 4 per SM
// the step is throughput-bound and one warp per tile (4 tiles per CTA) does
// the fewest instructions; below that it is latency-bound and 4 warps per tile
// shorten each warp's chain, with RT the largest of {1, 2, 4} that still gives
// about one CTA per SM (at least 85% of the SM count).
template <int D>
cudaError_t launch_mma(const Geometry &g, const __nv_bfloat16 *q, const __nv_bfloat16 *kb,
                       const __nv_bfloat16 *vb, const fbk_partial &pfx, void *out, float *lse,
                       cudaStream_t st, const DriftArgs &da) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long units = (long long)g.batch * g.hkv, t16 = (g.rows + STEP_ROWS - 1) / STEP_ROWS;
  if (units * t16 >= 4ll * sms) return launch_mma_cfg<D, 1, 4>(g, q, kb, vb, pfx, out, lse, st, da);
  int rt = 1;
  for (int c = 4; c > 1; c >>= 1)
    if (c <= t16 && units * ((t16 + c - 1) / c) * 20 >= 17ll * sms) { rt = c; break; }
  switch (rt) {
    case 4: return launch_mma_cfg<D, 4, 4>(g, q, kb, vb, pfx, out, lse, st, da);
    case 2: return launch_mma_cfg<D, 4, 2>(g, q, kb, vb, pfx, out, lse, st, da);
    default: return launch_mma_cfg<D, 4, 1>(g, q, kb, vb, pfx, out, lse, st, da);
  }
}

// ====================================================================== fp32 check (CUDA cores)

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

template <int D, int RPW>
__global__ void __launch_bounds__(THREADS) block_merge_f32_kernel(
    Geometry g, const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ kb,
    const __nv_bfloat16 *__restrict__ vb, fbk_partial pfx, float *__restrict__ out,
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
  const double rope_f = freq_over_pi(tid % HALF, D, g.log2_base);
  pdl_wait();
  pdl_release();
  int L = g.lens[b];
  if (L < 0) {
    raise_flag(g, FBK_DEVERR_PREFIX_LEN);
    L = 0;
  }

  const long long kv_row0 = ((long long)b * blk) * g.hkv + kvh;
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
  {  // RoPE table, accurate sincospi (check mode); each thread keeps one frequency
    const int i = tid % HALF;
    for (int t = tid / HALF; t < blk; t += THREADS / HALF) cs[t * HALF + i] = rope_cs_f32(L + t, rope_f);
  }
  cp_async_wait_all();
  __syncthreads();

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
    float *dst = out + (((long long)b * blk + t) * g.hq + h) * D + lane * CPL;
#pragma unroll
    for (int c = 0; c < CPL; ++c) dst[c] = (w1 * o1[c] + w2 * ob[c]) * inv;
    if (lse && lane == 0) lse[((long long)b * g.hq + h) * blk + t] = mm + logf(lt);
    __syncwarp();
  }
}

template <int D, int RPW>
cudaError_t launch_f32_cfg(const Geometry &g, const __nv_bfloat16 *q, const __nv_bfloat16 *kb,
                           const __nv_bfloat16 *vb, const fbk_partial &pfx, void *out, float *lse,
                           cudaStream_t st) {
  constexpr int RC = WARPS * RPW;
  const Layout lay(D, g.blk, RC);
  auto kern = block_merge_f32_kernel<D, RPW>;
  if (lay.bytes > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, lay.bytes);
    if (e != cudaSuccess) return e;
  }
  dim3 grid((g.rows + RC - 1) / RC, g.batch * g.hkv);
  return launch_pdl(kern, grid, dim3(THREADS), lay.bytes, st, g, q, kb, vb, pfx,
                    static_cast<float *>(out), lse);
}

template <int D>
cudaError_t launch_f32(const Geometry &g, const __nv_bfloat16 *q, const __nv_bfloat16 *kb,
                       const __nv_bfloat16 *vb, const fbk_partial &pfx, void *out, float *lse,
                       cudaStream_t st) {
  const long long units = (long long)g.batch * g.hkv;
  if (units * ((g.rows + 7) / 8) <= 512) return launch_f32_cfg<D, 2>(g, q, kb, vb, pfx, out, lse, st);
  return launch_f32_cfg<D, 8>(g, q, kb, vb, pfx, out, lse, st);
}

}  // namespace

cudaError_t launch_block_merge(const Geometry &g, const __nv_bfloat16 *q,
                               const __nv_bfloat16 *kb, const __nv_bfloat16 *vb,
                               const fbk_partial &pfx, void *out, float *lse, bool f32_out,
                               cudaStream_t st, const DriftArgs *drift) {
  if (f32_out) {
    if (drift) return cudaErrorInvalidValue;  // the adaptive refresh runs on the bf16 path
    return g.d == 128 ? launch_f32<128>(g, q, kb, vb, pfx, out, lse, st)
                      : launch_f32<64>(g, q, kb, vb, pfx, out, lse, st);
  }
  const DriftArgs da = drift ? *drift : DriftArgs{nullptr, 0, nullptr, -1, nullptr, nullptr, 0, 0.f, nullptr};
  return g.d == 128 ? launch_mma<128>(g, q, kb, vb, pfx, out, lse, st, da)
                    : launch_mma<64>(g, q, kb, vb, pfx, out, lse, st, da);
}

}  // namespace fbk
