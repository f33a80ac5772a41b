// Shared device helpers of the cached block attention kernels (sm_100a).
//
// Contents: the kernel-side view of a call (Geometry), prefix-length checks,
// the work list that splits the prefix keys into equal shares, RoPE angle
// helpers, bf16 conversions and the device error flag.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math_constants.h>
#include <stdint.h>

#include "fbk.h"

namespace fbk {

// Keys per work-list tile: the prefix of every (sequence, kv-head) pair is cut
// into ceil(L_b / KV_TILE) tiles, and all tiles of all pairs form one list.
constexpr int KV_TILE = 64;

// Everything a kernel needs to know about one call. Passed by value.
struct Geometry {
  int batch, hq, hkv, group, d, blk, rows;  // rows = group * blk (query rows per kv-head)
  float tau;                                // softmax scale
  double log2_base;                         // log2(rope base)
  double inv_freq_over_pi[64];              // base^(-2i/d) / pi, i < d/2 (host pow())
  // cache
  const __nv_bfloat16 *kc, *vc;
  int paged, page_size, page_shift, max_pages;
  long long cap, num_pages;
  const int *page_table;
  const int *lens;
  int *err;
};

__device__ __forceinline__ void raise_flag(const Geometry &g, unsigned bits) {
  if (g.err) atomicOr(g.err, (int)bits);
}

// Number of tokens the cache can hold for one sequence.
__host__ __device__ __forceinline__ long long seq_capacity(const Geometry &g) {
  return g.paged ? (long long)g.max_pages * g.page_size : g.cap;
}

// Committed prefix length of sequence b as the prefix kernels see it: a value
// outside [0, capacity] is flagged and the sequence is treated as empty, so no
// kernel reads outside the cache.
__device__ __forceinline__ int prefix_len(const Geometry &g, int b) {
  int L = g.lens[b];
  if (L < 0 || (long long)L > seq_capacity(g)) {
    raise_flag(g, FBK_DEVERR_PREFIX_LEN);
    return 0;
  }
  return L;
}

__host__ __device__ __forceinline__ int tiles_of(int L) { return (L + KV_TILE - 1) / KV_TILE; }

// In the work list every non-empty unit occupies UNIT_LEAD positions before
// its tiles. They carry no work: a share whose range starts a new unit pays
// for the switch (a piece epilogue and the next piece's start, a few tiles'
// time) in list positions, so the shares that hold several pieces get fewer
// tiles and finish with the others.
constexpr int UNIT_LEAD = 4;
__host__ __device__ __forceinline__ int span_of(int L) {
  const int tb = tiles_of(L);
  return tb > 0 ? tb + UNIT_LEAD : 0;
}

// Share c of P covers list positions [c*T/P, (c+1)*T/P).
// floor(n / d) for 0 <= n, 1 <= d < 2^31. Below 2^53 the quotient comes from
// one fp64 division (correctly rounded, so within one of the true quotient)
// and one integer correction, instead of a 64-bit integer division routine.
__host__ __device__ __forceinline__ long long floordiv_nonneg(long long n, long long d) {
  if (n >= (1ll << 53)) return n / d;
  long long q = (long long)((double)n / (double)d);
  if (q * d > n) --q;
  else if ((q + 1) * d <= n) ++q;
  return q;
}

__host__ __device__ __forceinline__ long long share_begin(long long c, long long T, long long P) {
  return floordiv_nonneg(c * T, P);
}

// The share that holds list position x (largest c with share_begin(c) <= x).
__device__ __forceinline__ long long share_of(long long x, long long T, long long P) {
  return floordiv_nonneg((x + 1) * P - 1, T);
}

// Per-sequence list lengths, loaded once per CTA: s_len[b] = validated L_b,
// s_scan[b] = Hkv * sum_{b' <= b} span_of(L_b') (inclusive scan; the host
// keeps the total below 2^31). All threads call it; the loads are issued in
// parallel, one per thread. Returns T, the total list length.
constexpr int MAX_BATCH = 1024;  // sequences per call (shared-memory scan)

__device__ __forceinline__ int load_tile_scan(const Geometry &g, int *s_len, int *s_scan) {
  for (int b = threadIdx.x; b < g.batch; b += blockDim.x) s_len[b] = prefix_len(g, b);
  __syncthreads();
  if (threadIdx.x < 32) {  // one warp scans 32 sequences per round
    int carry = 0;
    for (int b0 = 0; b0 < g.batch; b0 += 32) {
      const int b = b0 + (int)threadIdx.x;
      int v = b < g.batch ? g.hkv * span_of(s_len[b]) : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if ((int)threadIdx.x >= o) v += n;
      }
      if (b < g.batch) s_scan[b] = carry + v;
      carry += __shfl_sync(0xffffffffu, v, 31);
    }
  }
  __syncthreads();
  return g.batch > 0 ? s_scan[g.batch - 1] : 0;
}

// A piece: the intersection of one share with one (sequence, kv-head) unit.
// Unit u = b * Hkv + kvh. Its state goes to workspace slot (share + u), which
// is unique because every new piece of the list advances the share, the unit,
// or both.
struct Piece {
  int b, kvh, u, L;
  int tile_begin, tile_end;  // tile indices inside the unit
};

// Walks the pieces of one share in list order, reading the shared-memory
// scan. Every warp role of a kernel runs its own copy; the walk is
// deterministic, so all copies agree.
struct PieceWalker {
  long long pos, end;  // list positions still to cover
  int b;               // current sequence
  const int *len;
  const int *scan;

  __device__ __forceinline__ void init(const Geometry &g, const int *s_len, const int *s_scan,
                                       long long share, long long T, long long P) {
    pos = share_begin(share, T, P);
    end = share_begin(share + 1, T, P);
    len = s_len;
    scan = s_scan;
    // first sequence whose scan passes pos (binary search; scan is non-decreasing)
    int lo = 0, hi = g.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (scan[mid] > pos) hi = mid; else lo = mid + 1;
    }
    b = lo;
  }

  __device__ __forceinline__ bool next(const Geometry &g, Piece &p) {
    while (pos < end) {
      while (pos >= scan[b]) {
        if (++b >= g.batch) {  // unreachable while the scan is consistent
          pos = end;
          return false;
        }
      }
      const int L = len[b], tb = tiles_of(L), span = tb + UNIT_LEAD;  // tb > 0: the scan grew at b
      const long long acc = scan[b] - (long long)g.hkv * span;       // list position where sequence b starts
      const int kvh = (int)(pos - acc) / span;                       // < Hkv * span < 2^31
      const long long ustart = acc + (long long)kvh * span, first = ustart + UNIT_LEAD;
      const long long stop = ustart + span < end ? ustart + span : end;
      const long long lo = pos > first ? pos : first;
      pos = stop;
      if (lo >= stop) continue;  // only lead positions of this unit in the share
      p.b = b;
      p.kvh = kvh;
      p.u = b * g.hkv + kvh;
      p.L = L;
      p.tile_begin = (int)(lo - first);
      p.tile_end = (int)(stop - first);
      return true;
    }
    return false;
  }
};

// Row (of the 2-D [rows, d] view of the cache) that holds token `pos` of
// sequence b, kv-head kvh; -1 (and a flag) for a bad page id.
__device__ __forceinline__ long long cache_row(const Geometry &g, int b, int kvh, long long pos) {
  if (!g.paged) return ((long long)b * g.hkv + kvh) * g.cap + pos;
  int page = g.page_table[(long long)b * g.max_pages + (pos >> g.page_shift)];
  if (page < 0 || (long long)page >= g.num_pages) {
    raise_flag(g, FBK_DEVERR_PAGE_ID);
    return -1;
  }
  return ((long long)page * g.hkv + kvh) * g.page_size + (pos & (g.page_size - 1));
}

// ------------------------------------------------------------------ RoPE
// Rotate-half RoPE: pair (x_i, x_{i+d/2}) turns by pos * theta_i with
// theta_i = base^(-2i/d) (LaCache §3.3.2, Eq. 1; RoFormer). The angle is
// formed in fp64 as a multiple of pi, reduced to [-1, 1] exactly in fp64, and
// only then handed to CUDA's sincospi, so positions near 1.3e5 keep full
// fp32 accuracy.
// theta_i / pi computed in registers (no divergent parameter-space reads):
// exp2(-(2i/d) log2(base)) in fp64, relative error ~2e-15, i.e. < 3e-10 rad at
// position 1.3e5. The commit kernel, whose rounded output is compared bit for
// bit, reads the host-computed pow() table instead.
__device__ __forceinline__ double freq_over_pi(int i, int d, double log2_base) {
  return exp2(-2.0 * i / d * log2_base) * (1.0 / CUDART_PI);
}

__device__ __forceinline__ double rope_turns(int pos, double inv_freq_over_pi) {
  double t = (double)pos * inv_freq_over_pi;
  return t - 2.0 * rint(0.5 * t);
}

__device__ __forceinline__ float2 rope_cs_f32(int pos, double inv_freq_over_pi) {
  float s, c;
  sincospif((float)rope_turns(pos, inv_freq_over_pi), &s, &c);
  return make_float2(c, s);
}

// Same angle, fp64-reduced to [-pi, pi], then CUDA's fast __sincosf: absolute
// error ~5e-7, for the per-step kernels where a full sincospi per element would
// dominate the latency.
__device__ __forceinline__ float2 rope_cs_fast(int pos, double inv_freq_over_pi) {
  float s, c;
  __sincosf((float)(rope_turns(pos, inv_freq_over_pi) * CUDART_PI), &s, &c);
  return make_float2(c, s);
}

__device__ __forceinline__ void rope_cs_f64(int pos, double inv_freq_over_pi, double *c, double *s) {
  sincospi(rope_turns(pos, inv_freq_over_pi), s, c);
}

// ------------------------------------------------------------------ bf16
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
  return __uint_as_float(((uint32_t)h) << 16);
}

// fp64 -> bf16 with a single rounding to nearest even, through fp32 rounded
// to odd (Boldo and Melquiond, "When double rounding is odd"): truncate to
// fp32, set its last bit when the truncation was inexact, then round that fp32
// value to nearest-even bf16. fp32 carries 16 more significand bits than bf16
// (the method needs 2), in the normal and the subnormal range alike, since
// both formats share the 8-bit exponent, so the two roundings give the result
// of one.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  const float f = __double2float_rz(x);
  uint32_t u = __float_as_uint(f);
  if ((double)f != x) u |= 1u;
  return __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(u)));
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Scale factor e^(m_part - m) of a state whose max is m_part when the merged
// max is m; an empty state (m_part = -inf) contributes 0.
__device__ __forceinline__ float lse_weight(float m_part, float m) {
  return m_part == -CUDART_INF_F ? 0.f : expf(m_part - m);
}

// Ampere-style asynchronous global -> shared copies (issued together, waited once).
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gsrc)
               : "memory");
}

__device__ __forceinline__ void cp_async4(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gsrc)
               : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Programmatic dependent launch. Every kernel of the library is launched with
// programmatic stream serialization, so it may become resident while the
// kernel before it in the stream is still running. pdl_wait() returns once
// that predecessor has completed and its writes are visible: each kernel calls
// it before its first read of anything another kernel may have written
// (inputs, prefix lengths, states), and before its first global write. Only
// work on kernel parameters and shared memory comes before it. pdl_release()
// lets the next kernel in the stream start launching; each kernel calls it
// right after its wait, so that only the next kernel runs ahead (its CTAs do
// their parameter-only set-up while this one works) instead of the whole
// chain piling up on the SMs. Both are no-ops for a kernel launched without
// the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_release() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Workspace view of the per-share states written by the prefix kernels.
struct Workspace {
  float *o;  // [slots, rows, d]
  float *m;  // [slots, rows]
  float *l;  // [slots, rows]
  long long slots;
  __nv_bfloat16 *qrot;  // [units, MT * 128, d]: rotated block queries (bf16 mode)
};

}  // namespace fbk
