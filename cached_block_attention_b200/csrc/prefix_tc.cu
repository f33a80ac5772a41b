// Prefix state on the 5th-generation tensor cores (FBK_BF16).
//
// What it computes: for every (sequence b, kv-head) unit, the online-softmax
// state (O~, m, l) of the G*B block query rows of that kv-head over the cached
// prefix keys 0..L_b-1: the FlashAttention recurrence of LaCache §3.3.3
// (Eq. 2-6) whose result FACache keeps in HBM, here for the block's own query
// rows (FlashBlock, Abstract: cached block-external attention).
//
// How (one CTA per SM-sized share of the flattened (unit, 64-key tile) list,
// each unit preceded by a few lead positions that stand for the cost of
// switching units), warp-specialised, each role one elected lane or one
// warpgroup. The block queries were rotated beforehand by rope_q_kernel into
// the workspace, in this kernel's M-tile order:
//  * warps 0 and 3: TMA producers of 64-key K and V tiles of the bf16 cache
//    (contiguous rows or pages) into NS-stage rings, 128-byte swizzled, L2
//    evict-first (each KV byte is read once). K and V have separate rings and
//    producers: a K stage frees as soon as S = Q K^T is done, a V stage only
//    after O += P~ V, so K runs ahead of V.
//  * warp 1: loads each piece's rotated query rows by TMA (into one of two Q
//    buffers where shared memory allows, so the next piece's rows arrive
//    while this one streams) and issues S = Q K^T (M = 128 query rows, N = 64
//    keys, K = d) into a double-buffered TMEM S; warp 2: issues O += P~ V (M = 128, N = d,
//    K = 64 keys) into a TMEM accumulator. Both are tcgen05.mma kind::f16 with
//    fp32 accumulation; two issuers keep a late K tile from holding back a
//    ready PV product.
//  * warps 4..4+4*MT-1: one warpgroup per 128-row M-tile (MT = ceil(G*B/128)).
//    GQA packing: all G query heads of a kv-head share each staged K/V tile,
//    so every KV byte is read from HBM once per unit. Each thread owns one
//    query row = one TMEM lane: it reads its S row from TMEM, applies the
//    recurrence in the log2 domain (paired fp32 instructions where they
//    apply: the loop is issue-bound) and writes P~ (bf16) for the PV MMA.
//    The O accumulator stays in TMEM; it is rescaled only when the running
//    max grows by more than 2^8 over the reference max, which leaves the
//    state exact (O~ and l share one reference max) and bounds P~ by 256.
//    At the end of a piece the state is rebased to the true max and written
//    to this share's workspace slot.
// Every mbarrier wait is bounded (about a second); a timeout flags
// FBK_DEVERR_TIMEOUT and all roles drain and return.
#include <cudaTypedefs.h>

#include <algorithm>

#include "launch.h"
#include "prefix_at.h"
#include "tc.cuh"

namespace fbk {
namespace {

using namespace tc;

template <int D, int MT>
struct Cfg {
  static constexpr int NS = (D == 128) ? 4 : 8;        // K and V ring depth
  // Q buffers: two where shared memory allows (all but d = 128 with two
  // M-tiles), so the next piece's query rows load while this piece streams
  static constexpr int QB = (D == 128 && MT == 2) ? 1 : 2;
  static constexpr int Q_BYTES = 128 * D * 2;          // one M-tile of Q
  static constexpr int KV_BYTES = KV_TILE * D * 2;     // one K (or V) stage
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + QB * MT * Q_BYTES;
  static constexpr int V_OFF = K_OFF + NS * KV_BYTES;
  static constexpr int BAR_OFF = V_OFF + NS * KV_BYTES;
  // barrier indices
  static constexpr int B_KFULL = 0, B_KEMPTY = NS, B_VFULL = 2 * NS, B_VEMPTY = 3 * NS;
  static constexpr int B_QLOAD = 4 * NS;              // [QB]: a piece's rotated query rows landed (TMA)
  static constexpr int B_SFULL = B_QLOAD + QB;        // [MT][2]
  static constexpr int B_SEMPTY = B_SFULL + 2 * MT;   // [MT][2]: S buffer (and the P~ in it) free
  // [MT][2]: P~ of the tile in S buffer `buf` is written. One barrier per S
  // buffer, so an arrival for tile i+1 can never count toward tile i.
  static constexpr int B_PFULL = B_SEMPTY + 2 * MT;
  static constexpr int B_ODONE = B_PFULL + 2 * MT;
  static constexpr int B_OFREE = B_ODONE + MT;
  static constexpr int B_DRAIN = B_OFREE + MT;  // [2]: S issuer, PV issuer
  static constexpr int B_VTAIL = B_DRAIN + 2;   // a partial V tile's own loads landed (V producer only)
  static constexpr int NBAR = B_VTAIL + 1;
  static constexpr int LEN_OFF = BAR_OFF + NBAR * 8;  // [MAX_BATCH] int: validated L_b
  static constexpr int SCAN_OFF = LEN_OFF + MAX_BATCH * 4;  // [MAX_BATCH] int: tile scan
  static constexpr int MISC_OFF = SCAN_OFF + MAX_BATCH * 4;
  static constexpr int SMEM = MISC_OFF + 16 + 1024;   // + slack to align the base to 1024
  static constexpr int THREADS = 128 + 128 * MT;
  static constexpr int TMEM_S = 0;                    // S[mt][buf] at (2*mt + buf) * 64
  static constexpr int TMEM_O = MT * 2 * KV_TILE;     // O[mt] at TMEM_O + mt * D
  static constexpr int TMEM_USED = TMEM_O + MT * D;
  static constexpr int TMEM_COLS = TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(TMEM_USED <= 512, "tensor memory budget");
};

__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_test(bar, parity))
    if (clock64() - t0 > wait_limit()) return false;
  return true;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

// Keys of list tile j of piece p that exist (the unit's last tile may be partial).
__device__ __forceinline__ int tile_keys(const Piece &p, int j) { return min(KV_TILE, p.L - j * KV_TILE); }

// Rows a tile load brings in for n valid keys: whole boxes of boxh rows, then
// 8-row boxes for the rest, so up to 7 rows past the unit's last key may be
// loaded (their K only meets masked scores; their V rows are zeroed before the
// P~ V product reads them).
__device__ __forceinline__ int tile_rows(int n, int boxh) {
  const int full = n / boxh * boxh;
  return full + ((n - full + 7) & ~7);
}

// TMA loads of the n valid keys of tile j into a stage (each 64-column block
// of the stage holds KV_TILE rows of 128 bytes, 128B swizzle). Rows past the
// unit's keys are never requested in whole boxes: they may lie in memory the
// caller never wrote.
template <int D>
__device__ __forceinline__ void load_kv_tile(const Geometry &g, const CUtensorMap *map, const CUtensorMap *map8,
                                             uint32_t dst, const Piece &p, int j, int n, int boxh, uint32_t bar,
                                             uint64_t pol) {
  int r = 0;
  while (r < n) {
    const bool whole = n - r >= boxh;
    long long row = cache_row(g, p.b, p.kvh, (long long)j * KV_TILE + r);
    if (row < 0) row = 0;  // bad page id: flagged; any row keeps the arithmetic going
#pragma unroll
    for (int cb = 0; cb < D / 64; ++cb)
      tma_load_2d(dst + cb * (KV_TILE * 128) + r * 128, whole ? map : map8, cb * 64, (int)row, bar, pol);
    r += whole ? boxh : 8;
  }
}

template <int D, int MT>
__global__ void __launch_bounds__(Cfg<D, MT>::THREADS, 1)
    prefix_tc_kernel(const __grid_constant__ Geometry g, const __nv_bfloat16 *__restrict__ q,
                     const Workspace ws, const int shares, const __grid_constant__ CUtensorMap tmk,
                     const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmk8,
                     const __grid_constant__ CUtensorMap tmv8, const int boxh,
                     const __grid_constant__ CUtensorMap tmq, const int *gate) {
  using C = Cfg<D, MT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t pad = ((raw_addr + 1023u) & ~1023u) - raw_addr;
  uint8_t *smem = smem_raw + pad;
  const uint32_t sb = raw_addr + pad;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int *s_len = reinterpret_cast<int *>(smem + C::LEN_OFF);
  int *s_scan = reinterpret_cast<int *>(smem + C::SCAN_OFF);
  auto bar = [&](int idx) -> uint32_t { return sb + C::BAR_OFF + 8 * idx; };
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::MISC_OFF + 4);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::MISC_OFF);

  // ---- before the wait: nothing another kernel writes is touched here
  // The V ring starts at zero: a stage only ever holds these zeros, rows of
  // committed keys, or rows zeroed after a partial load, so every V row that
  // meets a zero weight in O += P~ V is finite.
  for (int o = threadIdx.x * 16; o < C::NS * C::KV_BYTES; o += C::THREADS * 16)
    *reinterpret_cast<uint4 *>(smem + C::V_OFF + o) = make_uint4(0, 0, 0, 0);
  fence_proxy_async();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) {
      mbar_init(bar(C::B_KFULL + s), 1);
      mbar_init(bar(C::B_KEMPTY + s), 1);
      mbar_init(bar(C::B_VFULL + s), 1);
      mbar_init(bar(C::B_VEMPTY + s), 1);
    }
    for (int qb = 0; qb < C::QB; ++qb) mbar_init(bar(C::B_QLOAD + qb), 1);
    for (int mt = 0; mt < MT; ++mt) {
      mbar_init(bar(C::B_SFULL + 2 * mt), 1);
      mbar_init(bar(C::B_SFULL + 2 * mt + 1), 1);
      mbar_init(bar(C::B_SEMPTY + 2 * mt), 1);
      mbar_init(bar(C::B_SEMPTY + 2 * mt + 1), 1);
      mbar_init(bar(C::B_PFULL + 2 * mt), 128);
      mbar_init(bar(C::B_PFULL + 2 * mt + 1), 128);
      mbar_init(bar(C::B_ODONE + mt), 1);
      mbar_init(bar(C::B_OFREE + mt), 128);
    }
    mbar_init(bar(C::B_DRAIN), 1);
    mbar_init(bar(C::B_DRAIN + 1), 1);
    mbar_init(bar(C::B_VTAIL), 1);
    *abort_flag = 0;
    mbar_fence_init();
    prefetch_tmap(&tmk);
    prefetch_tmap(&tmv);
    prefetch_tmap(&tmq);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_wait();
  pdl_release();
  if (gate && *gate == 0) {  // no refresh of this state at this step (the same for every thread)
    fence_before_sync();
    __syncthreads();  // the allocation's address is in shared memory
    fence_after_sync();
    if (warp == 1) tmem_dealloc(*tmem_slot, C::TMEM_COLS);  // nothing was issued on it
    return;
  }
  fence_before_sync();
  const long long T = load_tile_scan(g, s_len, s_scan);  // reads prefix_lens; two CTA barriers
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  if (T == 0 || share_begin(blockIdx.x, T, shares) == share_begin(blockIdx.x + 1, T, shares)) {
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);  // nothing was issued on it
    return;
  }

  PieceWalker sm_walk;
  Piece sm_piece;
  bool sm_more = false;
  if (warp >= 4) {
    sm_walk.init(g, s_len, s_scan, blockIdx.x, T, shares);
    sm_more = sm_walk.next(g, sm_piece);
  }

  if (warp == 0 || warp == 3) {
    // ---------------------------------------------------------------- producers
    // warp 0 streams K tiles, warp 3 streams V tiles: K stages are released as
    // soon as S = Q K^T is done, V stages only after O += P~ V, so separate
    // producers let the K stream run ahead of the V stream.
    if (lane == 0) {
      const bool is_k = warp == 0;
      const CUtensorMap *map = is_k ? &tmk : &tmv;
      const CUtensorMap *map8 = is_k ? &tmk8 : &tmv8;
      const int b_full = is_k ? C::B_KFULL : C::B_VFULL, b_empty = is_k ? C::B_KEMPTY : C::B_VEMPTY;
      const uint32_t ring = sb + (is_k ? C::K_OFF : C::V_OFF);
      const uint64_t pol = policy_evict_first();
      PieceWalker walk;
      walk.init(g, s_len, s_scan, blockIdx.x, T, shares);
      Piece p;
      int i = 0, ntail = 0;
      bool ok = true;
      while (ok && walk.next(g, p)) {
        for (int j = p.tile_begin; j < p.tile_end; ++j, ++i) {
          const int st = i % C::NS;
          if (!mbar_wait(bar(b_empty + st), ((i / C::NS) & 1) ^ 1, abort_flag)) { ok = false; break; }
#ifdef FBK_TEST_HOOKS
          if (is_k && blockIdx.x == 0 && i == g_test_withhold_stage) continue;  // a tile that never lands
#endif
          const int n = tile_keys(p, j), nrows = tile_rows(n, boxh);
          const uint32_t bytes = (uint32_t)nrows * 128u * (D / 64);
          if (is_k || nrows == n) {
            mbar_expect_tx(bar(b_full + st), bytes);
            load_kv_tile<D>(g, map, map8, ring + st * C::KV_BYTES, p, j, n, boxh, bar(b_full + st), pol);
          } else {
            // a partial V tile (once per unit): its loads land on a barrier of
            // their own, the up to 7 rows past the unit's last key are zeroed,
            // and only then is the stage marked full for O += P~ V
            mbar_expect_tx(bar(C::B_VTAIL), bytes);
            load_kv_tile<D>(g, map, map8, ring + st * C::KV_BYTES, p, j, n, boxh, bar(C::B_VTAIL), pol);
            if (!mbar_wait(bar(C::B_VTAIL), ntail & 1, abort_flag)) {
              mbar_wait_drain(bar(C::B_VTAIL), ntail & 1);  // no TMA write may be in flight when the CTA leaves
              ok = false;
              break;
            }
            ++ntail;
            uint8_t *stage = smem + C::V_OFF + st * C::KV_BYTES;
            for (int rr = n; rr < nrows; ++rr)
#pragma unroll
              for (int cb = 0; cb < D / 64; ++cb)
#pragma unroll
                for (int c = 0; c < 8; ++c)
                  *reinterpret_cast<uint4 *>(stage + cb * (KV_TILE * 128) + rr * 128 + c * 16) = make_uint4(0, 0, 0, 0);
            fence_proxy_async();
            mbar_arrive(bar(b_full + st));
          }
        }
      }
      // no TMA write may be in flight when the CTA leaves
      for (int n = max(0, i - C::NS); n < i; ++n) mbar_wait_drain(bar(b_full + n % C::NS), (n / C::NS) & 1);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- S = Q K^T issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, KV_TILE, false);
      const uint64_t qpol = policy_evict_last();
      PieceWalker walk;
      walk.init(g, s_len, s_scan, blockIdx.x, T, shares);
      Piece p, pn;
      bool have = walk.next(g, p);
      bool have_next = have && walk.next(g, pn);
      int i = 0, pi = 0;
      bool ok = true;
      // rotated query rows of piece `pc` (M-tile order) by TMA into Q buffer qb
      auto load_q = [&](const Piece &pc, int qb) {
        mbar_expect_tx(bar(C::B_QLOAD + qb), MT * C::Q_BYTES);
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
          for (int cb = 0; cb < D / 64; ++cb)
            tma_load_2d(sb + C::Q_OFF + (qb * MT + mt) * C::Q_BYTES + cb * 16384, &tmq, cb * 64,
                        (pc.u * MT + mt) * 128, bar(C::B_QLOAD + qb), qpol);
      };
      // the previous piece's last S products (the last readers of its Q buffer) have completed
      auto prev_s_done = [&]() {
        bool good = true;
        for (int mt = 0; mt < MT && good; ++mt)
          good = mbar_wait(bar(C::B_SFULL + 2 * mt + ((i - 1) & 1)), ((i - 1) >> 1) & 1, abort_flag);
        return good;
      };
      if (have) load_q(p, 0);
      while (ok && have) {
        const int qb = C::QB == 2 ? (pi & 1) : 0;
        const uint32_t qpar = C::QB == 2 ? ((pi >> 1) & 1) : (pi & 1);
        if (!mbar_wait(bar(C::B_QLOAD + qb), qpar, abort_flag)) {
          mbar_wait_drain(bar(C::B_QLOAD + qb), qpar);  // no TMA write may be in flight when the CTA leaves
          ok = false;
          break;
        }
        fence_after_sync();
        if (C::QB == 2 && have_next) {  // prefetch the next piece's rows into the other buffer
          if (pi > 0 && !prev_s_done()) { ok = false; break; }
          load_q(pn, qb ^ 1);
        }
        const uint32_t q_base = sb + C::Q_OFF + qb * MT * C::Q_BYTES;
        for (int j = p.tile_begin; j < p.tile_end && ok; ++j, ++i) {
          const int st = i % C::NS, buf = i & 1;
          if (!mbar_wait(bar(C::B_KFULL + st), (i / C::NS) & 1, abort_flag)) { ok = false; break; }
          fence_after_sync();
          for (int mt = 0; mt < MT && ok; ++mt) {
            if (!mbar_wait(bar(C::B_SEMPTY + 2 * mt + buf), ((i >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
            fence_after_sync();
            const uint32_t d_tmem = tmem + C::TMEM_S + (2 * mt + buf) * KV_TILE;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const int cb = kk >> 2, ko = (kk & 3) * 32;
              const uint64_t a = sdesc_sw128(q_base + mt * C::Q_BYTES + cb * 128 * 128 + ko, 16, 1024);
              const uint64_t b = sdesc_sw128(sb + C::K_OFF + st * C::KV_BYTES + cb * KV_TILE * 128 + ko, 16, 1024);
              mma_bf16(d_tmem, a, b, IDESC_S, kk > 0 ? 1u : 0u);
            }
            mma_commit(bar(C::B_SFULL + 2 * mt + buf));
          }
          if (ok) mma_commit(bar(C::B_KEMPTY + st));
        }
        if (ok && C::QB == 1 && have_next) {  // one Q buffer: reload once this piece's S products are done
          if (!prev_s_done()) { ok = false; break; }
          load_q(pn, 0);
        }
        ++pi;
        p = pn;
        have = have_next;
        have_next = have && walk.next(g, pn);
      }
      // a prefetched load may still be in flight after an early exit
      if (!ok && C::QB == 2 && have)
        mbar_wait_drain(bar(C::B_QLOAD + (pi & 1)), (pi >> 1) & 1);
      mma_commit(bar(C::B_DRAIN));
      mbar_wait_drain(bar(C::B_DRAIN), 0);
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---------------------------------------------------------------- O += P~ V issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(128, D, true);
      PieceWalker walk;
      walk.init(g, s_len, s_scan, blockIdx.x, T, shares);
      Piece p;
      int i = 0, pi = 0;
      bool ok = true;
      while (ok && walk.next(g, p)) {
        for (int j = p.tile_begin; j < p.tile_end && ok; ++j, ++i) {
          const bool first = j == p.tile_begin;  // the piece's first tile overwrites O
          const int st = i % C::NS;
          if (!mbar_wait(bar(C::B_VFULL + st), (i / C::NS) & 1, abort_flag)) { ok = false; break; }
          if (first && pi > 0)  // the previous piece's epilogue has read O
            for (int mt = 0; mt < MT && ok; ++mt) ok = mbar_wait(bar(C::B_OFREE + mt), (pi - 1) & 1, abort_flag);
          for (int mt = 0; mt < MT && ok; ++mt) {
            if (!mbar_wait(bar(C::B_PFULL + 2 * mt + (i & 1)), (i >> 1) & 1, abort_flag)) { ok = false; break; }
            fence_after_sync();
            const uint32_t d_tmem = tmem + C::TMEM_O + mt * D;
            const uint32_t p_tmem = tmem + C::TMEM_S + (2 * mt + (i & 1)) * KV_TILE;
#pragma unroll
            for (int kk = 0; kk < KV_TILE / 16; ++kk) {
              const uint64_t b = sdesc_sw128(sb + C::V_OFF + st * C::KV_BYTES + kk * 2048, KV_TILE * 128, 1024);
              mma_bf16_ts(d_tmem, p_tmem + kk * 8, b, IDESC_PV, (first && kk == 0) ? 0u : 1u);
            }
            mma_commit(bar(C::B_ODONE + mt));
            mma_commit(bar(C::B_SEMPTY + 2 * mt + (i & 1)));  // S / P~ buffer reusable
          }
          if (ok) mma_commit(bar(C::B_VEMPTY + st));
        }
        ++pi;
      }
      mma_commit(bar(C::B_DRAIN + 1));
      mbar_wait_drain(bar(C::B_DRAIN + 1), 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- softmax
    const int mt = (warp - 4) >> 2, wq = warp & 3;
    const int row = wq * 32 + lane;                 // row inside the M-tile = TMEM lane
    const int r = mt * 128 + row;                   // query row inside the unit
    const bool wact = mt * 128 + wq * 32 < g.rows;  // warp holds at least one real row
    const uint32_t tl = (uint32_t)(wq * 32) << 16;
    const float sl2 = g.tau * 1.4426950408889634f;  // scores in log2 units
    // waits are made warp-uniform so that warp-collective TMEM accesses never diverge
    auto wwait = [&](uint32_t b, uint32_t ph) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(b, ph, abort_flag));
    };
    Piece& p = sm_piece;
    int i = 0;
    bool ok = true;
    while (ok && sm_more) {

      float m_ref = -CUDART_INF_F, m_true = -CUDART_INF_F, lsum = 0.f;
      const int n = p.tile_end - p.tile_begin;
      for (int jj = 0; jj < n; ++jj, ++i) {
        const int buf = i & 1;
        if (!wwait(bar(C::B_SFULL + 2 * mt + buf), (i >> 1) & 1)) { ok = false; break; }
        fence_after_sync();
        if (wact) {
          const uint32_t ts = tmem + tl + C::TMEM_S + (2 * mt + buf) * KV_TILE;
          uint32_t sr[64];
          tmem_ld32(ts, *reinterpret_cast<uint32_t(*)[32]>(sr));
          tmem_ld32(ts + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
          tmem_wait_ld();
          const int j = p.tile_begin + jj;
          const int nval = p.L - j * KV_TILE;
          if (nval < KV_TILE) {  // the unit's partial last tile (warp-uniform)
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c >= nval) sr[c] = __float_as_uint(-CUDART_INF_F);
          }
          // tile max of the raw scores (tau > 0): 8 independent chains of
          // three-input maxima, then a tree
          auto sv = [&](int c) { return __uint_as_float(sr[c]); };
          float mx[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = fmax3(sv(k), sv(k + 8), sv(k + 16));
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], sv(k + 24), sv(k + 32));
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], sv(k + 40), sv(k + 48));
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = fmaxf(mx[k], sv(k + 56));
          const float tmax = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(fmax3(mx[3], mx[4], mx[5]), mx[6], mx[7])) * sl2;
          m_true = fmaxf(m_true, tmax);
          const bool need = jj > 0 && tmax > m_ref + 8.f;
          if (jj == 0) m_ref = tmax;
          if (__any_sync(0xffffffffu, need)) {
            // rescale this row's O~ (and l) to the new reference max, once every
            // PV product issued so far has landed
            if (!wwait(bar(C::B_ODONE + mt), (i - 1) & 1)) ok = false;
            fence_after_sync();
            const float f = need ? exp2f(m_ref - tmax) : 1.f;
            if (ok) {
#pragma unroll 1
              for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                const uint32_t ta = tmem + tl + C::TMEM_O + mt * D + cc * 32;
                tmem_ld32(ta, o);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                tmem_st32(ta, o);
              }
              tmem_wait_st();
            }
            if (need) {
              lsum *= f;
              m_ref = tmax;
            }
          }
          if (ok) {
            // P~ = 2^(s*tau*log2(e) - m_ref) (one FFMA and one exp2 per element),
            // packed to bf16 pairs in place (pair c overwrites sr[c] after sr[2c],
            // sr[2c+1] are read) and stored over the first 32 columns of this
            // S buffer, where the PV issuer reads it as the A operand
            // (paired FP32 instructions for the scale-and-shift and the sums)
            const float2 sc2 = make_float2(sl2, sl2), ng2 = make_float2(-m_ref, -m_ref);
            float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
            for (int c = 0; c < 32; ++c) {
              const float2 x = ffma2(make_float2(sv(2 * c), sv(2 * c + 1)), sc2, ng2);
              const float2 pp = make_float2(ex2(x.x), ex2(x.y));
              sr[c] = pack_bf16(pp.x, pp.y);
              acc[c & 1] = fadd2(acc[c & 1], pp);
            }
            lsum += (acc[0].x + acc[0].y) + (acc[1].x + acc[1].y);
            tmem_st32(ts, *reinterpret_cast<uint32_t(*)[32]>(sr));
            tmem_wait_st();
          }
        }
        if (!ok) break;
        // Track every phase of O_DONE in order: a parity wait is only exact when
        // the barrier is at most one phase away, so each tile waits for the
        // previous tile's PV here (normally long done), which keeps the rescale
        // and epilogue waits below unambiguous.
        if (i > 0 && !wwait(bar(C::B_ODONE + mt), (i - 1) & 1)) { ok = false; break; }
        fence_before_sync();
        mbar_arrive(bar(C::B_PFULL + 2 * mt + buf));
      }
      if (!ok) break;
      // epilogue: rebase to the true max and store this piece's state
      if (!wwait(bar(C::B_ODONE + mt), (i - 1) & 1)) { ok = false; break; }
      fence_after_sync();
      if (wact) {
        const float f = exp2f(m_ref - m_true);
        const long long srow = ((long long)blockIdx.x + p.u) * g.rows + r;
        float *dst = ws.o + srow * D;
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[32];
          tmem_ld32(tmem + tl + C::TMEM_O + mt * D + cc * 32, o);
          tmem_wait_ld();
          if (r < g.rows) {
#pragma unroll
            for (int e = 0; e < 32; e += 4)
              *reinterpret_cast<float4 *>(dst + cc * 32 + e) =
                  make_float4(__uint_as_float(o[e]) * f, __uint_as_float(o[e + 1]) * f,
                              __uint_as_float(o[e + 2]) * f, __uint_as_float(o[e + 3]) * f);
          }
        }
        if (r < g.rows) {
          ws.m[srow] = m_true * 0.6931471805599453f;  // back to natural-log units
          ws.l[srow] = lsum * f;
        }
      }
      fence_before_sync();
      mbar_arrive(bar(C::B_OFREE + mt));
      sm_more = sm_walk.next(g, p);
    }
  }

  // ------------------------------------------------------------------ teardown
  fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    fence_after_sync();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0 && *abort_flag) raise_flag(g, FBK_DEVERR_TIMEOUT);
}

// Rotated block queries for the prefix kernel, in its M-tile order: row
// (u * MT * 128 + r) of qrot holds query row r = hl * B + t of unit u =
// (b, kvh), i.e. head kvh * G + hl at position L_b + t, RoPE-rotated (rotate
// half, fp64-reduced angle, fast sine/cosine) and rounded to bf16; rows r >=
// G*B are zero. One thread per 8 rotation pairs (chunk c of each half of a row).
template <int D, int MT>
__global__ void __launch_bounds__(256) rope_q_kernel(Geometry g, const __nv_bfloat16 *__restrict__ q,
                                                    __nv_bfloat16 *__restrict__ qrot, const int *__restrict__ qpos,
                                                    PrefixGate gate) {
  constexpr int HALF = D / 2, KI = D / 16, ROWS = MT * 128;
  __shared__ double theta[HALF];
  for (int i = threadIdx.x; i < HALF; i += blockDim.x) theta[i] = freq_over_pi(i, D, g.log2_base);
  __syncthreads();
  pdl_wait();
  pdl_release();
  if (gate.gate) {  // the adaptive refresh: run only when asked, and record that it ran
    if (*gate.gate == 0) return;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
      *gate.mark = 1;
      *gate.last = gate.step;
    }
  }
  const long long n_items = (long long)g.batch * g.hkv * ROWS * KI;
  for (long long item = (long long)blockIdx.x * blockDim.x + threadIdx.x; item < n_items;
       item += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(item % KI);
    const long long rowi = item / KI;
    const int r = (int)(rowi % ROWS);
    const int u = (int)(rowi / ROWS), b = u / g.hkv, kvh = u % g.hkv;
    uint4 y1 = make_uint4(0, 0, 0, 0), y2 = make_uint4(0, 0, 0, 0);
    if (r < g.rows) {
      const int t = r % g.blk, h = kvh * g.group + r / g.blk;
      const int L = qpos ? qpos[b] : prefix_len(g, b);  // rotation base of the block's rows
      const uint4 *src = reinterpret_cast<const uint4 *>(q + (((long long)b * g.blk + t) * g.hq + h) * D);
      const uint4 a = src[c], bq = src[c + KI];
      const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {bq.x, bq.y, bq.z, bq.w};
      uint32_t o1[4], o2[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 c0 = rope_cs_fast(L + t, theta[8 * c + 2 * e]);
        const float2 c1 = rope_cs_fast(L + t, theta[8 * c + 2 * e + 1]);
        const float x1l = __uint_as_float(aw[e] << 16), x1h = __uint_as_float(aw[e] & 0xffff0000u);
        const float x2l = __uint_as_float(bw[e] << 16), x2h = __uint_as_float(bw[e] & 0xffff0000u);
        o1[e] = pack_bf16(x1l * c0.x - x2l * c0.y, x1h * c1.x - x2h * c1.y);
        o2[e] = pack_bf16(x2l * c0.x + x1l * c0.y, x2h * c1.x + x1h * c1.y);
      }
      y1 = make_uint4(o1[0], o1[1], o1[2], o1[3]);
      y2 = make_uint4(o2[0], o2[1], o2[2], o2[3]);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(qrot + rowi * D);
    dst[c] = y1;
    dst[c + KI] = y2;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;  // driver entry point, looked up once
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D map over the cache viewed as [rows, d] bf16, boxes of 64 columns x boxh rows, 128B swizzle.
bool make_map(CUtensorMap *m, const void *base, long long rows, int d, int boxh) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)boxh};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int MT>
cudaError_t launch_cfg(const Geometry &g, const __nv_bfloat16 *q, const int *qpos, const Workspace &ws, int shares,
                       cudaStream_t st, const PrefixGate *pg) {
  const PrefixGate gate = pg ? *pg : PrefixGate{nullptr, nullptr, nullptr, 0};
  using C = Cfg<D, MT>;
  const long long rows = g.paged ? g.num_pages * g.hkv * g.page_size : (long long)g.batch * g.hkv * g.cap;
  const int boxh = g.paged ? min(g.page_size, KV_TILE) : KV_TILE;
  CUtensorMap mk, mv, mk8, mv8;  // whole tiles; 8-row boxes for a unit's partial last tile
  if (!make_map(&mk, g.kc, rows, D, boxh) || !make_map(&mv, g.vc, rows, D, boxh) ||
      !make_map(&mk8, g.kc, rows, D, 8) || !make_map(&mv8, g.vc, rows, D, 8))
    return cudaErrorInvalidValue;
  // the rotated query rows: [units * MT * 128, D], boxes of 64 columns x 128 rows
  CUtensorMap mq;
  const long long qrows = (long long)g.batch * g.hkv * MT * 128;
  if (qrows > 0x7fffffffll || !make_map(&mq, ws.qrot, qrows, D, 128)) return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long items = qrows * (D / 16);
  const int rq_ctas = (int)std::min<long long>((items + 255) / 256, 8ll * sms);
  cudaError_t e = launch_pdl(rope_q_kernel<D, MT>, dim3(rq_ctas), dim3(256), 0, st, g, q, ws.qrot, qpos, gate);
  if (e != cudaSuccess) return e;
  auto kern = prefix_tc_kernel<D, MT>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(shares), dim3(C::THREADS), C::SMEM, st, g, q, ws, shares, mk, mv, mk8, mv8, boxh,
                    mq, gate.gate);
}

}  // namespace

cudaError_t launch_prefix_tc_at(const Geometry &g, const __nv_bfloat16 *q, const int *qpos, const Workspace &ws,
                                int shares, cudaStream_t st, const PrefixGate *gate) {
  const bool two = g.rows > 128;
  if (g.d == 128)
    return two ? launch_cfg<128, 2>(g, q, qpos, ws, shares, st, gate)
               : launch_cfg<128, 1>(g, q, qpos, ws, shares, st, gate);
  return two ? launch_cfg<64, 2>(g, q, qpos, ws, shares, st, gate)
             : launch_cfg<64, 1>(g, q, qpos, ws, shares, st, gate);
}

namespace {
__global__ void adaptive_init_kernel(int *flags, int *last_refresh, float *drift, int *refreshed, int n, int steps) {
  pdl_wait();
  pdl_release();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < steps * n; i += gridDim.x * blockDim.x) {
    drift[i] = 0.f;
    refreshed[i] = 0;
    if (i < n) {
      flags[i] = 1;      // step 0 computes every layer's state
      flags[n + i] = 0;  // no request for step 1 yet
      last_refresh[i] = 0;
    }
  }
}
}  // namespace

cudaError_t launch_adaptive_init(int *flags, int *last_refresh, float *drift, int *refreshed, int n_layers,
                                 int steps, cudaStream_t st) {
  const long long items = (long long)n_layers * steps;
  const int ctas = (int)std::min<long long>((items + 255) / 256, 1024);
  return launch_pdl(adaptive_init_kernel, dim3(ctas), dim3(256), 0, st, flags, last_refresh, drift, refreshed,
                    n_layers, steps);
}

cudaError_t launch_prefix_tc(const Geometry &g, const __nv_bfloat16 *q, const Workspace &ws,
                             int shares, cudaStream_t st) {
  return launch_prefix_tc_at(g, q, nullptr, ws, shares, st);
}

}  // namespace fbk

#ifdef FBK_TEST_HOOKS
// Test build only: see include/fbk_test_hooks.h.
extern "C" int fbk_test_set_wait_fault(long long wait_limit_clocks, int withhold_stage) {
  cudaError_t e = cudaMemcpyToSymbol(fbk::tc::g_test_wait_limit, &wait_limit_clocks, sizeof(long long));
  if (e == cudaSuccess) e = cudaMemcpyToSymbol(fbk::tc::g_test_withhold_stage, &withhold_stage, sizeof(int));
  return (int)e;
}
#endif
