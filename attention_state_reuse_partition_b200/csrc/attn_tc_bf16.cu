// Partition attention on the sm_100a tensor cores (bf16 in, fp32 state out).
//
// Computes attention states of DiTango (arXiv 2607.15650; review page,
// "What carries the argument"): for the query rows of a CTA and a list of KV
// token ranges it runs the blockwise online softmax over 128-key tiles and
// emits (OUT, LSE) per accumulation group -- the composite of every code-1
// partition (the composition of Eq. 1-2 done on chip) and one state per
// code-2 partition.
//
// One CTA per (256 query rows, head): two 128-row query tiles Q0, Q1 share
// every K/V tile.  Warp roles:
//   warp 0      TMA producer: Q0 and Q1 once, then K and V tiles (2-stage rings)
//   warp 1      TMEM allocator and UMMA issuer (one elected lane)
//   warps 4-7   softmax of Q0, warps 8-11 softmax of Q1: thread r owns row r of
//               its tile (TMEM lane r)
// TMEM columns: S_t = Q_t K^T at [128 t, 128 t + 128) (fp32), overwritten in
// place by P_t (bf16 pairs, 64 columns) once the softmax has read it; O_t at
// [256 + D t, 256 + D t + D).  S = Q K^T is an SS MMA (both operands in
// 128-byte-swizzled shared memory), O += P V a TS MMA (P from TMEM, V from
// shared memory, MN-major).  Per KV tile j the issuer sends, for t = 0, 1,
// one uninterrupted burst PV_t,j + QK_t,j+1 (16 MMAs, 1024 cycles at d = 128,
// all waits done before the burst, because the issuing thread runs only a few
// MMAs ahead of the tensor core), so the tensor core works on one tile while
// the other tile's softmax runs.  A commit after QK_t completes only when
// every earlier MMA has, so when the softmax of tile t sees S_t its previous
// PV has finished: O_t may be rescaled and P_t written without a further
// wait.  O is rescaled only when a row maximum grows by more than 2^8; OUT and
// the row sum share the same reference maximum, so the result is unchanged.
// At a group end each softmax warp moves its 32 rows of O through a small
// shared-memory block, 32 columns and 16 rows at a time, so that the global
// stores write whole 128-byte row segments; O_t is released to the next group
// as soon as it has been read.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "as_device.cuh"

namespace asp {
namespace {

constexpr int NQ = 2;          // query tiles per CTA
constexpr int BM = 128;        // rows per query tile
constexpr int BN = 128;        // keys per KV tile
constexpr int NST = 2;         // K and V ring depth
constexpr int REGION = 128 * 128;  // one 64-column bf16 chunk of a 128-row tile (bytes)
constexpr int NTHREADS = 128 * (1 + NQ);
constexpr uint32_t TMEM_COLS = 512;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 domain
#ifndef ASP_POLY_PAIR_EVERY
#define ASP_POLY_PAIR_EVERY 0
#endif
constexpr int POLY_PAIR_EVERY = ASP_POLY_PAIR_EVERY;  // every n-th pair of exponentials on the FMA pipe
constexpr int POLY_PERIOD = POLY_PAIR_EVERY > 0 ? POLY_PAIR_EVERY : 1;
// registers: launched at LAUNCH_REGS per thread; the control warpgroup (TMA,
// MMA, two idle warps) gives up registers to the softmax warpgroups.
// 128 * CTRL_REGS + 128 * NQ * SOFTMAX_REGS == NTHREADS * LAUNCH_REGS
constexpr int LAUNCH_REGS = 168;
constexpr int CTRL_REGS = 88;
constexpr int SOFTMAX_REGS = 208;
static_assert(128 * CTRL_REGS + 128 * NQ * SOFTMAX_REGS == NTHREADS * LAUNCH_REGS, "register split");

template <int D>
struct Layout {
  static constexpr int NREG = D / 64;                 // 64-column chunks per row
  static constexpr int TILE_BYTES = 128 * D * 2;      // one Q, K or V tile
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + NQ * TILE_BYTES;
  static constexpr int V_OFF = K_OFF + NST * TILE_BYTES;
  static constexpr int CTRL_OFF = V_OFF + NST * TILE_BYTES;
  static constexpr uint32_t O_COL = 256;              // O_t at O_COL + t * D
};

struct Ctrl {
  uint64_t q_full;
  // load unit u carries K_u and V_{u-1} (K stage u % 2, V stage (u-1) % 2):
  // exactly what the burst of tile u-1 needs
  uint64_t kv_full[NST], kv_empty[NST];
  uint64_t s_full[NQ], p_full[NQ], o_ready[NQ], o_free[NQ];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int n_tiles;
  KvSchedule sched;
};

// Output staging: each softmax warp moves its 32 rows, 32 columns at a
// time, through a 16 x 32-float block, one half-warp's 16 rows per pass (row
// stride STAGE_LD floats: the float4 accesses of 8 consecutive rows, or of 8
// lanes along one row, cover all 32 banks), so that each global store
// instruction writes four whole 128-byte row segments instead of 32
// scattered 16-byte pieces.  Against 64-byte segments (16 columns at a
// time) this is 5% faster when a CTA emits one state per KV partition.
constexpr int STAGE_LD = 36;
constexpr int STAGE_FLOATS = 16 * STAGE_LD;  // per softmax warp
constexpr int CTRL_BYTES = (static_cast<int>(sizeof(Ctrl)) + 15) & ~15;

template <int D>
constexpr int smem_bytes() {
  // at least 116 KB so that only one CTA (and one 512-column TMEM allocation)
  // fits on an SM
  constexpr int need = Layout<D>::CTRL_OFF + CTRL_BYTES + 4 * NQ * STAGE_FLOATS * 4 + 1024;
  return need > 116 * 1024 ? need : 116 * 1024;
}

// Walks the tiles of a schedule in order, the same way in every role.  The
// bounds of the current range and group are cached in registers; shared
// memory is read only when the walk enters a new range.
struct TileWalk {
  const KvSchedule* s;
  int g, r, t;
  int r_lo, r_hi, g_first_r, g_last_r, n_groups;
  __device__ void load_range() {
    r_lo = s->range_lo[r];
    r_hi = s->range_hi[r];
  }
  __device__ void load_group() {
    g_first_r = s->group_first[g];
    g_last_r = g_first_r + s->group_count[g] - 1;
  }
  __device__ void start(const KvSchedule* sched) {
    s = sched;
    n_groups = s->n_groups;
    g = 0;
    if (n_groups > 0) {
      load_group();
      r = g_first_r;
      load_range();
      t = r_lo;
    }
  }
  __device__ bool valid() const { return g < n_groups; }
  __device__ bool first() const { return r == g_first_r && t == r_lo; }
  __device__ bool last() const { return r == g_last_r && t + BN >= r_hi; }
  __device__ int nvalid() const { return min(BN, r_hi - t); }
  __device__ void next() {
    t += BN;
    if (t < r_hi) return;
    ++r;
    if (r <= g_last_r) {
      load_range();
      t = r_lo;
      return;
    }
    ++g;
    if (g < n_groups) {
      load_group();
      r = g_first_r;
      load_range();
      t = r_lo;
    }
  }
};

__device__ int count_tiles(const KvSchedule& s) {
  int n = 0;
  for (int r = 0; r < s.n_ranges; ++r) n += (s.range_hi[r] - s.range_lo[r] + BN - 1) / BN;
  return n;
}

// a wait for work already in flight (copies, MMAs) before the CTA exits;
// it ignores the abort flag, and is bounded in time like every other wait
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint32_t t0 = global_ns32();
  while (global_ns32() - t0 <= KERNEL_WAIT_NS)
    if (mbar_try_wait(bar, parity)) return true;
  raise_dev_error(AS_DEVERR_TIMEOUT);
  return false;
}

// all lanes of a warp wait; the result is the same in every lane
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const bool ok = mbar_wait(bar, parity, abort_flag);
  return __all_sync(0xffffffffu, ok);
}

template <int D>
__global__ void __launch_bounds__(NTHREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ AttnLaunch L) {
  using Lay = Layout<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl& c = *reinterpret_cast<Ctrl*>(smem + Lay::CTRL_OFF);
  volatile int* abort_flag = &c.abort;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tiles_per_block = (L.block_rows + NQ * BM - 1) / (NQ * BM);
  const int blk = blockIdx.x / tiles_per_block;
  const int qt = blockIdx.x % tiles_per_block;
  const int bh = blockIdx.y;
  const int block_lo = L.block_row0 + blk * L.block_rows;
  const int q_lo = block_lo + qt * NQ * BM;
  const int q_hi = min(block_lo + L.block_rows, L.S);  // rows at or beyond q_hi are not written

  if (threadIdx.x == 0) {
    mbar_init(&c.q_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&c.kv_full[s], 1);
      mbar_init(&c.kv_empty[s], 1);
    }
    for (int t = 0; t < NQ; ++t) {
      mbar_init(&c.s_full[t], 1);
      mbar_init(&c.p_full[t], 128);
      mbar_init(&c.o_ready[t], 1);
      mbar_init(&c.o_free[t], 128);
    }
    mbar_init(&c.drain, 1);
    c.abort = 0;
    build_schedule(L.code + blk * L.P, L.dest_of, L.kv_row0, L.P, L.n, c.sched);
    c.n_tiles = count_tiles(c.sched);
    mbar_fence_init();
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, TMEM_COLS);
    tmem_relinquish();
    tc_fence_before();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  const int n_tiles = c.n_tiles;

  if (warp < 4) {
  regs_dealloc<CTRL_REGS>();
  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&c.q_full, NQ * Lay::TILE_BYTES);
      for (int t = 0; t < NQ; ++t)
        for (int rg = 0; rg < Lay::NREG; ++rg)
          tma_load_3d(smem + Lay::Q_OFF + t * Lay::TILE_BYTES + rg * REGION, &tm_q, &c.q_full, rg * 64,
                      q_lo + t * BM, bh);
      // units 0..n_tiles: K_u (u < n_tiles) and V_{u-1} (u >= 1)
      TileWalk w;
      w.start(&c.sched);
      int prev_t = 0;  // KV row of tile u-1
      int u = 0;
      for (; u <= n_tiles; ++u) {
        const int slot = u % NST;
        if (!mbar_wait(&c.kv_empty[slot], ((u / NST) & 1) ^ 1, abort_flag)) break;
        const bool has_k = u < n_tiles, has_v = u >= 1;
        mbar_arrive_expect_tx(&c.kv_full[slot], (has_k ? Lay::TILE_BYTES : 0) + (has_v ? Lay::TILE_BYTES : 0));
        if (has_v) {
          uint8_t* sV = smem + Lay::V_OFF + ((u - 1) % NST) * Lay::TILE_BYTES;
          for (int rg = 0; rg < Lay::NREG; ++rg)
            tma_load_3d(sV + rg * REGION, &tm_v, &c.kv_full[slot], rg * 64, prev_t, bh);
        }
        if (has_k) {
          uint8_t* sK = smem + Lay::K_OFF + (u % NST) * Lay::TILE_BYTES;
          for (int rg = 0; rg < Lay::NREG; ++rg)
            tma_load_3d(sK + rg * REGION, &tm_k, &c.kv_full[slot], rg * 64, w.t, bh);
          prev_t = w.t;
          w.next();
        }
      }
      // before the CTA may exit, every issued load must have landed
      if (*abort_flag) {
        drain_wait(&c.q_full, 0);
        for (int uu = max(0, u - NST); uu < u; ++uu) drain_wait(&c.kv_full[uu % NST], (uu / NST) & 1);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, false, true);
      // descriptors of stage 0; stages, query tiles and k-steps only move the
      // start address field (16-byte units), which stays below 2^14 for 227 KB
      const uint64_t dq0 = smem_desc_sw128(smem_u32(smem + Lay::Q_OFF), 16, 1024);
      const uint64_t dk0 = smem_desc_sw128(smem_u32(smem + Lay::K_OFF), 16, 1024);
      const uint64_t dv0 = smem_desc_sw128(smem_u32(smem + Lay::V_OFF), REGION, 1024);
      constexpr uint32_t TILE16 = Lay::TILE_BYTES >> 4;
      auto issue_qk = [&](int t, int j) {
        const uint64_t dq = dq0 + t * TILE16;
        const uint64_t dk = dk0 + (j % NST) * TILE16;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off16 = ((kk >> 2) * REGION + (kk & 3) * 32) >> 4;
          umma_bf16_ss(tmem + t * BN, dq + off16, dk + off16, IDESC_QK, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, int j, bool first) {
        const uint64_t dv = dv0 + (j % NST) * TILE16;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          umma_bf16_ts(tmem + Lay::O_COL + t * D, tmem + t * BN + kk * 8, dv + ((kk * 16 * 128) >> 4),
                       IDESC_PV, (kk > 0 || !first) ? 1u : 0u);
      };
      // unit 0 (K_0) for the first QKs, unit 1 (V_0, K_1) for the first burst
      bool ok = mbar_wait(&c.q_full, 0, abort_flag) && mbar_wait(&c.kv_full[0], 0, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < NQ; ++t) {
          issue_qk(t, 0);
          umma_commit(&c.s_full[t]);
        }
        umma_commit(&c.kv_empty[0]);
        ok = mbar_wait(&c.kv_full[1 % NST], (1 / NST) & 1, abort_flag);
        TileWalk w;
        int j = 0, group = 0;
        for (w.start(&c.sched); w.valid() && ok; w.next(), ++j) {
          const bool first = w.first(), last = w.last();
          if (first && j > 0) ++group;
          const bool has_next = j + 1 < n_tiles;
          for (int t = 0; t < NQ; ++t) {
            // the burst's data (unit j+1) was waited for earlier; here only
            // the softmax handshake, then the 16 MMAs back to back
            if (first && group > 0 && !mbar_wait(&c.o_free[t], (group - 1) & 1, abort_flag)) ok = false;
            if (ok && !mbar_wait(&c.p_full[t], j & 1, abort_flag)) ok = false;
            if (!ok) break;
            tc_fence_after();
            issue_pv(t, j, first);
            if (has_next) issue_qk(t, j + 1);
            if (last) umma_commit(&c.o_ready[t]);
            if (has_next) umma_commit(&c.s_full[t]);
            if (t == NQ - 1) {
              umma_commit(&c.kv_empty[(j + 1) % NST]);  // unit j+1: V_j and K_{j+1} consumed
            } else if (has_next) {
              // data of the next burst, waited for while the other tile's softmax runs
              const int u = j + 2;
              if (!mbar_wait(&c.kv_full[u % NST], (u / NST) & 1, abort_flag)) {
                ok = false;
                break;
              }
            }
          }
        }
      }
      // all issued MMAs must be complete before TMEM is released
      umma_commit(&c.drain);
      drain_wait(&c.drain, 0);
    }
  }
  } else {
    regs_alloc<SOFTMAX_REGS>();
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;          // query tile of this warpgroup
    const int quarter = warp & 3;           // TMEM lane quarter of this warp
    const int row = quarter * 32 + lane;
    const int s_row = q_lo + t * BM + row;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t s_col = t * BN;
    const uint32_t o_col = Lay::O_COL + t * D;
    const float sl2 = L.scale * 1.4426950408889634f;
    float m = -INFINITY, l = 0.f;
    int group = 0;
    TileWalk w;
    int j = 0;
    for (w.start(&c.sched); w.valid(); w.next(), ++j) {
      const bool first = w.first();
      const bool last = w.last();
      const int nv = w.nvalid();
      if (first && j > 0) ++group;
      if (!warp_wait(&c.s_full[t], j & 1, abort_flag)) break;
      tc_fence_after();
      float s[BN];
      {
        uint32_t r[128];
        tmem_ld128(t_lane + s_col, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 128; ++e) s[e] = __uint_as_float(r[e]);
      }
      if (nv < BN) {
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (e >= nv) s[e] = -INFINITY;
      }
      // row maximum: four independent chains of 3-input max
      float mx4[4] = {s[0], s[1], s[2], s[3]};
#pragma unroll
      for (int e = 4; e < BN; e += 8) {
        mx4[0] = max3(mx4[0], s[e + 0], s[e + 1]);
        mx4[1] = max3(mx4[1], s[e + 2], s[e + 3]);
        mx4[2] = max3(mx4[2], s[e + 4], s[e + 5]);
        if (e + 7 < BN) mx4[3] = max3(mx4[3], s[e + 6], s[e + 7]);
      }
      const float m_tile = max3(mx4[0], mx4[1], fmaxf(mx4[2], mx4[3])) * sl2;
      float m_use = m, alpha = 1.f;
      bool rescale = false;
      if (first) {
        m_use = m_tile;
      } else if (m_tile > m + RESCALE_THRESHOLD) {
        m_use = m_tile;
        alpha = ex2_approx(m - m_use);
        rescale = true;
      }
      // p = 2^(s * scale * log2 e - m): scale-subtract and row sum on packed
      // pairs; one pair in POLY_PAIR_EVERY evaluated on the FMA pipe
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      const uint64_t negm2 = f2_pack(-m_use, -m_use);
      uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
      uint32_t pk[BN / 2];  // P as bf16 pairs, written to TMEM over S
#pragma unroll
      for (int i = 0; i < BN / 2; ++i) {
        const uint64_t x2 = f2_fma(f2_pack(s[2 * i], s[2 * i + 1]), sl2x2, negm2);
        float x0, x1;
        f2_unpack(x2, x0, x1);
        uint64_t p2;
        if (POLY_PAIR_EVERY > 0 && i % POLY_PERIOD == POLY_PERIOD - 1)
          p2 = exp2_poly2(x0, x1);
        else
          p2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
        sum2[i & 3] = f2_add(sum2[i & 3], p2);
        float p0, p1;
        f2_unpack(p2, p0, p1);
        pk[i] = pack_bf16x2(p0, p1);
      }
      // the previous PV of this tile has completed (see the header), so P may
      // be written over S and O rescaled now; P goes first, which frees its
      // registers for the rescale
      tmem_st64(t_lane + s_col, pk);
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int ch = 0; ch < D / 16; ++ch) {
          uint32_t r[16];
          tmem_ld16(t_lane + o_col + ch * 16, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st16(t_lane + o_col + ch * 16, r);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&c.p_full[t]);
      float rs;
      {
        const uint64_t a = f2_add(f2_add(sum2[0], sum2[1]), f2_add(sum2[2], sum2[3]));
        float lo, hi;
        f2_unpack(a, lo, hi);
        rs = lo + hi;
      }
      l = first ? rs : fmaf(l, alpha, rs);
      m = m_use;
      if (last) {
        if (!warp_wait(&c.o_ready[t], group & 1, abort_flag)) break;
        tc_fence_after();
        // the warp's 32 rows are consecutive in the destination: s_row0 + rr
        const int s_row0 = s_row - lane;
        const int dest = c.sched.group_dest[group];
        // checked build: the destination plane and the warp's rows lie inside
        // the destination (rows at or beyond q_hi are never written)
        const bool in_dest = ASP_CHECK(dest < L.dst_planes &&
                                       s_row0 >= (dest < 0 ? L.out_row0 : L.dst_row0) &&
                                       min(s_row0 + 32, q_hi) <= (dest < 0 ? L.out_row0 + L.out_rows
                                                                           : L.dst_row0 + L.dst_rows));
        float* orow0;  // row s_row0 (fp32 destinations)
        __nv_bfloat16* brow0 = nullptr;  // row s_row0 (bf16 cache planes)
        float* lrow;
        if (dest < 0) {
          const long long r_idx = static_cast<long long>(bh) * L.out_rows + (s_row0 - L.out_row0);
          orow0 = L.out + r_idx * D;
          lrow = L.lse + r_idx + lane;
        } else {
          const long long r_idx = static_cast<long long>(bh) * L.dst_rows + (s_row0 - L.dst_row0);
          const long long e_idx = dest * L.dst_plane_out + r_idx * D;
          orow0 = static_cast<float*>(L.dst_out) + e_idx;
          if (L.dst_bf16) brow0 = static_cast<__nv_bfloat16*>(L.dst_out) + e_idx;
          lrow = L.dst_lse + dest * L.dst_plane_lse + r_idx + lane;
        }
        const float inv_l = 1.0f / l;
        float* stage = reinterpret_cast<float*>(smem + Lay::CTRL_OFF + CTRL_BYTES) + (warp - 4) * STAGE_FLOATS;
        // read-back role of this lane: staged rows 4 i + lane / 8, columns 4 (lane % 8) .. + 3
        const int rb_row = lane >> 3, rb_col = (lane & 7) * 4;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(t_lane + o_col + ch * 32, r);
          tmem_wait_ld();
          if (ch == D / 32 - 1) {
            // O has been read: the next group may overwrite it
            tc_fence_before();
            mbar_arrive(&c.o_free[t]);
          }
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            if ((lane >> 4) == half) {
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                *reinterpret_cast<float4*>(stage + (lane & 15) * STAGE_LD + e) =
                    make_float4(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l,
                                __uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int rs = 4 * i + rb_row;     // row in the staging block
              const int rr = 16 * half + rs;     // row among the warp's 32
              const float4 v4 = *reinterpret_cast<const float4*>(stage + rs * STAGE_LD + rb_col);
              const long long off = static_cast<long long>(rr) * D + ch * 32 + rb_col;
              if (s_row0 + rr < q_hi && in_dest) {
                if (brow0)
                  *reinterpret_cast<uint2*>(brow0 + off) = make_uint2(pack_bf16x2(v4.x, v4.y), pack_bf16x2(v4.z, v4.w));
                else
                  *reinterpret_cast<float4*>(orow0 + off) = v4;
              }
            }
            __syncwarp();
          }
        }
        if (s_row < q_hi && in_dest) *lrow = (m + log2f(l)) * 0.6931471805599453f;
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [B*H, S, d] bf16, box = 64 columns x 128 rows x 1 head, 128-byte swizzle,
// rows beyond S read as zero
bool make_tmap(CUtensorMap* m, const void* base, int BH, int S, int d) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(S) * d * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
cudaError_t launch_d(const AttnLaunch& L, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  const int BH = L.B * L.H;
  if (!make_tmap(&tq, L.q, BH, L.S, D) || !make_tmap(&tk, L.k, BH, L.S_kv, D) || !make_tmap(&tv, L.v, BH, L.S_kv, D))
    return cudaErrorInvalidValue;
  constexpr int smem = smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // the in-kernel register split assumes exactly LAUNCH_REGS per thread at launch
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_tc_kernel<D>);
  if (e != cudaSuccess) return e;
  if (fa.numRegs != LAUNCH_REGS) return cudaErrorInvalidConfiguration;
  const int tiles_per_block = (L.block_rows + NQ * BM - 1) / (NQ * BM);
  dim3 grid(L.n_blocks * tiles_per_block, BH);
  attn_tc_kernel<D><<<grid, NTHREADS, smem, st>>>(tq, tk, tv, L);
  return cudaGetLastError();
}

// One thread waits, with the given limit, on a barrier that nothing completes.
__global__ void timeout_probe_kernel(unsigned int polls, unsigned int ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_bounded<true>(&bar, 0, &abort_flag, polls, ns);
}

__global__ void exp2_probe_kernel(const float* x, float* y, long long n, int mode) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
  {
    float lo = 0.f, hi = 0.f;
    if (mode == 0) f2_unpack(exp2_poly2(x[i], x[i]), lo, hi);
    y[i] = mode == 0 ? lo : ex2_approx(x[i]);
  }
}

}  // namespace

cudaError_t launch_exp2_probe(const float* x, float* y, long long n, int mode, cudaStream_t st) {
  const long long blocks = (n + 255) / 256;
  exp2_probe_kernel<<<static_cast<unsigned>(blocks < 4096 ? (blocks > 0 ? blocks : 1) : 4096), 256, 0, st>>>(
      x, y, n, mode);
  return cudaGetLastError();
}

cudaError_t launch_timeout_probe(unsigned int polls, unsigned int ns, cudaStream_t st) {
  timeout_probe_kernel<<<1, 32, 0, st>>>(polls, ns);
  return cudaGetLastError();
}

cudaError_t dev_error_attn_tc(unsigned int* bits) { return read_and_clear_local_dev_error(bits); }

#if ASP_DEBUG
__global__ void bounds_probe_kernel(float* buf, long long n) {
  const long long idx = n;  // one past the logical end
  if (ASP_CHECK(idx < n)) buf[idx] = 1.0f;
}
#endif

cudaError_t launch_bounds_probe(float* buf, long long n, cudaStream_t st) {
#if ASP_DEBUG
  bounds_probe_kernel<<<1, 1, 0, st>>>(buf, n);
  return cudaGetLastError();
#else
  (void)buf;
  (void)n;
  (void)st;
  return cudaErrorNotSupported;
#endif
}

cudaError_t launch_attn_tc_bf16(const AttnLaunch& L, cudaStream_t st) {
  if (L.d == 128) return launch_d<128>(L, st);
  if (L.d == 64) return launch_d<64>(L, st);
  return cudaErrorInvalidValue;
}

}  // namespace asp
