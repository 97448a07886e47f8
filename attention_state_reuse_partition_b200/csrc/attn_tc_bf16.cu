// Partition attention on the sm_100a tensor cores (bf16 in, fp32 state out).
//
// Computes attention states of DiTango (arXiv 2607.15650; review page,
// "What carries the argument"): for a 128-row query tile and a list of KV
// token ranges it runs the blockwise online softmax over 128-key tiles and
// emits (OUT, LSE) per accumulation group -- the composite of every code-1
// partition (the composition of Eq. 1-2 done on chip) and one state per
// code-2 partition.
//
// One CTA per (query tile, head).  Warp roles:
//   warp 0     TMA producer: Q once, then K and V tiles into 2-stage rings
//   warp 1     TMEM allocator and UMMA issuer (one elected lane)
//   warps 4-7  softmax: thread r owns query row r of the tile (TMEM lane r)
// TMEM: S double buffer in columns [0,128) and [128,256), O in [256,256+D).
// S = Q K^T and O += P V are tcgen05.mma kind::f16 (M=128, N=128 / D, K=16)
// with operands in 128-byte-swizzled shared memory; P goes through shared
// memory as bf16.  The issue order S_0, S_1, PV_0, S_2, PV_1, ... lets the
// tensor core compute S_{j+1} and PV_{j-1} while the softmax warps work on S_j.
// O is rescaled only when a row maximum grows by more than 2^8, which keeps
// the result exact (OUT and the row sum share the same reference maximum).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "as_device.cuh"

namespace asp {
namespace {

constexpr int BM = 128;       // query rows per tile
constexpr int BN = 128;       // keys per KV tile
constexpr int NST = 2;        // K and V ring depth
constexpr int REGION = 128 * 128;  // one 64-column bf16 chunk of a 128-row tile (bytes)
constexpr int NTHREADS = 256;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TMEM_O = 256;
constexpr float RESCALE_THRESHOLD = 8.0f;  // log2 domain

template <int D>
struct Layout {
  static constexpr int NREG = D / 64;                 // 64-column chunks per row
  static constexpr int TILE_BYTES = 128 * D * 2;      // Q, K or V tile
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE_BYTES;
  static constexpr int V_OFF = K_OFF + NST * TILE_BYTES;
  static constexpr int P_OFF = V_OFF + NST * TILE_BYTES;
  static constexpr int CTRL_OFF = P_OFF + BM * BN * 2;
};

struct Ctrl {
  uint64_t q_full;
  uint64_t k_full[NST], k_empty[NST];
  uint64_t v_full[NST], v_empty[NST];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full;
  uint64_t o_ready;
  uint64_t o_free;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  KvSchedule sched;
};

template <int D>
constexpr int smem_bytes() {
  return Layout<D>::CTRL_OFF + static_cast<int>(sizeof(Ctrl)) + 1024;
}

// Walks the tiles of a schedule in order, the same way in every role.
struct TileWalk {
  const KvSchedule* s;
  int g, r, t;
  __device__ void start(const KvSchedule* sched) {
    s = sched;
    g = 0;
    r = s->n_groups > 0 ? s->group_first[0] : 0;
    t = s->n_groups > 0 ? s->range_lo[r] : 0;
  }
  __device__ bool valid() const { return g < s->n_groups; }
  __device__ bool first() const {
    return r == s->group_first[g] && t == s->range_lo[r];
  }
  __device__ bool last() const {
    return r == s->group_first[g] + s->group_count[g] - 1 && t + BN >= s->range_hi[r];
  }
  __device__ int nvalid() const { return min(BN, s->range_hi[r] - t); }
  __device__ void next() {
    t += BN;
    if (t < s->range_hi[r]) return;
    ++r;
    if (r < s->group_first[g] + s->group_count[g]) {
      t = s->range_lo[r];
      return;
    }
    ++g;
    if (g < s->n_groups) {
      r = s->group_first[g];
      t = s->range_lo[r];
    }
  }
};

__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, uint32_t budget) {
  for (uint32_t it = 0; it < budget; ++it)
    if (mbar_try_wait(bar, parity)) return true;
  raise_dev_error(AS_DEVERR_TIMEOUT);
  return false;
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
  const int tiles_per_block = (L.block_rows + BM - 1) / BM;
  const int blk = blockIdx.x / tiles_per_block;
  const int qt = blockIdx.x % tiles_per_block;
  const int bh = blockIdx.y;
  const int block_lo = L.block_row0 + blk * L.block_rows;
  const int q_lo = block_lo + qt * BM;
  const int q_hi = min(min(q_lo + BM, block_lo + L.block_rows), L.S);
  const uint32_t budget = L.poll_budget;

  if (threadIdx.x == 0) {
    mbar_init(&c.q_full, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&c.k_full[s], 1);
      mbar_init(&c.k_empty[s], 1);
      mbar_init(&c.v_full[s], 1);
      mbar_init(&c.v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&c.s_full[b], 1);
      mbar_init(&c.s_free[b], 128);
    }
    mbar_init(&c.p_full, 128);
    mbar_init(&c.o_ready, 1);
    mbar_init(&c.o_free, 128);
    mbar_init(&c.drain, 1);
    c.abort = 0;
    build_schedule(L.code + blk * L.P, L.dest_of, L.P, L.n, c.sched);
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

  uint8_t* sQ = smem + Lay::Q_OFF;
  uint8_t* sP = smem + Lay::P_OFF;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && c.sched.n_groups > 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&c.q_full, Lay::TILE_BYTES);
      for (int rg = 0; rg < Lay::NREG; ++rg)
        tma_load_3d(sQ + rg * REGION, &tm_q, &c.q_full, rg * 64, q_lo, bh);
      TileWalk w;
      int j = 0;
      for (w.start(&c.sched); w.valid(); w.next(), ++j) {
        const int st = j % NST;
        const uint32_t ph = (j / NST) & 1;
        if (!mbar_wait(&c.k_empty[st], ph ^ 1, abort_flag, budget)) break;
        uint8_t* sK = smem + Lay::K_OFF + st * Lay::TILE_BYTES;
        mbar_arrive_expect_tx(&c.k_full[st], Lay::TILE_BYTES);
        for (int rg = 0; rg < Lay::NREG; ++rg)
          tma_load_3d(sK + rg * REGION, &tm_k, &c.k_full[st], rg * 64, w.t, bh);
        if (!mbar_wait(&c.v_empty[st], ph ^ 1, abort_flag, budget)) { ++j; break; }
        uint8_t* sV = smem + Lay::V_OFF + st * Lay::TILE_BYTES;
        mbar_arrive_expect_tx(&c.v_full[st], Lay::TILE_BYTES);
        for (int rg = 0; rg < Lay::NREG; ++rg)
          tma_load_3d(sV + rg * REGION, &tm_v, &c.v_full[st], rg * 64, w.t, bh);
      }
      // before the CTA may exit, every issued load must have landed
      if (*abort_flag) {
        drain_wait(&c.q_full, 0, budget);
        for (int jj = max(0, j - NST); jj < j; ++jj) {
          drain_wait(&c.k_full[jj % NST], (jj / NST) & 1, budget);
          drain_wait(&c.v_full[jj % NST], (jj / NST) & 1, budget);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0 && c.sched.n_groups > 0) {
      constexpr uint32_t IDESC_QK = idesc_bf16_f32(BM, BN, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16_f32(BM, D, false, true);
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t p_base = smem_u32(sP);
      bool ok = mbar_wait(&c.q_full, 0, abort_flag, budget);
      tc_fence_after();
      // the PV of tile j-1 is issued after the QK of tile j
      int prev_st = 0, prev_group = 0;
      bool prev_first = false;
      int group = 0;
      auto issue_pv = [&](int jp) -> bool {
        if (prev_first && prev_group > 0)
          if (!mbar_wait(&c.o_free, (prev_group - 1) & 1, abort_flag, budget)) return false;
        if (!mbar_wait(&c.p_full, jp & 1, abort_flag, budget)) return false;
        if (!mbar_wait(&c.v_full[prev_st], (jp / NST) & 1, abort_flag, budget)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(smem + Lay::V_OFF + prev_st * Lay::TILE_BYTES);
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t a = smem_desc_sw128(p_base + (kk >> 2) * REGION + (kk & 3) * 32, 16, 1024);
          const uint64_t b = smem_desc_sw128(v_base + kk * 16 * 128, REGION, 1024);
          umma_bf16_ss(tmem + TMEM_O, a, b, IDESC_PV, (kk > 0 || !prev_first) ? 1u : 0u);
        }
        umma_commit(&c.o_ready);
        umma_commit(&c.v_empty[prev_st]);
        return true;
      };
      TileWalk w;
      int j = 0;
      if (ok) {
        for (w.start(&c.sched); w.valid(); w.next(), ++j) {
          const int st = j % NST;
          if (!mbar_wait(&c.k_full[st], (j / NST) & 1, abort_flag, budget)) { ok = false; break; }
          if (j >= 2 && !mbar_wait(&c.s_free[j & 1], ((j - 2) >> 1) & 1, abort_flag, budget)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_base = smem_u32(smem + Lay::K_OFF + st * Lay::TILE_BYTES);
          const uint32_t s_col = (j & 1) * BN;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * REGION + (kk & 3) * 32;
            const uint64_t a = smem_desc_sw128(q_base + off, 16, 1024);
            const uint64_t b = smem_desc_sw128(k_base + off, 16, 1024);
            umma_bf16_ss(tmem + s_col, a, b, IDESC_QK, kk > 0 ? 1u : 0u);
          }
          umma_commit(&c.s_full[j & 1]);
          umma_commit(&c.k_empty[st]);
          if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
          if (w.first() && j > 0) ++group;
          prev_st = st;
          prev_first = w.first();
          prev_group = group;
        }
        if (ok && j >= 1) issue_pv(j - 1);
      }
      // all issued MMAs must be complete before TMEM is released
      umma_commit(&c.drain);
      drain_wait(&c.drain, 0, budget);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int quarter = warp - 4;
    const int row = quarter * 32 + lane;
    const int s_row = q_lo + row;
    const uint32_t t_lane = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float sl2 = L.scale * 1.4426950408889634f;
    float m = -INFINITY, l = 0.f;
    int pv_done = 0;
    int group = 0;
    TileWalk w;
    int j = 0;
    for (w.start(&c.sched); w.valid(); w.next(), ++j) {
      const bool first = w.first();
      const bool last = w.last();
      const int nv = w.nvalid();
      if (first && j > 0) ++group;
      if (!mbar_wait(&c.s_full[j & 1], (j >> 1) & 1, abort_flag, budget)) break;
      tc_fence_after();
      float s[BN];
      {
        uint32_t r[32];
#pragma unroll
        for (int ch = 0; ch < BN / 32; ++ch) {
          tmem_ld32(t_lane + (j & 1) * BN + ch * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) s[ch * 32 + e] = __uint_as_float(r[e]);
        }
      }
      tc_fence_before();
      mbar_arrive(&c.s_free[j & 1]);
      float mx = -INFINITY;
#pragma unroll
      for (int e = 0; e < BN; ++e) {
        if (e >= nv) s[e] = -INFINITY;
        mx = fmaxf(mx, s[e]);
      }
      const float m_tile = mx * sl2;
      float m_use = m, alpha = 1.f;
      bool rescale = false;
      if (first) {
        m_use = m_tile;
      } else if (m_tile > m + RESCALE_THRESHOLD) {
        m_use = m_tile;
        alpha = ex2_approx(m - m_use);
        rescale = true;
      }
      float rs = 0.f;
#pragma unroll
      for (int e = 0; e < BN; ++e) {
        s[e] = ex2_approx(fmaf(s[e], sl2, -m_use));
        rs += s[e];
      }
      // O and the P buffer are free once the previous PV has completed
      bool ok = true;
      while (pv_done < j) {
        if (!mbar_wait(&c.o_ready, pv_done & 1, abort_flag, budget)) { ok = false; break; }
        ++pv_done;
      }
      if (!ok) break;
      tc_fence_after();
      if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(t_lane + TMEM_O + ch * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(t_lane + TMEM_O + ch * 32, r);
        }
        tmem_wait_st();
      }
      l = first ? rs : fmaf(l, alpha, rs);
      m = m_use;
      // P row -> shared memory, K-major 128-byte swizzle (two 64-key chunks)
#pragma unroll
      for (int ch = 0; ch < BN / 8; ++ch) {
        uint4 pk;
        pk.x = pack_bf16x2(s[ch * 8 + 0], s[ch * 8 + 1]);
        pk.y = pack_bf16x2(s[ch * 8 + 2], s[ch * 8 + 3]);
        pk.z = pack_bf16x2(s[ch * 8 + 4], s[ch * 8 + 5]);
        pk.w = pack_bf16x2(s[ch * 8 + 6], s[ch * 8 + 7]);
        const int region = ch >> 3;
        const int phys = (ch & 7) ^ (row & 7);
        *reinterpret_cast<uint4*>(sP + region * REGION + row * 128 + phys * 16) = pk;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&c.p_full);
      if (last) {
        while (pv_done < j + 1) {
          if (!mbar_wait(&c.o_ready, pv_done & 1, abort_flag, budget)) { ok = false; break; }
          ++pv_done;
        }
        if (!ok) break;
        tc_fence_after();
        const int dest = c.sched.group_dest[group];
        float* orow;
        float* lrow;
        if (dest < 0) {
          const long long r_idx = static_cast<long long>(bh) * L.out_rows + (s_row - L.out_row0);
          orow = L.out + r_idx * D;
          lrow = L.lse + r_idx;
        } else {
          const long long r_idx = static_cast<long long>(bh) * L.dst_rows + (s_row - L.dst_row0);
          orow = L.dst_out + dest * L.dst_plane_out + r_idx * D;
          lrow = L.dst_lse + dest * L.dst_plane_lse + r_idx;
        }
        const bool write = s_row < q_hi;
        const float inv_l = 1.0f / l;
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t r[32];
          tmem_ld32(t_lane + TMEM_O + ch * 32, r);
          tmem_wait_ld();
          if (write) {
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              float4 o4 = make_float4(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l,
                                      __uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
              *reinterpret_cast<float4*>(orow + ch * 32 + e) = o4;
            }
          }
        }
        if (write) *lrow = (m + log2f(l)) * 0.6931471805599453f;
        tc_fence_before();
        mbar_arrive(&c.o_free);
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
  if (!make_tmap(&tq, L.q, BH, L.S, D) || !make_tmap(&tk, L.k, BH, L.S, D) || !make_tmap(&tv, L.v, BH, L.S, D))
    return cudaErrorInvalidValue;
  constexpr int smem = smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int tiles_per_block = (L.block_rows + BM - 1) / BM;
  dim3 grid(L.n_blocks * tiles_per_block, BH);
  attn_tc_kernel<D><<<grid, NTHREADS, smem, st>>>(tq, tk, tv, L);
  return cudaGetLastError();
}

// One thread waits, with a bounded budget, on a barrier that nothing completes.
__global__ void timeout_probe_kernel(unsigned int budget) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, budget);
}

}  // namespace

cudaError_t launch_timeout_probe(unsigned int poll_budget, cudaStream_t st) {
  timeout_probe_kernel<<<1, 32, 0, st>>>(poll_budget);
  return cudaGetLastError();
}

cudaError_t read_and_clear_dev_error(unsigned int* bits, cudaStream_t st) {
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(v));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return e;
  }
  *bits = v;
  return cudaSuccess;
}

cudaError_t launch_attn_tc_bf16(const AttnLaunch& L, cudaStream_t st) {
  if (L.d == 128) return launch_d<128>(L, st);
  if (L.d == 64) return launch_d<64>(L, st);
  return cudaErrorInvalidValue;
}

}  // namespace asp
