// State composition kernels (HBM-bound).
//
// DiTango (arXiv 2607.15650; review page, Axiom & Free-Parameter Ledger,
// Eq. 1-2): attention states compose associatively and commutatively.  For N
// states of one query row, LSE = m + ln sum_k exp(LSE_k - m) with m = max_k
// LSE_k, and OUT = sum_k exp(LSE_k - LSE) * OUT_k.  A row whose states are all
// empty (LSE = -inf) stays empty: OUT = 0, LSE = -inf.
//
// One warp composes a block of up to 8 consecutive rows that share their
// source list.  Lane k holds the LSEs of source k for the 8 rows (one 32-byte
// sector per source), so the max and the sum are warp reductions; the OUT
// rows are read with 128-bit loads, one 512-byte row per warp instruction
// (d = 128), several sources in flight per lane.  Every input byte is read
// once from HBM (the LSE re-reads of the third pass hit L1) and the output is
// written once.  Grids are persistent: 8 CTAs of 8 warps per SM of the
// current device.
#include "as_device.cuh"

namespace asp {
namespace {

constexpr int RB = 8;        // rows per warp block
constexpr int WARPS = 8;     // warps per CTA
constexpr int CTAS_PER_SM = 8;

template <int D>
struct Vec;
// a packed pair of bf16 (low half = first element) widened to fp32
__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

template <>
struct Vec<128> {
  using T = float4;
  static __device__ __forceinline__ float4 zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
  // this lane's 4 elements of row `row` of a state stored as E (fp32 or bf16)
  template <class E>
  static __device__ __forceinline__ float4 load(const void* base, long long row, int lane) {
    if constexpr (sizeof(E) == 2) {
      const uint2 u = reinterpret_cast<const uint2*>(static_cast<const E*>(base) + row * 128)[lane];
      return make_float4(bf_lo(u.x), bf_hi(u.x), bf_lo(u.y), bf_hi(u.y));
    } else {
      return reinterpret_cast<const float4*>(static_cast<const E*>(base) + row * 128)[lane];
    }
  }
  static __device__ __forceinline__ void fma(float4& a, float c, const float4& x) {
    a.x = fmaf(c, x.x, a.x);
    a.y = fmaf(c, x.y, a.y);
    a.z = fmaf(c, x.z, a.z);
    a.w = fmaf(c, x.w, a.w);
  }
};
template <>
struct Vec<64> {
  using T = float2;
  static __device__ __forceinline__ float2 zero() { return make_float2(0.f, 0.f); }
  template <class E>
  static __device__ __forceinline__ float2 load(const void* base, long long row, int lane) {
    if constexpr (sizeof(E) == 2) {
      const uint32_t u = reinterpret_cast<const uint32_t*>(static_cast<const E*>(base) + row * 64)[lane];
      return make_float2(bf_lo(u), bf_hi(u));
    } else {
      return reinterpret_cast<const float2*>(static_cast<const E*>(base) + row * 64)[lane];
    }
  }
  static __device__ __forceinline__ void fma(float2& a, float c, const float2& x) {
    a.x = fmaf(c, x.x, a.x);
    a.y = fmaf(c, x.y, a.y);
  }
};

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

struct Ptrs {
  const void* first;    // OUT base
  const float* second;  // LSE base
};

// Composes rows [row0, row0+nr) (nr <= RB) of `nsrc` sources.  src(k) gives the
// base pointers (out_base, lse_base) of source k such that row r's state is at
// row r of out_base and lse_base + r.  Sources [0, nf) keep OUT in fp32, the
// others in E (fp32 or bf16), so that every batch of loads has one type.  The
// output may alias a source: every source row is read before the output row
// is written, by the same warp.
template <int D, class E, int UNROLL, class SrcFn>
__device__ __forceinline__ void compose_rows(long long row0, int nr, int nsrc, int nf, SrcFn src, float* out,
                                             float* lse, int lane) {
  using V = Vec<D>;
  using T = typename V::T;
  float m[RB], tot[RB], inv[RB];
  // up to 32 sources (one per lane; the common case): lane k loads the LSEs
  // of source k once and keeps them, and each weight is one exponential
  float ev[RB];
  const bool one_chunk = nsrc <= 32;
  if (one_chunk) {
    const float* lb = lane < nsrc ? src(lane).second + row0 : nullptr;
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) ev[rr] = (lb != nullptr && rr < nr) ? lb[rr] : -INFINITY;
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) m[rr] = warp_max(ev[rr]);
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) ev[rr] = m[rr] != -INFINITY ? __expf(ev[rr] - m[rr]) : 0.f;
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) tot[rr] = warp_sum(ev[rr]);
  } else {
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) m[rr] = -INFINITY;
    for (int k0 = 0; k0 < nsrc; k0 += 32) {
      const int k = k0 + lane;
      if (k < nsrc) {
        const float* lb = src(k).second + row0;
#pragma unroll
        for (int rr = 0; rr < RB; ++rr)
          if (rr < nr) m[rr] = fmaxf(m[rr], lb[rr]);
      }
    }
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) {
      m[rr] = warp_max(m[rr]);
      tot[rr] = 0.f;
    }
    for (int k0 = 0; k0 < nsrc; k0 += 32) {
      const int k = k0 + lane;
      if (k < nsrc) {
        const float* lb = src(k).second + row0;
#pragma unroll
        for (int rr = 0; rr < RB; ++rr)
          if (rr < nr && m[rr] != -INFINITY) tot[rr] += __expf(lb[rr] - m[rr]);
      }
    }
#pragma unroll
    for (int rr = 0; rr < RB; ++rr) tot[rr] = warp_sum(tot[rr]);
  }
#pragma unroll
  for (int rr = 0; rr < RB; ++rr) inv[rr] = tot[rr] > 0.f ? 1.0f / tot[rr] : 0.f;

  T acc[RB];
#pragma unroll
  for (int rr = 0; rr < RB; ++rr) acc[rr] = V::zero();
  for (int k0 = 0; k0 < nsrc; k0 += 32) {
    const int k = k0 + lane;
    float coef[RB];
    if (one_chunk) {
#pragma unroll
      for (int rr = 0; rr < RB; ++rr) coef[rr] = ev[rr] * inv[rr];
    } else if (k < nsrc) {
      const float* lb = src(k).second + row0;
#pragma unroll
      for (int rr = 0; rr < RB; ++rr)
        coef[rr] = (rr < nr && tot[rr] > 0.f) ? __expf(lb[rr] - m[rr]) * inv[rr] : 0.f;
    } else {
#pragma unroll
      for (int rr = 0; rr < RB; ++rr) coef[rr] = 0.f;
    }
    const int kn = min(32, nsrc - k0);
    // one source at a time (its pointers resolved once), its rows' loads in
    // flight together
#pragma unroll UNROLL
    for (int kk = 0; kk < kn; ++kk) {
      const Ptrs sp = src(k0 + kk);
      T x[RB];
      if (k0 + kk < nf) {
#pragma unroll
        for (int rr = 0; rr < RB; ++rr)
          if (rr < nr) x[rr] = V::template load<float>(sp.first, row0 + rr, lane);
      } else {
#pragma unroll
        for (int rr = 0; rr < RB; ++rr)
          if (rr < nr) x[rr] = V::template load<E>(sp.first, row0 + rr, lane);
      }
#pragma unroll
      for (int rr = 0; rr < RB; ++rr)
        if (rr < nr) V::fma(acc[rr], __shfl_sync(0xffffffffu, coef[rr], kk), x[rr]);
    }
  }
#pragma unroll
  for (int rr = 0; rr < RB; ++rr) {
    if (rr >= nr) break;
    reinterpret_cast<T*>(out + (row0 + rr) * D)[lane] = acc[rr];
    if (lane == 0) lse[row0 + rr] = tot[rr] > 0.f ? m[rr] + __logf(tot[rr]) : -INFINITY;
  }
}

template <int D>
__global__ void __launch_bounds__(WARPS * 32, 2) compose_strided_kernel(const __grid_constant__ ComposeStrided a) {
  const int lane = threadIdx.x & 31;
  const long long nblk = (a.rows + RB - 1) / RB;
  const long long gw = static_cast<long long>(blockIdx.x) * WARPS + (threadIdx.x >> 5);
  const long long stride = static_cast<long long>(gridDim.x) * WARPS;
  auto src = [&](int k) {
    return Ptrs{a.outs + k * a.stride_out, a.lses + k * a.stride_lse};
  };
  for (long long b = gw; b < nblk; b += stride) {
    const long long row0 = b * RB;
    const int nr = static_cast<int>(min(static_cast<long long>(RB), a.rows - row0));
    // three sources' loads in flight: measured 6.95 against 6.90 TB/s with two
    compose_rows<D, float, 3>(row0, nr, a.n_states, 0, src, a.out, a.lse, lane);
  }
}

// E: type of the cache planes' OUT entries
template <int D, class E>
__global__ void __launch_bounds__(WARPS * 32, 2) compose_plan_kernel(const __grid_constant__ ComposePlan a) {
  const int lane = threadIdx.x & 31;
  const int bpp = (a.n + RB - 1) / RB;  // warp blocks per (head, partition)
  const long long nblk = static_cast<long long>(a.B) * a.H * a.P * bpp;
  const long long gw = static_cast<long long>(blockIdx.x) * WARPS + (threadIdx.x >> 5);
  const long long stride = static_cast<long long>(gridDim.x) * WARPS;
  for (long long b = gw; b < nblk; b += stride) {
    const int rb = static_cast<int>(b % bpp);
    const int i = static_cast<int>((b / bpp) % a.P);
    if (a.nsrc[i] == 0) continue;  // the composite already is the final state
    const long long bh = b / (static_cast<long long>(bpp) * a.P);
    const int s0 = i * a.n + rb * RB;
    const int nr = min(RB, (i + 1) * a.n - s0);
    const long long row0 = bh * a.S + s0;
    const int8_t* list = a.src[i];
    // branch-free pointer selection: the LSE pass evaluates a different
    // source in every lane
    auto src = [&](int k) {
      const int j = list[k];
      // checked build: a source is the composite, the local state or a plane of the cache
      const long long jj = (j < 0 || !ASP_CHECK(j >= -2 && j < a.n_planes)) ? 0 : j;
      const void* o = static_cast<const E*>(a.cache_out) + jj * a.plane_out;
      const float* l = a.cache_lse + jj * a.plane_lse;
      o = j == -2 ? static_cast<const void*>(a.local_out) : o;
      l = j == -2 ? a.local_lse : l;
      o = j == -1 ? static_cast<const void*>(a.out) : o;
      l = j == -1 ? a.lse : l;
      return Ptrs{o, l};
    };
    // the fp32 sources (composite, local state) lead the list
    const int nf = (a.nsrc[i] > 0 && list[0] < 0) + (a.nsrc[i] > 1 && list[1] < 0);
    // measured: bf16 planes (half the bytes per load) gain from four
    // sources' loads in flight (496 against 582 us per step compose with
    // two, although the d = 128 instance then spills about 180 bytes at the
    // two-CTA register cap); fp32 planes gain nothing from a second
    compose_rows<D, E, sizeof(E) == 2 ? 4 : 1>(row0, nr, a.nsrc[i], nf, src, a.out, a.lse, lane);
  }
}

// Step compose with bf16 cache planes, all loads of a block issued at once.
//
// compose_rows takes one source per trip to memory (its loop branches on the
// source's type, so the compiler does not hoist the next source's loads), and
// with few sources per row (bf16 groups: the composite and three or four
// planes) the warps spend their time waiting: 0.47 of HBM bandwidth.  Here a
// warp block of BRB rows issues, before using any of them, the LSEs of every
// source, the rows of the fp32 sources (composite, local state: at most two)
// and the packed rows of up to PLANES_PER_TRIP bf16 planes, so one trip to
// memory serves the whole block (a further trip per PLANES_PER_TRIP planes).
// Measured on the video reuse step with bf16 groups of 4 (ncu, per launch):
// 2 CTAs per SM with 4 planes per trip 367 us, 4 CTAs with 2-row blocks 366,
// 3 CTAs with 2-row blocks 412, 3 CTAs with 4-row blocks and 3 planes per
// trip 334 (used; 32 bytes of register spill at the 85-register cap), against
// 496 us for compose_rows.
constexpr int BRB = 4;               // rows per warp block
constexpr int PLANES_PER_TRIP = 3;   // bf16 planes whose rows are in flight together
constexpr int BATCHED_CTAS_PER_SM = 3;

template <int D>
struct Packed;  // this lane's share of one bf16 row: D / 32 values
template <>
struct Packed<128> {
  using T = uint2;
  static __device__ __forceinline__ void fma(float4& a, float c, const uint2& u) {
    a.x = fmaf(c, bf_lo(u.x), a.x);
    a.y = fmaf(c, bf_hi(u.x), a.y);
    a.z = fmaf(c, bf_lo(u.y), a.z);
    a.w = fmaf(c, bf_hi(u.y), a.w);
  }
};
template <>
struct Packed<64> {
  using T = uint32_t;
  static __device__ __forceinline__ void fma(float2& a, float c, const uint32_t& u) {
    a.x = fmaf(c, bf_lo(u), a.x);
    a.y = fmaf(c, bf_hi(u), a.y);
  }
};

template <int D>
__global__ void __launch_bounds__(WARPS * 32, BATCHED_CTAS_PER_SM) compose_plan_bf16_kernel(
    const __grid_constant__ ComposePlan a) {
  using V = Vec<D>;
  using T = typename V::T;
  using PK = typename Packed<D>::T;
  const int lane = threadIdx.x & 31;
  const int bpp = (a.n + BRB - 1) / BRB;  // warp blocks per (head, partition)
  const long long nblk = static_cast<long long>(a.B) * a.H * a.P * bpp;
  const long long gw = static_cast<long long>(blockIdx.x) * WARPS + (threadIdx.x >> 5);
  const long long stride = static_cast<long long>(gridDim.x) * WARPS;
  for (long long b = gw; b < nblk; b += stride) {
    const int rb = static_cast<int>(b % bpp);
    const int i = static_cast<int>((b / bpp) % a.P);
    const int nsrc = a.nsrc[i];
    if (nsrc == 0) continue;  // the composite already is the final state
    const long long bh = b / (static_cast<long long>(bpp) * a.P);
    const int s0 = i * a.n + rb * BRB;
    const int nr = min(BRB, (i + 1) * a.n - s0);
    const long long row0 = bh * a.S + s0;
    const int8_t* list = a.src[i];
    const int nf = (list[0] < 0) + (nsrc > 1 && list[1] < 0);  // the fp32 sources lead
    auto out_of = [&](int k) -> const void* {
      const int j = list[k];
      if (j == -1) return a.out;
      if (j == -2) return a.local_out;
      const long long jj = ASP_CHECK(j >= 0 && j < a.n_planes) ? j : 0;
      return static_cast<const __nv_bfloat16*>(a.cache_out) + jj * a.plane_out;
    };
    auto lse_of = [&](int k) -> const float* {
      const int j = list[k];
      if (j == -1) return a.lse;
      if (j == -2) return a.local_lse;
      const long long jj = ASP_CHECK(j >= 0 && j < a.n_planes) ? j : 0;
      return a.cache_lse + jj * a.plane_lse;
    };
    // every load of the block's first trip: LSEs (lane k: source k), fp32 rows, bf16 rows
    float lv[BRB];
    {
      const float* lp = lane < nsrc ? lse_of(lane) + row0 : nullptr;
#pragma unroll
      for (int rr = 0; rr < BRB; ++rr) lv[rr] = (lp != nullptr && rr < nr) ? lp[rr] : -INFINITY;
    }
    T xf[2][BRB];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const float* base = k < nf ? static_cast<const float*>(out_of(k)) + row0 * D : nullptr;
#pragma unroll
      for (int rr = 0; rr < BRB; ++rr)
        xf[k][rr] = (base != nullptr && rr < nr) ? reinterpret_cast<const T*>(base + rr * D)[lane] : V::zero();
    }
    PK xe[PLANES_PER_TRIP][BRB];
    auto load_planes = [&](int k0) {
#pragma unroll
      for (int e = 0; e < PLANES_PER_TRIP; ++e) {
        const __nv_bfloat16* base =
            k0 + e < nsrc ? static_cast<const __nv_bfloat16*>(out_of(k0 + e)) + row0 * D : nullptr;
#pragma unroll
        for (int rr = 0; rr < BRB; ++rr)
          xe[e][rr] = (base != nullptr && rr < nr) ? reinterpret_cast<const PK*>(base + rr * D)[lane] : PK{};
      }
    };
    load_planes(nf);
    // weights: this lane's source weight per row; lane rr keeps row rr's LSE
    float coef[BRB];
    float lse_out = -INFINITY;
#pragma unroll
    for (int rr = 0; rr < BRB; ++rr) {
      const float m = warp_max(lv[rr]);
      const float e = m != -INFINITY ? __expf(lv[rr] - m) : 0.f;
      const float tot = warp_sum(e);
      coef[rr] = tot > 0.f ? e / tot : 0.f;
      if (lane == rr && tot > 0.f) lse_out = m + __logf(tot);
    }
    T acc[BRB];
#pragma unroll
    for (int rr = 0; rr < BRB; ++rr) acc[rr] = V::zero();
#pragma unroll
    for (int k = 0; k < 2; ++k)
#pragma unroll
      for (int rr = 0; rr < BRB; ++rr) {
        const float c = __shfl_sync(0xffffffffu, coef[rr], k);
        if (k < nf) V::fma(acc[rr], c, xf[k][rr]);
      }
    for (int k0 = nf; k0 < nsrc; k0 += PLANES_PER_TRIP) {
      if (k0 > nf) load_planes(k0);
#pragma unroll
      for (int e = 0; e < PLANES_PER_TRIP; ++e)
#pragma unroll
        for (int rr = 0; rr < BRB; ++rr) {
          const float c = __shfl_sync(0xffffffffu, coef[rr], min(k0 + e, 31));
          if (k0 + e < nsrc) Packed<D>::fma(acc[rr], c, xe[e][rr]);
        }
    }
#pragma unroll
    for (int rr = 0; rr < BRB; ++rr)
      if (rr < nr) reinterpret_cast<T*>(a.out + (row0 + rr) * D)[lane] = acc[rr];
    if (lane < nr) a.lse[row0 + lane] = lse_out;
  }
}

// SMs of the current device
cudaError_t sm_count(int* n) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  return cudaDeviceGetAttribute(n, cudaDevAttrMultiProcessorCount, dev);
}

// persistent grid: at most CTAS_PER_SM CTAs per SM, fewer when there is less work
cudaError_t grid_for(long long nblk, unsigned* grid) {
  int sms = 0;
  cudaError_t e = sm_count(&sms);
  if (e != cudaSuccess) return e;
  const long long ctas = (nblk + WARPS - 1) / WARPS;
  const long long cap = static_cast<long long>(sms) * CTAS_PER_SM;
  *grid = static_cast<unsigned>(ctas < cap ? (ctas > 0 ? ctas : 1) : cap);
  return cudaSuccess;
}

}  // namespace

cudaError_t dev_error_compose(unsigned int* bits) { return read_and_clear_local_dev_error(bits); }

cudaError_t launch_compose_strided(const ComposeStrided& a, cudaStream_t st) {
  const long long nblk = (a.rows + RB - 1) / RB;
  unsigned grid = 0;
  cudaError_t e = grid_for(nblk, &grid);
  if (e != cudaSuccess) return e;
  if (a.d == 128)
    compose_strided_kernel<128><<<grid, WARPS * 32, 0, st>>>(a);
  else if (a.d == 64)
    compose_strided_kernel<64><<<grid, WARPS * 32, 0, st>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_compose_plan(const ComposePlan& a, cudaStream_t st) {
  // bf16 planes with at most two fp32 sources and 32 sources per row: the
  // batched kernel
  bool batched = a.cache_bf16 != 0;
  for (int i = 0; i < a.P && batched; ++i) {
    int nf = 0;
    while (nf < a.nsrc[i] && a.src[i][nf] < 0) ++nf;
    batched = nf <= 2 && a.nsrc[i] <= 32;
  }
  if (batched) {
    const long long nblk = static_cast<long long>(a.B) * a.H * a.P * ((a.n + BRB - 1) / BRB);
    unsigned grid = 0;
    cudaError_t e = grid_for(nblk, &grid);
    if (e != cudaSuccess) return e;
    if (a.d == 128)
      compose_plan_bf16_kernel<128><<<grid, WARPS * 32, 0, st>>>(a);
    else if (a.d == 64)
      compose_plan_bf16_kernel<64><<<grid, WARPS * 32, 0, st>>>(a);
    else
      return cudaErrorInvalidValue;
    return cudaGetLastError();
  }
  const long long nblk = static_cast<long long>(a.B) * a.H * a.P * ((a.n + RB - 1) / RB);
  unsigned grid = 0;
  cudaError_t e = grid_for(nblk, &grid);
  if (e != cudaSuccess) return e;
  if (a.d == 128 && a.cache_bf16)
    compose_plan_kernel<128, __nv_bfloat16><<<grid, WARPS * 32, 0, st>>>(a);
  else if (a.d == 128)
    compose_plan_kernel<128, float><<<grid, WARPS * 32, 0, st>>>(a);
  else if (a.d == 64 && a.cache_bf16)
    compose_plan_kernel<64, __nv_bfloat16><<<grid, WARPS * 32, 0, st>>>(a);
  else if (a.d == 64)
    compose_plan_kernel<64, float><<<grid, WARPS * 32, 0, st>>>(a);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace asp
