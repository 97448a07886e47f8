// Residual compression of the rows that context-parallel ranks exchange.
//
// CompactFusion ("Accelerating Parallel Diffusion Model Serving with Residual
// Compression", arXiv 2507.17511; Abstract on its listing page) sends, step
// after step, compressed residuals (step-wise activation differences) with
// lightweight error feedback so that compression errors do not accumulate.
// Here a row of d values (one token of one head of K or V, bf16) is coded
// against the receiver's reconstruction of it, which the sender tracks as
// well: r = x - base, s = max|r| / 127, q = round-half-even(r * (127 /
// max|r|)) in [-127, 127] (int8), and both sides move the reconstruction to
// bf16(base + q * s).  A step's coding error therefore enters the next
// step's residual (the error feedback).  Every operation is one float32
// operation rounded on its own (no fused multiply-add), so the codes and the
// reconstruction are bit-reproducible on the host.
//
// One warp per row, d / 32 values per lane, four rows in flight per warp;
// persistent grid.  HBM-bound:
// per row the encoder reads 2 d bf16 values and writes d codes, 4 bytes of
// scale and d bf16 values; the decoder reads d codes, the scale and d bf16
// values and writes d bf16 values.
#include "as_device.cuh"

namespace asp {
namespace {

constexpr int WARPS = 8;
constexpr int CTAS_PER_SM = 8;

__device__ __forceinline__ float warp_max_f(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}

// E = D / 32 bf16 values per lane: 4 (one 8-byte load) or 2 (4 bytes)
template <int E>
struct Lane;
template <>
struct Lane<4> {
  using B16 = uint2;     // 4 bf16
  using Q8 = uint32_t;   // 4 int8
};
template <>
struct Lane<2> {
  using B16 = uint32_t;  // 2 bf16
  using Q8 = uint16_t;   // 2 int8
};

template <int E>
__device__ __forceinline__ void unpack_bf16(const typename Lane<E>::B16& u, float (&v)[E]) {
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&u);
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    v[e] = __uint_as_float(w[e / 2] << 16);
    v[e + 1] = __uint_as_float(w[e / 2] & 0xffff0000u);
  }
}

template <int E>
__device__ __forceinline__ typename Lane<E>::B16 pack_bf16(const float (&v)[E]) {
  typename Lane<E>::B16 u;
  uint32_t* w = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
  for (int e = 0; e < E; e += 2) {
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(v[e]));
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(v[e + 1]));
    w[e / 2] = lo | (hi << 16);
  }
  return u;
}

// bf16(base + q * s), the product and the sum each rounded to float32
__device__ __forceinline__ float apply_one(float base, int q, float s) {
  return __fadd_rn(base, __fmul_rn(static_cast<float>(q), s));
}

// Each warp takes ROWS_PER_TRIP rows per iteration, their loads issued
// before any of them is used (one row per trip left the encoder at about
// half of HBM bandwidth, bound by latency).
constexpr int ROWS_PER_TRIP = 4;

template <int D>
__global__ void __launch_bounds__(WARPS * 32) residual_encode_kernel(const __nv_bfloat16* __restrict__ x,
                                                                     __nv_bfloat16* __restrict__ base,
                                                                     int8_t* __restrict__ codes,
                                                                     float* __restrict__ scales, long long rows) {
  constexpr int E = D / 32;
  using L = Lane<E>;
  const int lane = threadIdx.x & 31;
  const long long nw = static_cast<long long>(gridDim.x) * WARPS;
  const long long w = static_cast<long long>(blockIdx.x) * WARPS + (threadIdx.x >> 5);
  for (long long r0 = w; r0 < rows; r0 += nw * ROWS_PER_TRIP) {
    typename L::B16 xu[ROWS_PER_TRIP], bu[ROWS_PER_TRIP];
#pragma unroll
    for (int k = 0; k < ROWS_PER_TRIP; ++k) {
      const long long row = r0 + k * nw;
      if (row < rows) {
        const long long off = row * D + lane * E;
        xu[k] = *reinterpret_cast<const typename L::B16*>(x + off);
        bu[k] = *reinterpret_cast<const typename L::B16*>(base + off);
      }
    }
#pragma unroll
    for (int k = 0; k < ROWS_PER_TRIP; ++k) {
      const long long row = r0 + k * nw;
      if (row >= rows) break;
      const long long off = row * D + lane * E;
      float xv[E], bv[E], r[E];
      unpack_bf16<E>(xu[k], xv);
      unpack_bf16<E>(bu[k], bv);
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        r[e] = __fsub_rn(xv[e], bv[e]);
        amax = fmaxf(amax, fabsf(r[e]));
      }
      amax = warp_max_f(amax);
      const float inv = amax > 0.f ? __fdiv_rn(127.f, amax) : 0.f;
      const float s = __fdiv_rn(amax, 127.f);
      typename L::Q8 qp = 0;
      float nb[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int q = static_cast<int>(fminf(fmaxf(rintf(__fmul_rn(r[e], inv)), -127.f), 127.f));
        qp |= static_cast<typename L::Q8>(static_cast<uint8_t>(static_cast<int8_t>(q))) << (8 * e);
        nb[e] = apply_one(bv[e], q, s);
      }
      *reinterpret_cast<typename L::Q8*>(codes + off) = qp;
      *reinterpret_cast<typename L::B16*>(base + off) = pack_bf16<E>(nb);
      if (lane == 0) scales[row] = s;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(WARPS * 32) residual_decode_kernel(const int8_t* __restrict__ codes,
                                                                     const float* __restrict__ scales,
                                                                     __nv_bfloat16* __restrict__ base,
                                                                     long long rows) {
  constexpr int E = D / 32;
  using L = Lane<E>;
  const int lane = threadIdx.x & 31;
  const long long nw = static_cast<long long>(gridDim.x) * WARPS;
  const long long w = static_cast<long long>(blockIdx.x) * WARPS + (threadIdx.x >> 5);
  for (long long r0 = w; r0 < rows; r0 += nw * ROWS_PER_TRIP) {
    typename L::Q8 qu[ROWS_PER_TRIP];
    typename L::B16 bu[ROWS_PER_TRIP];
    float su[ROWS_PER_TRIP];
#pragma unroll
    for (int k = 0; k < ROWS_PER_TRIP; ++k) {
      const long long row = r0 + k * nw;
      if (row < rows) {
        const long long off = row * D + lane * E;
        qu[k] = *reinterpret_cast<const typename L::Q8*>(codes + off);
        bu[k] = *reinterpret_cast<const typename L::B16*>(base + off);
        su[k] = scales[row];
      }
    }
#pragma unroll
    for (int k = 0; k < ROWS_PER_TRIP; ++k) {
      const long long row = r0 + k * nw;
      if (row >= rows) break;
      const long long off = row * D + lane * E;
      float bv[E], nb[E];
      unpack_bf16<E>(bu[k], bv);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int q = static_cast<int8_t>(static_cast<uint8_t>(qu[k] >> (8 * e)));
        nb[e] = apply_one(bv[e], q, su[k]);
      }
      *reinterpret_cast<typename L::B16*>(base + off) = pack_bf16<E>(nb);
    }
  }
}

cudaError_t grid_for_rows(long long rows, unsigned* grid) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long ctas = (rows + WARPS * ROWS_PER_TRIP - 1) / (WARPS * ROWS_PER_TRIP);
  const long long cap = static_cast<long long>(sms) * CTAS_PER_SM;
  *grid = static_cast<unsigned>(ctas < cap ? (ctas > 0 ? ctas : 1) : cap);
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_residual_encode(const void* x, void* base, int8_t* codes, float* scales, long long rows, int d,
                                   cudaStream_t st) {
  unsigned grid = 0;
  cudaError_t e = grid_for_rows(rows, &grid);
  if (e != cudaSuccess) return e;
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  auto* bb = static_cast<__nv_bfloat16*>(base);
  if (d == 128)
    residual_encode_kernel<128><<<grid, WARPS * 32, 0, st>>>(xb, bb, codes, scales, rows);
  else if (d == 64)
    residual_encode_kernel<64><<<grid, WARPS * 32, 0, st>>>(xb, bb, codes, scales, rows);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_residual_decode(const int8_t* codes, const float* scales, void* base, long long rows, int d,
                                   cudaStream_t st) {
  unsigned grid = 0;
  cudaError_t e = grid_for_rows(rows, &grid);
  if (e != cudaSuccess) return e;
  auto* bb = static_cast<__nv_bfloat16*>(base);
  if (d == 128)
    residual_decode_kernel<128><<<grid, WARPS * 32, 0, st>>>(codes, scales, bb, rows);
  else if (d == 64)
    residual_decode_kernel<64><<<grid, WARPS * 32, 0, st>>>(codes, scales, bb, rows);
  else
    return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace asp
