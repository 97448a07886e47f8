// Reductions of the anchor-guided planner (DiTango, arXiv 2607.15650; review
// page, Referee Report major comments 1-3 and the Axiom & Free-Parameter
// Ledger: Eq. 8 partition importance, Eq. 9 scale ratio, Eq. 10 local drift).
//
// Both kernels reduce in fp64 and in a fixed order: one CTA per
// (partition i[, partition j], head bh) writes its partial sums to the scratch
// buffer, and a second kernel adds the partials over bh in index order, so the
// result does not depend on scheduling.
//
//   drift: for every partition i, sum over its rows (all b, h) of
//          |now - anchor|^2 and |anchor|^2 (d columns each)
//   stats: for every selected pair (i, j), sum over the rows of i of
//          exp(LSE_ij - LSE_i) and |OUT_ij|^2
#include <mutex>

#include "as_device.cuh"

namespace asp {

// Fixed scratch for the allocation-free drift entry point
// (as_plan_drift_static): partials [P][B*H][2] doubles, then sums [P][2].
// 1 MiB, held by every device that loads the library until the process exits.
constexpr size_t STATIC_DRIFT_DOUBLES = size_t(1) << 17;
static __device__ __align__(256) double g_static_drift_scratch[STATIC_DRIFT_DOUBLES];

namespace {

constexpr int THREADS = 256;

__device__ __forceinline__ double block_sum(double x, double* sh) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) sh[warp] = x;
  __syncthreads();
  double tot = 0.0;
  if (threadIdx.x == 0)
    for (int w = 0; w < THREADS / 32; ++w) tot += sh[w];
  return tot;  // valid in thread 0
}

// partials[(i * BH + bh) * 2 + {0, 1}]
__global__ void __launch_bounds__(THREADS) drift_partials_kernel(const float* __restrict__ now,
                                                                 const float* __restrict__ anchor, int BH, int S,
                                                                 int d, int n, double* __restrict__ partials) {
  __shared__ double sh[THREADS / 32];
  const int i = blockIdx.x, bh = blockIdx.y;
  const long long base = (static_cast<long long>(bh) * S + static_cast<long long>(i) * n) * d;
  // the partition's n rows are contiguous: 16-byte loads, each element's
  // difference and square in fp64, four independent accumulators per sum
  const long long nvec = static_cast<long long>(n) * d / 4;
  const float4* nv = reinterpret_cast<const float4*>(now + base);
  const float4* av = reinterpret_cast<const float4*>(anchor + base);
  double dd[4] = {0.0, 0.0, 0.0, 0.0}, aa[4] = {0.0, 0.0, 0.0, 0.0};
  for (long long e = threadIdx.x; e < nvec; e += THREADS) {
    const float4 x4 = nv[e], a4 = av[e];
    const float xs[4] = {x4.x, x4.y, x4.z, x4.w}, as[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const double a = as[c];
      const double x = static_cast<double>(xs[c]) - a;
      dd[c] = fma(x, x, dd[c]);
      aa[c] = fma(a, a, aa[c]);
    }
  }
  const double sdd = block_sum((dd[0] + dd[1]) + (dd[2] + dd[3]), sh);
  const double saa = block_sum((aa[0] + aa[1]) + (aa[2] + aa[3]), sh);
  if (threadIdx.x == 0) {
    partials[(static_cast<long long>(i) * BH + bh) * 2 + 0] = sdd;
    partials[(static_cast<long long>(i) * BH + bh) * 2 + 1] = saa;
  }
}

// partials[((i * NG + G) * BH + bh) * 2 + {0, 1}] for selected entries (i, G);
// OUT entries in fp32 or bf16 (OutT)
template <class OutT>
__global__ void __launch_bounds__(THREADS) stats_partials_kernel(const OutT* __restrict__ cache_out,
                                                                 const float* __restrict__ cache_lse,
                                                                 const float* __restrict__ lse_full,
                                                                 long long plane_out, long long plane_lse, int NG,
                                                                 int BH, int S, int d, int n,
                                                                 const __grid_constant__ PlanRows sel,
                                                                 double* __restrict__ partials) {
  __shared__ double sh[THREADS / 32];
  const int pair = blockIdx.x, bh = blockIdx.y;
  const int i = pair / NG, j = pair % NG;  // j: the entry's plane (its group)
  if (!sel.v[pair]) {
    if (threadIdx.x == 0) {
      partials[(static_cast<long long>(pair) * BH + bh) * 2 + 0] = 0.0;
      partials[(static_cast<long long>(pair) * BH + bh) * 2 + 1] = 0.0;
    }
    return;
  }
  const long long row0 = static_cast<long long>(bh) * S + static_cast<long long>(i) * n;
  const float* lse_ij = cache_lse + j * plane_lse + row0;
  const float* lse_i = lse_full + row0;
  const OutT* out_ij = cache_out + j * plane_out + row0 * d;
  double ws = 0.0;
  for (int r = threadIdx.x; r < n; r += THREADS) ws += exp(static_cast<double>(lse_ij[r]) - lse_i[r]);
  // the entry's n rows of OUT are contiguous: 16-byte loads, every element
  // squared and summed in fp64 over four independent accumulators
  constexpr int EPV = 16 / static_cast<int>(sizeof(OutT));  // elements per 16-byte vector
  const long long nvec = static_cast<long long>(n) * d / EPV;
  const uint4* vec = reinterpret_cast<const uint4*>(out_ij);
  double sq4[4] = {0.0, 0.0, 0.0, 0.0};
  for (long long e = threadIdx.x; e < nvec; e += THREADS) {
    const uint4 u = vec[e];
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      if constexpr (sizeof(OutT) == 2) {
        const double lo = __uint_as_float(w[c] << 16), hi = __uint_as_float(w[c] & 0xffff0000u);
        sq4[c] = fma(lo, lo, sq4[c]);
        sq4[c] = fma(hi, hi, sq4[c]);
      } else {
        const double x = __uint_as_float(w[c]);
        sq4[c] = fma(x, x, sq4[c]);
      }
    }
  }
  const double sws = block_sum(ws, sh);
  const double ssq = block_sum((sq4[0] + sq4[1]) + (sq4[2] + sq4[3]), sh);
  if (threadIdx.x == 0) {
    partials[(static_cast<long long>(pair) * BH + bh) * 2 + 0] = sws;
    partials[(static_cast<long long>(pair) * BH + bh) * 2 + 1] = ssq;
  }
}

// out[k * 2 + c] = sum over bh of partials[(k * BH + bh) * 2 + c], in bh order
__global__ void sum_over_heads_kernel(const double* __restrict__ partials, int K, int BH, double* __restrict__ out) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  double a = 0.0, b = 0.0;
  for (int bh = 0; bh < BH; ++bh) {
    a += partials[(static_cast<long long>(k) * BH + bh) * 2 + 0];
    b += partials[(static_cast<long long>(k) * BH + bh) * 2 + 1];
  }
  out[k * 2 + 0] = a;
  out[k * 2 + 1] = b;
}

}  // namespace

cudaError_t launch_drift(const float* now, const float* anchor, int BH, int S, int d, int P, double* partials,
                         double* sums, cudaStream_t st) {
  const int n = S / P;
  drift_partials_kernel<<<dim3(P, BH), THREADS, 0, st>>>(now, anchor, BH, S, d, n, partials);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sum_over_heads_kernel<<<(P + 127) / 128, 128, 0, st>>>(partials, P, BH, sums);
  return cudaGetLastError();
}

// Device address of the fixed drift scratch on the current device.  In host
// code the array's name only stands in for the symbol, so the address comes
// from cudaGetSymbolAddress, once per device (the first call on a device does
// it, with that device current), and is cached.
cudaError_t static_drift_scratch(double** ptr, size_t* capacity_doubles) {
  constexpr int MAX_DEVICES = 64;
  static double* addr[MAX_DEVICES] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_drift_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = static_cast<double*>(p);
  }
  *ptr = addr[dev];
  *capacity_doubles = STATIC_DRIFT_DOUBLES;
  return cudaSuccess;
}

cudaError_t launch_anchor_stats(const void* cache_out, bool out_bf16, const float* cache_lse, const float* lse_full,
                                long long plane_out, long long plane_lse, int P, int NG, int BH, int S, int d,
                                const PlanRows& sel, double* partials, double* sums, cudaStream_t st) {
  const int n = S / P;
  if (out_bf16)
    stats_partials_kernel<__nv_bfloat16><<<dim3(P * NG, BH), THREADS, 0, st>>>(
        static_cast<const __nv_bfloat16*>(cache_out), cache_lse, lse_full, plane_out, plane_lse, NG, BH, S, d, n, sel,
        partials);
  else
    stats_partials_kernel<float><<<dim3(P * NG, BH), THREADS, 0, st>>>(
        static_cast<const float*>(cache_out), cache_lse, lse_full, plane_out, plane_lse, NG, BH, S, d, n, sel,
        partials);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sum_over_heads_kernel<<<(P * NG + 127) / 128, 128, 0, st>>>(partials, P * NG, BH, sums);
  return cudaGetLastError();
}

}  // namespace asp
