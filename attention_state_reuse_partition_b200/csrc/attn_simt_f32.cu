// Partition attention in fp32 on the CUDA cores.
//
// Same contract as the tensor-core path (one state per accumulation group of
// the KV schedule; see as_device.cuh) for fp32 inputs.  tcgen05 has no fp32
// operand type and TF32 rounding would exceed a 1e-5 tolerance, so this path
// uses FFMA: one thread per query row, K/V tiles of 32 keys staged in shared
// memory, the online softmax of each row kept in registers, expf/logf for the
// exponentials.  It exists for fp32 workloads (small sizes); it is not tuned.
#include "as_device.cuh"

namespace asp {
namespace {

constexpr int ROWS = 128;  // query rows per CTA (one per thread)
constexpr int KT = 32;     // keys per shared-memory tile

template <int D>
__global__ void __launch_bounds__(ROWS) attn_simt_kernel(const __grid_constant__ AttnLaunch L) {
  extern __shared__ float sm[];
  float* sQ = sm;                       // [ROWS][D+1]
  float* sK = sQ + ROWS * (D + 1);      // [KT][D]
  float* sV = sK + KT * D;              // [KT][D]
  __shared__ KvSchedule sched;

  const int tiles_per_block = (L.block_rows + ROWS - 1) / ROWS;
  const int blk = blockIdx.x / tiles_per_block;
  const int qt = blockIdx.x % tiles_per_block;
  const int bh = blockIdx.y;
  const int block_lo = L.block_row0 + blk * L.block_rows;
  const int q_lo = block_lo + qt * ROWS;
  const int q_hi = min(min(q_lo + ROWS, block_lo + L.block_rows), L.S);
  const float* Q = static_cast<const float*>(L.q) + static_cast<long long>(bh) * L.S * D;
  const float* K = static_cast<const float*>(L.k) + static_cast<long long>(bh) * L.S_kv * D;
  const float* V = static_cast<const float*>(L.v) + static_cast<long long>(bh) * L.S_kv * D;

  if (threadIdx.x == 0) build_schedule(L.code + blk * L.P, L.dest_of, L.kv_row0, L.P, L.n, sched);
  for (int i = threadIdx.x; i < ROWS * D; i += ROWS) {
    const int r = i / D, col = i % D;
    sQ[r * (D + 1) + col] = (q_lo + r < L.S) ? Q[static_cast<long long>(q_lo + r) * D + col] : 0.f;
  }
  __syncthreads();

  const int row = threadIdx.x;
  const int s_row = q_lo + row;
  const float* qrow = sQ + row * (D + 1);
  float o[D];
  float m = -INFINITY, l = 0.f;

  for (int g = 0; g < sched.n_groups; ++g) {
#pragma unroll
    for (int e = 0; e < D; ++e) o[e] = 0.f;
    m = -INFINITY;
    l = 0.f;
    for (int r = sched.group_first[g]; r < sched.group_first[g] + sched.group_count[g]; ++r) {
      for (int t = sched.range_lo[r]; t < sched.range_hi[r]; t += KT) {
        const int nv = min(KT, sched.range_hi[r] - t);
        __syncthreads();
        for (int i = threadIdx.x; i < KT * D; i += ROWS) {
          const int kr = i / D;
          const long long src = static_cast<long long>(t + kr) * D + (i % D);
          sK[i] = kr < nv ? K[src] : 0.f;
          sV[i] = kr < nv ? V[src] : 0.f;
        }
        __syncthreads();
        float sc[KT];
        float mx = -INFINITY;
#pragma unroll 4
        for (int kr = 0; kr < KT; ++kr) {
          float acc = 0.f;
#pragma unroll 16
          for (int e = 0; e < D; ++e) acc = fmaf(qrow[e], sK[kr * D + e], acc);
          sc[kr] = kr < nv ? acc * L.scale : -INFINITY;
          mx = fmaxf(mx, sc[kr]);
        }
        const float m_new = fmaxf(m, mx);
        const float alpha = (m == -INFINITY) ? 0.f : expf(m - m_new);
        l *= alpha;
#pragma unroll
        for (int e = 0; e < D; ++e) o[e] *= alpha;
        for (int kr = 0; kr < nv; ++kr) {
          const float p = expf(sc[kr] - m_new);
          l += p;
#pragma unroll
          for (int e = 0; e < D; ++e) o[e] = fmaf(p, sV[kr * D + e], o[e]);
        }
        m = m_new;
      }
    }
    const int dest = sched.group_dest[g];
    const int row0 = dest < 0 ? L.out_row0 : L.dst_row0;
    const int rows = dest < 0 ? L.out_rows : L.dst_rows;
    if (s_row < q_hi && ASP_CHECK(dest < L.dst_planes && s_row >= row0 && s_row < row0 + rows)) {
      float* orow;
      __nv_bfloat16* brow = nullptr;  // bf16 cache planes
      float* lrow;
      if (dest < 0) {
        const long long r_idx = static_cast<long long>(bh) * L.out_rows + (s_row - L.out_row0);
        orow = L.out + r_idx * D;
        lrow = L.lse + r_idx;
      } else {
        const long long r_idx = static_cast<long long>(bh) * L.dst_rows + (s_row - L.dst_row0);
        const long long e_idx = dest * L.dst_plane_out + r_idx * D;
        orow = static_cast<float*>(L.dst_out) + e_idx;
        if (L.dst_bf16) brow = static_cast<__nv_bfloat16*>(L.dst_out) + e_idx;
        lrow = L.dst_lse + dest * L.dst_plane_lse + r_idx;
      }
      const float inv_l = 1.0f / l;
      if (brow) {
#pragma unroll
        for (int e = 0; e < D; ++e) brow[e] = __float2bfloat16_rn(o[e] * inv_l);
      } else {
#pragma unroll
        for (int e = 0; e < D; ++e) orow[e] = o[e] * inv_l;
      }
      *lrow = m + logf(l);
    }
  }
}

template <int D>
cudaError_t launch_d(const AttnLaunch& L, cudaStream_t st) {
  const int smem = (ROWS * (D + 1) + 2 * KT * D) * static_cast<int>(sizeof(float));
  cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int tiles_per_block = (L.block_rows + ROWS - 1) / ROWS;
  dim3 grid(L.n_blocks * tiles_per_block, L.B * L.H);
  attn_simt_kernel<D><<<grid, ROWS, smem, st>>>(L);
  return cudaGetLastError();
}

}  // namespace

cudaError_t dev_error_attn_simt(unsigned int* bits) { return read_and_clear_local_dev_error(bits); }

cudaError_t launch_attn_simt_f32(const AttnLaunch& L, cudaStream_t st) {
  if (L.d == 128) return launch_d<128>(L, st);
  if (L.d == 64) return launch_d<64>(L, st);
  return cudaErrorInvalidValue;
}

}  // namespace asp
