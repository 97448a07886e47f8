// Internal interface between the C-ABI dispatcher (as_api.cu) and the kernels.
// Not installed; the public boundary is include/as_partition.h.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#ifndef AS_MAX_P
#define AS_MAX_P 64
#endif

// kernel codes for one (query row block, KV partition) pair
#define AS_KCODE_SKIP 0     // partition not read
#define AS_KCODE_COMPOSE 1  // partition folded into the block's composite state
#define AS_KCODE_EMIT 2     // partition emitted as its own state to a destination plane

// bits of the device error word
#define AS_DEVERR_TIMEOUT 1u
#define AS_DEVERR_BOUNDS 2u  // checked build (ASP_DEBUG): an index check failed and its access was skipped

namespace asp {

// Everything an attention launch needs, passed by value as a kernel parameter.
struct AttnLaunch {
  const void* q;  // [B,H,S,d] (used by the SIMT path; the TMA path reads via tensor maps)
  const void* k;  // [B,H,S_kv,d]
  const void* v;
  int B, H, S, d, P, n;  // S: query (and output) rows per head; n: rows per partition
  // K/V rows per head, and the first K/V row of each KV partition j (its
  // n rows are contiguous); for one GPU holding every partition S_kv = S and
  // kv_row0[j] = j * n
  int S_kv;
  int kv_row0[AS_MAX_P];
  float scale;
  // query rows: n_blocks blocks of block_rows rows starting at block_row0; block b
  // uses row b of `code` ([n_blocks][P])
  int n_blocks, block_rows, block_row0;
  uint8_t code[AS_MAX_P * AS_MAX_P];
  // destination plane of each AS_KCODE_EMIT partition; consecutive emitted
  // partitions with the same destination form one accumulation group
  int8_t dest_of[AS_MAX_P];
  // composite output: row s of head bh at ((bh * out_rows) + s - out_row0)
  float* out;
  float* lse;
  int out_rows, out_row0;
  // emitted planes: plane p, row s of head bh at p * plane + (bh * dst_rows + s - dst_row0);
  // OUT in fp32, or in bf16 (round to nearest even) when dst_bf16
  void* dst_out;
  float* dst_lse;
  int dst_bf16;
  int dst_planes;  // planes the destination holds (the checked build's bound on dest_of)
  int dst_rows, dst_row0;
  long long dst_plane_out, dst_plane_lse;
};

// compose of N states per row with strided state storage (as_compose)
struct ComposeStrided {
  const float* outs;
  const float* lses;
  int n_states, d;
  long long rows;
  long long stride_out, stride_lse;  // distance between consecutive states, in elements
  float* out;
  float* lse;
};

// final compose of a step: composite (in out/lse) + cache planes, chosen per
// query partition from the step plan
struct ComposePlan {
  int B, H, S, d, P, n;
  // per query partition: -1 = composite, -2 = local state, G = cache plane G
  int8_t src[AS_MAX_P][AS_MAX_P + 2];
  uint8_t nsrc[AS_MAX_P];
  const void* cache_out;  // fp32, or bf16 when cache_bf16
  int cache_bf16;
  int n_planes;  // cache planes (the checked build's bound on src)
  const float* cache_lse;
  long long plane_out, plane_lse;
  const float* local_out;  // [B,H,S,d] local states AS(i,i) (source -2), may be null
  const float* local_lse;
  float* out;  // [B,H,S,d]: holds the composite on entry (where used), the final state on exit
  float* lse;
};

// entry selection for the planner's anchor statistics ([P][n_groups], 1 = reduce)
struct PlanRows {
  uint8_t v[AS_MAX_P * AS_MAX_P];
};

cudaError_t launch_attn_tc_bf16(const AttnLaunch& L, cudaStream_t st);
// planner reductions: partials scratch [K][BH][2] doubles, sums [K][2] doubles
cudaError_t launch_drift(const float* now, const float* anchor, int BH, int S, int d, int P, double* partials,
                         double* sums, cudaStream_t st);
// address (on the current device) and size of the fixed drift scratch
cudaError_t static_drift_scratch(double** ptr, size_t* capacity_doubles);
cudaError_t launch_anchor_stats(const void* cache_out, bool out_bf16, const float* cache_lse, const float* lse_full,
                                long long plane_out, long long plane_lse, int P, int NG, int BH, int S, int d,
                                const PlanRows& sel, double* partials, double* sums, cudaStream_t st);
cudaError_t launch_attn_simt_f32(const AttnLaunch& L, cudaStream_t st);
cudaError_t launch_compose_strided(const ComposeStrided& a, cudaStream_t st);
cudaError_t launch_compose_plan(const ComposePlan& a, cudaStream_t st);
// residual compression of exchanged rows [rows, d] (bf16 values, int8 codes,
// fp32 scales); base is updated in place to the new reconstruction
cudaError_t launch_residual_encode(const void* x, void* base, int8_t* codes, float* scales, long long rows, int d,
                                   cudaStream_t st);
cudaError_t launch_residual_decode(const int8_t* codes, const float* scales, void* base, long long rows, int d,
                                   cudaStream_t st);
cudaError_t launch_timeout_probe(unsigned int polls, unsigned int ns, cudaStream_t st);
cudaError_t launch_exp2_probe(const float* x, float* y, long long n, int mode, cudaStream_t st);
// Each translation unit holds its own device error word (no relocatable
// device code); each returns and clears its own.
cudaError_t dev_error_attn_tc(unsigned int* bits);
cudaError_t dev_error_attn_simt(unsigned int* bits);
cudaError_t dev_error_compose(unsigned int* bits);
// checked build only: one thread writes buf[n] behind an index check against n
cudaError_t launch_bounds_probe(float* buf, long long n, cudaStream_t st);

}  // namespace asp
