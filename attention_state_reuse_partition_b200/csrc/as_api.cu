// C-ABI boundary: argument checks, plan resolution, cache bookkeeping and
// kernel dispatch.  Every step of the computation runs in the kernels; this
// file only decides what to launch.
//
// Semantics follow DiTango (arXiv 2607.15650; review page: "What carries the
// argument" for the attention state, Axiom & Free-Parameter Ledger Eq. 1-2 for
// composition, Core claim and Referee Report "Summary" for fresh/reuse steps).
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <tuple>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "as_kernels.h"
#include "as_partition.h"

namespace {

#ifdef ASP_DEBUG
constexpr bool ASP_CHECKED_BUILD = ASP_DEBUG != 0;
#else
constexpr bool ASP_CHECKED_BUILD = false;
#endif

constexpr uint32_t CACHE_MAGIC = 0x41535043u;    // "ASPC"
constexpr uint32_t PLANNER_MAGIC = 0x41535050u;  // "ASPP"
thread_local std::string g_err;

as_status fail(as_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

as_status ok() {
  g_err.clear();
  return AS_OK;
}

// NVTX range around an entry point, so that profiler timelines show each call
// (a no-op unless a tool is attached)
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
};

as_status cuda_fail(cudaError_t e, const char* what) {
  return fail(AS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

as_status check_shape(int B, int H, int S, int d, int P) {
  if (B < 1 || H < 1 || S < 1) return fail(AS_ERR_INVALID_ARG, "B, H, S must be >= 1 (got %d, %d, %d)", B, H, S);
  if (d != 64 && d != 128) return fail(AS_ERR_INVALID_ARG, "d must be 64 or 128 (got %d)", d);
  if (P < 1 || P > AS_MAX_P) return fail(AS_ERR_INVALID_ARG, "P must be in [1, %d] (got %d)", AS_MAX_P, P);
  if (S % P != 0) return fail(AS_ERR_INVALID_ARG, "S (%d) must be a multiple of P (%d)", S, P);
  if (static_cast<long long>(B) * H > 65535) return fail(AS_ERR_INVALID_ARG, "B*H must be <= 65535");
  if (static_cast<long long>(S) * d >= (1ll << 31)) return fail(AS_ERR_INVALID_ARG, "S*d too large");
  return AS_OK;
}

// The kernels are built for sm_100a only.
as_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0)
    return fail(AS_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev, major, minor);
  return AS_OK;
}

as_status launch_attn(const asp::AttnLaunch& L, as_dtype dt, cudaStream_t st) {
  cudaError_t e = (dt == AS_BF16) ? asp::launch_attn_tc_bf16(L, st) : asp::launch_attn_simt_f32(L, st);
  if (e != cudaSuccess) return cuda_fail(e, dt == AS_BF16 ? "attention (tensor-core) launch" : "attention (fp32) launch");
  return AS_OK;
}

void base_launch(asp::AttnLaunch& L, const void* q, const void* k, const void* v, int B, int H, int S, int d,
                 int P, float scale) {
  std::memset(&L, 0, sizeof(L));
  L.q = q;
  L.k = k;
  L.v = v;
  L.B = B;
  L.H = H;
  L.S = S;
  L.d = d;
  L.P = P;
  L.n = S / P;
  L.scale = scale;
  L.S_kv = S;
  for (int j = 0; j < P; ++j) L.kv_row0[j] = j * (S / P);
}

// bit mask of the members of group (i, G) that carry plan code `code`
uint64_t group_mask(const uint8_t* plan, int P, int g, int i, int G, uint8_t code) {
  uint64_t m = 0;
  for (int j = G * g; j < std::min((G + 1) * g, P); ++j)
    if (plan[i * P + j] == code) m |= uint64_t(1) << j;
  return m;
}

// hit / age of a plan against the cache bookkeeping; codes checked first, then
// groups that mix reuse and store, then misses (never stored, or other members)
// rows q_first .. q_first + q_count - 1 of the plan belong to the cache's
// query partitions (all of them unless the cache is one rank's); the other
// rows are only checked for valid codes, and their hit and age are 0
as_status resolve(const as_cache* c, const uint8_t* plan, int step, uint8_t* hit, int32_t* age) {
  const int P = c->P, g = c->g, NG = c->n_groups;
  const int i0 = c->q_first, i1 = c->q_first + c->q_count;
  for (int x = 0; x < P * P; ++x)
    if (plan[x] > AS_PLAN_FRESH_STORE)
      return fail(AS_ERR_INVALID_ARG, "plan[%d][%d] = %d is not 0, 1 or 2", x / P, x % P, plan[x]);
  for (int i = i0; i < i1; ++i)
    for (int G = 0; G < NG; ++G)
      if (group_mask(plan, P, g, i, G, AS_PLAN_REUSE) && group_mask(plan, P, g, i, G, AS_PLAN_FRESH_STORE))
        return fail(AS_ERR_INVALID_ARG, "group (%d, %d) of size %d both reuses and stores members", i, G, g);
  for (int i = i0; i < i1; ++i)
    for (int G = 0; G < NG; ++G) {
      const uint64_t r = group_mask(plan, P, g, i, G, AS_PLAN_REUSE);
      if (!r) continue;
      if (c->t_c[i * NG + G] < 0)
        return fail(AS_ERR_CACHE_MISS, "group (%d, %d) is reused but its cache entry was never stored", i, G);
      if (r != c->member[i * NG + G])
        return fail(AS_ERR_CACHE_MISS, "group (%d, %d) reuses members 0x%llx but stores 0x%llx", i, G,
                    static_cast<unsigned long long>(r), static_cast<unsigned long long>(c->member[i * NG + G]));
    }
  for (int x = 0; x < P * P; ++x) {
    const bool r = plan[x] == AS_PLAN_REUSE && x / P >= i0 && x / P < i1;
    if (hit) hit[x] = r ? 1 : 0;
    if (age) age[x] = r ? step - c->t_c[(x / P) * NG + (x % P) / g] : 0;
  }
  return AS_OK;
}

// planner scratch: partials [P*P][BH][2] doubles, then sums [P*P][2] doubles
size_t planner_scratch(int B, int H, int P) {
  return (static_cast<size_t>(P) * P * B * H * 2 + static_cast<size_t>(P) * P * 2) * sizeof(double);
}

as_status check_scratch(void* scratch, size_t bytes, int B, int H, int P) {
  if (!scratch || (reinterpret_cast<uintptr_t>(scratch) & 7u) != 0)
    return fail(AS_ERR_INVALID_ARG, "planner scratch must be non-null and 8-byte aligned");
  if (bytes < planner_scratch(B, H, P))
    return fail(AS_ERR_INVALID_ARG, "planner scratch has %zu bytes, needs %zu", bytes, planner_scratch(B, H, P));
  return AS_OK;
}

// selection from ASE values per (i, G) unit (groups of g KV partitions, ase
// [P][NG]): |i-j| <= window fresh; the units are the groups with a member
// outside the window; the floor(R * count) units with the smallest ASE (ties
// by (i, G)) have their remote members reused, the others stored
void select_plan(const double* ase, int P, int g, int window, double ratio, uint8_t* plan) {
  const int NG = (P + g - 1) / g;
  std::vector<std::tuple<double, int, int>> units;
  for (int i = 0; i < P; ++i) {
    for (int j = 0; j < P; ++j)
      plan[i * P + j] = std::abs(i - j) <= window ? AS_PLAN_FRESH : AS_PLAN_FRESH_STORE;
    for (int G = 0; G < NG; ++G) {
      bool remote = false;
      for (int j = G * g; j < std::min((G + 1) * g, P); ++j) remote |= std::abs(i - j) > window;
      if (remote) units.emplace_back(ase[i * NG + G], i, G);
    }
  }
  std::sort(units.begin(), units.end());
  const size_t n_reuse = static_cast<size_t>(std::floor(ratio * static_cast<double>(units.size()) + 1e-9));
  for (size_t x = 0; x < n_reuse && x < units.size(); ++x) {
    const int i = std::get<1>(units[x]), G = std::get<2>(units[x]);
    for (int j = G * g; j < std::min((G + 1) * g, P); ++j)
      if (std::abs(i - j) > window) plan[i * P + j] = AS_PLAN_REUSE;
  }
}

void anchor_plan(int P, int window, uint8_t* plan) {
  for (int i = 0; i < P; ++i)
    for (int j = 0; j < P; ++j) plan[i * P + j] = std::abs(i - j) <= window ? AS_PLAN_FRESH : AS_PLAN_FRESH_STORE;
}

// drift and anchor norms of every partition, host values
as_status run_drift(const float* now, const float* anchor, int B, int H, int S, int d, int P, void* scratch,
                    cudaStream_t st, double* h_sums /*[P][2]*/) {
  double* partials = static_cast<double*>(scratch);
  double* sums = partials + static_cast<size_t>(P) * P * B * H * 2;
  cudaError_t e = asp::launch_drift(now, anchor, B * H, S, d, P, partials, sums, st);
  if (e != cudaSuccess) return cuda_fail(e, "drift launch");
  e = cudaMemcpyAsync(h_sums, sums, static_cast<size_t>(P) * 2 * sizeof(double), cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "drift copy");
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "drift sync");
  return AS_OK;
}

// the drift reduction reads both tensors with 16-byte loads
as_status check_drift_inputs(const float* now, const float* anchor) {
  if (!aligned16(now) || !aligned16(anchor))
    return fail(AS_ERR_INVALID_ARG, "local-state tensors must be 16-byte aligned");
  return AS_OK;
}

as_status check_planner(const as_planner* pl) {
  if (!pl || pl->magic != PLANNER_MAGIC) return fail(AS_ERR_INVALID_ARG, "planner not initialised by as_planner_init");
  return AS_OK;
}

as_status check_cache(const as_cache* c) {
  if (!c || c->magic != CACHE_MAGIC) return fail(AS_ERR_INVALID_ARG, "cache not initialised by as_cache_init");
  return AS_OK;
}

}  // namespace

extern "C" {

const char* as_last_error(void) { return g_err.c_str(); }

const char* as_version(void) {
  return ASP_CHECKED_BUILD ? "attention-state-reuse-partition b200 0.2 (sm_100a, checked)"
                           : "attention-state-reuse-partition b200 0.2 (sm_100a)";
}

as_status as_partition_attn(const void* q, const void* k, const void* v, as_dtype dt, int B, int H, int S, int d,
                            int P, float scale, int q_part, const int32_t* h_kv_parts, int n_kv_parts, int compose,
                            float* out, float* lse, void* stream) {
  Range nvtx_range("as_partition_attn");
  as_status s = check_shape(B, H, S, d, P);
  if (s != AS_OK) return s;
  if (dt != AS_F32 && dt != AS_BF16) return fail(AS_ERR_INVALID_ARG, "unknown dtype %d", static_cast<int>(dt));
  if (!q || !k || !v || !out || !lse) return fail(AS_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(AS_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (q_part < -1 || q_part >= P) return fail(AS_ERR_INVALID_ARG, "q_part %d out of [-1, %d)", q_part, P);
  if (!h_kv_parts || n_kv_parts < 1 || n_kv_parts > P)
    return fail(AS_ERR_INVALID_ARG, "need 1..P KV partitions (got %d)", n_kv_parts);
  if (compose != 0 && compose != 1) return fail(AS_ERR_INVALID_ARG, "compose must be 0 or 1");
  if (!(scale > 0.f)) return fail(AS_ERR_INVALID_ARG, "scale must be > 0");
  asp::AttnLaunch L;
  base_launch(L, q, k, v, B, H, S, d, P, scale);
  const int R = q_part >= 0 ? S / P : S;
  L.n_blocks = 1;
  L.block_rows = R;
  L.block_row0 = q_part >= 0 ? q_part * (S / P) : 0;
  for (int x = 0; x < n_kv_parts; ++x) {
    const int j = h_kv_parts[x];
    if (j < 0 || j >= P) return fail(AS_ERR_INVALID_ARG, "KV partition %d out of [0, %d)", j, P);
    if (L.code[j] != AS_KCODE_SKIP) return fail(AS_ERR_INVALID_ARG, "KV partition %d listed twice", j);
    L.code[j] = compose ? AS_KCODE_COMPOSE : AS_KCODE_EMIT;
    L.dest_of[j] = static_cast<int8_t>(x);
  }
  L.out = out;
  L.lse = lse;
  L.out_rows = R;
  L.out_row0 = L.block_row0;
  L.dst_out = out;
  L.dst_lse = lse;
  L.dst_rows = R;
  L.dst_row0 = L.block_row0;
  L.dst_plane_out = static_cast<long long>(B) * H * R * d;
  L.dst_plane_lse = static_cast<long long>(B) * H * R;
  L.dst_planes = compose ? 1 : n_kv_parts;
  if ((s = check_device()) != AS_OK) return s;
  if ((s = launch_attn(L, dt, static_cast<cudaStream_t>(stream))) != AS_OK) return s;
  return ok();
}

as_status as_compose(const float* outs, const float* lses, int n_states, int64_t rows, int d,
                     int64_t state_stride_out, int64_t state_stride_lse, float* out, float* lse, void* stream) {
  Range nvtx_range("as_compose");
  if (d != 64 && d != 128) return fail(AS_ERR_INVALID_ARG, "d must be 64 or 128 (got %d)", d);
  if (n_states < 1) return fail(AS_ERR_INVALID_ARG, "n_states must be >= 1");
  if (rows < 0) return fail(AS_ERR_INVALID_ARG, "rows must be >= 0");
  if (rows == 0) return ok();
  if (!outs || !lses || !out || !lse) return fail(AS_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(outs) || !aligned16(out)) return fail(AS_ERR_INVALID_ARG, "OUT pointers must be 16-byte aligned");
  if (n_states > 1 && (state_stride_out < rows * d || state_stride_lse < rows || (state_stride_out % 4) != 0))
    return fail(AS_ERR_INVALID_ARG, "state strides must cover a whole state (and OUT stride be a multiple of 4)");
  asp::ComposeStrided a;
  a.outs = outs;
  a.lses = lses;
  a.n_states = n_states;
  a.d = d;
  a.rows = rows;
  a.stride_out = state_stride_out;
  a.stride_lse = state_stride_lse;
  a.out = out;
  a.lse = lse;
  as_status s = check_device();
  if (s != AS_OK) return s;
  cudaError_t e = asp::launch_compose_strided(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "compose launch");
  return ok();
}

size_t as_cache_cp_bytes(int B, int H, int S, int d, int P, int g, as_dtype cache_dt, int q_count) {
  if (cache_dt != AS_F32 && cache_dt != AS_BF16) return 0;
  if (check_shape(B, H, S, d, P) != AS_OK || g < 1 || g > P || q_count < 1 || q_count > P) return 0;
  const size_t NG = static_cast<size_t>((P + g - 1) / g);
  const size_t rows = static_cast<size_t>(B) * H * q_count * (S / P);
  return NG * rows * (static_cast<size_t>(d) * (cache_dt == AS_BF16 ? 2 : 4) + sizeof(float));
}

size_t as_cache_group_bytes(int B, int H, int S, int d, int P, int g, as_dtype cache_dt) {
  return as_cache_cp_bytes(B, H, S, d, P, g, cache_dt, P);
}

size_t as_cache_bytes(int B, int H, int S, int d, int P, as_dtype cache_dt) {
  return as_cache_group_bytes(B, H, S, d, P, 1, cache_dt);
}

as_status as_cache_cp_init(as_cache* c, void* buf, size_t bytes, int B, int H, int S, int d, int P, int g,
                           as_dtype cache_dt, int q_first, int q_count) {
  if (!c) return fail(AS_ERR_INVALID_ARG, "null cache struct");
  if (cache_dt != AS_F32 && cache_dt != AS_BF16)
    return fail(AS_ERR_INVALID_ARG, "cache dtype %d is not AS_F32 or AS_BF16", static_cast<int>(cache_dt));
  as_status s = check_shape(B, H, S, d, P);
  if (s != AS_OK) return s;
  if (g < 1 || g > P) return fail(AS_ERR_INVALID_ARG, "group size %d outside [1, %d]", g, P);
  if (q_first < 0 || q_count < 1 || q_first + q_count > P)
    return fail(AS_ERR_INVALID_ARG, "query partitions [%d, %d) outside [0, %d)", q_first, q_first + q_count, P);
  const size_t need = as_cache_cp_bytes(B, H, S, d, P, g, cache_dt, q_count);
  if (!buf || (reinterpret_cast<uintptr_t>(buf) & 255u) != 0)
    return fail(AS_ERR_INVALID_ARG, "cache buffer must be non-null and 256-byte aligned");
  if (bytes < need) return fail(AS_ERR_INVALID_ARG, "cache buffer has %zu bytes, needs %zu", bytes, need);
  std::memset(c, 0, sizeof(*c));
  c->magic = CACHE_MAGIC;
  c->B = B;
  c->H = H;
  c->S = S;
  c->d = d;
  c->P = P;
  c->g = g;
  c->n_groups = (P + g - 1) / g;
  c->cache_dt = cache_dt;
  c->q_first = q_first;
  c->q_count = q_count;
  c->out_planes = buf;
  const size_t out_bytes =
      static_cast<size_t>(c->n_groups) * B * H * q_count * (S / P) * d * (cache_dt == AS_BF16 ? 2 : 4);
  c->lse_planes = reinterpret_cast<float*>(static_cast<char*>(buf) + out_bytes);
  for (int x = 0; x < AS_MAX_P * AS_MAX_P; ++x) c->t_c[x] = -1;
  return ok();
}

as_status as_cache_group_init(as_cache* c, void* buf, size_t bytes, int B, int H, int S, int d, int P, int g,
                              as_dtype cache_dt) {
  return as_cache_cp_init(c, buf, bytes, B, H, S, d, P, g, cache_dt, 0, P);
}

as_status as_cache_init(as_cache* c, void* buf, size_t bytes, int B, int H, int S, int d, int P, as_dtype cache_dt) {
  return as_cache_group_init(c, buf, bytes, B, H, S, d, P, 1, cache_dt);
}

as_status as_plan_resolve(const as_cache* c, const uint8_t* h_plan, int step, uint8_t* h_hit, int32_t* h_age) {
  as_status s = check_cache(c);
  if (s != AS_OK) return s;
  if (!h_plan) return fail(AS_ERR_INVALID_ARG, "null plan");
  if ((s = resolve(c, h_plan, step, h_hit, h_age)) != AS_OK) return s;
  return ok();
}

// K/V layout of a step: kv_rows rows per head in k and v, KV partition j at
// rows [kv_slot[j] * n, (kv_slot[j] + 1) * n) (kv_slot == nullptr: slot j,
// the whole sequence in place)
struct KvLayout {
  int kv_rows;
  const int32_t* kv_slot;
};

// as_step, as_step_local and as_step_cp.  The cache's query partitions
// [q_first, q_first + q_count) are the query rows of q, out and lse
// (q_count * n rows per head); local_out == nullptr: no precomputed local
// states.
static as_status step_impl(as_cache* c, const void* q, const void* k, const void* v, as_dtype dt, float scale,
                           const uint8_t* h_plan, int step, const float* local_out, const float* local_lse,
                           float* out, float* lse, uint8_t* h_hit, int32_t* h_age, void* stream,
                           const KvLayout& kvl, const char* name) {
  Range nvtx_range(name);
  as_status s = check_cache(c);
  if (s != AS_OK) return s;
  if (dt != AS_F32 && dt != AS_BF16) return fail(AS_ERR_INVALID_ARG, "unknown dtype %d", static_cast<int>(dt));
  if (!q || !k || !v || !out || !lse || !h_plan) return fail(AS_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(AS_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (local_out && (!local_lse || !aligned16(local_out) || !aligned16(local_lse)))
    return fail(AS_ERR_INVALID_ARG, "local states must be non-null and 16-byte aligned");
  if (!(scale > 0.f)) return fail(AS_ERR_INVALID_ARG, "scale must be > 0");
  const int B = c->B, H = c->H, S = c->S, d = c->d, P = c->P, n = S / P, g = c->g, NG = c->n_groups;
  const int i0 = c->q_first, nq = c->q_count, Sq = nq * n;
  if (local_out && nq != P)
    return fail(AS_ERR_UNSUPPORTED, "local states need a cache over every query partition");
  uint8_t hit[AS_MAX_P * AS_MAX_P];
  int32_t age[AS_MAX_P * AS_MAX_P];
  if ((s = resolve(c, h_plan, step, hit, age)) != AS_OK) return s;
  // every KV partition the cache's rows compute must be in k / v
  if (kvl.kv_slot) {
    uint64_t used = 0;
    for (int j = 0; j < P; ++j) {
      bool needed = false;
      for (int i = i0; i < i0 + nq; ++i) needed |= h_plan[i * P + j] != AS_PLAN_REUSE;
      const int sl = kvl.kv_slot[j];
      if (sl < 0) {
        if (needed) return fail(AS_ERR_INVALID_ARG, "KV partition %d is computed by the plan but not in the buffer", j);
        continue;
      }
      if (static_cast<long long>(sl + 1) * n > kvl.kv_rows)
        return fail(AS_ERR_INVALID_ARG, "KV partition %d at slot %d lies beyond the buffer's %d rows", j, sl,
                    kvl.kv_rows);
      if (sl >= 64 || (used >> sl) & 1u) return fail(AS_ERR_INVALID_ARG, "KV slot %d given twice (or >= 64)", sl);
      used |= uint64_t(1) << sl;
    }
  }
  if ((s = check_device()) != AS_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // a plain-fresh diagonal pair whose state the caller already holds
  auto local_of = [&](int i) { return local_out != nullptr && h_plan[i * P + i] == AS_PLAN_FRESH; };

  // fresh pairs: composite of the plain-fresh partitions -> out/lse; the
  // stored members of each group -> one composed state in the group's plane.
  // Block b is query partition i0 + b, at local rows [b n, (b + 1) n).
  asp::AttnLaunch L;
  base_launch(L, q, k, v, B, H, S, d, P, scale);
  L.S = Sq;
  L.S_kv = kvl.kv_rows;
  for (int j = 0; j < P; ++j) L.kv_row0[j] = kvl.kv_slot ? std::max(0, kvl.kv_slot[j]) * n : j * n;
  L.n_blocks = nq;
  L.block_rows = n;
  L.block_row0 = 0;
  bool any_fresh = false;
  for (int b = 0; b < nq; ++b) {
    const int i = i0 + b;
    for (int j = 0; j < P; ++j) {
      const uint8_t pc = h_plan[i * P + j];
      uint8_t kc = pc == AS_PLAN_FRESH ? AS_KCODE_COMPOSE : pc == AS_PLAN_FRESH_STORE ? AS_KCODE_EMIT : AS_KCODE_SKIP;
      if (j == i && local_of(i)) kc = AS_KCODE_SKIP;
      L.code[b * P + j] = kc;
      any_fresh |= kc != AS_KCODE_SKIP;
    }
  }
  for (int j = 0; j < P; ++j) L.dest_of[j] = static_cast<int8_t>(j / g);
  // every query partition reads the same KV list: one block of all rows, so
  // query tiles are not cut at partition boundaries
  bool uniform = true;
  for (int b = 1; b < nq && uniform; ++b) uniform = std::memcmp(L.code, L.code + b * P, P) == 0;
  if (uniform) {
    L.n_blocks = 1;
    L.block_rows = Sq;
  }
  L.out = out;
  L.lse = lse;
  L.out_rows = Sq;
  L.out_row0 = 0;
  L.dst_out = c->out_planes;
  L.dst_bf16 = c->cache_dt == AS_BF16;
  L.dst_lse = c->lse_planes;
  L.dst_rows = Sq;
  L.dst_row0 = 0;
  L.dst_plane_out = static_cast<long long>(B) * H * Sq * d;
  L.dst_plane_lse = static_cast<long long>(B) * H * Sq;
  L.dst_planes = NG;
  if (any_fresh && (s = launch_attn(L, dt, st)) != AS_OK) return s;

  // final composition: composite + local state + stored and reused group entries
  asp::ComposePlan a;
  std::memset(&a, 0, sizeof(a));
  bool need_compose = false;
  for (int b = 0; b < nq; ++b) {
    const int i = i0 + b;
    int cnt = 0;
    bool composite = false;
    for (int j = 0; j < P; ++j) composite |= L.code[(uniform ? 0 : b) * P + j] == AS_KCODE_COMPOSE;
    if (composite) a.src[b][cnt++] = -1;
    if (local_of(i)) a.src[b][cnt++] = -2;
    for (int G = 0; G < NG; ++G)
      if (group_mask(h_plan, P, g, i, G, AS_PLAN_REUSE) || group_mask(h_plan, P, g, i, G, AS_PLAN_FRESH_STORE))
        a.src[b][cnt++] = static_cast<int8_t>(G);
    // a row whose only source is the composite already holds its final state
    a.nsrc[b] = (cnt == 1 && composite) ? 0 : static_cast<uint8_t>(cnt);
    need_compose |= a.nsrc[b] > 0;
  }
  if (need_compose) {
    a.B = B;
    a.H = H;
    a.S = Sq;
    a.d = d;
    a.P = nq;
    a.n = n;
    a.cache_out = c->out_planes;
    a.cache_bf16 = c->cache_dt == AS_BF16;
    a.n_planes = NG;
    a.cache_lse = c->lse_planes;
    a.plane_out = L.dst_plane_out;
    a.plane_lse = L.dst_plane_lse;
    a.local_out = local_out;
    a.local_lse = local_lse;
    a.out = out;
    a.lse = lse;
    cudaError_t e = asp::launch_compose_plan(a, st);
    if (e != cudaSuccess) return cuda_fail(e, "step compose launch");
  }

  for (int i = i0; i < i0 + nq; ++i)
    for (int G = 0; G < NG; ++G) {
      const uint64_t m = group_mask(h_plan, P, g, i, G, AS_PLAN_FRESH_STORE);
      if (!m) continue;
      c->t_c[i * NG + G] = step;
      c->member[i * NG + G] = m;
    }
  if (h_hit) std::memcpy(h_hit, hit, static_cast<size_t>(P) * P);
  if (h_age) std::memcpy(h_age, age, static_cast<size_t>(P) * P * sizeof(int32_t));
  return ok();
}

as_status as_step(as_cache* c, const void* q, const void* k, const void* v, as_dtype dt, float scale,
                  const uint8_t* h_plan, int step, float* out, float* lse, uint8_t* h_hit, int32_t* h_age,
                  void* stream) {
  as_status s = check_cache(c);
  if (s != AS_OK) return s;
  if (c->q_count != c->P)
    return fail(AS_ERR_INVALID_ARG, "as_step needs a cache over every query partition; use as_step_cp");
  return step_impl(c, q, k, v, dt, scale, h_plan, step, nullptr, nullptr, out, lse, h_hit, h_age, stream,
                   KvLayout{c->S, nullptr}, "as_step");
}

as_status as_step_local(as_cache* c, const void* q, const void* k, const void* v, as_dtype dt, float scale,
                        const uint8_t* h_plan, int step, const float* local_out, const float* local_lse, float* out,
                        float* lse, uint8_t* h_hit, int32_t* h_age, void* stream) {
  if (!local_out || !local_lse) return fail(AS_ERR_INVALID_ARG, "null local states");
  as_status s = check_cache(c);
  if (s != AS_OK) return s;
  return step_impl(c, q, k, v, dt, scale, h_plan, step, local_out, local_lse, out, lse, h_hit, h_age, stream,
                   KvLayout{c->S, nullptr}, "as_step_local");
}

as_status as_step_cp(as_cache* c, const void* q, const void* k_buf, const void* v_buf, int kv_rows,
                     const int32_t* h_kv_slot, as_dtype dt, float scale, const uint8_t* h_plan, int step, float* out,
                     float* lse, uint8_t* h_hit, int32_t* h_age, void* stream) {
  as_status s = check_cache(c);
  if (s != AS_OK) return s;
  if (!h_kv_slot) return fail(AS_ERR_INVALID_ARG, "null KV slot map");
  if (kv_rows < 1 || static_cast<long long>(kv_rows) * c->d >= (1ll << 31))
    return fail(AS_ERR_INVALID_ARG, "kv_rows must be >= 1 and kv_rows * d < 2^31 (got %d)", kv_rows);
  return step_impl(c, q, k_buf, v_buf, dt, scale, h_plan, step, nullptr, nullptr, out, lse, h_hit, h_age, stream,
                   KvLayout{kv_rows, h_kv_slot}, "as_step_cp");
}

as_status as_device_status(void* stream, uint32_t* h_bits) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "device status");
  unsigned int bits = 0;
  for (auto reader : {asp::dev_error_attn_tc, asp::dev_error_attn_simt, asp::dev_error_compose}) {
    unsigned int b = 0;
    if ((e = reader(&b)) != cudaSuccess) return cuda_fail(e, "device status");
    bits |= b;
  }
  if (h_bits) *h_bits = bits;
  if (bits & AS_DEVERR_TIMEOUT) return fail(AS_ERR_TIMEOUT, "a kernel's bounded wait ran out (bits 0x%x)", bits);
  if (bits & AS_DEVERR_BOUNDS)
    return fail(AS_ERR_BOUNDS, "a checked build's index check failed and skipped its access (bits 0x%x)", bits);
  return ok();
}

as_status as_debug_bounds_probe(float* buf, int64_t n, void* stream) {
  if (!ASP_CHECKED_BUILD) return fail(AS_ERR_UNSUPPORTED, "as_debug_bounds_probe needs the checked build (ASP_DEBUG)");
  if (!buf || n < 0 || !aligned16(buf)) return fail(AS_ERR_INVALID_ARG, "bounds probe: bad buffer");
  as_status s = check_device();
  if (s != AS_OK) return s;
  cudaError_t e = asp::launch_bounds_probe(buf, n, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "bounds probe launch");
  return ok();
}

as_status as_debug_timeout_probe(uint32_t poll_budget, uint32_t limit_ns, void* stream) {
  if (poll_budget < 1) return fail(AS_ERR_INVALID_ARG, "poll_budget must be >= 1");
  if (limit_ns > 4000000000u) return fail(AS_ERR_INVALID_ARG, "limit_ns must be <= 4e9");
  as_status s = check_device();
  if (s != AS_OK) return s;
  cudaError_t e = asp::launch_timeout_probe(poll_budget, limit_ns, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "timeout probe launch");
  return ok();
}

as_status as_planner_group_init(as_planner* pl, int P, int g, int window, double reuse_ratio, double eps_local) {
  if (!pl) return fail(AS_ERR_INVALID_ARG, "null planner");
  if (P < 1 || P > AS_MAX_P) return fail(AS_ERR_INVALID_ARG, "P must be in [1, %d]", AS_MAX_P);
  if (g < 1 || g > P) return fail(AS_ERR_INVALID_ARG, "group size %d outside [1, %d]", g, P);
  if (window < 0) return fail(AS_ERR_INVALID_ARG, "window must be >= 0");
  if (!(reuse_ratio >= 0.0 && reuse_ratio <= 1.0)) return fail(AS_ERR_INVALID_ARG, "reuse_ratio must be in [0, 1]");
  if (!(eps_local >= 0.0)) return fail(AS_ERR_INVALID_ARG, "eps_local must be >= 0");
  std::memset(pl, 0, sizeof(*pl));
  pl->magic = PLANNER_MAGIC;
  pl->P = P;
  pl->window = window;
  pl->reuse_ratio = reuse_ratio;
  pl->eps_local = eps_local;
  pl->g = g;
  return ok();
}

as_status as_planner_init(as_planner* pl, int P, int window, double reuse_ratio, double eps_local) {
  return as_planner_group_init(pl, P, 1, window, reuse_ratio, eps_local);
}

size_t as_planner_scratch_bytes(int B, int H, int P) {
  if (B < 1 || H < 1 || P < 1 || P > AS_MAX_P) return 0;
  return planner_scratch(B, H, P);
}

as_status as_local_states(const void* q, const void* k, const void* v, as_dtype dt, int B, int H, int S, int d,
                          int P, float scale, float* out, float* lse, void* stream) {
  Range nvtx_range("as_local_states");
  as_status s = check_shape(B, H, S, d, P);
  if (s != AS_OK) return s;
  if (dt != AS_F32 && dt != AS_BF16) return fail(AS_ERR_INVALID_ARG, "unknown dtype %d", static_cast<int>(dt));
  if (!q || !k || !v || !out || !lse) return fail(AS_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(lse))
    return fail(AS_ERR_INVALID_ARG, "device pointers must be 16-byte aligned");
  if (!(scale > 0.f)) return fail(AS_ERR_INVALID_ARG, "scale must be > 0");
  asp::AttnLaunch L;
  base_launch(L, q, k, v, B, H, S, d, P, scale);
  L.n_blocks = P;
  L.block_rows = S / P;
  L.block_row0 = 0;
  for (int i = 0; i < P; ++i) L.code[i * P + i] = AS_KCODE_EMIT;  // block i: its own partition only
  L.out = out;
  L.lse = lse;
  L.out_rows = S;
  L.out_row0 = 0;
  L.dst_out = out;  // every emitted state goes to plane 0 at its own rows
  L.dst_lse = lse;
  L.dst_rows = S;
  L.dst_row0 = 0;
  L.dst_planes = 1;
  if ((s = check_device()) != AS_OK) return s;
  if ((s = launch_attn(L, dt, static_cast<cudaStream_t>(stream))) != AS_OK) return s;
  return ok();
}

as_status as_plan_drift(const float* now, const float* anchor, int B, int H, int S, int d, int P, void* scratch,
                        size_t scratch_bytes, double* h_drift, double* h_norm, void* stream) {
  Range nvtx_range("as_plan_drift");
  as_status s = check_shape(B, H, S, d, P);
  if (s != AS_OK) return s;
  if (!now || !anchor || !h_drift || !h_norm) return fail(AS_ERR_INVALID_ARG, "null pointer");
  if ((s = check_drift_inputs(now, anchor)) != AS_OK) return s;
  if ((s = check_scratch(scratch, scratch_bytes, B, H, P)) != AS_OK) return s;
  if ((s = check_device()) != AS_OK) return s;
  std::vector<double> sums(static_cast<size_t>(P) * 2);
  if ((s = run_drift(now, anchor, B, H, S, d, P, scratch, static_cast<cudaStream_t>(stream), sums.data())) != AS_OK)
    return s;
  for (int i = 0; i < P; ++i) {
    h_drift[i] = std::sqrt(sums[i * 2 + 0]);
    h_norm[i] = std::sqrt(sums[i * 2 + 1]);
  }
  return ok();
}

as_status as_plan_drift_static(const float* now, const float* anchor, int B, int H, int S, int d, int P,
                               double* h_drift, double* h_norm, void* stream) {
  Range nvtx_range("as_plan_drift_static");
  as_status s = check_shape(B, H, S, d, P);
  if (s != AS_OK) return s;
  if (!now || !anchor || !h_drift || !h_norm) return fail(AS_ERR_INVALID_ARG, "null pointer");
  if ((s = check_drift_inputs(now, anchor)) != AS_OK) return s;
  if ((s = check_device()) != AS_OK) return s;
  double* scratch = nullptr;
  size_t capacity = 0;
  cudaError_t e = asp::static_drift_scratch(&scratch, &capacity);
  if (e != cudaSuccess) return cuda_fail(e, "fixed drift scratch address");
  // partials [P][B*H][2] then sums [P][2]; every slot read is written first
  // by the same call, so nothing needs clearing
  const size_t need = static_cast<size_t>(P) * B * H * 2 + static_cast<size_t>(P) * 2;
  if (need > capacity)
    return fail(AS_ERR_INVALID_ARG,
                "as_plan_drift_static: P*(B*H*2 + 2) = %zu doubles exceeds the fixed scratch of %zu doubles; "
                "use as_plan_drift with a caller scratch buffer",
                need, capacity);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  double* partials = scratch;
  double* sums = scratch + static_cast<size_t>(P) * B * H * 2;
  e = asp::launch_drift(now, anchor, B * H, S, d, P, partials, sums, st);
  if (e != cudaSuccess) return cuda_fail(e, "drift launch");
  std::vector<double> h(static_cast<size_t>(P) * 2);
  e = cudaMemcpyAsync(h.data(), sums, h.size() * sizeof(double), cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "drift copy");
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "drift sync");
  for (int i = 0; i < P; ++i) {
    h_drift[i] = std::sqrt(h[i * 2 + 0]);
    h_norm[i] = std::sqrt(h[i * 2 + 1]);
  }
  return ok();
}

as_status as_plan_select_grouped(const double* h_ase, int P, int g, int window, double reuse_ratio,
                                 uint8_t* h_plan) {
  if (!h_ase || !h_plan) return fail(AS_ERR_INVALID_ARG, "null pointer");
  if (P < 1 || P > AS_MAX_P || g < 1 || g > P || window < 0 || !(reuse_ratio >= 0.0 && reuse_ratio <= 1.0))
    return fail(AS_ERR_INVALID_ARG, "bad P, g, window or reuse_ratio");
  select_plan(h_ase, P, g, window, reuse_ratio, h_plan);
  return ok();
}

as_status as_plan_select(const double* h_ase, int P, int window, double reuse_ratio, uint8_t* h_plan) {
  return as_plan_select_grouped(h_ase, P, 1, window, reuse_ratio, h_plan);
}

as_status as_planner_next(as_planner* pl, const float* local_now, float* local_anchor, int B, int H, int S, int d,
                          void* scratch, size_t scratch_bytes, uint8_t* h_plan, int* h_is_anchor, double* h_ase,
                          void* stream) {
  Range nvtx_range("as_planner_next");
  as_status s = check_planner(pl);
  if (s != AS_OK) return s;
  const int P = pl->P;
  if ((s = check_shape(B, H, S, d, P)) != AS_OK) return s;
  if (!local_now || !local_anchor || !h_plan || !h_is_anchor) return fail(AS_ERR_INVALID_ARG, "null pointer");
  if ((s = check_drift_inputs(local_now, local_anchor)) != AS_OK) return s;
  if ((s = check_scratch(scratch, scratch_bytes, B, H, P)) != AS_OK) return s;
  if ((s = check_device()) != AS_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  bool anchor = !pl->has_anchor;
  for (int i = 0; i < P; ++i) pl->drift[i] = pl->rel_drift[i] = 0.0;
  if (!anchor) {
    std::vector<double> sums(static_cast<size_t>(P) * 2);
    if ((s = run_drift(local_now, local_anchor, B, H, S, d, P, scratch, st, sums.data())) != AS_OK) return s;
    double worst = 0.0;
    for (int i = 0; i < P; ++i) {
      pl->drift[i] = std::sqrt(sums[i * 2 + 0]);
      const double nrm = std::sqrt(sums[i * 2 + 1]);
      pl->rel_drift[i] = nrm > 0.0 ? pl->drift[i] / nrm : 0.0;
      worst = std::max(worst, pl->rel_drift[i]);
    }
    anchor = worst > pl->eps_local;
  }
  const int g = pl->g, NG = (P + g - 1) / g;
  if (h_ase) std::memset(h_ase, 0, static_cast<size_t>(P) * NG * sizeof(double));
  if (anchor) {
    anchor_plan(P, pl->window, h_plan);
    const size_t bytes = static_cast<size_t>(B) * H * S * d * sizeof(float);
    cudaError_t e = cudaMemcpyAsync(local_anchor, local_now, bytes, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "anchor local-state copy");
  } else {
    std::vector<double> a(static_cast<size_t>(P) * NG);
    for (int i = 0; i < P; ++i)
      for (int G = 0; G < NG; ++G) a[i * NG + G] = pl->w[i * NG + G] * pl->alpha[i * NG + G] * pl->drift[i];
    select_plan(a.data(), P, g, pl->window, pl->reuse_ratio, h_plan);
    if (h_ase) std::memcpy(h_ase, a.data(), a.size() * sizeof(double));
  }
  *h_is_anchor = anchor ? 1 : 0;
  return ok();
}

as_status as_planner_commit_anchor(as_planner* pl, const as_cache* c, const float* lse_full,
                                   const float* local_anchor, const uint8_t* h_plan, void* scratch,
                                   size_t scratch_bytes, void* stream) {
  Range nvtx_range("as_planner_commit_anchor");
  as_status s = check_planner(pl);
  if (s != AS_OK) return s;
  if ((s = check_cache(c)) != AS_OK) return s;
  const int P = pl->P;
  if (c->P != P) return fail(AS_ERR_INVALID_ARG, "cache and planner disagree on P");
  if (c->g != pl->g)
    return fail(AS_ERR_INVALID_ARG, "cache groups of %d partitions, planner groups of %d", c->g, pl->g);
  if (c->q_count != c->P) return fail(AS_ERR_UNSUPPORTED, "the planner needs a cache over every query partition");
  if (!lse_full || !local_anchor || !h_plan) return fail(AS_ERR_INVALID_ARG, "null pointer");
  if ((s = check_drift_inputs(local_anchor, local_anchor)) != AS_OK) return s;
  const int B = c->B, H = c->H, S = c->S, d = c->d, n = S / P;
  if ((s = check_scratch(scratch, scratch_bytes, B, H, P)) != AS_OK) return s;
  if ((s = check_device()) != AS_OK) return s;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  // units: the (i, G) entries this anchor stored
  const int g = c->g, NG = c->n_groups;
  asp::PlanRows sel;
  std::memset(&sel, 0, sizeof(sel));
  for (int i = 0; i < P; ++i)
    for (int G = 0; G < NG; ++G) sel.v[i * NG + G] = group_mask(h_plan, P, g, i, G, AS_PLAN_FRESH_STORE) ? 1 : 0;
  double* partials = static_cast<double*>(scratch);
  double* sums = partials + static_cast<size_t>(P) * NG * B * H * 2;
  cudaError_t e = asp::launch_anchor_stats(c->out_planes, c->cache_dt == AS_BF16, c->lse_planes, lse_full,
                                           static_cast<long long>(B) * H * S * d, static_cast<long long>(B) * H * S,
                                           P, NG, B * H, S, d, sel, partials, sums, st);
  if (e != cudaSuccess) return cuda_fail(e, "anchor statistics launch");
  std::vector<double> stats(static_cast<size_t>(P) * NG * 2);
  e = cudaMemcpyAsync(stats.data(), sums, stats.size() * sizeof(double), cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return cuda_fail(e, "anchor statistics copy");
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "anchor statistics sync");
  // norms of the anchor's local states (drift of the anchor against itself)
  std::vector<double> norms(static_cast<size_t>(P) * 2);
  if ((s = run_drift(local_anchor, local_anchor, B, H, S, d, P, scratch, st, norms.data())) != AS_OK) return s;
  const double rows = static_cast<double>(B) * H * n;
  for (int i = 0; i < P; ++i) {
    const double local_norm = std::sqrt(norms[i * 2 + 1]);
    for (int G = 0; G < NG; ++G) {
      if (!sel.v[i * NG + G]) continue;
      pl->w[i * NG + G] = stats[(i * NG + G) * 2 + 0] / rows;
      pl->alpha[i * NG + G] = local_norm > 0.0 ? std::sqrt(stats[(i * NG + G) * 2 + 1]) / local_norm : 0.0;
    }
  }
  pl->has_anchor = 1;
  return ok();
}

as_status as_residual_encode(const void* x, void* base, int8_t* codes, float* scales, int64_t rows, int d,
                             void* stream) {
  Range nvtx_range("as_residual_encode");
  if (d != 64 && d != 128) return fail(AS_ERR_INVALID_ARG, "d must be 64 or 128 (got %d)", d);
  if (rows < 0) return fail(AS_ERR_INVALID_ARG, "rows must be >= 0");
  if (rows == 0) return ok();
  if (!x || !base || !codes || !scales) return fail(AS_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(x) || !aligned16(base) || !aligned16(codes) || !aligned16(scales))
    return fail(AS_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  as_status s = check_device();
  if (s != AS_OK) return s;
  cudaError_t e = asp::launch_residual_encode(x, base, codes, scales, rows, d, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "residual encode launch");
  return ok();
}

as_status as_residual_decode(const int8_t* codes, const float* scales, void* base, int64_t rows, int d,
                             void* stream) {
  Range nvtx_range("as_residual_decode");
  if (d != 64 && d != 128) return fail(AS_ERR_INVALID_ARG, "d must be 64 or 128 (got %d)", d);
  if (rows < 0) return fail(AS_ERR_INVALID_ARG, "rows must be >= 0");
  if (rows == 0) return ok();
  if (!codes || !scales || !base) return fail(AS_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(base))
    return fail(AS_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  as_status s = check_device();
  if (s != AS_OK) return s;
  cudaError_t e = asp::launch_residual_decode(codes, scales, base, rows, d, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "residual decode launch");
  return ok();
}

as_status as_debug_exp2(const float* x, float* y, int64_t n, int mode, void* stream) {
  if (n < 0 || (mode != 0 && mode != 1) || (n > 0 && (!x || !y)))
    return fail(AS_ERR_INVALID_ARG, "as_debug_exp2: bad arguments");
  if (n == 0) return ok();
  as_status s = check_device();
  if (s != AS_OK) return s;
  cudaError_t e = asp::launch_exp2_probe(x, y, n, mode, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "exp2 probe launch");
  return ok();
}

}  // extern "C"
