/* Attention states over sequence partitions, with cached-state reuse: C ABI.
 *
 * The operations follow DiTango ("DiTango: Cost-Effective Parallel Diffusion
 * Generation with Selective Attention State Reuse", arXiv 2607.15650), as
 * summarised on its pith.science review page:
 *   - "What carries the argument": for a sequence (KV) partition j the
 *     attention state is AS(j) = (OUT(j), LSE(j)), the partial attention
 *     output of j's keys and the log-sum-exp of their scores;
 *   - Axiom & Free-Parameter Ledger, Eq. 1-2: states compose associatively and
 *     commutatively by LSE weighting;
 *   - Core claim and Referee Report "Summary": at a denoising step, fresh
 *     states are computed for some partitions and cached composed states from
 *     earlier steps are reused for the others, under a per-(query partition,
 *     KV partition) compute/reuse plan; anchor steps compute every state.
 *
 * Conventions for every call:
 *   - Tensors are row-major.  Q, K, V are [B, H, S, d] (d contiguous); a state
 *     is OUT [.., S, d] fp32 (normalised partial output) and LSE [.., S] fp32
 *     (natural log, softmax scale included).  The empty state is OUT = 0,
 *     LSE = -inf.
 *   - Partition j covers tokens [j*n, (j+1)*n) with n = S / P.  Query
 *     partitions use the same split.  Attention is bidirectional (no mask).
 *   - Pointers without an h_ prefix are device pointers; h_ pointers are host
 *     memory.  The caller owns all memory.  The library allocates no device
 *     memory and does not synchronise the caller's stream; results follow
 *     stream order on `stream` (a cudaStream_t, NULL = legacy default stream).
 *   - Device pointers must be 16-byte aligned.  Supported: d in {64, 128},
 *     1 <= P <= AS_MAX_P, S % P == 0, B*H <= 65535.
 *   - Every call returns an as_status; on failure as_last_error() gives a
 *     message (thread-local).  Argument errors are reported before any launch.
 */
#ifndef AS_PARTITION_H
#define AS_PARTITION_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define AS_MAX_P 64

typedef enum {
  AS_OK = 0,
  AS_ERR_INVALID_ARG = 1,  /* shapes, alignment, plan values, cache mismatch */
  AS_ERR_UNSUPPORTED = 2,  /* valid request outside the built paths */
  AS_ERR_CACHE_MISS = 3,   /* the plan reuses an entry never stored, or other members than stored */
  AS_ERR_CUDA = 4,         /* a CUDA runtime call failed (message in as_last_error) */
  AS_ERR_TIMEOUT = 5,      /* a kernel's bounded wait ran out (see as_device_status) */
  AS_ERR_BOUNDS = 6        /* checked build only: a device index check failed (see as_device_status) */
} as_status;

typedef enum {
  AS_F32 = 0,   /* fp32 inputs: CUDA-core path */
  AS_BF16 = 1   /* bf16 inputs, fp32 accumulation and states: tensor-core path */
} as_dtype;

/* plan codes for as_step (uint8 per (query partition i, KV partition j)) */
#define AS_PLAN_REUSE 0        /* read the cached state of (i, j) */
#define AS_PLAN_FRESH 1        /* compute the state of (i, j); cache untouched */
#define AS_PLAN_FRESH_STORE 2  /* compute the state of (i, j) and refresh its cache entry */

/* Message of the last failed call on this thread ("" if none). */
const char* as_last_error(void);

/* Library version string. */
const char* as_version(void);

/* Attention states of one query partition (or of all query rows) against a
 * list of KV partitions.  DiTango review, "What carries the argument" (the
 * state) and Eq. 1-2 (composition).
 *
 *   q, k, v       [B,H,S,d] of type dt.
 *   scale         softmax scale (scores are scale * <q, k>).
 *   q_part        query partition i in [0, P), or -1 for all S query rows.
 *   h_kv_parts    host array of n_kv_parts distinct KV partition indices.
 *   compose = 1:  one state per query row, the composition of the listed
 *                 partitions' states: out [B,H,R,d], lse [B,H,R] with R = n
 *                 (q_part >= 0) or S (q_part = -1).
 *   compose = 0:  one state per listed partition: out [n_kv_parts,B,H,R,d],
 *                 lse [n_kv_parts,B,H,R]; plane k holds h_kv_parts[k].
 * Errors: AS_ERR_INVALID_ARG for a bad shape, index, duplicate or alignment;
 * AS_ERR_CUDA if the launch fails. */
as_status as_partition_attn(const void* q, const void* k, const void* v, as_dtype dt,
                            int B, int H, int S, int d, int P, float scale,
                            int q_part, const int32_t* h_kv_parts, int n_kv_parts, int compose,
                            float* out, float* lse, void* stream);

/* Compose n_states states per row into one (DiTango review, Eq. 1-2).
 *   State k, row r: OUT at outs + k*state_stride_out + r*d, LSE at
 *   lses + k*state_stride_lse + r (strides in elements).  rows >= 0.
 *   out [rows, d], lse [rows].  out/lse must not overlap the inputs.
 * Rows whose states are all empty come out empty (OUT = 0, LSE = -inf). */
as_status as_compose(const float* outs, const float* lses, int n_states, int64_t rows, int d,
                     int64_t state_stride_out, int64_t state_stride_lse,
                     float* out, float* lse, void* stream);

/* State cache.  KV partitions are merged into groups of g consecutive
 * partitions (group G = {j : j / g = G}, n_groups = ceil(P / g); the last
 * group may be short), following DiTango's memory-aware state merging
 * (review page, "If this is right", second bullet: composed states "can be
 * merged into coarser groups under memory pressure"; Axiom & Free-Parameter
 * Ledger: group size g = 4/8/16).  The cache holds one composed state per
 * (query partition i, group G): the composition of the states of the members
 * stored at its last refresh.  g = 1 gives one entry per (i, j) pair.
 *
 * Storage, in one caller-owned device buffer: OUT planes [n_groups][B,H,S,d]
 * (fp32, or bf16 rounded to nearest even when cache_dt = AS_BF16), then LSE
 * planes [n_groups][B,H,S] (fp32 always); entry (i, G) is plane G at the rows
 * of partition i.  Host side: t_c[i*n_groups+G] is the step of the entry's
 * last store (-1 = never stored) and member[i*n_groups+G] the bit mask (bit
 * j) of the KV partitions it was composed from.  The struct is caller-owned
 * host memory; initialise it with as_cache_init or as_cache_group_init. */
typedef struct as_cache {
  uint32_t magic;
  int B, H, S, d, P;
  as_dtype cache_dt;  /* type of the OUT planes: AS_F32 or AS_BF16 */
  void* out_planes;   /* device, [n_groups][B,H,S,d] of cache_dt */
  float* lse_planes;  /* device, [n_groups][B,H,S] */
  int32_t t_c[AS_MAX_P * AS_MAX_P];
  int g, n_groups;
  uint64_t member[AS_MAX_P * AS_MAX_P];
  /* the cache's query partitions [q_first, q_first + q_count): every one
   * (0, P) except for one rank of a context-parallel group (as_cache_cp_init);
   * its planes then hold q_count * S/P rows per head instead of S */
  int q_first, q_count;
} as_cache;

/* Bytes of device memory a cache with one entry per pair (g = 1) needs.
 * cache_dt: AS_F32 or AS_BF16 (the type of the OUT entries).  Returns 0 for
 * invalid sizes. */
size_t as_cache_bytes(int B, int H, int S, int d, int P, as_dtype cache_dt);

/* Carve a g = 1 cache out of `buf` (device, >= as_cache_bytes, 256-byte
 * aligned) and mark every entry empty.  No device access happens here. */
as_status as_cache_init(as_cache* c, void* buf, size_t bytes, int B, int H, int S, int d, int P,
                        as_dtype cache_dt);

/* As as_cache_bytes for groups of g partitions (1 <= g <= P):
 * n_groups * B*H*S * (d * sizeof(OUT entry) + 4).  Returns 0 for invalid
 * sizes. */
size_t as_cache_group_bytes(int B, int H, int S, int d, int P, int g, as_dtype cache_dt);

/* As as_cache_init for groups of g partitions.  AS_ERR_INVALID_ARG for g
 * outside [1, P] or a short buffer. */
as_status as_cache_group_init(as_cache* c, void* buf, size_t bytes, int B, int H, int S, int d, int P, int g,
                              as_dtype cache_dt);

/* Check a plan against the cache and derive the reuse bookkeeping, on the host
 * only (no launch, no state change).  h_plan [P*P] row-major (row = query
 * partition), one code per pair.  Per (i, G) the code-0 members are the
 * reused set and the code-2 members the stored set; a group is stored or
 * reused as a whole.  h_hit[i*P+j] = 1 for reused pairs, else 0;
 * h_age[i*P+j] = step - t_c(i, j/g) for reused pairs, else 0.  Checks, in
 * this order: AS_ERR_INVALID_ARG for a code other than 0/1/2, then for a
 * group with both reused and stored members; AS_ERR_CACHE_MISS if a reused
 * group was never stored or its reused set differs from the stored member
 * set. */
as_status as_plan_resolve(const as_cache* c, const uint8_t* h_plan, int step,
                          uint8_t* h_hit, int32_t* h_age);

/* One denoising step's attention under a compute/reuse plan (DiTango review:
 * Core claim; Referee Report, Summary).
 *   C(i,G) <- compose({AS_step(i,j) : j in G, plan AS_PLAN_FRESH_STORE})
 *             for every group with stored members (OUT rounded to the
 *             cache type), member(i,G) <- those j, t_c(i,G) <- step;
 *   final(i) = compose({AS_step(i,j) : plan AS_PLAN_FRESH}
 *                      U {C(i,G) : G stored or reused by row i})
 * written to out [B,H,S,d], lse [B,H,S].  Entries are written on the device in
 * stream order; t_c and member change on the host at return.  With g = 1 and
 * fp32 entries this is compose over every pair's fresh state or cached
 * entry.  h_hit / h_age (may be NULL) as in as_plan_resolve.  The plan is
 * checked before any launch: on AS_ERR_CACHE_MISS or AS_ERR_INVALID_ARG
 * nothing is launched and the cache is unchanged.  The cache must have been
 * initialised for the same B, H, S, d, P, over every query partition
 * (AS_ERR_INVALID_ARG otherwise; one rank's cache goes to as_step_cp): q, k,
 * v are read and out, lse written with the cache's sizes, which the library
 * cannot check against the caller's buffers (the Python binding does).  The call neither allocates nor
 * synchronises, so it can be captured in a CUDA graph: a replay repeats the
 * device work with the captured plan and pointers, while the host
 * bookkeeping (checks, hit/age, t_c, member) happens once, at the captured
 * call; capture steps that store nothing, or account for that yourself. */
as_status as_step(as_cache* c, const void* q, const void* k, const void* v, as_dtype dt, float scale,
                  const uint8_t* h_plan, int step, float* out, float* lse,
                  uint8_t* h_hit, int32_t* h_age, void* stream);

/* as_step for a caller that already holds the step's local states
 * AS_step(i,i) (as_local_states on the same q, k, v and scale, which the
 * anchor-guided planner computes every step to measure its drift).  Every
 * diagonal pair the plan marks AS_PLAN_FRESH is composed from local_out
 * [B,H,S,d] / local_lse [B,H,S] (fp32, device, 16-byte aligned) instead of
 * being recomputed; everything else is as_step's.  The review page
 * ("Circularity Check", on Eq. 10) describes the local state as the one
 * computed at every step; this entry point keeps it from being computed
 * twice. */
as_status as_step_local(as_cache* c, const void* q, const void* k, const void* v, as_dtype dt, float scale,
                        const uint8_t* h_plan, int step, const float* local_out, const float* local_lse,
                        float* out, float* lse, uint8_t* h_hit, int32_t* h_age, void* stream);

/* ---------------------------------------------------------------------------
 * Context parallelism: one rank of a group that splits the P partitions by
 * query partition (DiTango review page: Referee Report "Summary", group-wise
 * KV transfer across GPUs; "Core claim", cached states stand in for far
 * partitions, so a reused pair needs no KV transfer).  The rank owns query
 * partitions [q_first, q_first + q_count) and their cache entries; before a
 * step it fetches (by its own collectives) only the K/V partitions that its
 * rows of the plan compute fresh, into a compact buffer.
 * ------------------------------------------------------------------------ */

/* Bytes of a cache for q_count query partitions (1 <= q_count <= P):
 * n_groups * B*H*q_count*(S/P) * (d * sizeof(OUT entry) + 4).  0 for invalid
 * sizes. */
size_t as_cache_cp_bytes(int B, int H, int S, int d, int P, int g, as_dtype cache_dt, int q_count);

/* As as_cache_group_init for the query partitions [q_first, q_first +
 * q_count) of a sequence of S rows in P partitions: OUT planes
 * [n_groups][B,H,q_count*S/P,d], LSE planes [n_groups][B,H,q_count*S/P],
 * entry (i, G) at the local rows of partition i ((i - q_first) * S/P).
 * AS_ERR_INVALID_ARG if the run leaves [0, P). */
as_status as_cache_cp_init(as_cache* c, void* buf, size_t bytes, int B, int H, int S, int d, int P, int g,
                           as_dtype cache_dt, int q_first, int q_count);

/* as_step for the rank that owns the cache's query partitions.
 *   q, out [B,H,q_count*S/P,d] and lse [B,H,q_count*S/P]: the rank's query
 *   rows (partition q_first at local row 0).  k_buf, v_buf [B,H,kv_rows,d]
 *   (dt, device, 16-byte aligned): KV partition j at rows
 *   [h_kv_slot[j] * S/P, (h_kv_slot[j] + 1) * S/P) when h_kv_slot[j] >= 0
 *   (host int32 [P]; -1 = not in the buffer).
 *   h_plan is the group's [P*P] plan; only rows q_first .. q_first+q_count-1
 *   are read beyond their codes, and h_hit / h_age are 0 in the other rows.
 * Errors, before any launch: AS_ERR_INVALID_ARG if a pair of the rank's rows
 * with code 1 or 2 names a KV partition that is not in the buffer, if a slot
 * lies beyond kv_rows or is given twice; then as as_step.  The result equals
 * as_step's rows for those partitions on the whole sequence. */
as_status as_step_cp(as_cache* c, const void* q, const void* k_buf, const void* v_buf, int kv_rows,
                     const int32_t* h_kv_slot, as_dtype dt, float scale, const uint8_t* h_plan, int step, float* out,
                     float* lse, uint8_t* h_hit, int32_t* h_age, void* stream);

/* Residual compression of what a rank sends (CompactFusion, "Accelerating
 * Parallel Diffusion Model Serving with Residual Compression", arXiv
 * 2507.17511, Abstract on its listing page: transmit compressed step-wise
 * residuals, with lightweight error feedback against error accumulation).
 * Applied to the KV partitions of the context-parallel exchange (cp.py):
 * sender and receiver each keep the receiver's reconstruction `base` of a
 * partition's rows, and from the second send on only the coded residual
 * crosses the link: d int8 codes and one fp32 scale per row instead of d
 * bf16 values (132 against 256 bytes at d = 128).
 *   Per row of d values (x, base: bf16; all float32 arithmetic, each product
 *   and sum rounded on its own): r = x - base, s = max|r| / 127,
 *   q = round-half-even(r * (127 / max|r|)) clamped to [-127, 127] (q = 0,
 *   s = 0 for a zero residual), base <- bf16(base + q * s) (round to
 *   nearest even).  Because the residual is taken against the reconstruction,
 *   a step's coding error enters the next step's residual: the error
 *   feedback; |x - base| <= s/2 plus the bf16 rounding after every step.
 * x, base [rows, d] bf16; codes [rows, d] int8; scales [rows] fp32; all
 * device, 16-byte aligned; d in {64, 128}.  Stream-ordered, no allocation.
 * AS_ERR_INVALID_ARG for other d, negative rows, null or misaligned
 * pointers (rows = 0 is a no-op). */
as_status as_residual_encode(const void* x, void* base, int8_t* codes, float* scales, int64_t rows, int d,
                             void* stream);

/* The receiver's half: base <- bf16(base + q * s) for every row, exactly as
 * as_residual_encode moved the sender's copy.  Same arguments and errors. */
as_status as_residual_decode(const int8_t* codes, const float* scales, void* base, int64_t rows, int d,
                             void* stream);

/* Synchronise `stream`, then read and clear the device error word that the
 * kernels' bounded waits set.  *h_bits receives the raw bits (may be NULL).
 * Returns AS_ERR_TIMEOUT if a wait ran out since the last call, AS_ERR_BOUNDS
 * if a checked build's index check failed, else AS_OK.
 *   Every wait inside the attention kernel is bounded by 1 s of the GPU's
 *   %globaltimer.  A CTA whose pipeline stops therefore gives up at most 1 s
 *   after its wait began, then waits (again at most 1 s each, three at most)
 *   for the copies and MMAs it already issued, frees its TMEM and exits: the
 *   launch ends at most about 4 s after the stall, and this call then
 *   reports AS_ERR_TIMEOUT. */
as_status as_device_status(void* stream, uint32_t* h_bits);

/* The checked build.  `python -m attention_state_reuse_partition_b200.build`
 * also builds libasp_debug.so with ASP_DEBUG=1 (the Python binding loads it
 * when the environment sets ASP_DEBUG=1; as_version then ends in "checked").
 * compute-sanitizer being closed on the GPU pool this library targets, its
 * kernels check, before each store whose index comes from a launch's
 * arguments, that the index lies inside its destination (the attention
 * epilogues' destination plane and rows, the step compose's source planes);
 * a failed check skips the access and sets a bit that as_device_status
 * reports as AS_ERR_BOUNDS.  The normal build compiles the checks away.
 *
 * Test hook of the checked build: one thread writes buf[n], one past a
 * logical length n, behind the index check, which must refuse it.  Give buf
 * more than n floats, so that even a missing check writes inside the
 * allocation.  AS_ERR_UNSUPPORTED in the normal build (nothing launched). */
as_status as_debug_bounds_probe(float* buf, int64_t n, void* stream);

/* Test hook for failure detection: launches one CTA that waits on a barrier
 * that nothing completes, with the kernels' wait code and a limit of
 * `poll_budget` rounds of try_wait (>= 1) or `limit_ns` (<= 4e9) nanoseconds
 * of the GPU's %globaltimer, whichever comes first.  The wait runs out, sets the
 * device error word and the kernel returns; the context stays usable.  Read
 * the outcome with as_device_status. */
as_status as_debug_timeout_probe(uint32_t poll_budget, uint32_t limit_ns, void* stream);

/* ---------------------------------------------------------------------------
 * The anchor-guided planner (DiTango review: Referee Report major comments 1-3
 * and the Axiom & Free-Parameter Ledger -- Eq. 7-10, 12, 13, Algorithm 1).
 * Readings of the page:
 *   w(i,j)     = mean over the rows of query partition i (all b, h) of
 *                exp(LSE_ij - LSE_i), measured at an anchor (Eq. 8);
 *   alpha(i,j) = ||OUT_ij||_F / ||OUT_ii||_F at the anchor (Eq. 9);
 *   D(i,t)     = ||OUT_t(i,i) - OUT_ta(i,i)||_F, the local drift (Eq. 10);
 *   ASE(i,j,t) = w(i,j) * alpha(i,j) * D(i,t) (Eq. 7, groups of one pair);
 *   selection  : |i-j| <= window always fresh; of the other pairs, the
 *                floor(R * count) with the smallest ASE are reused (ties by
 *                (i, j)), the rest fresh and stored (Eq. 13, Algorithm 1);
 *   anchor     : when there is none yet, or max_i D(i,t)/||OUT_ta(i,i)||_F >
 *                eps_local; every pair fresh, every pair outside the window
 *                stored.
 *   groups     : with cache groups of g partitions the planner decides per
 *                group (Eq. 12, ASE of a group G_i): the unit (i, G) is the
 *                set of G's members outside the window, w(i,G) and
 *                alpha(i,G) come from its composed entry (w(i,G) is the sum of
 *                its members' weights), the selection runs over the units,
 *                and a unit's remote members are reused or stored together.
 *                g = 1 is the per-pair planner.
 * A step with the planner:
 *   as_local_states(q,k,v,...) -> local_now            (device)
 *   as_planner_next(pl, local_now, local_anchor, ...)  -> plan, is_anchor
 *   as_step(cache, q,k,v, plan, ...)                   -> out, lse
 *   if is_anchor: as_planner_commit_anchor(pl, cache, lse, local_anchor, plan, ...)
 * ------------------------------------------------------------------------- */
typedef struct as_planner {
  uint32_t magic;
  int P, window;
  double reuse_ratio, eps_local;
  int has_anchor;
  double w[AS_MAX_P * AS_MAX_P];      /* w(i,G) of the last anchor at [i*n_groups+G] */
  double alpha[AS_MAX_P * AS_MAX_P];  /* alpha(i,G) of the last anchor */
  double drift[AS_MAX_P];             /* D(i,t) of the last as_planner_next (0 at anchors) */
  double rel_drift[AS_MAX_P];         /* D(i,t) / ||OUT_ta(i,i)||_F */
  int g;                              /* cache group size the planner plans for */
} as_planner;

/* window >= 0, 0 <= reuse_ratio <= 1, eps_local >= 0, 1 <= P <= AS_MAX_P;
 * per-pair planning (g = 1). */
as_status as_planner_init(as_planner* pl, int P, int window, double reuse_ratio, double eps_local);

/* As as_planner_init for a cache of groups of g partitions (1 <= g <= P);
 * the cache passed to as_planner_commit_anchor must have the same g. */
as_status as_planner_group_init(as_planner* pl, int P, int g, int window, double reuse_ratio, double eps_local);

/* Bytes of device scratch the planner reductions need (8-byte aligned buffer,
 * caller-owned). */
size_t as_planner_scratch_bytes(int B, int H, int P);

/* The local (diagonal) states AS(i,i) of every query partition i in one
 * launch: out [B,H,S,d], lse [B,H,S], partition i at rows [i n, (i+1) n).
 * Same arguments and errors as as_partition_attn. */
as_status as_local_states(const void* q, const void* k, const void* v, as_dtype dt, int B, int H, int S, int d,
                          int P, float scale, float* out, float* lse, void* stream);

/* For every partition i: h_drift[i] = ||now_i - anchor_i||_F and h_norm[i] =
 * ||anchor_i||_F over its rows (all b, h, d), reduced in fp64 in a fixed
 * order.  now, anchor [B,H,S,d] fp32 device, 16-byte aligned (read with
 * 16-byte loads; AS_ERR_INVALID_ARG otherwise).  Uses `scratch`; synchronises
 * `stream` (the results are host values). */
as_status as_plan_drift(const float* now, const float* anchor, int B, int H, int S, int d, int P, void* scratch,
                        size_t scratch_bytes, double* h_drift, double* h_norm, void* stream);

/* as_plan_drift without a scratch argument, for callers that cannot allocate
 * device memory: a host that owns every device allocation itself and hands
 * this library only fixed, pre-sized buffers, or a loop that must not
 * allocate once running (cudaMalloc may synchronise the device and can fail
 * under memory pressure), and so cannot provide the scratch buffer that
 * as_plan_drift needs.  The paper has no counterpart: this is an interface
 * variant, not a step of the method.
 *   Same arguments, results and synchronisation as as_plan_drift.  The
 *   scratch is a fixed 1 MiB array inside the library (held on every device
 *   that loads it until the process exits); the call allocates nothing.
 *   Limit: P * (B*H*2 + 2) <= 131072 doubles, else AS_ERR_INVALID_ARG with the
 *   sizes in as_last_error().
 *   The first call on a device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   The address is kept for the life of the process: after cudaDeviceReset
 *   on a device (which unloads the library's device code there), do not
 *   call this entry point on that device again in the same process.
 *   local-state pointers must be 16-byte aligned (AS_ERR_INVALID_ARG).
 *   Every call uses the same array and leaves its contents behind; each call
 *   writes every slot it reads, so nothing has to be cleared.  Calls that
 *   overlap on the GPU (different streams, or different host threads on one
 *   device) race on the array: serialise them. */
as_status as_plan_drift_static(const float* now, const float* anchor, int B, int H, int S, int d, int P,
                               double* h_drift, double* h_norm, void* stream);

/* Host-only selection from ASE values h_ase [P*P] (see the readings above). */
as_status as_plan_select(const double* h_ase, int P, int window, double reuse_ratio, uint8_t* h_plan);

/* The same per (i, G) unit for groups of g partitions: h_ase [P*n_groups]
 * (entries of units without a remote member are ignored), h_plan [P*P]. */
as_status as_plan_select_grouped(const double* h_ase, int P, int g, int window, double reuse_ratio,
                                 uint8_t* h_plan);

/* Plan of the next step.  local_now: the step's local states (as_local_states);
 * local_anchor [B,H,S,d]: the planner's copy of the anchor's local states,
 * overwritten (stream-ordered copy) when this step becomes an anchor.  Writes
 * h_plan [P*P], *h_is_anchor, and h_ase [P*n_groups] (may be NULL; zeros at
 * anchors).  local_now and local_anchor must be 16-byte aligned
 * (AS_ERR_INVALID_ARG otherwise).  Synchronises `stream`. */
as_status as_planner_next(as_planner* pl, const float* local_now, float* local_anchor, int B, int H, int S, int d,
                          void* scratch, size_t scratch_bytes, uint8_t* h_plan, int* h_is_anchor, double* h_ase,
                          void* stream);

/* After an anchor step (the as_step that used the anchor plan h_plan):
 * measure w and alpha for every entry (pair or group) the plan stored, from
 * the cache (fp32 or bf16 entries), the step's composed LSE lse_full [B,H,S]
 * and local_anchor (16-byte aligned).  The cache's group size must be the
 * planner's (AS_ERR_INVALID_ARG otherwise).  Synchronises. */
as_status as_planner_commit_anchor(as_planner* pl, const as_cache* c, const float* lse_full,
                                   const float* local_anchor, const uint8_t* h_plan, void* scratch,
                                   size_t scratch_bytes, void* stream);

/* Test hook for the two exp2 evaluations the attention kernel mixes:
 * y[i] = 2^x[i] for n device floats, mode 0 = the FMA-pipe polynomial
 * (range reduction to [-1/2, 1/2], degree-4 minimax fit, relative error
 * <= 3e-6, inputs clamped below at -125), mode 1 = the MUFU ex2.approx. */
as_status as_debug_exp2(const float* x, float* y, int64_t n, int mode, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* AS_PARTITION_H */
