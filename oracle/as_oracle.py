"""Float64 CPU oracle for attention states over sequence partitions.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may use it.  It shares no code with
the CUDA path; both sides receive the same inputs from the seeded generators.

It is a plain restatement of what DiTango ("DiTango: Cost-Effective Parallel
Diffusion Generation with Selective Attention State Reuse", arXiv 2607.15650)
computes, as summarised on its pith.science review page:

* attention state (section "What carries the argument"): for a query row and
  a KV partition j, AS(j) = (OUT(j), LSE(j)), the partial attention output of
  the keys of j and the log-sum-exp of their scores;
* composition (Axiom & Free-Parameter Ledger, Eq. 1-2, "standard result from
  FlashAttention/FlashInfer"): states compose associatively and commutatively
  by LSE weighting;
* selective reuse (Core claim; Referee Report, Summary): at a step t the query
  partition i computes fresh states for some KV partitions and reuses cached
  states from an earlier step for the others; the final output is the
  composition of both kinds.

Readings where the page is silent (each is listed in the design notes):
OUT is the *normalised* partial output; logs are natural; the LSE includes the
softmax scale; attention is bidirectional with no mask or bias; partitions are
contiguous, equal and in token order; the empty state is (OUT=0, LSE=-inf); a
plan entry is 0=reuse, 1=fresh, 2=fresh and refresh the cached entry; hit is 1
exactly for reused pairs and age = t - t_c for them (0 otherwise).

Memory-aware merging (review page, "If this is right", second bullet: composed
states "can be merged into coarser groups under memory pressure"; ledger:
group size g = 4/8/16): KV partition j belongs to group j // g, and the cache
holds one composed state per (query partition i, group G) together with the
set of members it was composed from.  A group is refreshed or reused as a
whole; a reuse must name exactly the stored members.  Entries may keep OUT in
bf16 (round to nearest even from fp32); the LSE stays fp32.  A step composes
what the cache holds, so at a store step the stored groups enter the final
state with the cache's precision.

Residual compression of what ranks exchange (CompactFusion, "Accelerating
Parallel Diffusion Model Serving with Residual Compression", arXiv
2507.17511, as its listing page gives the Abstract: compressed step-wise
residuals with lightweight error feedback): see the last section of this
module.

Every pin of this module lives in ``tests/test_oracle.py``.
"""
from __future__ import annotations

import numpy as np

PLAN_REUSE = 0
PLAN_FRESH = 1
PLAN_FRESH_STORE = 2


class CacheMiss(Exception):
    """A plan reuses a pair whose cache entry has never been written, or (with
    groups) reuses a member set other than the one stored."""


class PlanError(Exception):
    """A plan matrix holds a value other than 0, 1 or 2, has a wrong shape, or
    (with groups) both reuses and stores members of one group."""


def round_bf16(x):
    """Round to bfloat16 and back: float64 -> float32 (nearest even), then the
    low 16 bits of the float32 rounded off to nearest even.  Finite inputs."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> np.uint64(16)) & np.uint64(1)
    bits = (bits + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return bits.astype(np.uint32).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# the attention state of one KV partition
# ---------------------------------------------------------------------------

def attention_state(q, k, v, scale):
    """AS = (OUT, LSE) of the query rows ``q`` against the keys ``k``/``v``.

    For a query row q_r: s_m = scale * <q_r, k_m> over the keys m of the
    partition, LSE = ln sum_m exp(s_m), OUT = sum_m exp(s_m - LSE) * v_m.
    Shapes: q [..., nq, d], k and v [..., nk, d]; returns OUT [..., nq, d] and
    LSE [..., nq], float64.  With no keys the state is the empty state.
    (DiTango review, "What carries the argument": AS_t(i) = (OUT_t(i), LSE_t(i)).)
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if k.shape[-2] == 0:
        return empty_state(q.shape[:-1], v.shape[-1])
    s = scale * (q @ np.swapaxes(k, -1, -2))            # [..., nq, nk]
    m = s.max(axis=-1, keepdims=True)                     # shift for exp range only
    e = np.exp(s - m)
    l = e.sum(axis=-1, keepdims=True)
    lse = (m + np.log(l))[..., 0]
    out = (e @ v) / l
    return out, lse


def empty_state(row_shape, d):
    """The neutral element of composition: OUT = 0, LSE = -inf."""
    return np.zeros(tuple(row_shape) + (d,)), np.full(tuple(row_shape), -np.inf)


# ---------------------------------------------------------------------------
# composition (DiTango review, Axiom & Free-Parameter Ledger, Eq. 1-2)
# ---------------------------------------------------------------------------

def compose_pair(a, b):
    """Compose two states: LSE = ln(e^{LSE_a} + e^{LSE_b}),
    OUT = e^{LSE_a - LSE} OUT_a + e^{LSE_b - LSE} OUT_b.  Rows where both
    states are empty stay empty."""
    oa, la = a
    ob, lb = b
    m = np.maximum(la, lb)
    safe_m = np.where(np.isfinite(m), m, 0.0)
    ea = np.exp(la - safe_m)
    eb = np.exp(lb - safe_m)
    tot = ea + eb
    lse = np.where(tot > 0, safe_m + np.log(np.where(tot > 0, tot, 1.0)), -np.inf)
    wa = np.where(tot > 0, ea / np.where(tot > 0, tot, 1.0), 0.0)
    wb = np.where(tot > 0, eb / np.where(tot > 0, tot, 1.0), 0.0)
    out = wa[..., None] * oa + wb[..., None] * ob
    return out, lse


def compose(states):
    """Compose any number of states in one pass (the N-ary form of the binary
    rule; equal to any tree of ``compose_pair`` because composition is
    associative and commutative).  ``states`` is a non-empty sequence of
    (OUT, LSE) with matching shapes."""
    states = list(states)
    outs = np.stack([np.asarray(o, dtype=np.float64) for o, _ in states])  # [N, ..., d]
    lses = np.stack([np.asarray(l, dtype=np.float64) for _, l in states])  # [N, ...]
    m = lses.max(axis=0)
    safe_m = np.where(np.isfinite(m), m, 0.0)
    w = np.exp(lses - safe_m)                                              # [N, ...]
    tot = w.sum(axis=0)
    nz = tot > 0
    lse = np.where(nz, safe_m + np.log(np.where(nz, tot, 1.0)), -np.inf)
    coef = np.where(nz, w / np.where(nz, tot, 1.0), 0.0)
    out = (coef[..., None] * outs).sum(axis=0)
    return out, lse


# ---------------------------------------------------------------------------
# partitions
# ---------------------------------------------------------------------------

def partition_bounds(S, P):
    """Contiguous equal partitions in token order: j covers [j*S/P, (j+1)*S/P)."""
    if P <= 0 or S % P != 0:
        raise ValueError("S must be a positive multiple of P")
    n = S // P
    return [(j * n, (j + 1) * n) for j in range(P)]


def partition_states(q, k, v, scale, P):
    """States of the query rows ``q`` [B,H,nq,d] against every KV partition of
    ``k``/``v`` [B,H,S,d]."""
    S = k.shape[-2]
    return [attention_state(q, k[..., a:b, :], v[..., a:b, :], scale)
            for a, b in partition_bounds(S, P)]


def full_attention(q, k, v, scale):
    """Plain softmax attention over all keys, returned as a state."""
    return attention_state(q, k, v, scale)


# ---------------------------------------------------------------------------
# plan resolution and the state cache
# ---------------------------------------------------------------------------

def n_groups(P, g):
    """Number of KV groups of size g over P partitions (the last may be short)."""
    return (P + g - 1) // g


def resolve_plan(plan, t_c, t, g=1, member=None):
    """Check a plan against the cache timestamps and derive hit and age.

    plan [P,P] uint8 (row i = query partition, column j = KV partition), t_c
    [P, n_groups(P, g)] int (step of the entry's last write, -1 = never
    written), t the current step.  hit[i,j] = 1 for reused pairs, else 0;
    age[i,j] = t - t_c[i, j // g] for reused pairs, else 0.  A reuse of a
    never-written entry raises CacheMiss, and so does a reuse whose member set
    differs from ``member[i][G]`` (the members stored, when given); a group
    with both reused and stored members, or any value other than 0/1/2,
    raises PlanError.  With g = 1 each pair is its own group.
    """
    plan = np.asarray(plan)
    t_c = np.asarray(t_c)
    P = plan.shape[0]
    NG = n_groups(P, g)
    if plan.ndim != 2 or plan.shape != (P, P) or t_c.shape != (P, NG):
        raise PlanError("plan must be [P, P] and t_c [P, n_groups]")
    for i in range(P):
        for j in range(P):
            if int(plan[i, j]) not in (PLAN_REUSE, PLAN_FRESH, PLAN_FRESH_STORE):
                raise PlanError(f"plan[{i},{j}] = {int(plan[i, j])}")
    hit = np.zeros((P, P), dtype=np.uint8)
    age = np.zeros((P, P), dtype=np.int32)

    def members(i, G, code):
        return frozenset(j for j in range(G * g, min((G + 1) * g, P)) if int(plan[i, j]) == code)

    for i in range(P):
        for G in range(NG):
            if members(i, G, PLAN_REUSE) and members(i, G, PLAN_FRESH_STORE):
                raise PlanError(f"group ({i},{G}) both reuses and stores members")
    for i in range(P):
        for G in range(NG):
            reused = members(i, G, PLAN_REUSE)
            if not reused:
                continue
            if t_c[i, G] < 0:
                raise CacheMiss(f"group ({i},{G}) reused before any store")
            if member is not None and reused != member[i][G]:
                raise CacheMiss(f"group ({i},{G}) reuses members {sorted(reused)}, "
                                f"stored {sorted(member[i][G])}")
            for j in reused:
                hit[i, j] = 1
                age[i, j] = t - int(t_c[i, G])
    return hit, age


class StateCache:
    """One cached state per (query partition i, KV group G) for the query rows
    the oracle evaluates, the member set it was composed from, and the step
    t_c of its last write.  g = 1 and cache_dt "f32" give one exact entry per
    pair; cache_dt "bf16" keeps OUT rounded to bf16."""

    def __init__(self, P, g=1, cache_dt="f32"):
        if g < 1 or g > P:
            raise PlanError(f"group size {g} outside [1, {P}]")
        if cache_dt not in ("f32", "bf16"):
            raise PlanError(f"cache dtype {cache_dt}")
        self.P, self.g, self.cache_dt = P, g, cache_dt
        self.NG = n_groups(P, g)
        self.t_c = np.full((P, self.NG), -1, dtype=np.int64)
        self.member = [[frozenset() for _ in range(self.NG)] for _ in range(P)]
        self.entry = {}


def step(cache, q, k, v, plan, t, scale, rows=None):
    """One denoising step's attention under a compute/reuse plan.

    final(i) = compose({AS_t(i,j) : plan[i,j] = fresh}
                       U {C(i,G) : G stored at this step}
                       U {C(i,G) : G reused}),
    where a stored group's entry C(i,G) <- compose({AS_t(i,j) : plan[i,j] =
    fresh-and-store, j in G}) (OUT rounded to the cache dtype), member(i,G)
    <- those j, and t_c(i,G) <- t.  (DiTango review: Core claim and Referee
    Report Summary -- fresh states for near partitions, cached composed
    states from earlier steps for far ones; "If this is right" -- composed
    states merged into coarser groups.)  With g = 1 and an fp32 cache this is
    compose of every pair's fresh state or cached entry.

    q, k, v: [B,H,S,d].  ``rows``: sorted token indices of the query rows to
    evaluate (default all); the same rows must be used at every step of one
    cache.  Returns OUT [B,H,len(rows),d], LSE [B,H,len(rows)], hit, age.
    The plan is validated (and CacheMiss raised) before anything changes.
    """
    q = np.asarray(q, dtype=np.float64)
    S = k.shape[-2]
    P, g = cache.P, cache.g
    n = S // P
    rows = np.arange(S) if rows is None else np.asarray(rows)
    hit, age = resolve_plan(plan, cache.t_c, t, g, cache.member)
    B, H, _, d = q.shape
    out = np.zeros((B, H, len(rows), d))
    lse = np.zeros((B, H, len(rows)))
    bounds = partition_bounds(S, P)
    updates = []
    for i in range(P):
        sel = np.nonzero((rows >= i * n) & (rows < (i + 1) * n))[0]
        if sel.size == 0:
            continue
        qi = q[:, :, rows[sel], :]
        parts = []
        for G in range(cache.NG):
            js = range(G * g, min((G + 1) * g, P))
            to_store = []
            reused = False
            for j in js:
                c = int(plan[i, j])
                if c == PLAN_REUSE:
                    reused = True
                    continue
                a, b = bounds[j]
                st = attention_state(qi, k[..., a:b, :], v[..., a:b, :], scale)
                if c == PLAN_FRESH_STORE:
                    to_store.append(st)
                else:
                    parts.append(st)
            if reused:
                parts.append(cache.entry[(i, G)])
            if to_store:
                o, l = compose(to_store)
                if cache.cache_dt == "bf16":
                    o = round_bf16(o)
                parts.append((o, l))
                members = frozenset(j for j in js if int(plan[i, j]) == PLAN_FRESH_STORE)
                updates.append(((i, G), (o, l), members))
        o, l = compose(parts)
        out[:, :, sel, :] = o
        lse[:, :, sel] = l
    for key, st, members in updates:
        cache.entry[key] = st
        cache.t_c[key] = t
        cache.member[key[0]][key[1]] = members
    return out, lse, hit, age


def mse(a, b):
    """Mean squared difference, used to report reuse error against full attention."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.mean((a - b) ** 2))


# ---------------------------------------------------------------------------
# the anchor-guided planner (DiTango review: Referee Report major comments
# 1-3 and the Axiom & Free-Parameter Ledger; Eq. 7-10, 12, 13, Algorithm 1)
# ---------------------------------------------------------------------------
# Readings (the page names the quantities but prints few formulas):
# * the importance of KV partition j for query partition i is the softmax of
#   the partitions' LSEs, w(i,j) = mean over the rows r of i (and over b, h)
#   of exp(LSE_ij[r] - LSE_i[r]), taken at an anchor (Eq. 8); sum_j w = 1;
# * the scale ratio is alpha(i,j) = ||OUT_ij||_F / ||OUT_ii||_F at the anchor,
#   the Frobenius norms running over the rows of i, b, h and d (Eq. 9);
# * the local drift is D(i,t) = ||OUT_t(i,i) - OUT_ta(i,i)||_F against the
#   anchor's local state, and delta(i,j,t) = alpha(i,j) * D(i,t) (Eq. 10);
# * ASE(i,j,t) = w(i,j) * delta(i,j,t) (Eq. 7; groups of one pair, Eq. 12);
# * selection (Eq. 13 with the adaptive threshold of Algorithm 1): pairs with
#   |i-j| <= window are always fresh; of the remaining pairs, the
#   floor(R * count) with the smallest ASE are reused (threshold = that
#   order statistic), ties broken by (i, j); the others are fresh and refresh
#   their cache entry;
# * with cache groups (Eq. 12, ASE of a group G_i) the unit is a group's set
#   of remote members: w and alpha come from its composed entry (w of the
#   group is the sum of its members' weights), and the selection above runs
#   over these units;
# * an anchor is taken when no anchor exists or when the relative local drift
#   max_i D(i,t) / ||OUT_ta(i,i)||_F exceeds eps_local; at an anchor every pair
#   is fresh and every remote pair is stored.

def anchor_weights(lse_pairs, lse_full):
    """w(i, j) for one query partition i: lse_pairs [P, ...rows] holds LSE_ij
    for every j, lse_full [...rows] the LSE of the composition."""
    lse_pairs = np.asarray(lse_pairs, dtype=np.float64)
    lse_full = np.asarray(lse_full, dtype=np.float64)
    return np.exp(lse_pairs - lse_full[None]).reshape(lse_pairs.shape[0], -1).mean(axis=1)


def frob(x):
    return float(np.sqrt(np.sum(np.asarray(x, dtype=np.float64) ** 2)))


def scale_ratios(out_pairs, i):
    """alpha(i, j) = ||OUT_ij|| / ||OUT_ii|| for one query partition i;
    out_pairs is a sequence of P states' OUT ([...rows, d] each), entry i the
    local state (Eq. 9)."""
    norms = np.array([frob(o) for o in out_pairs])
    return norms / norms[i]


def local_drift(out_now, out_anchor):
    """(||OUT_t - OUT_ta||_F, ||OUT_ta||_F) of one query partition's local state."""
    return frob(np.asarray(out_now, dtype=np.float64) - np.asarray(out_anchor, dtype=np.float64)), frob(out_anchor)


def ase(w, alpha, drift):
    """ASE(i, j) = w(i, j) * alpha(i, j) * D(i): w, alpha [P, P], drift [P]."""
    return np.asarray(w, dtype=np.float64) * np.asarray(alpha, dtype=np.float64) * \
        np.asarray(drift, dtype=np.float64)[:, None]


def select_plan(ase_ij, window, reuse_ratio, g=1):
    """Plan codes from ASE values (see the readings above).

    With cache groups of g partitions the planner decides per group (Eq. 12:
    ASE of a group G_i): ase_ij is [P, n_groups(P, g)], the units are the
    groups (i, G) with at least one member outside the window, and a unit's
    remote members are reused or stored together; members inside the window
    stay fresh.  g = 1 is the per-pair selection."""
    ase_ij = np.asarray(ase_ij, dtype=np.float64)
    P = ase_ij.shape[0]
    plan = np.full((P, P), PLAN_FRESH_STORE, dtype=np.uint8)
    units = []
    for i in range(P):
        for j in range(P):
            if abs(i - j) <= window:
                plan[i, j] = PLAN_FRESH
        for G in range(n_groups(P, g)):
            if any(abs(i - j) > window for j in range(G * g, min((G + 1) * g, P))):
                units.append((ase_ij[i, G], i, G))
    units.sort()
    n_reuse = int(np.floor(reuse_ratio * len(units) + 1e-9))
    for _, i, G in units[:n_reuse]:
        for j in range(G * g, min((G + 1) * g, P)):
            if abs(i - j) > window:
                plan[i, j] = PLAN_REUSE
    return plan


def anchor_plan(P, window):
    """Every pair fresh; every pair outside the window stored."""
    i = np.arange(P)[:, None]
    j = np.arange(P)[None, :]
    return np.where(np.abs(i - j) <= window, PLAN_FRESH, PLAN_FRESH_STORE).astype(np.uint8)


class Planner:
    """The planner's state between steps: the anchor's w, alpha and local
    states (OUT_ta(i,i) for every i, [B,H,S,d])."""

    def __init__(self, P, window, reuse_ratio, eps_local, g=1):
        self.P, self.window, self.g = P, window, g
        self.reuse_ratio, self.eps_local = reuse_ratio, eps_local
        self.has_anchor = False
        self.w = np.zeros((P, n_groups(P, g)))
        self.alpha = np.zeros((P, n_groups(P, g)))
        self.local_anchor = None


def planner_next(pl, local_now, n):
    """Plan of the next step from the current local states (OUT_t(i,i) for
    every i, [B,H,S,d] with partition i at rows [i n, (i+1) n)).  Returns
    (plan, is_anchor, drift [P], ase [P,P] or None)."""
    P = pl.P
    if not pl.has_anchor:
        pl.local_anchor = np.array(local_now, dtype=np.float64, copy=True)
        return anchor_plan(P, pl.window), True, np.zeros(P), None
    drift = np.zeros(P)
    rel = np.zeros(P)
    for i in range(P):
        dd, nrm = local_drift(local_now[..., i * n:(i + 1) * n, :], pl.local_anchor[..., i * n:(i + 1) * n, :])
        drift[i] = dd
        rel[i] = dd / nrm if nrm > 0 else 0.0
    if rel.max() > pl.eps_local:
        pl.local_anchor = np.array(local_now, dtype=np.float64, copy=True)
        return anchor_plan(P, pl.window), True, drift, None
    a = ase(pl.w, pl.alpha, drift)
    return select_plan(a, pl.window, pl.reuse_ratio, pl.g), False, drift, a


def planner_commit_anchor(pl, cache, lse_full, rows_of, n):
    """After an anchor step: w and alpha of every stored entry (a pair, or a
    group of remote members: its composed state stands for the group, Eq. 12)
    from the cache entries, the composed LSE and the anchor's local states.
    ``rows_of(i)`` gives the positions, within the evaluated rows, of
    partition i's rows (the same rows the cache entries hold)."""
    P = pl.P
    for i in range(P):
        sel = rows_of(i)
        local = pl.local_anchor[..., i * n:(i + 1) * n, :]
        lse_i = np.asarray(lse_full)[..., sel]
        for G in range(n_groups(P, pl.g)):
            if (i, G) not in cache.entry or cache.t_c[i, G] < 0:
                continue
            o, l = cache.entry[(i, G)]
            # Eq. 8 and Eq. 9 for the one entry: the entry against the
            # composed LSE, and its norm against the local state's
            pl.w[i, G] = float(anchor_weights(np.asarray(l)[None], lse_i)[0])
            pl.alpha[i, G] = float(scale_ratios([local, o], 0)[1])
    pl.has_anchor = True


# ---------------------------------------------------------------------------
# residual compression of what crosses a link (CompactFusion, arXiv
# 2507.17511, Abstract on its listing page: transmit compressed residuals --
# step-wise activation differences -- with lightweight error feedback against
# error accumulation), applied to the KV partitions that ranks exchange each
# step
# ---------------------------------------------------------------------------
# Readings (the page names the method, not the compressor): the residual of a
# row is taken against the receiver's reconstruction of it, which sender and
# receiver both track (so the compression error of a step is carried into the
# next residual: the error feedback); a row of d values is compressed to d
# int8 codes and one fp32 scale, s = max|r| / 127, q = round-half-even(r *
# (127 / max|r|)) clamped to [-127, 127]; the reconstruction is rounded to
# bf16 (the attention inputs' type) after adding q * s.  Every operation is
# taken in float32, each product and sum rounded on its own, as the kernel
# takes them: the codes are integers decided by floating point, so both sides
# decide them in the same precision.

def residual_apply(base, q, s):
    """x_hat = bf16(base + q * s) for rows of d values: base [..., d] (bf16
    values), q [..., d] int8, s [...] float32."""
    prod = (np.asarray(q).astype(np.float32) * np.asarray(s, dtype=np.float32)[..., None]).astype(np.float32)
    tot = (np.asarray(base, dtype=np.float32) + prod).astype(np.float32)
    return round_bf16(tot)


def residual_encode(x, base):
    """Compress the rows of x [..., d] against the reconstruction `base`
    (both bf16 values): returns (q int8 [..., d], s float32 [...], the new
    reconstruction residual_apply(base, q, s))."""
    r = (np.asarray(x, dtype=np.float32) - np.asarray(base, dtype=np.float32)).astype(np.float32)
    amax = np.max(np.abs(r), axis=-1).astype(np.float32)
    nz = amax > 0
    inv = np.where(nz, np.float32(127.0) / np.where(nz, amax, np.float32(1.0)), np.float32(0.0)).astype(np.float32)
    q = np.clip(np.rint((r * inv[..., None]).astype(np.float32)), -127, 127).astype(np.int8)
    s = (amax / np.float32(127.0)).astype(np.float32)
    return q, s, residual_apply(base, q, s)
