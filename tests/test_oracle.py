"""Pins for the float64 oracle, checked against things other than itself.

Each ``pin_*`` takes the oracle module and raises on a mismatch.  The real
oracle must pass every pin; each planted mistake in ``MUTANTS`` (a dropped
term, a wrong sign, a transposed operand, a wrong index, wrong bookkeeping)
must fail at least one pin, which shows the pins would notice it.

What the pins compare against (none of it is the oracle's own formula):
* pure-Python loops over math.exp on tiny inputs (brute force);
* torch's scaled_dot_product_attention in float64 on the CPU (library);
* scipy.special.logsumexp (library);
* closed forms: zero query (uniform weights), identical keys, a single key,
  equal-LSE halves, the empty state;
* invariants the pages state: composition is associative and commutative
  (DiTango review, Axiom & Free-Parameter Ledger, Eq. 1-2), composing the
  states of all partitions gives full attention, one partition is plain
  attention;
* the hand-computed plan/cache fixture tests/golden/plan_4x4.txt;
* reuse identities: cached states of KV partitions whose inputs did not move
  are exact, so a reuse step then equals full attention over the mixed inputs.
"""
import math

import numpy as np
import pytest
import scipy.special
import torch

from oracle import as_oracle
from tests._golden import load_plan_fixture, load_select_fixture

TOL = 1e-11


def _rng(seed):
    return np.random.default_rng(seed)


def _sdpa(q, k, v, scale):
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), scale=scale)
    return out.numpy()


def _expect_raises(exc, fn, *args, **kw):
    """Like pytest.raises, but a miss is an AssertionError (an Exception), so
    the planted-mistake harness sees it."""
    try:
        fn(*args, **kw)
    except exc:
        return
    raise AssertionError(f"{exc.__name__} not raised")


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    finite = np.isfinite(b)
    assert np.array_equal(np.isfinite(a), finite), f"{what}: finiteness differs"
    assert np.array_equal(a[~finite], b[~finite]), f"{what}: infinities differ"
    err = np.max(np.abs(a[finite] - b[finite])) if finite.any() else 0.0
    assert err <= tol, f"{what}: max abs err {err}"


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------

def pin_bruteforce_loops(o):
    r = _rng(1)
    nq, nk, d = 5, 9, 4
    q, k, v = r.normal(size=(nq, d)), r.normal(size=(nk, d)), r.normal(size=(nk, d))
    scale = 0.7
    out, lse = o.attention_state(q, k, v, scale)
    for a in range(nq):
        scores = [scale * sum(q[a][c] * k[m][c] for c in range(d)) for m in range(nk)]
        z = sum(math.exp(s) for s in scores)
        _close(lse[a], math.log(z), 1e-12, "bruteforce LSE")
        for c in range(d):
            ref = sum(math.exp(scores[m]) / z * v[m][c] for m in range(nk))
            _close(out[a][c], ref, 1e-12, "bruteforce OUT")


def pin_torch_sdpa_full(o):
    r = _rng(2)
    B, H, S, d, P = 2, 3, 40, 16, 5
    q, k, v = (r.normal(size=(B, H, S, d)) for _ in range(3))
    scale = 1 / math.sqrt(d)
    ref = _sdpa(q, k, v, scale)
    out, _ = o.compose(o.partition_states(q, k, v, scale, P))
    _close(out, ref, TOL, "composed vs sdpa")
    out1, _ = o.full_attention(q, k, v, scale)
    _close(out1, ref, TOL, "full vs sdpa")


def pin_scipy_lse(o):
    r = _rng(3)
    q, k, v = r.normal(size=(7, 8)), r.normal(size=(11, 8)), r.normal(size=(11, 8))
    scale = 0.3
    _, lse = o.attention_state(q, k, v, scale)
    for a in range(7):
        scores = np.array([scale * np.dot(q[a], k[m]) for m in range(11)])
        _close(lse[a], scipy.special.logsumexp(scores), 1e-12, "lse vs scipy")


def pin_closed_forms(o):
    r = _rng(4)
    nk, d = 13, 6
    k, v = r.normal(size=(nk, d)), r.normal(size=(nk, d))
    # zero query: uniform weights, LSE = ln nk
    out, lse = o.attention_state(np.zeros((2, d)), k, v, 0.9)
    _close(out, np.tile(v.mean(axis=0), (2, 1)), 1e-12, "zero query OUT")
    _close(lse, np.full(2, math.log(nk)), 1e-12, "zero query LSE")
    # identical keys: LSE = scale<q,k0> + ln nk, OUT = mean v
    q = r.normal(size=(3, d))
    k0 = r.normal(size=d)
    out, lse = o.attention_state(q, np.tile(k0, (nk, 1)), v, 0.5)
    _close(out, np.tile(v.mean(axis=0), (3, 1)), 1e-12, "equal keys OUT")
    _close(lse, 0.5 * (q @ k0) + math.log(nk), 1e-12, "equal keys LSE")
    # a single key: OUT = v0, LSE = score
    out, lse = o.attention_state(q, k0[None, :], v[:1], 0.5)
    _close(out, np.tile(v[0], (3, 1)), 1e-12, "single key OUT")
    _close(lse, 0.5 * (q @ k0), 1e-12, "single key LSE")
    # no keys: the empty state
    out, lse = o.attention_state(q, np.zeros((0, d)), np.zeros((0, d)), 0.5)
    assert np.all(out == 0) and np.all(lse == -np.inf)


def pin_compose_closed(o):
    r = _rng(5)
    oa, ob, oc = (r.normal(size=(4, 3)) for _ in range(3))
    L = r.normal(size=4)
    for f in (lambda a, b: o.compose([a, b]), o.compose_pair):
        out, lse = f((oa, L), (ob, L))
        _close(lse, L + math.log(2), 1e-12, "equal halves LSE")
        _close(out, (oa + ob) / 2, 1e-12, "equal halves OUT")
        out, lse = f((oa, L), (ob, np.full(4, -np.inf)))
        _close(lse, L, 1e-12, "with empty LSE")
        _close(out, oa, 1e-12, "with empty OUT")
        out, lse = f((oa, np.full(4, -np.inf)), (ob, np.full(4, -np.inf)))
        assert np.all(lse == -np.inf) and np.all(out == 0) and not np.isnan(out).any()
    out, lse = o.compose([(oa, L), (ob, L + math.log(2)), (oc, L + math.log(3))])
    _close(lse, L + math.log(6), 1e-12, "1:2:3 LSE")
    _close(out, (oa + 2 * ob + 3 * oc) / 6, 1e-12, "1:2:3 OUT")


def pin_assoc_comm(o):
    r = _rng(6)
    n = 7
    states = [(r.normal(size=(5, 4)), r.normal(size=5) * 3) for _ in range(n)]
    ref_o, ref_l = o.compose(states)
    for trial in range(6):
        perm = r.permutation(n)
        pool = [states[p] for p in perm]
        while len(pool) > 1:
            a = r.integers(len(pool) - 1)
            merged = o.compose_pair(pool[a], pool[a + 1])
            pool[a:a + 2] = [merged]
        _close(pool[0][0], ref_o, TOL, "random tree OUT")
        _close(pool[0][1], ref_l, TOL, "random tree LSE")
        po, pl = o.compose([states[p] for p in perm])
        _close(po, ref_o, TOL, "permuted OUT")
        _close(pl, ref_l, TOL, "permuted LSE")


def pin_split_invariance(o):
    r = _rng(7)
    nk, d = 37, 8
    q, k, v = r.normal(size=(6, d)), r.normal(size=(nk, d)), r.normal(size=(nk, d))
    whole_o, whole_l = o.attention_state(q, k, v, 0.4)
    for trial in range(4):
        cuts = np.sort(r.choice(np.arange(1, nk), size=r.integers(1, 6), replace=False))
        edges = [0] + list(cuts) + [nk]
        parts = [o.attention_state(q, k[a:b], v[a:b], 0.4) for a, b in zip(edges[:-1], edges[1:])]
        po, pl = o.compose(parts)
        _close(po, whole_o, TOL, "split OUT")
        _close(pl, whole_l, TOL, "split LSE")


def pin_single_partition(o):
    r = _rng(8)
    q, k, v = (r.normal(size=(1, 2, 24, 8)) for _ in range(3))
    (out, _), = o.partition_states(q, k, v, 0.35, 1)
    _close(out, _sdpa(q, k, v, 0.35), TOL, "P=1 vs sdpa")


def pin_plan_golden(o):
    P, cases = load_plan_fixture()
    r = _rng(9)
    S, d = 2 * P, 3
    q, k, v = (r.normal(size=(1, 1, S, d)) for _ in range(3))
    cache = o.StateCache(P)
    for c in cases:
        if c["expect"] == "cache_miss":
            before = cache.t_c.copy()
            _expect_raises(o.CacheMiss, o.step, cache, q, k, v, c["plan"], c["step"], 0.5)
            assert np.array_equal(cache.t_c, before), "cache changed on a miss"
            continue
        if c["expect"] == "invalid":
            _expect_raises(o.PlanError, o.step, cache, q, k, v, c["plan"], c["step"], 0.5)
            continue
        _, _, hit, age = o.step(cache, q, k, v, c["plan"], c["step"], 0.5)
        assert np.array_equal(hit, c["hit"]), f"hit at step {c['step']}"
        assert np.array_equal(age, c["age"]), f"age at step {c['step']}"


def _window_plans(P, w):
    i = np.arange(P)[:, None]
    j = np.arange(P)[None, :]
    near = np.abs(i - j) <= w
    anchor = np.where(near, o_FRESH, o_STORE).astype(np.uint8)
    reuse = np.where(near, o_FRESH, o_REUSE).astype(np.uint8)
    return anchor, reuse


o_REUSE, o_FRESH, o_STORE = 0, 1, 2


def pin_step_all_fresh(o):
    r = _rng(10)
    B, H, S, d, P = 1, 2, 48, 8, 6
    q, k, v = (r.normal(size=(B, H, S, d)) for _ in range(3))
    cache = o.StateCache(P)
    out, lse, hit, age = o.step(cache, q, k, v, np.ones((P, P), np.uint8), 0, 0.3)
    _close(out, _sdpa(q, k, v, 0.3), TOL, "all fresh vs sdpa")
    _close(lse, scipy.special.logsumexp(0.3 * np.einsum("bhqd,bhkd->bhqk", q, k), axis=-1),
           TOL, "all fresh LSE vs scipy")
    assert not hit.any() and not age.any()
    assert (cache.t_c == -1).all(), "fresh (code 1) pairs must not be stored"


def pin_step_reuse_identical(o):
    r = _rng(11)
    B, H, S, d, P = 1, 2, 64, 8, 8
    q, k, v = (r.normal(size=(B, H, S, d)) for _ in range(3))
    anchor, reuse = _window_plans(P, 1)
    cache = o.StateCache(P)
    o.step(cache, q, k, v, anchor, 0, 0.3)
    out, _, hit, age = o.step(cache, q, k, v, reuse, 1, 0.3)
    _close(out, _sdpa(q, k, v, 0.3), TOL, "reuse of unchanged inputs vs sdpa")
    assert np.array_equal(hit, (reuse == 0).astype(np.uint8))
    assert np.array_equal(age, (reuse == 0).astype(np.int32))


def pin_step_reuse_mixed(o):
    """Q fixed, K/V move between steps: a reused pair must see the step-0 K/V
    of its partition and a fresh pair the step-1 K/V, so each query partition
    equals full attention over K/V stitched per partition (computed by sdpa)."""
    r = _rng(12)
    B, H, S, d, P = 1, 2, 40, 8, 5
    n = S // P
    q = r.normal(size=(B, H, S, d))
    k0, v0 = r.normal(size=(B, H, S, d)), r.normal(size=(B, H, S, d))
    k1, v1 = k0 + r.normal(size=k0.shape), v0 + r.normal(size=v0.shape)
    anchor, reuse = _window_plans(P, 1)
    reuse[0, 4] = o_STORE  # a forced-fresh far pair
    cache = o.StateCache(P)
    rows = np.array([0, 3, 9, 17, 22, 31, 38])
    o.step(cache, q, k0, v0, anchor, 0, 0.4, rows=rows)
    out, _, _, _ = o.step(cache, q, k1, v1, reuse, 1, 0.4, rows=rows)
    for idx, row in enumerate(rows):
        i = row // n
        km, vm = k0.copy(), v0.copy()
        for j in range(P):
            if reuse[i, j] != o_REUSE:
                km[..., j * n:(j + 1) * n, :] = k1[..., j * n:(j + 1) * n, :]
                vm[..., j * n:(j + 1) * n, :] = v1[..., j * n:(j + 1) * n, :]
        ref = _sdpa(q[..., row:row + 1, :], km, vm, 0.4)[..., 0, :]
        _close(out[:, :, idx, :], ref, TOL, f"mixed row {row}")
    assert cache.t_c[0, 4] == 1 and cache.t_c[0, 3] == 0


# ---------------------------------------------------------------------------
# grouped cache and bf16 entries (DiTango review: "If this is right" -- merged
# composed states under memory pressure; ledger: group size g)
# ---------------------------------------------------------------------------

def pin_round_bf16(o):
    """bf16 rounding against torch's float32 -> bfloat16 conversion (round to
    nearest even), on random magnitudes and on exact halfway cases."""
    r = _rng(30)
    x = np.concatenate([r.normal(size=2000) * 10.0 ** r.integers(-6, 6, size=2000),
                        [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 0.0, -0.0, 1.5, 2.0 ** -100]])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    got = o.round_bf16(x)
    assert np.array_equal(got, ref), f"bf16 rounding differs at {np.nonzero(got != ref)[0][:5]}"
    assert o.round_bf16(1.0 + 2.0 ** -8) == 1.0 and o.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6


def pin_plan_grouped_golden(o):
    P, g, cases = load_plan_fixture("plan_grouped_4x4.txt", with_group=True)
    r = _rng(31)
    S, d = 2 * P, 3
    q, k, v = (r.normal(size=(1, 1, S, d)) for _ in range(3))
    cache = o.StateCache(P, g)
    for c in cases:
        if c["expect"] in ("cache_miss", "invalid"):
            before = (cache.t_c.copy(), [list(m) for m in cache.member])
            _expect_raises(o.CacheMiss if c["expect"] == "cache_miss" else o.PlanError,
                           o.step, cache, q, k, v, c["plan"], c["step"], 0.5)
            assert np.array_equal(cache.t_c, before[0]) and cache.member == before[1], "cache changed on an error"
            continue
        _, _, hit, age = o.step(cache, q, k, v, c["plan"], c["step"], 0.5)
        assert np.array_equal(hit, c["hit"]), f"grouped hit at step {c['step']}"
        assert np.array_equal(age, c["age"]), f"grouped age at step {c['step']}"


def pin_step_grouped_identical(o):
    """Window plans with grouped entries (g = 2, 3, 4 over P = 6, the last
    group short for g = 4): reusing entries of unchanged inputs gives full
    attention (sdpa), and hit/age follow the pairs."""
    r = _rng(32)
    B, H, S, d, P = 1, 2, 48, 8, 6
    q, k, v = (r.normal(size=(B, H, S, d)) for _ in range(3))
    anchor, reuse = _window_plans(P, 1)
    for g in (2, 3, 4):
        cache = o.StateCache(P, g)
        out0, _, _, _ = o.step(cache, q, k, v, anchor, 0, 0.3)
        _close(out0, _sdpa(q, k, v, 0.3), TOL, f"grouped anchor g={g}")
        assert cache.t_c.shape == (P, (P + g - 1) // g)
        out, _, hit, age = o.step(cache, q, k, v, reuse, 1, 0.3)
        _close(out, _sdpa(q, k, v, 0.3), TOL, f"grouped reuse g={g}")
        assert np.array_equal(hit, (reuse == 0).astype(np.uint8)) and np.array_equal(age, hit.astype(np.int32))


def pin_step_grouped_mixed(o):
    """K/V move between steps; a reused group must carry the step-0 K/V of
    exactly its stored members, so each row equals sdpa over K/V stitched per
    partition.  Row 0 refreshes its far group at step 1."""
    r = _rng(33)
    B, H, S, d, P, g = 1, 2, 48, 8, 6, 2
    n = S // P
    q = r.normal(size=(B, H, S, d))
    k0, v0 = r.normal(size=(B, H, S, d)), r.normal(size=(B, H, S, d))
    k1, v1 = k0 + r.normal(size=k0.shape), v0 + r.normal(size=v0.shape)
    anchor, reuse = _window_plans(P, 1)
    reuse[0, 4:6] = o_STORE
    cache = o.StateCache(P, g)
    rows = np.array([1, 9, 15, 22, 30, 37, 41, 47])  # every partition has rows
    o.step(cache, q, k0, v0, anchor, 0, 0.4, rows=rows)
    out, _, _, _ = o.step(cache, q, k1, v1, reuse, 1, 0.4, rows=rows)
    for idx, row in enumerate(rows):
        i = row // n
        km, vm = k0.copy(), v0.copy()
        for j in range(P):
            if reuse[i, j] != o_REUSE:
                km[..., j * n:(j + 1) * n, :] = k1[..., j * n:(j + 1) * n, :]
                vm[..., j * n:(j + 1) * n, :] = v1[..., j * n:(j + 1) * n, :]
        _close(out[:, :, idx, :], _sdpa(q[..., row:row + 1, :], km, vm, 0.4)[..., 0, :], TOL, f"grouped row {row}")
    assert cache.t_c[0, 2] == 1 and cache.t_c[1, 2] == 0 and cache.member[0][2] == frozenset({4, 5})


def pin_step_bf16_cache(o):
    """bf16 entries: a reuse of unchanged inputs differs from full attention
    by no more than the rounding of the reused OUT (relative 2^-8 of its
    magnitude), and it does differ (the entries are rounded)."""
    r = _rng(34)
    B, H, S, d, P = 1, 2, 48, 8, 6
    q, k, v = (r.normal(size=(B, H, S, d)) for _ in range(3))
    anchor, reuse = _window_plans(P, 1)
    ref = _sdpa(q, k, v, 0.3)
    for g in (1, 3):
        cache = o.StateCache(P, g, "bf16")
        o.step(cache, q, k, v, anchor, 0, 0.3)
        out, _, _, _ = o.step(cache, q, k, v, reuse, 1, 0.3)
        bound = 2.0 ** -8 * max(float(np.max(np.abs(e[0]))) for e in cache.entry.values())
        err = float(np.max(np.abs(out - ref)))
        assert 0.0 < err <= bound, f"bf16 cache g={g}: err {err}, bound {bound}"


# ---------------------------------------------------------------------------
# planner pins (DiTango review: Eq. 7-10, 12, 13 and Algorithm 1 as read in
# the oracle's planner section)
# ---------------------------------------------------------------------------

def pin_planner_weights(o):
    r = _rng(20)
    q, k, v = (r.normal(size=(1, 2, 24, 8)) for _ in range(3))
    states = o.partition_states(q, k, v, 0.4, 4)
    _, full_l = o.full_attention(q, k, v, 0.4)
    w = o.anchor_weights(np.stack([l for _, l in states]), full_l)
    _close(w.sum(), 1.0, 1e-12, "weights sum to 1")       # softmax over partitions
    assert np.all(w > 0)
    w_eq = o.anchor_weights(np.zeros((5, 7)), np.full(7, math.log(5)))
    _close(w_eq, np.full(5, 0.2), 1e-12, "equal LSEs: uniform weights")
    a, b = 0.3, -1.1
    lse2 = np.array([[a] * 3, [b] * 3])
    w2 = o.anchor_weights(lse2, np.full(3, math.log(math.exp(a) + math.exp(b))))
    _close(w2, np.array([math.exp(a), math.exp(b)]) / (math.exp(a) + math.exp(b)), 1e-12, "two-partition weights")


def pin_planner_ratios(o):
    r = _rng(21)
    base = r.normal(size=(2, 6, 4))
    outs = np.stack([base, 3.0 * base, -0.5 * base, np.zeros_like(base)])
    al = o.scale_ratios(outs, 0)
    _close(al, np.array([1.0, 3.0, 0.5, 0.0]), 1e-12, "scale ratios")
    _close(o.scale_ratios(outs, 1)[1], 1.0, 1e-12, "local ratio is 1")


def pin_planner_drift(o):
    r = _rng(22)
    anchor = r.normal(size=(2, 5, 4))
    d0, n0 = o.local_drift(anchor, anchor)
    assert d0 == 0.0
    _close(n0, math.sqrt(float(np.sum(anchor ** 2))), 1e-12, "anchor norm")
    d1, _ = o.local_drift(anchor + 0.25, anchor)
    _close(d1, 0.25 * math.sqrt(anchor.size), 1e-12, "drift of a constant shift")


def pin_planner_select(o):
    P, window, a, cases = load_select_fixture()
    for ratio, plan in cases:
        assert np.array_equal(o.select_plan(a, window, ratio), plan), f"selection at R={ratio}"
    assert (o.select_plan(a, P, 0.7) == o_FRESH).all(), "window covering everything: all fresh"
    # ASE = w * alpha * drift (Eq. 7 with Eq. 10): with w = 1/2 everywhere,
    # alpha decides the order; by hand the smallest remote ASE is (0, 1)
    w = np.full((2, 2), 0.5)
    alpha = np.array([[1.0, 0.2], [4.0, 1.0]])
    aa = o.ase(w, alpha, np.array([1.0, 0.5]))
    _close(aa, np.array([[0.5, 0.1], [1.0, 0.25]]), 1e-12, "ASE worked example")
    assert np.array_equal(o.select_plan(aa, 0, 0.5), np.array([[1, 0], [2, 1]], np.uint8))


def pin_planner_trajectory(o):
    """Inputs that do not move: the first step is an anchor, the next one
    reuses exactly floor(R * #remote) pairs (all ASE are 0) and still equals
    full attention; a large change triggers a new anchor."""
    r = _rng(23)
    B, H, S, d, P = 1, 1, 32, 4, 4
    n = S // P
    q, k, v = (r.normal(size=(B, H, S, d)) for _ in range(3))
    pl = o.Planner(P, window=0, reuse_ratio=0.5, eps_local=0.05)
    cache = o.StateCache(P)
    rows = np.arange(S)
    local = np.concatenate([o.attention_state(q[..., i * n:(i + 1) * n, :], k[..., i * n:(i + 1) * n, :],
                                              v[..., i * n:(i + 1) * n, :], 0.5)[0] for i in range(P)], axis=-2)
    plan0, anchor0, _, _ = o.planner_next(pl, local, n)
    assert anchor0 and np.array_equal(plan0, o.anchor_plan(P, 0))
    _, lse0, _, _ = o.step(cache, q, k, v, plan0, 0, 0.5)
    o.planner_commit_anchor(pl, cache, lse0, lambda i: np.arange(i * n, (i + 1) * n), n)
    # the stored (remote) weights plus the local partition's weight sum to 1
    w_loc = np.array([float(np.mean(np.exp(o.attention_state(
        q[..., i * n:(i + 1) * n, :], k[..., i * n:(i + 1) * n, :], v[..., i * n:(i + 1) * n, :], 0.5)[1]
        - lse0[..., i * n:(i + 1) * n]))) for i in range(P)])
    _close(pl.w.sum(axis=1) + w_loc, np.ones(P), 1e-12, "anchor weights of a query partition")
    plan1, anchor1, drift1, a1 = o.planner_next(pl, local, n)
    assert not anchor1 and np.all(drift1 == 0) and np.all(a1 == 0)
    assert int((plan1 == o_REUSE).sum()) == (P * P - P) // 2
    out1, _, _, _ = o.step(cache, q, k, v, plan1, 1, 0.5)
    _close(out1, _sdpa(q, k, v, 0.5), TOL, "reuse of unchanged states")
    k2 = r.normal(size=k.shape)
    local2 = np.concatenate([o.attention_state(q[..., i * n:(i + 1) * n, :], k2[..., i * n:(i + 1) * n, :],
                                               v[..., i * n:(i + 1) * n, :], 0.5)[0] for i in range(P)], axis=-2)
    _, anchor2, _, _ = o.planner_next(pl, local2, n)
    assert anchor2, "a large local drift must trigger an anchor"


def pin_planner_group_weights(o):
    """Grouped anchor weights: the weight of a group entry is the sum of its
    members' weights (exp of a composed LSE is the sum of the members' exps),
    computed here from scipy log-sum-exps of the raw scores.  The scale
    ratios of the commit path are pinned by pin_planner_commit_closed_form."""
    r = _rng(35)
    B, H, S, d, P, g = 1, 2, 48, 8, 6, 2
    n = S // P
    q, k, v = (r.normal(size=(B, H, S, d)) for _ in range(3))
    pl = o.Planner(P, window=1, reuse_ratio=0.5, eps_local=0.1, g=g)
    cache = o.StateCache(P, g)
    local = np.concatenate([o.attention_state(q[..., i * n:(i + 1) * n, :], k[..., i * n:(i + 1) * n, :],
                                              v[..., i * n:(i + 1) * n, :], 0.3)[0] for i in range(P)], axis=-2)
    plan0, anchor0, _, _ = o.planner_next(pl, local, n)
    assert anchor0
    _, lse0, _, _ = o.step(cache, q, k, v, plan0, 0, 0.3)
    o.planner_commit_anchor(pl, cache, lse0, lambda i: np.arange(i * n, (i + 1) * n), n)
    sc = 0.3 * np.einsum("bhqd,bhkd->bhqk", q, k)
    full = scipy.special.logsumexp(sc, axis=-1)
    for i in range(P):
        rows = slice(i * n, (i + 1) * n)
        for G in range(P // g):
            remote = [j for j in range(G * g, (G + 1) * g) if abs(i - j) > 1]
            if not remote:
                assert pl.w[i, G] == 0.0
                continue
            w_sum = sum(float(np.mean(np.exp(scipy.special.logsumexp(sc[..., rows, j * n:(j + 1) * n], axis=-1)
                                             - full[..., rows]))) for j in remote)
            _close(pl.w[i, G], w_sum, 1e-12, f"group weight ({i},{G})")


def _scaled_copies(seed, B, H, n, d, c, scale):
    """Q random; every KV partition holds the same keys k0, and partition j
    the values c_j * v0.  Then every pair (i, j) has the same scores, so
    OUT_ij = c_j * A_i with A_i = softmax(scale q_i k0^T) v0 and every LSE_ij
    is the same: the composed LSE is LSE_ij + ln P."""
    r = _rng(seed)
    P = len(c)
    q = r.normal(size=(B, H, P * n, d))
    k0 = r.normal(size=(B, H, n, d))
    v0 = r.normal(size=(B, H, n, d))
    k = np.concatenate([k0] * P, axis=-2)
    v = np.concatenate([cj * v0 for cj in c], axis=-2)
    return q, k, v


def pin_planner_commit_closed_form(o):
    """Anchor statistics and ASE in closed form (DiTango review, Axiom &
    Free-Parameter Ledger: Eq. 8 importance, Eq. 9 scale ratio
    alpha(i) = ||AS_ta(i)|| / ||AS_ta(i_loc)|| at the anchor, Eq. 10 and 7).

    With the inputs of _scaled_copies, OUT_ij = c_j * A_i and all LSE_ij are
    equal, so at the anchor w(i,j) = 1/P and alpha(i,j) = |c_j| / |c_i| for
    every stored pair.  A group entry of members M composes equal-LSE states,
    so its OUT is mean_{j in M}(c_j) * A_i: w(i,G) = |M| / P and
    alpha(i,G) = |mean c_M| / |c_i|.  A local state shifted by the constant s_i
    has drift D(i) = |s_i| sqrt(#elements), so ASE(i,G) = w * alpha * D(i)."""
    B, H, n, d, scale = 1, 2, 6, 8, 0.35
    c = [1.0, -2.0, 0.5, 3.0, -0.25]
    P = len(c)
    q, k, v = _scaled_copies(40, B, H, n, d, c, scale)
    shift = np.array([0.01, 0.02, 0.005, 0.03, 0.015])
    for g in (1, 2):
        pl = o.Planner(P, window=0, reuse_ratio=0.5, eps_local=1e9, g=g)
        cache = o.StateCache(P, g)
        local = np.concatenate([o.attention_state(q[..., i * n:(i + 1) * n, :], k[..., i * n:(i + 1) * n, :],
                                                  v[..., i * n:(i + 1) * n, :], scale)[0] for i in range(P)],
                               axis=-2)
        plan0, anchor0, _, _ = o.planner_next(pl, local, n)
        assert anchor0
        _, lse0, _, _ = o.step(cache, q, k, v, plan0, 0, scale)
        o.planner_commit_anchor(pl, cache, lse0, lambda i: np.arange(i * n, (i + 1) * n), n)
        NG = (P + g - 1) // g
        want_w = np.zeros((P, NG))
        want_a = np.zeros((P, NG))
        for i in range(P):
            for G in range(NG):
                members = [j for j in range(G * g, min((G + 1) * g, P)) if j != i]
                if not members:
                    continue
                want_w[i, G] = len(members) / P
                want_a[i, G] = abs(sum(c[j] for j in members) / len(members)) / abs(c[i])
        _close(pl.w, want_w, 1e-12, f"anchor weights, g={g}")
        _close(pl.alpha, want_a, 1e-12, f"anchor scale ratios, g={g}")
        now = local.copy()
        for i in range(P):
            now[..., i * n:(i + 1) * n, :] += shift[i]
        _, anchor1, drift1, a1 = o.planner_next(pl, now, n)
        assert not anchor1
        _close(drift1, shift * math.sqrt(B * H * n * d), 1e-12, f"drift of constant shifts, g={g}")
        _close(a1, want_w * want_a * (shift * math.sqrt(B * H * n * d))[:, None], 1e-12, f"ASE, g={g}")


def pin_planner_select_grouped(o):
    """Selection over groups, worked by hand: P = 4, g = 2, window 0, R = 0.5.
    Units (8, each with a remote member) sorted by ASE: (2,1) (0,0) (1,0)
    (2,0) are reused; window members stay fresh, the rest are stored."""
    a = np.array([[0.1, 0.5], [0.2, 0.9], [0.3, 0.05], [0.8, 0.4]])
    want = np.array([[1, 0, 2, 2], [0, 1, 2, 2], [0, 0, 1, 0], [2, 2, 2, 1]], np.uint8)
    assert np.array_equal(o.select_plan(a, 0, 0.5, 2), want), o.select_plan(a, 0, 0.5, 2)
    assert (o.select_plan(a, 0, 0.0, 2) != o_REUSE).all()
    # groups fully inside the window are no unit: window 1 leaves (0,1)...(3,0) as units only
    full = o.select_plan(a, 1, 1.0, 2)
    assert np.array_equal(full, np.array([[1, 1, 0, 0], [1, 1, 1, 0], [0, 1, 1, 1], [0, 0, 1, 1]], np.uint8))


def pin_planner_trajectory_grouped(o):
    """The trajectory pin with groups of 2: an anchor, then a reuse of
    floor(R * #units) units of unchanged inputs that equals full attention."""
    r = _rng(36)
    B, H, S, d, P, g = 1, 1, 48, 4, 6, 2
    n = S // P
    q, k, v = (r.normal(size=(B, H, S, d)) for _ in range(3))
    pl = o.Planner(P, window=0, reuse_ratio=0.5, eps_local=0.05, g=g)
    cache = o.StateCache(P, g)
    local = np.concatenate([o.attention_state(q[..., i * n:(i + 1) * n, :], k[..., i * n:(i + 1) * n, :],
                                              v[..., i * n:(i + 1) * n, :], 0.5)[0] for i in range(P)], axis=-2)
    plan0, _, _, _ = o.planner_next(pl, local, n)
    _, lse0, _, _ = o.step(cache, q, k, v, plan0, 0, 0.5)
    o.planner_commit_anchor(pl, cache, lse0, lambda i: np.arange(i * n, (i + 1) * n), n)
    plan1, anchor1, _, _ = o.planner_next(pl, local, n)
    assert not anchor1
    reused_units = sum(bool((plan1[i, G * g:(G + 1) * g] == o_REUSE).any()) for i in range(P) for G in range(P // g))
    assert reused_units == (P * (P // g)) // 2, reused_units   # every (i, G) has a remote member at window 0
    out1, _, _, _ = o.step(cache, q, k, v, plan1, 1, 0.5)
    _close(out1, _sdpa(q, k, v, 0.5), TOL, "grouped planner reuse of unchanged states")


# ---------------------------------------------------------------------------
# residual compression pins (CompactFusion, arXiv 2507.17511, Abstract on its
# listing page: compressed step-wise residuals with error feedback; the
# compressor read as int8 codes with one fp32 scale per row)
# ---------------------------------------------------------------------------

def _bf16_values(r, shape, scale=1.0):
    return as_oracle.round_bf16(r.normal(size=shape) * scale)


def pin_residual_exact(o):
    """A residual that is k * 2^-6 with integer |k| <= 127 and 127 reached in
    every row is coded exactly: q = k, s = 2^-6, and the reconstruction is
    the input (k * 2^-6 needs 7 significant bits, which bf16 holds)."""
    r = _rng(50)
    k = r.integers(-127, 128, size=(5, 64))
    k[:, 3] = 127
    k[1, 3] = -127
    x = k * 2.0 ** -6
    q, s, xh = o.residual_encode(x, np.zeros_like(x))
    assert np.array_equal(q.astype(np.int64), k)
    assert np.all(s == np.float32(2.0 ** -6))
    assert np.array_equal(xh, x)


def pin_residual_bound(o):
    """|x - x_hat| <= s / 2 (the quantisation step, half of it) plus the bf16
    rounding of the reconstruction (2^-8 relative); |q| <= 127 with the
    largest residual of every row coded as +-127; s = max|r| / 127; the
    reconstruction holds bf16 values."""
    r = _rng(51)
    for d in (64, 128):
        x = _bf16_values(r, (7, 3, d))
        base = _bf16_values(r, (7, 3, d), 0.9)
        q, s, xh = o.residual_encode(x, base)
        res = x - base
        amax = np.max(np.abs(res), axis=-1)
        _close(s, amax / 127.0, 1e-6 * float(amax.max()), "scale")
        assert np.all(np.abs(q.astype(np.int64)) <= 127)
        assert np.all(np.max(np.abs(q.astype(np.int64)), axis=-1) == 127)
        err = np.abs(x - xh)
        assert np.all(err <= s[..., None] * 0.5 * (1 + 1e-5) + 2.0 ** -8 * np.abs(xh) + 1e-30), float(err.max())
        assert np.array_equal(as_oracle.round_bf16(xh), xh)


def pin_residual_zero(o):
    r = _rng(52)
    x = _bf16_values(r, (4, 64))
    q, s, xh = o.residual_encode(x, x)
    assert not q.any() and not s.any() and np.array_equal(xh, x)


def pin_residual_error_feedback(o):
    """The page's point of error feedback: coding each step's residual against
    the reconstruction keeps the error of every step within that step's own
    bound over a 32-step random walk, while coding the difference of the true
    consecutive values and accumulating the decoded differences drifts
    beyond it."""
    r = _rng(53)
    x = _bf16_values(r, (16, 64))
    rec = x.copy()                       # both sides start from one exact send
    acc = x.copy()                       # no feedback: decoded differences accumulated
    prev = x.copy()
    drift = 0.0
    for t in range(32):
        x = as_oracle.round_bf16(x + 0.05 * r.normal(size=x.shape))
        q, s, rec = o.residual_encode(x, rec)
        bound = s[..., None] * 0.5 * (1 + 1e-5) + 2.0 ** -8 * np.abs(rec)
        assert np.all(np.abs(x - rec) <= bound + 1e-30), t
        qd, sd, _ = o.residual_encode(x, prev)
        acc = as_oracle.round_bf16(acc + qd.astype(np.float64) * sd[..., None])
        prev = x
        drift = max(drift, float(np.max(np.abs(x - acc) - bound)))
    assert drift > 0, "without feedback the error should leave the per-step bound"


PINS = [pin_bruteforce_loops, pin_torch_sdpa_full, pin_scipy_lse, pin_closed_forms,
        pin_compose_closed, pin_assoc_comm, pin_split_invariance, pin_single_partition,
        pin_plan_golden, pin_step_all_fresh, pin_step_reuse_identical, pin_step_reuse_mixed,
        pin_planner_weights, pin_planner_ratios, pin_planner_drift, pin_planner_select, pin_planner_trajectory,
        pin_round_bf16, pin_plan_grouped_golden, pin_step_grouped_identical, pin_step_grouped_mixed,
        pin_step_bf16_cache,
        pin_planner_group_weights, pin_planner_select_grouped, pin_planner_trajectory_grouped,
        pin_planner_commit_closed_form,
        pin_residual_exact, pin_residual_bound, pin_residual_zero, pin_residual_error_feedback]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_passes_pin(pin):
    pin(as_oracle)


# ---------------------------------------------------------------------------
# planted mistakes: each must fail at least one pin
# ---------------------------------------------------------------------------

_orig = {name: getattr(as_oracle, name) for name in
         ("attention_state", "compose", "compose_pair", "resolve_plan", "step", "partition_bounds",
          "anchor_weights", "scale_ratios", "local_drift", "select_plan", "ase", "round_bf16", "n_groups",
          "planner_commit_anchor", "residual_encode", "residual_apply")}


def _m_no_normalise(q, k, v, scale):
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    if k.shape[-2] == 0:
        return as_oracle.empty_state(q.shape[:-1], v.shape[-1])
    s = scale * (q @ np.swapaxes(k, -1, -2))
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=-1, keepdims=True)
    return e @ v, (m + np.log(l))[..., 0]


def _m_lse_unscaled(q, k, v, scale):
    out, _ = _orig["attention_state"](q, k, v, scale)
    _, lse = _orig["attention_state"](q, k, v, 1.0)
    return out, lse


def _m_transposed(q, k, v, scale):
    return _orig["attention_state"](q, k, k, scale)


def _m_log2(q, k, v, scale):
    out, lse = _orig["attention_state"](q, k, v, scale)
    return out, lse / math.log(2)


def _m_compose_unnormalised(states):
    states = list(states)
    _, lse = _orig["compose"](states)
    m = np.max(np.stack([l for _, l in states]), axis=0)
    out = sum(np.exp(l - m)[..., None] * oo for oo, l in states)
    return out, lse


def _m_compose_sign(states):
    states = [(oo, -l) for oo, l in states]
    out, lse = _orig["compose"](states)
    return out, -lse


def _m_compose_drop_last(states):
    states = list(states)
    return _orig["compose"](states[:-1] if len(states) > 1 else states)


def _m_pair_max_only(a, b):
    out, _ = _orig["compose_pair"](a, b)
    return out, np.maximum(a[1], b[1])


def _m_age_sign(plan, t_c, t, g=1, member=None):
    hit, age = _orig["resolve_plan"](plan, t_c, t, g, member)
    return hit, -age


def _m_hit_fresh(plan, t_c, t, g=1, member=None):
    hit, age = _orig["resolve_plan"](plan, t_c, t, g, member)
    return (1 - hit).astype(np.uint8), age


def _m_members_unchecked(plan, t_c, t, g=1, member=None):
    return _orig["resolve_plan"](plan, t_c, t, g, None)


def _m_group_stores_fresh_members(cache, q, k, v, plan, t, scale, rows=None):
    plan2 = np.array(plan, dtype=np.uint8, copy=True)
    P, g = cache.P, cache.g
    for i in range(P):
        for G in range((P + g - 1) // g):
            js = range(G * g, min((G + 1) * g, P))
            if any(plan2[i, j] == 2 for j in js):
                for j in js:
                    if plan2[i, j] == 1:
                        plan2[i, j] = 2
    return _orig["step"](cache, q, k, v, plan2, t, scale, rows)


def _m_bf16_truncate(x):
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32).astype(np.float64)


def _m_bf16_not_rounded(x):
    return np.asarray(x, dtype=np.float64)


def _m_groups_floor(P, g):
    return P // g


def _m_select_group_window(ase_ij, window, reuse_ratio, g=1):
    plan = _orig["select_plan"](ase_ij, window, reuse_ratio, g)
    P = plan.shape[0]
    for i in range(P):
        for G in range((P + g - 1) // g):
            js = range(G * g, min((G + 1) * g, P))
            if any(plan[i, j] == 0 for j in js):
                for j in js:
                    plan[i, j] = 0
    return plan


def _m_store_all_fresh(cache, q, k, v, plan, t, scale, rows=None):
    res = _orig["step"](cache, q, k, v, plan, t, scale, rows)
    cache.t_c[np.asarray(plan) == 1] = t
    return res


def _m_bounds_shift(S, P):
    b = _orig["partition_bounds"](S, P)
    return b[1:] + b[:1]


def _m_weights_unnormalised(lse_pairs, lse_full):
    lse_pairs = np.asarray(lse_pairs, dtype=np.float64)
    return np.exp(lse_pairs).reshape(lse_pairs.shape[0], -1).mean(axis=1)


def _m_ratios_inverted(out_pairs, i):
    r = _orig["scale_ratios"](out_pairs, i)
    with np.errstate(divide="ignore"):
        return np.where(r > 0, 1.0 / r, 0.0)


def _m_drift_relative(out_now, out_anchor):
    d, nrm = _orig["local_drift"](out_now, out_anchor)
    return (d / nrm if nrm > 0 else 0.0), nrm


def _m_select_largest(ase_ij, window, reuse_ratio, g=1):
    return _orig["select_plan"](-np.asarray(ase_ij), window, reuse_ratio, g)


def _m_select_window(ase_ij, window, reuse_ratio, g=1):
    return _orig["select_plan"](ase_ij, window - 1, reuse_ratio, g)


def _m_ase_no_alpha(w, alpha, drift):
    return _orig["ase"](w, np.ones_like(np.asarray(alpha, dtype=np.float64)), drift)


def _m_residual_scale_255(x, base):
    r = (np.asarray(x, np.float32) - np.asarray(base, np.float32)).astype(np.float32)
    amax = np.max(np.abs(r), axis=-1).astype(np.float32)
    inv = np.where(amax > 0, np.float32(255.0) / np.where(amax > 0, amax, 1), 0).astype(np.float32)
    q = np.clip(np.rint(r * inv[..., None]), -127, 127).astype(np.int8)
    s = (amax / np.float32(255.0)).astype(np.float32)
    return q, s, as_oracle.residual_apply(base, q, s)


def _m_residual_truncate(x, base):
    r = (np.asarray(x, np.float32) - np.asarray(base, np.float32)).astype(np.float32)
    amax = np.max(np.abs(r), axis=-1).astype(np.float32)
    inv = np.where(amax > 0, np.float32(127.0) / np.where(amax > 0, amax, 1), 0).astype(np.float32)
    q = np.clip(np.trunc(r * inv[..., None]), -127, 127).astype(np.int8)
    s = (amax / np.float32(127.0)).astype(np.float32)
    return q, s, as_oracle.residual_apply(base, q, s)


def _m_residual_no_bf16(base, q, s):
    prod = (np.asarray(q).astype(np.float32) * np.asarray(s, np.float32)[..., None]).astype(np.float32)
    return (np.asarray(base, np.float32) + prod).astype(np.float64)


def _m_commit_alpha_inverted(pl, cache, lse_full, rows_of, n):
    _orig["planner_commit_anchor"](pl, cache, lse_full, rows_of, n)
    pl.alpha = np.where(pl.alpha > 0, 1.0 / np.where(pl.alpha > 0, pl.alpha, 1.0), 0.0)



MUTANTS = {
    "attention_state: OUT not normalised": ("attention_state", _m_no_normalise),
    "attention_state: LSE without the scale": ("attention_state", _m_lse_unscaled),
    "attention_state: K in place of V": ("attention_state", _m_transposed),
    "attention_state: log2 instead of ln": ("attention_state", _m_log2),
    "compose: weights not normalised": ("compose", _m_compose_unnormalised),
    "compose: sign of the LSE": ("compose", _m_compose_sign),
    "compose: drops a state": ("compose", _m_compose_drop_last),
    "compose_pair: LSE = max": ("compose_pair", _m_pair_max_only),
    "resolve_plan: age sign": ("resolve_plan", _m_age_sign),
    "resolve_plan: hit on fresh": ("resolve_plan", _m_hit_fresh),
    "step: stores plain-fresh pairs": ("step", _m_store_all_fresh),
    "partition_bounds: off by one partition": ("partition_bounds", _m_bounds_shift),
    "anchor_weights: not normalised by the composed LSE": ("anchor_weights", _m_weights_unnormalised),
    "scale_ratios: inverted": ("scale_ratios", _m_ratios_inverted),
    "local_drift: relative instead of absolute": ("local_drift", _m_drift_relative),
    "select_plan: reuses the largest ASE": ("select_plan", _m_select_largest),
    "select_plan: window off by one": ("select_plan", _m_select_window),
    "ase: drops the scale ratio": ("ase", _m_ase_no_alpha),
    "resolve_plan: reused member set not checked": ("resolve_plan", _m_members_unchecked),
    "step: a stored group takes its plain-fresh members too": ("step", _m_group_stores_fresh_members),
    "round_bf16: truncates": ("round_bf16", _m_bf16_truncate),
    "round_bf16: no rounding": ("round_bf16", _m_bf16_not_rounded),
    "n_groups: drops the short last group": ("n_groups", _m_groups_floor),
    "select_plan: a reused group takes its window members too": ("select_plan", _m_select_group_window),
    "planner_commit_anchor: inverted scale ratio": ("planner_commit_anchor", _m_commit_alpha_inverted),
    "residual_encode: scale max/255": ("residual_encode", _m_residual_scale_255),
    "residual_encode: codes truncated": ("residual_encode", _m_residual_truncate),
    "residual_apply: reconstruction not rounded to bf16": ("residual_apply", _m_residual_no_bf16),
}


@pytest.mark.parametrize("name", list(MUTANTS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(as_oracle, attr, fn)
    failed = []
    for pin in PINS:
        try:
            pin(as_oracle)
        except Exception as e:  # noqa: BLE001 - any failure counts
            failed.append(pin.__name__)
    assert failed, f"no pin notices the planted mistake: {name}"
