"""The C-ABI library on a machine without a GPU: it loads, exports every
entry point that include/as_partition.h declares, rejects bad arguments before
touching the device, and resolves plans (host-side bookkeeping) exactly as the
hand-computed fixture says."""
import ctypes
import os
import re

import numpy as np
import pytest

from attention_state_reuse_partition_b200 import build
from tests._golden import load_plan_fixture

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def api():
    build.build()
    from attention_state_reuse_partition_b200 import api as a
    return a


def _declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"^\s*(?:const\s+)?[\w\*\s]+?\b(as_\w+)\s*\(", text, re.M))
    return names


def test_library_exports_every_declared_symbol(api):
    from attention_state_reuse_partition_b200 import _lib
    declared = _declared_symbols()
    assert {"as_partition_attn", "as_compose", "as_step", "as_cache_init"} <= declared
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for name in sorted(declared):
        assert hasattr(lib, name), f"{name} declared but not exported"
    assert declared == set(_lib.EXPORTS)


def test_version(api):
    assert "sm_100a" in api.as_version()


def test_cache_bytes(api):
    assert api.as_cache_bytes(1, 24, 32768, 128, 16) == 16 * 24 * 32768 * 129 * 4
    assert api.as_cache_bytes(1, 2, 100, 128, 3) == 0      # S % P != 0
    assert api.as_cache_bytes(1, 2, 96, 96, 3) == 0        # d not supported
    assert api.as_cache_bytes(1, 2, 130, 64, 65) == 0      # P > AS_MAX_P


def _status(call):
    from attention_state_reuse_partition_b200 import _lib
    st = call()
    return st, _lib.LIB.as_last_error().decode()


def test_partition_attn_rejects_bad_arguments_before_launch(api):
    from attention_state_reuse_partition_b200 import _lib
    L = _lib.LIB
    parts = (ctypes.c_int32 * 2)(0, 1)
    dup = (ctypes.c_int32 * 2)(1, 1)
    p = 1 << 20  # aligned placeholder address, never dereferenced

    def call(d=128, S=512, P=4, q_part=0, kv=parts, n=2, compose=1, ptr=p, scale=0.1):
        return L.as_partition_attn(ptr, p, p, 1, 1, 2, S, d, P, scale, q_part, kv, n, compose, p, p, None)

    for kw, frag in [(dict(d=96), "d must be"), (dict(S=510), "multiple of P"), (dict(q_part=4), "q_part"),
                     (dict(kv=dup), "twice"), (dict(n=0), "KV partitions"), (dict(compose=3), "compose"),
                     (dict(ptr=p + 4), "aligned"), (dict(ptr=0), "null"), (dict(scale=0.0), "scale"),
                     (dict(P=65, S=65 * 8), "P must be")]:
        st, msg = _status(lambda: call(**kw))
        assert st == _lib.AS_ERR_INVALID_ARG, (kw, st, msg)
        assert frag in msg, (kw, msg)


def test_compose_rejects_bad_arguments(api):
    from attention_state_reuse_partition_b200 import _lib
    L = _lib.LIB
    p = 1 << 20
    assert L.as_compose(p, p, 4, 100, 96, 100 * 96, 100, p, p, None) == _lib.AS_ERR_INVALID_ARG
    assert L.as_compose(p, p, 0, 100, 128, 100 * 128, 100, p, p, None) == _lib.AS_ERR_INVALID_ARG
    assert L.as_compose(p, p, 4, 100, 128, 10, 100, p, p, None) == _lib.AS_ERR_INVALID_ARG
    assert L.as_compose(p, p, 4, 0, 128, 0, 0, p, p, None) == _lib.AS_OK  # empty: nothing to do


def test_cache_init_validation(api):
    from attention_state_reuse_partition_b200 import _lib
    s = _lib.AsCacheStruct()
    L = _lib.LIB
    need = api.as_cache_bytes(1, 2, 64, 64, 4)
    assert L.as_cache_init(ctypes.byref(s), 1 << 20, need - 1, 1, 2, 64, 64, 4, 0) == _lib.AS_ERR_INVALID_ARG
    assert L.as_cache_init(ctypes.byref(s), (1 << 20) + 16, need, 1, 2, 64, 64, 4, 0) == _lib.AS_ERR_INVALID_ARG
    assert L.as_cache_init(ctypes.byref(s), 1 << 20, need, 1, 2, 64, 64, 4, 7) == _lib.AS_ERR_INVALID_ARG
    assert L.as_cache_init(ctypes.byref(s), 1 << 20, need, 1, 2, 64, 64, 4, 0) == _lib.AS_OK
    assert s.out_planes == 1 << 20
    assert s.lse_planes == (1 << 20) + 4 * 1 * 2 * 64 * 64 * 4
    assert all(s.t_c[x] == -1 for x in range(16)) and s.g == 1 and s.n_groups == 4
    # bf16 entries: OUT planes of 2-byte elements, LSE planes fp32
    need_bf = L.as_cache_bytes(1, 2, 64, 64, 4, 1)
    assert need_bf == 4 * 1 * 2 * 64 * (64 * 2 + 4)
    assert L.as_cache_init(ctypes.byref(s), 1 << 20, need_bf, 1, 2, 64, 64, 4, 1) == _lib.AS_OK
    assert s.lse_planes == (1 << 20) + 4 * 1 * 2 * 64 * 64 * 2


def test_cache_group_sizes(api):
    """Grouped caches: ceil(P / g) planes; g outside [1, P] is rejected."""
    from attention_state_reuse_partition_b200 import _lib
    L = _lib.LIB
    rows = 2 * 3 * 120
    for P, g, dt, esz in [(6, 1, 0, 4), (6, 2, 0, 4), (6, 4, 0, 4), (6, 6, 1, 2), (5, 2, 1, 2)]:
        NG = (P + g - 1) // g
        need = L.as_cache_group_bytes(2, 3, 120, 128, P, g, dt)
        assert need == NG * rows * (128 * esz + 4), (P, g, dt)
        s = _lib.AsCacheStruct()
        assert L.as_cache_group_init(ctypes.byref(s), 1 << 24, need, 2, 3, 120, 128, P, g, dt) == _lib.AS_OK
        assert s.g == g and s.n_groups == NG
        assert s.lse_planes == (1 << 24) + NG * rows * 128 * esz
    for g in (0, 7):
        s = _lib.AsCacheStruct()
        assert L.as_cache_group_bytes(2, 3, 96, 128, 6, g, 0) == 0
        assert L.as_cache_group_init(ctypes.byref(s), 1 << 24, 1 << 30, 2, 3, 96, 128, 6, g, 0) == \
            _lib.AS_ERR_INVALID_ARG


def _replay_fixture(api, cache, cases, P, g):
    """as_plan_resolve against a hand-computed fixture.  Between steps the
    bookkeeping follows the fixture's rule: every group with stored (code 2)
    members gets t_c = step and member = those members; a miss or an invalid
    plan changes nothing."""
    from attention_state_reuse_partition_b200 import _lib
    NG = (P + g - 1) // g
    t_c = np.full((P, NG), -1)
    member = np.zeros((P, NG), dtype=np.uint64)
    for c in cases:
        if c["expect"] in ("cache_miss", "invalid"):
            with pytest.raises(api.AsError) as ei:
                api.as_plan_resolve(cache, c["plan"], c["step"])
            want = _lib.AS_ERR_CACHE_MISS if c["expect"] == "cache_miss" else _lib.AS_ERR_INVALID_ARG
            assert ei.value.status == want, (c["step"], c["expect"])
            continue
        hit, age = api.as_plan_resolve(cache, c["plan"], c["step"])
        assert np.array_equal(hit, c["hit"]), c["step"]
        assert np.array_equal(age, c["age"]), c["step"]
        for i in range(P):
            for G in range(NG):
                m = sum(1 << j for j in range(G * g, min((G + 1) * g, P)) if c["plan"][i, j] == 2)
                if m:
                    t_c[i, G] = c["step"]
                    member[i, G] = m
        cache.set_t_c(t_c)
        cache.set_member(member)


def test_plan_resolve_matches_fixture(api):
    """Host-side hit/age from the C library against the hand-computed
    fixture; the store timestamps between steps follow the fixture's rule
    (code 2 refreshes t_c, a miss or invalid plan changes nothing)."""
    from attention_state_reuse_partition_b200 import _lib
    P, cases = load_plan_fixture()
    cache = api.AsCache.host_only(1, 1, 4 * P, 64, P)
    _replay_fixture(api, cache, cases, P, 1)


def test_plan_resolve_matches_grouped_fixture(api):
    """The same for grouped entries (g = 2): member sets, mixed groups."""
    P, g, cases = load_plan_fixture("plan_grouped_4x4.txt", with_group=True)
    cache = api.AsCache.host_only(1, 1, 4 * P, 64, P, g=g, cache_dtype="bf16")
    _replay_fixture(api, cache, cases, P, g)


def test_plan_resolve_matches_oracle_on_random_plans(api):
    """Random plans and group sizes: the C resolve and the oracle agree on
    hit, age and the kind of error, with the bookkeeping replayed from the
    oracle's cache."""
    from oracle import as_oracle as O
    from attention_state_reuse_partition_b200 import _lib
    r = np.random.default_rng(11)
    for trial in range(30):
        P = int(r.integers(2, 9))
        g = int(r.integers(1, P + 1))
        ocache = O.StateCache(P, g)
        cache = api.AsCache.host_only(1, 1, 2 * P, 64, P, g=g)
        q = r.normal(size=(1, 1, 2 * P, 2))
        for t in range(5):
            plan = r.choice([0, 1, 2], size=(P, P), p=[0.4, 0.3, 0.3]).astype(np.uint8)
            try:
                _, _, ohit, oage = O.step(ocache, q, q, q, plan, t, 0.5)
                oerr = None
            except O.CacheMiss:
                oerr = _lib.AS_ERR_CACHE_MISS
            except O.PlanError:
                oerr = _lib.AS_ERR_INVALID_ARG
            try:
                hit, age = api.as_plan_resolve(cache, plan, t)
                err = None
            except api.AsError as e:
                err = e.status
            assert err == oerr, (trial, t)
            if err is None:
                assert np.array_equal(hit, ohit) and np.array_equal(age, oage), (trial, t)
            cache.set_t_c(ocache.t_c)
            cache.set_member([[sum(1 << j for j in m) for m in row] for row in ocache.member])


def test_planner_and_cache_must_share_the_group_size(api):
    """The anchor statistics read one entry per (i, G): a planner for groups
    of g needs a cache of the same g (checked on the host, before any launch)."""
    from attention_state_reuse_partition_b200 import _lib
    plan = np.ones((4, 4), np.uint8)
    for pg, cg, dt in [(1, 2, "f32"), (2, 1, "bf16"), (4, 2, "bf16")]:
        pl = api.AsPlanner(4, 1, 0.5, 0.1, g=pg)
        cache = api.AsCache.host_only(1, 1, 64, 64, 4, g=cg, cache_dtype=dt)
        st = _lib.LIB.as_planner_commit_anchor(ctypes.byref(pl.struct), ctypes.byref(cache.struct), 1 << 20,
                                               1 << 20, plan.ctypes.data, 1 << 20, 1 << 30, None)
        assert st == _lib.AS_ERR_INVALID_ARG, (pg, cg, dt)
        assert "groups" in _lib.LIB.as_last_error().decode()


def test_grouped_selection_matches_oracle(api):
    """The C per-group selection against the hand-worked case and, bit-exactly,
    the oracle's on random ASE values with ties, group sizes and windows."""
    from oracle import as_oracle as O
    a = np.array([[0.1, 0.5], [0.2, 0.9], [0.3, 0.05], [0.8, 0.4]])
    want = np.array([[1, 0, 2, 2], [0, 1, 2, 2], [0, 0, 1, 0], [2, 2, 2, 1]], np.uint8)
    assert np.array_equal(api.as_plan_select(a, 0, 0.5, g=2), want)
    r = np.random.default_rng(8)
    for trial in range(60):
        P = int(r.integers(1, 24))
        g = int(r.integers(1, P + 1))
        window = int(r.integers(0, 4))
        ase = np.round(r.random((P, (P + g - 1) // g)) * 4) / 4
        ratio = float(r.choice([0.0, 0.25, 0.5, 0.9, 1.0, r.random()]))
        assert np.array_equal(api.as_plan_select(ase, window, ratio, g=g), O.select_plan(ase, window, ratio, g)), \
            (P, g, window, ratio)
    with pytest.raises(api.AsError):
        api.as_plan_select(np.zeros((4, 3)), 0, 0.5, g=2)


def test_step_cache_miss_is_reported_before_any_launch(api):
    """A reuse of a never-stored entry fails on the host, with the cache untouched."""
    from attention_state_reuse_partition_b200 import _lib
    P = 4
    cache = api.AsCache.host_only(1, 1, 64, 64, P)
    plan = np.ones((P, P), np.uint8)
    plan[0, 3] = 0
    p = 1 << 20
    st = _lib.LIB.as_step(ctypes.byref(cache.struct), p, p, p, 0, 0.125, plan.ctypes.data, 1, p, p, None, None,
                          None)
    assert st == _lib.AS_ERR_CACHE_MISS
    assert "(0, 3)" in _lib.LIB.as_last_error().decode()
    assert (cache.t_c == -1).all()


def test_plan_select_matches_fixture_and_oracle(api):
    """The C selection against the hand-computed fixture and, bit-exactly, the
    oracle's selection on random ASE values with ties."""
    from oracle import as_oracle as O
    from tests._golden import load_select_fixture
    P, window, a, cases = load_select_fixture()
    for ratio, plan in cases:
        assert np.array_equal(api.as_plan_select(a, window, ratio), plan), ratio
    r = np.random.default_rng(7)
    for trial in range(40):
        P = int(r.integers(1, 20))
        window = int(r.integers(0, 4))
        ase = np.round(r.random((P, P)) * 4) / 4  # many ties
        ratio = float(r.choice([0.0, 0.1, 0.33, 0.5, 0.9, 1.0, r.random()]))
        assert np.array_equal(api.as_plan_select(ase, window, ratio), O.select_plan(ase, window, ratio)), \
            (P, window, ratio)


def test_planner_init_validation(api):
    from attention_state_reuse_partition_b200 import _lib
    for args in [(0, 1, 0.5, 0.1), (65, 1, 0.5, 0.1), (4, -1, 0.5, 0.1), (4, 1, 1.5, 0.1), (4, 1, 0.5, -1.0)]:
        with pytest.raises(api.AsError) as ei:
            api.AsPlanner(*args)
        assert ei.value.status == _lib.AS_ERR_INVALID_ARG
    pl = api.AsPlanner(8, 2, 0.6, 0.05)
    assert not pl.has_anchor and pl.P == 8
    assert api.as_planner_scratch_bytes(1, 40, 32) == (32 * 32 * 40 * 2 + 32 * 32 * 2) * 8


def test_cache_bookkeeping_round_trip(api):
    """The host bookkeeping of a cache survives state_dict (no device buffer
    on a machine without a GPU)."""
    cache = api.AsCache.host_only(1, 1, 64, 64, 8, g=3, cache_dtype="bf16")
    t_c = np.arange(8 * 3).reshape(8, 3) - 5
    member = np.arange(8 * 3, dtype=np.uint64).reshape(8, 3) * 7
    cache.set_t_c(t_c)
    cache.set_member(member)
    sd = cache.state_dict()
    assert sd["g"] == 3 and sd["cache_dtype"] == "bf16" and sd["buffer"] is None
    other = api.AsCache.host_only(1, 1, 64, 64, 8, g=3, cache_dtype="bf16")
    other.set_t_c(sd["t_c"])
    other.set_member(sd["member"])
    assert np.array_equal(other.t_c, t_c) and np.array_equal(other.member, member)


def test_python_entry_points_check_q_k_v(api):
    """The binding refuses K or V that differ from Q in shape or dtype (the
    library would read them with Q's element type), before any device call."""
    import torch
    from attention_state_reuse_partition_b200 import _lib
    q = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16)
    good = torch.zeros_like(q)
    cache = api.AsCache.host_only(1, 2, 64, 64, 4)
    plan = np.ones((4, 4), np.uint8)
    calls = [lambda k, v: api.as_partition_attn(q, k, v, 4, -1, [0, 1, 2, 3]),
             lambda k, v: api.as_step(cache, q, k, v, plan, 0),
             lambda k, v: api.as_local_states(q, k, v, 4)]
    for bad, what in [(good.float(), "dtype"), (torch.zeros(1, 2, 32, 64, dtype=torch.bfloat16), "shape")]:
        for fn in calls:
            for args in [(bad, good), (good, bad)]:
                with pytest.raises(api.AsError) as ei:
                    fn(*args)
                assert ei.value.status == _lib.AS_ERR_INVALID_ARG and "does not match q" in str(ei.value), what


def test_python_entry_points_check_buffers(api):
    """Caller-supplied outputs must be fp32 of exactly the shape the library
    writes; compose and drift inputs must agree with each other."""
    import torch
    from attention_state_reuse_partition_b200 import _lib
    q = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16)
    cache = api.AsCache.host_only(1, 2, 64, 64, 4)
    plan = np.ones((4, 4), np.uint8)
    short = torch.zeros(1, 2, 32, 64)
    bad_cases = [
        lambda: api.as_step(cache, q, q, q, plan, 0, out=short),
        lambda: api.as_step(cache, q, q, q, plan, 0, lse=torch.zeros(1, 2, 64, dtype=torch.float64)),
        lambda: api.as_partition_attn(q, q, q, 4, 1, [0, 1], out=torch.zeros(1, 2, 64, 64)),
        lambda: api.as_partition_attn(q, q, q, 4, -1, [0, 1], compose=False, lse=torch.zeros(1, 2, 64)),
        lambda: api.as_local_states(q, q, q, 4, out=short),
        lambda: api.as_step_local(cache, q, q, q, plan, 0, short, torch.zeros(1, 2, 64)),
        lambda: api.as_compose(torch.zeros(3, 10, 64), torch.zeros(3, 11)),
        lambda: api.as_compose(torch.zeros(3, 10, 64), torch.zeros(3, 10), out=torch.zeros(10, 32)),
        lambda: api.as_plan_drift(torch.zeros(1, 2, 64, 64), torch.zeros(1, 2, 64, 32), 4, torch.zeros(8)),
        lambda: api.as_plan_drift_static(torch.zeros(1, 2, 64, 64), torch.zeros(1, 2, 64, 64).double(), 4),
    ]
    # inputs of another shape than the cache's: the library would index them with the cache's sizes
    for qq in [torch.zeros(1, 2, 32, 64, dtype=torch.bfloat16), torch.zeros(1, 1, 64, 64, dtype=torch.bfloat16)]:
        for fn in [lambda: api.as_step(cache, qq, qq, qq, plan, 0),
                   lambda: api.as_step_local(cache, qq, qq, qq, plan, 0, torch.zeros(qq.shape), torch.zeros(qq.shape[:3]))]:
            with pytest.raises(api.AsError) as ei:
                fn()
            assert "the cache's shape" in str(ei.value)
    for k, fn in enumerate(bad_cases):
        with pytest.raises(api.AsError) as ei:
            fn()
        assert ei.value.status == _lib.AS_ERR_INVALID_ARG, (k, str(ei.value))
        assert "float32" in str(ei.value), (k, str(ei.value))  # not the later device-pointer check


def test_planner_entry_points_check_shapes(api):
    """as_planner_next and as_planner_commit_anchor read the planner's anchor
    states with the caller's or the cache's sizes: mismatches are refused."""
    import torch
    pl = api.AsPlanner(4, 1, 0.5, 0.1, 1, 2, 64, 64, device="cpu")
    cache = api.AsCache.host_only(1, 2, 64, 64, 4)
    other = api.AsCache.host_only(1, 2, 128, 64, 4)
    plan = np.ones((4, 4), np.uint8)
    for fn in [lambda: api.as_planner_next(pl, torch.zeros(1, 2, 32, 64)),
               lambda: api.as_planner_next(pl, torch.zeros(1, 2, 64, 64, dtype=torch.float64)),
               lambda: api.as_planner_commit_anchor(pl, cache, torch.zeros(1, 2, 32), plan),
               lambda: api.as_planner_commit_anchor(pl, other, torch.zeros(1, 2, 128), plan),
               lambda: api.as_planner_next(api.AsPlanner(4, 1, 0.5, 0.1), torch.zeros(1, 2, 64, 64))]:
        with pytest.raises(api.AsError) as ei:
            fn()
        assert "must be float32" in str(ei.value) or "do not match" in str(ei.value) or "no device state" in str(ei.value)


def test_drift_entry_points_reject_misaligned_local_states(api):
    """The drift reduction reads the local-state tensors with 16-byte loads:
    every entry point that feeds it refuses a pointer off that boundary on the
    host (a view whose storage offset is not a multiple of four floats), so no
    kernel ever sees it."""
    from attention_state_reuse_partition_b200 import _lib
    L = _lib.LIB
    p, bad = 1 << 20, (1 << 20) + 4
    B, H, S, d, P = 1, 2, 64, 64, 4
    h2 = (ctypes.c_double * P)()
    h3 = (ctypes.c_double * P)()
    plan = np.ones((P, P), np.uint8)
    pl = api.AsPlanner(P, 1, 0.5, 0.1)
    cache = api.AsCache.host_only(B, H, S, d, P)
    is_anchor = ctypes.c_int(0)
    calls = {
        "as_plan_drift now": lambda: L.as_plan_drift(bad, p, B, H, S, d, P, p, 1 << 30, h2, h3, None),
        "as_plan_drift anchor": lambda: L.as_plan_drift(p, bad, B, H, S, d, P, p, 1 << 30, h2, h3, None),
        "as_plan_drift_static now": lambda: L.as_plan_drift_static(bad, p, B, H, S, d, P, h2, h3, None),
        "as_plan_drift_static anchor": lambda: L.as_plan_drift_static(p, bad, B, H, S, d, P, h2, h3, None),
        "as_planner_next now": lambda: L.as_planner_next(ctypes.byref(pl.struct), bad, p, B, H, S, d, p, 1 << 30,
                                                         plan.ctypes.data, ctypes.byref(is_anchor), None, None),
        "as_planner_next anchor": lambda: L.as_planner_next(ctypes.byref(pl.struct), p, bad, B, H, S, d, p,
                                                            1 << 30, plan.ctypes.data, ctypes.byref(is_anchor),
                                                            None, None),
        "as_planner_commit_anchor": lambda: L.as_planner_commit_anchor(ctypes.byref(pl.struct),
                                                                       ctypes.byref(cache.struct), p, bad,
                                                                       plan.ctypes.data, p, 1 << 30, None),
    }
    for name, call in calls.items():
        st, msg = _status(call)
        assert st == _lib.AS_ERR_INVALID_ARG, (name, st, msg)
        assert "16-byte aligned" in msg, (name, msg)


def test_rank_cache_and_step_cp_checks(api):
    """One rank's cache (context parallelism) and as_step_cp's checks, all on
    the host before any launch: a KV partition that the rank's rows compute
    but the buffer lacks, a slot beyond the buffer or given twice, and a rank
    cache passed to as_step are refused; misses are checked only in the
    rank's own rows."""
    from attention_state_reuse_partition_b200 import _lib
    L = _lib.LIB
    B, H, S, d, P = 1, 2, 8 * 64, 64, 8
    n = S // P
    assert api.as_cache_cp_bytes(B, H, S, d, P, 3) == 3 * n * B * H * (d * 4 + 4) * P
    assert api.as_cache_cp_bytes(B, H, S, d, P, 0) == 0 and api.as_cache_cp_bytes(B, H, S, d, P, P + 1) == 0
    with pytest.raises(api.AsError):
        api.AsCache.host_only(B, H, S, d, P, q_first=6, q_count=3)
    c = api.AsCache.host_only(B, H, S, d, P, q_first=3, q_count=3)
    p = 1 << 20
    # rows 3..5 (the rank's) compute every KV partition (window fresh, the rest
    # fresh-and-store); every other row reuses entries nobody stored, which
    # concerns other ranks only
    plan = np.zeros((P, P), np.uint8)
    for i in range(3, 6):
        plan[i] = [1 if abs(i - j) <= 1 else 2 for j in range(P)]
    hit, age = api.as_plan_resolve(c, plan, 0)
    assert hit.sum() == 0 and age.sum() == 0
    own_miss = plan.copy()
    own_miss[4, 7] = 0
    with pytest.raises(api.AsError) as ei:
        api.as_plan_resolve(c, own_miss, 0)
    assert ei.value.status == _lib.AS_ERR_CACHE_MISS and "(4, 7)" in str(ei.value)

    def step_cp(slots, kv_rows):
        arr = np.ascontiguousarray(plan.reshape(-1))
        sl = np.ascontiguousarray(np.asarray(slots, np.int32))
        return L.as_step_cp(ctypes.byref(c.struct), p, p, p, kv_rows, sl.ctypes.data, 1, 0.125, arr.ctypes.data,
                            0, p, p, None, None, None)
    for slots, kv_rows, frag in [([-1, 1, 2, 3, 4, 5, 6, 7], 8 * n, "not in the buffer"),
                                 ([0, 1, 2, 3, 4, 5, 6, 8], 8 * n, "beyond"),
                                 ([0, 1, 2, 3, 3, 5, 6, 7], 8 * n, "twice"),
                                 ([0, 1, 2, 3, 4, 5, 6, 7], 7 * n, "beyond")]:
        st, msg = _status(lambda: step_cp(slots, kv_rows))
        assert st == _lib.AS_ERR_INVALID_ARG and frag in msg, (slots, st, msg)
    assert (c.t_c == -1).all()
    full = api.AsCache.host_only(B, H, S, d, P)
    st, msg = _status(lambda: L.as_step(ctypes.byref(c.struct), p, p, p, 1, 0.125,
                                        np.ascontiguousarray(plan.reshape(-1)).ctypes.data, 0, p, p, None, None,
                                        None))
    assert st == _lib.AS_ERR_INVALID_ARG and "as_step_cp" in msg
    assert full.rows == S and c.rows == 3 * n


def test_residual_codec_checks(api):
    """as_residual_encode / decode refuse bad sizes and pointers on the host;
    zero rows is a no-op even without a GPU."""
    from attention_state_reuse_partition_b200 import _lib
    L = _lib.LIB
    p = 1 << 20
    assert L.as_residual_encode(p, p, p, p, 0, 128, None) == _lib.AS_OK
    for args, frag in [((p, p, p, p, 10, 96, None), "d must be"), ((p, p, p, p, -1, 128, None), "rows"),
                       ((p, 0, p, p, 10, 128, None), "null"), ((p + 8, p, p, p, 10, 128, None), "aligned")]:
        st, msg = _status(lambda: L.as_residual_encode(*args))
        assert st == _lib.AS_ERR_INVALID_ARG and frag in msg, (args, msg)
    st, msg = _status(lambda: L.as_residual_decode(p, p, p + 4, 10, 64, None))
    assert st == _lib.AS_ERR_INVALID_ARG and "aligned" in msg


def test_checked_build_probe_needs_the_checked_library(api):
    """The normal library refuses the bounds probe before any launch."""
    from attention_state_reuse_partition_b200 import _lib
    if _lib.CHECKED:
        pytest.skip("checked library loaded")
    st, msg = _status(lambda: _lib.LIB.as_debug_bounds_probe(1 << 20, 32, None))
    assert st == _lib.AS_ERR_UNSUPPORTED and "checked build" in msg
