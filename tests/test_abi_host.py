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
    assert L.as_cache_init(ctypes.byref(s), 1 << 20, need, 1, 2, 64, 64, 4, 1) == _lib.AS_ERR_UNSUPPORTED
    assert L.as_cache_init(ctypes.byref(s), 1 << 20, need, 1, 2, 64, 64, 4, 0) == _lib.AS_OK
    assert s.out_planes == 1 << 20
    assert s.lse_planes == (1 << 20) + 4 * 1 * 2 * 64 * 64 * 4
    assert all(s.t_c[x] == -1 for x in range(16))


def test_plan_resolve_matches_fixture(api):
    """Host-side hit/age from the C library against the hand-computed
    fixture; the store timestamps between steps follow the fixture's rule
    (code 2 refreshes t_c, a miss or invalid plan changes nothing)."""
    from attention_state_reuse_partition_b200 import _lib
    P, cases = load_plan_fixture()
    cache = api.AsCache.host_only(1, 1, 4 * P, 64, P)
    t_c = np.full((P, P), -1)
    for c in cases:
        if c["expect"] == "cache_miss":
            with pytest.raises(api.AsError) as ei:
                api.as_plan_resolve(cache, c["plan"], c["step"])
            assert ei.value.status == _lib.AS_ERR_CACHE_MISS
            continue
        if c["expect"] == "invalid":
            with pytest.raises(api.AsError) as ei:
                api.as_plan_resolve(cache, c["plan"], c["step"])
            assert ei.value.status == _lib.AS_ERR_INVALID_ARG
            continue
        hit, age = api.as_plan_resolve(cache, c["plan"], c["step"])
        assert np.array_equal(hit, c["hit"]), c["step"]
        assert np.array_equal(age, c["age"]), c["step"]
        t_c[c["plan"] == 2] = c["step"]
        cache.set_t_c(t_c)


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
