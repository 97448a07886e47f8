"""Grouped cache entries and bf16 entries on the GPU against the float64
oracle (DiTango review: "If this is right" -- composed states merged into
coarser groups under memory pressure; ledger: group size g).

Same tolerances as the other parity tests (bf16 inputs: OUT max-abs 2e-2 and
relative Frobenius 5e-3, LSE max-abs 1e-3; fp32 inputs with fp32 entries:
1e-5); hit, age, store timestamps and member sets bit-exact.  The oracle rounds its stored entries to bf16 the
way the kernels do (round to nearest even), so both sides compose the same
cached values up to accumulation order."""
import numpy as np
import pytest
import torch

from attention_state_reuse_partition_b200 import workloads as W
from oracle import as_oracle as O
from tests.test_gpu_parity import check_bf16, check_f32, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from attention_state_reuse_partition_b200 import build
    build.build()
    from attention_state_reuse_partition_b200 import api as a
    return a


def _members(ocache):
    return np.array([[sum(1 << j for j in m) for m in row] for row in ocache.member], dtype=np.uint64)


def _run_grouped(api, s, qkv_steps, plans, g, cache_dt, rows=None, heads=None, dtype_check=check_bf16):
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P, g=g, cache_dtype=cache_dt)
    ocache = O.StateCache(s.P, g, "bf16" if cache_dt == "bf16" else "f32")
    for t, (q, k, v) in enumerate(qkv_steps):
        plan = np.asarray(plans[t])
        out, lse, hit, age = api.as_step(cache, q, k, v, plan, t)
        torch.cuda.synchronize()
        hs = slice(None) if heads is None else heads
        qn = f64(q[:, hs])
        kn, vn = f64(k[:, hs]), f64(v[:, hs])
        r = np.arange(s.S) if rows is None else np.asarray(rows)
        ref_o, ref_l, ref_hit, ref_age = O.step(ocache, qn, kn, vn, plan, t, s.scale, rows=r)
        assert np.array_equal(hit, ref_hit), f"hit at step {t}"
        assert np.array_equal(age, ref_age), f"age at step {t}"
        assert np.array_equal(cache.t_c, ocache.t_c), f"t_c at step {t}"
        assert np.array_equal(cache.member, _members(ocache)), f"members at step {t}"
        rt = torch.as_tensor(r, device=out.device)
        dtype_check(out[:, hs][:, :, rt], lse[:, hs][:, :, rt], ref_o, ref_l, f"g={g} {cache_dt} step {t}")
    return cache


@pytest.mark.parametrize("g", [2, 3, 4, 16])
@pytest.mark.parametrize("cache_dt", ["f32", "bf16"])
def test_step_grouped_video_long_small(api, g, cache_dt):
    """Four steps of the long-trajectory construction (forced pairs lift whole
    groups to fresh-and-store); g = 3 leaves a short last group, g = 16 puts
    every partition in one group."""
    s = W.spec("video_long", H=2, rows=8, cols=16, S=16 * 8 * 16)
    steps = [(q.cuda(), k.cuda(), v.cuda()) for _, q, k, v in W.video_trajectory(s)]
    plans = [W.grouped_plan_for_step(s, t, g).numpy() for t in range(s.steps)]
    assert any((p == W.PLAN_REUSE).any() for p in plans[1:])
    _run_grouped(api, s, steps, plans, g, cache_dt)


@pytest.mark.parametrize("g", [1, 4])
def test_step_bf16_cache_video_reuse_small(api, g):
    s = W.spec("video_reuse", H=2, rows=12, cols=16, S=16 * 12 * 16)
    steps = [(q.cuda(), k.cuda(), v.cuda()) for _, q, k, v in W.video_trajectory(s)]
    plans = [W.grouped_plan_for_step(s, t, g).numpy() for t in range(s.steps)]
    _run_grouped(api, s, steps, plans, g, "bf16")


def test_step_grouped_f32_inputs(api):
    """fp32 inputs (CUDA-core path) with grouped fp32 entries: 1e-5."""
    s = W.spec("tiny_f32", P=8)
    q, k, v = (x.cuda() for x in W.iid_qkv(s))
    k2 = k + 0.1 * torch.randn(k.shape, generator=torch.Generator(device="cuda").manual_seed(5), device="cuda")
    near = np.abs(np.arange(8)[:, None] - np.arange(8)[None, :]) <= 1
    plans = [np.where(near, 1, 2).astype(np.uint8), np.where(near, 1, 0).astype(np.uint8)]
    _run_grouped(api, s, [(q, k, v), (q, k2, v)], plans, 3, "f32", dtype_check=check_f32)


def test_step_grouped_fixture_on_gpu(api):
    """The hand-computed grouped fixture through as_step with bf16 entries:
    bit-exact bookkeeping, errors leave the cache unchanged, and every step's
    states match the oracle."""
    from tests._golden import load_plan_fixture
    from attention_state_reuse_partition_b200 import _lib
    P, g, cases = load_plan_fixture("plan_grouped_4x4.txt", with_group=True)
    s = W.spec("flux_image", H=2, S=64 * P, d=64, P=P)
    q, k, v = (x.cuda() for x in W.flux_qkv(s))
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P, g=g, cache_dtype="bf16")
    ocache = O.StateCache(P, g, "bf16")
    qn, kn, vn = (f64(x) for x in (q, k, v))
    for c in cases:
        if c["expect"] in ("cache_miss", "invalid"):
            before = (cache.t_c, cache.member)
            with pytest.raises(api.AsError) as ei:
                api.as_step(cache, q, k, v, c["plan"], c["step"])
            want = _lib.AS_ERR_CACHE_MISS if c["expect"] == "cache_miss" else _lib.AS_ERR_INVALID_ARG
            assert ei.value.status == want
            assert np.array_equal(cache.t_c, before[0]) and np.array_equal(cache.member, before[1])
            continue
        out, lse, hit, age = api.as_step(cache, q, k, v, c["plan"], c["step"])
        assert np.array_equal(hit, c["hit"]) and np.array_equal(age, c["age"])
        ref_o, ref_l, _, _ = O.step(ocache, qn, kn, vn, c["plan"], c["step"], s.scale)
        check_bf16(out, lse, ref_o, ref_l, f"grouped fixture step {c['step']}")
        assert np.array_equal(cache.t_c, ocache.t_c) and np.array_equal(cache.member, _members(ocache))


def test_bf16_entries_are_the_rounded_fp32_entries(api):
    """The same anchor step with an fp32 and a bf16 cache: every bf16 entry is
    the round-to-nearest-even bf16 of the fp32 entry (bit-exact: both come
    from the same kernel arithmetic), and the LSE planes are identical."""
    s = W.spec("video_reuse", H=2, rows=4, cols=8, S=16 * 4 * 8)
    _, q, k, v = next(iter(W.video_trajectory(s)))
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    plan = W.grouped_plan_for_step(s, 0, 4).numpy()
    c32 = api.AsCache(s.B, s.H, s.S, s.d, s.P, g=4, cache_dtype="f32")
    c16 = api.AsCache(s.B, s.H, s.S, s.d, s.P, g=4, cache_dtype="bf16")
    api.as_step(c32, q, k, v, plan, 0)
    api.as_step(c16, q, k, v, plan, 0)
    torch.cuda.synchronize()
    o32, l32 = c32.planes()
    o16, l16 = c16.planes()
    stored = torch.zeros(((s.P + 3) // 4, s.S), dtype=torch.bool)  # [group plane, token]
    for i in range(s.P):
        for G in range(stored.shape[0]):
            if (plan[i, G * 4:(G + 1) * 4] == W.PLAN_FRESH_STORE).any():
                stored[G, i * s.n:(i + 1) * s.n] = True
    stored = stored.cuda()
    a = o32.permute(0, 3, 1, 2, 4)[stored]
    b = o16.permute(0, 3, 1, 2, 4)[stored]
    assert a.numel() > 0
    assert torch.equal(a.to(torch.bfloat16), b)
    assert torch.equal(l32.permute(0, 3, 1, 2)[stored], l16.permute(0, 3, 1, 2)[stored])


def test_step_grouped_video_long_full(api):
    """video_long at full size with g = 4 and bf16 entries (a 5.4 GB cache
    instead of 43.3 GB): seeded samples of 4 rows per partition on two heads
    against the oracle, and the whole bookkeeping bit-exact."""
    s = W.spec("video_long")
    steps = [(q, k, v) for _, q, k, v in W.video_trajectory(s, device="cuda")]
    plans = [W.grouped_plan_for_step(s, t, 4).numpy() for t in range(s.steps)]
    cache = _run_grouped(api, s, steps, plans, 4, "bf16", rows=W.sample_rows(s, 4).numpy(), heads=[0, 39])
    assert cache.buffer.numel() == api.as_cache_bytes(s.B, s.H, s.S, s.d, s.P, 4, "bf16")
    del steps, cache
    torch.cuda.empty_cache()


@pytest.mark.parametrize("g,cache_dt,d,B", [(1, "f32", 64, 2), (3, "bf16", 128, 1), (8, "bf16", 64, 2)])
def test_step_edge_plans(api, g, cache_dt, d, B):
    """Rows with nothing fresh (every group reused), rows with no plain-fresh
    partition (only stored groups, so no composite), a row of only fresh
    pairs, and P at its maximum of 64 partitions for g = 8: the same
    bookkeeping and states as the oracle over three steps."""
    P = 64 if g == 8 else 6
    n = 32 if P == 64 else 64
    s = W.spec("flux_image", B=B, H=2, S=P * n, d=d, P=P)
    steps = []
    gen = torch.Generator(device="cuda").manual_seed(40 + g)
    q, k, v = (x.cuda() for x in W.flux_qkv(s))
    for t in range(3):
        steps.append((q, (k.float() + 0.05 * t * torch.randn(k.shape, generator=gen, device="cuda")).to(k.dtype), v))
    stored = np.full((P, P), W.PLAN_FRESH_STORE, np.uint8)
    reuse = np.zeros((P, P), np.uint8)
    reuse[1] = W.PLAN_FRESH            # a row of only fresh pairs
    reuse[2] = W.PLAN_FRESH_STORE      # a row of only stored groups: no composite
    reuse[3, 0:g] = W.PLAN_FRESH       # a row with one plain-fresh group, the rest reused
    plans = [stored, reuse, reuse.copy()]
    plans[2][2] = 0                    # row 2 reuses what step 1 stored
    _run_grouped(api, s, steps, plans, g, cache_dt,
                 dtype_check=check_bf16 if s.dtype == "bf16" else check_f32)


@pytest.mark.parametrize("g,cache_dt", [(1, "f32"), (4, "bf16")])
def test_step_local_reuses_the_local_states(api, g, cache_dt):
    """as_step_local with the step's local states from as_local_states: the
    same bookkeeping and, within the parity tolerances, the same states as
    the oracle and as as_step (which recomputes the diagonal pairs).  The
    plans also hold rows whose diagonal is stored or reused, where the local
    states are not used."""
    s = W.spec("video_long", H=2, rows=8, cols=16, S=16 * 8 * 16)
    steps = [(q.cuda(), k.cuda(), v.cuda()) for _, q, k, v in W.video_trajectory(s)]
    plans = [W.grouped_plan_for_step(s, t, g).numpy() for t in range(s.steps)]
    plans[1][0, :] = W.PLAN_FRESH_STORE   # row 0 stores everything, its diagonal included
    plans[2][0, :] = W.PLAN_REUSE         # ... and reuses exactly those entries afterwards
    plans[3][0, :] = W.PLAN_REUSE
    ca = api.AsCache(s.B, s.H, s.S, s.d, s.P, g=g, cache_dtype=cache_dt)
    cb = api.AsCache(s.B, s.H, s.S, s.d, s.P, g=g, cache_dtype=cache_dt)
    ocache = O.StateCache(s.P, g, cache_dt)
    for t, (q, k, v) in enumerate(steps):
        plan = plans[t]
        lo, ll = api.as_local_states(q, k, v, s.P)
        out, lse, hit, age = api.as_step_local(ca, q, k, v, plan, t, lo, ll)
        out_b, lse_b, hit_b, age_b = api.as_step(cb, q, k, v, plan, t)
        torch.cuda.synchronize()
        ref_o, ref_l, ref_hit, ref_age = O.step(ocache, f64(q), f64(k), f64(v), plan, t, s.scale)
        assert np.array_equal(hit, ref_hit) and np.array_equal(age, ref_age), t
        assert np.array_equal(hit, hit_b) and np.array_equal(ca.t_c, cb.t_c) and np.array_equal(ca.member, cb.member)
        check_bf16(out, lse, ref_o, ref_l, f"as_step_local g={g} step {t}")
        # the two differ where P is rounded to bf16: against the diagonal's own
        # running maximum here, against the whole window's in as_step
        check_bf16(out, lse, f64(out_b), f64(lse_b), f"as_step_local vs as_step g={g} step {t}")


def test_cache_checkpoint_and_resume(api, tmp_path):
    """A cache saved after the anchor step (torch.save of state_dict) and
    restored into a new buffer gives bit-identical reuse steps."""
    s = W.spec("video_long", H=2, rows=8, cols=16, S=16 * 8 * 16)
    steps = [(q.cuda(), k.cuda(), v.cuda()) for _, q, k, v in W.video_trajectory(s)]
    plans = [W.grouped_plan_for_step(s, t, 4).numpy() for t in range(s.steps)]
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P, g=4, cache_dtype="bf16")
    api.as_step(cache, *steps[0], plans[0], 0)
    torch.cuda.synchronize()
    path = tmp_path / "cache.pt"
    torch.save(cache.state_dict(), path)
    restored = api.AsCache.from_state_dict(torch.load(path, weights_only=False))
    assert np.array_equal(restored.t_c, cache.t_c) and np.array_equal(restored.member, cache.member)
    for t in range(1, s.steps):
        a = api.as_step(cache, *steps[t], plans[t], t)
        b = api.as_step(restored, *steps[t], plans[t], t)
        torch.cuda.synchronize()
        assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]), t
        assert np.array_equal(a[2], b[2]) and np.array_equal(a[3], b[3])


def test_step_replays_from_a_cuda_graph(api):
    """as_step captured in a CUDA graph (a step whose plan stores nothing, so
    it has no host bookkeeping): replays give the eager result bit for bit,
    including after the inputs change in place."""
    s = W.spec("video_reuse", H=2, rows=8, cols=16, S=16 * 8 * 16)
    traj = [(q.cuda(), k.cuda(), v.cuda()) for _, q, k, v in W.video_trajectory(s)]
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P)
    api.as_step(cache, *traj[0], W.plan_for_step(s, 0).numpy(), 0)   # anchor, stores
    plan = W.plan_for_step(s, 1).numpy()                              # reuse only
    assert not (plan == W.PLAN_FRESH_STORE).any()
    q, k, v = (x.clone() for x in traj[1])
    out = torch.empty((s.B, s.H, s.S, s.d), device="cuda")
    lse = torch.empty((s.B, s.H, s.S), device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        api.as_step(cache, q, k, v, plan, 1, out=out, lse=lse)       # warm-up outside capture
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        api.as_step(cache, q, k, v, plan, 1, out=out, lse=lse)
    ref_o, ref_l, _, _ = api.as_step(cache, q, k, v, plan, 1)
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
    q.copy_(traj[0][0])                                               # new inputs, same buffers
    ref_o, ref_l, _, _ = api.as_step(cache, q, k, v, plan, 1)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref_o) and torch.equal(lse, ref_l)
    del graph


@pytest.mark.parametrize("P,n,d", [(1, 640, 128), (8, 8, 64), (16, 8, 128)])
def test_step_extreme_partitions(api, P, n, d):
    """One partition (the first step is plain attention, stored; the next
    ones take the whole row from the cache), and partitions of 8 tokens
    (every KV range and query block far shorter than a 128-row tile): the
    same bookkeeping and states as the oracle over three steps."""
    s = W.spec("flux_image", B=1, H=2, S=P * n, d=d, P=P)
    q, k, v = (x.cuda() for x in W.flux_qkv(s))
    gen = torch.Generator(device="cuda").manual_seed(70 + P)
    steps = [(q, (k.float() + 0.05 * t * torch.randn(k.shape, generator=gen, device="cuda")).to(k.dtype), v)
             for t in range(3)]
    near = np.abs(np.arange(P)[:, None] - np.arange(P)[None, :]) <= 1
    anchor = np.where(near, W.PLAN_FRESH, W.PLAN_FRESH_STORE).astype(np.uint8)
    reuse = np.where(near, W.PLAN_FRESH, W.PLAN_REUSE).astype(np.uint8)
    if P == 1:
        anchor[:] = W.PLAN_FRESH_STORE
        reuse[:] = W.PLAN_REUSE
    _run_grouped(api, s, steps, [anchor, reuse, reuse], 1, "f32")


@pytest.mark.parametrize("cache_dt", ["f32", "bf16"])
def test_step_many_sources(api, cache_dt):
    """Rows with more than 32 sources, so the step compose takes its general
    path: 40 partitions, every pair stored at the first step and reused at
    the next ones (40 cache entries per row), plus a row mixing fresh, stored
    and reused pairs."""
    P, n = 40, 16
    s = W.spec("flux_image", B=1, H=2, S=P * n, d=64, P=P)
    q, k, v = (x.cuda() for x in W.flux_qkv(s))
    gen = torch.Generator(device="cuda").manual_seed(91)
    steps = [(q, (k.float() + 0.05 * t * torch.randn(k.shape, generator=gen, device="cuda")).to(k.dtype), v)
             for t in range(3)]
    stored = np.full((P, P), W.PLAN_FRESH_STORE, np.uint8)
    reuse = np.zeros((P, P), np.uint8)
    mixed = reuse.copy()
    mixed[5, :10] = W.PLAN_FRESH
    mixed[5, 10:20] = W.PLAN_FRESH_STORE
    _run_grouped(api, s, steps, [stored, reuse, mixed], 1, cache_dt)
