"""CUDA path against the float64 oracle, element by element, on the same
seeded inputs.  Tolerances (written here, applied everywhere below):

* fp32 inputs: max-abs 1e-5 on OUT and LSE;
* bf16 inputs (fp32 accumulation): OUT max-abs 2e-2 and relative Frobenius
  5e-3, LSE max-abs 1e-3;
* plan bookkeeping (hit, age, store timestamps): bit-exact.

Small cases cover ragged tiles (partitions of 576, 192, 64 and 32 tokens
against 128-key tiles), d = 64 and 128, B > 1, empty states, non-contiguous
KV lists and several steps of reuse.  Full-size cases run the workloads in the
launch configuration of the benchmark and compare seeded samples of rows."""
import math

import numpy as np
import pytest
import torch

from attention_state_reuse_partition_b200 import workloads as W
from oracle import as_oracle as O

pytestmark = pytest.mark.gpu

F32_TOL = 1e-5
BF16_OUT_ABS, BF16_OUT_RELFRO, BF16_LSE_ABS = 2e-2, 5e-3, 1e-3


@pytest.fixture(scope="module")
def api():
    from attention_state_reuse_partition_b200 import build
    build.build()
    from attention_state_reuse_partition_b200 import api as a
    return a


def f64(t):
    return t.detach().float().cpu().double().numpy()


def check_f32(out, lse, ref_out, ref_lse, what=""):
    out, lse = f64(out), f64(lse)
    assert np.array_equal(np.isfinite(lse), np.isfinite(ref_lse)), what
    fin = np.isfinite(ref_lse)
    e_out = np.max(np.abs(out - ref_out)) if out.size else 0.0
    e_lse = np.max(np.abs(lse[fin] - ref_lse[fin])) if fin.any() else 0.0
    assert e_out <= F32_TOL, f"{what}: OUT max-abs {e_out}"
    assert e_lse <= F32_TOL, f"{what}: LSE max-abs {e_lse}"


def check_bf16(out, lse, ref_out, ref_lse, what=""):
    out, lse = f64(out), f64(lse)
    e_out = np.max(np.abs(out - ref_out))
    rel = np.linalg.norm(out - ref_out) / np.linalg.norm(ref_out)
    e_lse = np.max(np.abs(lse - ref_lse))
    assert e_out <= BF16_OUT_ABS, f"{what}: OUT max-abs {e_out}"
    assert rel <= BF16_OUT_RELFRO, f"{what}: OUT rel-Frobenius {rel}"
    assert e_lse <= BF16_LSE_ABS, f"{what}: LSE max-abs {e_lse}"


# ---------------------------------------------------------------------------
# state composition
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N", [1, 5, 37])
def test_compose_small(api, d, N):
    rows = 1003
    g = torch.Generator().manual_seed(N * 1000 + d)
    outs = torch.randn(N, rows, d, generator=g)
    lses = 5 + 2 * torch.randn(N, rows, generator=g)
    lses[:, 7] = -math.inf                     # a row with only empty states
    if N > 1:
        lses[0, 11:40] = -math.inf             # some empty states
    out, lse = api.as_compose(outs.cuda(), lses.cuda())
    ref_o, ref_l = O.compose([(outs[k].double().numpy(), lses[k].double().numpy()) for k in range(N)])
    check_f32(out, lse, ref_o, ref_l, f"compose N={N} d={d}")
    assert torch.all(out[7] == 0) and lse[7].item() == -math.inf


def test_compose_bound_full(api):
    s = W.spec("compose_bound")
    outs, lses = W.compose_states(s, device="cuda")
    out, lse = api.as_compose(outs, lses)
    torch.cuda.synchronize()
    rows = torch.randperm(outs.shape[1], generator=torch.Generator().manual_seed(5))[:4096].cuda()
    ref_o, ref_l = O.compose([(f64(outs[k, rows]), f64(lses[k, rows])) for k in range(s.n_states)])
    check_f32(out[rows], lse[rows], ref_o, ref_l, "compose_bound sampled rows")


# ---------------------------------------------------------------------------
# fp32 partition attention (CUDA cores)
# ---------------------------------------------------------------------------

def test_attn_f32_tiny(api):
    s = W.spec("tiny_f32")
    q, k, v = W.iid_qkv(s)
    qn, kn, vn = (x.double().numpy() for x in (q, k, v))
    qc, kc, vc = (x.cuda() for x in (q, k, v))
    full_o, full_l = O.full_attention(qn, kn, vn, s.scale)
    out, lse = api.as_partition_attn(qc, kc, vc, s.P, -1, list(range(s.P)), compose=True)
    check_f32(out, lse, full_o, full_l, "f32 composed over all partitions")
    order = W.merge_order(s.P)
    po, pl = api.as_partition_attn(qc, kc, vc, s.P, -1, order, compose=False)
    ref = O.partition_states(qn, kn, vn, s.scale, s.P)
    for x, j in enumerate(order):
        check_f32(po[x], pl[x], ref[j][0], ref[j][1], f"f32 state of partition {j}")
    co, cl = api.as_compose(po.contiguous(), pl.contiguous())  # composed in the seeded random order
    check_f32(co, cl, full_o, full_l, "f32 partition states composed in random order")
    n = s.n
    for i in range(s.P):
        oi, li = api.as_partition_attn(qc, kc, vc, s.P, i, [3, 1], compose=True)
        ref_o, ref_l = O.compose([O.attention_state(qn[..., i * n:(i + 1) * n, :], kn[..., a:b, :],
                                                    vn[..., a:b, :], s.scale)
                                  for a, b in [(3 * n, 4 * n), (n, 2 * n)]])
        check_f32(oi, li, ref_o, ref_l, f"f32 q_part {i}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_attn_and_step_with_a_given_scale(api, dtype):
    """A softmax scale other than 1/sqrt(d), through the CUDA-core (fp32) and
    the tensor-core (bf16) kernels and through a reuse step."""
    scale = 0.2
    if dtype == "f32":
        s = W.spec("tiny_f32")
        q, k, v = W.iid_qkv(s)
        check = check_f32
    else:
        s = W.spec("flux_image", H=2, S=640, P=5)
        q, k, v = W.flux_qkv(s)
        check = check_bf16
    qn, kn, vn = (x.double().numpy() for x in (q, k, v))
    qc, kc, vc = (x.cuda() for x in (q, k, v))
    full_o, full_l = O.full_attention(qn, kn, vn, scale)
    out, lse = api.as_partition_attn(qc, kc, vc, s.P, -1, list(range(s.P)), scale=scale)
    check(out, lse, full_o, full_l, f"{dtype} attention, scale {scale}")
    P = s.P
    near = np.abs(np.arange(P)[:, None] - np.arange(P)[None, :]) <= 1
    anchor_plan = np.where(near, 1, 2).astype(np.uint8)
    reuse_plan = np.where(near, 1, 0).astype(np.uint8)
    cache = api.AsCache(s.B, s.H, s.S, s.d, P)
    ocache = O.StateCache(P)
    for t, plan in enumerate([anchor_plan, reuse_plan]):
        out, lse, hit, age = api.as_step(cache, qc, kc, vc, plan, t, scale=scale)
        ref_o, ref_l, ref_hit, ref_age = O.step(ocache, qn, kn, vn, plan, t, scale)
        assert np.array_equal(hit, ref_hit) and np.array_equal(age, ref_age)
        check(out, lse, ref_o, ref_l, f"{dtype} step {t}, scale {scale}")


# ---------------------------------------------------------------------------
# bf16 partition attention (tensor cores)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("d,S,P,B", [(128, 1152, 2, 1), (64, 1152, 2, 2), (128, 640, 5, 1), (128, 384, 12, 1)])
def test_attn_bf16_small(api, d, S, P, B):
    s = W.spec("flux_image", B=B, H=3, S=S, d=d, P=P)
    q, k, v = W.flux_qkv(s)
    qn, kn, vn = (f64(x) for x in (q, k, v))
    qc, kc, vc = (x.cuda() for x in (q, k, v))
    full_o, full_l = O.full_attention(qn, kn, vn, s.scale)
    out, lse = api.as_partition_attn(qc, kc, vc, P, -1, list(range(P)), compose=True)
    check_bf16(out, lse, full_o, full_l, f"bf16 full d={d} S={S} P={P}")
    parts = list(range(P))[::-1]
    po, pl = api.as_partition_attn(qc, kc, vc, P, -1, parts, compose=False)
    ref = O.partition_states(qn, kn, vn, s.scale, P)
    for x, j in enumerate(parts):
        check_bf16(po[x], pl[x], ref[j][0], ref[j][1], f"bf16 partition {j}")
    n = S // P
    i = P - 1
    sel = [0, P - 1] if P > 1 else [0]
    oi, li = api.as_partition_attn(qc, kc, vc, P, i, sel, compose=True)
    ref_o, ref_l = O.compose([O.attention_state(qn[..., i * n:(i + 1) * n, :], kn[..., j * n:(j + 1) * n, :],
                                                vn[..., j * n:(j + 1) * n, :], s.scale) for j in sel])
    check_bf16(oi, li, ref_o, ref_l, "bf16 q_part, non-contiguous KV list")


def test_attn_bf16_flux_full(api):
    s = W.spec("flux_image")
    q, k, v = W.flux_qkv(s, device="cuda")
    out, lse = api.as_partition_attn(q, k, v, s.P, -1, list(range(s.P)), compose=True)
    torch.cuda.synchronize()
    heads = [0, 11, 23]
    rows = W.sample_rows(s, 16)
    qn = f64(q[:, heads][:, :, rows])
    kn, vn = f64(k[:, heads]), f64(v[:, heads])
    ref_o, ref_l = O.full_attention(qn, kn, vn, s.scale)
    check_bf16(out[:, heads][:, :, rows], lse[:, heads][:, :, rows], ref_o, ref_l, "flux_image sampled rows")


@pytest.mark.parametrize("H,S,P,d", [(96, 512, 4, 128), (200, 128, 1, 64), (80, 640, 5, 128)])
def test_attn_bf16_many_heads(api, H, S, P, d):
    """More 256-row CTAs than SMs over many heads: one KV tile per CTA
    (S = 128), a ragged last row block (S = 640: 2.5 blocks of 256 rows per
    head), and one state per KV partition (several accumulation groups per
    CTA)."""
    s = W.spec("flux_image", B=1, H=H, S=S, d=d, P=P)
    q, k, v = W.flux_qkv(s)
    qc, kc, vc = (x.cuda() for x in (q, k, v))
    heads = [0, 1, H // 2, H - 2, H - 1]
    qn, kn, vn = (f64(x[:, heads]) for x in (q, k, v))
    out, lse = api.as_partition_attn(qc, kc, vc, P, -1, list(range(P)), compose=True)
    full_o, full_l = O.full_attention(qn, kn, vn, s.scale)
    check_bf16(out[:, heads], lse[:, heads], full_o, full_l, f"composite H={H} S={S}")
    po, pl = api.as_partition_attn(qc, kc, vc, P, -1, list(range(P)), compose=False)
    ref = O.partition_states(qn, kn, vn, s.scale, P)
    for j in range(P):
        check_bf16(po[j][:, heads], pl[j][:, heads], ref[j][0], ref[j][1], f"partition {j} H={H} S={S}")


def test_step_store_then_reuse_many_heads(api):
    """An anchor step that stores every pair (one accumulation group per KV
    partition, the same for every query partition, so one launch block of all
    rows), then a step that reuses every stored entry, over 96 heads."""
    s = W.spec("flux_image", B=1, H=96, S=512, P=4)
    q, k, v = (x.cuda() for x in W.flux_qkv(s))
    plans = [np.full((4, 4), 2, np.uint8), np.zeros((4, 4), np.uint8)]
    _run_steps(api, s, [(q, k, v), (q, k, v)], plans, heads=[0, 47, 95])


# ---------------------------------------------------------------------------
# steps under a compute/reuse plan
# ---------------------------------------------------------------------------

def _run_steps(api, s, qkv_steps, plans, rows=None, heads=None, dtype_check=check_bf16):
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P)
    ocache = O.StateCache(s.P)
    for t, (q, k, v) in enumerate(qkv_steps):
        plan = plans[t]
        out, lse, hit, age = api.as_step(cache, q, k, v, plan, t)
        torch.cuda.synchronize()
        hs = slice(None) if heads is None else heads
        qn = f64(q[:, hs])
        kn, vn = f64(k[:, hs]), f64(v[:, hs])
        r = np.arange(s.S) if rows is None else np.asarray(rows)
        ref_o, ref_l, ref_hit, ref_age = O.step(ocache, qn, kn, vn, np.asarray(plan), t, s.scale, rows=r)
        assert np.array_equal(hit, ref_hit), f"hit at step {t}"
        assert np.array_equal(age, ref_age), f"age at step {t}"
        assert np.array_equal(cache.t_c, ocache.t_c), f"t_c at step {t}"
        rt = torch.as_tensor(r, device=out.device)
        dtype_check(out[:, hs][:, :, rt], lse[:, hs][:, :, rt], ref_o, ref_l, f"step {t}")
    return cache


@pytest.mark.parametrize("rows_,cols_", [(4, 8), (12, 16)])
def test_step_video_reuse_small(api, rows_, cols_):
    s = W.spec("video_reuse", H=2, rows=rows_, cols=cols_, S=16 * rows_ * cols_)
    steps = [(q.cuda(), k.cuda(), v.cuda()) for _, q, k, v in W.video_trajectory(s)]
    plans = [W.plan_for_step(s, t).numpy() for t in range(s.steps)]
    _run_steps(api, s, steps, plans)


def test_step_video_long_small(api):
    s = W.spec("video_long", H=2, rows=8, cols=16, S=16 * 8 * 16)
    steps = [(q.cuda(), k.cuda(), v.cuda()) for _, q, k, v in W.video_trajectory(s)]
    plans = [W.plan_for_step(s, t).numpy() for t in range(s.steps)]
    assert any((p == W.PLAN_FRESH_STORE).any() for p in plans[1:])
    _run_steps(api, s, steps, plans)


def test_step_video_reuse_full(api):
    s = W.spec("video_reuse")
    steps = [(q, k, v) for _, q, k, v in W.video_trajectory(s, device="cuda")]
    plans = [W.plan_for_step(s, t).numpy() for t in range(s.steps)]
    _run_steps(api, s, steps, plans, rows=W.sample_rows(s, 8).numpy(), heads=[0, 13, 23])


def test_step_video_long_full(api):
    """The long-trajectory workload at full size (S=65536, H=40, P=32, 4 steps,
    a 43 GB state cache) in the benchmark's launch configuration: seeded
    samples of 4 rows per partition on two heads against the oracle, plus the
    whole hit/age/store bookkeeping, which must be bit-exact."""
    s = W.spec("video_long")
    steps = [(q, k, v) for _, q, k, v in W.video_trajectory(s, device="cuda")]
    plans = [W.plan_for_step(s, t).numpy() for t in range(s.steps)]
    _run_steps(api, s, steps, plans, rows=W.sample_rows(s, 4).numpy(), heads=[0, 39])
    del steps
    torch.cuda.empty_cache()


def test_step_f32_with_reuse(api):
    s = W.spec("tiny_f32", P=8)
    q, k, v = (x.cuda() for x in W.iid_qkv(s))
    k2 = k + 0.1 * torch.randn(k.shape, generator=torch.Generator(device="cuda").manual_seed(3), device="cuda")
    plans = [np.where(np.abs(np.arange(8)[:, None] - np.arange(8)[None, :]) <= 1, 1, 2).astype(np.uint8),
             np.where(np.abs(np.arange(8)[:, None] - np.arange(8)[None, :]) <= 1, 1, 0).astype(np.uint8)]
    _run_steps(api, s, [(q, k, v), (q, k2, v)], plans, dtype_check=check_f32)


def test_step_all_fresh_equals_attention(api):
    s = W.spec("flux_image", H=2, S=576 * 4, P=4)
    q, k, v = (x.cuda() for x in W.flux_qkv(s))
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P)
    out, lse, hit, age = api.as_step(cache, q, k, v, W.all_fresh_plan(s.P).numpy(), 0)
    ref_out, ref_lse = api.as_partition_attn(q, k, v, s.P, -1, list(range(s.P)))
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    assert not hit.any() and not age.any() and (cache.t_c == -1).all()


def test_step_fixture_on_gpu(api):
    """The hand-computed plan fixture replayed through as_step: bit-exact hit,
    age and store timestamps, misses and invalid plans change nothing, and
    every step's states match the oracle."""
    from tests._golden import load_plan_fixture
    from attention_state_reuse_partition_b200 import _lib
    P, cases = load_plan_fixture()
    s = W.spec("flux_image", H=2, S=64 * P, d=64, P=P)
    q, k, v = (x.cuda() for x in W.flux_qkv(s))
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P)
    ocache = O.StateCache(P)
    qn, kn, vn = (f64(x) for x in (q, k, v))
    for c in cases:
        if c["expect"] in ("cache_miss", "invalid"):
            before = cache.t_c
            with pytest.raises(api.AsError) as ei:
                api.as_step(cache, q, k, v, c["plan"], c["step"])
            want = _lib.AS_ERR_CACHE_MISS if c["expect"] == "cache_miss" else _lib.AS_ERR_INVALID_ARG
            assert ei.value.status == want
            assert np.array_equal(cache.t_c, before)
            continue
        out, lse, hit, age = api.as_step(cache, q, k, v, c["plan"], c["step"])
        assert np.array_equal(hit, c["hit"]) and np.array_equal(age, c["age"])
        ref_o, ref_l, _, _ = O.step(ocache, qn, kn, vn, c["plan"], c["step"], s.scale)
        assert np.array_equal(cache.t_c, ocache.t_c)
        check_bf16(out, lse, ref_o, ref_l, f"fixture step {c['step']}")


# ---------------------------------------------------------------------------
# failure detection: a bounded wait that runs out, without faulting the GPU
# ---------------------------------------------------------------------------

def test_timeout_is_reported_and_context_survives(api):
    from attention_state_reuse_partition_b200 import _lib
    assert api.as_device_status() == 0
    api.as_debug_timeout_probe(64)
    with pytest.raises(api.AsError) as ei:
        api.as_device_status()
    assert ei.value.status == _lib.AS_ERR_TIMEOUT
    assert api.as_device_status() == 0  # cleared
    outs = torch.randn(3, 64, 128, device="cuda")
    lses = torch.randn(3, 64, device="cuda")
    out, lse = api.as_compose(outs, lses)
    ref_o, ref_l = O.compose([(f64(outs[k]), f64(lses[k])) for k in range(3)])
    check_f32(out, lse, ref_o, ref_l, "after timeout")


def test_timeout_deadline_in_gpu_time(api):
    """The kernels bound each wait in time, not in polls: a probe with an
    unlimited poll count and a 20 ms limit gives up after 20 ms of GPU time
    (%globaltimer) and reports AS_ERR_TIMEOUT; the host sees the launch end
    within a bounded wall time, and the context still works afterwards."""
    import time
    from attention_state_reuse_partition_b200 import _lib
    assert api.as_device_status() == 0
    limit_ns = 20_000_000
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    api.as_debug_timeout_probe(0xFFFFFFFF, limit_ns)
    with pytest.raises(api.AsError) as ei:
        api.as_device_status()          # synchronises
    wall = time.perf_counter() - t0
    assert ei.value.status == _lib.AS_ERR_TIMEOUT
    assert limit_ns * 1e-9 <= wall < 2.0, wall
    assert api.as_device_status() == 0
    x = torch.randn(1 << 10, device="cuda")
    assert torch.allclose(api.as_debug_exp2(x, 1), torch.exp2(x), rtol=1e-5)


# ---------------------------------------------------------------------------
# the two exp2 evaluations mixed in the softmax, against CUDA's exp2
# ---------------------------------------------------------------------------

def test_exp2_paths_against_cuda(api):
    x = torch.linspace(-124.9, 9.0, 1 << 22, device="cuda")
    ref = torch.exp2(x.double())
    for mode, tol in ((0, 4e-6), (1, 2e-6)):
        y = api.as_debug_exp2(x, mode).double()
        rel = ((y / ref) - 1).abs().max().item()
        assert rel < tol, (mode, rel)
    masked = api.as_debug_exp2(torch.tensor([-math.inf, -200.0], device="cuda"), 0)
    assert torch.all(masked > 0) and torch.all(masked < 3e-38)
