"""The planner on the GPU against the float64 oracle.

* local states: element-wise, with the bf16/fp32 tolerances of the parity
  tests;
* the drift and anchor-statistics reductions: on the same random fp32 inputs,
  against float64 NumPy sums (relative 1e-9);
* a planner trajectory: drift and ASE element by element, anchor decisions
  and plans against the oracle planner.  Floating point decides these
  integers, so a unit whose oracle ASE lies within a relative band of the
  selection threshold, or a step whose relative drift lies within the band
  around eps_local, may legitimately go either way; there the oracle follows
  the GPU's choice, everything else must match exactly, and every step's
  states, hit and age are compared with the oracle's under the same plan."""
import math

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


def _oracle_local(qn, kn, vn, P, scale):
    S = qn.shape[-2]
    n = S // P
    outs, lses = [], []
    for i in range(P):
        o, l = O.attention_state(qn[..., i * n:(i + 1) * n, :], kn[..., i * n:(i + 1) * n, :],
                                 vn[..., i * n:(i + 1) * n, :], scale)
        outs.append(o)
        lses.append(l)
    return np.concatenate(outs, axis=-2), np.concatenate(lses, axis=-1)


@pytest.mark.parametrize("dtype,S,P", [("bf16", 16 * 8 * 16, 16), ("bf16", 5 * 192, 5), ("f32", 256, 4)])
def test_local_states(api, dtype, S, P):
    if dtype == "bf16":
        s = W.spec("flux_image", H=2, S=S, P=P)
        q, k, v = W.flux_qkv(s)
        check = check_bf16
    else:
        s = W.spec("tiny_f32", P=P)
        q, k, v = W.iid_qkv(s)
        check = check_f32
    out, lse = api.as_local_states(q.cuda(), k.cuda(), v.cuda(), P)
    ref_o, ref_l = _oracle_local(f64(q), f64(k), f64(v), P, s.scale)
    check(out, lse, ref_o, ref_l, f"local states {dtype} S={S} P={P}")


def test_drift_reduction(api):
    g = torch.Generator(device="cuda").manual_seed(11)
    B, H, S, d, P = 1, 5, 640, 128, 5
    now = torch.randn((B, H, S, d), generator=g, device="cuda")
    anc = torch.randn((B, H, S, d), generator=g, device="cuda")
    scratch = torch.empty(api.as_planner_scratch_bytes(B, H, P) // 8 + 1, dtype=torch.float64, device="cuda")
    drift, norm = api.as_plan_drift(now, anc, P, scratch)
    nn, aa = f64(now), f64(anc)
    n = S // P
    for i in range(P):
        rd, rn = O.local_drift(nn[..., i * n:(i + 1) * n, :], aa[..., i * n:(i + 1) * n, :])
        assert abs(drift[i] - rd) <= 1e-9 * rd and abs(norm[i] - rn) <= 1e-9 * rn


def _units(P, g, window):
    """[P, n_groups] mask of the planner's units: groups with a member outside the window."""
    NG = (P + g - 1) // g
    return np.array([[any(abs(i - j) > window for j in range(G * g, min((G + 1) * g, P))) for G in range(NG)]
                     for i in range(P)])


@pytest.mark.parametrize("g,cache_dt", [(1, "f32"), (3, "f32"), (2, "bf16")])
def test_anchor_statistics(api, g, cache_dt):
    """commit_anchor on a cache filled with known random states: w and alpha
    of the stored entries (pairs, or groups of g) against float64 NumPy."""
    B, H, S, d, P, window = 1, 3, 8 * 64, 64, 8, 1
    n = S // P
    cache = api.AsCache(B, H, S, d, P, g=g, cache_dtype=cache_dt)
    outs, lses = cache.planes()
    gen = torch.Generator(device="cuda").manual_seed(12)
    outs.copy_(torch.randn(outs.shape, generator=gen, device="cuda"))
    lses.copy_(torch.randn(lses.shape, generator=gen, device="cuda") + 2.0)
    lse_full = torch.randn((B, H, S), generator=gen, device="cuda") + 4.0
    pl = api.AsPlanner(P, window, 0.5, 0.1, B, H, S, d, g=g)
    pl.local_anchor.copy_(torch.randn((B, H, S, d), generator=gen, device="cuda"))
    plan = O.anchor_plan(P, window)
    api.as_planner_commit_anchor(pl, cache, lse_full, plan)
    assert pl.has_anchor
    on, ln, lf, la = f64(outs), f64(lses), f64(lse_full), f64(pl.local_anchor)
    units = _units(P, g, window)
    for i in range(P):
        local_norm = O.frob(la[..., i * n:(i + 1) * n, :])
        for G in range(units.shape[1]):
            if not units[i, G]:
                assert pl.w[i, G] == 0.0
                continue
            w_ref = float(np.mean(np.exp(ln[G][..., i * n:(i + 1) * n] - lf[..., i * n:(i + 1) * n])))
            a_ref = O.frob(on[G][..., i * n:(i + 1) * n, :]) / local_norm
            assert abs(pl.w[i, G] - w_ref) <= 1e-9 * w_ref, (i, G)
            assert abs(pl.alpha[i, G] - a_ref) <= 1e-9 * a_ref, (i, G)


# Tolerances of the trajectory comparison.  The GPU's local states and cache
# entries come from bf16 inputs through the tensor-core path (P rounded to
# bf16 in the PV product), so a state's OUT differs from the float64 oracle by
# about 1e-3 relative.  The drift D(i) is the norm of the difference of two
# such states 0.1 to 0.4 apart (relative), so its relative error is about
# 1e-3 / 0.1 = 1e-2; w carries the LSE error (exp of <= 1e-3 absolute: 1e-3
# relative) and alpha the norm error of two states (~2e-3).  ASE = w alpha D
# then sits within about 1.5e-2; DRIFT_RTOL and ASE_RTOL leave a factor of two.
DRIFT_RTOL = 2e-2
ASE_RTOL = 3e-2
# a decision whose oracle margin is within BAND (relative) may go either way
BAND = 3e-2


def _rel_drift(local, anchor, P, n):
    return np.array([O.local_drift(local[..., i * n:(i + 1) * n, :], anchor[..., i * n:(i + 1) * n, :])[0]
                     / O.frob(anchor[..., i * n:(i + 1) * n, :]) for i in range(P)])


@pytest.mark.parametrize("g,cache_dt", [(1, "f32"), (4, "bf16")])
def test_planner_trajectory_against_oracle(api, g, cache_dt):
    """Seven steps of the planner on a small video trajectory (window 2,
    R = 0.6, eps_local = 0.4: the oracle anchors at steps 0 and 4 with
    margins of 6% or more and reuses at steps 1-3, 5 and 6).

    At every step: the anchor decision must match unless the oracle's
    relative drift lies within BAND of eps_local; at every reuse step the
    drift and the ASE of every unit are compared element by element with the
    oracle's, and the plan must match except on units whose oracle ASE lies
    within BAND of the selection threshold, where either choice is valid (the
    GPU's plan must still reuse exactly floor(R * #units) units).  Wherever
    the two may legitimately part, the oracle follows the GPU's decision, so
    the caches never diverge; then both run the step under the same plan and
    every state, hit and age is compared.  At least three reuse steps must be
    compared."""
    s = W.spec("video_long", H=2, rows=8, cols=16, S=16 * 8 * 16, steps=7)
    P, n, window, ratio, eps_local = s.P, s.n, 2, 0.6, 0.4
    steps = [(q.cuda(), k.cuda(), v.cuda()) for _, q, k, v in W.video_trajectory(s)]
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P, g=g, cache_dtype=cache_dt)
    pl = api.AsPlanner(P, window, ratio, eps_local, s.B, s.H, s.S, s.d, g=g)
    ocache = O.StateCache(P, g, cache_dt)
    opl = O.Planner(P, window, ratio, eps_local, g)
    units = _units(P, g, window)
    NG = units.shape[1]
    member_of = np.array([[j // g for j in range(P)] for _ in range(P)])  # [i, j] -> G
    reuse_steps = anchors = 0
    for t, (q, k, v) in enumerate(steps):
        qn, kn, vn = f64(q), f64(k), f64(v)
        local, _ = api.as_local_states(q, k, v, P)
        plan, is_anchor, ase = api.as_planner_next(pl, local)
        olocal, _ = _oracle_local(qn, kn, vn, P, s.scale)
        saved_anchor = None if opl.local_anchor is None else opl.local_anchor.copy()
        rel = _rel_drift(olocal, saved_anchor, P, n) if opl.has_anchor else None
        oplan, o_anchor, odrift, oase = O.planner_next(opl, olocal, n)
        if t == 0:
            assert is_anchor and o_anchor
        if is_anchor != o_anchor:
            assert abs(rel.max() - eps_local) <= BAND * eps_local, f"anchor decision at step {t}"
            if is_anchor:   # follow the GPU: the oracle anchors too
                opl.local_anchor = olocal.copy()
                oplan, oase = O.anchor_plan(P, window), None
            else:           # follow the GPU: the oracle keeps its anchor
                opl.local_anchor = saved_anchor
                oase = O.ase(opl.w, opl.alpha, odrift)
                oplan = O.select_plan(oase, window, ratio, g)
        if is_anchor:
            assert np.array_equal(plan, O.anchor_plan(P, window))
        else:
            reuse_steps += 1
            assert np.allclose(pl.drift, odrift, rtol=DRIFT_RTOL, atol=0), (t, pl.drift, odrift)
            assert np.allclose(ase[units], oase[units], rtol=ASE_RTOL, atol=0), \
                (t, float(np.max(np.abs(ase[units] / oase[units] - 1))))
            vals = np.sort(oase[units])
            k_reuse = int(np.floor(ratio * vals.size + 1e-9))
            thr = vals[k_reuse - 1] if k_reuse > 0 else -np.inf
            amb_units = units & (np.abs(oase - thr) <= BAND * max(abs(thr), 1e-30))
            ambiguous = np.take_along_axis(amb_units, member_of, axis=1)
            assert np.array_equal(plan[~ambiguous], oplan[~ambiguous]), f"plan at step {t}"
            reused_units = sum(bool((plan[i, G * g:(G + 1) * g] == O.PLAN_REUSE).any())
                               for i in range(P) for G in range(NG))
            assert reused_units == k_reuse
        # both run the GPU's plan: equal to the oracle's but for ambiguous units
        out, lse, hit, age = api.as_step(cache, q, k, v, plan, t)
        torch.cuda.synchronize()
        ref_o, ref_l, ref_hit, ref_age = O.step(ocache, qn, kn, vn, plan, t, s.scale)
        assert np.array_equal(hit, ref_hit) and np.array_equal(age, ref_age), f"hit/age at step {t}"
        check_bf16(out, lse, ref_o, ref_l, f"step {t}")
        if is_anchor:
            anchors += 1
            api.as_planner_commit_anchor(pl, cache, lse, plan)
            O.planner_commit_anchor(opl, ocache, ref_l, lambda i: np.arange(i * n, (i + 1) * n), n)
            assert np.allclose(pl.w[units], opl.w[units], rtol=5e-3, atol=0)
            assert np.allclose(pl.alpha[units], opl.alpha[units], rtol=2e-2, atol=0)
    assert anchors >= 2 and reuse_steps >= 3, (anchors, reuse_steps)
