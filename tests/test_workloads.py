"""The seeded input generators: shapes, determinism and plan structure."""
import math

import torch

from attention_state_reuse_partition_b200 import workloads as W


def test_specs_match_the_workload_table():
    assert W.spec("tiny_f32").S == 256 and W.spec("tiny_f32").n == 64
    assert W.spec("flux_image").n == 576
    v = W.spec("video_reuse")
    assert v.frames * v.rows * v.cols == v.S == 32768 and v.n == 2048
    lv = W.spec("video_long")
    assert lv.frames * lv.rows * lv.cols == lv.S == 65536 and lv.n == 2048
    assert W.spec("compose_bound").n_states == 32


def test_draws_are_deterministic():
    s = W.spec("tiny_f32")
    a = W.iid_qkv(s)
    b = W.iid_qkv(s)
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    assert a[0].dtype == torch.float32 and a[0].shape == (1, 2, 256, 64)


def test_flux_inputs_are_rms_normalised_bf16():
    s = W.spec("flux_image", H=2, S=576 * 2, P=2)
    q, k, v = W.flux_qkv(s)
    assert q.dtype == torch.bfloat16
    rms = q.float().pow(2).mean(-1).sqrt()
    assert torch.allclose(rms, torch.ones_like(rms), atol=1e-2)
    assert abs(v.float().std().item() - 0.5) < 0.02


def test_video_trajectory_dynamics():
    s = W.spec("video_reuse", H=2, S=16 * 4 * 8, rows=4, cols=8)
    steps = list(W.video_trajectory(s))
    assert len(steps) == 2
    (_, q0, k0, v0), (_, q1, k1, v1) = steps
    dv = (v1.float() - v0.float()).std().item()
    assert abs(dv - 0.05) < 0.01  # inputs move by 0.05*N(0,1) per step
    g = W.fourier_features(s)
    assert g.shape == (2, s.S, s.d)
    assert torch.allclose((g * g).sum(-1), torch.full((2, s.S), 64.0), atol=1e-3)


def test_ar1_keeps_the_noise_variance():
    s = W.spec("video_long", H=1, S=16 * 4 * 4, rows=4, cols=4, P=16)
    vs = [v.float() for _, _, _, v in W.video_trajectory(s)]
    for v in vs:
        assert abs(v.std().item() - 0.5) < 0.05
    corr = torch.corrcoef(torch.stack([vs[0].flatten(), vs[1].flatten()]))[0, 1].item()
    assert abs(corr - 0.98) < 0.01


def test_plans():
    s = W.spec("video_long")
    p0 = W.plan_for_step(s, 0)
    assert (p0 != W.PLAN_REUSE).all()
    i = torch.arange(s.P)[:, None]
    j = torch.arange(s.P)[None, :]
    near = (i - j).abs() <= s.window
    assert (p0[near] == W.PLAN_FRESH).all() and (p0[~near] == W.PLAN_FRESH_STORE).all()
    p1 = W.plan_for_step(s, 1)
    assert (p1[near] == W.PLAN_FRESH).all()
    n_far = int((~near).sum())
    assert int((p1 == W.PLAN_FRESH_STORE).sum()) == round(0.1 * n_far)
    assert not torch.equal(p1, W.plan_for_step(s, 2))
    assert torch.equal(p1, W.plan_for_step(s, 1))
    r = W.plan_for_step(W.spec("video_reuse"), 1)
    assert int((r == W.PLAN_FRESH).sum()) == 74 and int((r == W.PLAN_REUSE).sum()) == 182


def test_sample_rows():
    s = W.spec("video_reuse")
    rows = W.sample_rows(s, 8)
    assert rows.numel() == 8 * s.P
    assert torch.equal(rows, W.sample_rows(s, 8))
    assert ((rows // s.n) == torch.arange(s.P).repeat_interleave(8)).all()


def test_compose_states():
    s = W.spec("compose_bound")
    out, lse = W.compose_states(s, rows=1000)
    assert out.shape == (32, 1000, 128) and lse.shape == (32, 1000)
    assert abs(lse.mean().item() - 5) < 0.1 and abs(lse.std().item() - 2) < 0.1
