"""Seeded synthetic inputs for the attention-state workloads.

This module draws random numbers and lays them out; it holds none of the
method's arithmetic (no attention, no state composition, no plan resolution).
Both the CUDA path and the float64 oracle consume what it produces, so every
parity comparison sees identical inputs.

Seeding: every tensor comes from its own ``torch.Generator`` seeded with
``BASE_SEED * 1000 + stream_id`` on the device the tensor is drawn on.  Stream
ids: q=0, k=1, v=2, Fourier frequencies=3, compose OUT=4, compose LSE=5,
per-step noise=10+t (q, k, v offset by 0/100/200... see ``_STREAM``),
plan draws=1000+t, merge order=2000, row samples=3000.  A CPU draw and a CUDA
draw with the same seed give different numbers; callers that need the same
data on both sides draw once and copy.

Workloads (shapes follow the DiT attention settings that DiTango, Fig. 11 and
§6, and the FLUX-style image DiTs of FastUSP evaluate; the data itself is
synthetic):

* ``tiny_f32``      B=1 H=2 S=256 d=64, fp32 N(0,1), P=4.
* ``flux_image``    B=1 H=24 S=4608 (4096 image + 512 text) d=128, bf16,
                    Q,K per-head RMS-normalised 0.5*N(0,1), V 0.5*N(0,1), P=8.
* ``video_reuse``   B=1 H=24 S=32768 (16 frames x 32x64) d=128, bf16, P=16,
                    Fourier-feature locality, random-walk step dynamics,
                    reuse window 2, two steps (anchor + reuse).
* ``video_long``    B=1 H=40 S=65536 (16 frames x 64x64) d=128, bf16, P=32,
                    AR(1) rho=0.98 dynamics over 4 steps, window 4, a seeded
                    10% of reused pairs forced fresh each non-anchor step.
* ``compose_bound`` B=2 H=24 S=16384 d=128, 32 fp32 states per row, OUT
                    N(0,1), LSE N(5, 2^2).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterator, Optional

import torch

BASE_SEED = 20261202

_STREAM = {
    "q": 0, "k": 1, "v": 2, "omega": 3, "c_out": 4, "c_lse": 5,
    "merge_order": 2000, "rows": 3000,
}

# plan codes shared by every consumer of a plan matrix (values, not arithmetic)
PLAN_REUSE = 0          # read the cached state of the pair
PLAN_FRESH = 1          # compute the pair's state now, leave the cache alone
PLAN_FRESH_STORE = 2    # compute the pair's state now and refresh its cache entry


def _gen(device, stream_id: int, seed: int = BASE_SEED) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(seed * 1000 + int(stream_id))
    return g


def _randn(shape, device, stream_id, seed=BASE_SEED, dtype=torch.float32):
    return torch.randn(shape, generator=_gen(device, stream_id, seed),
                       device=device, dtype=dtype)


@dataclasses.dataclass(frozen=True)
class Spec:
    name: str
    dtype: str              # "f32" or "bf16" (input dtype of Q, K, V)
    B: int
    H: int
    S: int
    d: int
    P: int
    frames: int = 0         # video layout (0 = not a video workload)
    rows: int = 0
    cols: int = 0
    window: int = -1        # |i-j| <= window computed fresh on non-anchor steps
    steps: int = 1
    dynamics: str = ""      # "walk" (x_t = x_{t-1} + sigma*N) or "ar1"
    sigma: float = 0.0      # walk step size
    rho: float = 0.0        # AR(1) coefficient
    forced_frac: float = 0.0
    n_states: int = 0       # compose-bound workload: states per row
    seed: int = BASE_SEED

    @property
    def n(self) -> int:
        return self.S // self.P

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def scaled(self, **kw) -> "Spec":
        return dataclasses.replace(self, **kw)


SPECS = {
    "tiny_f32": Spec("tiny_f32", "f32", B=1, H=2, S=256, d=64, P=4),
    "flux_image": Spec("flux_image", "bf16", B=1, H=24, S=4608, d=128, P=8),
    "video_reuse": Spec("video_reuse", "bf16", B=1, H=24, S=32768, d=128, P=16,
                        frames=16, rows=32, cols=64, window=2, steps=2,
                        dynamics="walk", sigma=0.05),
    "video_long": Spec("video_long", "bf16", B=1, H=40, S=65536, d=128, P=32,
                       frames=16, rows=64, cols=64, window=4, steps=4,
                       dynamics="ar1", rho=0.98, forced_frac=0.10),
    "compose_bound": Spec("compose_bound", "f32", B=2, H=24, S=16384, d=128, P=32,
                          n_states=32),
}


def spec(name: str, **overrides) -> Spec:
    s = SPECS[name]
    return s.scaled(**overrides) if overrides else s


def _to_input_dtype(x: torch.Tensor, dtype: str) -> torch.Tensor:
    # round-to-nearest-even from the fp32 master
    return x.to(torch.bfloat16) if dtype == "bf16" else x.contiguous()


# --------------------------------------------------------------------------
# tiny_f32 and flux_image: single-step inputs
# --------------------------------------------------------------------------

def iid_qkv(s: Spec, device="cpu"):
    """Q, K, V i.i.d. N(0,1), shape [B,H,S,d], in the workload's dtype."""
    shape = (s.B, s.H, s.S, s.d)
    q = _randn(shape, device, _STREAM["q"], s.seed)
    k = _randn(shape, device, _STREAM["k"], s.seed)
    v = _randn(shape, device, _STREAM["v"], s.seed)
    return tuple(_to_input_dtype(x, s.dtype) for x in (q, k, v))


def flux_qkv(s: Spec, device="cpu", eps: float = 1e-6):
    """FLUX-like image-DiT attention inputs.

    Q and K are 0.5*N(0,1) followed by per-head RMS normalisation over d (the
    QK-norm of FLUX-style DiTs), V is 0.5*N(0,1).  Text tokens sit after the
    image tokens; with no reuse their position does not matter.
    """
    shape = (s.B, s.H, s.S, s.d)
    q = 0.5 * _randn(shape, device, _STREAM["q"], s.seed)
    k = 0.5 * _randn(shape, device, _STREAM["k"], s.seed)
    v = 0.5 * _randn(shape, device, _STREAM["v"], s.seed)
    q = q * torch.rsqrt(q.pow(2).mean(-1, keepdim=True) + eps)
    k = k * torch.rsqrt(k.pow(2).mean(-1, keepdim=True) + eps)
    return tuple(_to_input_dtype(x, s.dtype) for x in (q, k, v))


# --------------------------------------------------------------------------
# video workloads: Fourier-feature locality and step dynamics
# --------------------------------------------------------------------------

def fourier_features(s: Spec, device="cpu", bandwidth: float = 0.1) -> torch.Tensor:
    """g[h, token, :] = [cos(w_k . x), sin(w_k . x)] for d/2 random frequencies.

    x = (frame/(F-1), row/(R-1), col/(C-1)) with tokens ordered frame-major,
    then row, then column.  Each frequency component is N(0, (1/bandwidth)^2),
    drawn per head.  Returns fp32 [H, S, d].
    """
    assert s.frames * s.rows * s.cols == s.S, "video layout must cover S"
    nf = s.d // 2
    omega = _randn((s.H, nf, 3), device, _STREAM["omega"], s.seed) / bandwidth
    f = torch.arange(s.frames, device=device, dtype=torch.float32) / max(s.frames - 1, 1)
    r = torch.arange(s.rows, device=device, dtype=torch.float32) / max(s.rows - 1, 1)
    c = torch.arange(s.cols, device=device, dtype=torch.float32) / max(s.cols - 1, 1)
    grid = torch.stack(torch.meshgrid(f, r, c, indexing="ij"), dim=-1).reshape(s.S, 3)
    phase = torch.einsum("sx,hkx->hsk", grid, omega)
    return torch.cat([torch.cos(phase), torch.sin(phase)], dim=-1)


def video_trajectory(s: Spec, device="cpu") -> Iterator[tuple]:
    """Yields (step, q, k, v) for steps 0..s.steps-1.

    Q = 0.5*z_q + g, K = 0.5*z_k + g, V = 0.5*z_v, with z the per-tensor noise
    state.  ``walk``: z_t = z_{t-1} + (sigma/0.5)*N(0,1), i.e. the inputs move
    by sigma*N(0,1) per step.  ``ar1``: z_t = rho*z_{t-1} + sqrt(1-rho^2)*eps_t
    with g fixed.  bf16 rounding is applied to each step's fp32 masters.
    """
    shape = (s.B, s.H, s.S, s.d)
    g = fourier_features(s, device).unsqueeze(0)
    z = {n: _randn(shape, device, _STREAM[n], s.seed) for n in ("q", "k", "v")}
    for t in range(s.steps):
        if t > 0:
            for idx, n in enumerate(("q", "k", "v")):
                eps = _randn(shape, device, 10 + t + 100 * idx, s.seed)
                if s.dynamics == "walk":
                    z[n].add_(eps, alpha=s.sigma / 0.5)
                elif s.dynamics == "ar1":
                    z[n].mul_(s.rho).add_(eps, alpha=math.sqrt(1.0 - s.rho * s.rho))
                else:
                    raise ValueError(f"unknown dynamics {s.dynamics!r}")
                del eps
        q = _to_input_dtype(0.5 * z["q"] + g, s.dtype)
        k = _to_input_dtype(0.5 * z["k"] + g, s.dtype)
        v = _to_input_dtype(0.5 * z["v"], s.dtype)
        yield t, q, k, v


def plan_for_step(s: Spec, t: int):
    """Plan matrix (uint8 [P, P], rows = query partition i, cols = KV partition j).

    Step 0 is an anchor: every pair fresh; pairs outside the window store their
    state so that later steps can reuse it.  Later steps: |i-j| <= window fresh
    (not stored), the rest reused, except a seeded ``forced_frac`` of the
    reused pairs (round(frac * #reused), drawn without replacement per step),
    which are computed fresh and refresh their cache entry.
    """
    P = s.P
    i = torch.arange(P).unsqueeze(1)
    j = torch.arange(P).unsqueeze(0)
    near = (i - j).abs() <= s.window if s.window >= 0 else torch.ones(P, P, dtype=torch.bool)
    plan = torch.empty(P, P, dtype=torch.uint8)
    if t == 0:
        plan[near] = PLAN_FRESH
        plan[~near] = PLAN_FRESH_STORE
        return plan
    plan[near] = PLAN_FRESH
    plan[~near] = PLAN_REUSE
    far = (~near).flatten().nonzero().flatten()
    n_forced = int(round(s.forced_frac * far.numel()))
    if n_forced > 0:
        perm = torch.randperm(far.numel(), generator=_gen("cpu", 1000 + t, s.seed))
        plan.view(-1)[far[perm[:n_forced]]] = PLAN_FRESH_STORE
    return plan


def grouped_plan_for_step(s: Spec, t: int, g: int):
    """plan_for_step for a cache of groups of g KV partitions (group j // g).

    A group is stored or reused as a whole, so the per-pair plan is lifted to
    groups: for query partition i and group G, the members outside the window
    are stored if the pair plan stores any of them (the anchor, or a forced
    pair), else reused; members inside the window stay fresh.
    """
    base = plan_for_step(s, t)
    plan = base.clone()
    P = s.P
    for i in range(P):
        for G in range((P + g - 1) // g):
            js = [j for j in range(G * g, min((G + 1) * g, P)) if base[i, j] != PLAN_FRESH]
            if not js:
                continue
            code = PLAN_FRESH_STORE if any(base[i, j] == PLAN_FRESH_STORE for j in js) else PLAN_REUSE
            for j in js:
                plan[i, j] = code
    return plan


def all_fresh_plan(P: int):
    return torch.full((P, P), PLAN_FRESH, dtype=torch.uint8)


def merge_order(n: int, seed: int = BASE_SEED):
    """A seeded random permutation used to compose states in random order."""
    return torch.randperm(n, generator=_gen("cpu", _STREAM["merge_order"], seed)).tolist()


def sample_rows(s: Spec, per_partition: int, seed_offset: int = 0) -> torch.Tensor:
    """Seeded sample of query rows: ``per_partition`` distinct rows in every
    query partition (sorted, int64 token indices in [0, S))."""
    g = _gen("cpu", _STREAM["rows"] + seed_offset, s.seed)
    n = s.n
    k = min(per_partition, n)
    out = []
    for i in range(s.P):
        out.append(i * n + torch.randperm(n, generator=g)[:k].sort().values)
    return torch.cat(out)


# --------------------------------------------------------------------------
# compose_bound: precomputed states
# --------------------------------------------------------------------------

def compose_states(s: Spec, device="cpu", rows: Optional[int] = None):
    """N states per row: OUT fp32 [N, rows, d] ~ N(0,1), LSE fp32 [N, rows]
    ~ N(5, 2^2), rows = B*H*S (row-major over b, h, s) unless overridden."""
    R = rows if rows is not None else s.B * s.H * s.S
    out = _randn((s.n_states, R, s.d), device, _STREAM["c_out"], s.seed)
    lse = 5.0 + 2.0 * _randn((s.n_states, R), device, _STREAM["c_lse"], s.seed)
    return out, lse
