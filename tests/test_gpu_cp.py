"""Context parallelism through the C ABI on one GPU: every rank of a 2- and a
3-way split is run in turn (its rows of Q, its own cache, and the compact
K/V buffer that the exchange would give it, gathered locally), four steps of
the long-trajectory construction with forced-fresh pairs.  Each rank's
states must match the float64 oracle's rows at the bf16 tolerances, and its
hit and age bit for bit; and, rank by rank, the single-GPU as_step's rows
within the same bounds.  (The exchange itself is tested with gloo in
test_cp.py; ranks whose kernels waited on one another are never run on one
GPU here -- each rank's step is independent.)"""
import numpy as np
import pytest
import torch

from attention_state_reuse_partition_b200 import workloads as W
from oracle import as_oracle as O
from tests.test_gpu_parity import check_bf16, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from attention_state_reuse_partition_b200 import build
    build.build()
    from attention_state_reuse_partition_b200 import api as a
    return a


@pytest.mark.parametrize("world,g,cache_dt", [(2, 1, "f32"), (3, 1, "f32"), (3, 4, "bf16")])
def test_step_cp_ranks_against_oracle(api, world, g, cache_dt):
    from attention_state_reuse_partition_b200 import cp
    s = W.spec("video_long", H=2, rows=8, cols=16, S=16 * 8 * 16)
    n = s.n
    layout = cp.CpLayout(s.P, world)
    steps = [(q.cuda(), k.cuda(), v.cuda()) for _, q, k, v in W.video_trajectory(s)]
    plans = [W.grouped_plan_for_step(s, t, g).numpy() for t in range(s.steps)]
    gcache = api.AsCache(s.B, s.H, s.S, s.d, s.P, g=g, cache_dtype=cache_dt)
    caches = [api.AsCache(s.B, s.H, s.S, s.d, s.P, g=g, cache_dtype=cache_dt, q_first=layout.parts(r).start,
                          q_count=len(layout.parts(r))) for r in range(world)]
    ocache = O.StateCache(s.P, g, cache_dt)
    for t, (q, k, v) in enumerate(steps):
        plan = plans[t]
        gout, glse, ghit, gage = api.as_step(gcache, q, k, v, plan, t)
        ref_o, ref_l, ref_hit, ref_age = O.step(ocache, f64(q), f64(k), f64(v), plan, t, s.scale)
        moved = 0
        for r in range(world):
            mine = layout.parts(r)
            rows = slice(mine.start * n, mine.stop * n)
            need = cp.needed_kv(plan, mine)
            k_buf, v_buf, slots = cp.gather_kv_local(k, v, need, n)
            out, lse, hit, age = api.as_step_cp(caches[r], q[:, :, rows].contiguous(), k_buf, v_buf, slots, plan, t)
            torch.cuda.synchronize()
            assert np.array_equal(hit[list(mine)], ref_hit[list(mine)]), (world, r, t)
            assert np.array_equal(age[list(mine)], ref_age[list(mine)]), (world, r, t)
            assert hit[[i for i in range(s.P) if i not in mine]].sum() == 0
            check_bf16(out, lse, ref_o[:, :, rows], ref_l[:, :, rows], f"world {world} rank {r} step {t}")
            check_bf16(out, lse, f64(gout[:, :, rows]), f64(glse[:, :, rows]), f"rank {r} vs as_step, step {t}")
            moved += len([j for j in need if j not in mine])
        if t > 0 and g == 1:
            # per-pair entries: the reused pairs move nothing, so less than an
            # all-gather (with groups, a forced pair refreshes its whole group
            # and a rank may need every partition)
            assert moved < sum(s.P - len(layout.parts(r)) for r in range(world))
