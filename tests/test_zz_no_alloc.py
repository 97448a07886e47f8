"""The allocation-free drift entry point (as_plan_drift_static), for callers
that cannot allocate device memory and so cannot pass the scratch buffer
as_plan_drift needs.  Collected last, so that a run that stops at the first
failure has already run every other test.

It must agree with as_plan_drift (same kernels, caller scratch) within the
reductions' tolerance (relative 1e-9), on two calls in a row -- the second
call finds the first call's contents in the shared fixed scratch -- and must
reject sizes beyond its fixed scratch with a clear error."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def api():
    from attention_state_reuse_partition_b200 import build
    build.build()
    from attention_state_reuse_partition_b200 import api as a
    return a


def _inputs(seed, B, H, S, d):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return (torch.randn((B, H, S, d), generator=g, device="cuda"),
            torch.randn((B, H, S, d), generator=g, device="cuda"))


def test_static_drift_matches_scratch_variant_twice(api):
    for call, (B, H, S, d, P) in enumerate([(1, 24, 16 * 256, 128, 16), (2, 3, 5 * 192, 64, 5)]):
        now, anc = _inputs(100 + call, B, H, S, d)
        scratch = torch.empty(api.as_planner_scratch_bytes(B, H, P) // 8 + 1, dtype=torch.float64, device="cuda")
        ref_drift, ref_norm = api.as_plan_drift(now, anc, P, scratch)
        drift, norm = api.as_plan_drift_static(now, anc, P)
        assert np.all(np.abs(drift - ref_drift) <= 1e-9 * ref_drift), call
        assert np.all(np.abs(norm - ref_norm) <= 1e-9 * ref_norm), call


def test_static_drift_rejects_sizes_beyond_its_scratch(api):
    from attention_state_reuse_partition_b200 import _lib
    B, H, S, d, P = 1, 2048, 64, 64, 32  # P * (B*H*2 + 2) = 131136 > 131072
    now = torch.zeros((B, H, S, d), device="cuda")
    with pytest.raises(api.AsError) as ei:
        api.as_plan_drift_static(now, now, P)
    assert ei.value.status == _lib.AS_ERR_INVALID_ARG
    assert "fixed scratch" in str(ei.value)
