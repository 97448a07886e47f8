"""The checked build (libasp_debug.so, ASP_DEBUG=1) on the GPU.

compute-sanitizer is closed on this machine; the checked build is its stand-in:
device-side index checks before the stores whose indices come from a launch's
arguments, reporting through the device error word (no trap).

* a reuse trajectory (fresh, stored and reused pairs; groups with bf16
  entries), a strided compose and the residual codec give, in the checked
  build, results bit-identical to the normal build's, and a clean device
  status: no check fires on valid work;
* the bounds probe writes one past a logical length behind the check: the
  checked build refuses the write (the buffer keeps its value, and the
  status is AS_ERR_BOUNDS); the normal build refuses the probe itself.
The checked build runs in a child process (ASP_DEBUG=1 selects its library
when the binding loads)."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from attention_state_reuse_partition_b200 import api, _lib, workloads as W
def run():
    out = {}
    s = W.spec("video_long", H=2, rows=8, cols=16, S=16 * 8 * 16)
    for g, dt in ((1, "f32"), (4, "bf16")):
        cache = api.AsCache(s.B, s.H, s.S, s.d, s.P, g=g, cache_dtype=dt)
        for t, q, k, v in W.video_trajectory(s):
            plan = W.grouped_plan_for_step(s, t, g).numpy()
            o, l, _, _ = api.as_step(cache, q.cuda(), k.cuda(), v.cuda(), plan, t)
            out[f"step{g}{dt}{t}"] = o.cpu().numpy()
            out[f"lse{g}{dt}{t}"] = l.cpu().numpy()
    gen = torch.Generator(device="cuda").manual_seed(5)
    outs = torch.randn(5, 3000, 128, generator=gen, device="cuda")
    lses = torch.randn(5, 3000, generator=gen, device="cuda")
    o, l = api.as_compose(outs, lses)
    out["compose"] = o.cpu().numpy()
    x = torch.randn(999, 128, generator=gen, device="cuda").to(torch.bfloat16)
    base = (x.float() + 0.1).to(torch.bfloat16)
    c, sc = api.as_residual_encode(x, base)
    out["codes"] = c.cpu().numpy()
    out["base"] = base.float().cpu().numpy()
    api.as_device_status()
    return out
res = run()
buf = torch.zeros(64, device="cuda")
st = _lib.LIB.as_debug_bounds_probe(buf.data_ptr(), 32, None)
res["probe_status"] = np.array(st)
res["probe_dev"] = np.array(_lib.LIB.as_device_status(None, None)) if st == 0 else np.array(-1)
res["probe_buf"] = buf.cpu().numpy()
res["version"] = np.array(api.as_version())
np.savez(sys.argv[2], **res)
'''


def _run(tmp_path, checked):
    path = str(tmp_path / ("checked.npz" if checked else "normal.npz"))
    env = dict(os.environ)
    env["ASP_DEBUG"] = "1" if checked else "0"
    p = subprocess.run([sys.executable, "-c", CHILD, ROOT, path], env=env, capture_output=True, text=True,
                       timeout=600)
    assert p.returncode == 0, p.stderr[-3000:]
    return dict(np.load(path))


def test_checked_build_matches_and_refuses_out_of_range(tmp_path):
    from attention_state_reuse_partition_b200 import _lib, build
    build.build_all()
    normal = _run(tmp_path, False)
    checked = _run(tmp_path, True)
    assert "checked" in str(checked["version"]) and "checked" not in str(normal["version"])
    for key in normal:
        if key.startswith("probe") or key == "version":
            continue
        assert np.array_equal(normal[key], checked[key]), key
    assert int(normal["probe_status"]) == _lib.AS_ERR_UNSUPPORTED
    assert int(checked["probe_status"]) == _lib.AS_OK
    assert int(checked["probe_dev"]) == _lib.AS_ERR_BOUNDS
    assert not checked["probe_buf"].any()      # the write one past the end was skipped
