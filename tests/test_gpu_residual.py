"""The residual codec of the context-parallel exchange on the GPU
(CompactFusion, arXiv 2507.17511, Abstract on its listing page: compressed
step-wise residuals with error feedback).

* as_residual_encode against the oracle over a 5-step trajectory, bit for
  bit: the int8 codes (integers decided in float32 on both sides), the fp32
  scales and the bf16 reconstruction; d = 64 and 128, row counts that are
  not a multiple of the kernel's rows per CTA;
* as_residual_decode reproduces the encoder's reconstruction bit for bit
  (the receiver's copy equals the sender's);
* one rank of a 2-way split attending to residual-reconstructed K/V through
  as_step_cp stays within the bf16 parity bounds of the oracle's exact step."""
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


@pytest.mark.parametrize("d,rows", [(128, 4093), (64, 1021)])
def test_residual_codec_against_oracle(api, d, rows):
    g = torch.Generator(device="cpu").manual_seed(70 + d)
    x = torch.randn((rows, d), generator=g).to(torch.bfloat16)
    base = x.clone().cuda()                # the first send is raw: both sides hold x_0
    recv = base.clone()
    obase = f64(x)
    for t in range(1, 6):
        step = 0.05 * torch.randn((rows, d), generator=g)
        if t == 3:
            step[:7] = 0.0                     # some rows with a zero residual
        x = (x.float() + step).to(torch.bfloat16)
        if t == 3:
            x[:7] = base[:7].cpu()
        codes, scales = api.as_residual_encode(x.cuda(), base)
        api.as_residual_decode(codes, scales, recv)
        torch.cuda.synchronize()
        q, s, nb = O.residual_encode(f64(x), obase)
        assert np.array_equal(codes.cpu().numpy(), q), t
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), s.view(np.uint32)), t
        assert np.array_equal(f64(base), nb), t
        assert torch.equal(recv, base), t
        if t == 3:
            assert not codes[:7].any().item() and not scales[:7].any().item()
        obase = nb


def test_rank_step_on_residual_reconstructions(api):
    from attention_state_reuse_partition_b200 import cp
    s = W.spec("video_long", H=2, rows=8, cols=16, S=16 * 8 * 16)
    n = s.n
    layout = cp.CpLayout(s.P, 2)
    r = 0
    mine = layout.parts(r)
    rows = slice(mine.start * n, mine.stop * n)
    cache = api.AsCache(s.B, s.H, s.S, s.d, s.P, q_first=mine.start, q_count=len(mine))
    ocache = O.StateCache(s.P)
    recon = {}  # remote partition j -> (k, v) reconstruction on the receiving rank
    for t, q, k, v in W.video_trajectory(s):
        plan = W.plan_for_step(s, t).numpy()
        q, k, v = q.cuda(), k.cuda(), v.cuda()
        need = cp.needed_kv(plan, mine)
        k_buf = torch.empty((s.B, s.H, n * len(need), s.d), dtype=k.dtype, device="cuda")
        v_buf = torch.empty_like(k_buf)
        slots = cp.kv_slots(need, s.P)
        for j in need:
            kj, vj = k[:, :, j * n:(j + 1) * n].contiguous(), v[:, :, j * n:(j + 1) * n].contiguous()
            if j not in mine:
                if j not in recon:
                    recon[j] = (kj.clone(), vj.clone())
                else:
                    for x, b in zip((kj, vj), recon[j]):
                        api.as_residual_encode(x, b)     # the sender's tracked copy moves like the receiver's
                kj, vj = recon[j]
            a = int(slots[j]) * n
            k_buf[:, :, a:a + n] = kj
            v_buf[:, :, a:a + n] = vj
        out, lse, _, _ = api.as_step_cp(cache, q[:, :, rows].contiguous(), k_buf, v_buf, slots, plan, t)
        torch.cuda.synchronize()
        ref_o, ref_l, _, _ = O.step(ocache, f64(q), f64(k), f64(v), plan, t, s.scale)
        check_bf16(out, lse, ref_o[:, :, rows], ref_l[:, :, rows], f"step {t} on reconstructed K/V")
