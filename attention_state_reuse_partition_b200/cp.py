"""Context parallelism over ranks for the attention-state step.

DiTango (arXiv 2607.15650; review page, Referee Report "Summary": group-wise
KV transfer and ring-based composition across GPUs; "Core claim": cached
states stand in for far KV partitions) runs the query partitions of one
sequence on several GPUs.  Here each rank owns a contiguous run of query
partitions and the K/V rows of the same partitions.  Before a step a rank
fetches from the other ranks only the KV partitions that its rows of the plan
compute fresh (codes 1 and 2); a reused pair moves nothing, because its
cached state lives on the rank that owns the query partition.  After the
exchange the rank runs ``as_step_cp`` on its own rows, its own cache and the
compact K/V buffer.

Everything here is host logic plus point-to-point sends and receives through
``torch.distributed`` (NCCL on GPUs, gloo on CPU); the arithmetic runs in the
library's kernels.  No TMA multicast is involved anywhere on this path.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Sequence, Tuple

import numpy as np
import torch

PLAN_REUSE = 0


@dataclasses.dataclass(frozen=True)
class CpLayout:
    """P partitions over `world` ranks: rank r owns the contiguous run
    ``parts(r)`` of query partitions (and of K/V partitions); the first
    P % world ranks own one partition more than the others."""
    P: int
    world: int

    def __post_init__(self):
        if self.world < 1 or self.P < self.world:
            raise ValueError(f"need 1 <= world <= P (P={self.P}, world={self.world})")

    def parts(self, rank: int) -> range:
        base, extra = divmod(self.P, self.world)
        lo = rank * base + min(rank, extra)
        return range(lo, lo + base + (1 if rank < extra else 0))

    def owner(self, j: int) -> int:
        for r in range(self.world):
            if j in self.parts(r):
                return r
        raise ValueError(f"partition {j} out of [0, {self.P})")


def needed_kv(plan, parts: Sequence[int]) -> List[int]:
    """KV partitions that the rows ``parts`` of the plan compute fresh, sorted."""
    plan = np.asarray(plan)
    return sorted({j for i in parts for j in range(plan.shape[1]) if int(plan[i, j]) != PLAN_REUSE})


def exchange_plan(plan, layout: CpLayout) -> Dict[Tuple[int, int], List[int]]:
    """{(src, dst): partitions src sends to dst} for src != dst: the
    partitions src owns that dst needs."""
    out = {}
    for dst in range(layout.world):
        need = needed_kv(plan, layout.parts(dst))
        for src in range(layout.world):
            if src != dst:
                js = [j for j in need if j in layout.parts(src)]
                if js:
                    out[(src, dst)] = js
    return out


def kv_slots(needed: Sequence[int], P: int) -> np.ndarray:
    """Slot of every KV partition in a rank's compact K/V buffer (int32 [P],
    -1 = not present): the needed partitions in increasing order."""
    slots = np.full(P, -1, dtype=np.int32)
    for s, j in enumerate(sorted(needed)):
        slots[j] = s
    return slots


def exchange_bytes(plan, layout: CpLayout, B: int, H: int, n: int, d: int, elem_bytes: int) -> Dict[str, int]:
    """Bytes a step's exchange moves between ranks (K and V), and what an
    all-gather of every partition would move."""
    per_part = 2 * B * H * n * d * elem_bytes
    moved = sum(len(js) for js in exchange_plan(plan, layout).values()) * per_part
    all_gather = sum(layout.P - len(layout.parts(r)) for r in range(layout.world)) * per_part
    return {"moved": moved, "all_gather": all_gather}


def _rows(t: torch.Tensor, js: Sequence[int], first: int, n: int) -> torch.Tensor:
    """Rows of partitions js (owned run starting at partition `first`) of a
    [B, H, rows, d] tensor, concatenated in order, contiguous."""
    return torch.cat([t[:, :, (j - first) * n:(j - first + 1) * n] for j in js], dim=2).contiguous()


def exchange_kv(k_local: torch.Tensor, v_local: torch.Tensor, plan, layout: CpLayout, rank: int, n: int,
                group=None) -> Tuple[torch.Tensor, torch.Tensor, np.ndarray]:
    """The exchange of one step on one rank.

    k_local, v_local: [B, H, n * len(parts(rank)), d], the rank's own
    partitions.  Returns (k_buf, v_buf, slots): [B, H, n * #needed, d] with
    KV partition j at rows [slots[j] * n, (slots[j] + 1) * n).  Every rank of
    the group must call this with the same plan (the sends and receives pair
    up); each message carries all the partitions of one (src, dst) pair, K
    and V separately."""
    import torch.distributed as dist
    mine = layout.parts(rank)
    need = needed_kv(plan, mine)
    slots = kv_slots(need, layout.P)
    B, H, _, d = k_local.shape
    k_buf = torch.empty((B, H, n * len(need), d), dtype=k_local.dtype, device=k_local.device)
    v_buf = torch.empty_like(k_buf)
    for j in need:
        if j in mine:
            s = int(slots[j])
            k_buf[:, :, s * n:(s + 1) * n] = k_local[:, :, (j - mine.start) * n:(j - mine.start + 1) * n]
            v_buf[:, :, s * n:(s + 1) * n] = v_local[:, :, (j - mine.start) * n:(j - mine.start + 1) * n]
    pairs = exchange_plan(plan, layout)
    ops, recvs = [], []
    for (src, dst), js in sorted(pairs.items()):
        if src == rank:
            for t in (k_local, v_local):
                ops.append(dist.P2POp(dist.isend, _rows(t, js, mine.start, n), dst, group=group))
        elif dst == rank:
            bufs = [torch.empty((B, H, n * len(js), d), dtype=k_local.dtype, device=k_local.device)
                    for _ in range(2)]
            for b in bufs:
                ops.append(dist.P2POp(dist.irecv, b, src, group=group))
            recvs.append((js, bufs))
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()
    for js, (kb, vb) in recvs:
        for x, j in enumerate(js):
            s = int(slots[j])
            k_buf[:, :, s * n:(s + 1) * n] = kb[:, :, x * n:(x + 1) * n]
            v_buf[:, :, s * n:(s + 1) * n] = vb[:, :, x * n:(x + 1) * n]
    return k_buf, v_buf, slots


def gather_kv_local(k: torch.Tensor, v: torch.Tensor, needed: Sequence[int], n: int):
    """The buffers exchange_kv would produce, built from the full K/V of one
    process (for a single-GPU stand-in of one rank)."""
    js = sorted(needed)
    return _rows(k, js, 0, n), _rows(v, js, 0, n), kv_slots(js, k.shape[2] // n)


class CudaCodec:
    """The library's residual codec (as_residual_encode / as_residual_decode)."""

    def encode(self, x, base):
        from attention_state_reuse_partition_b200 import api
        return api.as_residual_encode(x, base)

    def decode(self, codes, scales, base):
        from attention_state_reuse_partition_b200 import api
        api.as_residual_decode(codes, scales, base)


class ResidualExchange:
    """exchange_kv with CompactFusion's residual compression on the link
    ("Accelerating Parallel Diffusion Model Serving with Residual
    Compression", arXiv 2507.17511, Abstract on its listing page: transmit
    compressed step-wise residuals, with error feedback).

    The first time a rank sends KV partition j to a receiver it sends the
    rows as they are, and both keep them as the receiver's reconstruction.
    Later sends carry the residual against that reconstruction, coded per
    row (d int8 codes and an fp32 scale), and both sides move the
    reconstruction by the same coded residual (as_residual_encode on the
    sender, as_residual_decode on the receiver), so they stay bit-identical
    and a step's coding error is fed into the next residual.  The receiver
    attends to its reconstruction.  State: per (receiver, partition) on the
    sender and per partition on the receiver, [B, H, n, d] for K and for V.

    `codec` provides encode(x, base) -> (codes, scales) (moving base) and
    decode(codes, scales, base); the library's kernels by default."""

    def __init__(self, layout: CpLayout, rank: int, n: int, codec=None):
        self.layout, self.rank, self.n = layout, rank, n
        self.codec = codec if codec is not None else CudaCodec()
        self.send_base = {}   # (dst, j) -> (k, v): the receiver's reconstruction, as this sender tracks it
        self.recv_base = {}   # j -> (k, v): this receiver's reconstruction of a remote partition
        self.sent_bytes = 0   # bytes this rank sent in the last exchange

    def exchange(self, k_local: torch.Tensor, v_local: torch.Tensor, plan, group=None):
        """As exchange_kv; returns (k_buf, v_buf, slots), remote partitions as
        reconstructed."""
        import torch.distributed as dist
        lay, rank, n = self.layout, self.rank, self.n
        mine = lay.parts(rank)
        need = needed_kv(plan, mine)
        slots = kv_slots(need, lay.P)
        B, H, _, d = k_local.shape
        k_buf = torch.empty((B, H, n * len(need), d), dtype=k_local.dtype, device=k_local.device)
        v_buf = torch.empty_like(k_buf)
        for j in need:
            if j in mine:
                s = int(slots[j])
                k_buf[:, :, s * n:(s + 1) * n] = k_local[:, :, (j - mine.start) * n:(j - mine.start + 1) * n]
                v_buf[:, :, s * n:(s + 1) * n] = v_local[:, :, (j - mine.start) * n:(j - mine.start + 1) * n]
        ops, post = [], []
        sent = 0
        for (src, dst), js in sorted(exchange_plan(plan, lay).items()):
            if src == rank:
                for j in js:
                    rows = [_rows(t, [j], mine.start, n) for t in (k_local, v_local)]
                    key = (dst, j)
                    if key not in self.send_base:
                        self.send_base[key] = tuple(x.clone() for x in rows)
                        payload = rows
                    else:
                        payload = []
                        for x, base in zip(rows, self.send_base[key]):
                            payload.extend(self.codec.encode(x, base))
                    for p in payload:
                        ops.append(dist.P2POp(dist.isend, p, dst, group=group))
                        sent += p.numel() * p.element_size()
            elif dst == rank:
                for j in js:
                    shape = (B, H, n, d)
                    if j not in self.recv_base:
                        bufs = [torch.empty(shape, dtype=k_local.dtype, device=k_local.device) for _ in range(2)]
                        post.append((j, "raw", bufs))
                    else:
                        bufs = []
                        for _ in range(2):
                            bufs.append(torch.empty(shape, dtype=torch.int8, device=k_local.device))
                            bufs.append(torch.empty(shape[:-1], dtype=torch.float32, device=k_local.device))
                        post.append((j, "coded", bufs))
                    for b in bufs:
                        ops.append(dist.P2POp(dist.irecv, b, src, group=group))
        if ops:
            for req in dist.batch_isend_irecv(ops):
                req.wait()
        for j, kind, bufs in post:
            if kind == "raw":
                self.recv_base[j] = (bufs[0], bufs[1])
            else:
                kb, vb = self.recv_base[j]
                self.codec.decode(bufs[0], bufs[1], kb)
                self.codec.decode(bufs[2], bufs[3], vb)
            kb, vb = self.recv_base[j]
            s = int(slots[j])
            k_buf[:, :, s * n:(s + 1) * n] = kb
            v_buf[:, :, s * n:(s + 1) * n] = vb
        self.sent_bytes = sent
        return k_buf, v_buf, slots
