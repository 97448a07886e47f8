"""Python binding of the C ABI (include/as_partition.h), same names as the C
entry points.  Argument marshalling only: tensors are passed by device
pointer, outputs are allocated with torch when not given, streams are torch
streams.  Every computation runs in the library's CUDA kernels."""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np
import torch

from . import _lib
from ._lib import (AS_BF16, AS_F32, AS_PLAN_FRESH, AS_PLAN_FRESH_STORE, AS_PLAN_REUSE, AsCacheStruct,
                   AsError, AsPlannerStruct, LIB, check)

__all__ = ["as_partition_attn", "as_compose", "as_cache_bytes", "as_cache_init", "as_plan_resolve", "as_step",
           "as_device_status", "as_debug_timeout_probe", "as_version", "AsCache", "AsError",
           "AS_PLAN_REUSE", "AS_PLAN_FRESH", "AS_PLAN_FRESH_STORE", "AsPlanner", "as_planner_init",
           "as_planner_scratch_bytes", "as_local_states", "as_plan_drift", "as_plan_select", "as_planner_next", "as_residual_encode",
           "as_residual_decode",
           "as_planner_commit_anchor", "as_plan_drift_static", "as_step_local", "as_cache_cp_bytes", "as_step_cp"]


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return AS_BF16
    if t.dtype == torch.float32:
        return AS_F32
    raise AsError(_lib.AS_ERR_INVALID_ARG, f"unsupported input dtype {t.dtype}")


def _check_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> None:
    """Q, K and V must agree in shape [B, H, S, d], dtype and device: the
    library reads all three with Q's element type."""
    if q.dim() != 4:
        raise AsError(_lib.AS_ERR_INVALID_ARG, f"q must be [B, H, S, d], got shape {tuple(q.shape)}")
    for name, t in (("k", k), ("v", v)):
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device:
            raise AsError(_lib.AS_ERR_INVALID_ARG,
                          f"{name} ({tuple(t.shape)}, {t.dtype}, {t.device}) does not match q "
                          f"({tuple(q.shape)}, {q.dtype}, {q.device})")


def _buf(t: Optional[torch.Tensor], shape, device, name: str) -> torch.Tensor:
    """An fp32 buffer of exactly `shape`: allocated when not given, checked
    when given (the library writes all of it)."""
    shape = tuple(int(x) for x in shape)
    if t is None:
        return torch.empty(shape, device=device, dtype=torch.float32)
    if t.dtype != torch.float32 or tuple(t.shape) != shape:
        raise AsError(_lib.AS_ERR_INVALID_ARG,
                      f"{name} must be float32 of shape {shape}, got {t.dtype} of shape {tuple(t.shape)}")
    return t


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> Optional[int]:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream or None


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda or not t.is_contiguous():
        raise AsError(_lib.AS_ERR_INVALID_ARG, f"{name} must be a contiguous CUDA tensor")
    return t.data_ptr()


def as_version() -> str:
    return LIB.as_version().decode()


def as_partition_attn(q, k, v, P: int, q_part: int, kv_parts: Sequence[int], compose: bool = True,
                      scale: Optional[float] = None, out=None, lse=None, stream=None):
    """States of query partition ``q_part`` (or all rows, q_part=-1) against
    the listed KV partitions; composed (compose=True) or one per partition."""
    _check_qkv(q, k, v)
    B, H, S, d = q.shape
    R = S if q_part < 0 else S // P
    scale = 1.0 / d ** 0.5 if scale is None else scale
    planes = () if compose else (len(kv_parts),)
    out = _buf(out, planes + (B, H, R, d), q.device, "out")
    lse = _buf(lse, planes + (B, H, R), q.device, "lse")
    parts = (ctypes.c_int32 * len(kv_parts))(*[int(x) for x in kv_parts])
    check(LIB.as_partition_attn(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dtype_code(q), B, H, S, d, P,
                                float(scale), int(q_part), parts, len(kv_parts), 1 if compose else 0,
                                _dev(out, "out"), _dev(lse, "lse"), _stream_ptr(stream)))
    return out, lse


def as_compose(outs, lses, out=None, lse=None, stream=None):
    """Compose N states per row: outs [N, ..., d], lses [N, ...] (fp32)."""
    N = outs.shape[0]
    d = outs.shape[-1]
    if outs.dtype != torch.float32 or lses.dtype != torch.float32 or tuple(lses.shape) != tuple(outs.shape[:-1]):
        raise AsError(_lib.AS_ERR_INVALID_ARG,
                      f"outs [N, ..., d] and lses [N, ...] must be float32 with matching shapes, got "
                      f"{outs.dtype} {tuple(outs.shape)} and {lses.dtype} {tuple(lses.shape)}")
    rows = lses[0].numel()
    out = _buf(out, outs.shape[1:], outs.device, "out")
    lse = _buf(lse, lses.shape[1:], lses.device, "lse")
    check(LIB.as_compose(_dev(outs, "outs"), _dev(lses, "lses"), N, rows, d, rows * d, rows,
                         _dev(out, "out"), _dev(lse, "lse"), _stream_ptr(stream)))
    return out, lse


def _cache_dt(cache_dtype) -> int:
    if cache_dtype in (torch.float32, "f32", AS_F32):
        return AS_F32
    if cache_dtype in (torch.bfloat16, "bf16", AS_BF16):
        return AS_BF16
    raise AsError(_lib.AS_ERR_INVALID_ARG, f"unsupported cache dtype {cache_dtype}")


def as_cache_bytes(B: int, H: int, S: int, d: int, P: int, g: int = 1, cache_dtype=torch.float32) -> int:
    return int(LIB.as_cache_group_bytes(B, H, S, d, P, g, _cache_dt(cache_dtype)))


def as_cache_cp_bytes(B: int, H: int, S: int, d: int, P: int, q_count: int, g: int = 1,
                      cache_dtype=torch.float32) -> int:
    return int(LIB.as_cache_cp_bytes(B, H, S, d, P, g, _cache_dt(cache_dtype), q_count))


class AsCache:
    """A state cache: the C struct plus its device buffer (allocated with
    torch).  ``g``: KV partitions per cache group (one composed entry per
    (query partition, group)); ``cache_dtype``: torch.float32 or
    torch.bfloat16 for the OUT entries (LSE entries are fp32).  ``q_first``,
    ``q_count``: the query partitions the cache holds entries for (all of
    them by default; one rank's run for context parallelism, as_step_cp)."""

    def __init__(self, B: int, H: int, S: int, d: int, P: int, device="cuda", buffer: Optional[torch.Tensor] = None,
                 g: int = 1, cache_dtype=torch.float32, q_first: int = 0, q_count: Optional[int] = None):
        dt = _cache_dt(cache_dtype)
        q_count = P if q_count is None else q_count
        nbytes = as_cache_cp_bytes(B, H, S, d, P, q_count, g, dt)
        if nbytes == 0:
            raise AsError(_lib.AS_ERR_INVALID_ARG, "invalid cache sizes")
        if buffer is None:
            buffer = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.buffer = buffer
        self.struct = AsCacheStruct()
        check(LIB.as_cache_cp_init(ctypes.byref(self.struct), buffer.data_ptr(), buffer.numel(), B, H, S, d, P, g,
                                   dt, q_first, q_count))
        self._set_sizes(B, H, S, d, P, g, dt, q_first, q_count)

    def _set_sizes(self, B, H, S, d, P, g, dt, q_first=0, q_count=None):
        self.B, self.H, self.S, self.d, self.P, self.g = B, H, S, d, P, g
        self.q_first, self.q_count = q_first, (P if q_count is None else q_count)
        self.rows = self.q_count * (S // P)  # query rows per head of the cache's planes
        self.NG = (P + g - 1) // g
        self.cache_dtype = torch.bfloat16 if dt == AS_BF16 else torch.float32

    @classmethod
    def host_only(cls, B: int, H: int, S: int, d: int, P: int, g: int = 1, cache_dtype=torch.float32,
                  q_first: int = 0, q_count: Optional[int] = None) -> "AsCache":
        """A cache struct for host-side plan bookkeeping (as_plan_resolve) on a
        machine without a GPU.  Its planes point at a placeholder address that
        is never dereferenced; it must not be passed to as_step."""
        self = cls.__new__(cls)
        self.buffer = None
        self.struct = AsCacheStruct()
        dt = _cache_dt(cache_dtype)
        q_count = P if q_count is None else q_count
        check(LIB.as_cache_cp_init(ctypes.byref(self.struct), 1 << 30, as_cache_cp_bytes(B, H, S, d, P, q_count, g, dt),
                                   B, H, S, d, P, g, dt, q_first, q_count))
        self._set_sizes(B, H, S, d, P, g, dt, q_first, q_count)
        return self

    def set_t_c(self, t_c) -> None:
        """Overwrite the host-side store timestamps [P, n_groups] (for
        replaying bookkeeping)."""
        flat = np.asarray(t_c, dtype=np.int32).reshape(-1)
        for x in range(self.P * self.NG):
            self.struct.t_c[x] = int(flat[x])

    def set_member(self, member) -> None:
        """Overwrite the stored member masks [P, n_groups] (bit j = KV
        partition j), for replaying bookkeeping."""
        flat = np.asarray(member, dtype=np.uint64).reshape(-1)
        for x in range(self.P * self.NG):
            self.struct.member[x] = int(flat[x])

    @property
    def t_c(self) -> np.ndarray:
        return np.ctypeslib.as_array(self.struct.t_c)[: self.P * self.NG].reshape(self.P, self.NG).copy()

    @property
    def member(self) -> np.ndarray:
        return np.ctypeslib.as_array(self.struct.member)[: self.P * self.NG].reshape(self.P, self.NG).copy()

    def state_dict(self) -> dict:
        """Everything needed to resume: sizes, group size, entry dtype, the
        host bookkeeping (t_c, member masks) and a host copy of the device
        buffer (synchronises the current stream)."""
        return {"sizes": (self.B, self.H, self.S, self.d, self.P), "g": self.g,
                "q_first": self.q_first, "q_count": self.q_count,
                "cache_dtype": "bf16" if self.cache_dtype == torch.bfloat16 else "f32",
                "t_c": self.t_c, "member": self.member,
                "buffer": None if self.buffer is None else self.buffer.cpu()}

    @classmethod
    def from_state_dict(cls, sd: dict, device="cuda") -> "AsCache":
        """A cache restored from state_dict(): same entries and bookkeeping."""
        B, H, S, d, P = sd["sizes"]
        self = cls(B, H, S, d, P, device=device, g=sd["g"], cache_dtype=sd["cache_dtype"],
                   q_first=sd.get("q_first", 0), q_count=sd.get("q_count"))
        if sd["buffer"] is None or sd["buffer"].numel() != self.buffer.numel():
            raise AsError(_lib.AS_ERR_INVALID_ARG, "state dict buffer does not match the cache sizes")
        self.buffer.copy_(sd["buffer"])
        self.set_t_c(sd["t_c"])
        self.set_member(sd["member"])
        return self

    def planes(self):
        """Views of the cache planes: OUT [NG,B,H,rows,d] (the cache dtype),
        LSE [NG,B,H,rows] (fp32); rows = S unless the cache is one rank's."""
        n_out = self.NG * self.B * self.H * self.rows * self.d
        n_lse = self.NG * self.B * self.H * self.rows
        esz = 2 if self.cache_dtype == torch.bfloat16 else 4
        out = self.buffer[: n_out * esz].view(self.cache_dtype).view(self.NG, self.B, self.H, self.rows, self.d)
        lse = self.buffer[n_out * esz: n_out * esz + n_lse * 4].view(torch.float32).view(
            self.NG, self.B, self.H, self.rows)
        return out, lse


def as_cache_init(B, H, S, d, P, device="cuda", buffer=None, g: int = 1, cache_dtype=torch.float32) -> AsCache:
    return AsCache(B, H, S, d, P, device=device, buffer=buffer, g=g, cache_dtype=cache_dtype)


def _plan_bytes(plan, P):
    arr = np.ascontiguousarray(np.asarray(plan, dtype=np.uint8).reshape(P * P))
    return arr


def as_plan_resolve(cache: AsCache, plan, step: int):
    """Host-only plan check: returns (hit, age) as [P,P] numpy arrays."""
    P = cache.P
    arr = _plan_bytes(plan, P)
    hit = np.zeros(P * P, dtype=np.uint8)
    age = np.zeros(P * P, dtype=np.int32)
    check(LIB.as_plan_resolve(ctypes.byref(cache.struct), arr.ctypes.data, int(step), hit.ctypes.data,
                              age.ctypes.data))
    return hit.reshape(P, P), age.reshape(P, P)


def as_step(cache: AsCache, q, k, v, plan, step: int, scale: Optional[float] = None, out=None, lse=None,
            stream=None):
    """One step under a compute/reuse plan; returns (out, lse, hit, age)."""
    _check_qkv(q, k, v)
    _check_cache_shape(cache, q)
    B, H, S, d = q.shape
    P = cache.P
    scale = 1.0 / d ** 0.5 if scale is None else scale
    out = _buf(out, (B, H, S, d), q.device, "out")
    lse = _buf(lse, (B, H, S), q.device, "lse")
    arr = _plan_bytes(plan, P)
    hit = np.zeros(P * P, dtype=np.uint8)
    age = np.zeros(P * P, dtype=np.int32)
    check(LIB.as_step(ctypes.byref(cache.struct), _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dtype_code(q),
                      float(scale), arr.ctypes.data, int(step), _dev(out, "out"), _dev(lse, "lse"),
                      hit.ctypes.data, age.ctypes.data, _stream_ptr(stream)))
    return out, lse, hit.reshape(P, P), age.reshape(P, P)


def as_step_local(cache: AsCache, q, k, v, plan, step: int, local_out, local_lse, scale: Optional[float] = None,
                  out=None, lse=None, stream=None):
    """as_step with the step's local states AS(i, i) given (from
    as_local_states on the same inputs): plain-fresh diagonal pairs are
    composed from them instead of recomputed.  Returns (out, lse, hit, age)."""
    _check_qkv(q, k, v)
    _check_cache_shape(cache, q)
    B, H, S, d = q.shape
    P = cache.P
    scale = 1.0 / d ** 0.5 if scale is None else scale
    out = _buf(out, (B, H, S, d), q.device, "out")
    lse = _buf(lse, (B, H, S), q.device, "lse")
    _buf(local_out, (B, H, S, d), q.device, "local_out")
    _buf(local_lse, (B, H, S), q.device, "local_lse")
    arr = _plan_bytes(plan, P)
    hit = np.zeros(P * P, dtype=np.uint8)
    age = np.zeros(P * P, dtype=np.int32)
    check(LIB.as_step_local(ctypes.byref(cache.struct), _dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dtype_code(q),
                            float(scale), arr.ctypes.data, int(step), _dev(local_out, "local_out"),
                            _dev(local_lse, "local_lse"), _dev(out, "out"), _dev(lse, "lse"), hit.ctypes.data,
                            age.ctypes.data, _stream_ptr(stream)))
    return out, lse, hit.reshape(P, P), age.reshape(P, P)


# ---------------------------------------------------------------------------
# the anchor-guided planner
# ---------------------------------------------------------------------------

def as_step_cp(cache: AsCache, q, k_buf, v_buf, kv_slots, plan, step: int, scale: Optional[float] = None,
               out=None, lse=None, stream=None):
    """One step on the rank that owns the cache's query partitions: q [B, H,
    cache.rows, d] holds its query rows, k_buf / v_buf [B, H, kv_rows, d] the
    KV partitions its plan rows compute (partition j at rows kv_slots[j] * n,
    -1 = absent; see cp.exchange_kv).  Returns (out, lse, hit, age) for the
    rank's rows; hit and age are [P, P] with zeros outside them."""
    want = (cache.B, cache.H, cache.rows, cache.d)
    if q.dim() != 4 or tuple(q.shape) != want:
        raise AsError(_lib.AS_ERR_INVALID_ARG, f"q must have shape {want}, got {tuple(q.shape)}")
    for name, t in (("k_buf", k_buf), ("v_buf", v_buf)):
        if t.dim() != 4 or t.shape[:2] != q.shape[:2] or t.shape[3] != q.shape[3] or t.dtype != q.dtype \
                or t.device != q.device or t.shape != k_buf.shape:
            raise AsError(_lib.AS_ERR_INVALID_ARG,
                          f"{name} ({tuple(t.shape)}, {t.dtype}) must be [B, H, kv_rows, d] like k_buf, with q's "
                          f"B, H, d, dtype and device")
    P = cache.P
    slots = np.ascontiguousarray(np.asarray(kv_slots, dtype=np.int32).reshape(P))
    B, H, R, d = q.shape
    scale = 1.0 / d ** 0.5 if scale is None else scale
    out = _buf(out, (B, H, R, d), q.device, "out")
    lse = _buf(lse, (B, H, R), q.device, "lse")
    arr = _plan_bytes(plan, P)
    hit = np.zeros(P * P, dtype=np.uint8)
    age = np.zeros(P * P, dtype=np.int32)
    check(LIB.as_step_cp(ctypes.byref(cache.struct), _dev(q, "q"), _dev(k_buf, "k_buf"), _dev(v_buf, "v_buf"),
                         int(k_buf.shape[2]), slots.ctypes.data, _dtype_code(q), float(scale), arr.ctypes.data,
                         int(step), _dev(out, "out"), _dev(lse, "lse"), hit.ctypes.data, age.ctypes.data,
                         _stream_ptr(stream)))
    return out, lse, hit.reshape(P, P), age.reshape(P, P)


def _rows_d(t: torch.Tensor, name: str):
    if t.dtype != torch.bfloat16 or t.dim() < 2:
        raise AsError(_lib.AS_ERR_INVALID_ARG, f"{name} must be bfloat16 [..., d], got {t.dtype} {tuple(t.shape)}")
    return t.numel() // t.shape[-1], t.shape[-1]


def as_residual_encode(x, base, codes=None, scales=None, stream=None):
    """Residual-code the rows of x [..., d] (bf16) against the reconstruction
    `base` (same shape, bf16), which moves to the new reconstruction in
    place.  Returns (codes int8 [..., d], scales fp32 [...])."""
    rows, d = _rows_d(x, "x")
    if base.shape != x.shape or base.dtype != x.dtype:
        raise AsError(_lib.AS_ERR_INVALID_ARG, "base must match x in shape and dtype")
    if codes is None:
        codes = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    if codes.shape != x.shape or codes.dtype != torch.int8 or scales.shape != x.shape[:-1] \
            or scales.dtype != torch.float32:
        raise AsError(_lib.AS_ERR_INVALID_ARG, "codes must be int8 like x, scales float32 [...]")
    check(LIB.as_residual_encode(_dev(x, "x"), _dev(base, "base"), _dev(codes, "codes"), _dev(scales, "scales"),
                                 rows, d, _stream_ptr(stream)))
    return codes, scales


def as_residual_decode(codes, scales, base, stream=None):
    """The receiver's half: base <- bf16(base + codes * scales), in place."""
    rows, d = _rows_d(base, "base")
    if codes.shape != base.shape or codes.dtype != torch.int8 or scales.shape != base.shape[:-1] \
            or scales.dtype != torch.float32:
        raise AsError(_lib.AS_ERR_INVALID_ARG, "codes must be int8 like base, scales float32 [...]")
    check(LIB.as_residual_decode(_dev(codes, "codes"), _dev(scales, "scales"), _dev(base, "base"), rows, d,
                                 _stream_ptr(stream)))
    return base


def as_planner_scratch_bytes(B: int, H: int, P: int) -> int:
    return int(LIB.as_planner_scratch_bytes(B, H, P))


class AsPlanner:
    """The planner's C struct plus its device buffers (scratch and the anchor's
    local states), allocated with torch."""

    def __init__(self, P: int, window: int, reuse_ratio: float, eps_local: float, B: int = 0, H: int = 0,
                 S: int = 0, d: int = 0, device="cuda", g: int = 1):
        self.struct = AsPlannerStruct()
        check(LIB.as_planner_group_init(ctypes.byref(self.struct), P, g, window, float(reuse_ratio),
                                        float(eps_local)))
        self.P, self.g = P, g
        self.NG = (P + g - 1) // g
        self.scratch = None
        self.local_anchor = None
        if B:
            nbytes = as_planner_scratch_bytes(B, H, P)
            self.scratch = torch.empty(nbytes // 8 + 1, dtype=torch.float64, device=device)
            self.local_anchor = torch.zeros((B, H, S, d), dtype=torch.float32, device=device)

    def _arr(self, name, n):
        return np.ctypeslib.as_array(getattr(self.struct, name))[:n].copy()

    @property
    def has_anchor(self) -> bool:
        return bool(self.struct.has_anchor)

    @property
    def w(self):
        """w(i, G) of the last anchor, [P, n_groups]."""
        return self._arr("w", self.P * self.NG).reshape(self.P, self.NG)

    @property
    def alpha(self):
        """alpha(i, G) of the last anchor, [P, n_groups]."""
        return self._arr("alpha", self.P * self.NG).reshape(self.P, self.NG)

    @property
    def drift(self):
        return self._arr("drift", self.P)

    @property
    def rel_drift(self):
        return self._arr("rel_drift", self.P)


def as_planner_init(P, window, reuse_ratio, eps_local, B=0, H=0, S=0, d=0, device="cuda", g=1) -> AsPlanner:
    return AsPlanner(P, window, reuse_ratio, eps_local, B, H, S, d, device, g)


def as_local_states(q, k, v, P: int, scale: Optional[float] = None, out=None, lse=None, stream=None):
    """Local states AS(i, i) of every query partition: out [B,H,S,d], lse [B,H,S]."""
    _check_qkv(q, k, v)
    B, H, S, d = q.shape
    scale = 1.0 / d ** 0.5 if scale is None else scale
    out = _buf(out, (B, H, S, d), q.device, "out")
    lse = _buf(lse, (B, H, S), q.device, "lse")
    check(LIB.as_local_states(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dtype_code(q), B, H, S, d, P,
                              float(scale), _dev(out, "out"), _dev(lse, "lse"), _stream_ptr(stream)))
    return out, lse


def _check_cache_shape(cache: "AsCache", q: torch.Tensor) -> None:
    """The step reads Q, K, V and writes OUT with the cache's B, H, S, d."""
    want = (cache.B, cache.H, cache.S, cache.d)
    if tuple(q.shape) != want:
        raise AsError(_lib.AS_ERR_INVALID_ARG,
                      f"q, k, v must have the cache's shape {want} (B, H, S, d), got {tuple(q.shape)}")


def _check_drift_inputs(now, anchor):
    if now.dim() != 4 or now.dtype != torch.float32 or anchor.dtype != torch.float32 or anchor.shape != now.shape:
        raise AsError(_lib.AS_ERR_INVALID_ARG,
                      f"now and anchor must be float32 [B, H, S, d] of one shape, got {now.dtype} "
                      f"{tuple(now.shape)} and {anchor.dtype} {tuple(anchor.shape)}")


def as_plan_drift(now, anchor, P: int, scratch, stream=None):
    """(drift [P], norm [P]) of every partition's local state against the anchor's."""
    _check_drift_inputs(now, anchor)
    B, H, S, d = now.shape
    drift = np.zeros(P, dtype=np.float64)
    norm = np.zeros(P, dtype=np.float64)
    check(LIB.as_plan_drift(_dev(now, "now"), _dev(anchor, "anchor"), B, H, S, d, P, _dev(scratch, "scratch"),
                            scratch.numel() * scratch.element_size(), drift.ctypes.data, norm.ctypes.data,
                            _stream_ptr(stream)))
    return drift, norm


def as_plan_drift_static(now, anchor, P: int, stream=None):
    """as_plan_drift with the library's fixed scratch: for callers that cannot
    allocate device memory (see include/as_partition.h).  The library
    allocates nothing; the limit is P * (B*H*2 + 2) <= 131072."""
    _check_drift_inputs(now, anchor)
    B, H, S, d = now.shape
    drift = np.zeros(P, dtype=np.float64)
    norm = np.zeros(P, dtype=np.float64)
    check(LIB.as_plan_drift_static(_dev(now, "now"), _dev(anchor, "anchor"), B, H, S, d, P, drift.ctypes.data,
                                   norm.ctypes.data, _stream_ptr(stream)))
    return drift, norm


def as_plan_select(ase, window: int, reuse_ratio: float, g: int = 1):
    """Host-only plan selection from ASE values [P, n_groups] (groups of g
    KV partitions; [P, P] for g = 1); returns the plan [P, P]."""
    a = np.ascontiguousarray(np.asarray(ase, dtype=np.float64))
    P = a.shape[0]
    if a.shape != (P, (P + g - 1) // g):
        raise AsError(_lib.AS_ERR_INVALID_ARG, f"ASE must be [P, ceil(P/g)], got {a.shape}")
    plan = np.zeros(P * P, dtype=np.uint8)
    check(LIB.as_plan_select_grouped(a.ctypes.data, P, int(g), int(window), float(reuse_ratio), plan.ctypes.data))
    return plan.reshape(P, P)


def _check_planner_state(pl: AsPlanner) -> None:
    if pl.local_anchor is None:
        raise AsError(_lib.AS_ERR_INVALID_ARG, "the planner holds no device state: create it with B, H, S, d")


def as_planner_next(pl: AsPlanner, local_now, stream=None):
    """(plan [P,P], is_anchor, ase [P, n_groups]) of the next step."""
    _check_planner_state(pl)
    if local_now.dtype != torch.float32 or local_now.shape != pl.local_anchor.shape:
        raise AsError(_lib.AS_ERR_INVALID_ARG,
                      f"local_now must be float32 of the planner's shape {tuple(pl.local_anchor.shape)}, got "
                      f"{local_now.dtype} {tuple(local_now.shape)}")
    B, H, S, d = local_now.shape
    P = pl.P
    plan = np.zeros(P * P, dtype=np.uint8)
    ase = np.zeros(P * pl.NG, dtype=np.float64)
    is_anchor = ctypes.c_int(0)
    check(LIB.as_planner_next(ctypes.byref(pl.struct), _dev(local_now, "local_now"), _dev(pl.local_anchor, "anchor"),
                              B, H, S, d, _dev(pl.scratch, "scratch"), pl.scratch.numel() * 8, plan.ctypes.data,
                              ctypes.byref(is_anchor), ase.ctypes.data, _stream_ptr(stream)))
    return plan.reshape(P, P), bool(is_anchor.value), ase.reshape(P, pl.NG)


def as_planner_commit_anchor(pl: AsPlanner, cache: AsCache, lse_full, plan, stream=None):
    _check_planner_state(pl)
    want = (cache.B, cache.H, cache.S)
    if lse_full.dtype != torch.float32 or tuple(lse_full.shape) != want:
        raise AsError(_lib.AS_ERR_INVALID_ARG,
                      f"lse_full must be float32 of the cache's shape {want}, got {lse_full.dtype} "
                      f"{tuple(lse_full.shape)}")
    if tuple(pl.local_anchor.shape) != want + (cache.d,):
        raise AsError(_lib.AS_ERR_INVALID_ARG,
                      f"the planner's states {tuple(pl.local_anchor.shape)} do not match the cache {want + (cache.d,)}")
    arr = _plan_bytes(plan, pl.P)
    check(LIB.as_planner_commit_anchor(ctypes.byref(pl.struct), ctypes.byref(cache.struct), _dev(lse_full, "lse"),
                                       _dev(pl.local_anchor, "anchor"), arr.ctypes.data, _dev(pl.scratch, "scratch"),
                                       pl.scratch.numel() * 8, _stream_ptr(stream)))


def as_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device error bits;
    raises AsError(AS_ERR_TIMEOUT) when a bounded wait ran out."""
    bits = ctypes.c_uint32(0)
    status = LIB.as_device_status(_stream_ptr(stream), ctypes.byref(bits))
    if status not in (_lib.AS_OK, _lib.AS_ERR_TIMEOUT):
        check(status)
    if status == _lib.AS_ERR_TIMEOUT:
        raise AsError(status, LIB.as_last_error().decode())
    return bits.value


def as_debug_exp2(x, mode: int = 0, stream=None):
    """2^x on the device: mode 0 = FMA-pipe polynomial, 1 = MUFU ex2.approx."""
    y = torch.empty_like(x)
    check(LIB.as_debug_exp2(_dev(x, "x"), _dev(y, "y"), x.numel(), int(mode), _stream_ptr(stream)))
    return y


def as_debug_timeout_probe(poll_budget: int = 64, limit_ns: int = 4_000_000_000, stream=None) -> None:
    """One wait on a barrier that nothing completes, bounded by `poll_budget`
    try_wait rounds or `limit_ns` nanoseconds of GPU time."""
    check(LIB.as_debug_timeout_probe(int(poll_budget), int(limit_ns), _stream_ptr(stream)))
