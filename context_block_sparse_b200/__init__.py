"""Split-KV block-sparse anchor attention on NVIDIA B200 (sm_100a).

Thin Python binding of libsplitkv.so.  The functions carry the C entry points'
names and only marshal arguments (torch tensors -> device pointers, the
current CUDA stream -> cudaStream_t); every step of the computation runs in the
library's CUDA kernels.  Importing this package loads the shared library and
raises ImportError if it has not been built.

Method: "Split-KV: Efficient Context Parallelism for Training Diffusion
Drafters" (digest page, Abstract) and the news page "Split-KV speeds
diffusion drafter training by keeping long-context data local" (sections "Why
short queries change the problem", "Exchange the smaller side", "Balance actual
attention work").
"""

from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np

from . import _abi
from ._abi import (  # noqa: F401
    DTYPE_BF16, DTYPE_F32, EXPORT_BWD_LOADS, EXPORT_BWD_SCHEDULE, EXPORT_CHUNK_PAIRS,
    EXPORT_BWD_LPT_ORDER, EXPORT_CHUNK_OWNER, EXPORT_CONTIG_LOADS, EXPORT_ENTRIES, EXPORT_FWD_LOADS,
    EXPORT_FWD_LPT_ORDER, EXPORT_QUERY_SHARD, MAX_RANKS,
    EXPORT_FWD_SCHEDULE, FLAG_BLOCK_KEYS_IN_CONTEXT, FLAG_CONTIGUOUS_RANKS, FLAG_CONTIGUOUS_SCHEDULE,
    FLAG_DYNAMIC_CLAIM, FLAG_EQUAL_COUNT,
    FLAG_FWD_TILE_COST,
    FLAG_PARTIAL_BF16, FLAG_TILE_COST,
    STATIC_SCRATCH_BYTES, TIMES_DQ, WS_BWD, WS_FWD,
)

_lib = _abi.load()


class SplitKVError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        msg = _lib.splitkv_error_string(status).decode()
        super().__init__(f"{fn}: {msg} ({status})")


def _with_site(err: "SplitKVError", site: int) -> "SplitKVError":
    if site:
        err.args = (f"{err.args[0]} [first timed-out wait: file {site // 10000}, line {site % 10000}]",)
    return err


def _check(fn: str, status: int) -> None:
    if status != _abi.OK:
        raise SplitKVError(fn, status)


def _stream_ptr(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if hasattr(stream, "cuda_stream"):
        return stream.cuda_stream
    return int(stream)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return t.data_ptr()


def _bf16_ptr(t) -> int:
    import torch
    if t is None:
        return None
    if t.dtype != torch.bfloat16:
        raise ValueError("q, k, v, kb, vb and dout must be bfloat16")
    return _ptr(t)


def _f32_ptr(t) -> int:
    import torch
    if t is None:
        return None
    if t.dtype != torch.float32:
        raise ValueError("lse, dq, dk, dv, dkb and dvb must be float32")
    return _ptr(t)


def _dims(plan: "Plan") -> dict:
    """Element counts of every tensor of an attention call, from the plan's problem (cached on
    the plan until splitkv_plan_update)."""
    if plan._dims is not None:
        return plan._dims
    st = splitkv_plan_stats(plan)
    p = plan.problem
    N, Nq, Hq, Hkv, d = st["context_len"], st["num_queries"], p.num_q_heads, p.num_kv_heads, p.head_dim
    qs, ks, bs_ = Nq * Hq * d, N * Hkv * d, Nq * Hkv * d
    plan._dims = {"q": qs, "dout": qs, "o": qs, "dq": qs, "lse": Nq * Hq, "k": ks, "v": ks, "dk": ks, "dv": ks,
            "kb": bs_, "vb": bs_, "dkb": bs_, "dvb": bs_}
    return plan._dims


def _sizes(plan: "Plan", **tensors) -> None:
    """Every given tensor must hold exactly the elements the plan's layout gives it (the C
    entry points take bare pointers; a short tensor would be read or written past its end)."""
    want = _dims(plan)
    for name, t in tensors.items():
        if t is not None and t.numel() != want[name]:
            raise ValueError(f"{name} has {t.numel()} elements; the plan's layout needs {want[name]}")


def _o_dtype(o) -> int:
    import torch
    if o.dtype == torch.float32:
        return DTYPE_F32
    if o.dtype == torch.bfloat16:
        return DTYPE_BF16
    raise ValueError("o must be float32 or bfloat16")


class Plan:
    """Owner of a splitkv_plan_t handle (see splitkv_plan)."""

    def __init__(self, handle: ctypes.c_void_p, problem: _abi.Problem, keep):
        self._h = handle
        self.problem = problem
        self._keep = keep
        self._dims = None

    @property
    def handle(self) -> ctypes.c_void_p:
        if not self._h:
            raise ValueError("plan has been destroyed")
        return self._h

    def stats(self) -> dict:
        return splitkv_plan_stats(self)

    def export(self, what: int) -> np.ndarray:
        return splitkv_plan_export(self, what)

    def dump(self, path: str) -> None:
        """Write the plan to `path` (.npz): the problem, the stats and every exported table."""
        splitkv_plan_dump(self, path)

    def upload(self, stream=None) -> "Plan":
        splitkv_plan_upload(self, stream)
        return self

    def destroy(self) -> None:
        splitkv_plan_destroy(self)

    def __del__(self):
        try:
            if self._h:
                _lib.splitkv_plan_destroy(self._h)
                self._h = None
        except Exception:
            pass


def _problem(sample_lens, anchors, block_size, num_q_heads, num_kv_heads, head_dim, kv_chunk,
             num_workers, num_bwd_workers, q_slice, equal_count, block_keys_in_context=False,
             partial_bf16=False, tile_cost=False, fwd_tile_cost=False, dynamic_claim=False,
             contiguous_schedule=False, contiguous_ranks=False):
    lens = np.ascontiguousarray(sample_lens, dtype=np.int32)
    anc = np.ascontiguousarray(anchors, dtype=np.int32)
    p = _abi.Problem()
    p.num_samples = lens.size
    p.sample_lens = lens.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    p.num_anchors = anc.size
    p.anchors = anc.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    p.block_size = int(block_size)
    p.num_q_heads = int(num_q_heads)
    p.num_kv_heads = int(num_kv_heads)
    p.head_dim = int(head_dim)
    p.kv_chunk = int(kv_chunk)
    p.num_workers = int(num_workers)
    p.num_bwd_workers = int(num_bwd_workers)
    p.q_slice = int(q_slice)
    p.flags = ((FLAG_EQUAL_COUNT if equal_count else 0) | (FLAG_BLOCK_KEYS_IN_CONTEXT if block_keys_in_context else 0)
               | (FLAG_PARTIAL_BF16 if partial_bf16 else 0) | (FLAG_TILE_COST if tile_cost else 0)
               | (FLAG_FWD_TILE_COST if fwd_tile_cost else 0) | (FLAG_DYNAMIC_CLAIM if dynamic_claim else 0)
               | (FLAG_CONTIGUOUS_SCHEDULE if contiguous_schedule else 0)
               | (FLAG_CONTIGUOUS_RANKS if contiguous_ranks else 0))
    return p, (lens, anc)


def splitkv_plan(sample_lens: Sequence[int], anchors: Sequence[int], block_size: int, num_q_heads: int,
                 num_kv_heads: int, head_dim: int, kv_chunk: int, num_workers: int,
                 num_bwd_workers: int = 0, q_slice: int = 0, equal_count: bool = False,
                 block_keys_in_context: bool = False, partial_bf16: bool = False,
                 tile_cost: bool = False, fwd_tile_cost: bool = False, dynamic_claim: bool = False,
                 contiguous_schedule: bool = False, contiguous_ranks: bool = False) -> Plan:
    """Host-side mask metadata + LPT schedules (no CUDA call).  block_keys_in_context
    selects reading B of the block keys (SPLITKV_FLAG_BLOCK_KEYS_IN_CONTEXT);
    partial_bf16 stores the partial records as bf16 (SPLITKV_FLAG_PARTIAL_BF16);
    tile_cost / fwd_tile_cost cost the backward / forward LPT items by the executed
    tile work of their kernels (SPLITKV_FLAG_TILE_COST / SPLITKV_FLAG_FWD_TILE_COST);
    dynamic_claim lets the CTAs claim the items in LPT order at run time
    (SPLITKV_FLAG_DYNAMIC_CLAIM); contiguous_schedule replaces LPT by the contiguous
    baseline schedule (SPLITKV_FLAG_CONTIGUOUS_SCHEDULE); contiguous_ranks only matters to rank
    plans (SPLITKV_FLAG_CONTIGUOUS_RANKS)."""
    p, keep = _problem(sample_lens, anchors, block_size, num_q_heads, num_kv_heads, head_dim, kv_chunk,
                       num_workers, num_bwd_workers, q_slice, equal_count, block_keys_in_context, partial_bf16,
                       tile_cost, fwd_tile_cost, dynamic_claim, contiguous_schedule, contiguous_ranks)
    h = ctypes.c_void_p()
    _check("splitkv_plan", _lib.splitkv_plan(ctypes.byref(p), ctypes.byref(h)))
    return Plan(h, p, keep)


def splitkv_plan_shard(sample_lens: Sequence[int], anchors: Sequence[int], block_size: int, num_q_heads: int,
                       num_kv_heads: int, head_dim: int, kv_chunk: int, num_workers: int, num_ranks: int,
                       rank: int, **kw) -> Plan:
    """Rank `rank`'s plan of Split-KV over `num_ranks` ranks (splitkv_plan_shard): the
    chunks it owns and the in-block term of its block range; other options as
    splitkv_plan, plus contiguous_ranks (chunks owned in order, the unbalanced baseline)."""
    p, keep = _problem(sample_lens, anchors, block_size, num_q_heads, num_kv_heads, head_dim, kv_chunk,
                       num_workers, kw.pop("num_bwd_workers", 0), kw.pop("q_slice", 0),
                       kw.pop("equal_count", False), **kw)
    h = ctypes.c_void_p()
    _check("splitkv_plan_shard", _lib.splitkv_plan_shard(ctypes.byref(p), int(num_ranks), int(rank), ctypes.byref(h)))
    return Plan(h, p, keep)


def splitkv_plan_update(plan: Plan, sample_lens, anchors, **kw) -> Plan:
    """Rebuild `plan` in place for new sample lengths / anchors (other fields kept unless given)."""
    old = plan.problem
    args = dict(block_size=old.block_size, num_q_heads=old.num_q_heads, num_kv_heads=old.num_kv_heads,
                head_dim=old.head_dim, kv_chunk=old.kv_chunk, num_workers=old.num_workers,
                num_bwd_workers=old.num_bwd_workers, q_slice=old.q_slice,
                equal_count=bool(old.flags & FLAG_EQUAL_COUNT),
                block_keys_in_context=bool(old.flags & FLAG_BLOCK_KEYS_IN_CONTEXT),
                partial_bf16=bool(old.flags & FLAG_PARTIAL_BF16),
                tile_cost=bool(old.flags & FLAG_TILE_COST),
                fwd_tile_cost=bool(old.flags & FLAG_FWD_TILE_COST),
                dynamic_claim=bool(old.flags & FLAG_DYNAMIC_CLAIM),
                contiguous_schedule=bool(old.flags & FLAG_CONTIGUOUS_SCHEDULE),
                contiguous_ranks=bool(old.flags & FLAG_CONTIGUOUS_RANKS))
    args.update(kw)
    p, keep = _problem(sample_lens, anchors, **args)
    _check("splitkv_plan_update", _lib.splitkv_plan_update(plan.handle, ctypes.byref(p)))
    plan.problem, plan._keep, plan._dims = p, keep, None
    return plan


def splitkv_plan_upload(plan: Plan, stream=None) -> None:
    _check("splitkv_plan_upload", _lib.splitkv_plan_upload(plan.handle, _stream_ptr(stream)))


def splitkv_plan_destroy(plan: Plan) -> None:
    if plan._h:
        h, plan._h = plan._h, None
        _check("splitkv_plan_destroy", _lib.splitkv_plan_destroy(h))


def splitkv_plan_stats(plan: Plan) -> dict:
    s = _abi.Stats()
    _check("splitkv_plan_stats", _lib.splitkv_plan_stats(plan.handle, ctypes.byref(s)))
    return s.as_dict()


def splitkv_plan_export(plan: Plan, what: int) -> np.ndarray:
    n = ctypes.c_int64()
    _check("splitkv_plan_export", _lib.splitkv_plan_export(plan.handle, what, None, 0, ctypes.byref(n)))
    out = np.zeros(max(n.value, 1), dtype=np.int64)
    _check("splitkv_plan_export", _lib.splitkv_plan_export(
        plan.handle, what, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), out.size, ctypes.byref(n)))
    return out[:n.value]


_PROBLEM_FIELDS = ("block_size", "num_q_heads", "num_kv_heads", "head_dim", "kv_chunk", "num_workers",
                   "num_bwd_workers", "q_slice", "flags")
_EXPORTS = ("entries", "chunk_pairs", "fwd_schedule", "bwd_schedule", "fwd_loads", "bwd_loads", "contig_loads",
            "fwd_lpt_order", "bwd_lpt_order", "chunk_owner", "query_shard")


def splitkv_plan_dump(plan: Plan, path: str) -> None:
    """The plan as a reproducible record (.npz): sample lengths, anchors and the other problem
    fields, the stats (plan_us aside, which is a timing), and every SPLITKV_EXPORT_* table.
    Two plans of the same problem give identical dumps (the planner is integer arithmetic)."""
    p = plan.problem
    rec = {"sample_lens": np.ctypeslib.as_array(p.sample_lens, shape=(p.num_samples,)).copy(),
           "anchors": np.ctypeslib.as_array(p.anchors, shape=(p.num_anchors,)).copy()}
    for f in _PROBLEM_FIELDS:
        rec["problem_" + f] = np.int64(getattr(p, f))
    for k, v in splitkv_plan_stats(plan).items():
        if k != "plan_us":
            rec["stats_" + k] = np.asarray(v)
    for i, name in enumerate(_EXPORTS):
        rec[name] = splitkv_plan_export(plan, i)
    np.savez(path, **rec)


def splitkv_plan_load_dump(path: str) -> dict:
    """A dump written by splitkv_plan_dump, as a dict of numpy arrays."""
    with np.load(path) as z:
        return {k: z[k] for k in z.files}


def splitkv_workspace_size(plan: Plan, which: int) -> int:
    n = ctypes.c_size_t()
    _check("splitkv_workspace_size", _lib.splitkv_workspace_size(plan.handle, which, ctypes.byref(n)))
    return n.value


def splitkv_attn_fwd(plan: Plan, q, k, v, scale: float, ws, stream=None) -> None:
    """Chunk partial records into ws (uint8 CUDA tensor of splitkv_workspace_size(plan, WS_FWD) bytes)."""
    _sizes(plan, q=q, k=k, v=v)
    _check("splitkv_attn_fwd", _lib.splitkv_attn_fwd(
        plan.handle, _bf16_ptr(q), _bf16_ptr(k), _bf16_ptr(v), float(scale), _ptr(ws), ws.numel() * ws.element_size(),
        _stream_ptr(stream)))


def splitkv_merge(plan: Plan, q, kb, vb, scale: float, ws, o, lse, stream=None) -> None:
    """In-block term + exact LSE merge of the chunk records -> o (f32 or bf16), lse (f32)."""
    _sizes(plan, q=q, kb=kb, vb=vb, o=o, lse=lse)
    _check("splitkv_merge", _lib.splitkv_merge(
        plan.handle, _bf16_ptr(q), _bf16_ptr(kb), _bf16_ptr(vb), float(scale), _ptr(ws),
        ws.numel() * ws.element_size(), _ptr(o), _o_dtype(o), _f32_ptr(lse), _stream_ptr(stream)))


def splitkv_attn_bwd(plan: Plan, q, k, v, kb, vb, o, lse, dout, dq, dk, dv, dkb, dvb, scale: float, ws,
                     stream=None) -> None:
    """Gradients dq, dk, dv, dkb, dvb (float32) recomputed from the saved lse."""
    _sizes(plan, q=q, k=k, v=v, kb=kb, vb=vb, o=o, lse=lse, dout=dout, dq=dq, dk=dk, dv=dv, dkb=dkb, dvb=dvb)
    _check("splitkv_attn_bwd", _lib.splitkv_attn_bwd(
        plan.handle, _bf16_ptr(q), _bf16_ptr(k), _bf16_ptr(v), _bf16_ptr(kb), _bf16_ptr(vb), _ptr(o),
        _o_dtype(o), _f32_ptr(lse), _bf16_ptr(dout), _f32_ptr(dq), _f32_ptr(dk), _f32_ptr(dv), _f32_ptr(dkb),
        _f32_ptr(dvb), float(scale), _ptr(ws), ws.numel() * ws.element_size(), _stream_ptr(stream)))


def splitkv_bwd_delta(plan: Plan, o, dout, ws, stream=None) -> None:
    _sizes(plan, o=o, dout=dout)
    _check("splitkv_bwd_delta", _lib.splitkv_bwd_delta(
        plan.handle, _ptr(o), _o_dtype(o), _bf16_ptr(dout), _ptr(ws), ws.numel() * ws.element_size(),
        _stream_ptr(stream)))


def splitkv_bwd_partial(plan: Plan, q, k, v, lse, dout, dk, dv, scale: float, ws, stream=None) -> None:
    _sizes(plan, q=q, k=k, v=v, lse=lse, dout=dout, dk=dk, dv=dv)
    _check("splitkv_bwd_partial", _lib.splitkv_bwd_partial(
        plan.handle, _bf16_ptr(q), _bf16_ptr(k), _bf16_ptr(v), _f32_ptr(lse), _bf16_ptr(dout), _f32_ptr(dk),
        _f32_ptr(dv), float(scale), _ptr(ws), ws.numel() * ws.element_size(), _stream_ptr(stream)))


def splitkv_bwd_dkdv(plan: Plan, q, k, v, lse, dout, dk, dv, scale: float, ws, stream=None) -> None:
    _sizes(plan, q=q, k=k, v=v, lse=lse, dout=dout, dk=dk, dv=dv)
    _check("splitkv_bwd_dkdv", _lib.splitkv_bwd_dkdv(
        plan.handle, _bf16_ptr(q), _bf16_ptr(k), _bf16_ptr(v), _f32_ptr(lse), _bf16_ptr(dout), _f32_ptr(dk),
        _f32_ptr(dv), float(scale), _ptr(ws), ws.numel() * ws.element_size(), _stream_ptr(stream)))


def splitkv_bwd_dq(plan: Plan, q, k, v, lse, dout, scale: float, ws, stream=None) -> None:
    _sizes(plan, q=q, k=k, v=v, lse=lse, dout=dout)
    _check("splitkv_bwd_dq", _lib.splitkv_bwd_dq(
        plan.handle, _bf16_ptr(q), _bf16_ptr(k), _bf16_ptr(v), _f32_ptr(lse), _bf16_ptr(dout), float(scale),
        _ptr(ws), ws.numel() * ws.element_size(), _stream_ptr(stream)))


def splitkv_bwd_reduce(plan: Plan, q, kb, vb, lse, dout, dq, dkb, dvb, scale: float, ws, stream=None) -> None:
    _sizes(plan, q=q, kb=kb, vb=vb, lse=lse, dout=dout, dq=dq, dkb=dkb, dvb=dvb)
    _check("splitkv_bwd_reduce", _lib.splitkv_bwd_reduce(
        plan.handle, _bf16_ptr(q), _bf16_ptr(kb), _bf16_ptr(vb), _f32_ptr(lse), _bf16_ptr(dout), _f32_ptr(dq),
        _f32_ptr(dkb), _f32_ptr(dvb), float(scale), _ptr(ws), ws.numel() * ws.element_size(),
        _stream_ptr(stream)))


def splitkv_attn_fwd_static_scratch(plan: Plan, q, k, v, kb, vb, scale: float, o, lse, stream=None) -> None:
    """Forward + merge with the partial records in the library's static device buffer (no allocation)."""
    _sizes(plan, q=q, k=k, v=v, kb=kb, vb=vb, o=o, lse=lse)
    _check("splitkv_attn_fwd_static_scratch", _lib.splitkv_attn_fwd_static_scratch(
        plan.handle, _bf16_ptr(q), _bf16_ptr(k), _bf16_ptr(v), _bf16_ptr(kb), _bf16_ptr(vb), float(scale),
        _ptr(o), _o_dtype(o), _f32_ptr(lse), _stream_ptr(stream)))


def splitkv_plan_set_wait_limit(plan: Plan, ns: int) -> None:
    """Time limit (ns) of the mbarrier waits in this plan's tcgen05 kernels (default 2e9);
    from the next launch on."""
    _check("splitkv_plan_set_wait_limit", _lib.splitkv_plan_set_wait_limit(plan.handle, int(ns)))


def splitkv_plan_status(plan: Plan, stream=None) -> None:
    """Raise SplitKVError if a kernel of this plan recorded an error (e.g. a timed-out wait)."""
    site = ctypes.c_int32(0)
    st = _lib.splitkv_plan_status(plan.handle, _stream_ptr(stream), ctypes.byref(site))
    if st != _abi.OK:
        err = SplitKVError("splitkv_plan_status", st)
        err.site = site.value
        raise _with_site(err, site.value)


def splitkv_read_cta_times(plan: Plan, which: int, stream=None) -> np.ndarray:
    """Per-CTA busy nanoseconds of the last forward (WS_FWD), dK/dV (WS_BWD) or dQ (TIMES_DQ)
    partial kernel."""
    st = plan.stats()
    n = st["num_bwd_workers"] if which == WS_BWD else st["num_workers"]
    out = np.zeros(n, dtype=np.int64)
    _check("splitkv_read_cta_times", _lib.splitkv_read_cta_times(
        plan.handle, which, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n, _stream_ptr(stream)))
    return out


def splitkv_merge_to_owners(plan: Plan, q, kb, vb, scale: float, ws, o_dest, lse_dest, stream=None) -> None:
    """The merge of a rank plan writing each block's rows into its owner's receive buffers:
    o_dest, lse_dest are int64 CUDA tensors [R] of device addresses (o: float32 [R][rows_r][Hq][d],
    lse: float32 [R][rows_r][Hq] on rank r)."""
    import torch
    shard = splitkv_plan_export(plan, EXPORT_QUERY_SHARD).tolist()
    for name, t in (("o_dest", o_dest), ("lse_dest", lse_dest)):
        if t.dtype != torch.int64 or t.numel() != shard[1]:
            raise ValueError(f"{name} must be an int64 tensor of {shard[1]} device addresses")
    _sizes(plan, q=q, kb=kb, vb=vb)
    _check("splitkv_merge_to_owners", _lib.splitkv_merge_to_owners(
        plan.handle, _bf16_ptr(q), _bf16_ptr(kb), _bf16_ptr(vb), float(scale), _ptr(ws),
        ws.numel() * ws.element_size(), shard[1], shard[0], _ptr(o_dest), _ptr(lse_dest), _stream_ptr(stream)))


def splitkv_bwd_reduce_to_owners(plan: Plan, q, kb, vb, lse, dout, dkb, dvb, scale: float, ws, dq_dest,
                                 stream=None) -> None:
    """The dQ reduce of a rank plan writing each block's dq rows into its owner's receive
    buffer: dq_dest is an int64 CUDA tensor [R] of device addresses (float32 [R][rows_r][Hq][d]
    on rank r)."""
    import torch
    shard = splitkv_plan_export(plan, EXPORT_QUERY_SHARD).tolist()
    if dq_dest.dtype != torch.int64 or dq_dest.numel() != shard[1]:
        raise ValueError(f"dq_dest must be an int64 tensor of {shard[1]} device addresses")
    _sizes(plan, q=q, kb=kb, vb=vb, lse=lse, dout=dout, dkb=dkb, dvb=dvb)
    _check("splitkv_bwd_reduce_to_owners", _lib.splitkv_bwd_reduce_to_owners(
        plan.handle, _bf16_ptr(q), _bf16_ptr(kb), _bf16_ptr(vb), _f32_ptr(lse), _bf16_ptr(dout), _f32_ptr(dkb),
        _f32_ptr(dvb), float(scale), _ptr(ws), ws.numel() * ws.element_size(), shard[1], shard[0], _ptr(dq_dest),
        _stream_ptr(stream)))


def splitkv_enable_peer_access(peer_device: int) -> None:
    """Let kernels on the current device access memory of `peer_device` (no-op when it is
    the current device or access is already on)."""
    _check("splitkv_enable_peer_access", _lib.splitkv_enable_peer_access(int(peer_device)))


def splitkv_combine_ranks(o_parts, lse_parts, o, lse, stream=None) -> None:
    """o_parts [R, rows..., d] and lse_parts [R, rows...] float32 -> o [rows..., d] (float32 or
    bfloat16) and lse [rows...]: the exact combine of R ranks' results."""
    R = int(o_parts.shape[0])
    d = int(o_parts.shape[-1])
    rows = int(lse_parts[0].numel()) if R else 0
    if tuple(lse_parts.shape) != tuple(o_parts.shape[:-1]) or o.numel() != rows * d or lse.numel() != rows:
        raise ValueError("o_parts [R, rows..., d], lse_parts [R, rows...], o [rows..., d], lse [rows...]")
    _check("splitkv_combine_ranks", _lib.splitkv_combine_ranks(R, rows, d, _f32_ptr(o_parts), _f32_ptr(lse_parts),
                                                               _ptr(o), _o_dtype(o), _f32_ptr(lse),
                                                               _stream_ptr(stream)))


def splitkv_sum_ranks(parts, out, stream=None) -> None:
    """parts [R, ...] float32 -> out [...] = the sum over R, in rank order."""
    R = int(parts.shape[0])
    n = int(out.numel())
    if parts.numel() != R * n:
        raise ValueError("parts must be [R, *out.shape]")
    _check("splitkv_sum_ranks", _lib.splitkv_sum_ranks(R, n, _f32_ptr(parts), _f32_ptr(out), _stream_ptr(stream)))


def splitkv_cast_bf16(src, dst, stream=None) -> None:
    """dst (bfloat16) = src (float32) rounded to nearest even, element by element."""
    import torch
    if src.dtype != torch.float32 or dst.dtype != torch.bfloat16:
        raise ValueError("src must be float32 and dst bfloat16")
    if src.numel() != dst.numel() or not src.is_contiguous() or not dst.is_contiguous():
        raise ValueError("src and dst must be contiguous with the same number of elements")
    _check("splitkv_cast_bf16", _lib.splitkv_cast_bf16(int(src.numel()), _ptr(src), _ptr(dst), _stream_ptr(stream)))


def splitkv_selftest_wait_timeout(stream=None):
    """Run the bounded-wait self-test; returns the status words (code, site) it recorded."""
    out = (ctypes.c_int32 * 2)()
    _check("splitkv_selftest_wait_timeout", _lib.splitkv_selftest_wait_timeout(out, _stream_ptr(stream)))
    return int(out[0]), int(out[1])


def library_path() -> str:
    return _abi.LIB_PATH
