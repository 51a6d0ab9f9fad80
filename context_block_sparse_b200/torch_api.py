"""Convenience wrapper over the C entry points for torch users.

Allocates the outputs and workspaces with torch (device memory only) and calls
splitkv_attn_fwd / splitkv_merge / splitkv_attn_bwd in order on the current
stream.  No arithmetic happens here.
"""

from __future__ import annotations

from typing import Optional

import torch

from . import (
    WS_BWD, WS_FWD, Plan, splitkv_attn_bwd, splitkv_attn_fwd, splitkv_cast_bf16, splitkv_merge, splitkv_plan,
    splitkv_plan_upload, splitkv_workspace_size,
)


class SplitKVAttention:
    """One problem (packed samples + anchors + head layout) bound to a device plan."""

    def __init__(self, sample_lens, anchors, block_size: int, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, kv_chunk: int, num_workers: Optional[int] = None,
                 num_bwd_workers: int = 0, q_slice: int = 0, equal_count: bool = False,
                 device: Optional[torch.device] = None, block_keys_in_context: bool = False,
                 partial_bf16: bool = False, tile_cost: bool = False, fwd_tile_cost: bool = False,
                 dynamic_claim: bool = False, contiguous_schedule: bool = False):
        """block_keys_in_context: reading B of the block keys (the block's own tokens are
        the context positions after its anchor); kb, vb are then unused (pass None)
        and backward() returns no dkb, dvb.  partial_bf16: bf16 partial records.
        tile_cost / fwd_tile_cost: backward / forward LPT items costed by executed tile work.
        dynamic_claim: the CTAs claim the items in LPT order at run time.
        contiguous_schedule: the contiguous baseline schedule instead of LPT."""
        self.device = torch.device("cuda") if device is None else torch.device(device)
        if num_workers is None:
            num_workers = torch.cuda.get_device_properties(self.device).multi_processor_count
        self.plan: Plan = splitkv_plan(sample_lens, anchors, block_size, num_q_heads, num_kv_heads, head_dim,
                                       kv_chunk, num_workers, num_bwd_workers, q_slice, equal_count,
                                       block_keys_in_context, partial_bf16, tile_cost, fwd_tile_cost,
                                       dynamic_claim, contiguous_schedule)
        self.block_keys_in_context = bool(block_keys_in_context)
        splitkv_plan_upload(self.plan)
        self.block_size = block_size
        self.num_q_heads = num_q_heads
        self.num_kv_heads = num_kv_heads
        self.head_dim = head_dim
        self.ws_fwd = torch.empty(splitkv_workspace_size(self.plan, WS_FWD), dtype=torch.uint8, device=self.device)
        self._ws_bwd = None
        self._grad32 = None   # float32 gradients behind bf16 ones (grad_dtype=torch.bfloat16)

    def ws_bwd(self) -> torch.Tensor:
        if self._ws_bwd is None:
            self._ws_bwd = torch.empty(splitkv_workspace_size(self.plan, WS_BWD), dtype=torch.uint8,
                                       device=self.device)
        return self._ws_bwd

    def forward(self, q, k, v, kb, vb, scale: float, out_dtype=torch.float32, o=None, lse=None):
        Nq = q.shape[0]
        if o is None:
            o = torch.empty((Nq, self.num_q_heads, self.head_dim), dtype=out_dtype, device=q.device)
        if lse is None:
            lse = torch.empty((Nq, self.num_q_heads), dtype=torch.float32, device=q.device)
        splitkv_attn_fwd(self.plan, q, k, v, scale, self.ws_fwd)
        splitkv_merge(self.plan, q, kb, vb, scale, self.ws_fwd, o, lse)
        return o, lse

    def _grad_buffers(self, q, k, v, kb, vb, dtype):
        a = dict(dtype=dtype, device=q.device)
        return {
            "dq": torch.empty(q.shape, **a),
            "dk": torch.empty(k.shape, **a),
            "dv": torch.empty(v.shape, **a),
            "dkb": None if self.block_keys_in_context else torch.empty(kb.shape, **a),
            "dvb": None if self.block_keys_in_context else torch.empty(vb.shape, **a),
        }

    def backward(self, q, k, v, kb, vb, o, lse, dout, scale: float, grads=None, grad_dtype=torch.float32):
        """Gradients dq, dk, dv (and dkb, dvb).  grad_dtype=torch.bfloat16 returns them in bf16:
        the kernels still accumulate in fp32 (into buffers kept by this object), and
        splitkv_cast_bf16 rounds the finished arrays."""
        if grad_dtype not in (torch.float32, torch.bfloat16):
            raise ValueError("grad_dtype must be torch.float32 or torch.bfloat16")
        if grads is None:
            grads = self._grad_buffers(q, k, v, kb, vb, grad_dtype)
        if grad_dtype == torch.float32:
            g32 = grads
        else:
            if self._grad32 is None or self._grad32["dq"].shape != q.shape or self._grad32["dk"].shape != k.shape:
                self._grad32 = self._grad_buffers(q, k, v, kb, vb, torch.float32)
            g32 = self._grad32
        splitkv_attn_bwd(self.plan, q, k, v, kb, vb, o, lse, dout, g32["dq"], g32["dk"], g32["dv"],
                         g32["dkb"], g32["dvb"], scale, self.ws_bwd())
        if grad_dtype == torch.bfloat16:
            for n, t in grads.items():
                if t is not None:
                    splitkv_cast_bf16(g32[n], t)
        return grads
