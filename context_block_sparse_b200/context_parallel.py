"""Split-KV over the ranks of a process group: one rank per GPU.

The method (news page "Split-KV speeds diffusion drafter training by keeping
long-context data local", sections "Exchange the smaller side" and "Balance
actual attention work"; digest page "Split-KV: Efficient Context Parallelism for
Training Diffusion Drafters", Abstract): every rank keeps its own chunks of the
long context's keys and values; the short query side -- the draft blocks --
moves instead.  Each rank computes every query row's exact partial result over
its keys, and the owner of a query row combines the ranks' results with their
log-sum-exp statistics.  Chunks go to ranks by LPT on their realised attention
cost with equal chunk counts.

Per step, on every rank (R ranks, this one r):

  forward   q (the rank's block rows) --broadcast from each rank--> q of every row
            local: splitkv_attn_fwd + splitkv_merge on the rank plan -> O_r, LSE_r
            for every row; all-to-all of rows -> the R results of this rank's rows;
            splitkv_combine_ranks -> O, LSE of this rank's rows
  backward  dout, o, lse of the rank's rows --broadcast--> every row
            local: splitkv_attn_bwd on the rank plan -> every row's dq share,
            complete dk, dv of the rank's chunks, dkb, dvb of its blocks;
            all-to-all of dq rows; splitkv_sum_ranks -> dq of this rank's rows

dk and dv never leave the rank that owns their chunks.  Every arithmetic step
runs in the library's kernels; this module moves rows between ranks
(torch.distributed: NCCL between GPUs) and allocates buffers.
"""

from __future__ import annotations

from typing import Dict, List, Optional, Tuple

import torch
import torch.distributed as dist

from . import (
    EXPORT_CHUNK_OWNER, EXPORT_QUERY_SHARD, WS_BWD, WS_FWD, splitkv_attn_bwd, splitkv_attn_fwd, splitkv_bwd_delta,
    splitkv_bwd_partial, splitkv_bwd_reduce_to_owners, splitkv_combine_ranks, splitkv_enable_peer_access,
    splitkv_merge,
    splitkv_merge_to_owners, splitkv_plan_shard, splitkv_sum_ranks, splitkv_workspace_size,
)


def block_ranges(num_blocks: int, num_ranks: int) -> List[Tuple[int, int]]:
    """Blocks [lo, hi) of every rank: contiguous, rank r from floor(r A / R)."""
    return [((r * num_blocks) // num_ranks, ((r + 1) * num_blocks) // num_ranks) for r in range(num_ranks)]


class KernelOps:
    """The local steps of one rank on its GPU, through the C entry points."""

    def __init__(self, plan, num_queries: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 context_len: int, device, block_keys_in_context: bool):
        self.plan = plan
        self.Nq, self.Hq, self.Hkv, self.d, self.N = num_queries, num_q_heads, num_kv_heads, head_dim, context_len
        self.device = torch.device(device)
        self.rb = block_keys_in_context
        self.ws_fwd = torch.empty(splitkv_workspace_size(plan, WS_FWD), dtype=torch.uint8, device=self.device)
        self._ws_bwd = None
        self._dkv = None

    def local_fwd(self, q, k, v, kb, vb, scale: float):
        f32 = dict(dtype=torch.float32, device=self.device)
        o = torch.empty((self.Nq, self.Hq, self.d), **f32)
        lse = torch.empty((self.Nq, self.Hq), **f32)
        splitkv_attn_fwd(self.plan, q, k, v, scale, self.ws_fwd)
        splitkv_merge(self.plan, q, kb, vb, scale, self.ws_fwd, o, lse)
        return o, lse

    def local_fwd_to_owners(self, q, k, v, kb, vb, scale: float, dest_o, dest_lse):
        """The forward with the exchange fused into the merge: rows go straight into the
        owners' receive buffers (device addresses in dest_o / dest_lse)."""
        splitkv_attn_fwd(self.plan, q, k, v, scale, self.ws_fwd)
        splitkv_merge_to_owners(self.plan, q, kb, vb, scale, self.ws_fwd, dest_o, dest_lse)

    def combine(self, o_parts, lse_parts, out_dtype):
        o = torch.empty(o_parts.shape[1:], dtype=out_dtype, device=self.device)
        lse = torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=self.device)
        splitkv_combine_ranks(o_parts, lse_parts, o, lse)
        return o, lse

    def _bwd_buffers(self) -> Dict[str, torch.Tensor]:
        f32 = dict(dtype=torch.float32, device=self.device)
        if self._ws_bwd is None:
            self._ws_bwd = torch.empty(splitkv_workspace_size(self.plan, WS_BWD), dtype=torch.uint8,
                                       device=self.device)
            # rows of other ranks' chunks (blocks) are never written: zero them once
            self._dkv = {"dk": torch.zeros((self.N, self.Hkv, self.d), **f32),
                         "dv": torch.zeros((self.N, self.Hkv, self.d), **f32),
                         "dkb": None if self.rb else torch.zeros((self.Nq, self.Hkv, self.d), **f32),
                         "dvb": None if self.rb else torch.zeros((self.Nq, self.Hkv, self.d), **f32)}
        return dict(self._dkv)

    def local_bwd(self, q, k, v, kb, vb, o, lse, dout, scale: float) -> Dict[str, torch.Tensor]:
        g = self._bwd_buffers()
        g["dq"] = torch.empty((self.Nq, self.Hq, self.d), dtype=torch.float32, device=self.device)
        splitkv_attn_bwd(self.plan, q, k, v, kb, vb, o, lse, dout, g["dq"], g["dk"], g["dv"], g["dkb"], g["dvb"],
                         scale, self._ws_bwd)
        return g

    def local_bwd_to_owners(self, q, k, v, kb, vb, o, lse, dout, scale: float, dest_dq) -> Dict[str, torch.Tensor]:
        """The backward with the dq exchange fused into the dQ reduce: dq rows go straight into
        the owners' receive buffers (device addresses in dest_dq); returns dk, dv, dkb, dvb."""
        g = self._bwd_buffers()
        splitkv_bwd_delta(self.plan, o, dout, self._ws_bwd)
        splitkv_bwd_partial(self.plan, q, k, v, lse, dout, g["dk"], g["dv"], scale, self._ws_bwd)
        splitkv_bwd_reduce_to_owners(self.plan, q, kb, vb, lse, dout, g["dkb"], g["dvb"], scale, self._ws_bwd,
                                     dest_dq)
        return g

    def sum(self, parts):
        out = torch.empty(parts.shape[1:], dtype=torch.float32, device=self.device)
        splitkv_sum_ranks(parts, out)
        return out


class SplitKVContextParallel:
    """One rank of Split-KV over `group` (default: the world).

    Inputs of a step on this rank: the query-side rows of its blocks
    (`block_range`): q, kb, vb, and in the backward dout and its own o, lse; the
    context keys and values k, v [N, Hkv, d] addressed by global position, of
    which only the rows of its chunks (`owned_rows`) are read (other rows must
    hold finite values; zeros will do).  Outputs: o, lse, dq, dkb, dvb of its
    block rows; dk, dv [N, Hkv, d], complete on its chunks' rows and zero
    elsewhere.
    """

    def __init__(self, sample_lens, anchors, block_size: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 kv_chunk: int, group=None, num_workers: Optional[int] = None, device=None, ops=None,
                 exchange: str = "nccl", **plan_kw):
        """ops: the local steps (default: the library's kernels on `device`), or a factory
        called with this object; exchange: "nccl" (all-to-all of result rows) or "p2p" (the
        forward merge stores each row into its owner's receive buffer, mapped into every rank
        by CUDA IPC; ranks of one node with peer access); plan_kw: options of splitkv_plan
        (q_slice, tile_cost, ...)."""
        if exchange not in ("nccl", "p2p"):
            raise ValueError("exchange is 'nccl' or 'p2p'")
        self.exchange = exchange
        self.group = group
        self.R = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.bs = int(block_size)
        self.A = len(anchors)
        self.Hq, self.Hkv, self.d = int(num_q_heads), int(num_kv_heads), int(head_dim)
        self.N = int(sum(int(x) for x in sample_lens))
        self.kv_chunk = int(kv_chunk)
        self.rb = bool(plan_kw.get("block_keys_in_context", False))
        if num_workers is None:
            num_workers = torch.cuda.get_device_properties(device or "cuda").multi_processor_count
        self.plan = splitkv_plan_shard(sample_lens, anchors, block_size, num_q_heads, num_kv_heads, head_dim,
                                       kv_chunk, num_workers, self.R, self.rank, **plan_kw)
        shard = self.plan.export(EXPORT_QUERY_SHARD).tolist()
        self.ranges = block_ranges(self.A, self.R)
        if shard != [self.rank, self.R, *self.ranges[self.rank]]:
            raise RuntimeError(f"rank plan holds blocks {shard[2:]}, expected {self.ranges[self.rank]}")
        self.chunk_owner = self.plan.export(EXPORT_CHUNK_OWNER).tolist()
        self.row_counts = [(hi - lo) * self.bs for lo, hi in self.ranges]
        self.row_starts = [lo * self.bs for lo, _ in self.ranges]
        if ops is None:
            self.plan.upload()
            ops = KernelOps(self.plan, self.A * self.bs, self.Hq, self.Hkv, self.d, self.N,
                            device or torch.device("cuda", torch.cuda.current_device()), self.rb)
        elif not hasattr(ops, "local_fwd"):
            ops = ops(self)          # a factory given this rank's layout
        self.ops = ops
        self._saved = None
        self._bufs = {}
        self._p2p = None

    def _buffer(self, name: str, like: torch.Tensor, zero: bool = False) -> torch.Tensor:
        """A full-size (every query row) buffer kept across steps: the query side has the same
        shape every step, and rows other ranks never send stay as first written (zero)."""
        shape = (sum(self.row_counts),) + tuple(like.shape[1:])
        b = self._bufs.get(name)
        if b is None or tuple(b.shape) != shape or b.dtype != like.dtype or b.device != like.device:
            b = (torch.zeros if zero else torch.empty)(shape, dtype=like.dtype, device=like.device)
            self._bufs[name] = b
        return b

    # ---- layout
    @property
    def block_range(self) -> Tuple[int, int]:
        return self.ranges[self.rank]

    @property
    def rows(self) -> slice:
        """This rank's query rows (token-major, bs rows per block)."""
        return slice(self.row_starts[self.rank], self.row_starts[self.rank] + self.row_counts[self.rank])

    def owned_rows(self) -> List[Tuple[int, int]]:
        """Context rows [lo, hi) of the chunks this rank owns, ascending."""
        C = self.kv_chunk
        return [(c * C, min((c + 1) * C, self.N)) for c, o in enumerate(self.chunk_owner) if o == self.rank]

    # ---- row movement
    def _gather_rows(self, name: str, shard: torch.Tensor) -> torch.Tensor:
        """Every rank's block rows, in block order: one broadcast per rank into its rows."""
        full = self._buffer(name, shard)
        full[self.rows].copy_(shard)
        for r in range(self.R):
            if self.row_counts[r]:
                part = full[self.row_starts[r]:self.row_starts[r] + self.row_counts[r]]
                dist.broadcast(part, src=dist.get_global_rank(self.group, r) if self.group is not None else r,
                               group=self.group)
        return full

    def _place_rows(self, name: str, shard: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
        """A full-size buffer holding this rank's block rows (the only rows it reads)."""
        if shard is None:
            return None
        full = self._buffer(name, shard, zero=True)
        full[self.rows].copy_(shard)
        return full

    def _to_owners(self, full: torch.Tensor) -> torch.Tensor:
        """Rows of every query row, computed here, sent to the rows' owners: returns
        [R, rows of this rank, ...] (rank r's values at index r)."""
        mine = self.row_counts[self.rank]
        out = torch.empty((self.R * mine,) + tuple(full.shape[1:]), dtype=full.dtype, device=full.device)
        dist.all_to_all_single(out, full.contiguous(), [mine] * self.R, self.row_counts, group=self.group)
        return out.view((self.R, mine) + tuple(full.shape[1:]))

    def _p2p_buffers(self, device):
        """This rank's receive buffers ([R][rows][Hq][d], [R][rows][Hq]) and the device
        addresses of every rank's, mapped here through CUDA IPC (set up once)."""
        if self._p2p is None:
            from torch.multiprocessing.reductions import reduce_tensor
            mine = self.row_counts[self.rank]
            f32 = dict(dtype=torch.float32, device=device)
            recv_o = torch.zeros((self.R, mine, self.Hq, self.d), **f32)
            recv_l = torch.zeros((self.R, mine, self.Hq), **f32)
            handles = [None] * self.R
            if self.R > 1:
                # one-rank groups share nothing: an IPC handle that no other process opens
                # would stay registered with torch's producer-side reference count until exit
                dist.all_gather_object(handles, (reduce_tensor(recv_o), reduce_tensor(recv_l)),
                                       group=self.group)
            peers, ptr_o, ptr_l = [], [], []
            for r, h in enumerate(handles):
                to, tl = (recv_o, recv_l) if r == self.rank else (h[0][0](*h[0][1]), h[1][0](*h[1][1]))
                if to.device != recv_o.device:
                    # the IPC mapping is opened under the owner's device: this device's
                    # kernels store into it only with peer access switched on here
                    with torch.cuda.device(recv_o.device):
                        splitkv_enable_peer_access(to.device.index)
                peers.append((to, tl))          # keeps the mappings open
                ptr_o.append(to.data_ptr())
                ptr_l.append(tl.data_ptr())
            self._p2p = {"o": recv_o, "lse": recv_l, "peers": peers,
                         "dest_o": torch.tensor(ptr_o, dtype=torch.int64, device=device),
                         "dest_lse": torch.tensor(ptr_l, dtype=torch.int64, device=device),
                         "flag": torch.zeros(1, dtype=torch.float32, device=device)}
        return self._p2p

    def _stream_barrier(self, flag: torch.Tensor) -> None:
        """Every rank past this point in stream order: a one-element all-reduce."""
        dist.all_reduce(flag, group=self.group)

    # ---- steps
    def forward(self, q, k, v, kb, vb, scale: float, out_dtype=torch.float32):
        q_full = self._gather_rows("q", q)
        kb_full, vb_full = self._place_rows("kb", kb), self._place_rows("vb", vb)
        if self.exchange == "p2p":
            b = self._p2p_buffers(q.device)
            self.ops.local_fwd_to_owners(q_full, k, v, kb_full, vb_full, scale, b["dest_o"], b["dest_lse"])
            self._stream_barrier(b["flag"])          # every rank's rows have landed
            o, lse = self.ops.combine(b["o"], b["lse"], out_dtype)
            self._stream_barrier(b["flag"])          # every owner has read before the next writes
        else:
            o_r, lse_r = self.ops.local_fwd(q_full, k, v, kb_full, vb_full, scale)
            o, lse = self.ops.combine(self._to_owners(o_r), self._to_owners(lse_r), out_dtype)
        self._saved = (q_full, kb_full, vb_full)
        return o, lse

    def backward(self, k, v, o, lse, dout, scale: float) -> Dict[str, torch.Tensor]:
        if self._saved is None:
            raise RuntimeError("backward needs a forward first")
        q_full, kb_full, vb_full = self._saved
        o_full, lse_full, dout_full = (self._gather_rows("o", o), self._gather_rows("lse", lse),
                                       self._gather_rows("dout", dout))
        if self.exchange == "p2p":
            b = self._p2p_buffers(dout.device)      # the forward's receive buffers take the dq rows
            g = self.ops.local_bwd_to_owners(q_full, k, v, kb_full, vb_full, o_full, lse_full, dout_full, scale,
                                             b["dest_o"])
            self._stream_barrier(b["flag"])          # every rank's dq rows have landed
            dq = self.ops.sum(b["o"])
            self._stream_barrier(b["flag"])          # every owner has read before the next writes
        else:
            g = self.ops.local_bwd(q_full, k, v, kb_full, vb_full, o_full, lse_full, dout_full, scale)
            dq = self.ops.sum(self._to_owners(g["dq"]))
        out = {"dq": dq, "dk": g["dk"], "dv": g["dv"]}
        for n in ("dkb", "dvb"):
            out[n] = None if g[n] is None else g[n][self.rows]
        return out
