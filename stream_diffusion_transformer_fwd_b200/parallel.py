"""Multi-GPU layouts of the Ideogram 4 block: tensor parallelism over heads
(TP) and Ulysses sequence parallelism over the image tokens (SP).

Source: "SGLang cookbook: Ideogram 4", section 3 (tensor and sequence
parallelism): TP shards the DiT weights, with a degree that divides the 18
attention heads; Ulysses SP keeps the weights whole on every GPU and shards
the image-token sequence.  Both were validated there on two B200s at
1024 x 1024.

One process per GPU.  Each rank's share of the block runs in the library's
kernels (include/ig4.h, "multi-GPU layouts"); between those calls the ranks
exchange data through a torch.distributed process group (NCCL between GPUs).
The per-rank steps are passed in as an ``ops`` object, so the same exchange
logic drives the CUDA library (``Ig4TpOps``, ``Ig4SpOps``) or any other
implementation of the steps with the same buffer layouts.

TP, per block on rank r of P:
    attention(x) -> partial_r ; all-reduce(sum) ; reduce -> x1 (stream dtype)
    mlp(x1)      -> partial_r ; all-reduce(sum) ; reduce -> y
SP, per block on rank r of P (local tokens: the text and the r-th share of
the image tokens):
    pre(x_local)  -> phase-0 send buffer ; all-to-all
    attention     -> phase-1 send buffer ; all-to-all
    post(x_local) -> y_local
"""

from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


# ---------------------------------------------------------------- weights

def tp_shard_weights(w: dict, rank: int, size: int, D: int, H: int, I: int,
                     head_dim: int = 256) -> dict:
    """One block's weights (dict as for ig4.block_weights) cut to TP rank
    `rank` of `size`: the q, k and v rows of its heads, the matching columns
    of w_o, its rows of w_gate / w_up and columns of w_down (per-output-channel
    scales follow the rows); everything else whole.  Works on host or device
    tensors; FP8 codes are cut as bytes."""
    if H % size or I % size:
        raise ValueError(f"TP degree {size} must divide H={H} and I={I}")
    hs = H // size * head_dim
    q0, i0, i_s = rank * hs, rank * (I // size), I // size

    def cut_rows(t, starts, n):
        if t is None:
            return None
        b = t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t
        out = torch.cat([b[s:s + n] for s in starts]).contiguous()
        return out.view(t.dtype) if t.dtype == torch.float8_e4m3fn else out

    def cut_cols(t, start, n):
        b = t.view(torch.uint8) if t.dtype == torch.float8_e4m3fn else t
        out = b[:, start:start + n].contiguous()
        return out.view(t.dtype) if t.dtype == torch.float8_e4m3fn else out

    out = dict(w)
    qkv_starts = [q0, D + q0, 2 * D + q0]
    out["w_qkv"] = cut_rows(w["w_qkv"], qkv_starts, hs)
    out["s_qkv"] = cut_rows(w.get("s_qkv"), qkv_starts, hs)
    out["w_o"] = cut_cols(w["w_o"], q0, hs)
    for name in ("gate", "up"):
        out["w_" + name] = cut_rows(w["w_" + name], [i0], i_s)
        out["s_" + name] = cut_rows(w.get("s_" + name), [i0], i_s)
    out["w_down"] = cut_cols(w["w_down"], i0, i_s)
    return out


# ------------------------------------------------------------ exchanges

class Collectives:
    """The two exchanges the layouts use, over a torch.distributed group
    (NCCL for GPU tensors, gloo for CPU tensors)."""

    def __init__(self, group=None):
        self.group = group

    def all_reduce_sum(self, t: torch.Tensor):
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)

    def all_to_all(self, recv: torch.Tensor, send: torch.Tensor, recv_splits: list,
                   send_splits: list):
        dist.all_to_all_single(recv, send, recv_splits, send_splits, group=self.group)


# ------------------------------------------------------------------- TP

def tp_block_forward(ops, coll, x, y, partial, x1):
    """One block on one TP rank: y = block(x), x and y replicated on every
    rank.  partial: fp32 [B*L, D]; x1: the stream after the attention branch
    (x's dtype).  ops: attention(x, partial), mlp(x1, partial),
    reduce(list of partials, out)."""
    ops.attention(x, partial)
    coll.all_reduce_sum(partial)
    ops.reduce([partial], x1)
    ops.mlp(x1, partial)
    coll.all_reduce_sum(partial)
    ops.reduce([partial], y)


class Ig4TpOps:
    """The TP steps of one block on this rank, in the CUDA library."""

    def __init__(self, ig4, cfg, rank: int, size: int, w_shard: dict, pos, temb, workspace=None):
        self.ig4, self.rank, self.size = ig4, rank, size
        self.c = ig4.config_from(cfg)
        self._w = w_shard  # keeps the shard's tensors alive
        self.bw = ig4.block_weights(w_shard)
        self.pos, self.temb = pos, temb
        if workspace is None:
            workspace = torch.empty(ig4.ig4_tp_workspace_size(self.c, size), dtype=torch.uint8,
                                    device=temb.device)
        self.ws = workspace

    def attention(self, x, partial):
        self.ig4.ig4_block_tp_attention(self.c, self.rank, self.size, self.bw, x, self.pos,
                                        self.temb, partial, self.ws)

    def mlp(self, x1, partial):
        self.ig4.ig4_block_tp_mlp(self.c, self.rank, self.size, self.bw, x1, partial, self.ws)

    def reduce(self, srcs, out):
        self.ig4.ig4_tp_reduce(srcs, out)


# ------------------------------------------------------------------- SP

@dataclass
class SpPlan:
    """Exchange sizes of Ulysses rank `rank` of `size` (bytes, from the
    library's chunk layout): send[phase][d] to rank d, recv[phase][s] from s."""
    rank: int
    size: int
    send: tuple
    recv: tuple

    @classmethod
    def build(cls, ig4, c, rank: int, size: int) -> "SpPlan":
        send = tuple([ig4.ig4_sp_exchange_bytes(c, size, ph, rank, d) for d in range(size)]
                     for ph in (0, 1))
        recv = tuple([ig4.ig4_sp_exchange_bytes(c, size, ph, s, rank) for s in range(size)]
                     for ph in (0, 1))
        return cls(rank, size, send, recv)

    def buffers(self, device) -> dict:
        return {f"{k}{ph}": torch.empty(sum(getattr(self, k)[ph]), dtype=torch.uint8,
                                        device=device)
                for k in ("send", "recv") for ph in (0, 1)}


def sp_block_forward(ops, coll, plan: SpPlan, x_local, y_local, bufs: dict):
    """One block on one Ulysses rank: y_local = the block's output for this
    rank's local tokens (text + its image share).  bufs: SpPlan.buffers.
    ops: pre(x_local, send0), attention(recv0, send1), post(x_local, y_local,
    recv1)."""
    ops.pre(x_local, bufs["send0"])
    coll.all_to_all(bufs["recv0"], bufs["send0"], plan.recv[0], plan.send[0])
    ops.attention(bufs["recv0"], bufs["send1"])
    coll.all_to_all(bufs["recv1"], bufs["send1"], plan.recv[1], plan.send[1])
    ops.post(x_local, y_local, bufs["recv1"])


class Ig4SpOps:
    """The Ulysses steps of one block on this rank, in the CUDA library."""

    def __init__(self, ig4, cfg, rank: int, size: int, w: dict, temb, workspace=None):
        self.ig4, self.rank, self.size = ig4, rank, size
        self.c = ig4.config_from(cfg)
        self._w = w
        self.bw = ig4.block_weights(w)
        self.temb = temb
        self.pos = ig4.ig4_sp_positions(self.c, size, rank, device=temb.device)
        if workspace is None:
            workspace = torch.empty(ig4.ig4_sp_workspace_size(self.c, size, rank),
                                    dtype=torch.uint8, device=temb.device)
        self.ws = workspace

    def pre(self, x_local, send):
        self.ig4.ig4_block_sp_pre(self.c, self.rank, self.size, self.bw, x_local, self.pos,
                                  self.temb, send, self.ws)

    def attention(self, recv, send_o):
        self.ig4.ig4_block_sp_attention(self.c, self.rank, self.size, recv, send_o, self.ws)

    def post(self, x_local, y_local, recv_o):
        self.ig4.ig4_block_sp_post(self.c, self.rank, self.size, self.bw, x_local, y_local,
                                   recv_o, self.ws)


def sp_local_tokens(x, T: int, img_off: int, img_count: int):
    """[B, T + img_count, D] local sequence of a rank from the whole [B, L, D]."""
    return torch.cat([x[:, :T], x[:, T + img_off:T + img_off + img_count]], dim=1).contiguous()
