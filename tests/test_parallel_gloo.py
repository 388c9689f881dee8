"""The exchange logic of the multi-GPU layouts on the CPU, with gloo ranks.

tp_block_forward and sp_block_forward (stream_diffusion_transformer_fwd_b200
.parallel) run in 2 or 3 processes over a gloo process group.  Each rank's
steps are stand-ins written with the fp64 oracle's functions, exchanging
buffers in the layouts include/ig4.h documents for the library's kernels:
TP partial sums (fp32 there, fp64 here) and the Ulysses chunks (bf16 bytes,
sizes from the library's own ig4_sp_exchange_bytes, positions from
ig4_sp_positions).  The result assembled on rank 0 must match the oracle's
plain block: to fp64 rounding for TP, within bf16 exchange rounding for SP.
This checks the weight sharding, the order and sizes of the collectives and
the decomposition itself; the kernels are checked on the GPU
(test_gpu_parallel.py).
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
from oracle.inputs import block_weights_f64, to_f64
from synth import CONFIGS, make_block_activations, make_block_weights

CFGS = {
    "tp2": (CONFIGS["tiny"].with_(name="g_tp2", B=2, T_text=5, grid_h=4, grid_w=6, D=512, H=2,
                                  I=256), 2),
    "tp2_fp8": (CONFIGS["tiny"].with_(name="g_tp2_fp8", B=1, T_text=7, grid_h=5, grid_w=5,
                                      D=512, H=2, I=256, w_dtype="e4m3"), 2),
    "tp3": (CONFIGS["tiny"].with_(name="g_tp3", B=1, T_text=6, grid_h=4, grid_w=5, D=768, H=3,
                                  I=384), 3),
    "sp2": (CONFIGS["tiny"].with_(name="g_sp2", B=2, T_text=5, grid_h=5, grid_w=7, D=512, H=2,
                                  I=256), 2),
    "sp3": (CONFIGS["tiny"].with_(name="g_sp3", B=1, T_text=4, grid_h=4, grid_w=5, D=768, H=3,
                                  I=384), 3),
}


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _bf16_bytes(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.bfloat16).contiguous().view(
        torch.uint8).reshape(-1)


def _from_bf16_bytes(b: torch.Tensor, shape) -> np.ndarray:
    return b.contiguous().view(torch.bfloat16).to(torch.float64).numpy().reshape(shape)


def _qkv_heads(h, W, H, pos, cfg):
    """q, k, v [B, H, n, 256] of the rows h [B, n, D] (QK-norm and MRoPE on q, k)."""
    Dq = H * 256
    qkv = h @ W["w_qkv"].T
    q = O.split_heads(qkv[..., :Dq], H)
    k = O.split_heads(qkv[..., Dq:2 * Dq], H)
    v = O.split_heads(qkv[..., 2 * Dq:], H)
    q = O.apply_mrope(O.rms_norm(q, cfg.eps, W["g_q"]), pos, cfg.rope_theta, cfg.sections)
    k = O.apply_mrope(O.rms_norm(k, cfg.eps, W["g_k"]), pos, cfg.rope_theta, cfg.sections)
    return q, k, v


class TpStandIn:
    """One TP rank's steps in fp64 on its shard of the weights."""

    def __init__(self, cfg, rank, size, wts, temb, pos):
        from stream_diffusion_transformer_fwd_b200.parallel import tp_shard_weights

        self.cfg, self.rank = cfg, rank
        self.Hs = cfg.H // size
        self.W = block_weights_f64(tp_shard_weights(wts, rank, size, cfg.D, cfg.H, cfg.I))
        self.mod = O.adaln_modulation(temb, self.W["w_ada"], self.W["b_ada"], 6)
        self.pos = pos

    def attention(self, x, partial):
        sh, sc, g = self.mod[0], self.mod[1], self.mod[2]
        xn = x.numpy()
        h = O.modulate(xn, sh, sc, self.cfg.eps)
        q, k, v = _qkv_heads(h, self.W, self.Hs, self.pos, self.cfg)
        o = O.merge_heads(O.joint_attention(q, k, v))
        res = xn if self.rank == 0 else 0.0
        partial.copy_(torch.from_numpy(res + g[:, None, :] * (o @ self.W["w_o"].T)))

    def mlp(self, x1, partial):
        sh, sc, g = self.mod[3], self.mod[4], self.mod[5]
        x1n = x1.numpy()
        u = O.swiglu(O.modulate(x1n, sh, sc, self.cfg.eps), self.W["w_gate"], self.W["w_up"])
        res = x1n if self.rank == 0 else 0.0
        partial.copy_(torch.from_numpy(res + g[:, None, :] * (u @ self.W["w_down"].T)))

    def reduce(self, srcs, out):
        out.copy_(sum(srcs[1:], srcs[0].clone()))


class SpStandIn:
    """One Ulysses rank's steps in fp64, exchanging bf16 chunks laid out as
    include/ig4.h documents them."""

    def __init__(self, ig4, cfg, rank, size, wts, temb):
        self.cfg, self.r, self.P = cfg, rank, size
        self.c = ig4.config_from(cfg)
        self.W = block_weights_f64(wts)
        self.mod = O.adaln_modulation(temb, self.W["w_ada"], self.W["b_ada"], 6)
        self.Hg = cfg.H // size
        self.rng = [ig4.ig4_sp_image_range(self.c, size, s) for s in range(size)]
        self.pos = ig4.ig4_sp_positions(self.c, size, rank).numpy()
        self.nb = lambda ph, s, d: ig4.ig4_sp_exchange_bytes(self.c, size, ph, s, d)

    def pre(self, x_local, send):
        cfg, T, Hg, B = self.cfg, self.cfg.T_text, self.Hg, self.cfg.B
        h = O.modulate(x_local.numpy(), self.mod[0], self.mod[1], cfg.eps)
        self.q, self.k, self.v = _qkv_heads(h, self.W, cfg.H, self.pos, cfg)
        off = 0
        for d in range(self.P):
            hs = slice(d * Hg, (d + 1) * Hg)
            parts = [self.q[:, hs, T:], self.k[:, hs, T:], np.swapaxes(self.v[:, hs, T:], -1, -2)]
            chunk = torch.cat([_bf16_bytes(p) for p in parts])
            assert chunk.numel() == self.nb(0, self.r, d)
            send[off:off + chunk.numel()] = chunk
            off += chunk.numel()
        assert off == send.numel()

    def attention(self, recv, send_o):
        cfg, T, Hg, B, r = self.cfg, self.cfg.T_text, self.Hg, self.cfg.B, self.r
        hs = slice(r * Hg, (r + 1) * Hg)
        qs, ks, vs = [self.q[:, hs, :T]], [self.k[:, hs, :T]], [self.v[:, hs, :T]]
        off = 0
        for s in range(self.P):
            n = self.rng[s][1]
            part = B * Hg * n * 256 * 2
            ch = recv[off:off + self.nb(0, s, r)]
            qs.append(_from_bf16_bytes(ch[:part], (B, Hg, n, 256)))
            ks.append(_from_bf16_bytes(ch[part:2 * part], (B, Hg, n, 256)))
            vs.append(np.swapaxes(_from_bf16_bytes(ch[2 * part:], (B, Hg, 256, n)), -1, -2))
            off += self.nb(0, s, r)
        assert off == recv.numel()
        o = O.merge_heads(O.joint_attention(np.concatenate(qs, 2), np.concatenate(ks, 2),
                                            np.concatenate(vs, 2)))  # [B, L, Hg*256]
        off = 0
        for d in range(self.P):
            o_off, n = self.rng[d]
            rows = np.concatenate([o[:, :T], o[:, T + o_off:T + o_off + n]], axis=1)
            chunk = _bf16_bytes(rows)
            assert chunk.numel() == self.nb(1, r, d)
            send_o[off:off + chunk.numel()] = chunk
            off += chunk.numel()

    def post(self, x_local, y_local, recv_o):
        cfg, T, Hg, B, r = self.cfg, self.cfg.T_text, self.Hg, self.cfg.B, self.r
        Ls = T + self.rng[r][1]
        cols, off = [], 0
        for s in range(self.P):
            cols.append(_from_bf16_bytes(recv_o[off:off + self.nb(1, s, r)], (B, Ls, Hg * 256)))
            off += self.nb(1, s, r)
        o = np.concatenate(cols, axis=2)
        x = x_local.numpy()
        x1 = x + self.mod[2][:, None, :] * (o @ self.W["w_o"].T)
        u = O.swiglu(O.modulate(x1, self.mod[3], self.mod[4], cfg.eps), self.W["w_gate"],
                     self.W["w_up"])
        y_local.copy_(torch.from_numpy(x1 + self.mod[5][:, None, :] * (u @ self.W["w_down"].T)))


def _worker(rank, world, port, name, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from stream_diffusion_transformer_fwd_b200 import ig4
        from stream_diffusion_transformer_fwd_b200.parallel import (Collectives, SpPlan,
                                                                     sp_block_forward,
                                                                     sp_local_tokens,
                                                                     tp_block_forward)

        cfg, _ = CFGS[name]
        acts = make_block_activations(cfg, seed=41)
        wts = make_block_weights(cfg, seed=41, stress=True)
        x = torch.from_numpy(to_f64(acts["x"]))
        temb = to_f64(acts["temb"])
        pos = O.mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w)
        coll = Collectives()
        if name.startswith("tp"):
            ops = TpStandIn(cfg, rank, world, wts, temb, pos)
            partial, x1, y = torch.empty_like(x), torch.empty_like(x), torch.empty_like(x)
            tp_block_forward(ops, coll, x, y, partial, x1)
            outs = [torch.empty_like(y) for _ in range(world)]
            dist.all_gather(outs, y)
            y_all = y.numpy()
            same = all(torch.equal(o, outs[0]) for o in outs)
        else:
            c = ig4.config_from(cfg)
            plan = SpPlan.build(ig4, c, rank, world)
            ops = SpStandIn(ig4, cfg, rank, world, wts, temb)
            off, n = ig4.ig4_sp_image_range(c, world, rank)
            x_loc = sp_local_tokens(x, cfg.T_text, off, n)
            y_loc = torch.empty_like(x_loc)
            sp_block_forward(ops, coll, plan, x_loc, y_loc, plan.buffers("cpu"))
            shapes = [ig4.ig4_sp_image_range(c, world, s)[1] for s in range(world)]
            gathered = [torch.empty(cfg.B, cfg.T_text + n_s, cfg.D, dtype=torch.float64)
                        for n_s in shapes]
            for s in range(world):  # every rank's local result to every rank
                buf = y_loc.clone() if s == rank else gathered[s]
                dist.broadcast(buf, src=s)
                gathered[s] = buf
            T = cfg.T_text
            same = all(torch.equal(g[:, :T], gathered[0][:, :T]) for g in gathered)
            y_all = torch.cat([gathered[0][:, :T]] + [g[:, T:] for g in gathered], 1).numpy()
        if rank == 0:
            ref = O.block_forward(x.numpy(), temb, pos, block_weights_f64(wts), cfg.H,
                                  cfg.rope_theta, cfg.sections, cfg.eps)
            q.put((same, float(np.linalg.norm(y_all - ref) / np.linalg.norm(ref)),
                   float(np.linalg.norm((y_all - x.numpy()) - (ref - x.numpy())) /
                         np.linalg.norm(ref - x.numpy()))))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", list(CFGS))
def test_parallel_layouts_over_gloo(name):
    _, world = CFGS[name]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0] * world, codes
    same, e_y, e_d = q.get(timeout=10)
    print(f"{name}: ranks agree={same} relL2(y)={e_y:.3e} relL2(delta)={e_d:.3e}")
    assert same
    if name.startswith("tp"):
        assert e_y <= 1e-12 and e_d <= 1e-10
    else:
        # q, k, v and o cross the exchange as bf16 (relative rounding 2^-9)
        assert e_y <= 1e-2 and e_d <= 2e-2
