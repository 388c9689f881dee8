"""Sampler step on the GPU through the C ABI against the fp64 oracle.

The guided Euler kernel element by element; one full step with asymmetric CFG
(a conditional stack over [text | image] and a separate image-only
unconditional stack) in full at reduced width, in bf16 and with E4M3
weights, and at the full width with two blocks per branch; and the full-size
step (34 + 34 live blocks, 1024 px, FP8) as the exact composition of two
stacks whose blocks are checked against the oracle one by one."""

import numpy as np
import pytest
import torch

import oracle as O
from oracle import ig4_sampler as S
from oracle.inputs import block_weights_f64, to_f64, weight_f64
from synth import CONFIGS, make_block_weights, make_stack_inputs
from tests._util import rel_l2
from tests.gpu_common import (check_tapped_stack, lib, live_blocks, run_stack_tapped,
                              tap_ids_for, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ig4(cuda_device):
    return lib()


def _bf16(t):
    return t.to(torch.bfloat16)


@pytest.mark.parametrize("n", [8, 4096, 1 << 20])
def test_cfg_euler(ig4, n):
    g = torch.Generator().manual_seed(n)
    vc = _bf16(torch.randn(n, generator=g))
    vu = _bf16(torch.randn(n, generator=g))
    z = torch.randn(n, generator=g)
    gw, dt = 7.0, 0.0371
    ref = S.euler_update(to_f64(z), S.cfg_velocity(to_f64(vc), to_f64(vu), gw), dt, 0.0)
    zd = z.cuda()
    z16 = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    ig4.ig4_cfg_euler(vc.cuda(), vu.cuda(), gw, dt, zd, zd, z16)  # in place
    torch.cuda.synchronize()
    got = to_f64(zd.cpu())
    # fp32 arithmetic on exact bf16 velocities: a few fp32 roundings
    assert np.max(np.abs(got - ref) / (np.abs(ref) + 1.0)) <= 4e-7
    assert torch.equal(z16.cpu(), zd.cpu().to(torch.bfloat16))
    # conversion only
    z16b = torch.empty_like(z16)
    ig4.ig4_cfg_euler(None, None, 0.0, 0.0, z.cuda(), None, z16b)
    torch.cuda.synchronize()
    assert torch.equal(z16b.cpu(), z.to(torch.bfloat16))


def _stack_dict(cfg, st, seed, n_blocks, zero_gates=False):
    def blocks(i):
        return block_weights_f64(make_block_weights(cfg, seed=seed, block=0 if zero_gates else i,
                                                    stress=True, zero_adaln=zero_gates))

    return {"block_weights": blocks, "n_blocks": 0 if zero_gates else n_blocks,
            "w_in": weight_f64(st["w_in"], st["s_in"]), "b_in": to_f64(st["b_in"]),
            "w_f": weight_f64(st["w_f"], st["s_f"]), "b_f": to_f64(st["b_f"]),
            "w_out": weight_f64(st["w_out"], st["s_out"]), "b_out": to_f64(st["b_out"])}


def _stack_weights(ig4, cfg, st, blocks):
    sd = to_dev(st)
    bws = [ig4.block_weights(b) for b in blocks]
    sw = ig4.stack_weights(bws, sd["w_in"], sd["s_in"], sd["b_in"], sd["w_f"], sd["s_f"],
                           sd["b_f"], sd["w_out"], sd["s_out"], sd["b_out"], cfg.latent_ch)
    return sw, sd


def _run_step(ig4, cfg, st_c, st_u, blocks_c, blocks_u, z, t_cur, t_next, gw):
    c = ig4.config_from(cfg)
    sw_c, sd_c = _stack_weights(ig4, cfg, st_c, blocks_c)
    sw_u, sd_u = _stack_weights(ig4, cfg, st_u, blocks_u)
    pos_c = ig4.ig4_mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w, device="cuda")
    pos_u = ig4.ig4_mrope_positions(0, cfg.grid_t, cfg.grid_h, cfg.grid_w, device="cuda")
    ws = torch.empty(ig4.ig4_denoise_workspace_size(c, cfg.latent_ch), dtype=torch.uint8,
                     device="cuda")
    zd = z.cuda()
    ig4.ig4_denoise_step(c, sw_c, sw_u, zd, sd_c["text"], pos_c, pos_u, sd_c["temb"],
                         sd_u["temb"], t_cur, t_next, gw, ws)
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    return to_f64(zd.cpu())


@pytest.mark.parametrize("wdt", ["bf16", "e4m3"])
def test_denoise_step_small_full(ig4, wdt):
    cfg = CONFIGS["tiny"].with_(name="step_small", B=2, T_text=8, grid_h=4, grid_w=6, D=512, H=2,
                                I=256, x_dtype="bf16", w_dtype=wdt, n_blocks=2)
    st_c = make_stack_inputs(cfg, seed=4, stress=True)
    st_u = make_stack_inputs(cfg, seed=5, stress=True)
    blocks_c = [to_dev(make_block_weights(cfg, seed=4, block=i, stress=True)) for i in range(2)]
    blocks_u = [to_dev(make_block_weights(cfg, seed=5, block=i, stress=True)) for i in range(2)]
    t = S.flow_schedule(20, 0.0, 1.75, 256, 384)
    gw = float(S.guidance_schedule(20, 2)[5])
    z = torch.randn(cfg.B, cfg.n_img, cfg.latent_ch, generator=torch.Generator().manual_seed(3))
    got = _run_step(ig4, cfg, st_c, st_u, blocks_c, blocks_u, z, float(t[5]), float(t[6]), gw)
    ref = S.denoise_step(to_f64(z), to_f64(st_c["text"]), to_f64(st_c["temb"]),
                         to_f64(st_u["temb"]), float(t[5]), float(t[6]), gw,
                         (cfg.grid_t, cfg.grid_h, cfg.grid_w), _stack_dict(cfg, st_c, 4, 2),
                         _stack_dict(cfg, st_u, 5, 2), cfg.H, theta=cfg.rope_theta,
                         sections=cfg.sections, eps=cfg.eps)
    z0 = to_f64(z)
    e = rel_l2(got - z0, ref - z0)
    print(f"denoise step {wdt}: relL2(dz)={e:.3e}")
    # two stacks of two blocks each and their head; the guided difference keeps
    # the per-stack relative error
    assert e <= (3e-2 if wdt == "e4m3" else 1e-2)


@pytest.mark.parametrize("wdt", ["e4m3"])
def test_denoise_step_full_width_two_blocks(ig4, wdt):
    """One sampler step at the full width (D 4608, 18 heads, I 12288) with two
    live blocks per branch, B = 2, 128 text + 32 x 32 image tokens (the
    unconditional stack sees the 1024 image tokens alone), against the
    oracle's whole denoise_step on the same seeded inputs."""
    cfg = CONFIGS["step_1024px_fp8"].with_(name="step_fw2", B=2, T_text=128, grid_h=32,
                                           grid_w=32, w_dtype=wdt, n_blocks=2)
    st_c = make_stack_inputs(cfg, seed=14, stress=True)
    st_u = make_stack_inputs(cfg, seed=15, stress=True)
    host_c = [make_block_weights(cfg, seed=14, block=i, stress=True) for i in range(2)]
    host_u = [make_block_weights(cfg, seed=15, block=i, stress=True) for i in range(2)]
    t = S.flow_schedule(20, 0.0, 1.75, 512, 512)
    gw = float(S.guidance_schedule(20, 2)[3])
    z = torch.randn(cfg.B, cfg.n_img, cfg.latent_ch, generator=torch.Generator().manual_seed(6))
    got = _run_step(ig4, cfg, st_c, st_u, [to_dev(w) for w in host_c],
                    [to_dev(w) for w in host_u], z, float(t[3]), float(t[4]), gw)
    Wc = [block_weights_f64(w) for w in host_c]
    Wu = [block_weights_f64(w) for w in host_u]
    dc = _stack_dict(cfg, st_c, 14, 2)
    du = _stack_dict(cfg, st_u, 15, 2)
    dc["block_weights"] = lambda i: Wc[i]
    du["block_weights"] = lambda i: Wu[i]
    ref = S.denoise_step(to_f64(z), to_f64(st_c["text"]), to_f64(st_c["temb"]),
                         to_f64(st_u["temb"]), float(t[3]), float(t[4]), gw,
                         (cfg.grid_t, cfg.grid_h, cfg.grid_w), dc, du, cfg.H,
                         theta=cfg.rope_theta, sections=cfg.sections, eps=cfg.eps)
    z0 = to_f64(z)
    e = rel_l2(got - z0, ref - z0)
    print(f"denoise step full width, 2 + 2 blocks, {wdt}: relL2(dz)={e:.3e}")
    assert e <= (3e-2 if wdt == "e4m3" else 1e-2)


def test_denoise_step_full_size_live_blocks(ig4):
    """The full-size step (1024 px, FP8, two 34-block stacks with live
    weights).  The step's result must equal, bit for bit, the guided Euler
    update of the two stacks run on their own through the tapped stack entry
    point on the bf16-rounded latent; those two stack runs are checked against
    the oracle block by block (tests.gpu_common.check_tapped_stack: stack
    input, blocks 0 and 33 of each branch on sampled rows, final layer)."""
    cfg = CONFIGS["step_1024px_fp8"]
    cfg_u = cfg.with_(name="step_1024px_fp8_uncond", T_text=0)
    checked = (0, 33)
    st_c = make_stack_inputs(cfg, seed=16, stress=True)
    st_u = make_stack_inputs(cfg_u, seed=17, stress=True)
    host_c = {i: make_block_weights(cfg, seed=16, block=i, stress=True) for i in checked}
    host_u = {i: make_block_weights(cfg_u, seed=17, block=i, stress=True) for i in checked}
    blocks_c = live_blocks(cfg, host_c, seed=16)
    blocks_u = live_blocks(cfg_u, host_u, seed=17)
    t = S.flow_schedule(48, 0.0, 1.5, 1024, 1024)
    t_cur, t_next, gw = float(t[3]), float(t[4]), 7.0
    z = torch.randn(cfg.B, cfg.n_img, cfg.latent_ch, generator=torch.Generator().manual_seed(5))
    z_step = _run_step(ig4, cfg, st_c, st_u, blocks_c, blocks_u, z, t_cur, t_next, gw)

    z16 = z.to(torch.bfloat16)
    v_c, seq_c = run_stack_tapped(ig4, cfg, st_c, blocks_c, tap_ids_for(cfg, host_c), z16)
    v_u, seq_u = run_stack_tapped(ig4, cfg_u, st_u, blocks_u, tap_ids_for(cfg_u, host_u), z16)
    del blocks_c, blocks_u
    zd = z.cuda()
    z_comp = torch.empty_like(zd)
    # the step takes t_cur and t_next as fp32 and subtracts them in fp32
    dt = float(np.float32(t_cur) - np.float32(t_next))
    ig4.ig4_cfg_euler(v_c, v_u, gw, dt, zd, z_comp, None)
    torch.cuda.synchronize()
    assert np.array_equal(to_f64(z_comp.cpu()), z_step)

    z64 = to_f64(z16)
    check_tapped_stack(cfg, st_c, host_c, seq_c, v_c, z64)
    check_tapped_stack(cfg_u, st_u, host_u, seq_u, v_u, z64)


def test_denoise_step_argument_errors(ig4):
    cfg = CONFIGS["tiny"].with_(name="step_small", B=1, T_text=8, grid_h=4, grid_w=4, D=512, H=2,
                                I=256, x_dtype="bf16", w_dtype="bf16", n_blocks=1)
    st = make_stack_inputs(cfg, seed=1)
    blocks = [to_dev(make_block_weights(cfg, seed=1, block=0))]
    sw, sd = _stack_weights(ig4, cfg, st, blocks)
    c = ig4.config_from(cfg)
    pos = ig4.ig4_mrope_positions(cfg.T_text, 1, 4, 4, device="cuda")
    z = torch.zeros(1, 16, 128, device="cuda")
    need = ig4.ig4_denoise_workspace_size(c, 128)
    assert need > ig4.ig4_stack_workspace_size(c, 128)
    with pytest.raises(ig4.Ig4Error) as e:
        ig4.ig4_denoise_step(c, sw, sw, z, sd["text"], pos, pos, sd["temb"], sd["temb"], 0.5,
                             0.4, 7.0, torch.empty(need - 256, dtype=torch.uint8, device="cuda"))
    assert e.value.status == ig4.IG4_ERR_WORKSPACE
    with pytest.raises(ig4.Ig4Error) as e:
        ig4.ig4_denoise_step(c, sw, sw, z, sd["text"], pos, pos, sd["temb"], sd["temb"],
                             float("nan"), 0.4, 7.0,
                             torch.empty(need, dtype=torch.uint8, device="cuda"))
    assert e.value.status == ig4.IG4_ERR_INVALID_ARG
