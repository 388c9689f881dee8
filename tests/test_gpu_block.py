"""Whole-block and stack parity through the C-ABI against the fp64 oracle.

Small problems are compared element by element in full; full-width workloads
(in the launch configuration the benchmark times) are compared on sampled
token rows, which the oracle evaluates one by one.  Tolerances: rel-L2 <= 1e-2
and max-abs <= 5e-2 RMS on y for bf16 weights, rel-L2 <= 3e-2 for FP8
weights; delta = y - x is checked too (see gpu_common.delta_tolerance)."""

import numpy as np
import pytest
import torch

import oracle as O
from oracle.inputs import block_weights_f64, to_f64, weight_f64
from synth import CONFIGS, make_block_activations, make_block_weights, make_stack_inputs
from tests._util import max_abs_over_rms, rel_l2
from tests.gpu_common import (check_output, check_tapped_stack, lib, live_blocks, run_block,
                              run_stack_tapped, sample_rows, tap_ids_for, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ig4(cuda_device):
    return lib()


def _oracle_full(cfg, acts, wts):
    pos = O.mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w)
    return O.block_forward(to_f64(acts["x"]), to_f64(acts["temb"]), pos,
                           block_weights_f64(wts), cfg.H, cfg.rope_theta, cfg.sections, cfg.eps)


def _gpu(ig4, cfg, acts, wts):
    x = acts["x"].cuda()
    y = run_block(ig4, cfg, to_dev(wts), x, acts["temb"].cuda())
    return y.float().cpu().double().numpy()


# ------------------------------------------------------------- small, in full

SMALL = {
    "tiny": CONFIGS["tiny"],
    "tiny_fp8": CONFIGS["tiny"].with_(name="tiny_fp8", w_dtype="e4m3"),
    "tiny_bf16x": CONFIGS["tiny"].with_(name="tiny_bf16x", x_dtype="bf16"),
    # batch 2 with a ragged length: tiles straddle the sample boundary
    "ragged_b2": CONFIGS["tiny"].with_(name="ragged_b2", B=2, T_text=5, grid_h=7, grid_w=9, D=512,
                                       H=2, I=384),
    "ragged_b2_fp8": CONFIGS["tiny"].with_(name="ragged_b2_fp8", B=2, T_text=5, grid_h=7,
                                           grid_w=9, D=512, H=2, I=384, w_dtype="e4m3"),
    # text only / image only / a single token
    "text_only": CONFIGS["tiny"].with_(name="text_only", T_text=70, grid_h=0, grid_w=0, D=512,
                                       H=2, I=256),
    "image_only": CONFIGS["tiny"].with_(name="image_only", T_text=0, grid_h=5, grid_w=13, D=512,
                                        H=2, I=256),
    "one_token": CONFIGS["tiny"].with_(name="one_token", T_text=1, grid_h=0, grid_w=0, D=512, H=2,
                                       I=256),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_block_small_full(ig4, name):
    cfg = SMALL[name]
    acts = make_block_activations(cfg, seed=11)
    wts = make_block_weights(cfg, seed=11, stress=True)
    y = _gpu(ig4, cfg, acts, wts)
    y_ref = _oracle_full(cfg, acts, wts)
    x = to_f64(acts["x"])
    check_output(y.reshape(y_ref.shape), y_ref, x, cfg.w_dtype == "e4m3",
                 cfg.x_dtype == "bf16", name)


def test_block_512px_full(ig4):
    cfg = CONFIGS["512px"]
    acts = make_block_activations(cfg, seed=1)
    wts = make_block_weights(cfg, seed=1, stress=True)
    y = _gpu(ig4, cfg, acts, wts)
    y_ref = _oracle_full(cfg, acts, wts)
    check_output(y.reshape(y_ref.shape), y_ref, to_f64(acts["x"]), False, True, "512px")


# ------------------------------------------------ full size, sampled rows

@pytest.mark.parametrize("name", ["1024px", "1024px_fp8", "2048x352", "2048px"])
def test_block_full_size_sampled_rows(ig4, name):
    cfg = CONFIGS[name]
    acts = make_block_activations(cfg, seed=0)
    wts = make_block_weights(cfg, seed=0)
    y = _gpu(ig4, cfg, acts, wts).reshape(cfg.M, cfg.D)
    rows = sample_rows(cfg, n=24 if name == "2048px" else 48)
    pos = O.mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w)
    x = to_f64(acts["x"])
    y_ref = O.block_forward_rows(x, to_f64(acts["temb"]), pos, block_weights_f64(wts), cfg.H,
                                 rows, cfg.rope_theta, cfg.sections, cfg.eps)
    check_output(y[rows], y_ref, x.reshape(cfg.M, cfg.D)[rows], cfg.w_dtype == "e4m3", True,
                 name)


# ----------------------------------------------------------- exact properties

@pytest.mark.parametrize("name", ["tiny", "1024px"])
def test_zero_adaln_is_bit_exact_identity(ig4, name):
    cfg = CONFIGS[name]
    acts = make_block_activations(cfg, seed=5)
    wts = make_block_weights(cfg, seed=5, zero_adaln=True)
    x = acts["x"].cuda()
    y = run_block(ig4, cfg, to_dev(wts), x, acts["temb"].cuda())
    assert torch.equal(y, x)


def test_block_deterministic(ig4):
    cfg = SMALL["ragged_b2"]
    acts = make_block_activations(cfg, seed=2)
    wd = to_dev(make_block_weights(cfg, seed=2, stress=True))
    x = acts["x"].cuda()
    y1 = run_block(ig4, cfg, wd, x, acts["temb"].cuda())
    y2 = run_block(ig4, cfg, wd, x, acts["temb"].cuda())
    assert torch.equal(y1, y2)


def test_traced_events_cover_the_block(ig4):
    cfg = CONFIGS["tiny"]
    acts = make_block_activations(cfg, seed=3)
    wd = to_dev(make_block_weights(cfg, seed=3))
    c = ig4.config_from(cfg)
    x = acts["x"].cuda()
    y = torch.empty_like(x)
    pos = ig4.ig4_mrope_positions(cfg.T_text, 1, cfg.grid_h, cfg.grid_w, device="cuda")
    ws = torch.empty(ig4.ig4_workspace_size(c), dtype=torch.uint8, device="cuda")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(ig4.IG4_BLOCK_TRACE_EVENTS)]
    ig4.ig4_block_forward(c, ig4.block_weights(wd), x, y, pos, acts["temb"].cuda(), ws,
                          events=ev)
    torch.cuda.synchronize()
    times = [ev[i].elapsed_time(ev[i + 1]) for i in range(9)]
    assert all(t >= 0 for t in times)
    y2 = run_block(ig4, cfg, wd, x, acts["temb"].cuda())
    assert torch.equal(y, y2)


# --------------------------------------------------------------------- stack

def _stack_oracle(cfg, st, n_blocks, seed, same_block=False):
    pos = O.mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w)

    def blocks(i):
        return block_weights_f64(make_block_weights(cfg, seed=seed, block=0 if same_block else i,
                                                    stress=True))

    return O.stack_forward(to_f64(st["x_latent"]), to_f64(st["text"]), to_f64(st["temb"]), pos,
                           blocks, n_blocks, weight_f64(st["w_in"], st["s_in"]),
                           to_f64(st["b_in"]), weight_f64(st["w_f"], st["s_f"]),
                           to_f64(st["b_f"]), weight_f64(st["w_out"], st["s_out"]),
                           to_f64(st["b_out"]), cfg.H, cfg.rope_theta, cfg.sections, cfg.eps)


def _stack_gpu(ig4, cfg, st, block_dicts):
    c = ig4.config_from(cfg)
    bws = [ig4.block_weights(b) for b in block_dicts]
    sd = to_dev(st)
    sw = ig4.stack_weights(bws, sd["w_in"], sd["s_in"], sd["b_in"], sd["w_f"], sd["s_f"],
                           sd["b_f"], sd["w_out"], sd["s_out"], sd["b_out"], cfg.latent_ch)
    pos = ig4.ig4_mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w, device="cuda")
    ws = torch.empty(ig4.ig4_stack_workspace_size(c, cfg.latent_ch), dtype=torch.uint8,
                     device="cuda")
    out = torch.empty_like(sd["x_latent"])
    ig4.ig4_stack_forward(c, sw, sd["x_latent"], sd["text"], out, pos, sd["temb"], ws)
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    return out.float().cpu().double().numpy()


@pytest.mark.parametrize("wdt", ["bf16", "e4m3"])
def test_stack_small_full(ig4, wdt):
    cfg = CONFIGS["tiny"].with_(name="stack_small", B=2, T_text=8, grid_h=4, grid_w=6, D=512,
                                H=2, I=256, x_dtype="bf16", w_dtype=wdt, n_blocks=3)
    st = make_stack_inputs(cfg, seed=4, stress=True)
    blocks = [to_dev(make_block_weights(cfg, seed=4, block=i, stress=True)) for i in range(3)]
    got = _stack_gpu(ig4, cfg, st, blocks)
    ref = _stack_oracle(cfg, st, 3, seed=4)
    tol = 3e-2 if wdt == "e4m3" else 1e-2
    e = rel_l2(got, ref)
    print(f"stack {wdt}: relL2={e:.3e}")
    assert e <= tol


@pytest.mark.parametrize("wdt", ["e4m3", "bf16"])
def test_stack_full_width_two_blocks(ig4, wdt):
    """The stack at the full width and batch of the one-step workload (D 4608,
    18 heads, I 12288, B = 2) with two live blocks over 128 text + 32 x 32
    image tokens, against the oracle's whole stack_forward on the same seeded
    inputs (every output element)."""
    cfg = CONFIGS["stack_1024px_fp8"].with_(name="stack_fw2", T_text=128, grid_h=32, grid_w=32,
                                            w_dtype=wdt, n_blocks=2)
    st = make_stack_inputs(cfg, seed=13, stress=True)
    host = [make_block_weights(cfg, seed=13, block=i, stress=True) for i in range(2)]
    got = _stack_gpu(ig4, cfg, st, [to_dev(w) for w in host])
    Ws = [block_weights_f64(w) for w in host]
    pos = O.mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w)
    ref = O.stack_forward(to_f64(st["x_latent"]), to_f64(st["text"]), to_f64(st["temb"]), pos,
                          lambda i: Ws[i], 2, weight_f64(st["w_in"], st["s_in"]),
                          to_f64(st["b_in"]), weight_f64(st["w_f"], st["s_f"]),
                          to_f64(st["b_f"]), weight_f64(st["w_out"], st["s_out"]),
                          to_f64(st["b_out"]), cfg.H, cfg.rope_theta, cfg.sections, cfg.eps)
    tol = 3e-2 if wdt == "e4m3" else 1e-2
    e = rel_l2(got, ref)
    m = max_abs_over_rms(got, ref)
    print(f"stack full width, 2 blocks, {wdt}: relL2={e:.3e} maxabs/rms={m:.3e}")
    assert e <= tol
    if wdt == "bf16":
        assert m <= 5e-2


def test_stack_full_size_live_blocks(ig4):
    """The one-step workload in full: 34 live blocks with FP8 weights, batch 2,
    512 text + 64 x 64 image tokens.  The stack is run once with taps on the
    sequence entering blocks 0, 1, 16, 17, 33 and after block 33, and checked
    against the oracle (tests.gpu_common.check_tapped_stack): the sequence
    entering block 0 against the oracle's stack_input of the seeded latents
    and text; blocks 0, 16 and 33 on 48 sampled token rows of both samples;
    the final layer on every output element.  Blocks 0, 16 and 33 carry
    host-drawn seeded weights (stress biases and QK-norm weights); the other
    31 are drawn on the device with the same shapes and distributions (their
    values never reach the oracle)."""
    cfg = CONFIGS["stack_1024px_fp8"]
    checked = (0, 16, 33)
    st = make_stack_inputs(cfg, seed=12, stress=True)
    host = {i: make_block_weights(cfg, seed=12, block=i, stress=True) for i in checked}
    blocks = live_blocks(cfg, host, seed=12)
    out, seq = run_stack_tapped(ig4, cfg, st, blocks, tap_ids_for(cfg, host), st["x_latent"])
    del blocks
    check_tapped_stack(cfg, st, host, seq, out, to_f64(st["x_latent"]))


# --------------------------------------------------------- failure detection

def test_timeout_selftest_reports_and_context_survives(ig4):
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    ig4.ig4_selftest_timeout(20000)  # 20 ms wait on a barrier nothing completes
    assert ig4.ig4_last_device_error() == ig4.IG4_ERR_TIMEOUT
    assert ig4.ig4_last_device_error() == ig4.IG4_OK  # the word was cleared
    cfg = SMALL["one_token"]
    acts = make_block_activations(cfg, seed=1)
    wts = make_block_weights(cfg, seed=1)
    y = _gpu(ig4, cfg, acts, wts)
    y_ref = _oracle_full(cfg, acts, wts)
    assert rel_l2(y.reshape(y_ref.shape), y_ref) <= 1e-2


def test_sm_clock_probe_reads_a_plausible_clock(ig4):
    """The clock probe's cycles / global-timer ratio lies between idle and
    boost clocks of the part (a wrong unit would be off by 10^3)."""
    mhz = [ig4.ig4_sm_clock_mhz(50) for _ in range(3)]
    assert all(100.0 < m < 3500.0 for m in mhz), mhz


def test_invalid_arguments_launch_nothing(ig4):
    cfg = CONFIGS["tiny"]
    c = ig4.config_from(cfg)
    acts = make_block_activations(cfg)
    wd = to_dev(make_block_weights(cfg))
    x = acts["x"].cuda()
    pos = ig4.ig4_mrope_positions(cfg.T_text, 1, 8, 8, device="cuda")
    small = torch.empty(ig4.ig4_workspace_size(c) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(ig4.Ig4Error) as e:
        ig4.ig4_block_forward(c, ig4.block_weights(wd), x, torch.empty_like(x), pos,
                              acts["temb"].cuda(), small)
    assert e.value.status == ig4.IG4_ERR_WORKSPACE
    with pytest.raises(ig4.Ig4Error) as e:
        ig4.ig4_block_forward(c, ig4.block_weights(wd), x, x, pos, acts["temb"].cuda(),
                              torch.empty(ig4.ig4_workspace_size(c), dtype=torch.uint8,
                                          device="cuda"))
    assert e.value.status == ig4.IG4_ERR_INVALID_ARG


def test_stack_small_nvfp4_mixed(ig4):
    """The stack with NVFP4 Mixed weights (3 blocks, B = 2, 160 tokens).  Every
    block's attention gate is zero and the oracle stores the stream in bf16
    as the GPU does, so each block's FFN sees the same h2 on both sides and
    the NVFP4 decisions agree (see the NVFP4 block tests); the stack then
    checks the assembly, the ping-pong launches and the head."""
    cfg = CONFIGS["tiny"].with_(name="stack_nvfp4", B=2, T_text=16, grid_h=8, grid_w=8, D=512,
                                H=2, I=256, x_dtype="bf16", w_dtype="nvfp4_mixed", n_blocks=3)
    D = cfg.D
    st = make_stack_inputs(cfg, seed=6, stress=True)
    wts = []
    for i in range(3):
        w = make_block_weights(cfg, seed=6, block=i, stress=True)
        w["w_ada"].view(torch.uint8)[2 * D:3 * D] = 0
        w["b_ada"][2 * D:3 * D] = 0.0
        wts.append(w)
    got = _stack_gpu(ig4, cfg, st, [ig4.nvfp4_pack_block_scales(to_dev(w)) for w in wts])
    pos = O.mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w)
    Ws = [block_weights_f64(w) for w in wts]
    # the library runs the stack's in- and out-projections in bf16 with their
    # E4M3 weights decoded to bf16; the in-projection's output then feeds the
    # first block's NVFP4 decisions, so the oracle takes the same bf16 weights
    ref = O.stack_forward(to_f64(st["x_latent"]), to_f64(st["text"]), to_f64(st["temb"]), pos,
                          lambda i: Ws[i], 3, O.bf16_round(weight_f64(st["w_in"], st["s_in"])),
                          to_f64(st["b_in"]), weight_f64(st["w_f"], st["s_f"]),
                          to_f64(st["b_f"]), O.bf16_round(weight_f64(st["w_out"], st["s_out"])),
                          to_f64(st["b_out"]), cfg.H, cfg.rope_theta, cfg.sections, cfg.eps,
                          ffn_nvfp4=True, stream_bf16=True)
    e = rel_l2(got, ref)
    print(f"stack nvfp4-mixed, zero attention gates: relL2={e:.3e}")
    assert e <= 2e-2
