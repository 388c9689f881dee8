"""Tensor-parallel (heads) and Ulysses sequence-parallel (image tokens)
layouts of the block ("SGLang cookbook: Ideogram 4", section 3), on one GPU.

Every rank's share runs through the C ABI on the one device, one rank after
the other, and the exchange between the ranks is done by the test: the TP
all-reduce by ig4_tp_reduce over all ranks' partial buffers (the kernel a
peer-mapped all-reduce would run), the Ulysses all-to-all by cutting each
rank's send buffer into the chunks the library's exchange sizes give.  No
kernel waits for another rank.  The assembled output is compared with the
oracle's plain (unsharded) block: in full on small shapes, on sampled rows at
1024 px."""

import numpy as np
import pytest
import torch

import oracle as O
from oracle.inputs import block_weights_f64, to_f64
from stream_diffusion_transformer_fwd_b200.parallel import sp_local_tokens, tp_shard_weights
from synth import CONFIGS, make_block_activations, make_block_weights
from tests.gpu_common import check_output, lib, run_block, sample_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ig4(cuda_device):
    return lib()


def _oracle(cfg, acts, wts, rows=None):
    pos = O.mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w)
    x = to_f64(acts["x"])
    if rows is None:
        return O.block_forward(x, to_f64(acts["temb"]), pos, block_weights_f64(wts), cfg.H,
                               cfg.rope_theta, cfg.sections, cfg.eps)
    return O.block_forward_rows(x, to_f64(acts["temb"]), pos, block_weights_f64(wts), cfg.H, rows,
                                cfg.rope_theta, cfg.sections, cfg.eps)


# ------------------------------------------------------------------- TP

def _tp_run(ig4, cfg, wts, acts, P):
    c = ig4.config_from(cfg)
    x = acts["x"].cuda()
    temb = acts["temb"].cuda()
    pos = ig4.ig4_mrope_positions(cfg.T_text, cfg.grid_t, cfg.grid_h, cfg.grid_w, device="cuda")
    shards = [to_dev(tp_shard_weights(wts, r, P, cfg.D, cfg.H, cfg.I)) for r in range(P)]
    bws = [ig4.block_weights(s) for s in shards]
    wss = [torch.empty(ig4.ig4_tp_workspace_size(c, P), dtype=torch.uint8, device="cuda")
           for _ in range(P)]
    parts = [torch.empty(cfg.M, cfg.D, dtype=torch.float32, device="cuda") for _ in range(P)]
    x1 = torch.empty_like(x)
    y = torch.empty_like(x)
    for r in range(P):
        ig4.ig4_block_tp_attention(c, r, P, bws[r], x, pos, temb, parts[r], wss[r])
    ig4.ig4_tp_reduce(parts, x1)
    for r in range(P):
        ig4.ig4_block_tp_mlp(c, r, P, bws[r], x1, parts[r], wss[r])
    ig4.ig4_tp_reduce(parts, y)
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    return y


TP_SMALL = {
    "tp2_tiny": (CONFIGS["tiny"], 2),
    "tp2_tiny_fp8": (CONFIGS["tiny"].with_(name="tp2_tiny_fp8", w_dtype="e4m3"), 2),
    "tp2_ragged_b2": (CONFIGS["tiny"].with_(name="tp2_ragged_b2", B=2, T_text=5, grid_h=7,
                                            grid_w=9, D=1024, H=4, I=1024, x_dtype="bf16"), 2),
    "tp3_d768": (CONFIGS["tiny"].with_(name="tp3_d768", T_text=20, grid_h=6, grid_w=10, D=768,
                                       H=3, I=1152), 3),
    "tp4_tiny_fp8": (CONFIGS["tiny"].with_(name="tp4_tiny_fp8", I=2048, w_dtype="e4m3",
                                           x_dtype="bf16"), 4),
}


@pytest.mark.parametrize("name", list(TP_SMALL))
def test_tp_block_small_full(ig4, name):
    cfg, P = TP_SMALL[name]
    acts = make_block_activations(cfg, seed=31)
    wts = make_block_weights(cfg, seed=31, stress=True)
    y = _tp_run(ig4, cfg, wts, acts, P).double().cpu().numpy()
    y_ref = _oracle(cfg, acts, wts)
    check_output(y.reshape(y_ref.shape), y_ref, to_f64(acts["x"]), cfg.w_dtype == "e4m3",
                 cfg.x_dtype == "bf16", name)


@pytest.mark.parametrize("name", ["1024px", "1024px_fp8"])
def test_tp2_block_1024px_sampled_rows(ig4, name):
    cfg = CONFIGS[name]
    acts = make_block_activations(cfg, seed=32)
    wts = make_block_weights(cfg, seed=32)
    y = _tp_run(ig4, cfg, wts, acts, 2).float().cpu().double().numpy().reshape(cfg.M, cfg.D)
    rows = sample_rows(cfg, n=48)
    y_ref = _oracle(cfg, acts, wts, rows)
    x = to_f64(acts["x"]).reshape(cfg.M, cfg.D)
    check_output(y[rows], y_ref, x[rows], cfg.w_dtype == "e4m3", True, f"tp2 {name}")


def test_tp1_equals_the_block(ig4):
    """One shard holding every head: the TP path's arithmetic is the block's
    except that x1 and y pass through an fp32 partial before rounding, so
    the two agree to one rounding of the stream."""
    cfg = CONFIGS["tiny"].with_(name="tp1", x_dtype="bf16")
    acts = make_block_activations(cfg, seed=33)
    wts = make_block_weights(cfg, seed=33, stress=True)
    y_tp = _tp_run(ig4, cfg, wts, acts, 1).double().cpu().numpy()
    y = run_block(ig4, cfg, to_dev(wts), acts["x"].cuda(), acts["temb"].cuda())
    y = y.double().cpu().numpy()
    assert np.max(np.abs(y_tp - y) / (np.abs(y) + 1e-3)) <= 2.0 ** -7


def test_tp_reduce_sums_in_order(ig4):
    g = torch.Generator().manual_seed(1)
    srcs = [torch.randn(4096 + 8, generator=g).cuda() for _ in range(3)]
    out32 = torch.empty_like(srcs[0])
    out16 = torch.empty(srcs[0].shape, dtype=torch.bfloat16, device="cuda")
    ig4.ig4_tp_reduce(srcs, out32)
    ig4.ig4_tp_reduce(srcs, out16)
    torch.cuda.synchronize()
    ref = (srcs[0] + srcs[1]) + srcs[2]
    assert torch.equal(out32, ref)
    assert torch.equal(out16, ref.to(torch.bfloat16))


# ------------------------------------------------------------------- SP

def _all_to_all(ig4, c, P, sends, phase):
    """recv[d] = concat over s of the chunk (s -> d) of sends[s]."""
    recvs = []
    for d in range(P):
        parts = []
        for s in range(P):
            off = sum(ig4.ig4_sp_exchange_bytes(c, P, phase, s, k) for k in range(d))
            n = ig4.ig4_sp_exchange_bytes(c, P, phase, s, d)
            parts.append(sends[s][off:off + n])
        recvs.append(torch.cat(parts).contiguous())
    return recvs


def _sp_run(ig4, cfg, wts, acts, P):
    return _sp_run_dev(ig4, cfg, to_dev(wts), acts, P)


SP_SMALL = {
    # 63 image tokens over 2 ranks: shares of 32 and 31
    "sp2_ragged_b2": (CONFIGS["tiny"].with_(name="sp2_ragged_b2", B=2, T_text=5, grid_h=7,
                                            grid_w=9, D=512, H=2, I=384, x_dtype="bf16"), 2),
    "sp2_ragged_b2_fp8": (CONFIGS["tiny"].with_(name="sp2_ragged_b2_fp8", B=2, T_text=5,
                                                grid_h=7, grid_w=9, D=512, H=2, I=384,
                                                x_dtype="bf16", w_dtype="e4m3"), 2),
    "sp2_tiny": (CONFIGS["tiny"], 2),
    "sp2_image_only": (CONFIGS["tiny"].with_(name="sp2_image_only", T_text=0, grid_h=5,
                                             grid_w=13, D=512, H=2, I=256), 2),
    "sp3_d768": (CONFIGS["tiny"].with_(name="sp3_d768", T_text=20, grid_h=6, grid_w=11, D=768,
                                       H=3, I=1152), 3),
    "sp4_tiny": (CONFIGS["tiny"].with_(name="sp4_tiny", T_text=33, grid_h=9, grid_w=7), 4),
    "sp2_small_nvfp4": (CONFIGS["small_nvfp4"], 2),
}


@pytest.mark.parametrize("name", list(SP_SMALL))
def test_sp_block_small_full(ig4, name):
    cfg, P = SP_SMALL[name]
    acts = make_block_activations(cfg, seed=34)
    wts = make_block_weights(cfg, seed=34, stress=True)
    if cfg.w_dtype == "nvfp4_mixed":
        # the NVFP4 FFN quantises h2 and u row by row, so each rank's rows
        # take the same decisions as in the single-GPU block, whose parity
        # with the oracle is tested on its own: compare with that block
        wd = ig4.nvfp4_pack_block_scales(to_dev(wts))
        y = _sp_run_dev(ig4, cfg, wd, acts, P).double().cpu().numpy()
        y_ref = run_block(ig4, cfg, wd, acts["x"].cuda(), acts["temb"].cuda())
        y_ref = y_ref.double().cpu().numpy()
        e = float(np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref))
        print(f"{name}: relL2 vs single-GPU block {e:.3e}, equal={np.array_equal(y, y_ref)}")
        assert e <= 1e-3
        return
    y = _sp_run(ig4, cfg, wts, acts, P).float().cpu().double().numpy()
    y_ref = _oracle(cfg, acts, wts)
    check_output(y.reshape(y_ref.shape), y_ref, to_f64(acts["x"]), cfg.w_dtype == "e4m3",
                 cfg.x_dtype == "bf16", name)


def _sp_run_dev(ig4, cfg, wd, acts, P):
    """_sp_run with weights already on the device."""
    c = ig4.config_from(cfg)
    bw = ig4.block_weights(wd)
    x = acts["x"].cuda()
    temb = acts["temb"].cuda()
    T = cfg.T_text
    ranges = [ig4.ig4_sp_image_range(c, P, r) for r in range(P)]
    xs = [sp_local_tokens(x, T, off, n) for off, n in ranges]
    ys = [torch.empty_like(t) for t in xs]
    pos = [ig4.ig4_sp_positions(c, P, r, device="cuda") for r in range(P)]
    wss = [torch.empty(ig4.ig4_sp_workspace_size(c, P, r), dtype=torch.uint8, device="cuda")
           for r in range(P)]

    def send_buf(r, phase):
        n = sum(ig4.ig4_sp_exchange_bytes(c, P, phase, r, d) for d in range(P))
        return torch.empty(n, dtype=torch.uint8, device="cuda")

    send0 = [send_buf(r, 0) for r in range(P)]
    for r in range(P):
        ig4.ig4_block_sp_pre(c, r, P, bw, xs[r], pos[r], temb, send0[r], wss[r])
    recv0 = _all_to_all(ig4, c, P, send0, 0)
    send1 = [send_buf(r, 1) for r in range(P)]
    for r in range(P):
        ig4.ig4_block_sp_attention(c, r, P, recv0[r], send1[r], wss[r])
    recv1 = _all_to_all(ig4, c, P, send1, 1)
    for r in range(P):
        ig4.ig4_block_sp_post(c, r, P, bw, xs[r], ys[r], recv1[r], wss[r])
    torch.cuda.synchronize()
    assert ig4.ig4_last_device_error() == ig4.IG4_OK
    return torch.cat([ys[0][:, :T]] + [t[:, T:] for t in ys], dim=1)


@pytest.mark.parametrize("name", ["1024px", "1024px_fp8"])
def test_sp2_block_1024px_sampled_rows(ig4, name):
    cfg = CONFIGS[name]
    acts = make_block_activations(cfg, seed=35)
    wts = make_block_weights(cfg, seed=35)
    y = _sp_run(ig4, cfg, wts, acts, 2).float().cpu().double().numpy().reshape(cfg.M, cfg.D)
    rows = sample_rows(cfg, n=48)
    y_ref = _oracle(cfg, acts, wts, rows)
    x = to_f64(acts["x"]).reshape(cfg.M, cfg.D)
    check_output(y[rows], y_ref, x[rows], cfg.w_dtype == "e4m3", True, f"sp2 {name}")


def test_sp_bf16_equals_the_block_bit_for_bit(ig4):
    """With bf16 weights the Ulysses path runs the block's kernels on the
    same rows, except that QKV, out-projection and MLP see fewer tokens and
    attention fewer heads per launch; every output element is computed by
    the same arithmetic in the same order, so it equals the single-GPU
    block exactly."""
    cfg = CONFIGS["tiny"].with_(name="sp_exact", T_text=40, grid_h=9, grid_w=9, x_dtype="bf16")
    acts = make_block_activations(cfg, seed=36)
    wts = make_block_weights(cfg, seed=36, stress=True)
    wd = to_dev(wts)
    y_sp = _sp_run_dev(ig4, cfg, wd, acts, 2)
    y = run_block(ig4, cfg, wd, acts["x"].cuda(), acts["temb"].cuda())
    assert torch.equal(y_sp, y)


def test_parallel_argument_errors(ig4):
    cfg = CONFIGS["tiny"]
    c = ig4.config_from(cfg)
    assert ig4.ig4_tp_workspace_size(c, 3) == 0    # 3 does not divide 4 heads
    assert ig4.ig4_sp_workspace_size(c, 2, 2) == 0  # rank out of range
    assert ig4.ig4_sp_exchange_bytes(c, 2, 2, 0, 0) == 0  # no phase 2
    x = torch.zeros(cfg.M, cfg.D, device="cuda")
    part = torch.empty(cfg.M, cfg.D, device="cuda")
    wd = to_dev(make_block_weights(cfg, seed=1))
    ws = torch.empty(ig4.ig4_tp_workspace_size(c, 2), dtype=torch.uint8, device="cuda")
    pos = ig4.ig4_mrope_positions(cfg.T_text, 1, 8, 8, device="cuda")
    temb = torch.zeros(1, 512, device="cuda")
    with pytest.raises(ig4.Ig4Error) as e:
        ig4.ig4_block_tp_attention(c, 2, 2, ig4.block_weights(wd), x, pos, temb, part, ws)
    assert e.value.status == ig4.IG4_ERR_INVALID_ARG
    with pytest.raises(ig4.Ig4Error) as e:
        ig4.ig4_block_tp_attention(c, 0, 2, ig4.block_weights(wd), x, pos, temb, part, ws[:-256])
    assert e.value.status == ig4.IG4_ERR_WORKSPACE
