"""GPU parity: PBSA backward (dQ, dK/dV of persistent slots and local window) through the
C ABI against the fp64 oracle; relative L2 within the gradient tolerance."""
import dataclasses

import numpy as np
import pytest
import torch

from block_sparse_attention_35_b200 import pbsa as P
from block_sparse_attention_35_b200.synth import WORKLOADS, decode_inputs, training_inputs
from oracle import pbsa_oracle as orc
from tests.harness import (GRAD_REL_L2, Buffers, config, f64, rel_l2, ring_to_window,
                           run_fwd, run_select, window_to_ring)
from tests.test_gpu_select_fwd import ODDQB, RAGGED, RAGGED64

pytestmark = pytest.mark.gpu


def _grads(buf, dev, wl):
    f32 = dict(dtype=torch.float32, device=dev)
    W, tf = buf.W, buf.tf
    g = dict(dq=torch.full(buf.out.shape, float("nan"), **f32),
             dkp=torch.zeros(wl.B, wl.H, buf.S, 64, wl.D, **f32),
             dvp=torch.zeros(wl.B, wl.H, buf.S, 64, wl.D, **f32),
             dkl=torch.zeros(wl.B, W * tf, wl.H, wl.D, **f32),
             dvl=torch.zeros(wl.B, W * tf, wl.H, wl.D, **f32))
    return g


def run_bwd(buf, g, q, q_frames, kp, vp, plen, kl, vl, lf, rh, dout):
    P.pbsa_attn_bwd(buf.cfg, q, q_frames, kp, vp, plen, kl, vl, lf, rh, buf.idx, buf.idx_stride,
                    buf.cnt, buf.out, buf.lse, dout, g["dq"], g["dkp"], g["dvp"], g["dkl"],
                    g["dvl"], buf.ws_bwd, buf.status)


def _check_grads(g, want, plen, ring_head, lf, W, tf, what):
    dQ, dKp, dVp, dKw, dVw = want
    errs = {}
    errs["dq"] = rel_l2(f64(g["dq"]), dQ)
    mask = np.zeros(dKp.shape, dtype=bool)
    pl = plen.numpy()
    for b in range(pl.shape[0]):
        for h in range(pl.shape[1]):
            for s in range(pl.shape[2]):
                mask[b, h, s, :pl[b, h, s]] = True
    if mask.any():
        errs["dk_pers"] = rel_l2(f64(g["dkp"])[mask], dKp[mask])
        errs["dv_pers"] = rel_l2(f64(g["dvp"])[mask], dVp[mask])
    errs["dk_local"] = rel_l2(f64(ring_to_window(g["dkl"].cpu(), ring_head, lf, W, tf)), dKw)
    errs["dv_local"] = rel_l2(f64(ring_to_window(g["dvl"].cpu(), ring_head, lf, W, tf)), dVw)
    for k, v in errs.items():
        assert np.isfinite(v) and v <= GRAD_REL_L2, f"{what} {k}: rel L2 {v:.3e} ({errs})"
    return errs


def _run_case(wl, dev, ring_head=0, local_frames=None, persistent_filled=True, cfg_over=None):
    cfg = config(wl, **(cfg_over or {}))
    inp = decode_inputs(wl, persistent_filled=persistent_filled)
    W, tf = wl.window_frames, wl.tokens_per_frame
    lf = W if local_frames is None else local_frames
    kring = window_to_ring(inp["k_local"][:, :lf * tf], ring_head, W, tf)
    vring = window_to_ring(inp["v_local"][:, :lf * tf], ring_head, W, tf)
    d = {k: v.to(dev) for k, v in inp.items()}
    kring, vring = kring.to(dev), vring.to(dev)
    dout = torch.randn(inp["q"].shape, generator=torch.Generator().manual_seed(wl.seed + 77))
    dout = dout.to(torch.bfloat16)
    buf = Buffers(cfg, wl, wl.q_frames, lf, dev)
    run_select(buf, d["q"], wl.q_frames, kring, lf, ring_head)
    run_fwd(buf, d["q"], wl.q_frames, d["k_pers"], d["v_pers"], d["pers_len"], kring, vring,
            lf, ring_head, mass=False)
    g = _grads(buf, dev, wl)
    run_bwd(buf, g, d["q"], wl.q_frames, d["k_pers"], d["v_pers"], d["pers_len"], kring, vring,
            lf, ring_head, dout.to(dev))
    torch.cuda.synchronize()
    assert int(buf.status.item()) == 0
    kwin = ring_to_window(kring.cpu(), ring_head, lf, W, tf)
    vwin = ring_to_window(vring.cpu(), ring_head, lf, W, tf)
    idx = buf.idx.cpu().numpy()[..., :buf.k]
    bt, bh, bw = wl.block
    want = orc.attn_bwd(f64(inp["q"]), f64(inp["k_pers"]), f64(inp["v_pers"]),
                        inp["pers_len"].numpy(), f64(kwin), f64(vwin), idx, f64(dout),
                        wl.frame_h, wl.frame_w, bh, bw, bt=bt)
    return _check_grads(g, want, inp["pers_len"], ring_head, lf, W, tf, wl.name)


def test_bwd_tiny(cuda_dev):
    _run_case(WORKLOADS["tiny"], cuda_dev)


@pytest.mark.parametrize("ring_head", [0, 1])
def test_bwd_ragged(cuda_dev, ring_head):
    _run_case(RAGGED, cuda_dev, ring_head=ring_head)


def test_bwd_ragged_d64_partial_window(cuda_dev):
    _run_case(RAGGED64, cuda_dev, ring_head=3, local_frames=2)


def test_bwd_empty_persistent(cuda_dev):
    _run_case(RAGGED, cuda_dev, persistent_filled=False)


def test_bwd_odd_query_blocks(cuda_dev):
    _run_case(ODDQB, cuda_dev, ring_head=1)


def test_bwd_dense_local_flag_off(cuda_dev):
    _run_case(RAGGED, cuda_dev, cfg_over=dict(use_local_block_sparse_attn=False))


def test_bwd_decode_geometry_one_head(cuda_dev):
    """Full decode geometry (30x52 frames, 168 slots, 168 local blocks, k=21) on one head:
    every gradient against the oracle."""
    _run_case(dataclasses.replace(WORKLOADS["decode"], H=1), cuda_dev, ring_head=4)


def test_training_slice_two_chunks(cuda_dev):
    """Training configuration (chunk-causal 3-frame chunks over a 6-frame window, 168
    persistent slots, top-0.125) on a 6-frame slice: the first chunk sees a 3-frame window
    (k = 11), the second the full 6-frame window (k = 21); per-chunk gradients against the
    oracle."""
    wl = dataclasses.replace(WORKLOADS["train"], H=2)
    cfg = config(wl)
    tf, W = wl.tokens_per_frame, wl.window_frames
    inp = training_inputs(wl, frames=6)
    dev = cuda_dev
    kring = torch.zeros(wl.B, W * tf, wl.H, wl.D, dtype=torch.bfloat16)
    vring = torch.zeros_like(kring)
    for c in range(2):
        frames = slice(3 * c * tf, 3 * (c + 1) * tf)
        kring[:, 3 * c * tf:3 * (c + 1) * tf] = inp["k"][:, frames]
        vring[:, 3 * c * tf:3 * (c + 1) * tf] = inp["v"][:, frames]
        lf = 3 * (c + 1)
        q = inp["q"][:, frames].contiguous()
        do = inp["do"][:, frames].contiguous()
        buf = Buffers(cfg, wl, 3, lf, dev)
        kr, vr = kring.to(dev), vring.to(dev)
        kp, vp, pl = inp["k_pers"].to(dev), inp["v_pers"].to(dev), inp["pers_len"].to(dev)
        qd = q.to(dev)
        run_select(buf, qd, 3, kr, lf, 0)
        run_fwd(buf, qd, 3, kp, vp, pl, kr, vr, lf, 0, mass=False)
        g = _grads(buf, dev, wl)
        run_bwd(buf, g, qd, 3, kp, vp, pl, kr, vr, lf, 0, do.to(dev))
        torch.cuda.synchronize()
        assert int(buf.status.item()) == 0
        assert buf.k == (11 if c == 0 else 21)
        idx = buf.idx.cpu().numpy()[..., :buf.k]
        kwin, vwin = kring[:, :lf * tf], vring[:, :lf * tf]
        want = orc.attn_bwd(f64(q), f64(inp["k_pers"]), f64(inp["v_pers"]),
                            inp["pers_len"].numpy(), f64(kwin), f64(vwin), idx, f64(do),
                            wl.frame_h, wl.frame_w)
        _check_grads(g, want, inp["pers_len"], 0, lf, W, tf, f"train chunk {c}")
