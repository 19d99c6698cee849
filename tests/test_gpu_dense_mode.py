"""GPU parity for kv_cache_mode="dense" (one window of total_cache_size tokens, no
persistent slots, every block attended) and for the no-scoring selection path taken
whenever every window block is selected: through the C ABI against the fp64 oracle."""
import dataclasses

import numpy as np
import pytest
import torch

from block_sparse_attention_35_b200 import pbsa as P
from block_sparse_attention_35_b200.synth import decode_inputs
from oracle import pbsa_oracle as orc
from tests.harness import (Buffers, assert_close_bf16, config, f64, ring_to_window, run_fwd,
                           run_select, window_to_ring)
from tests.test_gpu_bwd import _check_grads, _grads, run_bwd
from tests.test_gpu_select_fwd import RAGGED

pytestmark = pytest.mark.gpu

# Inputs of a 5-frame dense window (the sizes the dense config below adds up to).
DENSE_IN = dataclasses.replace(RAGGED, name="dense5", local_cache_size=5 * 240,
                               persistent_cache_size=0, total_cache_size=5 * 240, seed=11)


def test_select_all_without_scores_is_the_full_ascending_list(cuda_dev):
    wl = RAGGED
    cfg = config(wl, use_local_block_sparse_attn=False)
    inp = decode_inputs(wl)
    buf = Buffers(cfg, wl, wl.q_frames, wl.window_frames, cuda_dev)
    run_select(buf, inp["q"].to(cuda_dev), wl.q_frames, inp["k_local"].to(cuda_dev),
               wl.window_frames, 0, scores=False)
    torch.cuda.synchronize()
    nl = wl.window_frames * buf.nbf
    assert buf.k == nl
    assert (buf.cnt.cpu().numpy() == nl).all()
    assert (buf.idx.cpu().numpy() == np.arange(nl)).all()
    # the same call through the static-scratch entry point
    buf.idx.fill_(-7)
    P.pbsa_select_blocks_noalloc(cfg, inp["q"].to(cuda_dev), wl.q_frames, inp["k_local"].to(cuda_dev),
                                 wl.window_frames, 0, buf.idx, buf.idx_stride, buf.cnt, None)
    torch.cuda.synchronize()
    assert (buf.idx.cpu().numpy() == np.arange(nl)).all()


@pytest.mark.parametrize("ring_head", [0, 3])
def test_dense_mode_forward_backward_slide(cuda_dev, ring_head):
    wl = DENSE_IN
    # the page-style split (local 3 frames + persistent 2 frames); dense mode uses all 5 as
    # one window and has no slots
    cfg = config(wl, kv_cache_mode="dense", local_cache_size=3 * 240, persistent_cache_size=2 * 240)
    W = P.pbsa_window_frames(cfg)
    assert W == 5 and P.pbsa_num_slots(cfg) == 0
    tf = wl.tokens_per_frame
    inp = decode_inputs(wl)
    kring = window_to_ring(inp["k_local"], ring_head, W, tf).to(cuda_dev)
    vring = window_to_ring(inp["v_local"], ring_head, W, tf).to(cuda_dev)
    q = inp["q"].to(cuda_dev)
    buf = Buffers(cfg, wl, wl.q_frames, W, cuda_dev)
    assert buf.k == W * buf.nbf
    run_select(buf, q, wl.q_frames, kring, W, ring_head, scores=False)
    run_fwd(buf, q, wl.q_frames, None, None, None, kring, vring, W, ring_head, mass=True)
    torch.cuda.synchronize()
    assert int(buf.status.item()) == 0
    kwin = ring_to_window(kring.cpu(), ring_head, W, W, tf)
    vwin = ring_to_window(vring.cpu(), ring_head, W, W, tf)
    idx = buf.idx.cpu().numpy()
    assert (idx == np.arange(buf.k)).all()
    B, H, D = wl.B, wl.H, wl.D
    kp0 = np.zeros((B, H, 0, 64, D))
    pl0 = np.zeros((B, H, 0), np.int64)
    O, lse, mp, ml = orc.attn_fwd(f64(inp["q"]), kp0, kp0, pl0, f64(kwin), f64(vwin), idx,
                                  wl.frame_h, wl.frame_w)
    assert_close_bf16(f64(buf.out), O, "dense out")
    assert np.abs(buf.lse.cpu().numpy() - lse).max() <= 1e-3
    # every row's probability lands on window blocks
    assert np.allclose(buf.mass_local.cpu().numpy().sum(-1), wl.nq, rtol=1e-4)

    # backward
    dout = torch.randn(inp["q"].shape, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    g = _grads(buf, cuda_dev, wl)
    run_bwd(buf, g, q, wl.q_frames, None, None, None, kring, vring, W, ring_head, dout.to(cuda_dev))
    torch.cuda.synchronize()
    assert int(buf.status.item()) == 0
    want = orc.attn_bwd(f64(inp["q"]), kp0, kp0, pl0, f64(kwin), f64(vwin), idx, f64(dout),
                        wl.frame_h, wl.frame_w)
    _check_grads(g, want, torch.zeros(B, H, 0, dtype=torch.int32), ring_head, W, W, tf, "dense")

    # slide: the oldest frame is dropped, nothing is admitted, its masses are cleared
    i32 = dict(dtype=torch.int32, device=cuda_dev)
    upd = torch.full((B, H, buf.nbf, 2), -3, **i32)
    n_upd = torch.full((B, H), -3, **i32)
    P.pbsa_cache_update(cfg, kring, vring, W, ring_head, buf.mass_local, 1, 0, None, None, None,
                        None, None, upd, n_upd)
    torch.cuda.synchronize()
    assert (n_upd.cpu().numpy() == 0).all()
    ml_after = buf.mass_local.cpu().numpy().reshape(B, H, W, buf.nbf)
    assert (ml_after[:, :, ring_head] == 0).all()
    assert (ml_after.sum((2, 3)) > 0).all()
