"""GPU parity of the key-mean cache: pooling the window's key blocks once per appended frame
(pbsa_pool_keys) and selecting from the cached means (pbsa_select_blocks_pooled) gives the
same scores and the same selection as pooling the whole window at every selection, and
both match the oracle's block scores and top-k sets."""
import numpy as np
import pytest
import torch

from block_sparse_attention_35_b200 import pbsa as P
from block_sparse_attention_35_b200.synth import decode_inputs
from oracle import pbsa_oracle as orc
from tests.harness import Buffers, check_topk, config, f64, ring_to_window, run_select
from tests.test_gpu_select_fwd import RAGGED

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("ring_head,local_frames", [(0, 3), (2, 3), (1, 2)])
def test_pooled_key_cache_matches_full_pooling(cuda_dev, ring_head, local_frames):
    wl = RAGGED
    cfg = config(wl)
    inp = decode_inputs(wl)
    q = inp["q"].to(cuda_dev)
    kring = inp["k_local"].to(cuda_dev)           # W frames in the ring's slots
    W, nbf = P.pbsa_window_frames(cfg), P.pbsa_blocks_per_frame(cfg)
    ref = Buffers(cfg, wl, wl.q_frames, local_frames, cuda_dev)
    run_select(ref, q, wl.q_frames, kring, local_frames, ring_head)
    # cache: slots pooled one "append" at a time, in ring order from the head
    kbar = torch.full((wl.B, wl.H, W * nbf, wl.D), float("nan"), dtype=torch.float32, device=cuda_dev)
    P.pbsa_pool_keys(cfg, kring, ring_head, 1, kbar)
    if local_frames > 1:
        P.pbsa_pool_keys(cfg, kring, (ring_head + 1) % W, local_frames - 1, kbar)
    got = Buffers(cfg, wl, wl.q_frames, local_frames, cuda_dev)
    P.pbsa_select_blocks_pooled(cfg, q, wl.q_frames, kbar, local_frames, ring_head, got.idx,
                                got.idx_stride, got.cnt, got.scores, got.ws_sel)
    torch.cuda.synchronize()
    assert torch.equal(got.scores, ref.scores)
    assert torch.equal(got.idx, ref.idx)
    assert torch.equal(got.cnt, ref.cnt)
    # against the oracle: scores to 1e-5, top-k sets exact where the margin allows
    kwin = ring_to_window(inp["k_local"], ring_head, local_frames, W, wl.tokens_per_frame)
    _, sc_o = orc.select_blocks(f64(inp["q"]), f64(kwin), wl.frame_h, wl.frame_w, wl.topk_ratio)
    assert np.allclose(got.scores.cpu().numpy(), sc_o, rtol=0, atol=1e-5)
    check_topk(got.idx.cpu().numpy(), got.cnt.cpu().numpy(), sc_o, got.k)
