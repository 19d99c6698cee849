"""GPU parity of the frame append fused with the key-mean cache (pbsa_append_frames):
window frames land in the ring bit for bit, their key means equal both pbsa_pool_keys'
(bit for bit) and the oracle's block means, and sink frames land in their slots exactly as
the oracle's append_frames puts them there."""
import dataclasses

import numpy as np
import pytest
import torch

from block_sparse_attention_35_b200 import pbsa as P
from block_sparse_attention_35_b200.synth import Workload
from oracle import pbsa_oracle as orc
from tests.harness import config, f64

pytestmark = pytest.mark.gpu

GRID = Workload("append", B=2, H=3, D=128, frame_h=14, frame_w=18, local_cache_size=6 * 252,
                persistent_cache_size=3 * 252, total_cache_size=9 * 252, max_seq_len=12 * 252,
                q_frames=3, topk_ratio=0.25, seed=51)


def _setup(wl, sink_frames, dev):
    cfg = config(wl, sink_frames=sink_frames)
    W, S, nbf = P.pbsa_window_frames(cfg), P.pbsa_num_slots(cfg), P.pbsa_blocks_per_frame(cfg)
    bt = wl.block[0]
    bf = dict(dtype=torch.bfloat16, device=dev)
    t = dict(kl=torch.zeros(wl.B, W * wl.tokens_per_frame, wl.H, wl.D, **bf),
             vl=torch.zeros(wl.B, W * wl.tokens_per_frame, wl.H, wl.D, **bf),
             kbar=torch.full((wl.B, wl.H, W // bt * nbf, wl.D), float("nan"), device=dev),
             kp=torch.full((wl.B, wl.H, S, 64, wl.D), 3.0, **bf),
             vp=torch.full((wl.B, wl.H, S, 64, wl.D), 3.0, **bf),
             plen=torch.zeros(wl.B, wl.H, S, dtype=torch.int32, device=dev),
             ps=torch.full((wl.B, wl.H, S), 9.0, device=dev),
             src=torch.full((wl.B, wl.H, S), -1, dtype=torch.int32, device=dev))
    return cfg, W, S, nbf, t


@pytest.mark.parametrize("block", [(1, 8, 8), (3, 4, 4)])
def test_append_window_frames_and_key_means(cuda_dev, block):
    wl = dataclasses.replace(GRID, block=block)
    cfg, W, S, nbf, t = _setup(wl, 0, cuda_dev)
    tf, bt = wl.tokens_per_frame, block[0]
    gen = torch.Generator().manual_seed(3)
    n = 3
    k = torch.randn(wl.B, n * tf, wl.H, wl.D, generator=gen).to(torch.bfloat16)
    v = torch.randn(wl.B, n * tf, wl.H, wl.D, generator=gen).to(torch.bfloat16)
    ring_slot = 3                                      # frames go to ring frames 3, 4, 5
    P.pbsa_append_frames(cfg, k.to(cuda_dev), v.to(cuda_dev), n, 6, t["kl"], t["vl"], ring_slot,
                         t["kbar"])
    torch.cuda.synchronize()
    kl, vl = t["kl"].cpu(), t["vl"].cpu()
    assert torch.equal(kl[:, 3 * tf:6 * tf], k) and torch.equal(vl[:, 3 * tf:6 * tf], v)
    assert (kl[:, :3 * tf] == 0).all()                 # other ring frames untouched
    # key means: bit-identical to pooling the same ring frames, and the oracle's means
    ref = torch.full_like(t["kbar"], float("nan"))
    P.pbsa_pool_keys(cfg, t["kl"], ring_slot, n, ref)
    torch.cuda.synchronize()
    rows = slice(ring_slot // bt * nbf, (ring_slot + n) // bt * nbf)
    assert torch.equal(t["kbar"][:, :, rows], ref[:, :, rows])
    assert torch.isnan(t["kbar"][:, :, :rows.start]).all()
    blocks = orc.frame_blocks(wl.frame_h, wl.frame_w, block[1], block[2], bt)
    for b in range(wl.B):
        for h in range(wl.H):
            want = orc.pool_blocks(f64(k[b, :, h]).reshape(n // bt, bt * tf, wl.D), blocks)
            assert np.allclose(t["kbar"][b, h, rows].cpu().numpy(), want, rtol=0, atol=1e-6)


@pytest.mark.parametrize("block,sink,n", [((1, 8, 8), 1, 3), ((1, 8, 8), 2, 2), ((3, 4, 4), 3, 6)])
def test_append_sink_frames_match_the_oracle(cuda_dev, block, sink, n):
    wl = dataclasses.replace(GRID, block=block)
    cfg, W, S, nbf, t = _setup(wl, sink, cuda_dev)
    bt, bh, bw = block
    tf = wl.tokens_per_frame
    n_sink = P.pbsa_sink_slots(cfg)
    assert n_sink == orc.sink_slots(sink, wl.frame_h, wl.frame_w, bh, bw, bt)
    gen = torch.Generator().manual_seed(4)
    k = torch.randn(wl.B, n * tf, wl.H, wl.D, generator=gen).to(torch.bfloat16)
    v = torch.randn(wl.B, n * tf, wl.H, wl.D, generator=gen).to(torch.bfloat16)
    P.pbsa_append_frames(cfg, k.to(cuda_dev), v.to(cuda_dev), n, 0, t["kl"], t["vl"], 0, t["kbar"],
                         t["kp"], t["vp"], t["plen"], t["ps"], t["src"])
    torch.cuda.synchronize()
    st0 = orc.DecodeState(np.zeros((wl.B, 0, wl.H, wl.D)), np.zeros((wl.B, 0, wl.H, wl.D)),
                          np.zeros((wl.B, wl.H, 0)), f64(t["kp"]) * 0 + 3.0, f64(t["vp"]) * 0 + 3.0,
                          np.zeros((wl.B, wl.H, S), np.int64), np.full((wl.B, wl.H, S), 9.0),
                          np.full((wl.B, wl.H, S), -1), 0)
    st = orc.append_frames(st0, f64(k), f64(v), sink, wl.frame_h, wl.frame_w, bh, bw, bt)
    assert np.array_equal(t["plen"].cpu().numpy(), st.pers_len)
    assert np.array_equal(t["src"].cpu().numpy(), st.pers_src)
    assert np.array_equal(t["ps"].cpu().double().numpy(), st.pers_score)
    # sink slots hold the blocks (rows past the length zero); the other slots are untouched
    assert np.array_equal(f64(t["kp"][:, :, :n_sink]), st.k_pers[:, :, :n_sink])
    assert np.array_equal(f64(t["vp"][:, :, :n_sink]), st.v_pers[:, :, :n_sink])
    assert (t["kp"][:, :, n_sink:] == 3.0).all()
    # the window frames went to the ring from slot 0 on
    nw = n - sink
    assert st.win_k.shape[1] == nw * tf and st.first_frame_global == sink
    assert np.array_equal(f64(t["kl"][:, :nw * tf]), st.win_k)
    assert np.array_equal(f64(t["vl"][:, :nw * tf]), st.win_v)
