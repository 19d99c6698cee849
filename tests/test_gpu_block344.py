"""GPU parity for the project page's [3,4,4] block size (blocks of 3 frames x 4 x 4
tokens, 48 tokens, ragged rows and columns clipped to the frame): selection, forward with
block mass, backward, merge and a short rollout through the C ABI against the fp64 oracle
with the same block shape."""
import dataclasses

import numpy as np
import pytest
import torch

from block_sparse_attention_35_b200 import pbsa as P
from block_sparse_attention_35_b200.synth import WORKLOADS, Workload, decode_inputs
from oracle import pbsa_oracle as orc
from tests.harness import config, f64, ring_to_window
from tests.test_gpu_bwd import _run_case as _bwd_case
from tests.test_gpu_rollout import _run_rollout
from tests.test_gpu_select_fwd import _run_case as _fwd_case

pytestmark = pytest.mark.gpu

# 14x18 frames in 4x4 columns: block rows 4, 4, 4, 2 and columns 4, 4, 4, 4, 2, so a
# 3-frame group has 20 blocks of 48, 24 and 12 tokens; window 6 frames (40 blocks, k=10),
# persistent 3 frames' worth (20 slots), 3-frame chunks (20 query blocks).
B344 = Workload("b344", B=2, H=2, D=128, frame_h=14, frame_w=18, local_cache_size=6 * 252,
                persistent_cache_size=3 * 252, total_cache_size=9 * 252, max_seq_len=12 * 252,
                q_frames=3, topk_ratio=0.25, block=(3, 4, 4), bias_fraction=0.1, seed=41)
# D=64, 13x10 frames: rows 4, 4, 4, 1 and columns 4, 4, 2 (blocks of 48, 24, 12, 6 tokens),
# a 2-group window, 2 query groups.
B344_64 = dataclasses.replace(B344, name="b344d64", D=64, frame_h=13, frame_w=10, seed=42,
                              local_cache_size=6 * 130, persistent_cache_size=6 * 130,
                              total_cache_size=12 * 130, max_seq_len=12 * 130, q_frames=6)


@pytest.mark.parametrize("ring_head", [0, 3])
def test_344_select_fwd_mass(cuda_dev, ring_head):
    _fwd_case(B344, cuda_dev, ring_head=ring_head)


def test_344_d64_partial_window(cuda_dev):
    _fwd_case(B344_64, cuda_dev, ring_head=3, local_frames=3)


def test_344_empty_persistent_dense_flag(cuda_dev):
    _fwd_case(B344, cuda_dev, persistent_filled=False, cfg_over=dict(use_local_block_sparse_attn=False))


@pytest.mark.parametrize("ring_head", [0, 3])
def test_344_bwd(cuda_dev, ring_head):
    _bwd_case(B344, cuda_dev, ring_head=ring_head)


def test_344_bwd_d64(cuda_dev):
    _bwd_case(B344_64, cuda_dev, ring_head=3, local_frames=3)


def test_344_decode_full_size_sampled(cuda_dev):
    """The page-sized decode step with [3,4,4] blocks (H=12, 30x52 frames, 208 slots, 208
    window blocks, k=26): sampled query blocks (ragged ones included) of sampled heads."""
    _fwd_case(WORKLOADS["decode344"], cuda_dev, qblocks=[0, 12, 51, 90, 103],
              heads=[(0, 0), (0, 6), (0, 11)])


def test_344_decode_geometry_one_head_bwd(cuda_dev):
    _bwd_case(dataclasses.replace(WORKLOADS["decode344"], H=1), cuda_dev, ring_head=3)


@pytest.mark.parametrize("n_ev,ring_head,fill", [(3, 0, 1.0), (3, 3, 0.5), (6, 0, 0.7)])
def test_344_merge(cuda_dev, n_ev, ring_head, fill):
    wl = B344
    dev = cuda_dev
    cfg = config(wl)
    W, tf = wl.window_frames, wl.tokens_per_frame
    nbf, S = P.pbsa_blocks_per_frame(cfg), P.pbsa_num_slots(cfg)
    Wg = W // 3
    gen = torch.Generator().manual_seed(7 + n_ev + ring_head)
    inp = decode_inputs(wl)
    plen = inp["pers_len"].clone()
    empty = torch.rand(wl.B, wl.H, S, generator=gen) > fill
    plen[empty] = 0
    kp, vp = inp["k_pers"].clone(), inp["v_pers"].clone()
    kp[empty] = 0
    vp[empty] = 0
    pscore = torch.where(empty, 0.0, torch.rand(wl.B, wl.H, S, generator=gen) * 10)
    ml = torch.rand(wl.B, wl.H, Wg * nbf, generator=gen) * 10
    psrc = torch.where(plen > 0, torch.arange(S, dtype=torch.int32) + 900, -1).to(torch.int32)
    g = {k: v.to(dev).contiguous() for k, v in dict(kl=inp["k_local"], vl=inp["v_local"], kp=kp,
                                                   vp=vp, plen=plen, ps=pscore, src=psrc, ml=ml).items()}
    n_blk = n_ev // 3 * nbf
    upd = torch.full((wl.B, wl.H, n_blk, 2), -9, dtype=torch.int32, device=dev)
    nupd = torch.zeros((wl.B, wl.H), dtype=torch.int32, device=dev)
    P.pbsa_cache_update(cfg, g["kl"], g["vl"], W, ring_head, g["ml"], n_ev, 9, g["kp"], g["vp"],
                        g["plen"], g["ps"], g["src"], upd, nupd)
    torch.cuda.synchronize()
    kwin = ring_to_window(inp["k_local"], ring_head, W, W, tf)
    vwin = ring_to_window(inp["v_local"], ring_head, W, W, tf)
    ml_log = np.zeros((wl.B, wl.H, Wg * nbf))
    for lid in range(Wg * nbf):
        ml_log[:, :, lid] = ml[:, :, ((ring_head // 3 + lid // nbf) % Wg) * nbf + lid % nbf].numpy()
    r = orc.cache_update(f64(kp), f64(vp), plen.numpy(), pscore.double().numpy(), psrc.numpy(),
                         f64(kwin), f64(vwin), ml_log, n_ev, 9, wl.frame_h, wl.frame_w, 4, 4, bt=3)
    assert np.array_equal(g["plen"].cpu().numpy(), r["pers_len"])
    assert np.array_equal(g["src"].cpu().numpy(), r["pers_src"])
    assert np.array_equal(g["ps"].cpu().double().numpy(), r["pers_score"])
    assert np.array_equal(f64(g["kp"]), r["k_pers"])
    assert np.array_equal(f64(g["vp"]), r["v_pers"])
    nu, uu = nupd.cpu().numpy(), upd.cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.H):
            assert [tuple(x) for x in uu[b, h, :nu[b, h]]] == r["updates"][b][h]
    mlg = g["ml"].cpu().numpy()
    for lid in range(Wg * nbf):
        phys = ((ring_head // 3 + lid // nbf) % Wg) * nbf + lid % nbf
        if lid < n_blk:
            assert np.all(mlg[:, :, phys] == 0)
        else:
            assert np.array_equal(mlg[:, :, phys], ml[:, :, phys].numpy())


def test_344_wrapper_rollout_against_decode_step(cuda_dev):
    """Six 3-frame chunks through SparseForcingAttention with [3,4,4] blocks (append ->
    select -> forward with mass -> slide + merge), each replayed by the oracle's
    decode_step from the GPU's state, the merge decisions compared exactly."""
    wl = dataclasses.replace(B344, B=1, H=1, chunks=6)
    gen = torch.Generator().manual_seed(99)
    shape = (1, wl.q_frames * wl.tokens_per_frame, 1, wl.D)
    chunks = [tuple(torch.randn(shape, generator=gen).to(torch.bfloat16) for _ in range(3))
              for _ in range(wl.chunks)]
    a, _, admitted = _run_rollout(wl, cuda_dev, wl.chunks, lambda s: chunks[s])
    assert sum(admitted) >= a.S


def test_344_rollout_with_a_sink_group(cuda_dev):
    """[3,4,4] blocks with the first 3-frame group as the sink: chunk 0 is all sink, so its
    queries attend the sink slots alone (an empty window); later chunks add the window and
    the merge, which never touches the 20 sink slots.  Replayed step by step by the oracle."""
    wl = dataclasses.replace(B344, B=1, H=1, chunks=5)
    gen = torch.Generator().manual_seed(7)
    shape = (1, wl.q_frames * wl.tokens_per_frame, 1, wl.D)
    chunks = [tuple(torch.randn(shape, generator=gen).to(torch.bfloat16) for _ in range(3))
              for _ in range(wl.chunks)]
    a, _, admitted = _run_rollout(wl, cuda_dev, wl.chunks, lambda s: chunks[s], sink_frames=3)
    assert a.n_sink == 20 and a.S == 40
    assert (a.pers_src[0, 0, :20].cpu() == torch.arange(20)).all()
    assert sum(admitted) > 0
