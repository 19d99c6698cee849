"""GPU parity: window slide + persistent merge through the C ABI against the oracle, on
the same masses (so every decision is comparable exactly)."""
import numpy as np
import pytest
import torch

from block_sparse_attention_35_b200 import pbsa as P
from block_sparse_attention_35_b200.synth import WORKLOADS, decode_inputs
from oracle import pbsa_oracle as orc
from tests.harness import config, f64, ring_to_window
from tests.test_gpu_select_fwd import RAGGED

pytestmark = pytest.mark.gpu


def _merge_case(wl, dev, ring_head, n_ev, fill, seed, tie_scores=False):
    cfg = config(wl)
    inp = decode_inputs(wl)
    W, tf = wl.window_frames, wl.tokens_per_frame
    nbf = P.pbsa_blocks_per_frame(cfg)
    S = P.pbsa_num_slots(cfg)
    gen = torch.Generator().manual_seed(seed)
    B, H = wl.B, wl.H
    plen = inp["pers_len"].clone()
    empty = torch.rand(B, H, S, generator=gen) > fill
    plen[empty] = 0
    kp, vp = inp["k_pers"].clone(), inp["v_pers"].clone()
    kp[empty] = 0
    vp[empty] = 0
    if tie_scores:
        pscore = torch.randint(0, 4, (B, H, S), generator=gen).float()
        ml = torch.randint(0, 4, (B, H, W * nbf), generator=gen).float()
    else:
        pscore = torch.rand(B, H, S, generator=gen) * 10
        ml = torch.rand(B, H, W * nbf, generator=gen) * 10
    pscore[empty] = 0
    psrc = torch.where(plen > 0, torch.arange(S, dtype=torch.int32) + 5000, -1).to(torch.int32)
    d = dict(kl=inp["k_local"], vl=inp["v_local"], kp=kp, vp=vp, plen=plen, ps=pscore,
             src=psrc, ml=ml)
    g = {k: v.to(dev).contiguous() for k, v in d.items()}
    n_evb = n_ev * nbf
    upd = torch.full((B, H, n_evb, 2), -9, dtype=torch.int32, device=dev)
    nupd = torch.zeros((B, H), dtype=torch.int32, device=dev)
    P.pbsa_cache_update(cfg, g["kl"], g["vl"], W, ring_head, g["ml"], n_ev, 11, g["kp"],
                        g["vp"], g["plen"], g["ps"], g["src"], upd, nupd)
    torch.cuda.synchronize()

    # oracle on the logical window with masses in logical order
    kwin = ring_to_window(inp["k_local"], ring_head, W, W, tf)
    vwin = ring_to_window(inp["v_local"], ring_head, W, W, tf)
    ml_log = np.zeros((B, H, W * nbf))
    for lid in range(W * nbf):
        ml_log[:, :, lid] = ml[:, :, ((ring_head + lid // nbf) % W) * nbf + lid % nbf].numpy()
    r = orc.cache_update(f64(kp), f64(vp), plen.numpy(), pscore.double().numpy(), psrc.numpy(),
                         f64(kwin), f64(vwin), ml_log, n_ev, 11, wl.frame_h, wl.frame_w)
    assert np.array_equal(g["plen"].cpu().numpy(), r["pers_len"])
    assert np.array_equal(g["src"].cpu().numpy(), r["pers_src"])
    assert np.array_equal(g["ps"].cpu().double().numpy(), r["pers_score"])
    assert np.array_equal(f64(g["kp"]), r["k_pers"])
    assert np.array_equal(f64(g["vp"]), r["v_pers"])
    nu = nupd.cpu().numpy()
    uu = upd.cpu().numpy()
    for b in range(B):
        for h in range(H):
            want = r["updates"][b][h]
            assert nu[b, h] == len(want)
            assert [tuple(x) for x in uu[b, h, :nu[b, h]]] == want
    # evicted blocks' masses are cleared, the others untouched
    mlg = g["ml"].cpu().numpy()
    for lid in range(W * nbf):
        phys = ((ring_head + lid // nbf) % W) * nbf + lid % nbf
        if lid < n_evb:
            assert np.all(mlg[:, :, phys] == 0)
        else:
            assert np.array_equal(mlg[:, :, phys], ml[:, :, phys].numpy())


@pytest.mark.parametrize("ring_head,n_ev,fill,seed", [(0, 1, 1.0, 0), (2, 1, 0.5, 1),
                                                      (1, 2, 0.9, 2), (0, 3, 0.0, 3)])
def test_merge_ragged(cuda_dev, ring_head, n_ev, fill, seed):
    _merge_case(RAGGED, cuda_dev, ring_head, n_ev, fill, seed)


def test_merge_with_ties(cuda_dev):
    _merge_case(RAGGED, cuda_dev, 1, 2, 0.8, 4, tie_scores=True)


def test_merge_tiny(cuda_dev):
    _merge_case(WORKLOADS["tiny"], cuda_dev, 0, 1, 1.0, 5)


def test_merge_decode_full_size(cuda_dev):
    _merge_case(WORKLOADS["decode"], cuda_dev, 3, 3, 1.0, 6)
