"""GPU parity on frame grids whose edge blocks hold a token count that is not a multiple of
8 (30x50: 64, 16, 48 and 12 tokens; 20x21: 64, 40, 32 and 20; 13x11: 64, 24, 40 and 15).
Persistent slots then carry lengths such as 12, 15 or 20, both in the synthetic initial
cache and after a merge admits edge blocks.  Each case runs, through the C ABI, select ->
forward with block mass -> slide + merge -> forward on the merged cache -> backward, and
compares every step with the fp64 oracle on the same inputs."""
import numpy as np
import pytest
import torch

from block_sparse_attention_35_b200 import pbsa as P
from block_sparse_attention_35_b200.synth import Workload, decode_inputs
from oracle import pbsa_oracle as orc
from tests.harness import (LSE_ABS, MASS_ABS, MASS_REL, Buffers, assert_close_bf16,
                           check_topk, config, f64, ring_to_window, run_fwd, run_select)
from tests.test_gpu_bwd import _check_grads, _grads, run_bwd

pytestmark = pytest.mark.gpu


def _grid_workload(name, fh, fw, D=128, seed=0):
    tf = fh * fw
    return Workload(name, B=2, H=2, D=D, frame_h=fh, frame_w=fw, local_cache_size=3 * tf,
                    persistent_cache_size=2 * tf, total_cache_size=5 * tf, max_seq_len=8 * tf,
                    q_frames=2, topk_ratio=0.25, bias_fraction=0.1, seed=seed)


GRIDS = [_grid_workload("g30x50", 30, 50, seed=31), _grid_workload("g20x21", 20, 21, seed=32),
         _grid_workload("g13x11", 13, 11, D=64, seed=33)]


def _logical(ml_phys, ring_head, local_frames, W, nbf):
    out = np.zeros(ml_phys.shape[:2] + (local_frames * nbf,))
    for lid in range(local_frames * nbf):
        out[:, :, lid] = ml_phys[:, :, ((ring_head + lid // nbf) % W) * nbf + lid % nbf]
    return out


def _fwd_check(buf, inp_q, kp, vp, plen, kwin, vwin, wl, what):
    idx = buf.idx.cpu().numpy()[..., :buf.k]
    O, lse, mp, ml = orc.attn_fwd(f64(inp_q), f64(kp), f64(vp), plen.numpy(), f64(kwin),
                                  f64(vwin), idx, wl.frame_h, wl.frame_w)
    assert int(buf.status.item()) == 0, what
    assert_close_bf16(f64(buf.out), O, what + " out")
    assert np.abs(buf.lse.cpu().numpy() - lse).max() <= LSE_ABS, what + " lse"
    return mp, ml


@pytest.mark.parametrize("wl", GRIDS, ids=[w.name for w in GRIDS])
def test_edge_block_lengths_select_fwd_merge_fwd_bwd(cuda_dev, wl):
    dev = cuda_dev
    cfg = config(wl)
    W, tf = wl.window_frames, wl.tokens_per_frame
    nbf, S = P.pbsa_blocks_per_frame(cfg), P.pbsa_num_slots(cfg)
    sizes = [len(b) for b in orc.frame_blocks(wl.frame_h, wl.frame_w)]
    assert any(s % 8 for s in sizes), "the grid must have edge blocks of non-multiple-of-8 size"
    inp = decode_inputs(wl)
    # keep one frame's worth of slots (every block size of the frame, edge blocks included)
    # and empty the rest, so that the one-frame slide below admits every evicted block
    inp["pers_len"][:, :, nbf:] = 0
    inp["k_pers"][:, :, nbf:] = 0
    inp["v_pers"][:, :, nbf:] = 0
    assert (inp["pers_len"].numpy() % 8 != 0).any()
    ring_head = 1
    kring = inp["k_local"].clone()
    vring = inp["v_local"].clone()
    # the generated window (logical order) placed at ring_head
    kring = torch.cat([kring[:, (W - ring_head) * tf:], kring[:, :(W - ring_head) * tf]], 1)
    vring = torch.cat([vring[:, (W - ring_head) * tf:], vring[:, :(W - ring_head) * tf]], 1)
    kwin = ring_to_window(kring, ring_head, W, W, tf)
    assert torch.equal(kwin, inp["k_local"])
    d = {k: v.to(dev).contiguous() for k, v in inp.items()}
    kr, vr = kring.to(dev), vring.to(dev)
    q = d["q"]

    # ---- 1. select + forward with block mass on the initial cache
    buf = Buffers(cfg, wl, wl.q_frames, W, dev)
    run_select(buf, q, wl.q_frames, kr, W, ring_head)
    run_fwd(buf, q, wl.q_frames, d["k_pers"], d["v_pers"], d["pers_len"], kr, vr, W, ring_head)
    torch.cuda.synchronize()
    idx_o, sc_o = orc.select_blocks(f64(inp["q"]), f64(inp["k_local"]), wl.frame_h, wl.frame_w,
                                    wl.topk_ratio)
    check_topk(buf.idx.cpu().numpy(), buf.cnt.cpu().numpy(), sc_o, buf.k)
    mp, ml = _fwd_check(buf, inp["q"], inp["k_pers"], inp["v_pers"], inp["pers_len"],
                        inp["k_local"], inp["v_local"], wl, wl.name + " fwd1")
    mlg = buf.mass_local.cpu().numpy()
    mpg = buf.mass_pers.cpu().numpy()
    assert np.allclose(mpg, mp, rtol=MASS_REL, atol=MASS_ABS)
    assert np.allclose(_logical(mlg, ring_head, W, W, nbf), ml, rtol=MASS_REL, atol=MASS_ABS)
    assert np.allclose(mlg.sum(-1) + mpg.sum(-1), wl.nq, rtol=1e-4)

    # ---- 2. slide by one frame and merge, on the GPU's own masses (exact decisions)
    n_ev = 1
    psrc = torch.where(d["pers_len"] > 0, torch.arange(S, dtype=torch.int32, device=dev), -1)
    psrc = psrc.to(torch.int32).contiguous()
    upd = torch.full((wl.B, wl.H, n_ev * nbf, 2), -9, dtype=torch.int32, device=dev)
    n_upd = torch.zeros((wl.B, wl.H), dtype=torch.int32, device=dev)
    kp_before, vp_before = d["k_pers"].cpu(), d["v_pers"].cpu()
    plen_before, src_before = d["pers_len"].cpu().numpy(), psrc.cpu().numpy()
    score_before = buf.mass_pers.cpu().double().numpy()
    ml_log = _logical(mlg, ring_head, W, W, nbf)
    P.pbsa_cache_update(cfg, kr, vr, W, ring_head, buf.mass_local, n_ev, 4, d["k_pers"],
                        d["v_pers"], d["pers_len"], buf.mass_pers, psrc, upd, n_upd)
    torch.cuda.synchronize()
    r = orc.cache_update(f64(kp_before), f64(vp_before), plen_before, score_before, src_before,
                         f64(inp["k_local"]), f64(inp["v_local"]), ml_log, n_ev, 4,
                         wl.frame_h, wl.frame_w)
    assert np.array_equal(d["pers_len"].cpu().numpy(), r["pers_len"])
    assert np.array_equal(psrc.cpu().numpy(), r["pers_src"])
    assert np.array_equal(f64(d["k_pers"]), r["k_pers"])
    assert np.array_equal(f64(d["v_pers"]), r["v_pers"])
    nu, uu = n_upd.cpu().numpy(), upd.cpu().numpy()
    for b in range(wl.B):
        for h in range(wl.H):
            assert [tuple(x) for x in uu[b, h, :nu[b, h]]] == r["updates"][b][h]
    adm_len = [len(orc.frame_blocks(wl.frame_h, wl.frame_w)[j % nbf])
               for bb in r["updates"] for u in bb for _, j in u]
    assert nu.sum() == wl.B * wl.H * nbf and any(n % 8 for n in adm_len), \
        "the merge must admit edge blocks whose length is not a multiple of 8"

    # ---- 3. forward on the merged cache: the window keeps its last two frames, the freed
    # ring slot receives a fresh frame
    ring_head2 = (ring_head + n_ev) % W
    gen = torch.Generator().manual_seed(wl.seed + 500)
    fresh_k = torch.randn(wl.B, n_ev * tf, wl.H, wl.D, generator=gen).to(torch.bfloat16)
    fresh_v = torch.randn(wl.B, n_ev * tf, wl.H, wl.D, generator=gen).to(torch.bfloat16)
    for p in range(n_ev):
        slot = (ring_head2 + (W - n_ev) + p) % W
        kr[:, slot * tf:(slot + 1) * tf] = fresh_k[:, p * tf:(p + 1) * tf].to(dev)
        vr[:, slot * tf:(slot + 1) * tf] = fresh_v[:, p * tf:(p + 1) * tf].to(dev)
    q2 = torch.randn(inp["q"].shape, generator=gen).to(torch.bfloat16)
    buf2 = Buffers(cfg, wl, wl.q_frames, W, dev)
    run_select(buf2, q2.to(dev), wl.q_frames, kr, W, ring_head2)
    run_fwd(buf2, q2.to(dev), wl.q_frames, d["k_pers"], d["v_pers"], d["pers_len"], kr, vr, W,
            ring_head2)
    torch.cuda.synchronize()
    kwin2 = ring_to_window(kr.cpu(), ring_head2, W, W, tf)
    vwin2 = ring_to_window(vr.cpu(), ring_head2, W, W, tf)
    plen2 = d["pers_len"].cpu()
    assert (plen2.numpy() % 8 != 0).any()
    mp2, _ = _fwd_check(buf2, q2, d["k_pers"].cpu(), d["v_pers"].cpu(), plen2, kwin2, vwin2,
                        wl, wl.name + " fwd2")
    assert np.allclose(buf2.mass_pers.cpu().numpy(), mp2, rtol=MASS_REL, atol=MASS_ABS)

    # ---- 4. backward of that forward
    dout = torch.randn(inp["q"].shape, generator=gen).to(torch.bfloat16)
    g = _grads(buf2, dev, wl)
    run_bwd(buf2, g, q2.to(dev), wl.q_frames, d["k_pers"], d["v_pers"], d["pers_len"], kr, vr,
            W, ring_head2, dout.to(dev))
    torch.cuda.synchronize()
    assert int(buf2.status.item()) == 0
    idx2 = buf2.idx.cpu().numpy()[..., :buf2.k]
    want = orc.attn_bwd(f64(q2), f64(d["k_pers"]), f64(d["v_pers"]), plen2.numpy(), f64(kwin2),
                        f64(vwin2), idx2, f64(dout), wl.frame_h, wl.frame_w)
    _check_grads(g, want, plen2, ring_head2, W, W, tf, wl.name)


def test_slot_rows_past_length_do_not_leak(cuda_dev):
    """Rows past a slot's length hold large finite garbage: outputs and gradients must not
    change (the kernels mask those rows with exact zeros)."""
    wl = GRIDS[0]
    dev = cuda_dev
    cfg = config(wl)
    W = wl.window_frames
    inp = decode_inputs(wl)
    d = {k: v.to(dev).contiguous() for k, v in inp.items()}
    plen = inp["pers_len"]
    kp_g, vp_g = inp["k_pers"].clone(), inp["v_pers"].clone()
    rows = torch.arange(64)[None, None, None, :] >= plen[..., None]
    gen = torch.Generator().manual_seed(3)
    junk = (torch.randn(kp_g.shape, generator=gen) * 1e4).to(torch.bfloat16)
    kp_g[rows] = junk[rows]
    vp_g[rows] = junk[rows]
    outs = []
    for kp, vp in [(d["k_pers"], d["v_pers"]), (kp_g.to(dev), vp_g.to(dev))]:
        buf = Buffers(cfg, wl, wl.q_frames, W, dev)
        run_select(buf, d["q"], wl.q_frames, d["k_local"], W, 0)
        run_fwd(buf, d["q"], wl.q_frames, kp, vp, d["pers_len"], d["k_local"], d["v_local"], W, 0)
        g = _grads(buf, dev, wl)
        dout = torch.ones_like(d["q"])
        run_bwd(buf, g, d["q"], wl.q_frames, kp, vp, d["pers_len"], d["k_local"], d["v_local"], W, 0,
                dout)
        torch.cuda.synchronize()
        assert int(buf.status.item()) == 0
        outs.append((buf.out.clone(), buf.lse.clone(), buf.mass_pers.clone(), g["dq"].clone(),
                     g["dkl"].clone()))
    # outputs, lse and dK/dV are deterministic; the masses and dQ are summed across CTAs
    # with fp32 reductions in any order, so they agree to rounding
    for i, (a, b) in enumerate(zip(*outs)):
        if i == 2:
            assert torch.allclose(a, b, rtol=1e-6, atol=0)
        elif i == 3:
            assert torch.allclose(a, b, rtol=1e-5, atol=1e-6)
        else:
            assert torch.equal(a, b)
